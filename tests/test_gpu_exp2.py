"""The FMA-pipe exponential of the compress kernels on the GPU (iamap_selftest_exp2): against
exact powers of two and against ex2.approx on the MUFU unit, element by element."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_exp2_fma_against_exact_and_mufu():
    from cross_model_attention_map_b200 import iamap as C
    rng = np.random.default_rng(11)
    x = np.concatenate([-rng.uniform(0.0, 126.0, 1_000_001), -np.linspace(0.0, 1.0, 4097),
                        np.array([0.0, -1.0, -126.0, -200.0, -1e30])]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    y_fma = torch.empty_like(xd)
    y_mufu = torch.empty_like(xd)
    C.iamap_selftest_exp2(xd, y_fma, y_mufu, x.size)
    torch.cuda.synchronize()
    yf = y_fma.cpu().numpy().astype(np.float64)
    ym = y_mufu.cpu().numpy().astype(np.float64)
    exact = np.exp2(np.maximum(x.astype(np.float64), -126.0))
    inside = x >= -126.0
    rel_fma = np.abs(yf[inside] / exact[inside] - 1.0)
    assert rel_fma.max() < 3e-7, rel_fma.max()
    # ex2.approx.ftz flushes results below 2^-126; compare where both are normal
    normal = inside & (x > -125.0)
    assert np.max(np.abs(yf[normal] / ym[normal] - 1.0)) < 6e-7
    # below the clamp the FMA form returns 2^-126 within the polynomial's error (never a
    # wrapped exponent)
    assert np.allclose(yf[~inside], 2.0 ** -126, rtol=3e-7, atol=0)
    assert np.all(np.isfinite(yf)) and np.all(yf > 0)


def test_exp2_fma_odd_count_and_empty():
    from cross_model_attention_map_b200 import iamap as C
    x = torch.tensor([-0.25, -3.5, -10.0], dtype=torch.float32, device="cuda")
    yf = torch.full_like(x, -1.0)
    ym = torch.full_like(x, -1.0)
    C.iamap_selftest_exp2(x, yf, ym, 3)
    C.iamap_selftest_exp2(x, yf, ym, 0)
    torch.cuda.synchronize()
    exact = np.exp2(x.cpu().numpy().astype(np.float64))
    assert np.allclose(yf.cpu().numpy(), exact, rtol=3e-7, atol=0)
