"""GPU parity of the paged decode form and of head matching against the float64 oracle."""

import numpy as np
import pytest
import torch

import oracle as O
from synth import decode_config, make_decode, make_head_match

from _gpu_common import bf16, check_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    from cross_model_attention_map_b200 import iamap
    return iamap


def _run_decode(dw):
    from cross_model_attention_map_b200.runner import DecodeStep
    max_pages = dw.page_table.shape[1]
    st = DecodeStep(dw.batch, dw.H_s, dw.H_r, dw.d_v, dw.ctx_lens, dw.p_rows.shape[2], max_pages,
                    dw.page_size, dw.v_pages.shape[0])
    out = st.run(torch.from_numpy(dw.p_rows).cuda(), torch.from_numpy(dw.W).cuda(),
                 bf16(dw.v_pages), torch.from_numpy(dw.page_table).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy()


def test_decode_config_parity(C):
    """Batch 4, context 8704, 14 sender heads, 64 receiver heads d_v=128, one-hot W, 16-token
    pages under a random page table."""
    dw = decode_config()
    out = _run_decode(dw)
    assert C.iamap_device_status() == 0
    check_output(out, O.mapped_av_paged(dw), "paged decode")


def test_decode_ragged_general_W(C):
    dw = make_decode(batch=5, ctx=300, H_s=6, H_r=12, d_v=64, page_size=16,
                     ctx_lens=[300, 1, 17, 0, 256], seed=31)
    dw.W = np.random.default_rng(32).standard_normal(dw.W.shape).astype(np.float32)
    out = _run_decode(dw)
    assert C.iamap_device_status() == 0
    check_output(out, O.mapped_av_paged(dw), "ragged decode")
    assert np.all(out[3] == 0)


def test_decode_bad_page_is_flagged(C):
    dw = make_decode(batch=2, ctx=64, H_s=2, H_r=4, d_v=64, page_size=16, seed=33)
    dw.page_table[1, 2] = 10_000
    _run_decode(dw)
    assert C.iamap_device_status() & C.IAMAP_DEV_BAD_INDEX


def _run_hm(hm, n_used=None):
    from cross_model_attention_map_b200.runner import HeadMatch
    r = HeadMatch(hm.L_s, hm.H_small, hm.d_small, hm.L_l, hm.H_large, hm.d_large, hm.n, n_used)
    arg, sim = r.run(bf16(hm.q_small), bf16(hm.k_small), bf16(hm.q_large), bf16(hm.k_large))
    torch.cuda.synchronize()
    return arg.cpu().numpy(), sim.cpu().numpy()


@pytest.mark.parametrize("n,n_used,d_small,d_large", [(200, 200, 64, 128), (300, 131, 64, 64),
                                                      (64, 64, 128, 128)])
def test_head_match_small_parity(C, n, n_used, d_small, d_large):
    hm = make_head_match(n=n, L_s=3, H_small=5, d_small=d_small, L_l=2, H_large=7,
                         d_large=d_large, noise=0.3, seed=34)
    arg, sim = _run_hm(hm, n_used)
    assert C.iamap_device_status() == 0
    C_ref, arg_ref = O.head_match(hm, n_used=n_used)
    np.testing.assert_allclose(sim, C_ref, rtol=0, atol=2e-3)
    np.testing.assert_array_equal(arg.reshape(arg_ref.shape), arg_ref)


def test_head_match_calibration_workload(C):
    """n=1024, small 24 x 14 heads d=64, large 8 x 64 heads d=128, noisy zero-padded copies: the
    GPU argmax equals the planted mapping (which the oracle also recovers: oracle pin tests) and
    the cosine of one large layer matches the oracle's."""
    hm = make_head_match()
    arg, sim = _run_hm(hm)
    assert C.iamap_device_status() == 0
    np.testing.assert_array_equal(arg.reshape(hm.planted.shape), hm.planted)
    # oracle cosines of large layer 0 against every small head
    sub = make_head_match()
    sub.L_l = 1
    sub.q_large = sub.q_large[:1]
    sub.k_large = sub.k_large[:1]
    C_ref, _ = O.head_match(sub)
    np.testing.assert_allclose(sim[:hm.H_large], C_ref, rtol=0, atol=2e-3)
