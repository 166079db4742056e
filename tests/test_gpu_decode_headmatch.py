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
                    dw.page_size, dw.v_pages.shape[0], H_kv=dw.v_pages.shape[2])
    out = st.run(torch.from_numpy(dw.p_rows).cuda(), torch.from_numpy(dw.W).cuda(),
                 bf16(dw.v_pages), torch.from_numpy(dw.page_table).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _gpu_sender_rows(C, dw):
    """The small model's decode rows on the GPU (iamap_sender_rows), as a device tensor."""
    max_ctx = int(dw.ctx_lens.max())
    rows = torch.empty(dw.batch, dw.H_s, max_ctx, dtype=torch.float32, device="cuda")
    ws = C.alloc_workspace(C.iamap_sender_rows_workspace_bytes(dw.batch, dw.H_s, max_ctx))
    C.iamap_sender_rows(bf16(dw.q_s), bf16(dw.k_pages_s), dw.k_pages_s.shape[0],
                        torch.from_numpy(dw.page_table).cuda(), dw.page_table.shape[1],
                        dw.page_size, torch.from_numpy(dw.ctx_lens).cuda(), dw.ctx_lens,
                        dw.batch, dw.H_s, dw.q_s.shape[2], rows, max_ctx, ws)
    torch.cuda.synchronize()
    return rows


def test_sender_rows_parity(C):
    """The small model's decode rows (softmax of q.k / 8 over 8704 paged keys, 14 heads) against
    the oracle: relative error of every row within the output tolerance, rows summing to 1."""
    dw = decode_config()
    rows = _gpu_sender_rows(C, dw).cpu().numpy()
    assert C.iamap_device_status() == 0
    ref = O.sender_decode_rows(dw)
    for b in range(dw.batch):
        check_output(rows[b], ref[b], "sender rows of sequence %d" % b)
    np.testing.assert_allclose(rows.sum(axis=2), 1.0, rtol=0, atol=1e-4)


def test_sender_rows_ragged_and_bad_page(C):
    dw = make_decode(batch=4, ctx=600, H_s=3, H_r=4, d_v=64, page_size=16,
                     ctx_lens=[600, 0, 17, 513], seed=34, d_s=128)
    rows = _gpu_sender_rows(C, dw).cpu().numpy()
    assert C.iamap_device_status() == 0
    ref = O.sender_decode_rows(dw)
    for b in (0, 2, 3):
        check_output(rows[b], ref[b], "sender rows of sequence %d" % b)
    assert np.all(rows[1] == 0) and np.all(rows[2, :, 17:] == 0)
    dw.page_table[3, 5] = dw.k_pages_s.shape[0] + 7          # a page outside the pool
    rows = _gpu_sender_rows(C, dw).cpu().numpy()
    assert C.iamap_device_status() & C.IAMAP_DEV_BAD_INDEX
    assert np.all(rows[3, :, 80:96] == 0)


def test_decode_config_parity(C):
    """Batch 4, context 8704, 14 sender heads, 64 receiver heads d_v=128, one-hot W, 16-token
    pages under a random page table; the sender rows are the small model's own softmax rows,
    computed on the GPU (iamap_sender_rows) and compared with the oracle's output on the
    oracle's rows."""
    dw = decode_config()
    gpu_rows = _gpu_sender_rows(C, dw)
    from cross_model_attention_map_b200.runner import DecodeStep
    st = DecodeStep(dw.batch, dw.H_s, dw.H_r, dw.d_v, dw.ctx_lens, gpu_rows.shape[2],
                    dw.page_table.shape[1], dw.page_size, dw.v_pages.shape[0])
    out = st.run(gpu_rows, torch.from_numpy(dw.W).cuda(), bf16(dw.v_pages),
                 torch.from_numpy(dw.page_table).cuda())
    torch.cuda.synchronize()
    assert C.iamap_device_status() == 0
    dw.p_rows = O.sender_decode_rows(dw)
    check_output(out.cpu().numpy(), O.mapped_av_paged(dw), "paged decode")


def test_decode_dirichlet_rows(C):
    """The same step on given rows (Dirichlet draws with a sink at position 0)."""
    dw = decode_config()
    out = _run_decode(dw)
    assert C.iamap_device_status() == 0
    check_output(out, O.mapped_av_paged(dw), "paged decode, given rows")


def test_decode_ragged_general_W(C):
    dw = make_decode(batch=5, ctx=300, H_s=6, H_r=12, d_v=64, page_size=16,
                     ctx_lens=[300, 1, 17, 0, 256], seed=31)
    dw.W = np.random.default_rng(32).standard_normal(dw.W.shape).astype(np.float32)
    out = _run_decode(dw)
    assert C.iamap_device_status() == 0
    check_output(out, O.mapped_av_paged(dw), "ragged decode")
    assert np.all(out[3] == 0)


def test_decode_grouped_values(C):
    """Grouped value heads in the page pool (8 receiver heads per value head), ragged contexts,
    a general W."""
    dw = make_decode(batch=3, ctx=1000, H_s=6, H_r=64, d_v=128, page_size=16,
                     ctx_lens=[1000, 513, 17], seed=44, H_kv=8)
    rng = np.random.default_rng(45)
    dw.W = rng.standard_normal(dw.W.shape).astype(np.float32)
    check_output(_run_decode(dw), O.mapped_av_paged(dw), "decode, grouped values")


def test_decode_bad_page_is_flagged(C):
    dw = make_decode(batch=2, ctx=64, H_s=2, H_r=4, d_v=64, page_size=16, seed=33)
    dw.page_table[1, 2] = 10_000
    _run_decode(dw)
    assert C.iamap_device_status() & C.IAMAP_DEV_BAD_INDEX


def _run_hm(hm, n_used=None, metric="cosine"):
    from cross_model_attention_map_b200.runner import HeadMatch
    r = HeadMatch(hm.L_s, hm.H_small, hm.d_small, hm.L_l, hm.H_large, hm.d_large, hm.n, n_used,
                  metric=metric)
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


@pytest.mark.parametrize("metric", ["cosine", "pearson"])
def test_head_match_long_prompt_tensor_core_maps(C, metric):
    """n_used >= 1024 builds the maps with the tensor-core compress kernels (row statistics, then
    dense head-major tiles with their sums and norms)."""
    hm = make_head_match(n=2304, L_s=2, H_small=3, d_small=64, L_l=1, H_large=4,
                         d_large=128, noise=0.3, seed=38)
    arg, sim = _run_hm(hm, 2100, metric)
    assert C.iamap_device_status() == 0
    S_ref, _ = O.head_match(hm, n_used=2100, metric=metric)
    np.testing.assert_allclose(sim, S_ref, rtol=0, atol=3e-3)
    _argmax_matches(arg, S_ref, 6e-3)


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


def _argmax_matches(arg, S_ref, tol):
    """GPU argmax equals the oracle's wherever the oracle's top two differ by more than tol;
    elsewhere it must be one of the heads within tol of the best."""
    for m in range(S_ref.shape[0]):
        row = S_ref[m]
        best = row.max()
        near = np.nonzero(row >= best - tol)[0]
        assert arg[m] in near, (m, arg[m], near)


@pytest.mark.parametrize("metric", ["pearson", "euclidean"])
@pytest.mark.parametrize("n,n_used,d_small,d_large", [(200, 200, 64, 128), (300, 131, 64, 64)])
def test_head_match_metric_parity(C, metric, n, n_used, d_small, d_large):
    """Pearson and Euclidean similarities (IAM notes, method section 1) against the oracle; the
    GPU computes them from the Gram of the bf16 maps and each map's sum and squared norm."""
    hm = make_head_match(n=n, L_s=3, H_small=5, d_small=d_small, L_l=2, H_large=7,
                         d_large=d_large, noise=0.3, seed=35)
    arg, sim = _run_hm(hm, n_used, metric)
    assert C.iamap_device_status() == 0
    S_ref, arg_ref = O.head_match(hm, n_used=n_used, metric=metric)
    tol = 3e-3 * max(1.0, np.abs(S_ref).max())
    np.testing.assert_allclose(sim, S_ref, rtol=0, atol=tol)
    _argmax_matches(arg, S_ref, 2 * tol)


def test_mapping_consistency_kernel(C):
    from cross_model_attention_map_b200.runner import mapping_consistency
    rng = np.random.default_rng(36)
    for n in (1, 31, 512, 5000):
        a = rng.integers(0, 4, size=n).astype(np.int32)
        b = rng.integers(0, 4, size=n).astype(np.int32)
        agree = mapping_consistency(torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda())
        assert int(agree.item()) == int(np.sum(a == b))


def test_prefill_vs_prefix_consistency(C):
    """Mappings found on the full prompt and on its first half: each matches the oracle's (up to
    near-ties), and the kernel's agreement count is that of the two GPU mappings."""
    from cross_model_attention_map_b200.runner import mapping_consistency
    hm = make_head_match(n=256, L_s=2, H_small=6, d_small=64, L_l=2, H_large=8, d_large=128,
                         noise=0.6, seed=37)
    a_full, _ = _run_hm(hm, 256)
    a_half, _ = _run_hm(hm, 128)
    S_full, _ = O.head_match(hm, n_used=256)
    S_half, _ = O.head_match(hm, n_used=128)
    _argmax_matches(a_full, S_full, 4e-3)
    _argmax_matches(a_half, S_half, 4e-3)
    agree = mapping_consistency(torch.from_numpy(a_full).cuda(), torch.from_numpy(a_half).cuda())
    assert int(agree.item()) == int(np.sum(a_full == a_half))
