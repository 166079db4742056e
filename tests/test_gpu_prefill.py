"""GPU parity of map_compress + mapped_av against the float64 oracle (through the C ABI).

Small workloads are compared element by element over everything the library writes: lse, block
masses, per-head kept sets (bit-exact except near-threshold blocks), the union BSR index, every
stored bf16 tile, and the output. The output is compared with the oracle evaluated on the GPU's
own kept sets (so a near-threshold flip is not mistaken for a kernel error) and, where no flip
happened, against the oracle's own kept sets too. The full-size workloads are checked on sampled
row blocks in the launch configuration the benchmark times.
"""

import numpy as np
import pytest
import torch

import oracle as O
from synth import bf16_bits_to_f64, make_prefill, prefill_config

from _gpu_common import (LSE_ATOL, MASS_NORM_ATOL, bsr_readback, check_bsr_structure,
                         check_kept_invariants, check_output, compare_kept, gpu_kept, head_tile,
                         upload_prefill)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    from cross_model_attention_map_b200 import iamap
    return iamap


def _run(wl, capacity=None):
    from cross_model_attention_map_b200.runner import PrefillLayer
    layer = PrefillLayer(wl.seqlens, wl.H_s, wl.d, wl.H_r, wl.d_v, wl.tau, wl.bias_window,
                         wl.bias_value, capacity_tiles=capacity, H_kv=wl.v.shape[1])
    q, k, v, W = upload_prefill(wl)
    layer.step(q, k, W, v)
    torch.cuda.synchronize()
    return layer


def _full_parity(C, wl):
    layer = _run(wl)
    assert C.iamap_device_status() == 0
    ref = O.compress(wl)
    lay = ref.layout
    # lse
    lse = layer.bufs["lse"].cpu().numpy()
    np.testing.assert_allclose(lse, ref.lse, rtol=0, atol=LSE_ATOL)
    # masses normalised by valid rows
    mass = layer.bufs["mass"].cpu().numpy()
    rows = np.zeros(lay.num_causal_blocks)
    for s, L in enumerate(lay.seqlens):
        for I in range(lay.nb[s]):
            R = min(wl.B, L - I * wl.B)
            c0 = lay.cb(s, I, 0)
            rows[c0:c0 + I + 1] = R
    assert np.abs((mass - ref.mass) / rows[None, :]).max() <= MASS_NORM_ATOL
    # kept sets: bit-exact outside near-threshold blocks, and the GPU's own sets satisfy the
    # cumulative-mass choice on the oracle's float64 masses
    kept = gpu_kept(layer)
    flips = compare_kept(kept, ref.kept, ref.near)
    for s in range(len(lay.seqlens)):
        for I in range(lay.nb[s]):
            c0 = lay.cb(s, I, 0)
            R = min(wl.B, lay.seqlens[s] - I * wl.B)
            check_kept_invariants(kept[:, c0:c0 + I + 1], ref.mass[:, c0:c0 + I + 1] / R, wl.tau)
    # BSR index from the GPU's own kept sets, and every stored tile
    row_ptr, col_idx, headmask, val_off = check_bsr_structure(layer, kept, lay)
    vals = layer.vals.float().cpu().numpy().reshape(-1, 64)
    rb = 0
    for s in range(len(lay.seqlens)):
        for I in range(lay.nb[s]):
            stats = {}
            for u in range(row_ptr[rb], row_ptr[rb + 1]):
                J = int(col_idx[u])
                m = int(headmask[u])
                rank = 0
                for h in range(wl.H_s):
                    if (m >> h) & 1:
                        if h not in stats:
                            stats[h] = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, s, h, I, wl.B,
                                                        wl.tau, wl.bias_window, wl.bias_value)
                        t_ref = O.masked_tile(stats[h], J, wl.B)
                        t_gpu = head_tile(vals, val_off[u], bin(m).count("1"), rank)
                        np.testing.assert_allclose(t_gpu, t_ref, rtol=8e-3, atol=2e-6)
                        rank += 1
            rb += 1
    # output on the GPU's kept sets; and on the oracle's own when nothing flipped
    out = layer.out.cpu().numpy()
    check_output(out, O.mapped_av(wl, kept), "mapped_av (GPU kept sets)")
    if flips == 0:
        check_output(out, O.mapped_av(wl, ref.kept), "end to end (oracle kept sets)")
    return flips


def test_tiny_config_full_parity(C):
    """The tiny configuration (n=512, 8 sender heads d=64, 4 receiver heads, tau=0.95)."""
    _full_parity(C, prefill_config("tiny"))


@pytest.mark.parametrize("seqlens,H_s,H_r,d,tau,bias", [
    ([200, 64, 1, 333], 5, 6, 64, 0.9, (0, 0.0)),        # ragged tails, a 1-token sequence
    ([1000, 130], 12, 10, 128, 0.95, (128, 2.0)),         # d=128, local bias, H_r % 4 != 0
    ([640], 3, 2, 128, 1.0, (0, 0.0)),                    # keep everything
    ([450, 70], 7, 9, 64, 0.3, (16, 2.0)),                # aggressive sparsity
    ([130, 0, 64, 0], 4, 4, 64, 0.9, (0, 0.0)),           # empty sequences inside the batch
    ([600, 77], 64, 32, 128, 0.9, (0, 0.0)),              # the largest head counts: every head-mask
                                                          # bit, 32 receivers in clusters of 8
])
def test_varlen_parity(C, seqlens, H_s, H_r, d, tau, bias):
    wl = make_prefill(seqlens, H_s=H_s, d=d, H_r=H_r, d_v=d, B=64, tau=tau, std=1.5, sink=True,
                      bias_window=bias[0], bias_value=bias[1], seed=21)
    _full_parity(C, wl)


@pytest.mark.parametrize("seqlens,H_s,H_r,H_kv,d", [
    ([300, 90], 20, 8, 2, 64),     # tensor-core cluster kernel (2 CTAs, H_s > 16), 4 receivers
                                   # per value head
    ([300, 90], 6, 8, 2, 64),      # the CUDA-core kernel (2-CTA cluster, few sender heads)
    ([200], 5, 12, 3, 128),        # tensor-core, groups across CTA boundaries
    ([260, 40], 4, 40, 8, 64),     # H_r > 32: the CUDA-core kernel
])
def test_grouped_values_parity(C, seqlens, H_s, H_r, H_kv, d):
    """Grouped receiver values (receiver head r reads value head r / (H_r / H_kv))."""
    wl = make_prefill(seqlens, H_s=H_s, d=d, H_r=H_r, d_v=d, B=64, tau=0.9, std=1.5, sink=True,
                      seed=43, H_kv=H_kv)
    _full_parity(C, wl)


def test_identity_mixing_keep_all_is_dense_attention(C):
    """W = I, tau = 1: the output is dense causal attention; compare with torch SDPA on the
    same bf16 inputs (float64 on the CPU)."""
    wl = make_prefill([300, 100], H_s=4, d=64, H_r=4, d_v=64, B=64, tau=1.0, seed=22)
    wl.W = np.eye(4, dtype=np.float32)
    layer = _run(wl)
    out = layer.out.cpu().numpy()
    q, k, v = (torch.from_numpy(bf16_bits_to_f64(x)) for x in (wl.q, wl.k, wl.v))
    ref = np.zeros_like(out, dtype=np.float64)
    for s in range(2):
        a, b = wl.cu_seqlens[s], wl.cu_seqlens[s + 1]
        ref[a:b] = torch.nn.functional.scaled_dot_product_attention(
            q[a:b].transpose(0, 1), k[a:b].transpose(0, 1), v[a:b].transpose(0, 1),
            is_causal=True).transpose(0, 1).numpy()
    check_output(out, ref, "identity mixing vs SDPA")


def test_capacity_shortfall_is_reported(C):
    wl = make_prefill([256], H_s=4, d=64, H_r=4, d_v=64, B=64, tau=1.0, seed=23)
    layer = _run(wl, capacity=3)
    assert layer.counts()[1] == 4 * 10
    assert C.iamap_device_status() & C.IAMAP_DEV_CAPACITY
    assert C.iamap_device_status() == 0  # cleared by the read


def test_two_phase_exact_allocation(C):
    """Stats, read the tile count, allocate exactly, extract: same tiles as the one-call path."""
    from cross_model_attention_map_b200.runner import PrefillLayer
    wl = make_prefill([500, 180], H_s=6, d=64, H_r=4, d_v=64, B=64, tau=0.9, seed=24)
    q, k, v, W = upload_prefill(wl)
    one = PrefillLayer(wl.seqlens, 6, 64, 4, 64, 0.9)
    one.step(q, k, W, v)
    two = PrefillLayer(wl.seqlens, 6, 64, 4, 64, 0.9, capacity_tiles=1)
    b = two.bufs
    C.iamap_compress_stats(q, k, two.cu, two.cu_host, two.num_seqs, two.n, 6, 64, 64, 0.9, 0, 0.0,
                           b["lse"], b["mass"], b["headmask_dense"], b["row_ptr"], b["col_idx"],
                           b["headmask"], b["val_off"], b["counts"], two.ws)
    nnz, tiles = two.counts()
    vals = torch.empty(tiles, 64, 64, dtype=torch.bfloat16, device="cuda")
    C.iamap_compress_extract(q, k, two.cu, two.cu_host, two.num_seqs, two.n, 6, 64, 64, 0, 0.0,
                             b["lse"], b["row_ptr"], b["col_idx"], b["headmask"], b["val_off"],
                             b["counts"], vals, tiles, two.ws)
    torch.cuda.synchronize()
    assert C.iamap_device_status() == 0
    assert torch.equal(vals, one.vals[:tiles])


# ------------------------------------------------------------------------------------------------
# Full-size configurations, sampled
# ------------------------------------------------------------------------------------------------

def _sampled_parity(C, wl, samples):
    layer = _run(wl)
    assert C.iamap_device_status() == 0
    lay = O.causal_layout(wl.seqlens, wl.B)
    kept = gpu_kept(layer)
    lse = layer.bufs["lse"].cpu().numpy()
    mass = layer.bufs["mass"].cpu().numpy()
    row_ptr, col_idx, headmask, val_off, tiles = bsr_readback(layer)
    vals = layer.vals.view(-1, 64)
    out = layer.out.cpu().numpy()
    flips = 0
    # invariants everywhere, on the GPU's own masses: the kept mass reaches tau, the kept set is
    # minimal, and no dropped block outweighs a kept one (up to fp32 rounding)
    for s in range(len(lay.seqlens)):
        for I in range(lay.nb[s]):
            c0 = lay.cb(s, I, 0)
            R = min(wl.B, lay.seqlens[s] - I * wl.B)
            check_kept_invariants(kept[:, c0:c0 + I + 1], mass[:, c0:c0 + I + 1] / R, wl.tau)
    for (s, I) in samples:
        c0 = lay.cb(s, I, 0)
        a = int(wl.cu_seqlens[s])
        st = {}
        for h in range(wl.H_s):
            st[h] = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, s, h, I, wl.B, wl.tau,
                                     wl.bias_window, wl.bias_value)
            np.testing.assert_allclose(lse[h, a + st[h].row0:a + st[h].row0 + st[h].R], st[h].lse,
                                       rtol=0, atol=LSE_ATOL)
            assert np.abs(mass[h, c0:c0 + I + 1] - st[h].masses).max() / st[h].R <= MASS_NORM_ATOL
            flips += compare_kept(kept[h, c0:c0 + I + 1], st[h].kept, st[h].near)
        rb = lay.rb_start[s] + I
        for u in list(range(row_ptr[rb], row_ptr[rb + 1]))[::7]:
            J, m = int(col_idx[u]), int(headmask[u])
            rank = 0
            for h in range(wl.H_s):
                if (m >> h) & 1:
                    k = bin(m).count("1")
                    blk = vals[int(val_off[u]) * 64:(int(val_off[u]) + k) * 64].float().cpu().numpy()
                    t_gpu = blk.reshape(64, k, 64)[:, rank, :]
                    np.testing.assert_allclose(t_gpu, O.masked_tile(st[h], J, wl.B), rtol=8e-3,
                                               atol=2e-6)
                    rank += 1
        ref = O.mapped_av_rows(wl, s, I, lambda h: kept[h, c0:c0 + I + 1], lambda h: st[h])
        row0 = a + I * wl.B
        check_output(out[row0:row0 + ref.shape[0]], ref, "rows of block (%d, %d)" % (s, I))
    return flips


def test_prefill8k_sampled(C):
    """n=8192, 32 sender heads d=128, 24 receiver heads, tau=0.95, sink, local bias +2.0."""
    wl = prefill_config("prefill8k")
    _sampled_parity(C, wl, [(0, 0), (0, 1), (0, 64), (0, 127)])


def test_varlen40k_sampled(C):
    """4 packed sequences 4096/8192/12288/16384, 40 sender heads, 32 receiver heads, tau=0.9."""
    wl = prefill_config("varlen40k")
    _sampled_parity(C, wl, [(0, 63), (1, 5), (2, 191), (3, 0), (3, 255)])


def test_sequence_longer_than_16384_tokens(C):
    """257 row blocks: the compress stages take the mma.sync kernels (the tensor-core statistics
    keep at most 256 column blocks per row in TMEM); mapped_av stays on the tensor cores."""
    wl = make_prefill([16448, 300], H_s=2, d=64, H_r=3, d_v=64, B=64, tau=0.9, std=1.5,
                      sink=True, seed=46)
    _sampled_parity(C, wl, [(0, 0), (0, 131), (0, 256), (1, 4)])


def test_host_pipeline_equals_direct_steps(C):
    """HostPrefillPipeline (uploads and read-backs overlapping the kernels of other steps) gives
    every step exactly the output of a direct step on the same inputs."""
    from cross_model_attention_map_b200.runner import HostPrefillPipeline, PrefillLayer
    wls = [make_prefill([300, 200], H_s=4, d=64, H_r=4, d_v=64, B=64, tau=0.9, seed=s)
           for s in (71, 72, 73)]
    layer = PrefillLayer(wls[0].seqlens, 4, 64, 4, 64, 0.9)

    def pinned(x):
        return x.cpu().pin_memory()

    ins = [tuple(pinned(t) for t in upload_prefill(wl)) for wl in wls]
    outs = [torch.empty(layer.out.shape, dtype=torch.float32).pin_memory() for _ in wls]
    pipe = HostPrefillPipeline(layer)
    pipe.run(ins, outs).synchronize()
    assert C.iamap_device_status() == 0
    for wl, o in zip(wls, outs):
        q, k, v, W = upload_prefill(wl)
        ref = layer.step(q, k, W, v).cpu()
        torch.cuda.synchronize()
        assert torch.equal(o, ref)
