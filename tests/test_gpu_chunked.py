"""GPU parity of the sender's own output (fused into compress) and of the chunked-prefill form of
compress and mapped_av, through the C ABI, against the float64 oracle (``oracle/chunked.py``).

Every chunk result is also compared with the GPU's whole-sequence result of the same rows: the
chunk kernels visit the same key tiles in the same order, so lse, masses, kept sets, stored
tiles and outputs must be bit-identical. Chunk starts are taken at 0, inside a sequence (at even
and odd row blocks: a row-block pair whose first block lies before the chunk), at its last block,
and with chunk ends in the middle of a block.
"""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import chunked as CH
from synth import chunk_of, make_prefill, make_sender_values, prefill_config

from _gpu_common import (LSE_ATOL, MASS_NORM_ATOL, bf16, check_kept_invariants, check_output,
                         compare_kept, gpu_kept, upload_prefill)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def C():
    from cross_model_attention_map_b200 import iamap
    return iamap


def _whole(wl, v_s=None):
    from cross_model_attention_map_b200.runner import PrefillLayer
    layer = PrefillLayer(wl.seqlens, wl.H_s, wl.d, wl.H_r, wl.d_v, wl.tau, wl.bias_window,
                         wl.bias_value, H_kv=wl.v.shape[1])
    q, k, v, W = upload_prefill(wl)
    o_s = None
    if v_s is None:
        layer.compress(q, k)
    else:
        o_s = torch.empty(wl.n, wl.H_s, v_s.shape[2], dtype=torch.float32, device="cuda")
        layer.compress_with_output(q, k, bf16(v_s), o_s)
    layer.mapped_av(W, v)
    torch.cuda.synchronize()
    return layer, o_s


def _chunk(wl, starts, ends, v_s_keys=None):
    from cross_model_attention_map_b200.runner import ChunkPrefillLayer
    cw = chunk_of(wl, starts, ends)
    layer = ChunkPrefillLayer(starts, [int(cw.cu_k[s + 1] - cw.cu_k[s]) for s in range(len(starts))],
                              wl.H_s, wl.d, wl.H_r, wl.d_v, wl.tau, wl.bias_window, wl.bias_value,
                              H_kv=wl.v.shape[1],
                              d_vs=None if v_s_keys is None else v_s_keys.shape[2])
    q, k, v = bf16(cw.q), bf16(cw.k), bf16(cw.v)
    W = torch.from_numpy(wl.W).cuda()
    layer.compress(q, k, None if v_s_keys is None else bf16(v_s_keys))
    layer.mapped_av(W, v)
    torch.cuda.synchronize()
    return cw, layer


def _keys_of(v_s, wl, ends):
    """Rows [0, ends[s]) of every sequence of a [n, H, d] array, packed like a chunk's keys."""
    return np.concatenate([v_s[int(wl.cu_seqlens[s]):int(wl.cu_seqlens[s]) + e]
                           for s, e in enumerate(ends)])


# ------------------------------------------------------------------------------------------------
# Sender output fused into compress
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("seqlens,H_s,d,d_vs,bias", [
    ([512], 8, 64, 64, (0, 0.0)),              # the tiny configuration's shapes
    ([200, 64, 1, 333], 5, 64, 128, (0, 0.0)),  # ragged tails, a 1-token sequence
    ([1000, 130], 6, 128, 128, (128, 2.0)),     # d = 128, local bias
    ([130, 0, 64], 3, 128, 64, (0, 0.0)),       # an empty sequence inside the batch
])
def test_sender_output_parity(C, seqlens, H_s, d, d_vs, bias):
    wl = make_prefill(seqlens, H_s=H_s, d=d, H_r=4, d_v=64, B=64, tau=0.9, std=1.5, sink=True,
                      bias_window=bias[0], bias_value=bias[1], seed=61)
    v_s = make_sender_values(wl, d_vs=d_vs)
    plain, _ = _whole(wl)
    layer, o_s = _whole(wl, v_s)
    assert C.iamap_device_status() == 0
    check_output(o_s.cpu().numpy(), CH.sender_output(wl, v_s), "sender output")
    # the map written beside it is the plain compress's, bit for bit
    for key in ("lse", "mass", "headmask_dense", "row_ptr"):
        assert torch.equal(layer.bufs[key], plain.bufs[key]), key
    tiles = plain.counts()[1]
    assert layer.counts() == plain.counts()
    assert torch.equal(layer.vals[:tiles], plain.vals[:tiles])
    assert torch.equal(layer.out, plain.out)


# ------------------------------------------------------------------------------------------------
# Chunked prefill
# ------------------------------------------------------------------------------------------------

def _chunk_parity(C, wl, starts, ends, with_sender=True):
    v_s = make_sender_values(wl) if with_sender else None
    cw, layer = _chunk(wl, starts, ends, None if v_s is None else _keys_of(v_s, wl, ends))
    assert C.iamap_device_status() == 0
    ref = CH.compress_chunk(cw)
    lay = ref.layout
    lse = layer.bufs["lse"].cpu().numpy()
    np.testing.assert_allclose(lse, ref.lse, rtol=0, atol=LSE_ATOL)
    mass = layer.bufs["mass"].cpu().numpy()
    hm = layer.bufs["headmask_dense"].cpu().numpy().view(np.uint64)
    kept = ((hm[None, :] >> np.arange(wl.H_s, dtype=np.uint64)[:, None]) & np.uint64(1)).astype(bool)
    compare_kept(kept, ref.kept, ref.near)
    for s in range(len(starts)):
        for I in range(lay.I0[s], lay.nb[s]):
            b0 = lay.cb(s, I, 0)
            R = min(wl.B, lay.ends[s] - I * wl.B)
            assert np.abs(mass[:, b0:b0 + I + 1] - ref.mass[:, b0:b0 + I + 1]).max() / R <= MASS_NORM_ATOL
            check_kept_invariants(kept[:, b0:b0 + I + 1], ref.mass[:, b0:b0 + I + 1] / R, wl.tau)
    # every stored tile against the oracle's probabilities of the chunk rows
    row_ptr = layer.bufs["row_ptr"].cpu().numpy()
    nnz, tiles = layer.counts()
    col_idx = layer.bufs["col_idx"].cpu().numpy()[:nnz]
    hmask = layer.bufs["headmask"].cpu().numpy().view(np.uint64)[:nnz]
    val_off = layer.bufs["val_off"].cpu().numpy()[:nnz]
    vals = layer.vals.float().cpu().numpy().reshape(-1, 64)
    rb = 0
    for s in range(len(starts)):
        for I in range(lay.I0[s], lay.nb[s]):
            st = {}
            for u in range(row_ptr[rb], row_ptr[rb + 1]):
                J, m = int(col_idx[u]), int(hmask[u])
                assert bool(kept[:, lay.cb(s, I, J)].any())
                k = bin(m).count("1")
                rank = 0
                for h in range(wl.H_s):
                    if (m >> h) & 1:
                        if h not in st:
                            st[h] = CH.chunk_rowblock_stats(cw, lay, s, h, I)
                        blk = vals[int(val_off[u]) * 64:(int(val_off[u]) + k) * 64]
                        t_gpu = blk.reshape(64, k, 64)[:, rank, :]
                        np.testing.assert_allclose(t_gpu, O.masked_tile(st[h], J, wl.B),
                                                   rtol=8e-3, atol=2e-6)
                        rank += 1
            rb += 1
    assert rb == layer.nrb
    check_output(layer.out.cpu().numpy(), CH.mapped_av_chunk(cw, kept), "chunk mapped_av")
    if v_s is not None:
        check_output(layer.o_s.cpu().numpy(),
                     CH.sender_output_chunk(cw, _keys_of(v_s, wl, ends)), "chunk sender output")
    return cw, layer


def _same_as_whole(wl, cw, layer, whole):
    """The chunk's rows equal the whole-sequence GPU results bit for bit."""
    lay = CH.chunk_layout(cw)
    wlay = O.causal_layout(wl.seqlens, wl.B)
    lse_c, lse_w = layer.bufs["lse"].cpu(), whole.bufs["lse"].cpu()
    mass_c, mass_w = layer.bufs["mass"].cpu(), whole.bufs["mass"].cpu()
    hm_c, hm_w = layer.bufs["headmask_dense"].cpu(), whole.bufs["headmask_dense"].cpu()
    out_c, out_w = layer.out.cpu(), whole.out.cpu()
    for s in range(len(cw.starts)):
        c0, e = cw.starts[s], lay.ends[s]
        a, qa = int(wl.cu_seqlens[s]), int(cw.cu_q[s])
        if e != wl.seqlens[s]:
            continue   # a chunk that ends early sees fewer keys than the whole sequence's rows
        assert torch.equal(lse_c[:, qa:qa + e - c0], lse_w[:, a + c0:a + e])
        assert torch.equal(out_c[qa:qa + e - c0], out_w[a + c0:a + e])
        for I in range(lay.I0[s], lay.nb[s]):
            b0, w0 = lay.cb(s, I, 0), wlay.cb(s, I, 0)
            assert torch.equal(mass_c[:, b0:b0 + I + 1], mass_w[:, w0:w0 + I + 1])
            assert torch.equal(hm_c[b0:b0 + I + 1], hm_w[w0:w0 + I + 1])


@pytest.mark.parametrize("seqlens,starts,ends,H_s,H_r,d,bias", [
    ([300, 200], [0, 0], None, 4, 4, 64, (0, 0.0)),               # whole sequences as chunks
    ([300, 200], [128, 64], None, 4, 6, 64, (0, 0.0)),            # even and odd first blocks
    ([1000, 130], [576, 128], None, 6, 10, 128, (128, 2.0)),      # d = 128, bias, last block
    ([500, 450, 64], [64, 192, 0], [420, 450, 64], 5, 9, 64, (0, 0.0)),  # a chunk ending mid-block
    ([260, 90], [256, 64], None, 3, 40, 64, (0, 0.0)),            # H_r > 32: CUDA-core mapped_av
])
def test_chunk_parity(C, seqlens, starts, ends, H_s, H_r, d, bias):
    wl = make_prefill(seqlens, H_s=H_s, d=d, H_r=H_r, d_v=d, B=64, tau=0.9, std=1.5, sink=True,
                      bias_window=bias[0], bias_value=bias[1], seed=62)
    ends = list(wl.seqlens) if ends is None else ends
    cw, layer = _chunk_parity(C, wl, starts, ends)
    whole, _ = _whole(wl)
    _same_as_whole(wl, cw, layer, whole)


def test_chunk_grouped_values(C):
    """Grouped receiver values (H_kv < H_r) in the chunk form."""
    wl = make_prefill([400, 150], H_s=5, d=64, H_r=8, d_v=64, B=64, tau=0.9, std=1.5, sink=True,
                      seed=63, H_kv=2)
    _chunk_parity(C, wl, [192, 64], list(wl.seqlens), with_sender=False)


def test_chunk_bad_start_is_rejected(C):
    wl = make_prefill([300], H_s=2, d=64, H_r=2, d_v=64, B=64, tau=0.9, seed=64)
    with pytest.raises(C.IamapError) as e:
        C.iamap_chunk_plan([0, 300 - 100], [0, 300], [100], 1, 64)
    assert e.value.code == -1


def test_varlen40k_chunks_sampled(C):
    """The packed 4096/8192/12288/16384 workload (40 sender heads, 32 receiver heads, tau 0.9) as
    chunks from 2048/4096/8192/12288: sampled row blocks against the oracle, all rows against the
    whole-sequence GPU results."""
    wl = prefill_config("varlen40k")
    starts = [2048, 4096, 8192, 12288]
    cw, layer = _chunk(wl, starts, list(wl.seqlens))
    assert C.iamap_device_status() == 0
    whole, _ = _whole(wl)
    _same_as_whole(wl, cw, layer, whole)
    lay = CH.chunk_layout(cw)
    out = layer.out.cpu().numpy()
    kept = gpu_kept(layer)
    for s, I in [(0, 32), (1, 127), (2, 128), (3, 255)]:
        b0 = lay.cb(s, I, 0)
        st = {h: CH.chunk_rowblock_stats(cw, lay, s, h, I) for h in range(wl.H_s)}
        for h in range(wl.H_s):
            compare_kept(kept[h, b0:b0 + I + 1], st[h].kept, st[h].near)
        a = int(wl.cu_seqlens[s])
        ref = O.mapped_av_rows(wl, s, I, lambda h: kept[h, b0:b0 + I + 1], lambda h: st[h])
        r0 = int(cw.cu_q[s]) + I * wl.B - starts[s]
        check_output(out[r0:r0 + ref.shape[0]], ref, "chunk rows of block (%d, %d)" % (s, I))


def test_two_phase_extract_with_output(C):
    """Stats, read the tile count, allocate exactly, then extract with the sender output: the same
    tiles and the same sender output as the one-call iamap_compress_with_output."""
    from cross_model_attention_map_b200.runner import PrefillLayer
    wl = make_prefill([500, 180], H_s=6, d=128, H_r=4, d_v=64, B=64, tau=0.9, seed=65)
    v_s = make_sender_values(wl)
    one, o_one = _whole(wl, v_s)
    q, k, v, W = upload_prefill(wl)
    two = PrefillLayer(wl.seqlens, 6, 128, 4, 64, 0.9, capacity_tiles=1)
    b = two.bufs
    C.iamap_compress_stats(q, k, two.cu, two.cu_host, two.num_seqs, two.n, 6, 128, 64, 0.9, 0, 0.0,
                           b["lse"], b["mass"], b["headmask_dense"], b["row_ptr"], b["col_idx"],
                           b["headmask"], b["val_off"], b["counts"], two.ws)
    nnz, tiles = two.counts()
    vals = torch.empty(tiles, 64, 64, dtype=torch.bfloat16, device="cuda")
    o_s = torch.empty(wl.n, 6, 128, dtype=torch.float32, device="cuda")
    C.iamap_compress_extract_with_output(q, k, two.cu, two.cu_host, two.num_seqs, two.n, 6, 128,
                                         64, 0, 0.0, bf16(v_s), 128, o_s, b["lse"], b["row_ptr"],
                                         b["col_idx"], b["headmask"], b["val_off"], b["counts"],
                                         vals, tiles, two.ws)
    torch.cuda.synchronize()
    assert C.iamap_device_status() == 0
    assert torch.equal(vals, one.vals[:tiles])
    assert torch.equal(o_s, o_one)
