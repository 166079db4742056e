"""Pins of the chunked-prefill and sender-output oracle (CPU only).

The sender's own output is checked against torch's float64 scaled_dot_product_attention. Every
chunk result is checked against the whole-sequence oracle (pinned separately): a chunk of rows
[c0, e) sees exactly the keys a whole-sequence row sees, so its statistics, kept sets and outputs
must equal the whole sequence's for those rows -- an off-by-c0 in a row index or in the causal
mask breaks that.
"""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import chunked as CH
from synth import bf16_bits_to_f64, chunk_of, make_prefill, make_sender_values


def _sdpa(q, k, v, bias_window=0, bias_value=0.0):
    L = q.shape[0]
    i = torch.arange(L)[:, None]
    j = torch.arange(L)[None, :]
    mask = torch.zeros(L, L, dtype=torch.float64)
    if bias_window:
        mask = mask + torch.where((i - j >= 0) & (i - j < bias_window),
                                  torch.tensor(bias_value, dtype=torch.float64),
                                  torch.tensor(0.0, dtype=torch.float64))
    mask = mask.masked_fill(j > i, float("-inf"))
    tq, tk, tv = (torch.from_numpy(np.ascontiguousarray(x))[None, None] for x in (q, k, v))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask[None, None])
    return out[0, 0].numpy()


@pytest.mark.parametrize("bias", [0, 24])
def test_sender_output_equals_sdpa(bias):
    wl = make_prefill([70, 33, 1], H_s=3, d=16, H_r=2, d_v=8, B=16, bias_window=bias,
                      bias_value=2.0, seed=5)
    vs = make_sender_values(wl, d_vs=12)
    out = CH.sender_output(wl, vs)
    q, k, v = (bf16_bits_to_f64(x) for x in (wl.q, wl.k, vs))
    for s in range(3):
        a, b = wl.cu_seqlens[s], wl.cu_seqlens[s + 1]
        for h in range(3):
            np.testing.assert_allclose(out[a:b, h], _sdpa(q[a:b, h], k[a:b, h], v[a:b, h], bias,
                                                          2.0), rtol=1e-10, atol=1e-12)


def _whole(wl):
    res = O.compress(wl)
    return res, O.mapped_av(wl, res.kept)


def _check_chunk_matches_whole(wl, res, out, starts, ends=None):
    cw = chunk_of(wl, starts, ends)
    cres = CH.compress_chunk(cw)
    cout = CH.mapped_av_chunk(cw, cres.kept)
    lay, wlay = cres.layout, res.layout
    for s in range(len(starts)):
        a, qa = int(wl.cu_seqlens[s]), int(cw.cu_q[s])
        c0, e = starts[s], lay.ends[s]
        # same arithmetic on the same numbers; only numpy's summation order over the masked
        # (zero) tail of a row can differ when e < L
        np.testing.assert_allclose(cres.lse[:, qa:qa + e - c0], res.lse[:, a + c0:a + e],
                                   rtol=1e-12, atol=0)
        np.testing.assert_allclose(cout[qa:qa + e - c0], out[a + c0:a + e], rtol=1e-12,
                                   atol=1e-13)
        for I in range(lay.I0[s], lay.nb[s]):
            c, w = lay.cb(s, I, 0), wlay.cb(s, I, 0)
            np.testing.assert_allclose(cres.mass[:, c:c + I + 1], res.mass[:, w:w + I + 1],
                                       rtol=1e-12, atol=1e-14)
            np.testing.assert_array_equal(cres.kept[:, c:c + I + 1], res.kept[:, w:w + I + 1])
            np.testing.assert_array_equal(cres.near[:, c:c + I + 1], res.near[:, w:w + I + 1])
    return cw, cres


def test_tail_chunks_equal_whole_sequence_rows():
    """Chunks running to the sequence end, starting at 0, inside, and at the end (empty)."""
    wl = make_prefill([150, 96, 64, 130], H_s=3, d=16, H_r=4, d_v=8, B=16, tau=0.8,
                      bias_window=20, bias_value=2.0, seed=6)
    res, out = _whole(wl)
    assert not res.kept.all()                      # tau < 1 drops blocks
    cw, cres = _check_chunk_matches_whole(wl, res, out, [0, 48, 64, 112])
    assert cres.layout.nb[2] == cres.layout.I0[2]  # the empty chunk has no row block
    assert int(cw.cu_q[3] - cw.cu_q[2]) == 0


def test_middle_chunks_ending_on_block_boundaries():
    """Chunks [c0, e) with e a multiple of B inside the sequence, and grouped receiver values."""
    wl = make_prefill([160, 100], H_s=2, d=16, H_r=4, d_v=8, B=16, tau=0.7, seed=7, H_kv=2)
    res, out = _whole(wl)
    _check_chunk_matches_whole(wl, res, out, [32, 16], [96, 64])


def test_chunk_ending_mid_block_keeps_row_results():
    """A chunk ending inside a block: its rows' lse and sender output equal the whole
    sequence's (they see the same keys); its last row block holds only the rows present."""
    wl = make_prefill([150], H_s=2, d=16, H_r=2, d_v=8, B=16, tau=0.9, seed=8)
    vs = make_sender_values(wl, d_vs=8)
    res = O.compress(wl)
    whole_os = CH.sender_output(wl, vs)
    cw = chunk_of(wl, [64], [103])
    cres = CH.compress_chunk(cw)
    np.testing.assert_allclose(cres.lse, res.lse[:, 64:103], rtol=1e-12, atol=0)
    vs_keys = vs[:103]
    np.testing.assert_allclose(CH.sender_output_chunk(cw, vs_keys), whole_os[64:103],
                               rtol=1e-12, atol=1e-13)
    lay = cres.layout
    assert lay.nb[0] == 7 and lay.I0[0] == 4          # row blocks 4, 5, 6 (the last: 7 rows)
    last = lay.cb(0, 6, 0)
    np.testing.assert_allclose(cres.mass[:, last:last + 7].sum(axis=1), 7.0, rtol=1e-12)


def test_sender_output_chunk_equals_whole_rows():
    wl = make_prefill([96, 80], H_s=2, d=16, H_r=2, d_v=8, B=16, bias_window=10,
                      bias_value=2.0, seed=9)
    vs = make_sender_values(wl, d_vs=16)
    whole = CH.sender_output(wl, vs)
    cw = chunk_of(wl, [32, 48])
    got = CH.sender_output_chunk(cw, np.concatenate([vs[0:96], vs[96:176]]))
    np.testing.assert_allclose(got[:64], whole[32:96], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got[64:], whole[96 + 48:176], rtol=1e-12, atol=1e-13)


def test_chunk_start_must_be_a_block_multiple():
    wl = make_prefill([64], H_s=1, d=16, H_r=1, d_v=8, B=16, seed=10)
    with pytest.raises(ValueError):
        CH.compress_chunk(chunk_of(wl, [8]))


def test_sender_output_of_empty_sequences_and_chunks():
    """Sequences and chunks without rows contribute no output rows (and do not disturb the
    others): the other sequences' rows equal those of the batch without the empty ones."""
    wl = make_prefill([40, 0, 20], H_s=2, d=16, H_r=2, d_v=8, B=16, seed=6)
    vs = make_sender_values(wl, d_vs=8)
    out = CH.sender_output(wl, vs)
    assert out.shape == (60, 2, 8)
    from synth import select_sequences
    sub = select_sequences(wl, [0, 2])
    np.testing.assert_array_equal(out, CH.sender_output(sub, np.concatenate([vs[:40], vs[40:]])))
    cw = chunk_of(wl, [16, 0, 16], [40, 0, 20])
    oc = CH.sender_output_chunk(cw, np.concatenate([vs[:40], vs[40:60]]))
    np.testing.assert_allclose(oc[:24], out[16:40], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(oc[24:], out[56:60], rtol=1e-12, atol=1e-14)
