"""Float64 CPU oracle: the sender's own attention output, and the chunked-prefill form of
map_compress and mapped_av.

TEST INFRASTRUCTURE ONLY, like ``oracle/iamap_oracle.py`` (whose steps it reuses): imported by
``tests/`` only, never by the product path; it shares no code with the CUDA library.

Sources:

[GLIDE II-B]    "GLIDE: Guided Layerwise Hybrid Attention for efficient LLM inference" page,
                Section II-B: O_i = sum_j alpha_ij v_j with alpha the causal softmax of q_i.k_j.
[MapFlow-vLLM]  "PKU MapFlow: cross-model attention map reuse" news page, the paragraph on the
                integration into vLLM: the fused retrieval kernel works with paged attention,
                chunked prefill and variable-length packing.
[MapFlow-C1]    same page, first component (block statistics, cumulative-mass selection).
[MapFlow-C3]    same page, third component (mixing on chip, times the receiver's V).
[MapFlow-maps]  same page, the attention map as the shared state: the sender runs its own
                attention; the receiver reuses the sender's probabilities with its own V.

Readings where the pages are silent:

* a chunk of sequence s is its query rows [c0, e); it attends to keys [0, e) with the same
  causal mask and bias as the whole sequence (absolute positions). c0 is a multiple of B, so the
  chunk's row blocks are the sequence's own row blocks I = c0/B .. ceil(e/B) - 1, each with
  column blocks J = 0..I, and every result of a chunk equals the whole-sequence result of those
  rows (rows past e in a partial last block are absent);
* the sender's own output is the dense attention output O_s = P V_s with the sender's values,
  computed from the same probabilities as the map (before any block is dropped).

Parity status: pinned by ``tests/test_chunked_oracle.py``: the sender output against torch's
scaled_dot_product_attention in float64, and every chunk result against the whole-sequence
oracle (itself pinned in ``tests/test_oracle_pins.py``) for chunk starts at 0, inside and at the
end of each sequence.
"""

from __future__ import annotations

import dataclasses

import numpy as np

from synth import bf16_bits_to_f64

from .iamap_oracle import (RowBlockStats, block_masses, head_rows, receiver_values, scores,
                           select_blocks, softmax_rows)

__all__ = ["ChunkLayout", "chunk_layout", "chunk_rowblock_stats", "ChunkCompressResult",
           "compress_chunk", "mapped_av_chunk", "sender_output", "sender_output_chunk"]


@dataclasses.dataclass
class ChunkLayout:
    """Row blocks I0[s] .. nb[s]-1 of each sequence's chunk. Global chunk row-block index =
    rb_start[s] + I - I0[s]; chunk causal block (I, J) has index
    cb_start[s] + I(I+1)/2 - I0(I0+1)/2 + J."""
    B: int
    I0: list
    nb: list
    ends: list
    rb_start: list
    cb_start: list

    @property
    def num_rowblocks(self) -> int:
        return self.rb_start[-1]

    @property
    def num_causal_blocks(self) -> int:
        return self.cb_start[-1]

    def cb(self, s: int, I: int, J: int) -> int:
        I0 = self.I0[s]
        return self.cb_start[s] + I * (I + 1) // 2 - I0 * (I0 + 1) // 2 + J


def chunk_layout(cw) -> ChunkLayout:
    B = cw.B
    I0, nb, ends, rb, cb = [], [], [], [0], [0]
    for s in range(len(cw.starts)):
        e = int(cw.cu_k[s + 1] - cw.cu_k[s])
        c0 = int(cw.starts[s])
        if c0 % B:
            raise ValueError("chunk start %d of sequence %d is not a multiple of B=%d"
                             % (c0, s, B))
        if int(cw.cu_q[s + 1] - cw.cu_q[s]) != e - c0:
            raise ValueError("sequence %d: %d query rows for a chunk [%d, %d)"
                             % (s, int(cw.cu_q[s + 1] - cw.cu_q[s]), c0, e))
        i0, n_b = c0 // B, (e + B - 1) // B
        I0.append(i0)
        nb.append(n_b)
        ends.append(e)
        rb.append(rb[-1] + max(n_b - i0, 0))
        cb.append(cb[-1] + sum(I + 1 for I in range(i0, n_b)))
    return ChunkLayout(B=B, I0=I0, nb=nb, ends=ends, rb_start=rb, cb_start=cb)


def chunk_rowblock_stats(cw, lay: ChunkLayout, s: int, h: int, I: int) -> RowBlockStats:
    """[MapFlow-C1] for one row block of a chunk: the rows' probabilities over keys [0, e),
    block masses over J <= I and the kept set. row0 and the causal mask use the sequence-local
    (absolute) row index; the query rows come from the chunk's packed rows."""
    B = cw.B
    ka, e = int(cw.cu_k[s]), lay.ends[s]
    c0 = lay.I0[s] * B
    row0 = I * B
    R = min(B, e - row0)
    qa = int(cw.cu_q[s]) + row0 - c0
    k = head_rows(cw.k, ka, ka + e, h)
    q = head_rows(cw.q, qa, qa + R, h)
    p, lse = softmax_rows(scores(q, k, row0, cw.bias_window, cw.bias_value))
    m = block_masses(p, B, I + 1)
    kept, near = select_blocks(m, R, cw.tau)
    return RowBlockStats(p=p, lse=lse, masses=m, kept=kept, near=near, row0=row0, R=R)


@dataclasses.dataclass
class ChunkCompressResult:
    layout: ChunkLayout
    lse: np.ndarray     # [H_s, n_q]
    mass: np.ndarray    # [H_s, num chunk causal blocks]
    kept: np.ndarray    # bool, same shape
    near: np.ndarray    # bool, same shape


def compress_chunk(cw) -> ChunkCompressResult:
    lay = chunk_layout(cw)
    n_q = int(cw.cu_q[-1])
    lse = np.zeros((cw.H_s, n_q))
    mass = np.zeros((cw.H_s, lay.num_causal_blocks))
    kept = np.zeros((cw.H_s, lay.num_causal_blocks), dtype=bool)
    near = np.zeros_like(kept)
    for s in range(len(cw.starts)):
        qa, c0 = int(cw.cu_q[s]), lay.I0[s] * cw.B
        for h in range(cw.H_s):
            for I in range(lay.I0[s], lay.nb[s]):
                st = chunk_rowblock_stats(cw, lay, s, h, I)
                lse[h, qa + st.row0 - c0:qa + st.row0 - c0 + st.R] = st.lse
                b0 = lay.cb(s, I, 0)
                mass[h, b0:b0 + I + 1] = st.masses
                kept[h, b0:b0 + I + 1] = st.kept
                near[h, b0:b0 + I + 1] = st.near
    return ChunkCompressResult(layout=lay, lse=lse, mass=mass, kept=kept, near=near)


def mapped_av_chunk(cw, kept: np.ndarray) -> np.ndarray:
    """[MapFlow-C3] on a chunk: O_r[i] = sum_j (sum_s W[r,s] Pt_s[i,j]) V_r[j] for the chunk's
    rows i, over keys and receiver values [0, e); kept [H_s, num chunk causal blocks]."""
    lay = chunk_layout(cw)
    B = cw.B
    O = np.zeros((int(cw.cu_q[-1]), cw.H_r, cw.d_v))
    for s in range(len(cw.starts)):
        ka, e = int(cw.cu_k[s]), lay.ends[s]
        qa, c0 = int(cw.cu_q[s]), lay.I0[s] * B
        V = receiver_values(bf16_bits_to_f64(cw.v[ka:ka + e]), cw.H_r)   # [e, H_r, d_v]
        for I in range(lay.I0[s], lay.nb[s]):
            R = min(B, e - I * B)
            Pr = np.zeros((cw.H_r, R, e))
            b0 = lay.cb(s, I, 0)
            for h in range(cw.H_s):
                st = chunk_rowblock_stats(cw, lay, s, h, I)
                kmask = np.zeros(e, dtype=bool)
                for J in np.flatnonzero(kept[h, b0:b0 + I + 1]):
                    kmask[J * B:(J + 1) * B] = True
                pt = np.where(kmask[None, :], st.p, 0.0)
                Pr += cw.W[:, h].astype(np.float64)[:, None, None] * pt[None, :, :]
            O[qa + I * B - c0:qa + I * B - c0 + R] = np.einsum("rij,jre->ire", Pr, V)
    return O


def _sender_rows(q, k, vs, row0, bias_window, bias_value):
    p, _ = softmax_rows(scores(q, k, row0, bias_window, bias_value))
    return p @ vs


def sender_output(wl, v_s: np.ndarray) -> np.ndarray:
    """[GLIDE II-B], [MapFlow-maps] the sender's own attention output: O_s[i, h] =
    sum_{j <= i} p_h(i, j) V_s[j, h] per packed sequence (same bias as the map).
    v_s: bf16 bits [n, H_s, d_vs]. Returns [n, H_s, d_vs]."""
    O = np.zeros((wl.n, wl.H_s, v_s.shape[2]))
    for s in range(len(wl.seqlens)):
        a, b = int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])
        if b == a:
            continue   # an empty sequence has no rows
        for h in range(wl.H_s):
            O[a:b, h] = _sender_rows(head_rows(wl.q, a, b, h), head_rows(wl.k, a, b, h),
                                     bf16_bits_to_f64(v_s[a:b, h]), 0, wl.bias_window,
                                     wl.bias_value)
    return O


def sender_output_chunk(cw, v_s_keys: np.ndarray) -> np.ndarray:
    """The sender output of a chunk's rows; v_s_keys: bf16 bits [n_k, H_s, d_vs] packed like the
    chunk's keys (rows [0, e) of every sequence). Returns [n_q, H_s, d_vs]."""
    lay = chunk_layout(cw)
    O = np.zeros((int(cw.cu_q[-1]), cw.H_s, v_s_keys.shape[2]))
    for s in range(len(cw.starts)):
        ka, e = int(cw.cu_k[s]), lay.ends[s]
        qa, qb = int(cw.cu_q[s]), int(cw.cu_q[s + 1])
        c0 = lay.I0[s] * cw.B
        if qb == qa:
            continue   # a chunk with no query rows
        for h in range(cw.H_s):
            O[qa:qb, h] = _sender_rows(head_rows(cw.q, qa, qb, h), head_rows(cw.k, ka, ka + e, h),
                                       bf16_bits_to_f64(v_s_keys[ka:ka + e, h]), c0,
                                       cw.bias_window, cw.bias_value)
    return O
