"""Float64 CPU oracle: cross-model attention-map reuse (compress, mapped A.V, head matching).

TEST INFRASTRUCTURE ONLY. Imported by ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs; never by the product path. It shares no code with the CUDA
library: its only import from this repository is ``synth`` (seeded draws and exact bf16 upcast).

Everything is plain numpy in float64, on inputs upcast exactly from bf16, following the pages'
steps in their order, with no blocking or fusion beyond what those steps state.

Sources (cited below by the short tag in brackets):

[GLIDE II-B]   "GLIDE: Guided Layerwise Hybrid Attention for efficient LLM inference" page,
               Section II-B (attention and KV-cache basics): alpha_ij is the softmax over
               j <= i of scaled dot products q_i.k_j, and O_i = sum_j alpha_ij v_j.
[GLIDE II-C]   same page, Section II-C: the attention weights as a normalised exponential over a
               restricted key range (here: the causal range, plus an additive logit bias).
[MapFlow-maps] "PKU MapFlow: cross-model attention map reuse" news page, the paragraphs on the
               attention map as the shared state: a receiver keeps its own Value and uses the
               sender's token-to-token attention probabilities; layer mapping pairs depths and
               head mapping is a learned linear combination of sender heads.
[MapFlow-C1]   same page, "storage and execution" part, first component: keep regular 2-D
               blocks chosen by cumulative attention probability, stored block-sparse; first
               block-level statistics, then extraction of the kept blocks, with no dense map.
[MapFlow-C3]   same page, third component: read the sparse blocks, combine the heads linearly on
               chip, multiply by the receiver's Value and accumulate the output.
[IAM-1]        "IAM: Efficient Inference through Attention Mapping between Different-scale LLMs"
               notes page, Method section 1 (similarity metric): attention matrices of the small
               and the large model are flattened to vectors; cosine similarity is the metric.
[IAM-4]        same page, Method section 4 (mapping and inference): at prefill, pairwise cosine
               similarity of all attention matrices gives, for each head of each mapped large
               layer, the most similar small-model head; at decode a mapped layer uses the small
               model's attention directly (no Q/K projection, no QK^T, no K cache); prompts longer
               than tau_t are truncated for the similarity computation.

Readings where the pages are silent:
* cumulative-mass selection is per (sender head, row block) and normalised by the row block's
  total mass, which equals its number of valid rows; tau >= 1 keeps every causal block;
* ties between equal block masses are broken by the lower column-block index;
* kept probabilities are not renormalised; absent (head, block) pairs count as zero in mixing;
* the local logit bias is added after the 1/sqrt(d) scaling, for 0 <= i - j < window.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py`` against an
independent definition (torch SDPA, closed forms in exact rationals, brute-force enumeration,
scikit-learn cosine similarity, planted ground truth) or an invariant; none is "parity unpinned".
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

from synth import bf16_bits_to_f64

NEAR_EPS = 1e-5

__all__ = [
    "NEAR_EPS", "CausalLayout", "causal_layout", "head_rows", "scores", "softmax_rows",
    "block_masses", "select_blocks", "RowBlockStats", "rowblock_stats", "CompressResult",
    "compress", "union_bsr", "masked_tile", "mapped_av_rows", "mapped_av", "mapped_av_paged",
    "attention_map", "head_match", "mapping_consistency", "receiver_values",
    "sender_decode_rows",
]


# ----------------------------------------------------------------------------------------------
# Block enumeration shared by all outputs (a layout convention, not arithmetic of the method)
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class CausalLayout:
    """Row blocks and causal blocks of packed sequences.

    Row block I of sequence s covers sequence-local rows [I*B, min((I+1)*B, L_s)). Global row-block
    index = rb_start[s] + I. Causal block (I, J), J <= I, of sequence s has index
    cb_start[s] + I*(I+1)/2 + J.
    """
    seqlens: list
    B: int
    nb: list
    rb_start: list
    cb_start: list

    @property
    def num_rowblocks(self) -> int:
        return self.rb_start[-1]

    @property
    def num_causal_blocks(self) -> int:
        return self.cb_start[-1]

    def cb(self, s: int, I: int, J: int) -> int:
        return self.cb_start[s] + I * (I + 1) // 2 + J


def causal_layout(seqlens, B: int) -> CausalLayout:
    nb = [(int(L) + B - 1) // B for L in seqlens]
    rb = [0]
    cb = [0]
    for x in nb:
        rb.append(rb[-1] + x)
        cb.append(cb[-1] + x * (x + 1) // 2)
    return CausalLayout(seqlens=[int(L) for L in seqlens], B=B, nb=nb, rb_start=rb, cb_start=cb)


def head_rows(bits: np.ndarray, start: int, stop: int, h: int) -> np.ndarray:
    """Rows [start, stop) of head h of a [n, H, d] bf16 tensor, upcast exactly to float64."""
    return bf16_bits_to_f64(bits[start:stop, h, :])


# ----------------------------------------------------------------------------------------------
# Attention probabilities [GLIDE II-B], [GLIDE II-C]
# ----------------------------------------------------------------------------------------------

def scores(q_rows: np.ndarray, k: np.ndarray, row0: int, bias_window: int = 0,
           bias_value: float = 0.0) -> np.ndarray:
    """Causal logits s_ij = q_i.k_j / sqrt(d) (+ bias_value if 0 <= i-j < bias_window), -inf for j > i.

    q_rows: [R, d] rows i = row0 .. row0+R-1 (sequence-local); k: [L, d] all keys of the sequence.
    """
    d = q_rows.shape[1]
    s = (q_rows @ k.T) / math.sqrt(d)
    i = np.arange(row0, row0 + q_rows.shape[0])[:, None]
    j = np.arange(k.shape[0])[None, :]
    if bias_window > 0:
        s = s + np.where((i - j >= 0) & (i - j < bias_window), bias_value, 0.0)
    return np.where(j <= i, s, -np.inf)


def softmax_rows(s: np.ndarray):
    """Row-wise softmax by max subtraction; returns (p, lse) with lse_i = log sum_j exp(s_ij)."""
    m = np.max(s, axis=1, keepdims=True)
    e = np.exp(s - m)
    l = np.sum(e, axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


# ----------------------------------------------------------------------------------------------
# Block statistics and cumulative-mass selection [MapFlow-C1]
# ----------------------------------------------------------------------------------------------

def block_masses(p_rows: np.ndarray, B: int, num_col_blocks: int) -> np.ndarray:
    """mass[J] = sum of p over the rows given and columns [J*B, (J+1)*B)."""
    L = p_rows.shape[1]
    out = np.zeros(num_col_blocks)
    for J in range(num_col_blocks):
        out[J] = np.sum(p_rows[:, J * B:min((J + 1) * B, L)])
    return out


def select_blocks(masses: np.ndarray, R: int, tau: float, eps: float = NEAR_EPS):
    """Keep the shortest prefix of blocks, in order of decreasing mass (ties: lower J first), whose
    cumulative mass reaches tau * R. tau >= 1 keeps all blocks.

    Returns (kept, near): boolean arrays over J. ``near`` marks blocks whose membership could flip
    under a perturbation of the normalised masses by eps. The selection threshold is the
    normalised mass t of the last kept block; three cases can flip:
      (a) a dropped block whose normalised mass is within eps of t: it can change places with the
          last kept block, so it, the last kept block and any other block within eps of t are
          near (the last kept block is never compared with its own mass: clear margins mark
          nothing);
      (b) the cumulative mass before the last kept block is within eps of tau: that block may not
          be needed, and neither may any kept block within eps of t that could take its place;
      (c) the cumulative mass through the last kept block is within eps of tau: the first dropped
          block may be needed, and so may any dropped block within eps of its mass.
    """
    nJ = len(masses)
    kept = np.zeros(nJ, dtype=bool)
    near = np.zeros(nJ, dtype=bool)
    if tau >= 1.0:
        kept[:] = True
        return kept, near
    mhat = masses / R
    order = sorted(range(nJ), key=lambda J: (-mhat[J], J))
    cum = 0.0
    last = -1
    cum_before_last = cum_through_last = 0.0
    for t, J in enumerate(order):
        if cum >= tau:
            break
        kept[J] = True
        last = t
        cum_before_last = cum
        cum += mhat[J]
        cum_through_last = cum
    if last < 0:
        return kept, near
    J_last = order[last]
    close_t = np.abs(mhat - mhat[J_last]) <= eps
    if (close_t & ~kept).any():                                       # (a)
        near |= close_t
    if abs(cum_before_last - tau) <= eps:                             # (b)
        near |= close_t & kept
        near[J_last] = True
    if last + 1 < nJ and abs(cum_through_last - tau) <= eps:          # (c)
        J_first = order[last + 1]
        near |= (np.abs(mhat - mhat[J_first]) <= eps) & ~kept
    return kept, near


@dataclasses.dataclass
class RowBlockStats:
    p: np.ndarray        # [R, L] float64 attention probabilities of the valid rows
    lse: np.ndarray      # [R]
    masses: np.ndarray   # [I+1]
    kept: np.ndarray     # [I+1] bool
    near: np.ndarray     # [I+1] bool
    row0: int            # sequence-local first row
    R: int               # valid rows


def rowblock_stats(q_bits, k_bits, cu_seqlens, s: int, h: int, I: int, B: int, tau: float,
                   bias_window: int = 0, bias_value: float = 0.0) -> RowBlockStats:
    """Steps of [MapFlow-C1] for one (sequence, sender head, row block): probabilities of the
    block's rows, block-level statistics (masses over J <= I), then the cumulative-mass choice."""
    a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
    L = b - a
    row0 = I * B
    R = min(B, L - row0)
    k = head_rows(k_bits, a, b, h)
    q = head_rows(q_bits, a + row0, a + row0 + R, h)
    p, lse = softmax_rows(scores(q, k, row0, bias_window, bias_value))
    m = block_masses(p, B, I + 1)
    kept, near = select_blocks(m, R, tau)
    return RowBlockStats(p=p, lse=lse, masses=m, kept=kept, near=near, row0=row0, R=R)


@dataclasses.dataclass
class CompressResult:
    layout: CausalLayout
    lse: np.ndarray     # [H_s, n]
    mass: np.ndarray    # [H_s, num_causal_blocks]
    kept: np.ndarray    # [H_s, num_causal_blocks] bool
    near: np.ndarray    # [H_s, num_causal_blocks] bool


def compress(wl) -> CompressResult:
    """Block statistics and kept sets of every (sender head, causal block) of a prefill workload."""
    lay = causal_layout(wl.seqlens, wl.B)
    n = int(wl.cu_seqlens[-1])
    lse = np.zeros((wl.H_s, n))
    mass = np.zeros((wl.H_s, lay.num_causal_blocks))
    kept = np.zeros((wl.H_s, lay.num_causal_blocks), dtype=bool)
    near = np.zeros((wl.H_s, lay.num_causal_blocks), dtype=bool)
    for s in range(len(wl.seqlens)):
        a = int(wl.cu_seqlens[s])
        for h in range(wl.H_s):
            for I in range(lay.nb[s]):
                st = rowblock_stats(wl.q, wl.k, wl.cu_seqlens, s, h, I, wl.B, wl.tau,
                                    wl.bias_window, wl.bias_value)
                lse[h, a + st.row0:a + st.row0 + st.R] = st.lse
                c0 = lay.cb(s, I, 0)
                mass[h, c0:c0 + I + 1] = st.masses
                kept[h, c0:c0 + I + 1] = st.kept
                near[h, c0:c0 + I + 1] = st.near
    return CompressResult(layout=lay, lse=lse, mass=mass, kept=kept, near=near)


def union_bsr(kept: np.ndarray, lay: CausalLayout):
    """Block-sparse storage of per-head kept sets: per row block the union of kept column blocks
    (ascending), a head bit mask per stored block, and the tile offset of its first present head
    (tiles of present heads are consecutive in head order). Returns
    (row_ptr [num_rowblocks+1], col_idx, headmask (uint64), val_off (int64), nnz_tiles)."""
    H_s = kept.shape[0]
    row_ptr = [0]
    col_idx, headmask, val_off = [], [], []
    tiles = 0
    for s in range(len(lay.seqlens)):
        for I in range(lay.nb[s]):
            for J in range(I + 1):
                c = lay.cb(s, I, J)
                m = 0
                for h in range(H_s):
                    if kept[h, c]:
                        m |= 1 << h
                if m:
                    col_idx.append(J)
                    headmask.append(m)
                    val_off.append(tiles)
                    tiles += bin(m).count("1")
            row_ptr.append(len(col_idx))
    return (np.array(row_ptr, dtype=np.int64), np.array(col_idx, dtype=np.int64),
            np.array(headmask, dtype=np.uint64), np.array(val_off, dtype=np.int64), tiles)


def masked_tile(st: RowBlockStats, J: int, B: int) -> np.ndarray:
    """The B x B probability tile of column block J for a row block (zeros for rows or columns
    outside the sequence; causal zeros come from p itself)."""
    t = np.zeros((B, B))
    L = st.p.shape[1]
    c1 = min((J + 1) * B, L)
    t[:st.R, :c1 - J * B] = st.p[:, J * B:c1]
    return t


# ----------------------------------------------------------------------------------------------
# Mapped attention output [MapFlow-maps], [MapFlow-C3], [GLIDE II-B]
# ----------------------------------------------------------------------------------------------

def receiver_values(V: np.ndarray, H_r: int) -> np.ndarray:
    """The value vectors each receiver head uses: V [tokens, H_kv, d_v] with H_kv dividing H_r;
    with grouped values (H_kv < H_r) receiver head r reads value head r // (H_r / H_kv), the
    consecutive-group sharing of grouped-query attention. Returns [tokens, H_r, d_v]."""
    H_kv = V.shape[1]
    if H_r % H_kv:
        raise ValueError("H_kv=%d does not divide H_r=%d" % (H_kv, H_r))
    return V[:, np.arange(H_r) // (H_r // H_kv)]


def mapped_av_rows(wl, s: int, I: int, kept_of, stats_of=None) -> np.ndarray:
    """O rows of one row block: O_r[i] = sum_j (sum_s W[r,s] Pt_s[i,j]) V_r[j], with Pt_s the
    sender head's probabilities restricted to its kept blocks (zero elsewhere).

    kept_of(h) -> bool array over J = 0..I (the kept set to use for sender head h).
    stats_of(h) -> RowBlockStats (optional cache). Returns [R, H_r, d_v].
    """
    a, b = int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])
    L = b - a
    B = wl.B
    row0 = I * B
    R = min(B, L - row0)
    Pr = np.zeros((wl.H_r, R, L))
    for h in range(wl.H_s):
        st = stats_of(h) if stats_of is not None else rowblock_stats(
            wl.q, wl.k, wl.cu_seqlens, s, h, I, B, wl.tau, wl.bias_window, wl.bias_value)
        kmask = np.zeros(L, dtype=bool)
        for J in np.flatnonzero(np.asarray(kept_of(h), dtype=bool)):
            kmask[J * B:(J + 1) * B] = True
        pt = np.where(kmask[None, :], st.p, 0.0)
        Pr += wl.W[:, h].astype(np.float64)[:, None, None] * pt[None, :, :]
    V = receiver_values(bf16_bits_to_f64(wl.v[a:b]), wl.H_r)   # [L, H_r, d_v]
    O = np.einsum("rij,jre->ire", Pr, V)
    return O


def mapped_av(wl, kept: np.ndarray) -> np.ndarray:
    """O [n, H_r, d_v] of a prefill workload for given per-head kept sets [H_s, num_causal_blocks]."""
    lay = causal_layout(wl.seqlens, wl.B)
    n = int(wl.cu_seqlens[-1])
    O = np.zeros((n, wl.H_r, wl.d_v))
    for s in range(len(wl.seqlens)):
        a = int(wl.cu_seqlens[s])
        for I in range(lay.nb[s]):
            c0 = lay.cb(s, I, 0)
            rows = mapped_av_rows(wl, s, I, lambda h: kept[h, c0:c0 + I + 1])
            O[a + I * wl.B:a + I * wl.B + rows.shape[0]] = rows
    return O


def sender_decode_rows(dw) -> np.ndarray:
    """The small model's attention row of a decode step [IAM-4] (the row a mapped layer reuses)
    and the textbook softmax of scaled dot products [GLIDE II-B]: p[b, h, j] = softmax over
    j < ctx_len[b] of q_s[b, h] . k_s[b, j, h] / sqrt(d_s), the keys gathered through the page
    table. Returns float64 [batch, H_s, max_ctx] with zeros at j >= ctx_len[b]."""
    d = dw.q_s.shape[2]
    max_ctx = int(np.max(dw.ctx_lens))
    P = np.zeros((dw.batch, dw.H_s, max_ctx))
    ps = dw.page_size
    for b in range(dw.batch):
        c = int(dw.ctx_lens[b])
        if c == 0:
            continue
        pages = dw.page_table[b, (np.arange(c) // ps)]
        K = bf16_bits_to_f64(dw.k_pages_s[pages, np.arange(c) % ps])      # [c, H_s, d]
        q = bf16_bits_to_f64(dw.q_s[b])                                      # [H_s, d]
        s = np.einsum("hd,jhd->hj", q, K) / math.sqrt(d)
        P[b, :, :c], _ = softmax_rows(s)
    return P


def mapped_av_paged(dw) -> np.ndarray:
    """Decode step on a mapped layer [IAM-4]: O[b, r] = sum_j (sum_s W[r,s] p[b,s,j]) V[b, j, r]
    for j < ctx_len[b], with V gathered through the page table. Returns [batch, H_r, d_v]."""
    O = np.zeros((dw.batch, dw.H_r, dw.d_v))
    ps = dw.page_size
    W = dw.W.astype(np.float64)
    for b in range(dw.batch):
        c = int(dw.ctx_lens[b])
        pr = W @ dw.p_rows[b, :, :c].astype(np.float64)            # [H_r, c]
        pages = dw.page_table[b, (np.arange(c) // ps)]
        V = receiver_values(bf16_bits_to_f64(dw.v_pages[pages, np.arange(c) % ps]), dw.H_r)
        O[b] = np.einsum("rj,jre->re", pr, V)
    return O


# ----------------------------------------------------------------------------------------------
# Head matching [IAM-1], [IAM-4]
# ----------------------------------------------------------------------------------------------

def attention_map(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Causal softmax map A = softmax(q k^T / sqrt(d)) over j <= i, [n, n] float64 (zeros above the
    diagonal)."""
    p, _ = softmax_rows(scores(q, k, 0))
    return p


def head_match(hm, n_used=None, metric="cosine"):
    """Similarity of the flattened causal maps of every large head with every small head, and
    the most similar small head per large head (ties: lowest index). IAM notes, method section 1
    (flatten the attention matrices, compare with cosine similarity, Minkowski distance or the
    Pearson correlation) and section 4 (for each head of a mapped large layer, the most similar
    small head; prompts longer than tau_t are truncated).

    metric: "cosine" (a.b / |a||b|), "pearson" (the correlation coefficient of the n*n entries of
    the two maps: the cosine of the maps less their means) or "euclidean" (the Minkowski distance
    with p = 2, negated so that the largest value is the most similar head).

    Small heads are indexed layer-major (layer * H_small + head), large heads likewise. Truncation
    to the first n_used tokens (tau_t) uses the maps of that prefix. Returns (S [L_l*H_large,
    L_s*H_small], argmax int32 [L_l, H_large])."""
    n = hm.n if n_used is None else int(n_used)
    ns = hm.L_s * hm.H_small

    def flat_maps(q, k, layers, heads):
        out = np.zeros((layers * heads, n * n))
        for l in range(layers):
            for h in range(heads):
                A = attention_map(bf16_bits_to_f64(q[l, :n, h]), bf16_bits_to_f64(k[l, :n, h]))
                out[l * heads + h] = A.ravel()
        return out

    small = flat_maps(hm.q_small, hm.k_small, hm.L_s, hm.H_small)
    if metric == "pearson":
        small = small - small.mean(axis=1, keepdims=True)
    C = np.zeros((hm.L_l * hm.H_large, ns))
    for l in range(hm.L_l):
        large = np.zeros((hm.H_large, n * n))
        for h in range(hm.H_large):
            A = attention_map(bf16_bits_to_f64(hm.q_large[l, :n, h]),
                              bf16_bits_to_f64(hm.k_large[l, :n, h]))
            large[h] = A.ravel()
        rows = slice(l * hm.H_large, (l + 1) * hm.H_large)
        if metric in ("cosine", "pearson"):
            if metric == "pearson":
                large = large - large.mean(axis=1, keepdims=True)
            C[rows] = (large @ small.T) / (np.linalg.norm(large, axis=1)[:, None]
                                           * np.linalg.norm(small, axis=1)[None, :])
        elif metric == "euclidean":
            for h in range(hm.H_large):
                C[l * hm.H_large + h] = -np.linalg.norm(small - large[h][None, :], axis=1)
        else:
            raise ValueError("unknown metric %r" % (metric,))
    arg = np.argmax(C, axis=1).astype(np.int32).reshape(hm.L_l, hm.H_large)
    return C, arg


def mapping_consistency(a, b) -> float:
    """Share of large heads that two head mappings send to the same small head (IAM notes,
    method section 3: the mapping built at prefill stays consistent during decode)."""
    a = np.asarray(a).ravel()
    b = np.asarray(b).ravel()
    return float(np.mean(a == b))
