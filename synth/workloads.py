"""Seeded synthetic workloads (shapes, value distributions, sinks, page tables, planted mappings).

Every array is drawn from ``numpy.random.default_rng(seed)`` (PCG64) in float32 in a fixed draw
order, then rounded to bf16 with round-to-nearest-even. bf16 tensors are carried as ``uint16``
bit patterns so that both the oracle (which upcasts them exactly to float64) and the CUDA path
(which views them as ``torch.bfloat16``) see the same numbers.

Workloads (one per configuration of the benchmark description):

* ``tiny``       n=512, H_s=8, d=64, H_r=4, d_v=64, B=64, tau=0.95, std 1.5, sink, seed 0
* ``prefill8k``  n=8192, H_s=32, d=128, H_r=24, d_v=128, tau=0.95, std 1.5, sink,
                 local bias +2.0 on |i-j| < 128
* ``varlen40k``  4 packed sequences 4096/8192/12288/16384 (40960 tokens), H_s=40, H_r=32,
                 d=d_v=128, tau=0.9, std 1.5, sink on token 0 of every sequence
* head match     n=1024, small 24 layers x 14 heads d=64, large 8 layers x 64 heads d=128,
                 each large head a noisy zero-padded copy of a uniformly drawn small head
* decode         batch 4, context 8704, sender 14 heads, receiver 64 heads d_v=128, one-hot
                 W, V cache in 16-token pages under a random page table
* prefix index   token ids of the varlen prompts as the cached set, 16 prompts sharing seeded
                 prefixes with them (block boundaries and mid-block), uniform over a 151936 vocab
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np


# ----------------------------------------------------------------------------------------------
# bf16 bit handling (rounding of random draws; not part of the method)
# ----------------------------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); return the uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns to float64."""
    return bf16_bits_to_f32(b).astype(np.float64)


def _normal_bits(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


# ----------------------------------------------------------------------------------------------
# Prefill workloads: map_compress + mapped_av
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class PrefillWorkload:
    name: str
    seqlens: list
    H_s: int
    d: int
    H_r: int
    d_v: int
    B: int
    tau: float
    bias_window: int
    bias_value: float
    q: np.ndarray          # uint16 bf16 bits [n, H_s, d]
    k: np.ndarray          # uint16 bf16 bits [n, H_s, d]
    v: np.ndarray          # uint16 bf16 bits [n, H_r, d_v]
    W: np.ndarray          # float32 [H_r, H_s]
    cu_seqlens: np.ndarray  # int32 [S+1]

    @property
    def n(self) -> int:
        return int(self.cu_seqlens[-1])

    @property
    def num_seqs(self) -> int:
        return len(self.seqlens)


PREFILL_CONFIGS = {
    "tiny": dict(seqlens=[512], H_s=8, d=64, H_r=4, d_v=64, B=64, tau=0.95, std=1.5,
                 sink=True, bias_window=0, bias_value=0.0),
    "prefill8k": dict(seqlens=[8192], H_s=32, d=128, H_r=24, d_v=128, B=64, tau=0.95, std=1.5,
                      sink=True, bias_window=128, bias_value=2.0),
    "varlen40k": dict(seqlens=[4096, 8192, 12288, 16384], H_s=40, d=128, H_r=32, d_v=128, B=64,
                      tau=0.9, std=1.5, sink=True, bias_window=0, bias_value=0.0),
}


def make_prefill(seqlens, H_s, d, H_r, d_v, B=64, tau=0.95, std=1.5, sink=True,
                 bias_window=0, bias_value=0.0, seed=0, name="custom",
                 q_zero=False, v_const=None, H_kv=None) -> PrefillWorkload:
    """Draw Q, K, V (bf16) and W (fp32) in the order Q, K, V, W.

    ``sink`` multiplies the key of token 0 of every sequence by 4 (a power of two, so exact) before
    bf16 rounding. ``q_zero`` zeroes Q (uniform attention rows); ``v_const`` replaces V by that
    constant. Both are for closed-form checks. ``H_kv`` (dividing H_r) draws grouped receiver
    values: V has H_kv heads.
    """
    seqlens = [int(x) for x in seqlens]
    n = int(sum(seqlens))
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    rng = np.random.default_rng(seed)
    q = _normal_bits(rng, (n, H_s, d), std)
    k = _normal_bits(rng, (n, H_s, d), std)
    v = _normal_bits(rng, (n, H_r if H_kv is None else int(H_kv), d_v), std)
    W = rng.standard_normal((H_r, H_s), dtype=np.float32) * np.float32(math.sqrt(1.0 / H_s))
    if sink:
        for s in range(len(seqlens)):
            if seqlens[s] > 0:
                k[cu[s]] *= np.float32(4.0)
    if q_zero:
        q[:] = 0.0
    if v_const is not None:
        v[:] = np.float32(v_const)
    return PrefillWorkload(name=name, seqlens=seqlens, H_s=H_s, d=d, H_r=H_r, d_v=d_v, B=B,
                           tau=float(tau), bias_window=int(bias_window),
                           bias_value=float(bias_value), q=bf16_bits(q), k=bf16_bits(k),
                           v=bf16_bits(v), W=np.ascontiguousarray(W, dtype=np.float32),
                           cu_seqlens=cu)


def prefill_config(name: str, seed: int = 0) -> PrefillWorkload:
    c = dict(PREFILL_CONFIGS[name])
    return make_prefill(seed=seed, name=name, **c)


# ----------------------------------------------------------------------------------------------
# Head-match calibration workload
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class HeadMatchWorkload:
    n: int
    L_s: int
    H_small: int
    d_small: int
    L_l: int
    H_large: int
    d_large: int
    q_small: np.ndarray   # uint16 bf16 [L_s, n, H_small, d_small]
    k_small: np.ndarray
    q_large: np.ndarray   # uint16 bf16 [L_l, n, H_large, d_large]
    k_large: np.ndarray
    planted: np.ndarray   # int32 [L_l, H_large]: small head index (layer * H_small + head)


def make_head_match(n=1024, L_s=24, H_small=14, d_small=64, L_l=8, H_large=64, d_large=128,
                    noise=0.3, seed=0) -> HeadMatchWorkload:
    """Small Q, K ~ N(0,1); each large head copies a uniformly drawn small head's Q and K into
    dims [0, d_small), zero elsewhere, plus N(0, noise^2) on every dim. Draw order: small Q,
    small K, planted assignment, large-Q noise, large-K noise."""
    rng = np.random.default_rng(seed)
    qs = rng.standard_normal((L_s, n, H_small, d_small), dtype=np.float32)
    ks = rng.standard_normal((L_s, n, H_small, d_small), dtype=np.float32)
    planted = rng.integers(0, L_s * H_small, size=(L_l, H_large)).astype(np.int32)
    nq = rng.standard_normal((L_l, n, H_large, d_large), dtype=np.float32) * np.float32(noise)
    nk = rng.standard_normal((L_l, n, H_large, d_large), dtype=np.float32) * np.float32(noise)
    ql = nq
    kl = nk
    dd = min(d_small, d_large)
    for ll in range(L_l):
        for h in range(H_large):
            s = int(planted[ll, h])
            ql[ll, :, h, :dd] += qs[s // H_small, :, s % H_small, :dd]
            kl[ll, :, h, :dd] += ks[s // H_small, :, s % H_small, :dd]
    return HeadMatchWorkload(n=n, L_s=L_s, H_small=H_small, d_small=d_small, L_l=L_l,
                             H_large=H_large, d_large=d_large, q_small=bf16_bits(qs),
                             k_small=bf16_bits(ks), q_large=bf16_bits(ql), k_large=bf16_bits(kl),
                             planted=planted)


def head_match_config(seed: int = 0) -> HeadMatchWorkload:
    return make_head_match(seed=seed)


# ----------------------------------------------------------------------------------------------
# Decode workload (paged V cache, one-hot W)
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class DecodeWorkload:
    batch: int
    ctx_lens: np.ndarray    # int32 [batch]
    H_s: int
    H_r: int
    d_v: int
    page_size: int
    p_rows: np.ndarray      # float32 [batch, H_s, max_ctx]; each row a probability vector
    W: np.ndarray           # float32 [H_r, H_s] (one-hot rows)
    assign: np.ndarray      # int32 [H_r]: the sender head of each receiver head
    v_pages: np.ndarray     # uint16 bf16 [num_pages, page_size, H_r, d_v]
    page_table: np.ndarray  # int32 [batch, max_pages]
    q_s: np.ndarray = None        # uint16 bf16 [batch, H_s, d_s]: the small model's query
    k_pages_s: np.ndarray = None  # uint16 bf16 [num_pages, page_size, H_s, d_s]: its keys, on
                                  # the same pages as the large model's values


def make_decode(batch=4, ctx=8704, H_s=14, H_r=64, d_v=128, page_size=16, sink_weight=64.0,
                ctx_lens=None, seed=0, H_kv=None, d_s=64) -> DecodeWorkload:
    """Draw order: sender rows, one-hot assignment, V pages, page-table permutation, the small
    model's query, its key pages.

    ``p_rows`` are drawn from a Dirichlet distribution (normalised Gamma draws) with a heavier
    concentration at position 0 (unused tail positions, ctx_len < max, are zero): an extra case
    of given rows. The configuration's rows are the small model's own softmax rows over its keys:
    ``q_s`` and ``k_pages_s`` (N(0, 1), head dim d_s, keys on the same pages as the values) are
    the inputs from which they are computed. ``H_kv`` (dividing H_r) gives the page pool that many
    value heads.
    """
    if ctx_lens is None:
        ctx_lens = [ctx] * batch
    ctx_lens = np.asarray(ctx_lens, dtype=np.int32)
    max_ctx = int(ctx_lens.max())
    max_pages = (max_ctx + page_size - 1) // page_size
    rng = np.random.default_rng(seed)
    g = rng.gamma(shape=1.0, scale=1.0, size=(batch, H_s, max_ctx))
    g[:, :, 0] *= sink_weight
    for b in range(batch):
        g[b, :, ctx_lens[b]:] = 0.0
    den = g.sum(axis=2, keepdims=True)
    den[den == 0] = 1.0
    p_rows = (g / den).astype(np.float32)
    assign = rng.integers(0, H_s, size=H_r).astype(np.int32)
    W = np.zeros((H_r, H_s), dtype=np.float32)
    W[np.arange(H_r), assign] = 1.0
    num_pages = batch * max_pages
    v = rng.standard_normal((num_pages, page_size, H_r if H_kv is None else int(H_kv), d_v),
                            dtype=np.float32)
    perm = rng.permutation(num_pages).astype(np.int32)
    page_table = perm.reshape(batch, max_pages)
    q_s = rng.standard_normal((batch, H_s, d_s), dtype=np.float32)
    k_s = rng.standard_normal((num_pages, page_size, H_s, d_s), dtype=np.float32)
    return DecodeWorkload(batch=batch, ctx_lens=ctx_lens, H_s=H_s, H_r=H_r, d_v=d_v,
                          page_size=page_size, p_rows=p_rows, W=W, assign=assign,
                          v_pages=bf16_bits(v), page_table=page_table, q_s=bf16_bits(q_s),
                          k_pages_s=bf16_bits(k_s))


def decode_config(seed: int = 0) -> DecodeWorkload:
    return make_decode(seed=seed)


# ----------------------------------------------------------------------------------------------
# Token ids for the prefix-hash block index
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class PrefixWorkload:
    B: int
    salt: int
    cached_tokens: np.ndarray   # int32, packed sequences already in the index
    cached_cu: np.ndarray       # int32 [S_c + 1]
    query_tokens: np.ndarray    # int32, packed prompts looked up
    query_cu: np.ndarray        # int32 [S_q + 1]
    shared: list                # per prompt: (cached sequence it copies from or -1, tokens copied)


def _pack(seqs):
    cu = np.zeros(len(seqs) + 1, dtype=np.int32)
    cu[1:] = np.cumsum([len(x) for x in seqs])
    toks = np.concatenate(seqs).astype(np.int32) if seqs else np.zeros(0, np.int32)
    return toks, cu


def make_prefix_requests(cached_lens, query_lens, B=64, vocab=151936, seed=0,
                         p_fresh=0.2) -> PrefixWorkload:
    """Draw order: salt, cached sequences, then per prompt its source, shared length and tokens.

    Token ids are uniform in [0, vocab). Cached sequence i > 0 copies a prefix of a uniformly
    drawn earlier cached sequence with probability 1/2 (so the cached set holds repeated prefix
    blocks). Each prompt copies the first m tokens of a uniformly drawn cached sequence (with
    probability 1 - p_fresh), m uniform in [0, min(lengths)], every third one rounded down to a
    multiple of B, and then differs at token m (when m is shorter than the prompt).
    """
    rng = np.random.default_rng(seed)
    salt = int(rng.integers(0, 2**63 - 1, dtype=np.int64))
    cached = []
    for i, L in enumerate(cached_lens):
        x = rng.integers(0, vocab, size=int(L), dtype=np.int64).astype(np.int32)
        if i > 0 and rng.random() < 0.5:
            src = cached[int(rng.integers(0, i))]
            m = int(rng.integers(0, min(len(src), len(x)) + 1))
            x[:m] = src[:m]
        cached.append(x)
    queries, shared = [], []
    for j, L in enumerate(query_lens):
        x = rng.integers(0, vocab, size=int(L), dtype=np.int64).astype(np.int32)
        if cached and rng.random() >= p_fresh:
            c = int(rng.integers(0, len(cached)))
            m = int(rng.integers(0, min(len(cached[c]), len(x)) + 1))
            if j % 3 == 0:
                m -= m % B
            x[:m] = cached[c][:m]
            if m < len(x) and m < len(cached[c]):
                x[m] = (cached[c][m] + 1 + int(rng.integers(0, vocab - 1))) % vocab
            shared.append((c, m))
        else:
            shared.append((-1, 0))
        queries.append(x)
    ct, ccu = _pack(cached)
    qt, qcu = _pack(queries)
    return PrefixWorkload(B=B, salt=salt, cached_tokens=ct, cached_cu=ccu, query_tokens=qt,
                          query_cu=qcu, shared=shared)


def prefix_config(seed: int = 0) -> PrefixWorkload:
    """The packed prompts of the varlen prefill workload (4096/8192/12288/16384 tokens) as the
    cached set, and 16 prompts of those lengths (four each) looked up against it."""
    lens = [4096, 8192, 12288, 16384]
    return make_prefix_requests(lens, lens * 4, seed=seed)


# ----------------------------------------------------------------------------------------------
# Chunked prefill (a slice of a prefill workload) and sender values
# ----------------------------------------------------------------------------------------------

@dataclasses.dataclass
class ChunkWorkload:
    """Query rows [start, end) of every sequence of a prefill workload, with the keys and values
    of rows [0, end): the state of a chunked prefill whose earlier chunks are cached."""
    B: int
    H_s: int
    d: int
    H_r: int
    d_v: int
    tau: float
    bias_window: int
    bias_value: float
    W: np.ndarray            # float32 [H_r, H_s]
    starts: list             # sequence-local first query row of each chunk
    q: np.ndarray            # uint16 bf16 bits [n_q, H_s, d], chunk rows only
    cu_q: np.ndarray         # int32 [S+1]
    k: np.ndarray            # uint16 bf16 bits [n_k, H_s, d], rows [0, end) of every sequence
    v: np.ndarray            # uint16 bf16 bits [n_k, H_kv, d_v]
    cu_k: np.ndarray         # int32 [S+1]


def chunk_of(wl: PrefillWorkload, starts, ends=None) -> ChunkWorkload:
    """Slices (no arithmetic): queries of rows [starts[s], ends[s]) and keys/values of rows
    [0, ends[s]) of sequence s; ends default to the sequence lengths."""
    ends = list(wl.seqlens) if ends is None else [int(e) for e in ends]
    qs, ks, vs = [], [], []
    cu_q, cu_k = [0], [0]
    for s, (a0, e) in enumerate(zip(starts, ends)):
        a = int(wl.cu_seqlens[s])
        if not 0 <= int(a0) <= e <= wl.seqlens[s]:
            raise ValueError("chunk [%d, %d) outside sequence %d" % (a0, e, s))
        qs.append(wl.q[a + int(a0):a + e])
        ks.append(wl.k[a:a + e])
        vs.append(wl.v[a:a + e])
        cu_q.append(cu_q[-1] + e - int(a0))
        cu_k.append(cu_k[-1] + e)
    return ChunkWorkload(B=wl.B, H_s=wl.H_s, d=wl.d, H_r=wl.H_r, d_v=wl.d_v, tau=wl.tau,
                         bias_window=wl.bias_window, bias_value=wl.bias_value, W=wl.W,
                         starts=[int(x) for x in starts], q=np.concatenate(qs),
                         cu_q=np.array(cu_q, dtype=np.int32), k=np.concatenate(ks),
                         v=np.concatenate(vs), cu_k=np.array(cu_k, dtype=np.int32))


def make_sender_values(wl: PrefillWorkload, d_vs=None, std=1.0, seed=1) -> np.ndarray:
    """The sender's own values V_s, bf16 bits [n, H_s, d_vs] ~ N(0, std^2), from a generator of
    their own (so the prefill workload's draws are unchanged)."""
    rng = np.random.default_rng(seed)
    return bf16_bits(_normal_bits(rng, (wl.n, wl.H_s, wl.d if d_vs is None else int(d_vs)), std))


def select_sequences(wl: PrefillWorkload, idx) -> PrefillWorkload:
    """The packed workload of sequences `idx` of `wl` (in that order): slices, no arithmetic."""
    idx = [int(s) for s in idx]
    parts = [slice(int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])) for s in idx]
    lens = [wl.seqlens[s] for s in idx]
    cu = np.zeros(len(idx) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens) if lens else []
    cat = (lambda a: np.concatenate([a[p] for p in parts]) if parts else a[:0])
    return dataclasses.replace(wl, seqlens=lens, q=cat(wl.q), k=cat(wl.k), v=cat(wl.v),
                               cu_seqlens=cu)
