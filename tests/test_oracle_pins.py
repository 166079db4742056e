"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against an independent definition or a property the mathematics
fixes: torch's scaled-dot-product attention (a library routine, in float64), closed forms in exact
rational arithmetic, a hand-derived golden fixture, brute-force enumeration of block subsets,
scikit-learn's cosine similarity, and a planted ground truth. A dropped term, a wrong sign or
index, or a transposed operand anywhere in the oracle fails at least one of them.
"""

import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
from synth import (bf16_bits, bf16_bits_to_f64, make_decode, make_head_match, make_prefill)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa_head(q, k, v, bias_window=0, bias_value=0.0):
    """torch float64 SDPA for one sequence and one head with a causal (+ local bias) mask."""
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


def _frac(sx):
    return Fraction(sx)


# ----------------------------------------------------------------------------------------------
# Golden fixture (hand-derived, exact)
# ----------------------------------------------------------------------------------------------

def test_golden_uniform_rows():
    fx = json.load(open(os.path.join(GOLDEN, "uniform_rows.json")))
    for case in fx["cases"]:
        n = sum(case["seqlens"])
        for tau_s, kept_exp in case["kept"].items():
            tau = float(tau_s)
            wl = make_prefill(case["seqlens"], H_s=1, d=8, H_r=1, d_v=1, B=case["B"], tau=tau,
                              sink=False, q_zero=True, seed=3)
            wl.v = bf16_bits(np.array(case["v"], dtype=np.float32).reshape(n, 1, 1))
            wl.W = np.ones((1, 1), dtype=np.float32)
            res = O.compress(wl)
            lay = res.layout
            for I in range(lay.nb[0]):
                key = "I%d" % I
                for J, mx in enumerate(case["masses"][key]):
                    assert abs(res.mass[0, lay.cb(0, I, J)] - float(_frac(mx))) < 1e-12
                got = [J for J in range(I + 1) if res.kept[0, lay.cb(0, I, J)]]
                assert got == kept_exp[key], (case["name"], tau, I)
            for i in range(n):
                assert abs(res.lse[0, i] - math.log(i + 1)) < 1e-12
            out = O.mapped_av(wl, res.kept)[:, 0, 0]
            exp = [float(_frac(x)) for x in case["O"][tau_s]]
            np.testing.assert_allclose(out, exp, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Identity mixing, keep-all equals dense causal attention (torch SDPA)
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("seqlens,bias", [([96], 0), ([37, 64, 1, 70], 0), ([130], 20)])
def test_identity_W_tau1_equals_sdpa(seqlens, bias):
    wl = make_prefill(seqlens, H_s=3, d=16, H_r=3, d_v=8, B=16, tau=1.0, sink=True,
                      bias_window=bias, bias_value=2.0, seed=1)
    wl.W = np.eye(3, dtype=np.float32)
    res = O.compress(wl)
    assert res.kept.all()
    out = O.mapped_av(wl, res.kept)
    q, k, v = (bf16_bits_to_f64(x) for x in (wl.q, wl.k, wl.v))
    for s in range(len(seqlens)):
        a, b = wl.cu_seqlens[s], wl.cu_seqlens[s + 1]
        for h in range(3):
            ref = _sdpa_head(q[a:b, h], k[a:b, h], v[a:b, h], bias, 2.0)
            np.testing.assert_allclose(out[a:b, h], ref, rtol=1e-10, atol=1e-12)


def test_one_hot_W_tau1_equals_sdpa_of_mapped_head():
    """Receiver head r with W[r, :] = e_{m(r)} and tau = 1 is dense attention of sender head
    m(r) applied to the receiver's own V_r (H_r != H_s, W not symmetric)."""
    H_s, H_r = 2, 3
    wl = make_prefill([50, 77], H_s=H_s, d=16, H_r=H_r, d_v=8, B=16, tau=1.0, seed=2)
    m = [1, 0, 1]
    wl.W = np.zeros((H_r, H_s), dtype=np.float32)
    wl.W[np.arange(H_r), m] = 1.0
    res = O.compress(wl)
    out = O.mapped_av(wl, res.kept)
    q, k, v = (bf16_bits_to_f64(x) for x in (wl.q, wl.k, wl.v))
    for s in range(2):
        a, b = wl.cu_seqlens[s], wl.cu_seqlens[s + 1]
        for r in range(H_r):
            ref = _sdpa_head(q[a:b, m[r]], k[a:b, m[r]], v[a:b, r])
            np.testing.assert_allclose(out[a:b, r], ref, rtol=1e-10, atol=1e-12)


def test_linearity_in_W():
    wl = make_prefill([100], H_s=4, d=16, H_r=3, d_v=8, B=16, tau=0.8, seed=4)
    res = O.compress(wl)
    rng = np.random.default_rng(9)   # dyadic weights: W1 + W2 is exact in fp32
    W1 = (rng.integers(-16, 17, wl.W.shape) / 8.0).astype(np.float32)
    W2 = (rng.integers(-16, 17, wl.W.shape) / 8.0).astype(np.float32)
    wl.W = W1
    o1 = O.mapped_av(wl, res.kept)
    wl.W = W2
    o2 = O.mapped_av(wl, res.kept)
    wl.W = W1 + W2
    o12 = O.mapped_av(wl, res.kept)
    np.testing.assert_allclose(o12, o1 + o2, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Invariants of probabilities and of the cumulative-mass choice
# ----------------------------------------------------------------------------------------------

def test_rows_sum_to_one_and_masses_sum_to_rows():
    wl = make_prefill([200, 45], H_s=3, d=32, H_r=2, d_v=8, B=32, tau=0.9, bias_window=16,
                      bias_value=2.0, seed=5)
    lay = O.causal_layout(wl.seqlens, wl.B)
    for s in range(2):
        for h in range(3):
            for I in range(lay.nb[s]):
                st = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, s, h, I, wl.B, wl.tau,
                                      wl.bias_window, wl.bias_value)
                np.testing.assert_allclose(st.p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
                assert abs(st.masses.sum() - st.R) < 1e-12
                assert (st.p[:, st.row0 + st.R:] == 0).all()


@pytest.mark.parametrize("tau", [0.5, 0.9, 0.95, 0.999])
def test_selection_invariants(tau):
    wl = make_prefill([300], H_s=4, d=32, H_r=2, d_v=8, B=32, tau=tau, seed=6)
    lay = O.causal_layout(wl.seqlens, wl.B)
    for h in range(4):
        for I in range(lay.nb[0]):
            st = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, 0, h, I, wl.B, tau)
            mh = st.masses / st.R
            kept = st.kept
            assert mh[kept].sum() >= tau                       # reaches tau
            if kept.sum() > 1:                                   # minimal: drop the smallest kept
                assert mh[kept].sum() - mh[kept].min() < tau
            if (~kept).any():                                   # greedy: kept dominate dropped
                assert mh[kept].min() >= mh[~kept].max()


def test_brute_force_selection_small():
    """n = 8, B = 2: among all subsets of causal column blocks, the kept set has the smallest size
    reaching tau * R and the largest mass among subsets of that size."""
    for seed in range(6):
        wl = make_prefill([8], H_s=3, d=8, H_r=1, d_v=4, B=2, tau=0.0, std=1.5, seed=seed)
        for tau in (0.3, 0.6, 0.85, 0.97):
            for h in range(3):
                for I in range(4):
                    st = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, 0, h, I, 2, tau)
                    m = st.masses
                    best = None
                    for k in range(1, I + 2):
                        for S in itertools.combinations(range(I + 1), k):
                            tot = sum(m[list(S)])
                            if tot >= tau * st.R and (best is None or tot > best[1]):
                                best = (S, tot)
                        if best is not None:
                            break
                    got = tuple(np.flatnonzero(st.kept))
                    assert len(got) == len(best[0])
                    assert abs(m[list(got)].sum() - best[1]) < 1e-12


# ----------------------------------------------------------------------------------------------
# Near-threshold blocks on hand-built mass vectors (the tolerance of the kept-set comparison)
# ----------------------------------------------------------------------------------------------

# Each case: normalised masses, tau, the kept set and the near set worked out by hand. R = 64
# rows, so the masses passed are 64 times these.
_NEAR_CASES = [
    # clear margins everywhere: nothing is near (the last kept block, J=2, is not compared with
    # its own mass)
    ("clear", [0.5, 0.3, 0.15, 0.05], 0.9, {0, 1, 2}, set()),
    # the last kept block (J=2) and a dropped block (J=3) have equal masses: the order between
    # them may swap, both are near
    ("equal", [0.5, 0.3, 0.1, 0.1], 0.85, {0, 1, 2}, {2, 3}),
    # a dropped block 4e-6 below the last kept one: both near
    ("close", [0.5, 0.3, 0.1, 0.1 - 4e-6], 0.85, {0, 1, 2}, {2, 3}),
    # a dropped block 3e-5 below the last kept one: a clear margin
    ("apart", [0.5, 0.3, 0.1, 0.1 - 3e-5], 0.85, {0, 1, 2}, set()),
    # the cumulative mass before the last kept block (J=2) lands 5e-6 below tau: J=2 is near
    ("cum_before", [0.6, 0.3 - 5e-6, 0.08 + 5e-6, 0.02], 0.9, {0, 1, 2}, {2}),
    # the cumulative mass through the last kept block (J=1) lands 5e-6 above tau: the first
    # dropped block (J=2) is near
    ("cum_through", [0.6, 0.3 + 5e-6, 0.08, 0.02 - 5e-6], 0.9, {0, 1}, {2}),
    # ties in the order: equal masses sort by lower J, so J=1 is kept before J=3; the last kept
    # block is J=3 and no other block is close to its mass
    ("tie_order", [0.1, 0.3, 0.55, 0.3, 0.0], 0.9, {1, 2, 3}, set()),
]


@pytest.mark.parametrize("name,mh,tau,kept_exp,near_exp", _NEAR_CASES, ids=[c[0] for c in _NEAR_CASES])
def test_near_threshold_hand_built(name, mh, tau, kept_exp, near_exp):
    R = 64
    kept, near = O.select_blocks(np.array(mh) * R, R, tau)
    assert set(np.flatnonzero(kept)) == kept_exp
    assert set(np.flatnonzero(near)) == near_exp


def test_near_threshold_is_rare_on_the_tiny_workload():
    """With the rule above, near-threshold blocks are the exception: on the tiny configuration
    (8 heads x 36 causal blocks) no block is near, and in particular no last kept block is."""
    from synth import prefill_config
    wl = prefill_config("tiny")
    res = O.compress(wl)
    assert res.near.sum() <= 2, int(res.near.sum())


def test_dropping_the_last_kept_block_is_caught():
    """A planted selection mistake (the oracle's own kept sets with the last kept block of one
    row block removed) fails the kept-set comparison the GPU tests use."""
    from _gpu_common import compare_kept
    wl = make_prefill([300], H_s=3, d=32, H_r=2, d_v=8, B=32, tau=0.9, std=1.5, sink=True, seed=6)
    res = O.compress(wl)
    lay = res.layout
    assert compare_kept(res.kept, res.kept, res.near, report=False) == 0
    I = 7
    st = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, 0, 1, I, wl.B, wl.tau)
    mh = st.masses / st.R
    kept_J = np.flatnonzero(st.kept)
    last = kept_J[np.argmin(mh[kept_J] + 1e-12 * kept_J)]   # smallest kept mass (ties: higher J)
    assert not res.near[1, lay.cb(0, I, last)]
    bad = res.kept.copy()
    bad[1, lay.cb(0, I, last)] = False
    with pytest.raises(AssertionError):
        compare_kept(bad, res.kept, res.near, report=False)


# ----------------------------------------------------------------------------------------------
# Closed form: Q = 0 gives uniform rows p_ij = 1/(i+1)
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("L,I,J", [(100, 1, 1), (100, 1, 0), (64, 0, 0), (70, 1, 1)])
def test_masked_tile_partial_blocks_closed_form(L, I, J):
    """masked_tile on uniform rows (Q = 0): entry (r, c) of the tile of column block J in row
    block I is 1/(i+1) for the global row i = 64 I + r and column j = 64 J + c when i < L and
    j <= i, and 0 otherwise (exact rationals; partial last blocks of a sequence of L tokens)."""
    B = 64
    wl = make_prefill([L], H_s=1, d=16, H_r=1, d_v=4, B=B, tau=1.0, q_zero=True, seed=3)
    st = O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, 0, 0, I, B, 1.0)
    t = O.masked_tile(st, J, B)
    assert t.shape == (B, B)
    for r in range(B):
        i = I * B + r
        for c in range(B):
            j = J * B + c
            exp = Fraction(1, i + 1) if (i < L and j <= i) else Fraction(0)
            assert abs(t[r, c] - float(exp)) < 1e-15, (r, c)


# ----------------------------------------------------------------------------------------------
# Closed form: Q = 0 gives uniform rows p_ij = 1/(i+1)
# ----------------------------------------------------------------------------------------------

def _uniform_expected(L, B, tau):
    """Exact masses and kept sets for uniform rows, in rational arithmetic."""
    nb = (L + B - 1) // B
    out = []
    for I in range(nb):
        rows = range(I * B, min((I + 1) * B, L))
        R = len(rows)
        ms = []
        for J in range(I + 1):
            ms.append(sum(Fraction(len([j for j in range(J * B, (J + 1) * B) if j <= i]), i + 1)
                          for i in rows))
        assert sum(ms) == R
        order = sorted(range(I + 1), key=lambda J: (-ms[J], J))
        kept, cum = set(), Fraction(0)
        for J in order:
            if tau >= 1 or cum < Fraction(tau).limit_denominator(10 ** 9) * R:
                kept.add(J)
                cum += ms[J]
            else:
                break
            # guard against a boundary that float rounding could flip
            assert abs(float(cum / R) - tau) > 1e-9 or tau >= 1
        out.append((ms, kept, R))
    return out


@pytest.mark.parametrize("L,B,tau", [(200, 16, 0.9), (130, 32, 0.75), (64, 8, 1.0)])
def test_uniform_rows_closed_form(L, B, tau):
    H_s, H_r, c = 2, 3, 0.5
    wl = make_prefill([L], H_s=H_s, d=16, H_r=H_r, d_v=4, B=B, tau=tau, q_zero=True,
                      v_const=c, seed=7)
    res = O.compress(wl)
    lay = res.layout
    exp = _uniform_expected(L, B, tau)
    keptfrac = np.zeros(L)
    for I, (ms, kept, R) in enumerate(exp):
        for h in range(H_s):
            for J in range(I + 1):
                assert abs(res.mass[h, lay.cb(0, I, J)] - float(ms[J])) < 1e-11
                assert bool(res.kept[h, lay.cb(0, I, J)]) == (J in kept)
        for i in range(I * B, I * B + R):
            keptfrac[i] = sum(1 for j in range(i + 1) if j // B in kept) / (i + 1)
    out = O.mapped_av(wl, res.kept)
    cval = float(bf16_bits_to_f64(bf16_bits(np.array([c], dtype=np.float32)))[0])
    wsum = wl.W.astype(np.float64).sum(axis=1)
    expO = wsum[None, :, None] * keptfrac[:, None, None] * cval
    np.testing.assert_allclose(out, np.broadcast_to(expO, out.shape), rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------------------------
# Block-sparse storage
# ----------------------------------------------------------------------------------------------

def test_union_bsr_structure():
    wl = make_prefill([150, 64, 10], H_s=5, d=16, H_r=2, d_v=4, B=16, tau=0.7, seed=8)
    res = O.compress(wl)
    lay = res.layout
    row_ptr, col_idx, hm, val_off, tiles = O.union_bsr(res.kept, lay)
    assert tiles == int(res.kept.sum())
    assert row_ptr[-1] == len(col_idx)
    seen = np.zeros_like(res.kept)
    rb = 0
    for s in range(3):
        for I in range(lay.nb[s]):
            js = col_idx[row_ptr[rb]:row_ptr[rb + 1]]
            assert (np.diff(js) > 0).all()
            for u in range(row_ptr[rb], row_ptr[rb + 1]):
                c = lay.cb(s, I, int(col_idx[u]))
                for h in range(5):
                    bit = (int(hm[u]) >> h) & 1
                    assert bit == int(res.kept[h, c])
                    seen[h, c] |= bool(bit)
                if u + 1 < len(val_off):
                    assert val_off[u + 1] - val_off[u] == bin(int(hm[u])).count("1")
            rb += 1
    assert (seen == res.kept).all()


# ----------------------------------------------------------------------------------------------
# Decode on a mapped layer
# ----------------------------------------------------------------------------------------------

def test_paged_decode_equals_dense_attention_row():
    """Sender rows that are softmax(q K^T / sqrt(d)) of a real query: the paged, one-hot mapped
    output equals torch SDPA of that sender head applied to the receiver's V (gathered to a
    contiguous cache by the page table)."""
    rng = np.random.default_rng(11)
    dw = make_decode(batch=3, ctx=70, H_s=3, H_r=4, d_v=8, page_size=16, ctx_lens=[70, 33, 1],
                     seed=12)
    d = 16
    qs = rng.standard_normal((dw.batch, dw.H_s, d))
    ks = rng.standard_normal((dw.batch, 70, dw.H_s, d))
    for b in range(dw.batch):
        c = int(dw.ctx_lens[b])
        for s in range(dw.H_s):
            logit = ks[b, :c, s] @ qs[b, s] / math.sqrt(d)
            p = torch.softmax(torch.from_numpy(logit), dim=0).numpy()
            dw.p_rows[b, s, :] = 0
            dw.p_rows[b, s, :c] = p.astype(np.float32)
    out = O.mapped_av_paged(dw)
    for b in range(dw.batch):
        c = int(dw.ctx_lens[b])
        vcont = np.zeros((c, dw.H_r, dw.d_v))
        for j in range(c):
            vcont[j] = bf16_bits_to_f64(dw.v_pages[dw.page_table[b, j // 16], j % 16])
        for r in range(dw.H_r):
            s = int(dw.assign[r])
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(qs[b, s])[None, None, None, :],
                torch.from_numpy(np.ascontiguousarray(ks[b, :c, s]))[None, None],
                torch.from_numpy(np.ascontiguousarray(vcont[:, r]))[None, None])
            # the sender rows are stored as fp32, hence the 1e-6 relative slack
            np.testing.assert_allclose(out[b, r], ref[0, 0, 0].numpy(), rtol=2e-6, atol=2e-6)


def test_paged_decode_general_W_linear():
    dw = make_decode(batch=2, ctx=40, H_s=3, H_r=2, d_v=4, page_size=16, seed=13)
    W1 = dw.W.copy()
    o1 = O.mapped_av_paged(dw)
    dw.W = np.full_like(W1, 0.25)
    o2 = O.mapped_av_paged(dw)
    dw.W = W1 + 0.25
    np.testing.assert_allclose(O.mapped_av_paged(dw), o1 + o2, rtol=1e-10, atol=1e-12)


# ----------------------------------------------------------------------------------------------
# Head matching
# ----------------------------------------------------------------------------------------------

def test_attention_map_equals_torch_softmax():
    rng = np.random.default_rng(14)
    q = rng.standard_normal((40, 16))
    k = rng.standard_normal((40, 16))
    A = O.attention_map(q, k)
    s = torch.from_numpy(q @ k.T / 4.0)
    s = s.masked_fill(torch.triu(torch.ones(40, 40, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(A, torch.softmax(s, dim=1).numpy(), rtol=1e-12, atol=1e-15)


def test_head_match_cosine_equals_sklearn():
    from sklearn.metrics.pairwise import cosine_similarity
    hm = make_head_match(n=48, L_s=2, H_small=3, d_small=8, L_l=2, H_large=4, d_large=16,
                         noise=0.5, seed=15)
    C, arg = O.head_match(hm)
    small = [O.attention_map(bf16_bits_to_f64(hm.q_small[l, :, h]),
                             bf16_bits_to_f64(hm.k_small[l, :, h])).ravel()
             for l in range(2) for h in range(3)]
    large = [O.attention_map(bf16_bits_to_f64(hm.q_large[l, :, h]),
                             bf16_bits_to_f64(hm.k_large[l, :, h])).ravel()
             for l in range(2) for h in range(4)]
    ref = cosine_similarity(np.array(large), np.array(small))
    np.testing.assert_allclose(C, ref, rtol=1e-12, atol=1e-14)
    assert (C >= 0).all() and (C <= 1 + 1e-12).all()
    np.testing.assert_array_equal(arg.ravel(), np.argmax(ref, axis=1))
    # truncation to a prefix uses the prefix maps
    Ct, _ = O.head_match(hm, n_used=20)
    small_t = [x.reshape(48, 48)[:20, :20].ravel() for x in small]
    large_t = [x.reshape(48, 48)[:20, :20].ravel() for x in large]
    np.testing.assert_allclose(Ct, cosine_similarity(np.array(large_t), np.array(small_t)),
                               rtol=1e-12, atol=1e-14)


def _flat_maps(hm, q, k, layers, heads, n):
    return np.array([O.attention_map(bf16_bits_to_f64(q[l, :n, h]),
                                     bf16_bits_to_f64(k[l, :n, h])).ravel()
                     for l in range(layers) for h in range(heads)])


def test_head_match_pearson_equals_scipy():
    """Pearson metric = scipy.stats.pearsonr of the flattened n x n maps, pair by pair."""
    from scipy.stats import pearsonr
    hm = make_head_match(n=40, L_s=2, H_small=3, d_small=8, L_l=1, H_large=4, d_large=16,
                         noise=0.5, seed=17)
    S, arg = O.head_match(hm, metric="pearson")
    small = _flat_maps(hm, hm.q_small, hm.k_small, 2, 3, 40)
    large = _flat_maps(hm, hm.q_large, hm.k_large, 1, 4, 40)
    ref = np.array([[pearsonr(a, b)[0] for b in small] for a in large])
    np.testing.assert_allclose(S, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(arg.ravel(), np.argmax(ref, axis=1))
    # every causal softmax row sums to 1, so every map's mean is 1/n
    np.testing.assert_allclose(small.mean(axis=1), 1.0 / 40, rtol=1e-12)


def test_head_match_euclidean_equals_scipy_cdist():
    """Euclidean metric = minus scipy's Minkowski (p = 2) distance of the flattened maps, also
    on a truncated prefix."""
    from scipy.spatial.distance import cdist
    hm = make_head_match(n=36, L_s=1, H_small=5, d_small=8, L_l=2, H_large=3, d_large=8,
                         noise=0.4, seed=18)
    for n_used in (36, 17):
        S, arg = O.head_match(hm, n_used=n_used, metric="euclidean")
        small = _flat_maps(hm, hm.q_small, hm.k_small, 1, 5, n_used)
        large = _flat_maps(hm, hm.q_large, hm.k_large, 2, 3, n_used)
        ref = -cdist(large, small, metric="minkowski", p=2)
        np.testing.assert_allclose(S, ref, rtol=1e-10, atol=1e-13)
        np.testing.assert_array_equal(arg.ravel(), np.argmax(ref, axis=1))


def test_head_match_metrics_agree_on_exact_copies():
    """Noise-free copies with equal head dims: every metric picks the planted head (cosine and
    Pearson 1, distance 0)."""
    hm = make_head_match(n=32, L_s=2, H_small=3, d_small=8, L_l=1, H_large=5, d_large=8,
                         noise=0.0, seed=19)
    for metric, best in (("cosine", 1.0), ("pearson", 1.0), ("euclidean", 0.0)):
        S, arg = O.head_match(hm, metric=metric)
        np.testing.assert_array_equal(arg, hm.planted)
        for h in range(5):
            assert abs(S[h, hm.planted[0, h]] - best) < 1e-10


def test_mapping_consistency_counts_equal_entries():
    a = np.array([3, 1, 4, 1, 5, 9, 2, 6], dtype=np.int32)
    b = np.array([3, 1, 4, 0, 5, 8, 2, 6], dtype=np.int32)
    assert O.mapping_consistency(a, b) == 6 / 8
    assert O.mapping_consistency(a, a) == 1.0


def test_head_match_exact_copy_has_cosine_one():
    hm = make_head_match(n=32, L_s=2, H_small=3, d_small=8, L_l=1, H_large=5, d_large=8,
                         noise=0.0, seed=16)
    C, arg = O.head_match(hm)
    for h in range(5):
        assert abs(C[h, hm.planted[0, h]] - 1.0) < 1e-12
    np.testing.assert_array_equal(arg, hm.planted)


@pytest.mark.slow
def test_head_match_planted_full_size():
    """The calibration workload (n=1024, 24x14 small heads d=64, 8x64 large heads d=128, noisy
    zero-padded copies): the argmax recovers every planted mapping."""
    hm = make_head_match()
    C, arg = O.head_match(hm)
    np.testing.assert_array_equal(arg, hm.planted)
    top2 = np.sort(C, axis=1)[:, -2:]
    assert (top2[:, 1] - top2[:, 0]).min() > 0.05


def test_grouped_values_equal_repeated_heads():
    """Grouped receiver values (H_kv < H_r): the output equals that of a workload whose V holds
    every value head repeated H_r / H_kv times in consecutive receiver heads (prefill and decode)."""
    import dataclasses
    wl = make_prefill([150, 70], H_s=4, d=16, H_r=6, d_v=8, B=16, tau=0.9, seed=41, H_kv=2)
    lay = O.causal_layout(wl.seqlens, wl.B)
    kept = np.ones((wl.H_s, lay.num_causal_blocks), dtype=bool)
    rep = dataclasses.replace(wl, v=np.repeat(wl.v, 3, axis=1))
    assert rep.v.shape[1] == 6
    np.testing.assert_array_equal(O.mapped_av(wl, kept), O.mapped_av(rep, kept))
    dw = make_decode(batch=2, ctx=70, H_s=3, H_r=8, d_v=8, page_size=16, seed=42, H_kv=2)
    drep = dataclasses.replace(dw, v_pages=np.repeat(dw.v_pages, 4, axis=2))
    np.testing.assert_array_equal(O.mapped_av_paged(dw), O.mapped_av_paged(drep))
    with pytest.raises(ValueError):
        O.receiver_values(np.zeros((3, 4, 2)), 6)


def test_sender_decode_rows_equal_torch_softmax():
    """The small model's decode rows: torch's float64 softmax of the scaled dot products of the
    query with the keys, gathered here by plain indexing of the page pool (no page-table walk),
    rows of different context lengths, zeros past each length."""
    dw = make_decode(batch=3, ctx=70, H_s=2, H_r=4, d_v=8, page_size=16, ctx_lens=[70, 5, 33],
                     seed=13, d_s=16)
    P = O.sender_decode_rows(dw)
    assert P.shape == (3, 2, 70)
    q = torch.from_numpy(bf16_bits_to_f64(dw.q_s))
    K = torch.from_numpy(bf16_bits_to_f64(dw.k_pages_s))
    for b in range(3):
        c = int(dw.ctx_lens[b])
        keys = torch.stack([K[int(dw.page_table[b, j // 16]), j % 16] for j in range(c)])  # [c, H, d]
        logits = torch.einsum("hd,jhd->hj", q[b], keys) / 4.0
        np.testing.assert_allclose(P[b, :, :c], torch.softmax(logits, dim=1).numpy(),
                                   rtol=1e-12, atol=1e-15)
        assert (P[b, :, c:] == 0).all()
        np.testing.assert_allclose(P[b, :, :c].sum(axis=1), 1.0, rtol=0, atol=1e-12)
