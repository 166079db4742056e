"""Pins of the prefix-hash block index oracle (CPU only).

The oracle is checked against things other than itself: the published FNV-1a-64 test vectors,
byte serialisation by numpy instead of the oracle's own int-to-bytes path, and brute-force
comparison of token prefixes that uses no hashing at all.
"""

import json
import os

import numpy as np

from oracle import prefix_index as px
from synth import make_prefix_requests, prefix_config

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fnv1a64.json")


def test_fnv1a64_published_vectors():
    with open(GOLDEN) as f:
        g = json.load(f)
    assert g["citation"]
    for v in g["vectors"]:
        assert px.fnv1a64(v["ascii"].encode("ascii")) == int(v["fnv1a64"], 16), v


def _brute_digest(tokens):
    # numpy serialises the token ids; the oracle serialises them itself
    return px.fnv1a64(np.asarray(tokens, dtype="<i4").tobytes())


def test_keys_are_fnv_of_concatenated_digests():
    """With salt = the offset basis, the key of block b is one FNV-1a-64 call over the
    little-endian digests of blocks 0..b (serialised by numpy): the chain continues the state
    across blocks in order, little-endian, with nothing else absorbed."""
    rng = np.random.default_rng(3)
    B = 8
    lens = [37, 8, 0, 5, 64]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    toks = rng.integers(-5, 1 << 20, size=int(cu[-1])).astype(np.int32)
    keys, key_cu = px.prefix_keys(toks, cu, B)
    assert list(np.diff(key_cu)) == [L // B for L in lens]
    for s, L in enumerate(lens):
        base = int(cu[s])
        digs = [_brute_digest(toks[base + j * B: base + (j + 1) * B]) for j in range(L // B)]
        for b in range(L // B):
            blob = np.array(digs[:b + 1], dtype="<u8").tobytes()
            assert int(keys[key_cu[s] + b]) == px.fnv1a64(blob)


def test_salt_continues_the_state():
    toks = np.arange(64 * 3, dtype=np.int32)
    cu = np.array([0, 64 * 3], dtype=np.int32)
    salt = 0x0123456789ABCDEF
    keys, _ = px.prefix_keys(toks, cu, 64, salt)
    digs = [_brute_digest(toks[j * 64:(j + 1) * 64]) for j in range(3)]
    h = salt
    for b, c in enumerate(digs):
        for octet in np.array([c], dtype="<u8").tobytes():
            h = ((h ^ octet) * 0x100000001B3) % (1 << 64)
        assert int(keys[b]) == h
    other, _ = px.prefix_keys(toks, cu, 64, salt ^ 1)
    assert not set(map(int, keys)) & set(map(int, other))


def test_key_depends_on_whole_prefix_only():
    """Changing one token of block j changes the keys of blocks j, j+1, ... and no earlier one;
    tokens of a partial last block change nothing."""
    rng = np.random.default_rng(4)
    B, L = 16, 16 * 6 + 5
    toks = rng.integers(0, 1000, size=L).astype(np.int32)
    cu = np.array([0, L], dtype=np.int32)
    k0, _ = px.prefix_keys(toks, cu, B)
    for j in range(6):
        t = toks.copy()
        t[j * B + int(rng.integers(0, B))] += 1
        k1, _ = px.prefix_keys(t, cu, B)
        assert np.array_equal(k0[:j], k1[:j])
        assert np.all(k0[j:] != k1[j:])
    t = toks.copy()
    t[-1] += 7
    assert np.array_equal(px.prefix_keys(t, cu, B)[0], k0)


def _lcp(a, b):
    n = min(len(a), len(b))
    i = 0
    while i < n and a[i] == b[i]:
        i += 1
    return i


def _brute_found(w):
    """Per prompt block: does some cached sequence hold the same first (b + 1) * B tokens? By
    direct token comparison."""
    cached = [w.cached_tokens[w.cached_cu[i]:w.cached_cu[i + 1]]
              for i in range(len(w.cached_cu) - 1)]
    found, hits = [], []
    for s in range(len(w.query_cu) - 1):
        q = w.query_tokens[w.query_cu[s]:w.query_cu[s + 1]]
        lcp = max([_lcp(q, c) for c in cached] + [0])
        blk = [(b + 1) * w.B <= lcp for b in range(len(q) // w.B)]
        found += blk
        hits.append(lcp // w.B)
    return np.array(found, dtype=bool), np.array(hits, dtype=np.int32)


def _index_found(w):
    ck, _ = px.prefix_keys(w.cached_tokens, w.cached_cu, w.B, w.salt)
    idx = px.PrefixIndex()
    idx.insert(ck, np.arange(len(ck), dtype=np.int64))
    qk, q_cu = px.prefix_keys(w.query_tokens, w.query_cu, w.B, w.salt)
    found = idx.lookup(qk)
    return found, px.prefix_hits(found, q_cu), q_cu


def test_found_blocks_equal_brute_force_small():
    w = make_prefix_requests([40, 64, 130, 7, 0, 96], [64, 129, 5, 0, 200, 96, 64, 33, 130, 70],
                             B=16, vocab=50, seed=11, p_fresh=0.1)
    # one more prompt: cached sequence 2 with a token of block 1 changed; its later blocks equal
    # the cached ones, but their prefixes do not, so they must not be found
    c2 = w.cached_tokens[w.cached_cu[2]:w.cached_cu[3]].copy()
    c2[20] = (c2[20] + 1) % 50
    w.query_tokens = np.concatenate([w.query_tokens, c2])
    w.query_cu = np.concatenate([w.query_cu, [w.query_cu[-1] + len(c2)]]).astype(np.int32)
    found, hits, _ = _index_found(w)
    bf, bh = _brute_found(w)
    assert np.array_equal(found >= 0, bf)
    assert np.array_equal(hits, bh)
    assert hits.max() > 0 and hits[-1] == 1


def test_found_blocks_equal_brute_force_full_size():
    w = prefix_config()
    found, hits, q_cu = _index_found(w)
    bf, bh = _brute_found(w)
    assert np.array_equal(found >= 0, bf)
    assert np.array_equal(hits, bh)
    # each prompt that copied m tokens from a cached sequence hits at least m // B blocks
    for s, (c, m) in enumerate(w.shared):
        assert hits[s] >= (m // w.B if c >= 0 else 0)
    # found locations point at cached blocks with the same position and token prefix
    cblk = [(c, j) for c in range(len(w.cached_cu) - 1)
            for j in range((w.cached_cu[c + 1] - w.cached_cu[c]) // w.B)]
    for s in range(len(q_cu) - 1):
        for b in range(int(hits[s])):
            c, j = cblk[int(found[q_cu[s] + b])]
            assert j == b
            a0, c0 = int(w.query_cu[s]), int(w.cached_cu[c])
            n = (b + 1) * w.B
            assert np.array_equal(w.query_tokens[a0:a0 + n], w.cached_tokens[c0:c0 + n])


def test_insert_keeps_first_location_and_skips_empty_key():
    idx = px.PrefixIndex()
    keys = np.array([5, 9, 5, px.EMPTY_KEY, 9, 7], dtype=np.uint64)
    stored = idx.insert(keys, np.array([10, 20, 30, 40, 50, 60]))
    assert list(stored) == [10, 20, 10, px.MISSING, 20, 60]
    assert list(idx.insert(np.array([7, 8], dtype=np.uint64), np.array([1, 2]))) == [60, 2]
    assert list(idx.lookup(np.array([5, 6, px.EMPTY_KEY], dtype=np.uint64))) == [10, -1, -1]
