"""GPU parity of the prefix-hash block index against the CPU oracle (through the C ABI).

Keys, found locations and longest cached prefixes are integers and are compared bit for bit.
Where several results are correct -- the location kept for a key inserted twice in one call --
the test checks that the kept one is one of the candidates and that every reader agrees on it.
"""

import numpy as np
import pytest
import torch

from oracle import prefix_index as px
from synth import make_prefix_requests, prefix_config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from cross_model_attention_map_b200 import iamap, runner
    return iamap, runner


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def keys_np(t):
    return t.cpu().numpy().view(np.uint64)


def gpu_keys(runner, idx, tokens, cu):
    keys, key_cu = idx.keys(dev_i32(tokens), dev_i32(cu), np.asarray(cu, dtype=np.int32))
    return keys, key_cu


def status(C):
    torch.cuda.synchronize()
    return C.iamap_device_status()


def test_keys_parity_ragged_small_blocks(lib):
    """B = 16 over sequences with ragged tails, shorter than a block, and empty; negative and
    large token ids (every byte of the little-endian encoding matters)."""
    C, runner = lib
    rng = np.random.default_rng(21)
    lens = [37, 16, 0, 5, 64, 1000, 15, 17]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    toks = rng.integers(-2**31, 2**31 - 1, size=int(cu[-1]), dtype=np.int64).astype(np.int32)
    for salt in (px.FNV64_OFFSET, 0x0123456789ABCDEF, 2**64 - 2):
        idx = runner.PrefixIndex(64, B=16, salt=salt)
        keys, key_cu = gpu_keys(runner, idx, toks, cu)
        ref, ref_cu = px.prefix_keys(toks, cu, 16, salt)
        assert np.array_equal(key_cu.cpu().numpy(), ref_cu)
        assert np.array_equal(keys_np(keys), ref)
    assert status(C) == 0


def test_keys_parity_prompts_longer_than_one_chunk(lib):
    """Prompts of 312 and 257 blocks: the keys kernel digests 256 blocks per pass and carries the
    chain state from one pass to the next."""
    C, runner = lib
    rng = np.random.default_rng(2)
    lens = [5000, 17, 0, 4113, 300]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    toks = rng.integers(-2**31, 2**31 - 1, size=int(cu[-1]), dtype=np.int64).astype(np.int32)
    salt = 0x1234567890ABCDEF
    idx = runner.PrefixIndex(64, B=16, salt=salt)
    keys, key_cu = gpu_keys(runner, idx, toks, cu)
    ref, ref_cu = px.prefix_keys(toks, cu, 16, salt)
    assert list(np.diff(ref_cu)) == [312, 1, 0, 257, 18]
    assert np.array_equal(key_cu.cpu().numpy(), ref_cu)
    assert np.array_equal(keys_np(keys), ref)
    assert status(C) == 0


def test_keys_parity_full_size_prompts(lib):
    """The varlen prompt set (4 cached prompts of 4096..16384 tokens, 16 prompts looked up),
    B = 64: every key bit-exact."""
    C, runner = lib
    w = prefix_config()
    idx = runner.PrefixIndex(1 << 12, B=w.B, salt=w.salt)
    for toks, cu in ((w.cached_tokens, w.cached_cu), (w.query_tokens, w.query_cu)):
        keys, key_cu = gpu_keys(runner, idx, toks, cu)
        ref, ref_cu = px.prefix_keys(toks, cu, w.B, w.salt)
        assert np.array_equal(key_cu.cpu().numpy(), ref_cu)
        assert np.array_equal(keys_np(keys), ref)
    assert status(C) == 0


def _check_insert(stored, keys, values, ref_table, prior):
    """stored[i] is the location now kept for keys[i]: the earlier one if the key was present,
    else one of this call's locations for that key, the same for every duplicate."""
    chosen = {}
    for k, v, st in zip(keys.tolist(), values.tolist(), stored.tolist()):
        if k == px.EMPTY_KEY:
            assert st == px.MISSING
            continue
        if k in prior:
            assert st == prior[k]
        else:
            cands = [vv for kk, vv in zip(keys.tolist(), values.tolist()) if kk == k]
            assert st in cands
        assert chosen.setdefault(k, st) == st
    return chosen


def test_insert_lookup_longest_prefix_parity(lib):
    """Insert the cached prompts' keys (repeated prefix blocks give duplicate keys in one call),
    then look up the 16 prompts: found locations and longest cached prefixes match the oracle."""
    C, runner = lib
    w = prefix_config()
    idx = runner.PrefixIndex(1 << 12, B=w.B, salt=w.salt)
    ckeys, _ = gpu_keys(runner, idx, w.cached_tokens, w.cached_cu)
    ck = keys_np(ckeys)
    vals = np.arange(len(ck), dtype=np.int64) * 7 + 3
    stored = idx.insert(ckeys, torch.from_numpy(vals).cuda()).cpu().numpy()
    kept = _check_insert(stored, ck, vals, None, {})
    assert len(kept) == len(set(ck.tolist()))
    assert len(kept) < len(ck)          # the workload does repeat prefix blocks

    qkeys, q_cu = gpu_keys(runner, idx, w.query_tokens, w.query_cu)
    found, hits = idx.lookup(qkeys, q_cu)
    qk = keys_np(qkeys)
    ref_found = np.array([kept.get(k, px.MISSING) for k in qk.tolist()], dtype=np.int64)
    assert np.array_equal(found.cpu().numpy(), ref_found)
    # longest cached prefix: unique whatever location a duplicate kept
    o = px.PrefixIndex()
    o.insert(ck, vals)
    ref_hits = px.prefix_hits(o.lookup(qk), q_cu.cpu().numpy())
    assert np.array_equal(hits.cpu().numpy(), ref_hits)
    assert ref_hits.sum() > 0 and (ref_hits == 0).any()

    # a second insert of the same keys keeps every earlier location
    again = idx.insert(ckeys, torch.from_numpy(vals + 1).cuda()).cpu().numpy()
    _check_insert(again, ck, vals + 1, None, kept)
    # flat lookup (no sequences) over more than one 4096-key segment
    many = np.concatenate([qk, ck, qk ^ np.uint64(1)] * 40)
    assert len(many) > 3 * 4096
    t = torch.from_numpy(many.view(np.int64)).cuda()
    f2, h2 = idx.lookup(t)
    assert h2 is None
    assert np.array_equal(f2.cpu().numpy(),
                          np.array([kept.get(k, -1) for k in many.tolist()], dtype=np.int64))
    assert status(C) == 0


def test_small_random_prompt_sets_parity(lib):
    """Several seeded prompt sets with B = 16 and a small vocabulary, end to end."""
    C, runner = lib
    for seed in range(6):
        w = make_prefix_requests([40, 64, 130, 7, 0, 96], [64, 129, 5, 0, 200, 96, 64, 33, 130],
                                 B=16, vocab=50, seed=seed, p_fresh=0.1)
        idx = runner.PrefixIndex(256, B=16, salt=w.salt)
        ckeys, _ = gpu_keys(runner, idx, w.cached_tokens, w.cached_cu)
        ck = keys_np(ckeys)
        vals = np.arange(len(ck), dtype=np.int64)
        idx.insert(ckeys, torch.from_numpy(vals).cuda())
        qkeys, q_cu = gpu_keys(runner, idx, w.query_tokens, w.query_cu)
        found, hits = idx.lookup(qkeys, q_cu)
        o = px.PrefixIndex()
        o.insert(ck, vals)
        ref_found = o.lookup(keys_np(qkeys))
        assert np.array_equal(found.cpu().numpy() >= 0, ref_found >= 0)
        assert np.array_equal(hits.cpu().numpy(), px.prefix_hits(ref_found, q_cu.cpu().numpy()))
    assert status(C) == 0


def test_full_table_and_reserved_key(lib):
    """A table of 16 slots takes exactly 16 of 40 distinct keys; the others report -1 and raise
    the capacity bit; the reserved all-ones key is never stored and raises nothing."""
    C, runner = lib
    status(C)
    idx = runner.PrefixIndex(16, B=64)
    rng = np.random.default_rng(5)
    k = np.unique(rng.integers(0, 2**63 - 1, size=40, dtype=np.int64))
    assert len(k) == 40
    stored = idx.insert(torch.from_numpy(k).cuda(), torch.from_numpy(k % 1000).cuda())
    st = stored.cpu().numpy()
    ok = st >= 0
    assert ok.sum() == 16
    assert np.array_equal(st[ok], (k % 1000)[ok])
    assert status(C) & C.IAMAP_DEV_CAPACITY
    found, _ = idx.lookup(torch.from_numpy(k).cuda())
    assert np.array_equal(found.cpu().numpy(), np.where(ok, k % 1000, -1))

    idx.clear()
    empty = torch.tensor([-1, 5], dtype=torch.int64, device="cuda")   # all-ones bits, then 5
    st = idx.insert(empty, torch.tensor([9, 10], dtype=torch.int64, device="cuda")).cpu()
    assert st.tolist() == [-1, 10]
    assert status(C) == 0
    found, _ = idx.lookup(empty)
    assert found.cpu().tolist() == [-1, 10]


def test_bad_offsets_and_short_key_buffer_are_flagged(lib):
    """Device offsets outside the tokens give the sequence no keys and raise the bad-index bit;
    a key buffer shorter than the keys is not overrun and raises the capacity bit; lookup
    offsets outside the keys report 0 cached blocks and raise the bad-index bit."""
    C, runner = lib
    status(C)
    toks = dev_i32(np.arange(256))
    key_cu = torch.empty(3, dtype=torch.int64, device="cuda")
    keys = torch.full((8,), 7, dtype=torch.int64, device="cuda")
    C.iamap_prefix_keys(toks, 256, dev_i32([0, 128, 999]), 2, 64, px.FNV64_OFFSET, keys, 8,
                        key_cu)
    assert key_cu.cpu().tolist() == [0, 2, 2]
    assert status(C) & C.IAMAP_DEV_BAD_INDEX
    ref, _ = px.prefix_keys(np.arange(256, dtype=np.int32), [0, 128], 64)
    assert np.array_equal(keys_np(keys)[:2], ref)

    guard = torch.full((4,), 7, dtype=torch.int64, device="cuda")
    C.iamap_prefix_keys(toks, 256, dev_i32([0, 256]), 1, 64, px.FNV64_OFFSET, guard, 2, key_cu)
    assert status(C) & C.IAMAP_DEV_CAPACITY
    assert guard.cpu().tolist()[2:] == [7, 7]

    idx = runner.PrefixIndex(16, B=64)
    hits = torch.full((2,), 9, dtype=torch.int32, device="cuda")
    found = torch.empty(2, dtype=torch.int64, device="cuda")
    bad_cu = torch.tensor([0, 5, 1], dtype=torch.int64, device="cuda")
    C.iamap_prefix_lookup(keys, 2, bad_cu, 2, idx.table_keys, idx.table_vals, 16, found, hits)
    assert hits.cpu().tolist() == [0, 0]
    assert status(C) & C.IAMAP_DEV_BAD_INDEX
    assert status(C) == 0
