"""The multi-process host paths on CPU: world_size 2 over gloo (no GPU).

- bench.py's barrier and max-over-ranks timing;
- head matching split by large layers across ranks, reassembled with one all_gather; each
  rank's shard is computed here by the float64 oracle (the GPU entry point is the same call on
  the shard's slice of the large model's q, k).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _bench_helpers(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    _init(rank, world, port)
    try:
        bench.barrier(world)
        out[rank] = bench.max_over_ranks(1.5 + rank, world)
    finally:
        dist.destroy_process_group()


def _sharded_head_match(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import dataclasses
    import oracle as O
    from synth import make_head_match
    from cross_model_attention_map_b200.runner import gather_head_mapping, shard_range
    _init(rank, world, port)
    try:
        hm = make_head_match(n=40, L_s=2, H_small=3, d_small=8, L_l=3, H_large=4, d_large=16,
                             noise=0.3, seed=51)
        lo, hi = shard_range(hm.L_l, world, rank)
        local = dataclasses.replace(hm, L_l=hi - lo, q_large=hm.q_large[lo:hi],
                                    k_large=hm.k_large[lo:hi])
        _, arg = O.head_match(local) if hi > lo else (None, np.zeros((0, 4), np.int32))
        full = gather_head_mapping(torch.from_numpy(np.ascontiguousarray(arg, dtype=np.int32)),
                                   hm.L_l, hm.H_large)
        out[rank] = full.numpy().tolist()
    finally:
        dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(fn, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        return dict(out)


def test_shard_range_covers_every_item_once():
    from cross_model_attention_map_b200.runner import shard_range
    for total in (0, 1, 7, 8, 9):
        for world in (1, 2, 3, 8):
            got = [i for r in range(world) for i in range(*shard_range(total, world, r))]
            assert got == list(range(total))


def test_bench_max_over_ranks_gloo():
    out = _run(_bench_helpers)
    assert out == {0: 2.5, 1: 2.5}


def test_sharded_head_match_equals_single_process():
    import oracle as O
    from synth import make_head_match
    out = _run(_sharded_head_match)
    hm = make_head_match(n=40, L_s=2, H_small=3, d_small=8, L_l=3, H_large=4, d_large=16,
                         noise=0.3, seed=51)
    _, ref = O.head_match(hm)
    for rank in (0, 1):
        np.testing.assert_array_equal(np.array(out[rank]), ref)


def _brute_makespan(work, world):
    best = None
    for assign in np.ndindex(*([world] * len(work))):
        loads = [0] * world
        for w, r in zip(work, assign):
            loads[r] += w
        best = max(loads) if best is None else min(best, max(loads))
    return best


def test_shard_sequences_balances_causal_work():
    """Every sequence goes to exactly one rank, and the most loaded rank is within the
    longest-first bound of the optimum found by brute force."""
    from cross_model_attention_map_b200.runner import causal_blocks, shard_sequences
    rng = np.random.default_rng(3)
    for trial in range(40):
        lens = [int(x) for x in rng.integers(0, 700, size=int(rng.integers(1, 8)))]
        for world in (1, 2, 3):
            parts = shard_sequences(lens, world, B=64)
            assert sorted(s for p in parts for s in p) == list(range(len(lens)))
            work = [causal_blocks(L, 64) for L in lens]
            got = max(sum(work[s] for s in p) for p in parts)
            opt = _brute_makespan(work, world)
            assert got * 3 * world <= opt * (4 * world - 1)
    # the varlen packing (4096/8192/12288/16384) on 2 ranks: 16384 alone against the rest
    assert shard_sequences([4096, 8192, 12288, 16384], 2) == [[3], [0, 1, 2]]


def test_prefill_split_by_sequence_equals_whole_batch():
    """Each rank's share of the packed sequences, run on its own, gives exactly the rows of the
    whole batch (the oracle stands in for each rank's GPU step; there is no exchange)."""
    import oracle as O
    from synth import make_prefill, select_sequences
    from cross_model_attention_map_b200.runner import shard_sequences
    wl = make_prefill([90, 30, 150, 64, 7], H_s=2, d=16, H_r=3, d_v=8, B=16, tau=0.8, seed=12)
    res = O.compress(wl)
    whole = O.mapped_av(wl, res.kept)
    for world in (2, 3):
        for part in shard_sequences(wl.seqlens, world, B=16):
            if not part:
                continue
            sub = select_sequences(wl, part)
            r = O.compress(sub)
            o = O.mapped_av(sub, r.kept)
            for i, s in enumerate(part):
                a, b = int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])
                c = int(sub.cu_seqlens[i])
                np.testing.assert_array_equal(o[c:c + b - a], whole[a:b])
                np.testing.assert_array_equal(r.lse[:, c:c + b - a], res.lse[:, a:b])


def _bench_sequence_split(rank, world, port, out):
    """The host side of `bench.py --split seq`: each rank takes its sequences of one packed batch
    (a rank without any follows the same barriers and max reductions with zero time), and the
    step time is the max over ranks."""
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from synth import make_prefill
    _init(rank, world, port)
    try:
        wl = make_prefill([300, 64, 700, 5], H_s=2, d=16, H_r=2, d_v=8, B=64, tau=0.9, seed=77)
        sub, mine = bench.split_by_sequence(wl, world, rank)
        rows = {s: sub.q[int(sub.cu_seqlens[i]):int(sub.cu_seqlens[i + 1])].tobytes()
                for i, s in enumerate(mine)}
        bench.barrier(world)
        bench.barrier(world)
        ms = bench.max_over_ranks(10.0 * (rank + 1), world)
        bench.barrier(world)
        e2e = bench.max_over_ranks(1.0 + rank, world)
        out[rank] = (mine, sub.n, {s: r for s, r in rows.items()}, ms, e2e)
    finally:
        dist.destroy_process_group()


def test_bench_sequence_split_world2():
    import sys
    sys.path.insert(0, ROOT)
    from synth import make_prefill
    out = _run(_bench_sequence_split)
    wl = make_prefill([300, 64, 700, 5], H_s=2, d=16, H_r=2, d_v=8, B=64, tau=0.9, seed=77)
    mine0, n0, rows0, ms0, e0 = out[0]
    mine1, n1, rows1, ms1, e1 = out[1]
    # every sequence on exactly one rank; the longest (700 tokens, 66 causal blocks) alone on
    # rank 0, the rest (15 + 1 + 1 blocks) on rank 1
    assert sorted(mine0 + mine1) == [0, 1, 2, 3]
    assert mine0 == [2] and mine1 == [0, 1, 3]
    assert n0 + n1 == wl.n
    # each rank's rows are the packed batch's rows of its sequences (slices, bit for bit)
    for rows in (rows0, rows1):
        for s, r in rows.items():
            a, b = int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])
            assert r == wl.q[a:b].tobytes()
    assert ms0 == ms1 == 20.0 and e0 == e1 == 2.0


def _bench_idle_rank(rank, world, port, out):
    """A rank with no sequence (4 ranks, 2 sequences) takes the working ranks' collectives."""
    import sys
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    from synth import make_prefill
    _init(rank, world, port)
    try:
        wl = make_prefill([200, 70], H_s=2, d=16, H_r=2, d_v=8, B=64, tau=0.9, seed=78)
        sub, mine = bench.split_by_sequence(wl, world, rank)
        if not mine:
            r = bench.idle_rank(argparse.Namespace(), world, wl.n)
            out[rank] = ("idle", r["ms"], r["e2e_ms"])
        else:
            bench.barrier(world)
            bench.barrier(world)
            ms = bench.max_over_ranks(3.0 + rank, world)
            bench.barrier(world)
            e2e = bench.max_over_ranks(4.0 + rank, world)
            out[rank] = (mine, ms, e2e)
    finally:
        dist.destroy_process_group()


def test_bench_sequence_split_idle_ranks():
    out = _run(_bench_idle_rank, world=4)
    assert out[0][0] == [0] and out[1][0] == [1]
    assert out[2][0] == "idle" and out[3][0] == "idle"
    for r in range(4):
        assert out[r][-2] == 4.0 and out[r][-1] == 5.0
