"""CPU checks of bench.py's command-line contract: the reference arm (the float64 oracle on the
host) prints one JSON line with the contract's keys; under torchrun only rank 0 prints it; fewer
than 3 warm-up steps are refused."""

import json

import numpy as np
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args,
                          capture_output=True, text=True, timeout=timeout, env=env, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _run(["--impl", "reference", "--config", "prefixindex", "--steps", "2", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]


def test_reference_arm_prints_nothing_on_other_ranks():
    r = _run(["--impl", "reference", "--config", "prefixindex", "--steps", "1", "--warmup", "3"],
             {"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_fewer_than_three_warmup_steps_are_refused():
    r = _run(["--impl", "reference", "--config", "prefixindex", "--steps", "1", "--warmup", "2"])
    assert r.returncode == 2
    assert "warmup" in r.stderr


def test_reference_arm_decode_line():
    r = _run(["--impl", "reference", "--config", "decode", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["unit"] == "rows/s" and d["value"] > 0
    assert d["cpu_baseline"]["cores"] >= 1


def test_oracle_timing_helpers_on_small_workloads():
    sys.path.insert(0, ROOT)
    import bench
    from synth import make_decode, make_head_match
    hm = make_head_match(n=64, L_s=2, H_small=3, d_small=16, L_l=2, H_large=4, d_large=32,
                         seed=1)
    full, t_full = bench.oracle_headmatch_sample(hm)
    half, t_half = bench.oracle_headmatch_sample(hm, 1)
    assert full > 0 and half > 0 and t_full > 0 and t_half > 0
    dw = make_decode(batch=2, ctx=100, H_s=3, H_r=4, d_v=16, seed=1)
    rows, dt = bench.oracle_decode_step(dw)
    assert abs(rows * dt - 2) < 1e-9


def test_reference_arm_prefill_times_what_it_reports():
    """The prefill reference arm times one row block of a fixed, stated sample per step, and its
    ms_per_step is that measured time (so steps x ms_per_step fits inside the run)."""
    import time
    t0 = time.time()
    r = _run(["--impl", "reference", "--config", "tiny", "--steps", "3", "--warmup", "3"])
    wall = time.time() - t0
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    assert d["steps"] * d["ms_per_step"] / 1e3 <= wall
    assert "fixed sample" in d["cpu_baseline"]["sample"]
    assert d["ms_per_workload_extrapolated"] > 0


def test_kept_set_check_counts_a_planted_mismatch():
    sys.path.insert(0, ROOT)
    import bench
    import oracle as O
    from synth import make_prefill
    wl = make_prefill([300, 200], H_s=3, d=32, H_r=2, d_v=8, B=64, tau=0.9, seed=79)
    blocks = bench.systematic_rowblocks(wl, 3)
    assert len(blocks) == 3 and len(set(blocks)) == 3
    _, rows, _, stats, text = bench.oracle_sample_prefill(wl, blocks)
    kept = O.compress(wl).kept
    chk = bench.kept_set_check(wl, kept, stats)
    assert chk["mismatches_outside_near"] == 0 and chk["flips"] == 0
    assert chk["blocks"] == 3 * sum(I + 1 for _, I in blocks)
    s, I = blocks[1]
    lay = O.causal_layout(wl.seqlens, wl.B)
    J = int(np.flatnonzero(stats[1][2][0].kept)[0])
    bad = kept.copy()
    bad[0, lay.cb(s, I, J)] = False
    assert bench.kept_set_check(wl, bad, stats)["mismatches_outside_near"] == 1
