"""CPU checks of bench.py's command-line contract: the reference arm (the float64 oracle on the
host) prints one JSON line with the contract's keys; under torchrun only rank 0 prints it; fewer
than 3 warm-up steps are refused."""

import json
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
