"""Benchmark of cross-model attention-map reuse on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

A step is one pass of the hot path over one synthetic batch: map_compress (block statistics +
selection + union index, then extraction of the kept tiles) followed by mapped_av, on the
packed-prefill workload (default ``varlen40k``: 4 causal sequences of 4096/8192/12288/16384
tokens = 40960 tokens, sender 40 heads d=128, receiver 32 heads d_v=128, B=64, tau=0.9). Inputs
are resident in HBM when the timed region starts; Q+K (840 MB) and the block-sparse values
(~17 GB) exceed the 126 MB L2, so no flush is needed between steps.

Other configs (for measurement of the other kernels): ``tiny``, ``prefill8k``, ``headmatch``
(head_match, n=1024, 24x14 small / 8x64 large heads), ``decode`` (paged decode, batch 4,
context 8704), ``prefixindex`` (prefix-hash block index: publish and look up prompts).

Multi-GPU (torchrun): every rank runs its own full batch (independent problems, no data-path
collective, weak scaling); rank 0 prints value = tokens of all ranks / max time over ranks.

``--impl reference`` times the float64 CPU oracle (rank 0 only) on a bounded sample of the same
workload, in the same metric.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mapped-attention tokens/s at n=32k (1 B200); achieved % HBM / tensor roofline"
PROFILES = os.path.join(ROOT, "profiles")

CONFIG_TEXT = {
    "varlen40k": ("varlen40k: 4 packed causal sequences 4096/8192/12288/16384 (40960 tokens), "
                  "sender H_s=40 d=128, receiver H_r=32 d_v=128, B=64, tau=0.9, sink; "
                  "compress + mapped_av"),
    "varlen40k_sender": ("varlen40k_sender: the varlen40k workload with the sender's own "
                         "attention output (values d_vs=128) fused into compress; compress + "
                         "sender output + mapped_av"),
    "prefill8k": ("prefill8k: 1 causal sequence n=8192, H_s=32 d=128, H_r=24 d_v=128, B=64, "
                  "tau=0.95, sink, local bias +2.0 on |i-j|<128; compress + mapped_av"),
    "tiny": "tiny: n=512, H_s=8 d=64, H_r=4 d_v=64, B=64, tau=0.95, sink; compress + mapped_av",
    "headmatch": ("headmatch: n=1024, small 24 layers x 14 heads d=64, large 8 layers x 64 heads "
                  "d=128, planted noisy copies; head_match"),
    "headmatch8k": ("headmatch8k: the headmatch calibration at prompt length n=8192 (small 24 "
                    "layers x 14 heads d=64, large 8 layers x 64 heads d=128, planted noisy "
                    "copies); head_match"),
    "decode": ("decode: batch 4, q_len 1, context 8704, sender 14 heads d=64 (its softmax rows "
               "over its paged keys, computed before the timed region), receiver 64 heads "
               "d_v=128, one-hot W, 16-token pages; mapped_av_paged"),
    "prefixindex": ("prefixindex: publish the 4 varlen prompts (40960 tokens, 640 blocks of 64) "
                    "into an empty 4096-slot prefix-hash index, then look up 16 prompts "
                    "(163840 tokens, 2560 blocks) sharing seeded prefixes with them"),
}


# MUFU ex2 issue rate of sm_100 (16 results per clock per SM) x 148 SMs x the maximum SM clock:
# the ALU peak of the exp-bound statistics kernel (4.65e12 ex2/s at 1965 MHz; 4.6e12 measured).
EX2_PER_CLK_SM = 16
B200_SMS = 148
L2_BYTES = 126e6


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    ex2_per_s=EX2_PER_CLK_SM * B200_SMS * d.get("sm_max_mhz", 1965.0) * 1e6,
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                ex2_per_s=EX2_PER_CLK_SM * B200_SMS * 1965.0e6, source="fallback")


def src_sha(files):
    """Hash of the code of the kernel's source files, comments and blank space removed, so that a
    captured DRAM traffic stays attached to the code it was measured on."""
    import re
    h = hashlib.sha256()
    for f in files:
        text = open(os.path.join(ROOT, "cross_model_attention_map_b200", "csrc", f)).read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload, files):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu summary, if it was
    taken on the current source; else None."""
    p = os.path.join(PROFILES, "dram_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel, {}).get(workload)
    if not d or d.get("source_sha") != src_sha(files):
        return None
    return d.get("bytes_per_launch")


# ------------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------------

class ClockSampler:
    """SM clocks and throttle reasons during the timed region (read-only queries).

    nvidia-smi samples every 100 ms; a region shorter than that may get no sample, so an NVML
    poller (every 2 ms, same GPU index) runs beside it and is used when nvidia-smi took none."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    # NVML clocks-event reason bits (nvml.h): SwPowerCap 0x4, HwSlowdown 0x8,
    # SwThermalSlowdown 0x20, HwThermalSlowdown 0x40
    NVML_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
                 ("hw_thermal_slowdown", 0x40))

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.nvml = []
        self.nvml_max = 0.0
        self._poll = None
        self._halt = threading.Event()

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.02)
            self.lines.clear()   # samples from before the timed region
        except (OSError, FileNotFoundError):
            self.proc = None
        self._start_nvml()

    def _start_nvml(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.nvml_max = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception:   # no NVML binding or no device: nvidia-smi alone
            return

        def poll():
            while not self._halt.is_set():
                try:
                    self.nvml.append((float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                                      int(reasons(h))))
                except Exception:
                    return
                self._halt.wait(0.002)

        self._poll = threading.Thread(target=poll, daemon=True)
        self._poll.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _stop_nvml(self):
        if self._poll is not None:
            self._halt.set()
            self._poll.join(timeout=2)
            try:
                import pynvml
                pynvml.nvmlShutdown()
            except Exception:
                pass

    def stop(self):
        self._stop_nvml()
        sm, mx, reasons = [], 0.0, set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in self.lines:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) < 7:
                    continue
                try:
                    sm.append(float(parts[0]))
                    mx = max(mx, float(parts[1]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[3:7]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if sm:
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                    "reasons": sorted(reasons), "samples": len(sm)}
        if self.nvml:
            for _, bits in self.nvml:
                reasons.update(nm for nm, b in self.NVML_BITS if bits & b)
            return {"sm_mhz": statistics.median(c for c, _ in self.nvml),
                    "sm_max_mhz": self.nvml_max, "reasons": sorted(reasons),
                    "samples": len(self.nvml), "source": "nvml, 2 ms polling"}
        return None


# ------------------------------------------------------------------------------------------------
# Distributed plumbing
# ------------------------------------------------------------------------------------------------

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest x over the ranks (a CPU tensor on gloo, a device tensor on NCCL)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------------------
# CPU baseline: the oracle on a bounded sample
# ------------------------------------------------------------------------------------------------

def systematic_rowblocks(wl, count=5):
    """A fixed sample of `count` row blocks of the workload: every (nrb // count)-th row block of
    the sequence-major enumeration, from the middle of the first stride. Row blocks later in a
    sequence cost more (more keys), and an evenly spaced sample follows that mix."""
    import oracle as O
    lay = O.causal_layout(wl.seqlens, wl.B)
    blocks = [(s, I) for s in range(len(wl.seqlens)) for I in range(lay.nb[s])]
    count = max(1, min(count, len(blocks)))
    stride = len(blocks) // count
    return [blocks[stride // 2 + j * stride] for j in range(count)]


def oracle_rowblock(wl, s, I):
    """Oracle compress (all sender heads) + mapped_av rows of one row block: the per-head stats
    (kept sets, near marks) and the number of query rows."""
    import oracle as O
    st = {h: O.rowblock_stats(wl.q, wl.k, wl.cu_seqlens, s, h, I, wl.B, wl.tau,
                              wl.bias_window, wl.bias_value) for h in range(wl.H_s)}
    O.mapped_av_rows(wl, s, I, lambda h: st[h].kept, lambda h: st[h])
    return st, st[0].R


def oracle_sample_prefill(wl, blocks):
    """Oracle compress + mapped_av on the given row blocks (all sender and receiver heads).
    Returns (tokens/s, rows, seconds, per-block stats, sample text)."""
    rows = 0
    stats = []
    t0 = time.perf_counter()
    for s, I in blocks:
        st, R = oracle_rowblock(wl, s, I)
        rows += R
        stats.append((s, I, st))
    dt = time.perf_counter() - t0
    text = ("%d row blocks %s (sequence, row block) of %d sequences (%d query rows, all %d sender "
            "and %d receiver heads): float64 compress + mapped_av"
            % (len(blocks), [tuple(b) for b in blocks], len(wl.seqlens), rows, wl.H_s, wl.H_r))
    return rows / dt, rows, dt, stats, text


def kept_set_check(wl, kept_gpu, stats):
    """Kept sets of the GPU against the oracle's on the sampled row blocks: blocks compared,
    near-threshold blocks, flips (all near-threshold) and mismatches outside them."""
    import oracle as O
    lay = O.causal_layout(wl.seqlens, wl.B)
    blocks = near = flips = bad = 0
    for s, I, st in stats:
        c0 = lay.cb(s, I, 0)
        for h in range(wl.H_s):
            g = kept_gpu[h, c0:c0 + I + 1]
            diff = g != st[h].kept
            blocks += I + 1
            near += int(st[h].near.sum())
            flips += int((diff & st[h].near).sum())
            bad += int((diff & ~st[h].near).sum())
    return {"sampled_rowblocks": len(stats), "blocks": blocks, "near_threshold": near,
            "flips": flips, "mismatches_outside_near": bad}


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ------------------------------------------------------------------------------------------------
# GPU arms
# ------------------------------------------------------------------------------------------------

def bf16_dev(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def base_config(name):
    """The prefill workload a bench configuration runs on (a "_sender" configuration adds the
    sender's own output to its base workload)."""
    return name[:-len("_sender")] if name.endswith("_sender") else name


def split_by_sequence(wl_full, world, rank):
    """This rank's sub-batch of a packed prefill batch split by sequence (longest first by
    causal blocks, runner.shard_sequences): (workload of its sequences, their indices)."""
    from synth import select_sequences
    from cross_model_attention_map_b200.runner import shard_sequences
    mine = shard_sequences(wl_full.seqlens, world, wl_full.B)[rank]
    return select_sequences(wl_full, mine), mine


def idle_rank(args, world, tokens_total):
    """A rank that holds no sequence of a split batch: it takes the same barriers and max
    reductions as the others (with zero time), and reports nothing."""
    for _ in range(2):
        barrier(world)
    ms = max_over_ranks(0.0, world)
    barrier(world)
    e2e_ms = max_over_ranks(0.0, world)
    return {"idle": True, "ms": ms, "e2e_ms": e2e_ms, "tokens_total": tokens_total}


def bench_prefill(args, world, rank, local, peaks):
    import torch
    from synth import prefill_config
    from cross_model_attention_map_b200 import iamap as C
    from cross_model_attention_map_b200.runner import PrefillLayer

    dev = torch.device("cuda", local)
    if args.split == "seq":
        # one packed batch split by sequence over the ranks (strong scaling, no collective on
        # the path)
        wl_full = prefill_config(base_config(args.config), seed=0)
        wl, mine = split_by_sequence(wl_full, world, rank)
        tokens_total = wl_full.n
    else:
        wl = prefill_config(base_config(args.config), seed=rank)
        mine = list(range(len(wl.seqlens)))
        tokens_total = wl.n * world
    if not mine:
        return idle_rank(args, world, tokens_total), wl
    q, k, v = bf16_dev(wl.q, dev), bf16_dev(wl.k, dev), bf16_dev(wl.v, dev)
    W = torch.from_numpy(wl.W).to(dev)
    layer = PrefillLayer(wl.seqlens, wl.H_s, wl.d, wl.H_r, wl.d_v, wl.tau, wl.bias_window,
                         wl.bias_value, device=dev)
    stream = torch.cuda.current_stream()
    b = layer.bufs

    def stats():
        C.iamap_compress_stats(q, k, layer.cu, layer.cu_host, layer.num_seqs, layer.n, wl.H_s,
                               wl.d, wl.B, wl.tau, wl.bias_window, wl.bias_value, b["lse"],
                               b["mass"], b["headmask_dense"], b["row_ptr"], b["col_idx"],
                               b["headmask"], b["val_off"], b["counts"], layer.ws, stream)

    sender = args.config.endswith("_sender")
    if sender:
        from synth import make_sender_values
        v_s = bf16_dev(make_sender_values(wl), dev)
        o_s = torch.empty(wl.n, wl.H_s, wl.d, dtype=torch.float32, device=dev)

    def extract():
        if sender:
            C.iamap_compress_extract_with_output(
                q, k, layer.cu, layer.cu_host, layer.num_seqs, layer.n, wl.H_s, wl.d, wl.B,
                wl.bias_window, wl.bias_value, v_s, wl.d, o_s, b["lse"], b["row_ptr"],
                b["col_idx"], b["headmask"], b["val_off"], b["counts"], layer.vals,
                layer.capacity, layer.ws, stream)
            return
        C.iamap_compress_extract(q, k, layer.cu, layer.cu_host, layer.num_seqs, layer.n, wl.H_s,
                                 wl.d, wl.B, wl.bias_window, wl.bias_value, b["lse"],
                                 b["row_ptr"], b["col_idx"], b["headmask"], b["val_off"],
                                 b["counts"], layer.vals, layer.capacity, layer.ws, stream)

    def mapped():
        layer.mapped_av(W, v, stream)

    # launches of our kernels per step: stats call 5 (tables, stats, row count/scan/fill),
    # extract call 3 (tables, extract, zero tail), mapped_av call 2 (tables, mapped_av)
    launches_per_step = 10
    for _ in range(args.warmup):
        stats(); extract(); mapped()
    torch.cuda.synchronize()
    assert C.iamap_device_status(stream) == 0
    nnz_blocks, nnz_tiles = layer.counts()
    # inputs that fit in the 126 MB L2 are flushed between timed steps (a 256 MB write outside
    # the step's events); larger ones are not
    step_bytes = 4.0 * layer.n * wl.H_s * wl.d + 8192.0 * nnz_tiles
    flush = (torch.empty(256 << 20, dtype=torch.uint8, device=dev) if step_bytes < L2_BYTES
             else None)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(stream); stats()
        ev[i][1].record(stream); extract()
        ev[i][2].record(stream); mapped()
        ev[i][3].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier(world)
    if flush is None:
        ms_local = t_start.elapsed_time(t_end) / args.steps
    else:
        ms_local = sum(e[0].elapsed_time(e[3]) for e in ev) / args.steps
    ms = max_over_ranks(ms_local, world)
    t_stats = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    t_extract = sum(e[1].elapsed_time(e[2]) for e in ev) / args.steps
    t_av = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    assert C.iamap_device_status(stream) == 0

    n = layer.n
    value = tokens_total / (ms * 1e-3)

    # algorithmic work per launch
    causal_pairs = sum(L * (L + 1) // 2 for L in wl.seqlens)
    qk_flops = 2.0 * wl.d * causal_pairs * wl.H_s                     # one causal QK^T
    exps = float(causal_pairs) * wl.H_s
    av_bytes = (8192.0 * nnz_tiles + 20.0 * nnz_blocks + 4.0 * (layer.nrb + 1)
                + 2.0 * n * wl.H_r * wl.d_v + 4.0 * n * wl.H_r * wl.d_v + 4.0 * wl.H_r * wl.H_s)
    extract_bytes = 8192.0 * nnz_tiles + 2.0 * 2 * n * wl.H_s * wl.d + 4.0 * n * wl.H_s
    if sender:   # the sender's values read once, its output written once
        extract_bytes += 2.0 * n * wl.H_s * wl.d + 4.0 * n * wl.H_s * wl.d
    kernels = {
        "compress_stats": {"ms": t_stats, "bound": "alu", "exps": exps,
                           "gex2_per_s": exps / (t_stats * 1e-3) / 1e9,
                           "ex2_frac": round(exps / (t_stats * 1e-3) / peaks["ex2_per_s"], 4),
                           "flops": qk_flops, "tflops": qk_flops / (t_stats * 1e-3) / 1e12},
        "compress_extract": {"ms": t_extract, "bound": "hbm", "bytes": extract_bytes,
                             "gbs": extract_bytes / (t_extract * 1e-3) / 1e9,
                             "tflops_qk_recompute": qk_flops * nnz_tiles / (wl.H_s * layer.ncb)
                             / (t_extract * 1e-3) / 1e12},
        "mapped_av": {"ms": t_av, "bound": "hbm", "bytes": av_bytes,
                      "gbs": av_bytes / (t_av * 1e-3) / 1e9},
    }
    dom = max(kernels, key=lambda kname: kernels[kname]["ms"])
    kd = kernels[dom]
    if kd["bound"] == "hbm":
        achieved = kd["gbs"]
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    elif kd["bound"] == "alu":
        achieved = kd["gex2_per_s"]
        peak = peaks["ex2_per_s"] / 1e9
        unit = "Gex2/s"
    else:
        achieved = kd["tflops"]
        peak = peaks["bf16_tflops_sustained"]
        unit = "TFLOP/s"
    files = {"mapped_av": ["mapped_av_tc.cu", "tc_utils.cuh"],
             "compress_stats": ["compress_tc.cu", "tc_utils.cuh"],
             "compress_extract": ["compress_tc.cu", "tc_utils.cuh"]}[dom]
    roofline = {"kernel": dom, "bound": kd["bound"], "achieved": round(achieved, 2),
                "peak": peak, "unit": unit, "frac": round(achieved / peak, 4),
                "traffic": load_traffic(dom, args.config, files),
                "peak_source": peaks["source"] + {"TFLOP/s": " sustained bf16", "GB/s": " HBM copy",
                                                   "Gex2/s": " (16 ex2/clk/SM x 148 SMs x max clock)"}[unit]}

    # end to end through the library's host-buffer entry point (iamap_prefill_steps_host, pinned
    # host buffers): every step uploads its q, k, v, W and reads its output back; the next step's
    # upload and the previous step's read-back overlap the current step's kernels. That entry
    # point runs compress without the sender's own output, so a "_sender" configuration has no
    # end-to-end figure (its base configuration's line has one).
    e2e = None
    if not sender:
        from cross_model_attention_map_b200.runner import HostPrefillPipeline
        hq = torch.empty(q.shape, dtype=q.dtype, pin_memory=True); hq.copy_(q)
        hk = torch.empty(k.shape, dtype=k.dtype, pin_memory=True); hk.copy_(k)
        hv = torch.empty(v.shape, dtype=v.dtype, pin_memory=True); hv.copy_(v)
        hW = torch.empty(W.shape, dtype=W.dtype, pin_memory=True); hW.copy_(W)
        houts = [torch.empty(layer.out.shape, dtype=torch.float32, pin_memory=True)
                 for _ in range(2)]
        pipe = HostPrefillPipeline(layer, device=dev)
        e2e_steps = max(3, args.steps)       # the same K as the device-timed region
        ins = [(hq, hk, hv, hW)] * e2e_steps
        outs = [houts[i % 2] for i in range(e2e_steps)]
        torch.cuda.synchronize()
        pipe.run(ins[:2], outs[:2], stream).synchronize()        # warm-up of the streams
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e1 = pipe.run(ins, outs, stream)
        torch.cuda.synchronize()
        h2d, d2h = pipe.bytes_per_step()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
        del pipe, houts
        e2e = {"value": round(tokens_total / (e2e_ms * 1e-3), 1), "unit": "tokens/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "strong" if args.split == "seq" else "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; the configuration's shapes and distributions)",
        "config": {"workload": CONFIG_TEXT[args.config], "tokens_per_gpu": n,
                   "split": ("sequences %s of the packed batch on rank %d (longest first by "
                             "causal blocks)" % (mine, rank)) if args.split == "seq"
                            else "one whole batch per GPU",
                   "nnz_blocks": nnz_blocks, "nnz_tiles": nnz_tiles,
                   "kept_tile_density": round(nnz_tiles / (wl.H_s * layer.ncb), 4),
                   "l2": ("inputs larger than L2 (Q+K %.0f MB, BSR values %.1f GB); no flush"
                          % (4.0 * n * wl.H_s * wl.d / 1e6, 8192.0 * nnz_tiles / 1e9)
                          if flush is None else
                          "inputs fit in L2 (%.1f MB): 256 MB buffer written between timed "
                          "steps, outside the step's events" % (step_bytes / 1e6)),
                   "parallelism": ("sequence split over %d GPUs (no collective)" % world
                                   if args.split == "seq" else
                                   "dp%d (independent batches per GPU, no collective)" % world)},
        "kernels": {kk: {x: (round(y, 4) if isinstance(y, float) else y) for x, y in kv.items()}
                    for kk, kv in kernels.items()},
        "roofline": roofline,
        "clocks": clocks,
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
    }
    if e2e is None:
        line["e2e_note"] = ("none: the host-buffer entry point runs compress without the "
                            "sender's own output; the base configuration's line has the figure")
    hm = layer.bufs["headmask_dense"].cpu().numpy().view(np.uint64)
    line["_kept"] = ((hm[None, :] >> np.arange(wl.H_s, dtype=np.uint64)[:, None])
                     & np.uint64(1)).astype(bool)
    return line, wl


def bench_decode(args, world, rank, local, peaks):
    import torch
    from synth import decode_config
    from cross_model_attention_map_b200 import iamap as C
    from cross_model_attention_map_b200.runner import DecodeStep

    dev = torch.device("cuda", local)
    dw = decode_config(seed=rank)
    st = DecodeStep(dw.batch, dw.H_s, dw.H_r, dw.d_v, dw.ctx_lens, dw.p_rows.shape[2],
                    dw.page_table.shape[1], dw.page_size, dw.v_pages.shape[0], device=dev)
    W = torch.from_numpy(dw.W).to(dev)
    vp = bf16_dev(dw.v_pages, dev)
    pt = torch.from_numpy(dw.page_table).to(dev)
    stream = torch.cuda.current_stream()
    # the sender rows: the small model's own softmax rows over its paged keys, computed by the
    # library before the timed region (the small model runs its attention anyway)
    max_ctx = int(dw.ctx_lens.max())
    p = torch.empty(dw.batch, dw.H_s, max_ctx, dtype=torch.float32, device=dev)
    rws = C.alloc_workspace(C.iamap_sender_rows_workspace_bytes(dw.batch, dw.H_s, max_ctx), dev)
    C.iamap_sender_rows(bf16_dev(dw.q_s, dev), bf16_dev(dw.k_pages_s, dev),
                        dw.k_pages_s.shape[0], pt, dw.page_table.shape[1], dw.page_size,
                        st.ctx_lens, dw.ctx_lens, dw.batch, dw.H_s, dw.q_s.shape[2], p, max_ctx,
                        rws, stream)
    for _ in range(args.warmup):
        st.run(p, W, vp, pt, stream)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    for a, b in evs:
        a.record(stream)
        st.run(p, W, vp, pt, stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    assert C.iamap_device_status(stream) == 0
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    ctx = int(dw.ctx_lens.sum())
    byts = 2.0 * ctx * dw.H_r * dw.d_v + 4.0 * ctx * dw.H_s + 4.0 * dw.batch * dw.H_r * dw.d_v
    gbs = byts / (ms * 1e-3) / 1e9
    return {
        "metric": "decode rows/s (paged mapped_av, batch 4, context 8704)",
        "value": round(dw.batch * world / (ms * 1e-3), 1), "unit": "rows/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": CONFIG_TEXT["decode"],
                                        "l2": "inputs larger than L2 (V pages %.0f MB); no flush"
                                              % (vp.numel() * 2 / 1e6)},
        "roofline": {"kernel": "paged_gemv", "bound": "hbm", "achieved": round(gbs, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 4),
                     "traffic": load_traffic("paged_gemv", "decode", ["decode.cu"])},
        "clocks": clocks, "gpu_launches": 2 * args.steps,
    }, dw


def bench_headmatch(args, world, rank, local, peaks):
    import torch
    from synth import head_match_config
    from cross_model_attention_map_b200 import iamap as C
    from cross_model_attention_map_b200.runner import HeadMatch

    dev = torch.device("cuda", local)
    if args.config == "headmatch8k":
        from synth import make_head_match
        hm = make_head_match(n=8192, seed=rank)
    else:
        hm = head_match_config(seed=rank)
    r = HeadMatch(hm.L_s, hm.H_small, hm.d_small, hm.L_l, hm.H_large, hm.d_large, hm.n,
                  want_sim=False, device=dev)
    qs, ks = bf16_dev(hm.q_small, dev), bf16_dev(hm.k_small, dev)
    ql, kl = bf16_dev(hm.q_large, dev), bf16_dev(hm.k_large, dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        r.run(qs, ks, ql, kl, stream)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    clk = ClockSampler(local)
    barrier(world)
    clk.start()
    for a, b in evs:
        a.record(stream)
        r.run(qs, ks, ql, kl, stream)
        b.record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    assert C.iamap_device_status(stream) == 0
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / args.steps, world)
    nb = (hm.n + 63) // 64
    K = nb * (nb + 1) // 2 * 4096
    NS, NL = hm.L_s * hm.H_small, hm.L_l * hm.H_large
    pairs = hm.n * (hm.n + 1) // 2
    gram = 2.0 * NS * NL * pairs
    maps = 2.0 * pairs * (NS * hm.d_small + NL * hm.d_large)
    tf = (gram + maps) / (ms * 1e-3) / 1e12
    planted = float((r.argmax.cpu().numpy().reshape(hm.L_l, hm.H_large) == hm.planted).mean())
    return {
        "metric": "head_match calibrations/s (n=%d, 336 small x 512 large heads)" % hm.n,
        "value": round(world / (ms * 1e-3), 2), "unit": "calibrations/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": {"workload": CONFIG_TEXT[args.config],
                                        "gram_K_padded": K,
                                        "planted_mapping_recovered": planted,
                                        "l2": "inputs larger than L2 (Q, K of both models "
                                              "%.0f MB); no flush" % (2.0 * (
                                                  qs.numel() + ks.numel() + ql.numel()
                                                  + kl.numel()) / 1e6)},
        "roofline": {"kernel": "head_match (maps + gram)", "bound": "tensor",
                     "achieved": round(tf, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(tf / peaks["bf16_tflops"], 4), "traffic": None,
                     "flops": {"gram": gram, "maps_qk": maps}},
        "clocks": clocks, "gpu_launches": 5 * args.steps,
    }, hm


def bench_prefixindex(args, world, rank, local, peaks):
    import torch
    from synth import prefix_config
    from cross_model_attention_map_b200 import iamap as C
    from cross_model_attention_map_b200.runner import PrefixIndex

    dev = torch.device("cuda", local)
    w = prefix_config(seed=rank)
    idx = PrefixIndex(1 << 12, B=w.B, salt=w.salt, device=dev)
    ct = torch.from_numpy(w.cached_tokens).to(dev)
    qt = torch.from_numpy(w.query_tokens).to(dev)
    ccu, qcu = torch.from_numpy(w.cached_cu).to(dev), torch.from_numpy(w.query_cu).to(dev)
    nc = C.iamap_prefix_num_keys(w.cached_cu, len(w.cached_cu) - 1, w.B)
    nq = C.iamap_prefix_num_keys(w.query_cu, len(w.query_cu) - 1, w.B)
    ckeys = torch.empty(nc, dtype=torch.int64, device=dev)
    ccu_k = torch.empty(len(w.cached_cu), dtype=torch.int64, device=dev)
    qkeys = torch.empty(nq, dtype=torch.int64, device=dev)
    qcu_k = torch.empty(len(w.query_cu), dtype=torch.int64, device=dev)
    locs = torch.arange(nc, dtype=torch.int64, device=dev)
    stored = torch.empty(nc, dtype=torch.int64, device=dev)
    found = torch.empty(nq, dtype=torch.int64, device=dev)
    hits = torch.empty(len(w.query_cu) - 1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    stream = torch.cuda.current_stream()
    S_c, S_q = len(w.cached_cu) - 1, len(w.query_cu) - 1

    def step(e=None):
        if e:
            e[0].record(stream)
        C.iamap_prefix_index_clear(idx.table_keys, idx.table_vals, idx.capacity, stream)
        C.iamap_prefix_keys(ct, ct.numel(), ccu, S_c, w.B, w.salt, ckeys, nc, ccu_k, stream)
        C.iamap_prefix_insert(ckeys, locs, nc, idx.table_keys, idx.table_vals, idx.capacity,
                              stored, stream)
        if e:
            e[1].record(stream)
        C.iamap_prefix_keys(qt, qt.numel(), qcu, S_q, w.B, w.salt, qkeys, nq, qcu_k, stream)
        if e:
            e[2].record(stream)
        C.iamap_prefix_lookup(qkeys, nq, qcu_k, S_q, idx.table_keys, idx.table_vals,
                              idx.capacity, found, hits, stream)
        if e:
            e[3].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clk = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clk.start()
    for e in evs:
        flush.zero_()            # L2 flush outside the timed events
        step(e)
    torch.cuda.synchronize()
    clocks = clk.stop()
    assert C.iamap_device_status(stream) == 0
    ms = max_over_ranks(sum(e[0].elapsed_time(e[3]) for e in evs) / args.steps, world)
    t_pub = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_qkeys = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    t_look = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    tokens = ct.numel() + qt.numel()
    # prompt keys kernel: token ids read (4 B), keys written (8 B), offsets (8 B per sequence)
    key_bytes = 4.0 * qt.numel() + 8.0 * nq + 8.0 * (S_q + 1)
    gbs = key_bytes / (t_qkeys * 1e-3) / 1e9
    return {
        "metric": "prefix-index prompt tokens/s (publish + look up, chained 64-token blocks)",
        "value": round(tokens * world / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u64",
        "data": "synthetic", "config": {"workload": CONFIG_TEXT["prefixindex"],
                                        "l2": "256 MB buffer written between timed steps",
                                        "ms_publish": round(t_pub, 4),
                                        "ms_prompt_keys": round(t_qkeys, 4),
                                        "ms_lookup": round(t_look, 4)},
        "roofline": {"kernel": "prefix_keys (16 prompts)", "bound": "hbm",
                     "achieved": round(gbs, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(gbs / peaks["hbm_gbs"], 5), "traffic": None},
        "clocks": clocks, "gpu_launches": 5 * args.steps,
    }, w


def oracle_prefix_step(w):
    """One oracle pass of the prefix-index step (publish the cached prompts, look up the others):
    (tokens/s, seconds)."""
    from oracle import prefix_index as px
    t0 = time.perf_counter()
    ck, _ = px.prefix_keys(w.cached_tokens, w.cached_cu, w.B, w.salt)
    idx = px.PrefixIndex()
    idx.insert(ck, np.arange(len(ck), dtype=np.int64))
    qk, q_cu = px.prefix_keys(w.query_tokens, w.query_cu, w.B, w.salt)
    px.prefix_hits(idx.lookup(qk), q_cu)
    dt = time.perf_counter() - t0
    return (len(w.cached_tokens) + len(w.query_tokens)) / dt, dt


def oracle_decode_step(dw):
    """One float64 oracle decode step (all rows of the batch): (rows/s, seconds)."""
    import oracle as O
    t0 = time.perf_counter()
    O.mapped_av_paged(dw)
    dt = time.perf_counter() - t0
    return dw.batch / dt, dt


def oracle_headmatch_sample(hm, layers=None):
    """The float64 oracle calibration on the first `layers` large layers (all of them by default)
    against every small head: (calibrations/s, seconds). A partial sample counts as
    layers / L_l of a calibration; the small maps are recomputed in full every time, so that
    count favours the GPU."""
    import dataclasses
    import oracle as O
    layers = hm.L_l if layers is None else int(layers)
    sub = dataclasses.replace(hm, L_l=layers, q_large=hm.q_large[:layers],
                              k_large=hm.k_large[:layers], planted=hm.planted[:layers])
    t0 = time.perf_counter()
    O.head_match(sub)
    dt = time.perf_counter() - t0
    return (layers / hm.L_l) / dt, dt


def _reference_line(args, metric, value, unit, ms, workload, cores_used, sample):
    print(json.dumps({
        "impl": "reference", "metric": metric, "value": round(value, 4), "unit": unit,
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload},
        "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": cores_used,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def reference_arm(args):
    """The float64 oracle on the host cores, same metric and unit, bounded sample per step."""
    from synth import prefill_config
    if args.config == "prefixindex":
        from synth import prefix_config
        w = prefix_config()
        for _ in range(args.warmup):
            oracle_prefix_step(w)
        vals = [oracle_prefix_step(w)[0] for _ in range(args.steps)]
        value = statistics.mean(vals)
        tokens = len(w.cached_tokens) + len(w.query_tokens)
        print(json.dumps({
            "impl": "reference",
            "metric": "prefix-index prompt tokens/s (publish + look up, chained 64-token blocks)",
            "value": round(value, 1), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * tokens / value, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u64",
            "data": "synthetic", "config": {"workload": CONFIG_TEXT["prefixindex"]},
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle", "sample": "the whole workload per step"},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }))
        return
    if args.config == "decode":
        from synth import decode_config
        dw = decode_config()
        for _ in range(args.warmup):
            oracle_decode_step(dw)
        runs = [oracle_decode_step(dw) for _ in range(args.steps)]
        value = statistics.mean(v for v, _ in runs)
        _reference_line(args, "decode rows/s (paged mapped_av, batch 4, context 8704)", value,
                        "rows/s", 1e3 * dw.batch / value, CONFIG_TEXT["decode"], cores(),
                        "one whole decode step (batch 4) per step")
        return
    if args.config == "headmatch":
        from synth import head_match_config
        hm = head_match_config()
        for _ in range(args.warmup):
            oracle_headmatch_sample(hm, 1)
        runs = [oracle_headmatch_sample(hm, 1) for _ in range(args.steps)]
        value = statistics.mean(v for v, _ in runs)
        _reference_line(args, "head_match calibrations/s (n=1024, 336 small x 512 large heads)",
                        value, "calibrations/s", 1e3 / value, CONFIG_TEXT["headmatch"], cores(),
                        "per step: 1 of the 8 large layers (64 large heads) against all 336 "
                        "small heads, counted as 1/8 calibration")
        return
    if args.config not in ("varlen40k", "prefill8k", "tiny"):
        print(json.dumps({"impl": "reference", "unavailable":
                          "no reference arm for this configuration"}))
        return
    wl = prefill_config(args.config)
    sample = systematic_rowblocks(wl)
    for i in range(args.warmup):
        oracle_rowblock(wl, *sample[i % len(sample)])
    rows = 0
    step_s = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        _, R = oracle_rowblock(wl, *sample[i % len(sample)])
        step_s.append(time.perf_counter() - t0)
        rows += R
    secs = sum(step_s)
    value = rows / secs
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / args.steps, 2),
        "ms_per_workload_extrapolated": round(1e3 * sum(wl.seqlens) / value, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": CONFIG_TEXT[args.config]},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores(),
                         "kind": "oracle",
                         "sample": "step i: row block i mod %d of the fixed sample %s (sequence, "
                                   "row block), all %d sender and %d receiver heads; %d query "
                                   "rows timed in %.1f s over %d steps"
                                   % (len(sample), [tuple(b) for b in sample], wl.H_s, wl.H_r,
                                      rows, secs, args.steps)},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="varlen40k", choices=sorted(CONFIG_TEXT))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--split", default="batch", choices=["batch", "seq"],
                    help="multi-GPU prefill: one whole batch per GPU (weak scaling) or one packed "
                         "batch split by sequence (strong scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        reference_arm(args)
        return

    world, rank, local = dist_setup(args)
    peaks = load_peaks()
    if base_config(args.config) in ("varlen40k", "prefill8k", "tiny"):
        line, wl = bench_prefill(args, world, rank, local, peaks)
    elif args.config == "decode":
        line, wl = bench_decode(args, world, rank, local, peaks)
    elif args.config == "prefixindex":
        line, wl = bench_prefixindex(args, world, rank, local, peaks)
    else:
        line, wl = bench_headmatch(args, world, rank, local, peaks)
    kept_gpu = line.pop("_kept", None)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and base_config(args.config) in (
            "varlen40k", "prefill8k", "tiny"):
        v, rows, dt, stats, text = oracle_sample_prefill(wl, systematic_rowblocks(wl))
        line["cpu_baseline"] = {"value": round(v, 2), "unit": "tokens/s", "cores": cores(),
                                "kind": "oracle", "sample": text + " in %.1f s" % dt}
        line["kept_set_check"] = kept_set_check(wl, kept_gpu, stats)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "decode":
        v, dt = oracle_decode_step(wl)
        line["cpu_baseline"] = {"value": round(v, 3), "unit": "rows/s", "cores": cores(),
                                "kind": "oracle",
                                "sample": "one whole decode step (batch 4) in %.1f s" % dt}
    if rank == 0 and world == 1 and args.config == "headmatch8k":
        line["cpu_baseline"] = None
        line["cpu_baseline_note"] = ("none: the float64 oracle would hold the 336 small heads' "
                                     "flattened 8192 x 8192 maps (180 GB)")
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "headmatch":
        v, dt = oracle_headmatch_sample(wl)
        line["cpu_baseline"] = {"value": round(v, 4), "unit": "calibrations/s",
                                "cores": cores(), "kind": "oracle",
                                "sample": "one whole calibration in %.1f s" % dt}
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.config == "prefixindex":
        v, dt = oracle_prefix_step(wl)
        line["cpu_baseline"] = {"value": round(v, 1), "unit": "tokens/s", "cores": 1,
                                "kind": "oracle",
                                "sample": "the whole workload, one pass in %.1f s" % dt}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
