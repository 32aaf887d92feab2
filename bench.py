#!/usr/bin/env python
"""Benchmark of one FCA decode step (one layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fca|reference]
                    [--config llama8b|longctx|forest|mixed|pairs|tiny] [--layers L]

A step is one pass of the whole hot path -- grouped prefix pass, per-request
pass, log-sum-exp merge -- over the configuration's synthetic batch, with the
plan built beforehand (plan time is reported separately).  Inputs are
resident in HBM; L2 is flushed (256 MiB write) before every timed step.
Every step is one fca_decode call (the two passes share the SMs, the
per-request pass taking over each SM the grouped pass frees, then the merge),
timed on the device with CUDA events on the
launching stream; ms_per_step is the mean over the K timed steps (max over
ranks).  The roofline times each pass alone on every SM through its own
entry point, in a second loop after the timed region.

value = unique KV bytes processed by all ranks per step / ms_per_step, in
GB/s (each shared block counted once).  Under torchrun every rank decodes its
own independent batch (seed = rank): weak scaling, no collective on the data
path; the only collectives are the barriers and the max-reduction of the
timings.

Extra keys: the flat paged decode of the same batch (speedup_vs_flat), the
per-kernel roofline of the dominant kernel, the CPU oracle as a baseline, an
end-to-end number through the public API with host buffers, and the SM clocks
sampled during the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FCA decode µs/step; unique-KV HBM GB/s (% peak); speedup vs flat paged decode"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
DOMINANT_SOURCES = {"prefix": "fca_prefix.cu", "suffix": "fca_suffix.cu", "merge": "fca_merge.cu"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["fca", "reference"], default="fca")
    ap.add_argument("--config", default="llama8b")
    ap.add_argument("--split", type=int, default=0, help="split-KV chunk tokens (0 = automatic)")
    ap.add_argument("--prompts", type=int, default=None,
                    help="shrink the configuration to this many prompts (profiling captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true",
                    help="no clock sampling and no untimed steps around the timed region (profiling runs)")
    ap.add_argument("--no-flat", action="store_true")
    ap.add_argument("--layers", type=int, default=1,
                    help="also time a multi-layer step: one plan, then this many layers' decodes")
    ap.add_argument("--cpu-budget-s", type=float, default=12.0,
                    help="approximate CPU seconds of the oracle baseline sample")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the lighter measurement of the other configurations")
    ap.add_argument("--per-config-steps", type=int, default=10,
                    help="timed steps per configuration in per_config")
    return ap.parse_args()


FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
PER_CONFIGS = ("tiny", "llama8b", "longctx", "forest", "mixed")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peaks():
    """(bf16 burst TFLOP/s, bf16 sustained TFLOP/s, 'measured' | 'fallback')."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


def prefix_flops(suffix_start, block_size: int, Hq: int, D: int) -> int:
    """Algorithmic flops of the grouped pass: every query head of a request
    attends every token its groups cover once (Q.K^T and P.V, 2 x 2 D flops
    per query row and key).  A request's groups cover tokens
    [0, suffix_start x block_size)."""
    import numpy as np
    return int(np.asarray(suffix_start, dtype=np.int64).sum()) * block_size * Hq * 4 * D


def prefix_roofline(prefix_bytes: int, flops: int, prefix_ms: float, hbm_gbs: float, tflops_burst: float,
                    tflops_sustained: float, peak_kind: str, tensor_pipe_pct=None):
    """The grouped pass timed alone on every SM: K/V bytes it streams (each
    shared token once per group) and its algorithmic flops over its duration,
    as fractions of the measured copy bandwidth and bf16 tensor peaks."""
    if prefix_ms is None or prefix_ms <= 0 or prefix_bytes <= 0:
        return None
    gbs = prefix_bytes / (prefix_ms * 1e-3) / 1e9
    tfs = flops / (prefix_ms * 1e-3) / 1e12
    return {"kernel": "k_prefix", "us": prefix_ms * 1e3, "algorithmic_bytes": int(prefix_bytes),
            "algorithmic_flops": int(flops), "achieved_gbs": gbs, "frac_hbm": gbs / hbm_gbs,
            "achieved_tflops": tfs, "frac_tensor_burst": tfs / tflops_burst,
            "frac_tensor_sustained": tfs / tflops_sustained, "tensor_pipe_pct": tensor_pipe_pct,
            "peak_note": f"{peak_kind} hbm_gbs, bf16_tflops and bf16_tflops_sustained"}


def workload_desc(w):
    return (f"{w.name}: {w.description}; {w.R} requests, heads {w.Hq}/{w.Hkv}/{w.D}, bf16 paged "
            f"KV, block {w.block_size}, {w.num_blocks} physical blocks")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return summarize_clock_samples(lines)


def _num(text: str):
    try:
        return float(text)
    except ValueError:
        return None


def summarize_clock_samples(lines, busy_watts: float = 200.0):
    """Summary of nvidia-smi rows in ClockSampler.FIELDS order (csv, no header,
    no units): the median SM clock over the samples drawn under load (power at
    least busy_watts; all samples if none was), the highest max clock, the
    throttle reasons seen active in any sample, and the sample counts.  Fields
    that are not numbers ("[N/A]") leave their sample out of that statistic."""
    rows = []
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) >= 9:
            rows.append(parts)
    if not rows:
        return None
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = set()
    sm, mx, pw, busy = [], [], [], []
    for r in rows:
        s_mhz, m_mhz, watts = _num(r[1]), _num(r[2]), _num(r[3])
        if s_mhz is not None:
            sm.append(s_mhz)
            if watts is not None and watts >= busy_watts:
                busy.append(s_mhz)
        if m_mhz is not None:
            mx.append(m_mhz)
        if watts is not None:
            pw.append(watts)
        for name, val in zip(names, r[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    loaded = busy or sm
    return {"sm_mhz": statistics.median(loaded) if loaded else None,
            "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(busy),
            "power_w_max": max(pw) if pw else None}


def gpu_id_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------------ ranks

class RankReducer:
    """Max / sum of one float over all ranks; the identity at world size 1.
    Every rank must make the same calls in the same order."""

    def __init__(self, world: int, device=None):
        self.world = world
        self.device = device

    def _reduce(self, x: float, op) -> float:
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist
        t = torch.tensor([float(x)], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x: float) -> float:
        import torch.distributed as dist
        return self._reduce(x, dist.ReduceOp.MAX)

    def sum(self, x: float) -> float:
        import torch.distributed as dist
        return self._reduce(x, dist.ReduceOp.SUM)


def aggregate_step(step_ms: float, unique_bytes_rank: int, red: RankReducer):
    """Whole-job throughput of one step: the unique KV bytes every rank
    processed over the slowest rank's step time.  Returns (max step ms,
    total bytes, GB/s)."""
    step = red.max(step_ms)
    total = red.sum(unique_bytes_rank)
    return step, total, total / (step * 1e-3) / 1e9


# ------------------------------------------------------------------ oracle legs

def oracle_sample(w, budget_s: float, seed: int = 0):
    """Time the oracle (as it stands) on whole requests, all heads, until about
    budget_s seconds of work; return (seconds, tokens covered, requests)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    order = rng.permutation(w.R)
    # calibrate on one request
    r0 = int(order[0])
    pairs = np.array([[r0, h] for h in range(w.Hq)], np.int32)
    t = time.perf_counter()
    oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, pairs=pairs)
    t1 = max(time.perf_counter() - t, 1e-4)
    per_token = t1 / float(w.seq_lens[r0])
    target_tokens = budget_s / per_token
    chosen, tok = [], 0
    for r in order:
        chosen.append(int(r))
        tok += int(w.seq_lens[r])
        if tok >= target_tokens:
            break
    pairs = np.array([[r, h] for r in chosen for h in range(w.Hq)], np.int32)
    t = time.perf_counter()
    oracle.paged_attention(w.q, w.k_cache, w.v_cache, w.block_tables, w.seq_lens, w.scale, pairs=pairs)
    return time.perf_counter() - t, tok, len(chosen)


def cpu_cores() -> int:
    v = os.environ.get("OMP_NUM_THREADS")
    if v and v.isdigit():
        return int(v)
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def unique_bytes(w) -> int:
    import oracle
    return oracle.unique_kv_tokens(w.block_tables, w.seq_lens, w.block_size, w.num_blocks) * w.Hkv * w.D * 4


def reference_arm(args):
    import fca_workloads
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = fca_workloads.make(args.config, seed=0, prompts=args.prompts)
    ub = unique_bytes(w)
    total_tok = int(w.seq_lens.sum())
    per_step_budget = max(0.5, 150.0 / max(1, args.steps + args.warmup))
    times = []
    for i in range(args.warmup + args.steps):
        sec, tok, nreq = oracle_sample(w, per_step_budget, seed=i)
        if i >= args.warmup:
            times.append(sec * total_tok / tok)   # extrapolated to the whole batch
    step_s = statistics.mean(times)
    value = ub / step_s / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(w)}, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"whole requests (all {w.Hq} heads) totalling about "
                                       f"{per_step_budget:.1f} s of CPU work per step, time scaled "
                                       f"to the full batch of {total_tok} tokens"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ FCA arm

def traffic_entry(kernel: str, workload: str):
    """The committed ncu record of a kernel on a workload (profiles/traffic.json),
    or None when there is none for this kernel source and workload."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        ent = rec[kernel][workload]
        src = os.path.join(ROOT, "shared_prefix_kv_fca_b200", "csrc", DOMINANT_SOURCES[kernel])
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if ent.get("source_sha256_16") != digest:
            return None
        return ent
    except Exception:
        return None


def traffic_record(dominant: str, workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary,
    or None when there is none for this kernel source and workload."""
    ent = traffic_entry(dominant, workload)
    try:
        return float(ent["dram_bytes_per_launch"]) if ent else None
    except Exception:
        return None


def measure_config(name, args, dev, rank, flush, red, peak, prefix_line):
    """One configuration, lighter than the headline: whole fca_decode steps
    (L2 flushed before each), the three passes alone on every SM, and the flat
    paged decode of the same batch; every rank decodes its own batch."""
    import torch
    import fca_workloads
    import shared_prefix_kv_fca_b200 as fca

    w = fca_workloads.make(name, seed=rank)
    q, k, v, bt, sl = w.torch_inputs(dev)
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device=dev)
    n, warm = args.per_config_steps, max(3, min(args.warmup, 5))

    def steps(p, flat=False):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(warm + n):
            flush.zero_()
            if i >= warm:
                ev[i - warm][0].record(stream)
            (fca.fca_flat_decode if flat else fca.fca_decode)(q, k, v, p, out, lse, w.scale, stream)
            if i >= warm:
                ev[i - warm][1].record(stream)
        torch.cuda.synchronize(dev)
        return red.max(statistics.mean(a.elapsed_time(b) for a, b in ev))

    def passes(p):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for i in range(warm + n):
            flush.zero_()
            e = ev[i - warm] if i >= warm else None
            if e: e[0].record(stream)
            fca.fca_prefix_pass(q, k, v, p, w.scale, stream)
            if e: e[1].record(stream)
            fca.fca_suffix_pass(q, k, v, p, w.scale, stream)
            if e: e[2].record(stream)
            fca.fca_merge_pass(p, out, lse, stream)
            if e: e[3].record(stream)
        torch.cuda.synchronize(dev)
        return {key: red.max(statistics.mean(e[i].elapsed_time(e[i + 1]) for e in ev))
                for i, key in enumerate(("prefix", "suffix", "merge"))}

    plan = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split)
    st, exp = plan.stats(), plan.export()
    step_ms = steps(plan)
    pass_ms = passes(plan)
    assert fca.fca_check_device_status(plan, stream) == 0
    flat_ms = None
    if not args.no_flat:
        flat = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, flat=True, split_tokens=args.split)
        flat_ms = steps(flat, flat=True)
        assert fca.fca_check_device_status(flat, stream) == 0
        flat.close()
    total = red.sum(st["unique_kv_bytes"])
    gbs = total / (step_ms * 1e-3) / 1e9
    res = {"us_per_step": step_ms * 1e3, "unique_kv_gbs": gbs, "pct_of_peak": 100.0 * gbs / (peak * red.world),
           "flat_us_per_step": flat_ms * 1e3 if flat_ms else None,
           "speedup_vs_flat": (flat_ms / step_ms) if flat_ms else None,
           "passes_us": {key: val * 1e3 for key, val in pass_ms.items()},
           "roofline_prefix": prefix_line(st, exp, w, pass_ms["prefix"], name),
           "unique_kv_bytes_per_rank": st["unique_kv_bytes"], "groups": st["num_groups"],
           "workload": workload_desc(w)}
    plan.close()
    del q, k, v, bt, sl, out, lse
    torch.cuda.empty_cache()
    return res


def fca_arm(args):
    import torch
    import torch.distributed as dist

    import fca_workloads
    import shared_prefix_kv_fca_b200 as fca

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    red = RankReducer(world, dev)
    max_over_ranks, sum_over_ranks = red.max, red.sum

    w = fca_workloads.make(args.config, seed=rank, prompts=args.prompts)
    q, k, v, bt, sl = w.torch_inputs(dev)
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(q)
    lse = torch.empty(w.R, w.Hq, dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    torch.cuda.synchronize(dev)
    t0 = time.perf_counter()
    plan = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split)
    torch.cuda.synchronize(dev)
    plan_ms = (time.perf_counter() - t0) * 1e3
    st = plan.stats()
    exp = plan.export()
    # the same plan again, as a decode loop that plans every step would: the
    # first plan above also pays for the process's first pool allocations
    steady = []
    for _ in range(10):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split).close()
        torch.cuda.synchronize(dev)
        steady.append((time.perf_counter() - t0) * 1e3)
    plan_ms_steady = statistics.median(steady)
    flat_plan = None if args.no_flat else fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, flat=True,
                                                       split_tokens=args.split)

    def run_steps(p, n, timed, flush_l2=True):
        """n whole decode steps (fca_decode: both passes at once, then the
        merge), each bracketed by events on the launching stream."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            if flush_l2:
                flush.zero_()
            ev[i][0].record(stream)
            fca.fca_decode(q, k, v, p, out, lse, w.scale, stream)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        if not timed:
            return None
        return statistics.mean(a.elapsed_time(b) for a, b in ev)

    def run_passes(p, n, timed):
        """n steps with the three passes launched one after another through
        their own entry points, each pass on every SM and bracketed by events
        on the launching stream: the per-kernel durations of the roofline."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
        for i in range(n):
            flush.zero_()
            e = ev[i]
            e[0].record(stream)
            fca.fca_prefix_pass(q, k, v, p, w.scale, stream)
            e[1].record(stream)
            fca.fca_suffix_pass(q, k, v, p, w.scale, stream)
            e[2].record(stream)
            fca.fca_merge_pass(p, out, lse, stream)
            e[3].record(stream)
        torch.cuda.synchronize(dev)
        if not timed:
            return None
        per = {"prefix": [], "suffix": [], "merge": [], "step": []}
        for e in ev:
            per["prefix"].append(e[0].elapsed_time(e[1]))
            per["suffix"].append(e[1].elapsed_time(e[2]))
            per["merge"].append(e[2].elapsed_time(e[3]))
            per["step"].append(e[0].elapsed_time(e[3]))
        return {key: statistics.mean(vals) for key, vals in per.items()}

    # ---- FCA, timed region
    run_steps(plan, args.warmup, False)
    sampler = ClockSampler(gpu_id_for(local)) if rank == 0 and not args.no_clocks else None
    barrier()
    torch.cuda.synchronize(dev)
    def keep_busy(seconds):
        """Untimed steps of the same workload around the timed region, so that
        the clock samples (every 200 ms) see the GPU under this load."""
        if args.no_clocks:
            return
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            run_steps(plan, 8, False)

    if sampler:
        sampler.start()
    keep_busy(0.6)   # every rank, so that the ranks' timed regions run at the same time
    barrier()
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_push("fca_decode: timed steps")
    step_ms_rank = run_steps(plan, args.steps, True)
    torch.cuda.synchronize(dev)
    torch.cuda.nvtx.range_pop()
    barrier()
    keep_busy(0.6)
    clocks = sampler.stop() if sampler else None
    barrier()
    assert fca.fca_check_device_status(plan, stream) == 0
    step_ms, total_unique, value = aggregate_step(step_ms_rank, st["unique_kv_bytes"], red)
    n_launch = (1 if (st["prefix_items"] > 0) else 0) + (1 if st["suffix_items"] > 0 else 0) + 1

    # ---- the same steps back to back without the L2 flush (warm L2)
    run_steps(plan, args.warmup, False, flush_l2=False)
    barrier()
    warm_ms = max_over_ranks(run_steps(plan, args.steps, True, flush_l2=False))
    barrier()

    # ---- the passes one at a time (per-kernel roofline)
    run_passes(plan, args.warmup, False)
    barrier()
    torch.cuda.nvtx.range_push("passes one at a time: timed steps")
    fca_t = run_passes(plan, args.steps, True)
    torch.cuda.nvtx.range_pop()
    barrier()
    assert fca.fca_check_device_status(plan, stream) == 0

    # ---- flat paged decode of the same batch
    flat_ms = None
    if flat_plan is not None:
        run_steps(flat_plan, args.warmup, False)
        barrier()
        torch.cuda.nvtx.range_push("flat decode: timed steps")
        flat_ms_rank = run_steps(flat_plan, args.steps, True)
        torch.cuda.nvtx.range_pop()
        flat_ms = max_over_ranks(flat_ms_rank)
        barrier()
        assert fca.fca_check_device_status(flat_plan, stream) == 0

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        q_h = q.cpu().pin_memory()
        bt_h = bt.cpu().pin_memory()
        sl_h = sl.cpu().pin_memory()
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        q_d, bt_d, sl_d = torch.empty_like(q), torch.empty_like(bt), torch.empty_like(sl)

        side = torch.cuda.Stream(dev)
        q_ready = torch.cuda.Event()

        parts = []

        def e2e_step(record=False):
            # the planner needs only the tables: q is uploaded on a side
            # stream meanwhile, and the decode waits for it
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            ev[0].record(stream)
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                q_d.copy_(q_h, non_blocking=True)
                q_ready.record(side)
            bt_d.copy_(bt_h, non_blocking=True)
            sl_d.copy_(sl_h, non_blocking=True)
            ev[1].record(stream)
            with fca.fca_plan(bt_d, sl_d, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split,
                              stream=stream) as p:
                stream.wait_event(q_ready)
                ev[2].record(stream)
                fca.fca_decode(q_d, k, v, p, out, lse, w.scale, stream)
                ev[3].record(stream)
                out_h.copy_(out, non_blocking=True)
                lse_h.copy_(lse, non_blocking=True)
                ev[4].record(stream)
                torch.cuda.synchronize(dev)
            if record:
                parts.append([ev[i].elapsed_time(ev[i + 1]) for i in range(4)])

        for _ in range(max(1, args.warmup)):
            flush.zero_()
            e2e_step()
        barrier()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step(record=True)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        e2e_ms = max_over_ranks(statistics.mean(times))
        e2e_parts = {key: max_over_ranks(statistics.mean(p[i] for p in parts))
                     for i, key in enumerate(("h2d_tables_ms", "plan_ms", "decode_ms", "d2h_ms"))}

        # the same step in a decode loop that keeps its plan: fca_plan_update
        # (the tables' shared entries unchanged) in place of a new plan, on a
        # plan built for asynchronous updates (no host synchronisation)
        kept = fca.fca_plan(bt_d, sl_d, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split, stream=stream,
                            async_update=True)

        def e2e_update_step():
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                q_d.copy_(q_h, non_blocking=True)
                q_ready.record(side)
            bt_d.copy_(bt_h, non_blocking=True)
            sl_d.copy_(sl_h, non_blocking=True)
            kept.update(bt_d, sl_d, stream)
            stream.wait_event(q_ready)
            fca.fca_decode(q_d, k, v, kept, out, lse, w.scale, stream)
            out_h.copy_(out, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)
            torch.cuda.synchronize(dev)

        for _ in range(max(1, args.warmup)):
            flush.zero_()
            e2e_update_step()
        barrier()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_update_step()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        upd_ms = max_over_ranks(statistics.mean(times))

        # the same kept-plan step captured once as a CUDA graph (uploads, update,
        # decode, downloads) and replayed: the host launches one graph a step
        graph_ms, graph_note, g = None, None, None
        try:
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            g = torch.cuda.CUDAGraph()
            # (thread-local capture: another thread's CUDA calls, a process
            # group's watchdog for one, do not invalidate it)
            with torch.cuda.graph(g, stream=cap, capture_error_mode="thread_local"):
                side.wait_stream(cap)
                with torch.cuda.stream(side):
                    q_d.copy_(q_h, non_blocking=True)
                    q_ready.record(side)
                bt_d.copy_(bt_h, non_blocking=True)
                sl_d.copy_(sl_h, non_blocking=True)
                kept.update(bt_d, sl_d, cap)
                cap.wait_event(q_ready)
                fca.fca_decode(q_d, k, v, kept, out, lse, w.scale, cap)
                out_h.copy_(out, non_blocking=True)
                lse_h.copy_(lse, non_blocking=True)
            stream.wait_stream(cap)
            for _ in range(max(1, args.warmup)):
                flush.zero_()
                g.replay()
        except Exception as ex:   # a capture this build's CUDA cannot take: report it, keep the rest
            graph_note = f"not captured: {type(ex).__name__}: {str(ex)[:160]}"
            g = None
        torch.cuda.synchronize(dev)
        barrier()                 # (every rank, captured or not)
        times = []
        if g is not None:
            for _ in range(args.steps):
                flush.zero_()
                torch.cuda.synchronize(dev)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                b.synchronize()
                times.append(a.elapsed_time(b))
        graph_local = statistics.mean(times) if times else -1.0
        graph_max = max_over_ranks(graph_local)
        graph_min = -max_over_ranks(-graph_local)
        graph_ms = graph_max if graph_min > 0 else None
        del g
        assert fca.fca_check_device_status(kept, stream) == 0
        kept.close()
        h2d = q.numel() * 2 + bt.numel() * 4 + sl.numel() * 4
        d2h = out.numel() * 2 + lse.numel() * 4
        e2e = {"value": sum_over_ranks(st["unique_kv_bytes"]) / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "includes": "H2D of the block tables, fca_plan (one host sync) while q uploads on a "
                           "side stream, fca_decode, D2H of out and lse; the KV cache is resident state",
               "parts": e2e_parts,
               "with_plan_update": {"value": sum_over_ranks(st["unique_kv_bytes"]) / (upd_ms * 1e-3) / 1e9,
                                    "ms_per_step": upd_ms,
                                    "includes": "the same, with fca_plan_update of a kept plan "
                                                "(FCA_PLAN_ASYNC_UPDATE: no host synchronisation) in place "
                                                "of fca_plan"},
               "with_plan_update_graph": {
                   "value": (sum_over_ranks(st["unique_kv_bytes"]) / (graph_ms * 1e-3) / 1e9) if graph_ms else None,
                   "ms_per_step": graph_ms,
                   "includes": graph_note or "the kept-plan step captured once as a CUDA graph (the same "
                                             "uploads, fca_plan_update, fca_decode and downloads) and "
                                             "replayed each step"}}

    # ---- a model-shaped step: one plan serves every layer
    multi = None
    if args.layers > 1:
        ks = [k] + [k.clone() for _ in range(args.layers - 1)]
        vs = [v] + [v.clone() for _ in range(args.layers - 1)]

        def layers_step():
            p = fca.fca_plan(bt, sl, w.num_blocks, w.Hq, w.Hkv, w.D, split_tokens=args.split, stream=stream)
            for kl, vl in zip(ks, vs):
                fca.fca_decode(q, kl, vl, p, out, lse, w.scale, stream)
            return p

        for _ in range(max(1, args.warmup)):
            flush.zero_()
            layers_step().close()
        barrier()
        times = []
        for _ in range(args.steps):
            flush.zero_()
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            p = layers_step()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
            p.close()
        ml_ms = max_over_ranks(statistics.mean(times))
        del ks, vs
        multi = {"layers": args.layers, "ms_per_step": ml_ms,
                 "unique_kv_gbs": args.layers * sum_over_ranks(st["unique_kv_bytes"]) / (ml_ms * 1e-3) / 1e9,
                 "plan_and_launch_share": max(0.0, 1.0 - args.layers * step_ms / ml_ms),
                 "includes": "fca_plan (one host sync) then one fca_decode per layer over distinct caches"}

    peak, peak_kind = peaks()
    tf_burst, tf_sust, tf_kind = tensor_peaks()

    # dominant kernel and its roofline
    pass_ms = {key: max_over_ranks(fca_t[key]) for key in ("prefix", "suffix", "merge")}
    serial_ms = max_over_ranks(fca_t["step"])
    dominant = max(pass_ms, key=pass_ms.get)
    alg_bytes = {"prefix": st["prefix_kv_bytes"], "suffix": st["suffix_kv_bytes"],
                 "merge": st["num_partials"] * (w.D + 1) * 4 + w.R * w.Hq * (w.D * 2 + 4)}
    achieved = alg_bytes[dominant] / (pass_ms[dominant] * 1e-3) / 1e9
    traffic = traffic_record(dominant, args.config)

    def prefix_line(stats, export, wk, prefix_ms, workload):
        ent = traffic_entry("prefix", workload)
        return prefix_roofline(stats["prefix_kv_bytes"], prefix_flops(export["suffix_start"], wk.block_size, wk.Hq, wk.D),
                               prefix_ms if stats["prefix_items"] > 0 else None, peak, tf_burst, tf_sust,
                               f"{peak_kind}/{tf_kind}", ent.get("tensor_pipe_pct") if ent else None)

    roof_prefix = prefix_line(st, exp, w, pass_ms["prefix"], args.config)

    # ---- the other configurations, lighter: whole steps, the passes alone, flat
    per_config = None
    if not args.no_per_config and args.prompts is None:
        per_config = {"steps": args.per_config_steps, "warmup": max(3, min(args.warmup, 5)),
                      "note": "L2 flushed before every step; the headline configuration's entry repeats its "
                              "own measurement"}
        for name in PER_CONFIGS:
            if name == args.config:
                per_config[name] = {"us_per_step": step_ms * 1e3, "unique_kv_gbs": value,
                                    "pct_of_peak": 100.0 * value / (peak * world),
                                    "flat_us_per_step": flat_ms * 1e3 if flat_ms else None,
                                    "speedup_vs_flat": (flat_ms / step_ms) if flat_ms else None,
                                    "passes_us": {key: val * 1e3 for key, val in pass_ms.items()},
                                    "roofline_prefix": roof_prefix}
                continue
            per_config[name] = measure_config(name, args, dev, rank, flush, red, peak, prefix_line)


    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            sec, tok, nreq = oracle_sample(w, args.cpu_budget_s)
            full_s = sec * float(w.seq_lens.sum()) / tok
            cpu = {"value": st["unique_kv_bytes"] / full_s / 1e9, "unit": "GB/s", "cores": cpu_cores(),
                   "kind": "oracle", "ms_per_step": full_s * 1e3, "cpu_model": cpu_model(),
                   "sample": f"{nreq} whole requests x {w.Hq} heads ({tok} tokens of "
                             f"{int(w.seq_lens.sum())}) in {sec:.1f} s, scaled to the full batch"}
            # the same oracle on one core, a smaller sample
            import oracle
            before = oracle.set_threads(1)
            try:
                sec1, tok1, nreq1 = oracle_sample(w, args.cpu_budget_s / 4, seed=1)
            finally:
                oracle.set_threads(before)
            full1 = sec1 * float(w.seq_lens.sum()) / tok1
            cpu["one_core"] = {"value": st["unique_kv_bytes"] / full1 / 1e9, "unit": "GB/s", "cores": 1,
                               "ms_per_step": full1 * 1e3,
                               "sample": f"{nreq1} whole requests x {w.Hq} heads ({tok1} tokens) in "
                                         f"{sec1:.1f} s, scaled to the full batch"}
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "us_per_step": step_ms * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; per-rank seed = rank)",
            "config": {"workload": workload_desc(w), "l2": "flushed before every step (256 MiB write)",
                       "split_tokens": st["split_tokens"], "groups": st["num_groups"],
                       "unique_kv_bytes_per_rank": st["unique_kv_bytes"],
                       "flat_kv_bytes_per_rank": st["flat_kv_bytes"], "replicas": world},
            "pct_of_peak": 100.0 * value / (peak * world), "peak_gbs": peak, "peak_kind": peak_kind,
            "plan_ms": plan_ms, "plan_ms_steady": plan_ms_steady,
            "warm_l2_us_per_step": warm_ms * 1e3,
            "passes_us": {key: val * 1e3 for key, val in pass_ms.items()},
            "serial_passes_us_per_step": serial_ms * 1e3,
            "flat_us_per_step": flat_ms * 1e3 if flat_ms else None,
            "speedup_vs_flat": (flat_ms / step_ms) if flat_ms else None,
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes": alg_bytes[dominant],
                         "peak_note": f"{peak_kind} copy bandwidth (MEASURED_PEAKS hbm_gbs)"},
            "roofline_prefix": roof_prefix, "per_config": per_config,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "multilayer": multi,
            "gpu_launches": n_launch * args.steps, "impl": "fca",
        }
        print(json.dumps(line), flush=True)

    plan.close()
    if flat_plan is not None:
        flat_plan.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return reference_arm(args)
    return fca_arm(args)


if __name__ == "__main__":
    sys.exit(main())
