#!/usr/bin/env python
"""Benchmark of zero-copy host/HBM split-KV decode attention on B200.

One step = one dkv_attn_decode call over one batch of the workload: the
pool-lists kernel, the zero-copy host-stream kernel (aux stream), the HBM
split-K kernel and the LSE merge.  Default workload: the largest single-GPU
configuration, long-context decode (B=1, Hq=32, Hkv=8, D=128, L=1,048,576
tokens, bf16 K/V, 64-token blocks, the oldest 90% of blocks in mapped pinned
host memory and the newest 10% in HBM: 4 GiB of KV per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl dkv|reference]
                    [--mode zero_copy|staged|planned] [--hbm-budget-frac F]

--mode planned measures the workload at its own placement first (and, when
the HBM budget allows, with the whole cache in HBM, for the HBM kernel's rate
alone), gives the measured rates to the offload planner (dkv_plan_offload),
rebuilds the cache at the planned host fraction and reports the planned step:
predicted against measured time and the HBM bytes the placement frees.

With N > 1 (launched by torchrun) every rank runs an independent replica of
the workload on its own GPU and PCIe link; rank 0 prints the JSON line with
the device time taken as the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kvgen  # noqa: E402

METRIC = "decode-attention µs/step & KV GB/s, fraction of PCIe+HBM roofline"
HBM_NOMINAL_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 10**6        # B200 L2
FLUSH_BYTES = 256 << 20       # written between timed steps when the KV of a step fits in L2


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long_ctx")
    ap.add_argument("--impl", choices=("dkv", "reference"), default="dkv")
    ap.add_argument("--mode", choices=("zero_copy", "staged", "planned", "append"), default="zero_copy",
                    help="staged: the prefetch comparator (host pool copied into HBM each step); "
                         "planned: the placement chosen by the offload planner from measured rates; "
                         "append: the write side, K/V projection of every sequence's new token and its store")
    ap.add_argument("--hbm-budget-frac", type=float, default=-1.0,
                    help="planned mode: HBM the cache may use, as a fraction of its bytes (< 0: unlimited)")
    ap.add_argument("--queries", type=int, default=1,
                    help="query tokens per sequence (>1: multi-token queries, e.g. speculative verification)")
    ap.add_argument("--host-ctas", type=int, default=0)
    ap.add_argument("--ctx", type=int, default=0,
                    help="override the context length (a reduced case of the workload, e.g. for profiler captures)")
    ap.add_argument("--host-fraction", type=float, default=-1.0,
                    help="replace the workload's share of blocks in host memory (0..1; < 0: the workload's own)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args(argv)
    if args.host_fraction > 1:
        ap.error("--host-fraction must be at most 1")
    return args


# ----------------------------------------------------------------------------- ranks

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0)))


def dist_init(backend: str):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def workload_for_rank(name: str, rank: int, ctx: int = 0, host_fraction: float = -1.0) -> kvgen.Workload:
    """Replica r draws its own inputs: same shapes and recipe, seed + 1000 r.  ctx > 0 replaces the
    context length (the workload is then named with a "_ctx<N>" suffix); host_fraction >= 0 replaces the
    share of blocks placed in host memory (suffix "_h<F>")."""
    w = kvgen.get(name)
    if ctx > 0:
        w = w.replace(name=f"{w.name}_ctx{ctx}", ctx=ctx)
    if host_fraction >= 0:
        w = w.replace(name=f"{w.name}_h{host_fraction:g}", host_fraction=host_fraction)
    return w if rank == 0 else w.replace(seed=w.seed + 1000 * rank)


# ----------------------------------------------------------------------------- measurements

class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 200 ms while active."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self._wait_rows(1, 5.0)   # nvidia-smi is up and sampling before the timed region starts

    def _rows(self) -> int:
        try:
            with open(self.file.name) as f:
                return sum(1 for line in f if line.strip())
        except OSError:
            return 0

    def _wait_rows(self, n: int, limit_s: float):
        t0 = time.monotonic()
        while self._rows() < n and time.monotonic() - t0 < limit_s and self.proc.poll() is None:
            time.sleep(0.02)

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        self._wait_rows(self._rows() + 1, 1.0)   # one sample taken at the end of a short timed region
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().splitlines() if r.strip()]
        self.file.close()
        os.unlink(self.file.name)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[4:8]):
                if v.strip() == "Active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm), "reasons": sorted(reasons)}


def measure_pcie_gbs(device, nbytes: int = 1 << 30, reps: int = 5) -> float:
    """Pinned host -> device cudaMemcpyAsync bandwidth (the PCIe roofline denominator)."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(nbytes, dtype=torch.uint8, device=device)
    s = torch.cuda.current_stream(device)
    best = float("inf")
    for i in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        dst.copy_(src, non_blocking=True)
        b.record(s)
        b.synchronize()
        if i:
            best = min(best, a.elapsed_time(b))
    del src, dst
    return nbytes / (best * 1e-3) / 1e9


def measured_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def kernel_source_sha() -> str:
    with open(os.path.join(ROOT, "decode_attention_host_b200", "csrc", "dkv_kernels.cuh"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """ncu DRAM + sysmem bytes per launch from profiles/traffic.json, if taken on the current kernel source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(f"{kernel}:{workload}")
    except (OSError, ValueError):
        return None
    if not rec or rec.get("kernel_source_sha") != kernel_source_sha():
        return None
    return rec


CPU_SAMPLE_S = 10.0   # the CPU baseline repeats its sample until at least this much CPU work is timed
CPU_SAMPLE_MAX_REPS = 100000


def oracle_gbs(w: kvgen.Workload, q, k, v, lens, group_mask, min_seconds: float = CPU_SAMPLE_S
               ) -> tuple[float, float, int, int]:
    """Time the fp64 oracle on the (batch, kv head) groups of group_mask, repeated until about
    min_seconds have run (once if 0): (GB/s, seconds, threads, repetitions)."""
    import oracle
    dt = oracle.KV_BF16 if w.kv_dtype == kvgen.BF16 else oracle.KV_F16
    reps, sec = 0, 0.0
    while reps == 0 or (sec < min_seconds and reps < CPU_SAMPLE_MAX_REPS):
        t0 = time.perf_counter()
        oracle.decode(q, k, v, lens, dt, w.rope_base, group_mask=group_mask)
        sec += time.perf_counter() - t0
        reps += 1
    tokens = sum(int(lens[b]) for b in range(w.batch) for h in range(w.num_kv_heads) if group_mask[b, h])
    nbytes = tokens * 2 * w.head_dim * 2 * reps
    return nbytes / sec / 1e9, sec, oracle.num_threads(), reps


# ----------------------------------------------------------------------------- reference arm (the oracle)

def plan_placement(plan_offload, measure_at, rates_of, x: float, budget: float, f0: float, meas0: dict):
    """The offload-planner rounds of --mode planned.

    plan_offload is dkv_plan_offload; measure_at(f) rebuilds the cache with host fraction f and measures a step
    there (a dict with "ms"); rates_of(m) gives the host-stream and HBM kernels' GB/s measured in m.  Rounds:
    the workload's own placement f0 (meas0); when the budget lets the whole cache sit in HBM, that placement,
    for the HBM kernel's rate alone; the side-by-side split, re-planned from the rates measured at the previous
    split (they depend on the operating point) until it settles; finally the plan that weighs that split
    against the whole cache in HBM, measured there unless the last round already was.  Returns the planner
    record and the measurement of the chosen placement, whose cache measure_at left built."""
    host_gbs, hbm_gbs = rates_of(meas0)
    rounds = [{"host_fraction": f0, "measured_step_ms": meas0["ms"], "host_stream_gbs": host_gbs,
               "hbm_split_k_gbs": hbm_gbs}]
    meas, f_cur = meas0, f0
    alone_gbs, all_hbm_ms = -1.0, None
    if f0 == 0:   # the workload's own placement is the whole cache in HBM
        alone_gbs, all_hbm_ms = hbm_gbs, meas0["ms"]
    elif budget < 0 or budget >= x:
        meas, f_cur = measure_at(0.0), 0.0
        alone_gbs, all_hbm_ms = rates_of(meas)[1], meas["ms"]
        rounds.append({"host_fraction": 0.0, "measured_step_ms": all_hbm_ms, "hbm_split_k_gbs": alone_gbs})
    split_fs = [f0] if f0 > 0 else []

    def measure_round(plan, used):
        m = measure_at(plan.host_fraction)
        h, d = rates_of(m)
        rounds.append({"host_fraction": plan.host_fraction, "rates_used_gbs": used,
                       "predicted_step_ms": plan.step_seconds * 1e3, "measured_step_ms": m["ms"],
                       "predicted_over_measured": plan.step_seconds * 1e3 / m["ms"],
                       "host_stream_gbs": h if plan.host_fraction > 0 else None, "hbm_split_k_gbs": d})
        return m

    for _ in range(2):
        split = plan_offload(x, host_gbs, hbm_gbs, budget, -1.0)   # the side-by-side split alone
        if any(abs(split.host_fraction - f) < 1e-3 for f in split_fs):
            break
        meas, f_cur = measure_round(split, [host_gbs, hbm_gbs, -1.0]), split.host_fraction
        split_fs.append(f_cur)
        host_gbs, hbm_gbs = rates_of(meas)
    plan = plan_offload(x, host_gbs, hbm_gbs, budget, alone_gbs)
    if abs(plan.host_fraction - f_cur) >= 1e-3:
        meas, f_cur = measure_round(plan, [host_gbs, hbm_gbs, alone_gbs]), plan.host_fraction
    elif "predicted_step_ms" not in rounds[-1]:
        rounds[-1].update({"rates_used_gbs": [host_gbs, hbm_gbs, alone_gbs],
                           "predicted_step_ms": plan.step_seconds * 1e3,
                           "predicted_over_measured": plan.step_seconds * 1e3 / meas["ms"]})
    last = rounds[-1]
    planner = {"rounds": rounds, "hbm_budget_bytes": budget if budget >= 0 else None,
               "hbm_alone_gbs": alone_gbs if alone_gbs > 0 else None, "all_hbm_step_ms": all_hbm_ms,
               "time_optimal_fraction": plan.time_optimal_fraction, "host_fraction": f_cur,
               "predicted_step_ms": last.get("predicted_step_ms"), "measured_step_ms": meas["ms"],
               "predicted_over_measured": last.get("predicted_over_measured")}
    return planner, meas


def cpu_model() -> str:
    """The host CPU's model name, as the kernel reports it."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    w = workload_for_rank(args.workload, 0, args.ctx, args.host_fraction)
    lens = kvgen.gen_seq_lens(w)
    q = kvgen.gen_q(w)
    k, v = kvgen.gen_kv(w, lens)
    threads = oracle.num_threads()
    ngroups = w.batch * w.num_kv_heads
    per_step = max(1, min(ngroups, threads))
    order = np.random.default_rng(0).permutation(ngroups)
    times, nbytes = [], []
    for i in range(args.warmup + args.steps):
        mask = np.zeros((w.batch, w.num_kv_heads), dtype=np.uint8)
        for g in order[(i * per_step) % ngroups:][:per_step]:
            mask.flat[g] = 1
        gbs, sec, _, _ = oracle_gbs(w, q, k, v, lens, mask, min_seconds=0.0)
        if i >= args.warmup:
            times.append(sec)
            nbytes.append(gbs * sec * 1e9)
    value = sum(nbytes) / sum(times) / 1e9
    total_bytes = float(lens.astype(np.int64).sum()) * w.num_kv_heads * 2 * w.head_dim * 2
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_bytes / (value * 1e9), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle", "cpu": cpu_model(),
                         "sample": f"{per_step} of {ngroups} (batch, kv head) groups per step; ms_per_step "
                                   f"extrapolates to the whole batch"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: kvgen.Workload, n: int) -> dict:
    return {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "seq_len": w.ctx if not isinstance(w.ctx, tuple) else list(w.ctx),
            "block_size": w.block_size, "kv_dtype": w.kv_dtype, "rope_base": w.rope_base,
            "placement": w.placement, "host_fraction": w.host_fraction,
            "parallelism": "replicas" if n > 1 else "single_gpu"}


# ----------------------------------------------------------------------------- our arm

def timed_steps(fn, steps, stream, flush_buf):
    """Device ms per step of fn over `steps` steps, CUDA events on `stream`.  With flush_buf, each step is
    timed alone and flush_buf (larger than L2) is written between steps, outside the events."""
    import torch
    if flush_buf is None:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        b.synchronize()
        return a.elapsed_time(b) / steps
    pairs = []
    for _ in range(steps):
        flush_buf.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        pairs.append((a, b))
    pairs[-1][1].synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs) / steps


def measure_placement(args, dkv, attn, kv, step, stream, device, b_pcie, hbm_peak, hbm_src, w_name, mode):
    """Warm-up, the timed region (nothing but the steps and the clock sampler), then a separate
    attribution pass with the library's per-kernel events.  Returns the measurements of this placement."""
    import torch
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if attn.status() != 0:
        raise RuntimeError("device status nonzero after warm-up")
    kv_bytes = kv.host_bytes + kv.dev_bytes
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device) if kv_bytes < 2 * L2_BYTES else None

    # ---- timed region: K steps, device time on the launching stream
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    ms_local = timed_steps(step, args.steps, stream, flush_buf)
    torch.cuda.synchronize(device)
    clock_info = clocks.stop()
    barrier()
    launches_per_step = attn.launches()
    ms = max_over_ranks(ms_local, device)

    # ---- attribution pass (not timed as the step): per-kernel events on each kernel's own stream
    n_prof = max(1, min(args.steps, 10))
    dkv.dkv_profile_begin(attn.handle, n_prof)
    timed_steps(step, n_prof, stream, flush_buf)
    timeline = dkv.dkv_profile_timeline(attn.handle, n_prof - 1)
    kernel_ms, kernel_counts = dkv.dkv_profile_end(attn.handle)

    kernels = []
    host_name = "staged_copy_then_hbm" if mode == "staged" else "host_stream"
    for idx, name, nbytes, bound, peak, unit_src in (
            (0, host_name, kv.host_bytes, "pcie", b_pcie, "pinned H2D cudaMemcpyAsync measured in this run"),
            (1, "hbm_split_k", kv.dev_bytes, "hbm", hbm_peak, hbm_src)):
        if kernel_counts[idx] == 0:
            continue
        avg_ms = kernel_ms[idx] / kernel_counts[idx]
        achieved = nbytes / (avg_ms * 1e-3) / 1e9
        traffic = recorded_traffic(name, w_name)
        kernels.append({"kernel": name, "bound": bound, "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "peak_source": unit_src, "avg_ms": avg_ms,
                        "algorithmic_bytes_per_launch": nbytes,
                        "traffic": traffic.get("bytes_per_launch") if traffic else None,
                        "traffic_detail": traffic})
    if kernel_counts[2]:
        kernels.append({"kernel": "merge", "avg_ms": kernel_ms[2] / kernel_counts[2]})
    names = ("host_stream", "hbm_split_k", "merge")
    tl = {n: [timeline[2 * i], timeline[2 * i + 1]] for i, n in enumerate(names) if timeline[2 * i] >= 0}
    if "host_stream" in tl and "hbm_split_k" in tl:
        h0, h1 = tl["host_stream"]
        d0, d1 = tl["hbm_split_k"]
        tl["overlap_ms"] = max(0.0, min(h1, d1) - max(h0, d0))
    return {"ms": ms, "clocks": clock_info, "launches_per_step": launches_per_step, "kernels": kernels,
            "timeline_ms": tl, "flush_buf": flush_buf, "kv_bytes": kv_bytes}


def run_dkv(args):
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    import decode_attention_host_b200 as dkv

    w = workload_for_rank(args.workload, rank, args.ctx, args.host_fraction)
    q = kvgen.gen_q(w)
    lens = kvgen.gen_seq_lens(w)
    k, v = kvgen.gen_kv(w, lens)
    placement = dkv.DKV_PLACE_PREFIX_HOST if w.placement == "prefix_host" else dkv.DKV_PLACE_RANDOM
    tq = args.queries
    planned = args.mode == "planned"

    def paged(f):
        # multi-token queries: the cache holds L + tq - 1 tokens, query i sits at position L + i
        c = dkv.PagedKV(k, v, lens, w.block_size, placement, f, w.shuffle, w.seed, device=local)
        if tq > 1:
            c.seq_lens_dev.copy_(torch.from_numpy(lens - (tq - 1)))
        return c

    kv = paged(w.host_fraction)
    attn = dkv.DecodeAttention(w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                               dkv.DKV_KV_BF16 if w.kv_dtype == kvgen.BF16 else dkv.DKV_KV_F16, w.rope_base,
                               w.batch * tq, kv.stride, device=local, host_ctas=args.host_ctas)
    keep_logical = rank == 0 and world == 1 and not args.no_cpu_baseline and args.queries == 1
    if not keep_logical and not planned:
        del k, v
    q_dev = torch.from_numpy(q).to(device)
    out = torch.empty_like(q_dev)
    stream = torch.cuda.current_stream(device)
    b_pcie = measure_pcie_gbs(device)
    peaks = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    hbm_src = "MEASURED_PEAKS.json hbm_gbs (copy, measured)" if "hbm_gbs" in peaks else "fallback 6650 GB/s"

    if tq > 1:
        q_dev = torch.from_numpy(np.random.default_rng(w.seed).standard_normal(
            (w.batch, tq, w.num_q_heads, w.head_dim)).astype(np.float32)).to(device)
        out = torch.empty_like(q_dev)
    k_stage = v_stage = None
    if args.mode == "staged":
        blk = w.num_kv_heads * w.block_size * w.head_dim
        k_stage = torch.empty(max(1, kv.host_split * blk), dtype=torch.int16, device=device)
        v_stage = torch.empty_like(k_stage)

    def step():
        if args.mode == "staged":
            attn.staged(q_dev, kv, out, k_stage, v_stage, stream)
        elif tq > 1:
            attn.multi(q_dev, kv, out, stream)
        else:
            attn(q_dev, kv, out, stream)

    meas = measure_placement(args, dkv, attn, kv, step, stream, device, b_pcie, hbm_peak, hbm_src, w.name,
                             args.mode)
    planner = None
    if planned:
        def rates_of(m):
            r = {k["kernel"]: k["achieved"] for k in m["kernels"] if "achieved" in k}
            return r.get("host_stream", b_pcie * 0.92), r.get("hbm_split_k", hbm_peak)

        def measure_at(f):
            nonlocal kv
            kv.free()
            kv = paged(f)
            return measure_placement(args, dkv, attn, kv, step, stream, device, b_pcie, hbm_peak, hbm_src, w.name,
                                     args.mode)
        x = float(meas["kv_bytes"])
        budget = args.hbm_budget_frac * x if args.hbm_budget_frac >= 0 else -1.0
        planner, meas = plan_placement(dkv.dkv_plan_offload, measure_at, rates_of, x, budget, w.host_fraction, meas)
        planner.update({"hbm_bytes_freed": float(kv.host_bytes), "hbm_bytes_used": float(kv.dev_bytes),
                        "hbm_fraction_freed": kv.host_bytes / max(1, kv.host_bytes + kv.dev_bytes)})
    ms = meas["ms"]
    flush_buf = meas["flush_buf"]

    # ---- end to end through the public API: inputs from pinned host memory, result back to the host
    e2e = None
    if not args.no_e2e:
        q_h = q_dev.cpu().pin_memory()
        lens_h = torch.from_numpy(kv.seq_lens - (tq - 1)).pin_memory()   # base lengths L
        table_h = torch.from_numpy(kv.table).pin_memory()
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        h2d = q_h.numel() * 4 + lens_h.numel() * 4 + table_h.numel() * 4
        d2h = out_h.numel() * 4

        def e2e_step():
            q_dev.copy_(q_h, non_blocking=True)
            kv.seq_lens_dev.copy_(lens_h, non_blocking=True)
            kv.table_dev.copy_(table_h, non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize(device)
        barrier()
        e2e_ms = max_over_ranks(timed_steps(e2e_step, args.steps, stream, flush_buf), device)
        e2e = {"value": None, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e2e_ms}

    if rank != 0:
        barrier()
        kv.free()
        return 0

    # ---- sampled parity: the fp64 oracle on two (batch, kv head) groups
    parity = None
    if keep_logical:
        import oracle
        mask = np.zeros((w.batch, w.num_kv_heads), dtype=np.uint8)
        mask[0, 0] = mask[-1, -1] = 1
        want = oracle.decode(q, k, v, lens, oracle.KV_BF16 if w.kv_dtype == kvgen.BF16 else oracle.KV_F16,
                             w.rope_base, group_mask=mask)
        got = out.cpu().numpy()
        rows = np.repeat(mask.astype(bool), w.group_size, axis=1)
        parity = {"groups": int(mask.sum()), "max_abs_err": float(np.abs(got[rows] - want[rows]).max()),
                  "tolerance": 2e-3}

    host_bytes, dev_bytes = kv.host_bytes, kv.dev_bytes
    total = (host_bytes + dev_bytes) * world
    value = total / (ms * 1e-3) / 1e9
    kernels = meas["kernels"]
    bw_kernels = [r for r in kernels if "bound" in r]
    dominant = max(bw_kernels, key=lambda r: r["avg_ms"]) if bw_kernels else None
    t_star_meas = max(host_bytes / (b_pcie * 1e9), dev_bytes / (hbm_peak * 1e9))
    t_star_nom = max(host_bytes / (b_pcie * 1e9), dev_bytes / (HBM_NOMINAL_GBS * 1e9))

    cpu = None
    if keep_logical:
        ngroups = w.batch * w.num_kv_heads
        mask = np.ones((w.batch, w.num_kv_heads), dtype=np.uint8)
        gbs, sec, threads, reps = oracle_gbs(w, q, k, v, lens, mask)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "cpu": cpu_model(),
               "sample": f"all {ngroups} (batch, kv head) groups of one step, run {reps} times: {sec:.1f} s"}

    if e2e is not None:
        e2e["value"] = total / (e2e["ms_per_step"] * 1e-3) / 1e9
    kv_bytes = meas["kv_bytes"]
    cfg = workload_config(w, world)
    if planned:
        cfg["host_fraction"] = planner["host_fraction"]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
        "config": dict(cfg, host_bytes=host_bytes, dev_bytes=dev_bytes, mode=args.mode,
                       query_tokens=tq,
                       l2=("inputs larger than L2: %.0f MiB of KV per step vs 126 MB L2" % (kv_bytes / 2**20)
                           if flush_buf is None else
                           "L2 flushed between timed steps (%d MiB write outside the step events): %.1f MiB of KV "
                           "per step vs 126 MB L2" % (FLUSH_BYTES >> 20, kv_bytes / 2**20))),
        "roofline": ({k2: dominant[k2] for k2 in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
                     if dominant else None),
        "roofline_kernels": kernels,
        "roofline_step": {"t_star_ms_measured_hbm": t_star_meas * 1e3, "frac_measured_hbm": t_star_meas / (ms * 1e-3),
                          "t_star_ms_nominal_hbm": t_star_nom * 1e3, "frac_nominal_hbm": t_star_nom / (ms * 1e-3),
                          "b_pcie_gbs": b_pcie, "b_hbm_measured_gbs": hbm_peak, "b_hbm_nominal_gbs": HBM_NOMINAL_GBS},
        "kernel_timeline_ms": meas["timeline_ms"],
        "e2e": e2e,
        "gpu_launches": meas["launches_per_step"] * args.steps,
        "clocks": meas["clocks"],
        "cpu_baseline": cpu,
        "parity": parity,
    }
    if planner is not None:
        line["planner"] = planner
    print(json.dumps(line), flush=True)
    barrier()
    kv.free()
    return 0


def append_bytes(w: kvgen.Workload, hidden: int, dev_stores: int, host_stores: int) -> tuple[int, int]:
    """Algorithmic bytes of one append step: (HBM bytes, host bytes).  HBM: the two weight matrices
    [Hkv*D][hidden] (16-bit), the fp32 hidden states and the K/V rows stored into device blocks; host: the K/V
    rows stored into host blocks (over PCIe)."""
    rows = w.num_kv_heads * w.head_dim
    row_bytes = 2 * rows * 2                      # one token's K and V, 16-bit
    return 2 * rows * hidden * 2 + w.batch * hidden * 4 + dev_stores * row_bytes, host_stores * row_bytes


def run_append(args):
    """--mode append: the K/V projection of each sequence's new token (hidden = Hq * D, the model width of the
    named workloads) and its store into the block holding position L - 1 of the workload's own cache, timed
    like a decode step.  HBM-bound: the weights are read once per step."""
    import torch
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist_init("nccl")
    import decode_attention_host_b200 as dkv

    w = workload_for_rank(args.workload, rank, args.ctx, args.host_fraction)
    lens = kvgen.gen_seq_lens(w)
    lmax = max(1, int(lens.max(initial=0)))
    zeros = np.zeros((w.batch, w.num_kv_heads, lmax, w.head_dim), dtype=np.uint16)   # contents do not matter here
    placement = dkv.DKV_PLACE_PREFIX_HOST if w.placement == "prefix_host" else dkv.DKV_PLACE_RANDOM
    kv = dkv.PagedKV(zeros, zeros, lens, w.block_size, placement, w.host_fraction, w.shuffle, w.seed, device=local)
    del zeros
    attn = dkv.DecodeAttention(w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                               dkv.DKV_KV_BF16 if w.kv_dtype == kvgen.BF16 else dkv.DKV_KV_F16, w.rope_base,
                               w.batch, kv.stride, device=local, host_ctas=args.host_ctas)
    hidden = w.num_q_heads * w.head_dim
    wdt = torch.bfloat16 if w.kv_dtype == kvgen.BF16 else torch.float16
    gen = torch.Generator(device=device).manual_seed(w.seed)
    x = torch.randn(w.batch, hidden, device=device, generator=gen)
    w_k = (torch.randn(w.num_kv_heads * w.head_dim, hidden, device=device, generator=gen) * hidden ** -0.5).to(wdt)
    w_v = (torch.randn(w.num_kv_heads * w.head_dim, hidden, device=device, generator=gen) * hidden ** -0.5).to(wdt)
    # the new token overwrites position L - 1, which the table covers (the timed quantity does not depend on it)
    pos = np.maximum(lens - 1, 0)
    kv.seq_lens_dev.copy_(torch.from_numpy(pos.astype(np.int32)))
    ids = kv.table[np.arange(w.batch), pos // w.block_size]
    live = lens > 0
    host_stores = int(np.count_nonzero(live & (ids < kv.host_split)))
    dev_stores = int(np.count_nonzero(live)) - host_stores
    hbm_bytes, host_bytes = append_bytes(w, hidden, dev_stores, host_stores)
    stream = torch.cuda.current_stream(device)

    def step():
        attn.append(x, w_k, w_v, kv, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if attn.status() != 0:
        raise RuntimeError("device status nonzero after warm-up")
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)   # the weights fit in L2
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize(device)
    clocks.start()
    ms_local = timed_steps(step, args.steps, stream, flush_buf)
    torch.cuda.synchronize(device)
    clock_info = clocks.stop()
    barrier()
    ms = max_over_ranks(ms_local, device)
    peaks = measured_peaks()
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
    hbm_src = "MEASURED_PEAKS.json hbm_gbs (copy, measured)" if "hbm_gbs" in peaks else "fallback 6650 GB/s"
    achieved = hbm_bytes / (ms * 1e-3) / 1e9
    total = (hbm_bytes + host_bytes) * world
    if rank == 0:
        line = {
            "metric": "KV append: K/V projection of the new token and its store, µs/step & GB/s", "value":
            total / (ms * 1e-3) / 1e9, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "us_per_step": ms * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp32", "data": "synthetic",
            "config": dict(workload_config(w, world), mode="append", hidden=hidden, hbm_bytes=hbm_bytes,
                           host_bytes=host_bytes, host_stores=host_stores, dev_stores=dev_stores,
                           l2="L2 flushed between timed steps (%d MiB write outside the step events): "
                              "%.1f MiB of weights per step" % (FLUSH_BYTES >> 20, hbm_bytes / 2**20)),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "peak_source": hbm_src, "traffic": None},
            "e2e": None, "gpu_launches": args.steps, "clocks": clock_info, "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    kv.free()
    attn.close()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    rc = run_append(args) if args.mode == "append" else run_dkv(args)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
