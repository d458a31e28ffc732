#!/usr/bin/env python
"""Benchmark one exact-attention training step on B200: forward + backward.

Workload: B=8, H=16, N=2048, d=128, causal, bf16 (the training-step
configuration). Inputs are synthetic (seeded iid N(0,1) -> bf16). A step is the
whole hot path through the library's public API: attn_fwd then attn_bwd. The
metric is attention TFLOP/s, with algorithmic FLOPs of 4*B*H*N^2*d/2 forward
and 2.5x that backward. Masked (skipped) tiles are not counted.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU. Each rank runs its own shard
of the batch (weak scaling, no data-path collective). The step time is the
maximum over ranks. Rank 0 prints one JSON line.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(rank 0 only), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "attention TFLOP/s (bf16 causal fwd/bwd) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = workloads.C5
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
CSRC = os.path.join(ROOT, "exact_attention_105_b200", "csrc")


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip the forward-only target workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["step", "fwd"], default="step",
                    help="step: forward + backward (default); fwd: forward only")
    ap.add_argument("--workload", default=None,
                    help="workload name from workloads.py (default: the training-step config)")
    return ap.parse_args()


def pick_workload(args):
    if args.workload is None:
        return WORKLOAD
    for w in workloads.ALL:
        if w.name == args.workload:
            return w
    sys.exit(f"unknown workload {args.workload!r}; choose from {[w.name for w in workloads.ALL]}")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    return {"bf16_tflops": FALLBACK_PEAKS["bf16_tflops"],
            "bf16_tflops_sustained": FALLBACK_PEAKS["bf16_tflops"],
            "hbm_gbs": FALLBACK_PEAKS["hbm_gbs"], "source": "fallback"}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources and this workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    if t.get("kernel_source_sha") != kernel_source_sha():
        return None
    k = t.get("kernels", {}).get(kernel)
    if not k or k.get("workload") != workload:
        return None
    return k.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler(threading.Thread):
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, device_index: int, period_s: float = 0.01):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._halt = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: record why, keep benchmarking
            self.err = str(e)

    def run(self):
        if not self.ok:
            return
        get_reasons = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._halt.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= int(get_reasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        self.join(timeout=2)

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "")}
        s = sorted(self.samples)
        med = s[len(s) // 2] if s else None
        reasons = [name for bit, name in REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(s)}


# ------------------------------------------------------------------ oracle timing

def oracle_sample_step(q, k, v, do, w, b, h, rows):
    """Oracle forward + backward for the last `rows` query rows of head (b, h)
    against all keys. With bottom-right causal alignment this is exactly the
    causal attention of those rows. Returns the algorithmic FLOPs covered."""
    import oracle
    N, d = w.N, w.d
    hk = h // w.group
    qs = oracle.to_f64(q[b, h, N - rows:])
    ks, vs = oracle.to_f64(k[b, hk]), oracle.to_f64(v[b, hk])
    dos = oracle.to_f64(do[b, h, N - rows:])
    oracle.attention_head(qs, ks, vs, w.scale, w.causal)
    oracle.attention_head_bwd(qs, ks, vs, dos, w.scale, w.causal)
    if w.causal:
        pairs = sum(i + 1 for i in range(N - rows, N))
    else:
        pairs = rows * N
    return pairs * 14.0 * d          # 4d forward + 10d backward FLOPs per visible pair


def pick_rows(q, k, v, do, w, budget_s):
    """Query-row count whose oracle step takes about budget_s seconds."""
    t0 = time.perf_counter()
    oracle_sample_step(q, k, v, do, w, 0, 0, 128)
    dt = max(time.perf_counter() - t0, 1e-3)
    rows = int(128 * budget_s / dt)
    return max(16, min(w.N, rows))


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 0) for i in info if i.get("user_api") == "blas"), default=0)
        if n:
            return n
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_baseline(w, inputs, steps, per_step_s, warmup=1):
    q, k, v, do = inputs
    rows = pick_rows(q, k, v, do, w, per_step_s)
    for s in range(warmup):
        oracle_sample_step(q, k, v, do, w, 0, s % w.Hq, rows)
    flops = 0.0
    t0 = time.perf_counter()
    for s in range(steps):
        b, h = s % w.B, (s * 5) % w.Hq
        flops += oracle_sample_step(q, k, v, do, w, b, h, rows)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"float64 numpy oracle, fwd+bwd of the last {rows} query rows of one head "
                      f"(all {w.N} keys, causal) per step, {steps} steps over rotating heads",
            "seconds": dt, "rows_per_step": rows, "gflops": flops / dt / 1e9,
            "blas": blas_info()}


def blas_info():
    """The BLAS library numpy uses and its thread count, as threadpoolctl reports it."""
    try:
        from threadpoolctl import threadpool_info
        libs = [f"{d.get('internal_api')} {d.get('version')} ({d.get('num_threads')} threads)"
                for d in threadpool_info() if d.get("user_api") == "blas"]
        return "; ".join(libs) or None
    except Exception:   # informational only
        return None


# ------------------------------------------------------------------ distributed

def rank_workload(w, rank: int):
    """The shard a rank runs: the same shape, its own seed (data parallel)."""
    return workloads.Workload(w.name, w.B, w.Hq, w.Hkv, w.N, w.d, w.causal, q_mult=w.q_mult,
                              backward=True, seed=w.seed + rank)


def max_over_ranks(x: float, dist, device) -> float:
    """The slowest rank's value (a no-op for one process)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step: float, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job TFLOP/s: the work every rank did over the slowest rank's time."""
    return flops_per_step * steps * world / (elapsed_ms / 1e3) / 1e12


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            sys.exit(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes")
    return world, rank, local


def config_dict(w, world):
    return {"workload": w.name, "B_per_gpu": w.B, "global_batch": w.B * world, "Hq": w.Hq,
            "Hkv": w.Hkv, "seq_len": w.N, "head_dim": w.d, "causal": w.causal,
            "parallelism": f"dp{world}" if world > 1 else "single_gpu",
            "l2": f"no flush: step working set {8 * w.B * w.Hq * w.N * w.d * 2 / 2**20:.0f} MiB "
                  "(q,k,v,o,dO,dq,dk,dv) exceeds the 126 MB L2"}


def run_reference(args):
    world, rank, _ = dist_setup(args)
    if rank != 0:
        return 0
    w = WORKLOAD
    inputs = workloads.make_inputs(w)
    budget = 120.0
    per_step = max(0.05, budget / max(1, args.steps + args.warmup))
    cb = oracle_baseline(w, inputs, args.steps, per_step, warmup=args.warmup)
    line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": cb["seconds"] * 1e3 / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded iid N(0,1) -> bf16 inputs, upcast to float64)",
            "config": dict(config_dict(w, args.gpus), mode="step"),
            "cpu_baseline": {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours

def visible_pairs(n_q, n_k, causal, window=(-1, -1)):
    """Number of (query, key) pairs the mask keeps for one head: bottom-right
    alignment, off = Nk - Nq; window (left, right), negative = unbounded."""
    import numpy as np
    i = np.arange(n_q, dtype=np.int64)
    off = n_k - n_q
    lo = i + off - window[0] if window[0] >= 0 else np.zeros_like(i)
    hi = np.full_like(i, n_k - 1)
    if causal:
        hi = np.minimum(hi, i + off)
    if window[1] >= 0:
        hi = np.minimum(hi, i + off + window[1])
    return int(np.maximum(0, np.minimum(n_k - 1, hi) - np.maximum(0, lo) + 1).sum())


def variant_targets(ea, torch, peak, iters=5, warmup=2):
    """Forward + backward TFLOP/s (14 d FLOPs per visible pair) of the variant
    paths: sliding window, Nq != Nk, softcapping and a packed varlen batch."""
    import numpy as np
    out = []

    def timed(name, step, pairs, d):
        for _ in range(warmup):
            step()
        ea.attn_check_status()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            step()
        b.record()
        torch.cuda.synchronize()
        ea.attn_check_status()
        ms = a.elapsed_time(b) / iters
        tf = 14.0 * d * pairs / ms / 1e9
        out.append({"workload": name, "ms": ms, "tflops": tf, "frac_of_measured_peak": tf / peak})

    fixed = [("swa1024_causal_B4_H16_N4096_d128", 4, 16, 4096, 4096, True, (1024, 0), 0.0),
             ("chunk_causal_B4_H16_Nq2048_Nk8192_d128", 4, 16, 2048, 8192, True, (-1, -1), 0.0),
             ("softcap50_causal_B4_H16_N4096_d128", 4, 16, 4096, 4096, True, (-1, -1), 50.0)]
    for name, B, H, Nq, Nk, causal, win, cap in fixed:
        q, k, v, do = (t.cuda() for t in workloads.make_inputs_qk(B, H, H, Nq, Nk, 128, seed=7))
        o, lse = torch.empty_like(q), torch.empty((B, H, Nq), dtype=torch.float32, device="cuda")
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(ea.attn_bwd_workspace_size(B, H, Nq, 128), dtype=torch.uint8,
                         device="cuda")

        def step():
            ea.attn_fwd_masked(q, k, v, o, lse, causal=causal, window=win, softcap=cap)
            ea.attn_bwd_masked(q, k, v, o, lse, do, dq, dk, dv, ws, causal=causal, window=win,
                               softcap=cap)
        timed(name, step, B * H * visible_pairs(Nq, Nk, causal, win), 128)
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()

    lens = [int(x) for x in np.random.default_rng(0).integers(256, 4097, 16)]
    H = 16
    q, k, v, do, cq, ck = (t.cuda() for t in workloads.make_packed_inputs(lens, lens, H, H, 128,
                                                                          seed=8))
    o, lse = torch.empty_like(q), torch.empty((H, q.shape[0]), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    mx = max(lens)
    ws = torch.empty(ea.attn_bwd_workspace_size(len(lens), H, mx, 128), dtype=torch.uint8,
                     device="cuda")

    def vstep():
        ea.attn_fwd_varlen(q, k, v, cq, ck, mx, mx, o, lse, causal=True)
        ea.attn_bwd_varlen(q, k, v, o, lse, do, cq, ck, mx, mx, dq, dk, dv, ws, causal=True)
    timed(f"varlen16_causal_H16_d128_total{sum(lens)}", vstep,
          H * sum(visible_pairs(n, n, True) for n in lens), 128)
    del q, k, v, do, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def small_target(ea, torch, w, hbm_gbs, iters=200, warmup=20):
    """The small configurations are latency-bound. Reports microseconds per
    forward and per forward + backward, called through the API from Python
    (host overhead included) and replayed from a CUDA graph that captured the
    same calls (device time only), plus the forward's HBM byte rate (q, k, v
    read and o, lse written once) from the graph timing. Each figure averages
    200 back-to-back calls: a call costs microseconds, so fewer calls let one
    host hiccup move the mean by tens of percent."""
    q, k, v, do = (t.cuda() for t in workloads.make_inputs(w, with_grad_out=True))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, ea.attn_bwd_workspace_size(w.B, w.Hq, w.N, w.d)), dtype=torch.uint8,
                     device="cuda")

    def fwd():
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)

    def fwd_bwd():
        fwd()
        ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, scale=w.scale, causal=w.causal)

    def timed(fn):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize()
        ea.attn_check_status()
        return a.elapsed_time(b) / iters * 1e3

    res = {"workload": w.name}
    for name, fn in (("fwd", fwd), ("fwd_bwd", fwd_bwd)):
        for _ in range(warmup):
            fn()
        res[f"{name}_api_us"] = timed(fn)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream().wait_stream(side)
        with torch.cuda.graph(g, capture_error_mode="relaxed"):
            fn()
        res[f"{name}_graph_us"] = timed(g.replay)
        del g
    fwd_bytes = 2.0 * w.d * (2 * w.B * w.Hq * w.N + 2 * w.B * w.Hkv * w.N) + 4.0 * w.B * w.Hq * w.N
    res["fwd_hbm_gbs"] = fwd_bytes / (res["fwd_graph_us"] * 1e-6) / 1e9
    res["fwd_hbm_frac_of_measured"] = res["fwd_hbm_gbs"] / hbm_gbs
    res["fwd_bwd_tflops"] = (w.fwd_flops() + w.bwd_flops()) / (res["fwd_bwd_graph_us"] * 1e-6) / 1e12
    return res


def fwd_target(ea, torch, w, iters=10, warmup=3):
    """Forward-only TFLOP/s on one workload (inputs resident, > L2)."""
    q, k, v = (t.cuda() for t in workloads.make_inputs(w, with_grad_out=False))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    for _ in range(warmup):
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
    ea.attn_check_status()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record()
    for _ in range(iters):
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
    b.record()
    torch.cuda.synchronize()
    ea.attn_check_status()
    ms = a.elapsed_time(b) / iters
    del q, k, v, o, lse
    return {"workload": w.name, "ms": ms, "tflops": w.fwd_flops() / ms / 1e9}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import exact_attention_105_b200 as ea

    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w = pick_workload(args)
    fwd_only = args.mode == "fwd"
    w_rank = rank_workload(w, rank)
    peaks = load_peaks()
    host = workloads.make_inputs(w_rank)
    q, k, v, do = (t.cuda() for t in host)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(ea.attn_bwd_workspace_size(w.B, w.Hq, w.N, w.d), dtype=torch.uint8,
                     device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
        if not fwd_only:
            ea.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, scale=w.scale, causal=w.causal)

    for _ in range(max(3, args.warmup)):
        step()
    ea.attn_check_status()

    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ea.profile_reset()
    ea.profile_enable(True)
    sampler.start()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev0, ev1 = evs[0], evs[-1]
    ev0.record(stream)
    for n_step in range(args.steps):
        step()
        evs[n_step + 1].record(stream)
    torch.cuda.synchronize()
    sampler.stop()
    ea.profile_enable(False)
    if world > 1:
        dist.barrier()
    ea.attn_check_status()
    elapsed = max_over_ranks(ev0.elapsed_time(ev1), dist, "cuda")
    per_step = sorted(evs[n].elapsed_time(evs[n + 1]) for n in range(args.steps))
    pick = lambda f: per_step[min(len(per_step) - 1, int(f * len(per_step)))]  # noqa: E731
    step_dist = {"p10_ms": pick(0.10), "median_ms": pick(0.50), "p90_ms": pick(0.90),
                 "rank": rank}
    prof = ea.profile_read()
    launches = sum(n for n, _ in prof.values())
    # Forward and backward separately, from the same timed region.
    fwd_ms = prof["fwd_kernel"][1] / max(1, prof["fwd_kernel"][0])
    bwd_ms = sum(prof[k2][1] for k2 in ("bwd_pre_kernel", "bwd_dkdv_kernel", "bwd_dq_kernel")) \
        / max(1, prof["bwd_dkdv_kernel"][0])
    split = {"fwd_ms": fwd_ms, "fwd_tflops": w.fwd_flops() / fwd_ms / 1e9}
    if not fwd_only:
        split.update({"bwd_ms": bwd_ms, "bwd_tflops": w.bwd_flops() / bwd_ms / 1e9})

    flops_step = w.fwd_flops() + (0.0 if fwd_only else w.bwd_flops())
    value = job_throughput(flops_step, args.steps, world, elapsed)

    # Roofline of the dominant kernel (largest share of the timed region).
    dom = max(prof, key=lambda kname: prof[kname][1])
    n_l, ms_tot = prof[dom]
    avg_ms = ms_tot / max(1, n_l)
    half_pairs = w.B * w.Hq * w.N * w.N / 2.0           # visible (query, key) pairs, causal
    pairs = half_pairs if w.causal else 2 * half_pairs
    alg = {"fwd_kernel": ("tensor", 4.0 * w.d * pairs),       # QK^T + PV
           "bwd_dkdv_kernel": ("tensor", 8.0 * w.d * pairs),  # S^T, dP^T, dV, dK
           "bwd_dq_kernel": ("tensor", 6.0 * w.d * pairs),    # S, dP, dQ
           "bwd_pre_kernel": ("hbm", 2.0 * 2 * w.B * w.Hq * w.N * w.d + 8.0 * w.B * w.Hq * w.N)}
    bound, work = alg[dom]
    if bound == "tensor":
        achieved = work / (avg_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = work / (avg_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    roofline = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": ncu_traffic(dom, w.name),
                "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json burst figure)"
                if peaks["source"] == "measured" else "fallback",
                "algorithmic_per_launch": work}
    kernels = {kn: {"launches": n, "avg_ms": (ms / n if n else None),
                    "share": (ms / sum(m for _, m in prof.values()) if n else 0.0)}
               for kn, (n, ms) in prof.items()}

    # End to end through the public API from pinned host buffers: every step
    # copies q, k, v, dO in, runs forward + backward, and copies o, lse, dq,
    # dk and dv out (forward mode: q, k, v in; o, lse out). Copies in,
    # compute and copies out run on three streams over two sets of device
    # tensors: step
    # i+1's inputs cross PCIe while step i computes and step i-1's results
    # come back. Events order each set's reuse.
    pin = [t.pin_memory() for t in host]
    n_in = 3 if fwd_only else 4
    e2e_steps = max(3, min(args.steps, 20))
    sets = []
    for _ in range(2):
        st = {"in": [torch.empty_like(t) for t in (q, k, v, do)[:n_in]],
              "o": torch.empty_like(o), "lse": torch.empty_like(lse)}
        # Every output of the step leaves the device: o and lse, and in step
        # mode dq, dk and dv as well.
        st["out"] = [st["o"], st["lse"]] if fwd_only else \
            [st["o"], st["lse"], torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)]
        sets.append(st)
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in sets[0]["out"]]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def compute(st):
        qb, kb, vb = st["in"][:3]
        ea.attn_fwd(qb, kb, vb, st["o"], st["lse"], scale=w.scale, causal=w.causal,
                    stream=s_comp)
        if not fwd_only:
            dq_b, dk_b, dv_b = st["out"][2:]
            ea.attn_bwd(qb, kb, vb, st["o"], st["lse"], st["in"][3], dq_b, dk_b, dv_b, ws,
                        scale=w.scale, causal=w.causal, stream=s_comp)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for sx in (s_in, s_comp, s_out):
        sx.wait_stream(stream)
    for i in range(e2e_steps):
        bi = i % 2
        st = sets[bi]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(comp_done[bi])      # compute of step i-2 read this set
            for dst, src in zip(st["in"], pin):
                dst.copy_(src, non_blocking=True)
            in_done[bi].record(s_in)
        s_comp.wait_event(in_done[bi])
        if i >= 2:
            s_comp.wait_event(out_done[bi])         # step i-2's results have left this set
        compute(st)
        comp_done[bi].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[bi])
            for dst, src in zip(host_out, st["out"]):
                dst.copy_(src, non_blocking=True)
            out_done[bi].record(s_out)
    stream.wait_stream(s_out)
    stream.wait_stream(s_comp)
    stream.wait_stream(s_in)
    e1.record(stream)
    torch.cuda.synchronize()
    ea.attn_check_status()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, "cuda")
    h2d = sum(t.numel() * t.element_size() for t in pin[:n_in])
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    del sets
    e2e = {"value": job_throughput(flops_step, e2e_steps, world, e2e_ms), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
           "overlap": "three streams (copy in / compute / copy out), two device buffer sets"}

    extra = None
    variants = None
    small = None
    if not args.no_extra and rank == 0 and not fwd_only:
        del pin, host_out
        torch.cuda.empty_cache()
        extra = []
        for tw in (workloads.C3_CAUSAL, workloads.C3_FULL, workloads.C3_STRESS, workloads.C4):
            r = fwd_target(ea, torch, tw)
            r["frac_of_measured_peak"] = r["tflops"] / peaks["bf16_tflops"]
            extra.append(r)
        variants = variant_targets(ea, torch, peaks["bf16_tflops"])
        small = [small_target(ea, torch, tw, peaks["hbm_gbs"]) for tw in (workloads.C1, workloads.C2)]

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not fwd_only:
        cpu = oracle_baseline(w, host, steps=3, per_step_s=4.0)
        cpu = {k2: cpu[k2] for k2 in ("value", "unit", "cores", "kind", "sample", "seconds",
                                    "gflops", "blas")}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    clocks = sampler.summary()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": elapsed / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded iid N(0,1) -> bf16)",
            "config": dict(config_dict(w, world), mode=args.mode),
            "frac_of_peak": value / peaks["bf16_tflops"],
            "frac_of_nominal_2250": value / 2250.0,
            "step_distribution": step_dist, "fwd_bwd_split": split,
            "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "fwd_targets": extra,
            "variants_fwd_bwd": variants, "small_configs": small,
            "kernel_source_sha": kernel_source_sha()}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
