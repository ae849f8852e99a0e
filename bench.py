#!/usr/bin/env python
"""Exact attention forward + backward on B200: throughput against the tensor roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME|all] [--impl ours|reference]

One step = the whole hot path over one batch of synthetic inputs already
resident in device memory: fa_fwd (O, LSE), fa_bwd_prep (D, log2 LSE, dQ := 0)
and fa_bwd_main (dQ, dK, dV).  `value` is whole-job TFLOP/s under the FLOP
convention 4*B*H*N^2*d forward, 2.5x that backward, halved under the causal
mask.  Kernels are timed with CUDA events on the launching stream; with N > 1
ranks each rank runs its own batch (weak scaling, no collective on the data
path) and the step time is the max over ranks.

--impl reference runs the fp64 CPU oracle on the host cores instead (one
head of the workload per step) and prints the same JSON line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOPS on 1 B200 and fraction of dense BF16 tensor peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "c4_bf16_4x16x4096x128_causal"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ ranks

def rank_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init_dist(world: int, backend: str, device=None):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = {"backend": backend, "timeout": datetime.timedelta(seconds=120)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(**kw)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (a timing collective, not a data-path one)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch of the same shape (weak scaling)."""
    return base_seed + 7919 * rank


# ------------------------------------------------------------------ peaks / clocks

def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded in profiles/traffic.txt for this kernel and
    workload, or None if absent or if the kernel's sources changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    for line in lines:
        if not line.strip() or line.startswith("#"):
            continue
        k, wl, sha, nbytes, files, _ = line.split()[:6]
        if k != kernel or wl != workload:
            continue
        h = hashlib.sha256()
        try:
            for f in files.split(","):
                with open(os.path.join(ROOT, f), "rb") as fh:
                    h.update(fh.read())
        except OSError:
            return None
        return int(nbytes) if h.hexdigest().startswith(sha) else None
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "of measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "of fallback"


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with nvidia-smi while running."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str, period_ms: int = 100):
        self.uuid = uuid
        self.period_ms = period_ms
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=5)
        sm, smax, power, reasons = [], [], [], set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9 or (self.uuid and parts[0] != self.uuid):
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names[1:], parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(w, heads: int, seed: int):
    """fp64 oracle forward + backward on `heads` heads of workload w; returns (seconds, flops, threads)."""
    from exact_io_aware_53_b200.workloads import make_inputs
    from oracle import oracle
    x = make_inputs(w, seed=seed, B=1, H=heads)
    q, k, v, do = (x[n] for n in ("q", "k", "v", "do"))
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, w.scale, w.causal)
    if w.backward:
        # the oracle's one-head backward spreads a head's rows over the threads
        for h in range(heads):
            oracle.attn_bwd_head(q[0, h], k[0, h], v[0, h], do[0, h], w.scale, w.causal)
    dt = time.perf_counter() - t0
    per_head = (w.flops_fwd() + (w.flops_bwd() if w.backward else 0.0)) / (w.B * w.H)
    return dt, per_head * heads, oracle.num_threads()


def cpu_baseline(w, seed: int, budget_s: float = 10.0):
    dt1, fl1, thr = oracle_sample(w, 1, seed)
    extra = max(0, min(int(budget_s / max(dt1, 1e-3)) - 1, w.B * w.H - 1))
    dt, fl = dt1, fl1
    if extra:
        dt2, fl2, _ = oracle_sample(w, extra, seed + 1)
        dt, fl = dt + dt2, fl + fl2
    heads = 1 + extra
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": "%d of %d heads (B=1, N=%d, d=%d, causal=%s), fwd%s, fp64, %.1f s" % (
                heads, w.B * w.H, w.N, w.d, w.causal, "+bwd" if w.backward else "", dt)}


def run_reference(args, w):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    for i in range(args.warmup):
        oracle_sample(w, 1, w.seed + i)
    times = []
    flops = 0.0
    thr = 1
    for i in range(args.steps):
        dt, fl, thr = oracle_sample(w, 1, w.seed + 100 + i)
        times.append(dt)
        flops = fl
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms / 1e3) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": 1, "H": 1, "N": w.N, "d": w.d, "causal": w.causal,
                       "sample": "one head per step", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": "one head of %s per step (fwd%s, fp64)" % (
                                 w.name, "+bwd" if w.backward else "")},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def run_ours(args, w, print_line=True):
    import torch
    from exact_io_aware_53_b200 import fa
    from exact_io_aware_53_b200.workloads import make_inputs

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl", torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    x = make_inputs(w, seed=rank_seed(w.seed, rank))
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    B, H, N, d = w.B, w.H, w.N, w.d
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    ws = torch.empty(max(1, fa.bwd_workspace_bytes(B, H, N, d)), dtype=torch.uint8, device=dev)
    scale, causal = w.scale, w.causal

    launches = [0]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rc = fa.fwd_raw(q, k, v, o, lse, scale, causal)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_fwd")
        if not w.backward:
            if ev is not None:
                ev[1].record(stream)
            return
        if ev is not None:
            ev[1].record(stream)
        rc = fa.bwd_prep_raw(o, lse, do, dq, ws)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_bwd_prep")
        if ev is not None:
            ev[2].record(stream)
        rc = fa.bwd_main_raw(q, k, v, do, dq, dk, dv, ws, scale, causal)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_bwd_main")
        if ev is not None:
            ev[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after warm-up: %s" % fa.status_string(st))

    # inputs smaller than twice L2 would stay cached from one step to the next:
    # then L2 is flushed (a write of twice its size) before each timed step,
    # outside that step's events, and the step time is the mean of the steps'
    # own event intervals
    in_bytes = (4 if w.backward else 3) * B * H * N * d * 2
    l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 << 20) or (126 << 20))
    flush = None
    if in_bytes < 2 * l2_bytes:
        flush = torch.empty(2 * l2_bytes // 4, dtype=torch.float32, device=dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(float(i))
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after timing: %s" % fa.status_string(st))
    timed_launches = launches[0]

    if flush is None:
        ms_local = t_start.elapsed_time(t_end) / args.steps
    else:
        last = 3 if w.backward else 1
        ms_local = statistics.mean(e[0].elapsed_time(e[last]) for e in evs)
    ms = max_over_ranks(ms_local, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    prep_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) if w.backward else 0.0
    main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs) if w.backward else 0.0
    flops_step = w.flops_fwd() + (w.flops_bwd() if w.backward else 0.0)
    value = world * flops_step / (ms / 1e3) / 1e12

    peaks, peak_src = load_peaks()
    long_region = ms * args.steps > 500.0
    peak_key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    if w.backward:
        dom_name, dom_ms, dom_flops = "bwd_main", main_ms, w.flops_bwd()
    else:
        dom_name, dom_ms, dom_flops = "fwd", fwd_ms, w.flops_fwd()
    achieved = dom_flops / (dom_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": dom_name, "achieved": achieved, "peak": peak, "unit": UNIT,
                "frac": achieved / peak, "peak_source": "%s %s" % (peak_key, peak_src),
                "frac_of_burst": achieved / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
                "algorithmic_flops_per_launch": dom_flops, "ms_per_launch": dom_ms,
                "traffic": measured_traffic(dom_name, w.name), "traffic_unit": "bytes per launch (ncu dram read+write)"}
    fwd_tflops = w.flops_fwd() / (fwd_ms / 1e3) / 1e12
    kernels = {"fwd": {"ms": fwd_ms, "tflops": fwd_tflops, "frac": fwd_tflops / peak}}
    if w.backward:
        bwd_tflops = w.flops_bwd() / ((prep_ms + main_ms) / 1e3) / 1e12
        kernels["bwd_prep"] = {"ms": prep_ms}
        kernels["bwd_main"] = {"ms": main_ms, "tflops": achieved, "frac": achieved / peak}
        kernels["bwd_total"] = {"ms": prep_ms + main_ms, "tflops": bwd_tflops, "frac": bwd_tflops / peak}

    # ---- end to end through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, w, fa, x, dev, stream, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, seed=w.seed)

    if flush is None:
        l2_note = "inputs larger than L2 (q,k,v,dO = %.0f MB per GPU)" % (in_bytes / 1e6)
    else:
        l2_note = ("L2 flushed before each timed step (inputs %.0f MB per GPU, below twice L2); step time = "
                   "mean of the steps' own event intervals" % (in_bytes / 1e6))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "backward": w.backward, "global_batch": B * world, "seq_len": N,
                       "parallelism": "dp%d (independent batches per GPU, no collective)" % world,
                       "l2": l2_note},
            "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": timed_launches, "clocks": clocks}
    if rank == 0 and print_line:
        print(json.dumps(line), flush=True)
    return line


def run_e2e(args, w, fa, x, dev, stream, world):
    import torch
    B, H, N, d = w.B, w.H, w.N, w.d
    E, R = B * H * N * d, B * H * N
    hq, hk, hv, hdo = (x[n].pin_memory() for n in ("q", "k", "v", "do"))
    outs = {"o": torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory(),
            "lse": torch.empty((B, H, N), dtype=torch.float32).pin_memory()}
    if w.backward:
        for n in ("dq", "dk", "dv"):
            outs[n] = torch.empty((B, H, N, d), dtype=torch.float32).pin_memory()
    arena = torch.empty(fa.attention_host_arena_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    if not w.backward:
        return None
    steps = max(3, min(args.steps, 20))
    for _ in range(2):
        fa.attention_host(hq, hk, hv, hdo, arena, outs, w.causal, w.scale)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        fa.attention_host(hq, hk, hv, hdo, arena, outs, w.causal, w.scale)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after e2e: %s" % fa.status_string(st))
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    flops = w.flops_fwd() + w.flops_bwd()
    return {"value": world * flops / (ms / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": 4 * E * 2, "d2h_bytes_per_step": E * 2 + R * 4 + 3 * E * 4,
            "steps": steps, "api": "fa_attention_host (pinned host buffers)"}


# ------------------------------------------------------------------ decode (split-KV)

DECODE_METRIC = "split-KV decode forward: HBM GB/s (q, k, v read + o, lse written) on 1 B200"
DECODE_UNIT = "GB/s"


def decode_oracle_sample(w, heads: int, seed: int):
    """fp64 oracle rectangular forward on `heads` heads of decode workload w;
    returns (seconds, algorithmic bytes of those heads, threads)."""
    from exact_io_aware_53_b200.workloads import make_decode_inputs
    from oracle import oracle
    x = make_decode_inputs(w, seed=seed, B=1, H=heads)
    t0 = time.perf_counter()
    oracle.attn_fwd_rect(x["q"], x["k"], x["v"], w.scale, w.causal)
    dt = time.perf_counter() - t0
    return dt, w.bytes_min() / (w.B * w.H) * heads, oracle.num_threads()


def decode_cpu_baseline(w, seed: int, budget_s: float = 10.0):
    dt1, b1, thr = decode_oracle_sample(w, 1, seed)
    heads = max(1, min(int(budget_s / max(dt1, 1e-3)), w.B * w.H))
    dt, by, _ = decode_oracle_sample(w, heads, seed + 1)
    return {"value": by / dt / 1e9, "unit": DECODE_UNIT, "cores": thr, "kind": "oracle",
            "sample": "%d of %d heads (Nq=%d, Nk=%d, d=%d, causal=%s), fp64, %.2f s" % (
                heads, w.B * w.H, w.Nq, w.Nk, w.d, w.causal, dt)}


def run_reference_decode(args, w):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    heads = min(8, w.B * w.H)
    for i in range(args.warmup):
        decode_oracle_sample(w, heads, w.seed + i)
    times, by, thr = [], 0.0, 1
    for i in range(args.steps):
        dt, by, thr = decode_oracle_sample(w, heads, w.seed + 100 + i)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = by / (ms / 1e3) / 1e9
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": 1, "H": heads, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
                       "causal": w.causal, "sample": "%d heads per step" % heads, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": DECODE_UNIT, "cores": thr, "kind": "oracle",
                             "sample": "%d heads of %s per step (fp64)" % (heads, w.name)},
            "e2e": {"value": value, "unit": DECODE_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args, w):
    """One step = fa_fwd_splitkv over the whole batch (range kernel + merge
    kernel) with q and the key/value cache resident in device memory."""
    import torch
    from exact_io_aware_53_b200 import fa
    from exact_io_aware_53_b200.workloads import make_decode_inputs

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl", torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    x = make_decode_inputs(w, seed=rank_seed(w.seed, rank))
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    B, H, Nq, Nk, d = w.B, w.H, w.Nq, w.Nk, w.d
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    n_split = args.n_split
    ws = torch.empty(max(16, fa.splitkv_workspace_bytes(B, H, Nq, Nk, d, n_split)), dtype=torch.uint8, device=dev)
    launches = [0]

    def step():
        rc = fa.fwd_splitkv_raw(q, k, v, o, lse, ws, w.scale, w.causal, n_split)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_fwd_splitkv")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after warm-up: %s" % fa.status_string(st))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after timing: %s" % fa.status_string(st))
    ms_local = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms = max_over_ranks(ms_local, world, dev)
    by = w.bytes_min()
    value = world * by / (ms / 1e3) / 1e9
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    achieved = by / (ms_local / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": "fa_fwd_splitkv (range + merge kernels)", "achieved": achieved,
                "peak": peak, "unit": DECODE_UNIT, "frac": achieved / peak, "peak_source": "hbm_gbs %s" % peak_src,
                "algorithmic_bytes_per_launch": by, "ms_per_launch": ms_local,
                "traffic": measured_traffic("decode", w.name),
                "traffic_unit": "bytes per launch (ncu dram read+write)"}

    # end to end: the query comes from pinned host memory and O, LSE go back
    # each step; the key/value cache stays resident (it is the decoder's state)
    e2e = None
    if not args.no_e2e:
        hq = x["q"].pin_memory()
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        steps = max(3, min(args.steps, 50))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        e2e = {"value": world * by / (ems / 1e3) / 1e9, "unit": DECODE_UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": hq.numel() * hq.element_size(),
               "d2h_bytes_per_step": ho.numel() * ho.element_size() + hl.numel() * hl.element_size(),
               "steps": steps, "api": "fa.fwd_splitkv_raw with q from and o, lse to pinned host memory; "
                                      "key/value cache resident on the device"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = decode_cpu_baseline(w, seed=w.seed)
    ranges = (Nk + 127) // 128 if n_split > (Nk + 127) // 128 else n_split
    line = {"metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "Nq": Nq, "Nk": Nk, "d": d, "causal": w.causal,
                       "n_split": ranges if n_split else "library choice",
                       "parallelism": "dp%d (independent batches per GPU, no collective)" % world,
                       "l2": "inputs larger than L2 (k, v = %.0f MB per GPU)" % (B * H * Nk * d * 4 / 1e6)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches[0], "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return line


def sized_oracle_sample(sample, max_heads: int, budget_s: float = 10.0):
    """Run `sample(heads)` -> (seconds, work, threads) once on one head, then on as
    many heads as fit the time budget (at most max_heads); returns the larger run."""
    dt, work, thr = sample(1)
    heads = max(1, min(max_heads, int(budget_s / max(dt, 1e-3))))
    if heads > 1:
        dt, work, thr = sample(heads)
    return dt, work, thr, heads


# ------------------------------------------------------------------ block-sparse forward

SPARSE_METRIC = "block-sparse attention forward TFLOPS (allowed 128x128 tile pairs) on 1 B200"


def sparse_oracle_sample(w, mask, heads: int, seed: int):
    """fp64 oracle block-mask forward on `heads` heads; returns (seconds, flops, threads)."""
    from exact_io_aware_53_b200.workloads import random_tensors
    from oracle import oracle
    q, k, v, _ = random_tensors((1, heads, w.N, w.d), torch_bf16(), seed=seed)
    t0 = time.perf_counter()
    oracle.attn_fwd_blockmask(q, k, v, w.scale, w.causal, mask.numpy())
    dt = time.perf_counter() - t0
    return dt, w.flops(mask) / (w.B * w.H) * heads, oracle.num_threads()


def torch_bf16():
    import torch
    return torch.bfloat16


def run_reference_sparse(args, w):
    from exact_io_aware_53_b200.workloads import make_block_mask
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    mask = make_block_mask(w)
    for i in range(args.warmup):
        sparse_oracle_sample(w, mask, 1, w.seed + i)
    times, fl, thr = [], 0.0, 1
    for i in range(args.steps):
        dt, fl, thr = sparse_oracle_sample(w, mask, 1, w.seed + 100 + i)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = fl / (ms / 1e3) / 1e12
    line = {"impl": "reference", "metric": SPARSE_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": 1, "H": 1, "N": w.N, "d": w.d, "causal": w.causal,
                       "density": w.density, "sample": "one head per step", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": "one head of %s per step (fp64)" % w.name},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_blocksparse(args, w):
    """One step = fa_fwd_blocksparse over the whole batch with q, k, v and the
    block mask resident in device memory."""
    import torch
    from exact_io_aware_53_b200 import fa
    from exact_io_aware_53_b200.workloads import make_block_mask, random_tensors

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl", torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    B, H, N, d = w.B, w.H, w.N, w.d
    hq, hk, hv, _ = random_tensors((B, H, N, d), torch.bfloat16, seed=rank_seed(w.seed, rank))
    q, k, v = (t.to(dev) for t in (hq, hk, hv))
    mask_cpu = make_block_mask(w)
    mask = mask_cpu.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    launches = [0]

    def step():
        rc = fa.fwd_blocksparse_raw(q, k, v, o, lse, mask, w.scale, w.causal)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_fwd_blocksparse")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after warm-up: %s" % fa.status_string(st))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after timing: %s" % fa.status_string(st))
    ms_local = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms = max_over_ranks(ms_local, world, dev)
    fl = w.flops(mask_cpu)
    value = world * fl / (ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    long_region = ms * args.steps > 500.0
    peak_key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    achieved = fl / (ms_local / 1e3) / 1e12
    pairs = int(mask_cpu.bool().sum())
    roofline = {"bound": "tensor", "kernel": "decode_partial_kernel (block-sparse, direct output)",
                "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "peak_source": "%s %s" % (peak_key, peak_src), "algorithmic_flops_per_launch": fl,
                "ms_per_launch": ms_local, "traffic": measured_traffic("blocksparse", w.name),
                "traffic_unit": "bytes per launch (ncu dram read+write)"}
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (t.pin_memory() for t in (hq, hk, hv))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        steps = max(3, min(args.steps, 20))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        e2e = {"value": world * fl / (ems / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": 3 * hq.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4,
               "steps": steps, "api": "fa.fwd_blocksparse_raw with q, k, v from and o, lse to pinned host memory"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, cfl, thr, nh = sized_oracle_sample(lambda h: sparse_oracle_sample(w, mask_cpu, h, w.seed), B * H)
        cpu = {"value": cfl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": "%d of %d heads (N=%d, d=%d, %d of %d tile pairs), fp64, %.1f s" % (
                   nh, B * H, N, d, pairs, w.tiles ** 2, dt)}
    line = {"metric": SPARSE_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "tile_pairs": pairs, "of_tile_pairs": w.tiles ** 2,
                       "parallelism": "dp%d (independent batches per GPU, no collective)" % world,
                       "l2": "inputs larger than L2 (q, k, v = %.0f MB per GPU)" % (3 * B * H * N * d * 2 / 1e6)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches[0], "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return line


# ------------------------------------------------------------------ e4m3 forward

FP8_METRIC = "FP8 (e4m3) attention forward TFLOPS on 1 B200 and fraction of the FP8 tensor peak"
FP8_OVER_BF16 = 4.5 / 2.25  # nominal dense fp8 : bf16 tensor throughput


def fp8_oracle_sample(w, heads: int, seed: int):
    """fp64 oracle forward on `heads` heads of the dequantized e4m3 inputs; returns (seconds, flops, threads)."""
    from exact_io_aware_53_b200.workloads import make_fp8_inputs
    from oracle import oracle
    x = make_fp8_inputs((1, heads, w.N, w.d), seed=seed)
    q, k, v = (x[n].double() * s for n, s in zip(("q", "k", "v"), x["descales"]))
    t0 = time.perf_counter()
    oracle.attn_fwd(q, k, v, w.scale, w.causal)
    dt = time.perf_counter() - t0
    return dt, w.flops() / (w.B * w.H) * heads, oracle.num_threads()


def run_reference_fp8(args, w):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    for i in range(args.warmup):
        fp8_oracle_sample(w, 1, w.seed + i)
    times, fl, thr = [], 0.0, 1
    for i in range(args.steps):
        dt, fl, thr = fp8_oracle_sample(w, 1, w.seed + 100 + i)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = fl / (ms / 1e3) / 1e12
    line = {"impl": "reference", "metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": 1, "H": 1, "N": w.N, "d": w.d, "causal": w.causal,
                       "sample": "one head per step (dequantized e4m3 inputs)", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": "one head of %s per step (fp64)" % w.name},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_fp8(args, w):
    """One step = fa_fwd_fp8 over the whole batch, e4m3 inputs resident in device memory."""
    import torch
    from exact_io_aware_53_b200 import fa
    from exact_io_aware_53_b200.workloads import make_fp8_inputs

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl", torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    B, H, N, d = w.B, w.H, w.N, w.d
    x = make_fp8_inputs((B, H, N, d), seed=rank_seed(w.seed, rank))
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    launches = [0]

    def step():
        rc = fa.fwd_fp8_raw(q, k, v, o, lse, x["descales"], w.scale, w.causal)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_fwd_fp8")

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after warm-up: %s" % fa.status_string(st))
    # inputs are 100 MB: flush L2 between timed calls by writing 2x its size
    flush = torch.empty(2 * 126 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.fill_(float(i))
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after timing: %s" % fa.status_string(st))
    ms_local = statistics.mean(a.elapsed_time(b) for a, b in evs)
    ms = max_over_ranks(ms_local, world, dev)
    fl = w.flops()
    value = world * fl / (ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak = bf16 * FP8_OVER_BF16
    achieved = fl / (ms_local / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "fwd_kernel<128, causal, e4m3> (persistent, kind::f8f6f4)", "achieved": achieved,
                "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "peak_source": "bf16_tflops %s x %.1f (nominal fp8 : bf16 ratio)" % (peak_src, FP8_OVER_BF16),
                "frac_of_bf16_peak": achieved / bf16, "algorithmic_flops_per_launch": fl, "ms_per_launch": ms_local,
                "traffic": measured_traffic("fp8", w.name), "traffic_unit": "bytes per launch (ncu dram read+write)"}
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        steps = max(3, min(args.steps, 20))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        e2e = {"value": world * fl / (ems / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": 3 * hq.numel(), "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4,
               "steps": steps, "api": "fa.fwd_fp8_raw with q, k, v from and o, lse to pinned host memory"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, cfl, thr, nh = sized_oracle_sample(lambda h: fp8_oracle_sample(w, h, w.seed), B * H)
        cpu = {"value": cfl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": "%d of %d heads (N=%d, d=%d, causal=%s, dequantized e4m3), fp64, %.1f s" % (
                   nh, B * H, N, d, w.causal, dt)}
    line = {"metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3 (fp32 accumulate, bf16 out)", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal,
                       "parallelism": "dp%d (independent batches per GPU, no collective)" % world,
                       "l2": "flushed before each timed call (q, k, v = %.0f MB per GPU)" % (3 * B * H * N * d / 1e6)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches[0], "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return line


# ------------------------------------------------------------------ forward with dropout

DROPOUT_METRIC = "attention fwd/bwd with dropout TFLOPS on 1 B200 and fraction of dense BF16 tensor peak"


def dropout_oracle_sample(w, heads: int, seed: int):
    """fp64 oracle dropout forward and backward on `heads` heads; returns
    (seconds, flops under the fwd + 2.5 x fwd convention, threads)."""
    from exact_io_aware_53_b200.workloads import random_tensors
    from oracle import oracle
    q, k, v, do = random_tensors((1, heads, w.N, w.d), torch_bf16(), seed=seed)
    t0 = time.perf_counter()
    oracle.attn_fwd_dropout(q, k, v, w.scale, w.causal, w.keep_t, w.seed, w.offset)
    for h in range(heads):
        oracle.attn_bwd_head(q[0, h], k[0, h], v[0, h], do[0, h], w.scale, w.causal, keep_t=w.keep_t, seed=w.seed,
                             offset=w.offset, bh=h)
    dt = time.perf_counter() - t0
    return dt, 3.5 * w.flops() / (w.B * w.H) * heads, oracle.num_threads()


def run_reference_dropout(args, w):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    for i in range(args.warmup):
        dropout_oracle_sample(w, 1, w.seed + i)
    times, fl, thr = [], 0.0, 1
    for i in range(args.steps):
        dt, fl, thr = dropout_oracle_sample(w, 1, w.seed + 100 + i)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = fl / (ms / 1e3) / 1e12
    line = {"impl": "reference", "metric": DROPOUT_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": 1, "H": 1, "N": w.N, "d": w.d, "causal": w.causal,
                       "keep_t": w.keep_t, "sample": "one head per step", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": "one head of %s per step (fp64)" % w.name},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)
    return 0


def run_dropout(args, w):
    """One step = fa_fwd_dropout then fa_bwd_dropout over the whole batch, inputs
    resident in device memory; FLOPs: forward 4 B H N^2 d (halved causal),
    backward 2.5 times that."""
    import torch
    from exact_io_aware_53_b200 import fa
    from exact_io_aware_53_b200.workloads import random_tensors

    rank, world, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        init_dist(world, "nccl", torch.device("cuda", local))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    B, H, N, d = w.B, w.H, w.N, w.d
    hq, hk, hv, hdo = random_tensors((B, H, N, d), torch.bfloat16, seed=rank_seed(w.seed, rank))
    q, k, v, do = (t.to(dev) for t in (hq, hk, hv, hdo))
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq = torch.empty(q.shape, dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty_like(dq)
    ws = torch.empty(max(1, fa.bwd_workspace_bytes(B, H, N, d)), dtype=torch.uint8, device=dev)
    launches = [0]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        rc = fa.fwd_dropout_raw(q, k, v, o, lse, w.scale, w.causal, w.keep_t, w.seed, w.offset)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_fwd_dropout")
        if ev is not None:
            ev[1].record(stream)
        rc = fa.bwd_dropout_raw(q, k, v, o, lse, do, dq, dk, dv, ws, w.scale, w.causal, w.keep_t, w.seed, w.offset)
        launches[0] += fa.last_launch_count()
        if rc:
            raise fa.FAError(rc, "fa_bwd_dropout")
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after warm-up: %s" % fa.status_string(st))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    launches[0] = 0
    barrier(world)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    st = fa.check_device_status()
    if st:
        raise RuntimeError("device status after timing: %s" % fa.status_string(st))
    timed_launches = launches[0]
    ms_local = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(ms_local, world, dev)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    fl_fwd = w.flops()
    fl_bwd = 2.5 * fl_fwd
    value = world * (fl_fwd + fl_bwd) / (ms / 1e3) / 1e12
    peaks, peak_src = load_peaks()
    long_region = ms * args.steps > 500.0
    peak_key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    peak = float(peaks.get(peak_key, FALLBACK_PEAKS[peak_key]))
    achieved = fl_bwd / (bwd_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "fa_bwd_dropout (pre-pass + bwd_kernel<128, causal, dropout>)",
                "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                "peak_source": "%s %s" % (peak_key, peak_src), "algorithmic_flops_per_launch": fl_bwd,
                "ms_per_launch": bwd_ms, "traffic": measured_traffic("bwd_dropout", w.name),
                "traffic_unit": "bytes per launch (ncu dram read+write)"}
    fwd_tf = fl_fwd / (fwd_ms / 1e3) / 1e12
    kernels = {"fwd_dropout": {"ms": fwd_ms, "tflops": fwd_tf, "frac": fwd_tf / peak},
               "bwd_dropout": {"ms": bwd_ms, "tflops": achieved, "frac": achieved / peak}}
    fl = fl_fwd + fl_bwd
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (t.pin_memory() for t in (hq, hk, hv, hdo))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hl = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        hg = [torch.empty(dq.shape, dtype=dq.dtype).pin_memory() for _ in range(3)]
        steps = max(3, min(args.steps, 20))

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            do.copy_(hdo, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            for h_, g_ in zip(hg, (dq, dk, dv)):
                h_.copy_(g_, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ems = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        e2e = {"value": world * fl / (ems / 1e3) / 1e12, "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": 4 * hq.numel() * 2,
               "d2h_bytes_per_step": ho.numel() * 2 + hl.numel() * 4 + 3 * dq.numel() * 4, "steps": steps,
               "api": "fa.fwd_dropout_raw + fa.bwd_dropout_raw with q, k, v, dO from and o, lse, dq, dk, dv to "
                      "pinned host memory"}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, cfl, thr, nh = sized_oracle_sample(lambda h: dropout_oracle_sample(w, h, w.seed), B * H)
        cpu = {"value": cfl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
               "sample": "%d of %d heads (N=%d, d=%d, causal=%s, keep %d/256), fp64, %.1f s" % (
                   nh, B * H, N, d, w.causal, w.keep_t, dt)}
    line = {"metric": DROPOUT_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": B, "H": H, "N": N, "d": d, "causal": w.causal, "keep_t": w.keep_t,
                       "backward": True,
                       "parallelism": "dp%d (independent batches per GPU, no collective)" % world,
                       "l2": "inputs larger than L2 (q, k, v, dO = %.0f MB per GPU)" % (4 * B * H * N * d * 2 / 1e6)},
            "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": timed_launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--n-split", type=int, default=0, help="key ranges for the decode workloads (0: library choice)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bwd-softmax-warps", type=int, default=0, choices=[0, 4, 8],
                    help="softmax warps per backward CTA (0: the library's choice)")
    args = ap.parse_args(argv)
    if args.bwd_softmax_warps and args.impl == "ours":
        from exact_io_aware_53_b200 import fa
        fa._lib.fa_set_bwd_softmax_warps(args.bwd_softmax_warps)
    from exact_io_aware_53_b200.workloads import (BLOCKSPARSE_WORKLOADS, DECODE_WORKLOADS, DROPOUT_WORKLOADS,
                                                  FP8_WORKLOADS, WORKLOADS)
    known = (list(WORKLOADS) + list(DECODE_WORKLOADS) + list(BLOCKSPARSE_WORKLOADS) + list(FP8_WORKLOADS) +
             list(DROPOUT_WORKLOADS))
    if args.workload != "all" and args.workload not in known:
        ap.error("unknown workload %s (choose from %s)" % (args.workload, ", ".join(known)))
    names = known if args.workload == "all" else [args.workload]
    rc = 0
    try:
        for name in names:
            if name in DROPOUT_WORKLOADS:
                w = DROPOUT_WORKLOADS[name]
                if args.impl == "reference":
                    rc |= run_reference_dropout(args, w)
                else:
                    run_dropout(args, w)
                continue
            if name in FP8_WORKLOADS:
                w = FP8_WORKLOADS[name]
                if args.impl == "reference":
                    rc |= run_reference_fp8(args, w)
                else:
                    run_fp8(args, w)
                continue
            if name in BLOCKSPARSE_WORKLOADS:
                w = BLOCKSPARSE_WORKLOADS[name]
                if args.impl == "reference":
                    rc |= run_reference_sparse(args, w)
                else:
                    run_blocksparse(args, w)
                continue
            if name in DECODE_WORKLOADS:
                w = DECODE_WORKLOADS[name]
                if args.impl == "reference":
                    rc |= run_reference_decode(args, w)
                else:
                    run_decode(args, w)
                continue
            w = WORKLOADS[name]
            if args.impl == "reference":
                rc |= run_reference(args, w)
            elif w.dtype != "bf16":
                continue  # the fp32 workload is a correctness case, not a bench line
            else:
                run_ours(args, w)
    finally:
        _, world, _ = rank_env()
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()
    return rc


if __name__ == "__main__":
    sys.exit(main())
