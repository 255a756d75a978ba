#!/usr/bin/env python
"""Benchmark of the training RMSNorm hot path on B200.

Headline workload (one "step"): the checkpointed training step on the large-T
configuration -- forward, forward recompute, backward (deterministic=False) -- for
x, dy BF16 [T=131072, H=6144] ~ N(0,1), BF16 weight 1 + 0.1 N(0,1), eps 1e-6, synthetic
and seeded.  Inputs are far larger than L2 and L2 is also flushed before every timed
step.  ``value`` is microseconds per step (lower is better); the pages report 1640.48 us
for this step on B200 (flashinfer PR #8848 table, H6144 T131072, BF16 weight).

Every launch inside the timed region is one of librmsnorm_train's kernels.  The JSON
line also carries the roofline of the dominant kernel (the backward), the CPU oracle
as a baseline, an end-to-end figure with host buffers, SM clocks sampled during the
timed region, and a per-configuration table (CUPTI span of a CUDA-graph replay, cold L2,
the pages' timing rule) with the achieved fraction of the measured HBM bandwidth.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--sweep all|none]
For N > 1 launch under torchrun: every rank runs its own replica (weak scaling, no
collective on the data path); the step time is the maximum over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "RMSNorm train bwd/fwd us per call and achieved HBM GB/s (% of B200 peak)"
PAGES_STEP_US = 1640.48  # B200, H6144 T131072 BF16 weight, non-det 2xfwd+bwd (PR #8848 table)
PAGES_STEP_DET_US = 1637.76  # the same row, deterministic
FALLBACK_HBM_GBS = 6650.0
HEAD_T, HEAD_H = 131072, 6144
WORKLOAD = ("large-T checkpointed step (fwd, fwd recompute, bwd), "
            "x/dy BF16 [131072, 6144] N(0,1), BF16 w 1+0.1N(0,1), eps 1e-6")


# ---- algorithmic bytes (minimal traffic) ------------------------------------------------------

def bytes_fwd(R, H, wb, res=False):
    return (8 if res else 4) * R * H + H * wb + 4 * R


def bytes_bwd(R, H, wb, res=False):
    return (8 if res else 6) * R * H + H * wb + 4 * R + 4 * H


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha():
    """Hash of the pipelined backward kernel's source (its section of bwd.cu) and of the
    shared device header: a recorded traffic figure stays valid while these are unchanged."""
    csrc = os.path.join(ROOT, "bwd_rmsnorm_fwd_b200", "csrc")
    with open(os.path.join(csrc, "bwd.cu")) as fh:
        text = fh.read()
    a = text.find("// Large-row kernel: a bulk-copy pipeline")
    b = text.find("// Fold kernel")
    h = hashlib.sha256(text[a:b].encode())
    with open(os.path.join(csrc, "common.cuh"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f).get(key)
        if d and d.get("source_sha") == source_sha():
            return int(d["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


# ---- clocks during the timed region -------------------------------------------------------------

class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML (read-only queries)."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hh)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hh
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                util = nv.nvmlDeviceGetUtilizationRates(h).gpu
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((sm, util, rs, pw))
            except Exception:
                pass
            time.sleep(0.02)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        self._stop.set()
        self.t.join()
        loaded = [s for s in self.samples if s[1] >= 50] or self.samples
        reasons = sorted({n for s in loaded for n, b in self.REASONS.items() if s[2] & b})
        sm = statistics.median([s[0] for s in loaded]) if loaded else None
        pw = max([s[3] for s in loaded], default=None)
        return {"sm_mhz": sm, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(loaded), "power_w_max": pw}


# ---- the reference arm: the FP64 CPU oracle ----------------------------------------------------

def oracle_step_seconds(rows, H, nthreads=0):
    """One checkpointed step (fwd, fwd, bwd) of the oracle on `rows` rows of width H."""
    import oracle
    from bwd_rmsnorm_fwd_b200 import synth
    x = synth.rows(0, "x", rows, H)
    dy = synth.rows(0, "dy", rows, H)
    w = synth.weight(0, H, "bf16")
    t0 = time.perf_counter()
    oracle.train_fwd(x, w, 1e-6, nthreads=nthreads)
    _, rstd = oracle.train_fwd(x, w, 1e-6, nthreads=nthreads)
    oracle.train_bwd(x, w, rstd, dy, nthreads=nthreads)
    return time.perf_counter() - t0


def oracle_sample_rows(target_s):
    t = oracle_step_seconds(256, HEAD_H)
    rows = int(256 * target_s / max(t, 1e-6))
    return max(256, min(HEAD_T, rows))


def cpu_baseline(target_s=10.0):
    import oracle
    rows = oracle_sample_rows(target_s)
    t = oracle_step_seconds(rows, HEAD_H)
    us = t * (HEAD_T / rows) * 1e6
    return {"value": round(us, 1), "unit": "us", "cores": oracle.hardware_threads(),
            "kind": "oracle",
            "sample": f"{rows} of {HEAD_T} rows of the headline step (fwd, fwd, bwd) on the "
                      f"FP64 C++ oracle, {t:.1f} s, scaled linearly to all rows"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    # per-step sample sized so that warmup + steps take about two minutes in all
    rows = oracle_sample_rows(min(3.0, 120.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_step_seconds(rows, HEAD_H)
    ts = [oracle_step_seconds(rows, HEAD_H) for _ in range(args.steps)]
    us = statistics.median(ts) * (HEAD_T / rows) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(us / 1e3, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "l2": "inputs larger than L2"},
        "cpu_baseline": {"value": round(us, 1), "unit": "us", "cores": oracle.hardware_threads(),
                         "kind": "oracle",
                         "sample": f"{rows} of {HEAD_T} rows per step, scaled linearly"},
        "e2e": {"value": round(us, 1), "unit": "us", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))
    return 0


# ---- multi-rank plumbing ----------------------------------------------------------------------

def max_over_ranks(value, dist, device):
    """The maximum of `value` over all ranks (the step time of a replica job is that of its
    slowest rank); `dist` is torch.distributed or None for one process."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- GPU timing helpers ----------------------------------------------------------------------

def make_inputs(T, H, wdt, seed, device, torch):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    x = torch.randn(T, H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    dy = torch.randn(T, H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    w = 1 + 0.1 * torch.randn(H, generator=g, device=device, dtype=torch.float32)
    w = w.to(torch.bfloat16) if wdt == "bf16" else w
    return x, dy, w


def graph_time_us(fn, flush, torch, reps=20):
    """Median per-replay time of fn captured in a CUDA graph, L2 flushed before every
    replay (outside the timed events)."""
    fn()  # warm: allocates outputs / workspace outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g):
            fn()
        run = g.replay
    except Exception:
        run = fn
    ts = []
    for i in range(reps + 3):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        run()
        b.record()
        b.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b) * 1e3)
    del g
    return statistics.median(ts)


def call_spans_us(events, flush_tag="FillFunctor"):
    """Per-call spans from device records (name, start_us, end_us) of a loop that flushes L2
    before every call: records sorted by start, cut at every flush kernel; a call's span runs
    from its first record's start to its last record's end."""
    spans, lo, hi = [], None, None
    for name, start, end in sorted(events, key=lambda e: e[1]):
        if flush_tag in name:
            if lo is not None:
                spans.append(hi - lo)
            lo = hi = None
        else:
            lo = start if lo is None else min(lo, start)
            hi = end if hi is None else max(hi, end)
    if lo is not None:
        spans.append(hi - lo)
    return spans


def span_time_us(fn, flush, torch, reps=30):
    """Median CUPTI span of one call replayed from a CUDA graph with L2 flushed before each
    replay (the pages' timing rule): first kernel start to last kernel end, every kernel of
    the call inside the span."""
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.graph(g):
            fn()
        run = g.replay
    except Exception:
        run = fn
    run()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(reps):
            flush.zero_()
            run()
        torch.cuda.synchronize()
    events = [(e.name, e.time_range.start, e.time_range.end) for e in prof.events()
              if e.device_type == DeviceType.CUDA]
    del g
    spans = call_spans_us(events)
    if not spans:
        raise RuntimeError("the profiler recorded no device activity for the call")
    return statistics.median(spans)


SWEEP_GROUPS = ("tiny", "small-T", "residual", "per-head", "large-T")


def sweep(torch, api, flush, peak, dev, groups=SWEEP_GROUPS):
    """Per-configuration table: us per call (CUPTI span of a graph replay, cold L2; CUDA events
    around the replay too where a call is long enough) and the fraction of the measured HBM
    bandwidth, for every configuration of the pages' tables."""
    out = []
    ws = api.Workspace(dev)

    def rec(cfg, form, H, T, wdt, op, fn, nbytes, replay):
        us = span_time_us(fn, flush, torch)
        gbs = nbytes / (us * 1e-6) / 1e9
        row = {"cfg": cfg, "form": form, "H": H, "T": T, "w": wdt, "op": op,
               "us": round(us, 2), "gbs": round(gbs, 1), "frac": round(gbs / peak, 3),
               "timer": "cupti_span"}
        if replay:
            row["replay_us"] = round(graph_time_us(fn, flush, torch), 2)
        out.append(row)

    def ops(cfg, form, x, dy, w, H, T, R, wdt, heads=1, res=None, dh=None, do=("fwd", "det", "nondet")):
        wb = 2 if wdt == "bf16" else 4
        isres = res is not None
        # CUDA events around a graph replay as well, where a call outlasts the launch latency
        replay = R * H > (1 << 22)
        if isres:
            h, _, rstd = api.rmsnorm_train_fwd(x, w, residual=res)
        else:
            _, rstd = api.rmsnorm_train_fwd(x, w)
            h = x
        if "fwd" in do:
            rec(cfg, form, H, T, wdt, "fwd", lambda: api.rmsnorm_train_fwd(x, w, residual=res),
                bytes_fwd(R, H, wb, isres), replay)
        for det in (True, False):
            if ("det" if det else "nondet") not in do:
                continue
            rec(cfg, form, H, T, wdt, "bwd_det" if det else "bwd_nondet",
                lambda: api.rmsnorm_train_bwd(h, w, rstd, dy, deterministic=det, dh=dh,
                                              workspace=ws),
                bytes_bwd(R, H, wb, isres), replay)

    # Tiny and small-T sweep (deterministic backward, single launch)
    if "tiny" in groups:
        x, dy, w = make_inputs(64, 512, "fp32", 1, dev, torch)
        ops("tiny", "plain", x, dy, w, 512, 64, 64, "fp32", do=("fwd", "det"))
    for H in (256, 512, 2048, 4096) if "small-T" in groups else ():
        for wdt in ("bf16", "fp32"):
            xa, dya, w = make_inputs(227, H, wdt, 2, dev, torch)
            for T in (1, 2, 8, 32, 87, 227):
                ops("small-T", "plain", xa[:T], dya[:T], w, H, T, T, wdt, do=("det",))
    # residual H 6144
    for T in (32, 4096, 65537) if "residual" in groups else ():
        x, dy, w = make_inputs(T, 6144, "bf16", 3, dev, torch)
        res, dh, _ = make_inputs(T, 6144, "bf16", 4, dev, torch)
        ops("residual", "res", x, dy, w, 6144, T, T, "bf16", res=res, dh=dh)
        del x, dy, res, dh
    # per-head views, FP32 weight
    for T in (1024, 16384) if "per-head" in groups else ():
        for name, heads, st, sk in (("24x256_pages", 24, 12288, 512),
                                    ("24x256_dense", 24, 6144, 256), ("4x256", 4, 1024, 256)):
            n = (T - 1) * st + (heads - 1) * sk + 256
            g = torch.Generator(device=dev)
            g.manual_seed(5)
            bx = torch.randn(n, generator=g, device=dev).to(torch.bfloat16)
            bd = torch.randn(n, generator=g, device=dev).to(torch.bfloat16)
            x = torch.as_strided(bx, (T, heads, 256), (st, sk, 1))
            dy = torch.as_strided(bd, (T, heads, 256), (st, sk, 1))
            w = 1 + 0.1 * torch.randn(256, generator=g, device=dev)
            ops("per-head", name, x, dy, w, 256, T, T * heads, "fp32", heads=heads)
            del bx, bd
    # large T
    for H in (1536, 2048, 4096, 5120, 6144) if "large-T" in groups else ():
        for wdt in ("bf16", "fp32"):
            xa, dya, w = make_inputs(131072, H, wdt, 6, dev, torch)
            for T in (65537, 98304, 131072):
                ops("large-T", "plain", xa[:T], dya[:T], w, H, T, T, wdt)
            del xa, dya
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", default="all", choices=["all", "none", *SWEEP_GROUPS],
                    help="per-configuration table: every group, none, or one group")
    ap.add_argument("--det", action="store_true",
                    help="the step's backward uses deterministic=True")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", type=int, default=HEAD_T, help="T of the headline step")
    ap.add_argument("--width", type=int, default=HEAD_H, help="H of the headline step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import torch
    from bwd_rmsnorm_fwd_b200 import api, build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    build.build()
    peak, peak_kind = peaks()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > L2

    R, H, wb = args.rows, args.width, 2
    x, dy, w = make_inputs(R, H, "bf16", 1234 + rank, dev, torch)
    ws = api.Workspace(dev)

    def step():
        api.rmsnorm_train_fwd(x, w)                       # forward
        _, rstd = api.rmsnorm_train_fwd(x, w)             # recompute (checkpointed)
        return rstd

    for _ in range(args.warmup):
        rstd = step()
        api.rmsnorm_train_bwd(x, w, rstd, dy, deterministic=args.det, workspace=ws)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    evs = []
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        flush.zero_()
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        e0.record()
        rstd = step()
        e1.record()
        api.rmsnorm_train_bwd(x, w, rstd, dy, deterministic=args.det, workspace=ws)
        e2.record()
        evs.append((e0, e1, e2))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    api.status(ws)
    step_us = [a.elapsed_time(c) * 1e3 for a, b, c in evs]
    bwd_us = [b.elapsed_time(c) * 1e3 for a, b, c in evs]
    ms_step = max_over_ranks(sum(step_us) / len(step_us) / 1e3, dist, dev)
    us_step = ms_step * 1e3
    bwd_avg_us = sum(bwd_us) / len(bwd_us)
    step_bytes = 2 * bytes_fwd(R, H, wb) + bytes_bwd(R, H, wb)
    bwd_bytes = bytes_bwd(R, H, wb)
    achieved = bwd_bytes / (bwd_avg_us * 1e-6) / 1e9

    # end to end through the public API with pinned host buffers
    xh = x.cpu().pin_memory()
    dyh = dy.cpu().pin_memory()
    dxh = torch.empty_like(xh).pin_memory()
    dwh = torch.empty(H, dtype=torch.float32).pin_memory()
    xd = torch.empty_like(x)
    dyd = torch.empty_like(dy)
    e2e = []
    for i in range(args.e2e_steps + 1 if args.e2e_steps > 0 else 0):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        xd.copy_(xh, non_blocking=True)
        dyd.copy_(dyh, non_blocking=True)
        api.rmsnorm_train_fwd(xd, w)
        _, r2 = api.rmsnorm_train_fwd(xd, w)
        dxd, dwd = api.rmsnorm_train_bwd(xd, w, r2, dyd, deterministic=args.det, workspace=ws)
        dxh.copy_(dxd, non_blocking=True)
        dwh.copy_(dwd, non_blocking=True)
        b.record()
        b.synchronize()
        if i:
            e2e.append(a.elapsed_time(b) * 1e3)
    del xd, dyd, xh, dyh, dxh
    e2e_us = statistics.median(e2e) if e2e else None

    per_cfg = None
    if args.sweep != "none" and rank == 0:
        del x, dy
        torch.cuda.empty_cache()
        per_cfg = sweep(torch, api, flush, peak, dev,
                        SWEEP_GROUPS if args.sweep == "all" else (args.sweep,))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(10.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(us_step, 2), "unit": "us", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "higher_is_better": False, "scaling": "weak",
            "vs_baseline": (round(us_step / (PAGES_STEP_DET_US if args.det else PAGES_STEP_US), 4)
                            if (R, H) == (HEAD_T, HEAD_H) else None),
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": (WORKLOAD if (R, H) == (HEAD_T, HEAD_H) else
                                    f"checkpointed step at T={R}, H={H} (reduced case)")
                       + f", backward deterministic={args.det}", "T": R, "H": H,
                       "w": "bf16",
                       "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                       "l2": "inputs larger than L2, and L2 flushed before every step"},
            "step_gbs": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
            "aggregate_gbs": round(world * step_bytes / (ms_step * 1e-3) / 1e9, 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": peak_kind,
                         "kernel": f"bwd_staged_kernel (deterministic={args.det}), H{H} T{R}",
                         "bytes_per_launch": bwd_bytes, "launch_us": round(bwd_avg_us, 2),
                         "traffic": recorded_traffic(
                             f"bwd_{'det' if args.det else 'nondet'}_h{H}_t{R}_bf16")},
            "e2e": {"value": round(e2e_us, 1) if e2e_us else None, "unit": "us",
                    "h2d_bytes_per_step": 2 * R * H * 2,
                    "d2h_bytes_per_step": R * H * 2 + H * 4},
            "gpu_launches": (4 if args.det else 3) * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        if per_cfg is not None:
            line["per_config"] = per_cfg
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
