#!/usr/bin/env python
"""Benchmark of the training RMSNorm hot path on B200.

Headline workload (one "step"): the checkpointed training step on the large-T
configuration -- forward, forward recompute, backward (deterministic=False), run through
the library's autograd wrapper under torch.utils.checkpoint, dw added into a float32
main-grad buffer -- for
x, dy BF16 [T=131072, H=6144] ~ N(0,1), BF16 weight 1 + 0.1 N(0,1), eps 1e-6, synthetic
and seeded.  Inputs are far larger than L2 and L2 is also flushed before every timed
step.  ``value`` is microseconds per step (lower is better); the pages report 1640.48 us
for this step on B200 (flashinfer PR #8848 table, H6144 T131072, BF16 weight).

Every launch inside the timed region is one of librmsnorm_train's kernels.  Output: one
JSON line on stdout, printed last and kept short (under MAX_LINE_BYTES): the step time, the
roofline of the dominant kernel (the backward), the CPU oracle as a baseline (all host
threads and one thread), an end-to-end figure with host buffers, SM clocks sampled during
the timed region, and a summary of the per-configuration table.  The table itself (every
configuration of the pages' tables: median, p10 and p90 of the CUPTI span of a CUDA-graph
replay with L2 flushed before each, 3 interleaved rounds x 67 replays per call, an A/A
floor per group, and the fraction of the measured HBM bandwidth) goes to its own file,
``--per-config-out``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--sweep all|none|<group>] [--per-config-out FILE]
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
            time.sleep(0.005)

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

def oracle_inputs(rows, H):
    from bwd_rmsnorm_fwd_b200 import synth
    return synth.rows(0, "x", rows, H), synth.rows(0, "dy", rows, H), synth.weight(0, H, "bf16")


def oracle_step_seconds(inputs, nthreads=0):
    """One checkpointed step (fwd, fwd, bwd) of the oracle on the given rows; nthreads = 0
    uses every hardware thread."""
    import oracle
    x, dy, w = inputs
    t0 = time.perf_counter()
    oracle.train_fwd(x, w, 1e-6, nthreads=nthreads)
    _, rstd = oracle.train_fwd(x, w, 1e-6, nthreads=nthreads)
    oracle.train_bwd(x, w, rstd, dy, nthreads=nthreads)
    return time.perf_counter() - t0


def oracle_sample_rows(target_s, nthreads=0):
    """Rows of the headline width that one oracle step covers in about target_s seconds."""
    probe = 256 if nthreads != 1 else 64
    t = oracle_step_seconds(oracle_inputs(probe, HEAD_H), nthreads)
    rows = int(probe * target_s / max(t, 1e-6))
    return max(probe, min(HEAD_T, rows))


def cpu_baseline(target_s=10.0):
    """The oracle, as it stands, on a bounded row sample of the headline step, with every
    hardware thread and with one thread; each scaled linearly to all rows."""
    import oracle
    out = None
    for nthreads in (0, 1):
        rows = oracle_sample_rows(target_s, nthreads)
        t = oracle_step_seconds(oracle_inputs(rows, HEAD_H), nthreads)
        cores = oracle.hardware_threads() if nthreads == 0 else 1
        rec = {"value": round(t * (HEAD_T / rows) * 1e6, 1), "unit": "us", "cores": cores,
               "kind": "oracle",
               "sample": f"{rows} of {HEAD_T} rows of the headline step (fwd, fwd, bwd), "
                         f"{t:.1f} s, scaled linearly to all rows"}
        if out is None:
            out = rec
        else:
            out["single_thread"] = {k: rec[k] for k in ("value", "cores", "sample")}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    # per-step sample sized so that warmup + steps take about two minutes in all; the
    # inputs are drawn once and every step recomputes from them
    rows = oracle_sample_rows(min(3.0, 120.0 / (args.steps + args.warmup)))
    inputs = oracle_inputs(rows, HEAD_H)
    for _ in range(args.warmup):
        oracle_step_seconds(inputs)
    ts = [oracle_step_seconds(inputs) for _ in range(args.steps)]
    us = statistics.median(ts) * (HEAD_T / rows) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": "us",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(us / 1e3, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "T": HEAD_T, "H": HEAD_H, "w": "bf16",
                   "l2": "inputs larger than L2"},
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


HEAD_VIEWS = {"24x256_pages": (24, 12288, 512), "24x256_dense": (24, 6144, 256),
              "4x256": (4, 1024, 256)}


def head_view_inputs(T, view, device, torch):
    """x, dy as a per-head view [T, heads, 256] of one allocation each (the pages' strided
    layout, a dense one, or four heads), and an FP32 weight of 256."""
    heads, st, sk = HEAD_VIEWS[view]
    n = (T - 1) * st + (heads - 1) * sk + 256
    g = torch.Generator(device=device)
    g.manual_seed(5)
    bx = torch.randn(n, generator=g, device=device).to(torch.bfloat16)
    bd = torch.randn(n, generator=g, device=device).to(torch.bfloat16)
    x = torch.as_strided(bx, (T, heads, 256), (st, sk, 1))
    dy = torch.as_strided(bd, (T, heads, 256), (st, sk, 1))
    w = 1 + 0.1 * torch.randn(256, generator=g, device=device)
    return x, dy, w


def profile_case(spec, torch, api, dev, calls=3):
    """Runs one library call of one configuration `calls` times with L2 flushed before each
    (the program a profiler capture runs).  spec = OP:H:T[:FORM[:W]]: OP fwd, bwd_det or
    bwd_nondet; FORM plain (default), res (H 6144 residual rows) or a per-head view
    (24x256_pages, 24x256_dense, 4x256; H is 256 there and T counts tokens); W bf16
    (default) or fp32."""
    parts = spec.split(":")
    op, H, T = parts[0], int(parts[1]), int(parts[2])
    form = parts[3] if len(parts) > 3 else "plain"
    wdt = parts[4] if len(parts) > 4 else "bf16"
    if op not in ("fwd", "bwd_det", "bwd_nondet"):
        raise SystemExit(f"unknown op {op!r}")
    res = dh = None
    if form in HEAD_VIEWS:
        x, dy, w = head_view_inputs(T, form, dev, torch)
    else:
        x, dy, w = make_inputs(T, H, wdt, 6, dev, torch)
        if form == "res":
            res, dh, _ = make_inputs(T, H, "bf16", 4, dev, torch)
        elif form != "plain":
            raise SystemExit(f"unknown form {form!r}")
    if res is not None:
        h, _, rstd = api.rmsnorm_train_fwd(x, w, residual=res)
    else:
        h = x
        _, rstd = api.rmsnorm_train_fwd(x, w)
    ws = api.Workspace(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > L2
    for _ in range(calls):
        flush.zero_()
        if op == "fwd":
            api.rmsnorm_train_fwd(x, w, residual=res)
        else:
            api.rmsnorm_train_bwd(h, w, rstd, dy, deterministic=op == "bwd_det", dh=dh,
                                  workspace=ws)
    if dev.type == "cuda":
        torch.cuda.synchronize(dev)
    api.status(ws)
    print("profile case done:", spec)


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


def interleaved_order(keys, rounds, reps):
    """Replay order of the timing protocol: `rounds` rounds; in round r the calls run in the
    list's order rotated by r; each call `reps` times in a row."""
    order = []
    n = len(keys)
    for r in range(rounds):
        k = r % n if n else 0
        for key in keys[k:] + keys[:k]:
            order.extend([key] * reps)
    return order


def quantile(xs, q):
    s = sorted(xs)
    if not s:
        return None
    i = q * (len(s) - 1)
    lo = int(i)
    hi = min(lo + 1, len(s) - 1)
    return s[lo] + (s[hi] - s[lo]) * (i - lo)


def time_group(calls, flush, torch, rounds=3, reps=67):
    """CUPTI spans of several calls, each captured in its own CUDA graph and replayed with L2
    flushed before every replay, in interleaved rounds (the pages' protocol: rounds x reps
    replays per call, rotated order).  `calls` is a list of (key, fn); every call runs once
    before any capture, so a growing workspace reaches its size outside the captures.
    Returns {key: [span_us, ...]}."""
    from torch.autograd import DeviceType
    from torch.profiler import ProfilerActivity, profile
    for _, fn in calls:
        fn()
    torch.cuda.synchronize()
    graphs = {}
    for key, fn in calls:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        graphs[key] = g
    for g in graphs.values():
        g.replay()
    torch.cuda.synchronize()
    order = interleaved_order([k for k, _ in calls], rounds, reps)
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for key in order:
            flush.zero_()
            graphs[key].replay()
        torch.cuda.synchronize()
    events = [(e.name, e.time_range.start, e.time_range.end) for e in prof.events()
              if e.device_type == DeviceType.CUDA]
    spans = call_spans_us(events)
    del graphs
    if len(spans) != len(order):
        raise RuntimeError(f"profiler gave {len(spans)} call spans for {len(order)} replays")
    out = {k: [] for k, _ in calls}
    for key, s in zip(order, spans):
        out[key].append(s)
    return out


def event_time_us(fn, flush, torch, reps=20):
    """Median CUDA-event time of fn's graph replay on the current stream, L2 flushed before
    every replay (outside the events)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    ts = []
    for i in range(reps + 3):
        flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        b.synchronize()
        if i >= 3:
            ts.append(a.elapsed_time(b) * 1e3)
    del g
    return statistics.median(ts)


SWEEP_GROUPS = ("tiny", "small-T", "residual", "per-head", "large-T", "long-256")


def sweep(torch, api, flush, peak, dev, groups=SWEEP_GROUPS, rounds=3, reps=67,
          device_index=None):
    """Per-configuration table for every configuration of the pages' tables: us per call
    (median, p10 and p90 of the CUPTI span of a CUDA-graph replay, cold L2, rounds x reps
    replays in interleaved rounds), an A/A floor per group (the group's first call captured
    twice and timed as two programs), CUDA-event time of the replay where a call is long
    enough, and the fraction of the measured HBM bandwidth.  With `device_index`, the SM clock
    (median over NVML samples while the group's spans are taken) and any clock-event reasons
    go into the group's first row."""
    out = []
    ws = api.Workspace(dev)

    def run_group(entries):
        # entries: (meta, fn, nbytes, replay); the first call is also timed as its own A/A twin
        calls = [(i, e[1]) for i, e in enumerate(entries)]
        calls.append(("aa", entries[0][1]))
        sampler = ClockSampler(device_index) if device_index is not None else None
        if sampler:
            sampler.start()
        spans = time_group(calls, flush, torch, rounds, reps)
        clk = sampler.stop() if sampler else None
        m0, ma = statistics.median(spans[0]), statistics.median(spans["aa"])
        aa = abs(m0 - ma) / ((m0 + ma) / 2)
        for i, (meta, fn, nbytes, replay) in enumerate(entries):
            us = statistics.median(spans[i])
            gbs = nbytes / (us * 1e-6) / 1e9
            row = dict(meta)
            row.update({"us": round(us, 2), "p10": round(quantile(spans[i], 0.1), 2),
                        "p90": round(quantile(spans[i], 0.9), 2), "gbs": round(gbs, 1),
                        "frac": round(gbs / peak, 3), "timer": "cupti_span",
                        "replays": len(spans[i])})
            if i == 0:
                row["aa_floor"] = round(aa, 4)
                if clk is not None:
                    row["group_sm_mhz"] = clk.get("sm_mhz")
                    row["group_clock_reasons"] = clk.get("reasons")
            if replay:
                row["replay_us"] = round(event_time_us(fn, flush, torch), 2)
            out.append(row)
        torch.cuda.synchronize()

    def ops(entries, cfg, form, x, dy, w, H, T, R, wdt, res=None, dh=None,
            do=("fwd", "det", "nondet")):
        wb = 2 if wdt == "bf16" else 4
        isres = res is not None
        # CUDA events around a graph replay as well, where a call outlasts the launch latency
        replay = R * H > (1 << 22)
        if isres:
            h, _, rstd = api.rmsnorm_train_fwd(x, w, residual=res)
        else:
            _, rstd = api.rmsnorm_train_fwd(x, w)
            h = x
        meta = {"cfg": cfg, "form": form, "H": H, "T": T, "w": wdt}
        if "fwd" in do:
            entries.append((dict(meta, op="fwd"),
                            lambda: api.rmsnorm_train_fwd(x, w, residual=res),
                            bytes_fwd(R, H, wb, isres), replay))
        for det in (True, False):
            if ("det" if det else "nondet") not in do:
                continue
            entries.append((dict(meta, op="bwd_det" if det else "bwd_nondet"),
                            (lambda d: lambda: api.rmsnorm_train_bwd(
                                h, w, rstd, dy, deterministic=d, dh=dh, workspace=ws))(det),
                            bytes_bwd(R, H, wb, isres), replay))

    if "tiny" in groups:
        e = []
        x, dy, w = make_inputs(64, 512, "fp32", 1, dev, torch)
        ops(e, "tiny", "plain", x, dy, w, 512, 64, 64, "fp32", do=("fwd", "det"))
        run_group(e)
    for H in (256, 512, 2048, 4096) if "small-T" in groups else ():
        for wdt in ("bf16", "fp32"):
            e = []
            xa, dya, w = make_inputs(227, H, wdt, 2, dev, torch)
            for T in (1, 2, 8, 32, 87, 227):
                ops(e, "small-T", "plain", xa[:T], dya[:T], w, H, T, T, wdt, do=("det",))
            run_group(e)
    for T in (32, 4096, 65537) if "residual" in groups else ():
        e = []
        x, dy, w = make_inputs(T, 6144, "bf16", 3, dev, torch)
        res, dh, _ = make_inputs(T, 6144, "bf16", 4, dev, torch)
        ops(e, "residual", "res", x, dy, w, 6144, T, T, "bf16", res=res, dh=dh)
        run_group(e)
        del e, x, dy, res, dh
    for T in (1024, 16384) if "per-head" in groups else ():
        for name in HEAD_VIEWS:
            e = []
            x, dy, w = head_view_inputs(T, name, dev, torch)
            heads = HEAD_VIEWS[name][0]
            ops(e, "per-head", name, x, dy, w, 256, T, T * heads, "fp32")
            run_group(e)
            del e, x, dy
    for H in (1536, 2048, 4096, 5120, 6144) if "large-T" in groups else ():
        for wdt in ("bf16", "fp32"):
            e = []
            xa, dya, w = make_inputs(131072, H, wdt, 6, dev, torch)
            for T in (65537, 98304, 131072):
                ops(e, "large-T", "plain", xa[:T], dya[:T], w, H, T, T, wdt)
            run_group(e)
            del e, xa, dya
            torch.cuda.empty_cache()
    if "long-256" in groups:
        # the very long narrow-row regime: H 256 rows at T 1048576, both weight dtypes
        for wdt in ("bf16", "fp32"):
            e = []
            x, dy, w = make_inputs(1048576, 256, wdt, 7, dev, torch)
            ops(e, "long-256", "plain", x, dy, w, 256, 1048576, 1048576, wdt)
            run_group(e)
            del e, x, dy
    torch.cuda.empty_cache()
    return out


def per_config_summary(rows):
    """Worst fraction of the measured bandwidth per large-T operation, and the largest A/A
    floor: the few figures of the table that go into the headline line."""
    s = {}
    for op in ("fwd", "bwd_det", "bwd_nondet"):
        fr = [r["frac"] for r in rows if r["cfg"] == "large-T" and r["op"] == op]
        if fr:
            s[f"large_T_min_frac_{op}"] = min(fr)
    aa = [r["aa_floor"] for r in rows if "aa_floor" in r]
    if aa:
        s["aa_floor_max"] = max(aa)
    return s


MAX_LINE_BYTES = 3000


def emit(line, per_cfg=None, per_cfg_path=None, peak=None, peak_kind=None, clocks=None,
         stream=None):
    """Writes the per-configuration table (when there is one) to its own file and prints the
    headline JSON line last, on its own, on stdout.  The table stays out of the line, which
    must fit in MAX_LINE_BYTES."""
    stream = stream or sys.stdout
    if per_cfg is not None:
        line["per_config"] = dict(per_config_summary(per_cfg), rows=len(per_cfg),
                                  file=os.path.relpath(per_cfg_path, ROOT) if per_cfg_path else None)
        if per_cfg_path:
            os.makedirs(os.path.dirname(os.path.abspath(per_cfg_path)), exist_ok=True)
            with open(per_cfg_path, "w") as f:
                json.dump({"peak_gbs": peak, "peak_kind": peak_kind, "clocks": clocks,
                           "timer": "CUPTI span of a CUDA-graph replay, L2 flushed before each "
                                    "replay; 3 interleaved rounds x 67 replays per call",
                           "rows": per_cfg}, f, indent=0)
    text = json.dumps(line, separators=(",", ":"))
    if len(text) > MAX_LINE_BYTES:
        raise RuntimeError(f"headline line of {len(text)} bytes exceeds {MAX_LINE_BYTES}")
    stream.write(text + "\n")
    stream.flush()
    return text


def headline_line(m):
    """The headline JSON object from the measured quantities `m` (R, H, det, world, steps,
    warmup, us_step, bwd_us, e2e_us, peak, peak_kind, clocks, cpu)."""
    R, H, wb, det = m["R"], m["H"], 2, m["det"]
    head = (R, H) == (HEAD_T, HEAD_H)
    us_step = m["us_step"]
    step_bytes = 2 * bytes_fwd(R, H, wb) + bytes_bwd(R, H, wb)
    bwd_bytes = bytes_bwd(R, H, wb)
    achieved = bwd_bytes / (m["bwd_us"] * 1e-6) / 1e9
    clocks = m["clocks"] or {}
    return {
        "metric": METRIC, "value": round(us_step, 2), "unit": "us", "n_gpus": m["world"],
        "steps": m["steps"], "warmup": m["warmup"], "ms_per_step": round(us_step / 1e3, 4),
        "higher_is_better": False, "scaling": "weak",
        "vs_baseline": (round(us_step / (PAGES_STEP_DET_US if det else PAGES_STEP_US), 4)
                        if head else None),
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD if head else
                   f"checkpointed step at T={R}, H={H} (reduced case)",
                   "T": R, "H": H, "w": "bf16", "deterministic": det,
                   "parallelism": f"replicas x{m['world']}" if m["world"] > 1 else "single GPU",
                   "l2": "inputs larger than L2, and L2 flushed before every step"},
        "step_gbs": round(step_bytes / (us_step * 1e-6) / 1e9, 1),
        "aggregate_gbs": round(m["world"] * step_bytes / (us_step * 1e-6) / 1e9, 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": m["peak"],
                     "unit": "GB/s", "frac": round(achieved / m["peak"], 4),
                     "peak_kind": m["peak_kind"],
                     "kernel": f"backward (deterministic={det}), H{H} T{R}",
                     "bytes_per_launch": bwd_bytes, "launch_us": round(m["bwd_us"], 2),
                     "traffic": recorded_traffic(
                         f"bwd_{'det' if det else 'nondet'}_h{H}_t{R}_bf16")},
        "e2e": {"value": round(m["e2e_us"], 1) if m["e2e_us"] else None, "unit": "us",
                "h2d_bytes_per_step": 2 * R * H * 2,
                "d2h_bytes_per_step": R * H * 2 + H * 4,
                "overlap": "step k+1's copy-in runs during step k's compute and copy-out"},
        "gpu_launches": (4 if det else 3) * m["steps"],
        "clocks": {k: clocks.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "power_w_max")},
        "cpu_baseline": m["cpu"],
    }


def e2e_pipelined(torch, step, x, dy, main_grad, steps, warm=2):
    """us per step of `step(x_leaf, dy)` fed from pinned host memory: copy-in, compute and
    copy-out on three streams, double-buffered device inputs; None when steps == 0."""
    if steps <= 0:
        return None
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xh, dyh = x.cpu().pin_memory(), dy.cpu().pin_memory()
    dxh = torch.empty_like(xh).pin_memory()
    dwh = torch.empty(main_grad.numel(), dtype=torch.float32).pin_memory()
    xin = [torch.empty_like(x) for _ in range(2)]
    dyin = [torch.empty_like(dy) for _ in range(2)]
    dwsnap = [torch.empty_like(main_grad) for _ in range(2)]
    n = warm + steps
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    comp.synchronize()
    for k in range(n):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_done[k - 2])  # step k-2 has finished with buffer b
            if k == warm:
                t0.record(s_in)
            xin[b].copy_(xh, non_blocking=True)
            dyin[b].copy_(dyh, non_blocking=True)
            ev_in[k].record(s_in)
        comp.wait_event(ev_in[k])
        xl = xin[b].detach().requires_grad_(True)
        dxd = step(xl, dyin[b])
        dwsnap[b].copy_(main_grad, non_blocking=True)
        ev_done[k].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[k])
            dxd.record_stream(s_out)
            dxh.copy_(dxd, non_blocking=True)
            dwh.copy_(dwsnap[b], non_blocking=True)
            if k == n - 1:
                t1.record(s_out)
    t1.synchronize()
    us = t0.elapsed_time(t1) * 1e3 / steps
    torch.cuda.synchronize()
    return us


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", default="all", choices=["all", "none", *SWEEP_GROUPS],
                    help="per-configuration table: every group, none, or one group")
    ap.add_argument("--per-config-out", default=os.path.join(ROOT, "profiles",
                                                             "per_config_b200.json"),
                    help="file the per-configuration table is written to")
    ap.add_argument("--det", action="store_true",
                    help="the step's backward uses deterministic=True")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", type=int, default=HEAD_T, help="T of the headline step")
    ap.add_argument("--width", type=int, default=HEAD_H, help="H of the headline step")
    ap.add_argument("--profile-case", default=None, metavar="OP:H:T[:FORM[:W]]",
                    help="run one call of one configuration three times (L2 flushed before "
                         "each) and exit: the program a profiler capture runs")
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
    if args.profile_case:
        build.build()
        return profile_case(args.profile_case, torch, api, dev)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    build.build()
    peak, peak_kind = peaks()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > L2

    R, H = args.rows, args.width
    x, dy, w = make_inputs(R, H, "bf16", 1234 + rank, dev, torch)
    ws = api.Workspace(dev)
    # the checkpointed training step through the autograd wrapper: the forward, then the
    # backward, which recomputes the forward (torch.utils.checkpoint) and runs the library's
    # backward; dw is added into a float32 main-grad buffer by the accumulate entry point
    from torch.utils.checkpoint import checkpoint
    xg = x.detach().requires_grad_(True)
    main_grad = torch.zeros(H, dtype=torch.float32, device=dev)

    def step(x_leaf, dy_in=None):
        x_leaf.grad = None
        y = checkpoint(api.rmsnorm_train, x_leaf, w, 1e-6, None, args.det, main_grad, ws,
                       use_reentrant=False)
        y.backward(dy if dy_in is None else dy_in)
        return x_leaf.grad

    for _ in range(args.warmup):
        step(xg)
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    evs, bwd_evs = [], []
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with api.record_backward_events(bwd_evs):
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            e0.record()
            step(xg)
            e1.record()
            evs.append((e0, e1))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    api.status(ws)
    if len(bwd_evs) != args.steps:
        raise RuntimeError(f"{len(bwd_evs)} backward calls recorded for {args.steps} steps")
    step_us = [a.elapsed_time(b) * 1e3 for a, b in evs]
    bwd_us = [a.elapsed_time(b) * 1e3 for a, b in bwd_evs]
    ms_step = max_over_ranks(sum(step_us) / len(step_us) / 1e3, dist, dev)
    us_step = ms_step * 1e3
    bwd_avg_us = sum(bwd_us) / len(bwd_us)

    # end to end through the public API (the autograd wrapper) with pinned host buffers: every
    # step's inputs go in from the host and its results (dx and the accumulated dw) come back.
    # The steps run as a pipeline, the way a training loop feeds a GPU: step k+1's inputs are
    # copied in on their own stream (into the other of two device buffers) while step k
    # computes and its results are copied out on a third stream.  Timed from the first timed
    # step's copy-in to the last one's copy-out, divided by the steps.
    e2e_us = e2e_pipelined(torch, step, x, dy, main_grad, args.e2e_steps)
    del xg

    per_cfg = None
    # the per-configuration table is a single-GPU measurement: with several ranks the others
    # would wait for it in the closing barrier
    if args.sweep != "none" and world == 1:
        del x, dy
        torch.cuda.empty_cache()
        per_cfg = sweep(torch, api, flush, peak, dev,
                        SWEEP_GROUPS if args.sweep == "all" else (args.sweep,),
                        device_index=local)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(10.0)

    if rank == 0:
        line = headline_line(dict(
            R=R, H=H, det=bool(args.det), world=world, steps=args.steps, warmup=args.warmup,
            us_step=us_step, bwd_us=bwd_avg_us, e2e_us=e2e_us, peak=peak, peak_kind=peak_kind,
            clocks=clocks, cpu=cpu))
        emit(line, per_cfg, args.per_config_out if per_cfg is not None else None, peak,
             peak_kind, clocks)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
