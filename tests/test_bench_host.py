"""Host-side logic of the benchmark, without a GPU: the max-over-ranks reduction of a
replica job (two gloo ranks on CPU), the reference arm's JSON line (the FP64 oracle on the
host cores), and the algorithmic byte counts."""

from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 15.0, 1: 15.0}
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                       timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "us"
    assert d["value"] > 0 and d["higher_is_better"] is False
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_algorithmic_bytes():
    R, H = 131072, 6144
    assert bench.bytes_fwd(R, H, 2) == 4 * R * H + 2 * H + 4 * R
    assert bench.bytes_bwd(R, H, 4) == 6 * R * H + 4 * H + 4 * R + 4 * H
    assert bench.bytes_fwd(R, H, 2, res=True) == 8 * R * H + 2 * H + 4 * R
    assert bench.bytes_bwd(R, H, 2, res=True) == 8 * R * H + 2 * H + 4 * R + 4 * H


def test_call_spans_cut_at_the_flush_kernel():
    """Spans run from a call's first record to its last one; every flush closes a call, and
    overlapping records (a dependent launch that starts before its producer ends) count once."""
    fill = "at::vectorized_elementwise_kernel<4, at::FillFunctor<float>>"
    ev = [(fill, 0.0, 50.0), ("rmsk::main", 51.0, 60.0), ("rmsk::fold", 59.0, 63.5),
          (fill, 70.0, 120.0), ("rmsk::one", 121.0, 125.0),
          (fill, 130.0, 180.0)]
    assert bench.call_spans_us(list(reversed(ev))) == [12.5, 4.0]
    assert bench.call_spans_us([(fill, 0.0, 1.0)]) == []
    assert bench.call_spans_us([("rmsk::k", 2.0, 5.0)]) == [3.0]
