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


def _fake_table(n=200):
    rows = []
    for i in range(n):
        rows.append({"cfg": "large-T" if i % 2 else "small-T", "form": "plain", "H": 6144,
                     "T": 131072, "w": "bf16", "op": ("fwd", "bwd_det", "bwd_nondet")[i % 3],
                     "us": 700.0 + i, "p10": 690.0, "p90": 720.0, "gbs": 6400.0,
                     "frac": 0.99 - 0.001 * i, "timer": "cupti_span", "replays": 201,
                     "replay_us": 705.0, **({"aa_floor": 0.004} if i % 9 == 0 else {})})
    return rows


def test_headline_line_is_last_short_and_complete(tmp_path):
    """The headline JSON line is the last stdout line, parses, stays under the size limit
    however long the per-configuration table is (the table goes to its own file), and
    carries every key of the bench contract."""
    import io
    cpu = {"value": 2.2e6, "unit": "us", "cores": 16, "kind": "oracle",
           "sample": "131072 of 131072 rows of the headline step (fwd, fwd, bwd), 2.2 s",
           "single_thread": {"value": 3.1e7, "cores": 1, "sample": "9000 of 131072 rows"}}
    clocks = {"sm_mhz": 1965.0, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"],
              "samples": 300, "power_w_max": 900.0}
    line = bench.headline_line(dict(R=bench.HEAD_T, H=bench.HEAD_H, det=False, world=1,
                                    steps=20, warmup=5, us_step=1790.0, bwd_us=745.0,
                                    e2e_us=88000.0, peak=6457.1, peak_kind="measured",
                                    clocks=clocks, cpu=cpu))
    table = _fake_table()
    out = io.StringIO()
    print("some earlier output", file=out)
    path = tmp_path / "per_config.json"
    bench.emit(line, table, str(path), 6457.1, "measured", clocks, stream=out)
    last = out.getvalue().rstrip("\n").splitlines()[-1]
    assert len(last.encode()) <= bench.MAX_LINE_BYTES
    d = json.loads(last)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert k in d, k
    assert d["value"] > 0 and d["metric"] == bench.METRIC
    assert d["config"]["deterministic"] is False and d["config"]["T"] == bench.HEAD_T
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s"
    assert abs(rf["achieved"] - rf["bytes_per_launch"] / (rf["launch_us"] * 1e-6) / 1e9) < 1.0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-3
    assert d["e2e"]["h2d_bytes_per_step"] == 2 * bench.HEAD_T * bench.HEAD_H * 2
    assert d["per_config"]["rows"] == len(table)
    assert d["per_config"]["large_T_min_frac_fwd"] <= 0.99
    assert d["per_config"]["aa_floor_max"] == 0.004
    saved = json.loads(path.read_text())
    assert len(saved["rows"]) == len(table) and saved["peak_gbs"] == 6457.1


def test_oversized_headline_line_is_refused():
    import io
    with pytest.raises(RuntimeError):
        bench.emit({"metric": "x", "blob": "y" * (bench.MAX_LINE_BYTES + 1)}, stream=io.StringIO())


def test_interleaved_rounds_rotate_the_order():
    order = bench.interleaved_order(["a", "b", "c"], rounds=3, reps=2)
    assert order == ["a", "a", "b", "b", "c", "c",
                     "b", "b", "c", "c", "a", "a",
                     "c", "c", "a", "a", "b", "b"]
    assert len(bench.interleaved_order(list(range(10)), 3, 67)) == 10 * 201
    assert bench.quantile([1, 2, 3, 4, 5], 0.5) == 3 and bench.quantile([4.0], 0.9) == 4.0


class _FakeApi:
    """Records the library calls profile_case makes (CPU tensors, no library)."""

    def __init__(self):
        self.calls = []

    class Workspace:
        def __init__(self, dev):
            pass

    def rmsnorm_train_fwd(self, x, w, residual=None):
        self.calls.append(("fwd", tuple(x.shape), residual is not None))
        rstd = torch.ones(x.numel() // x.shape[-1])
        return (x, x, rstd) if residual is not None else (x, rstd)

    def rmsnorm_train_bwd(self, h, w, rstd, dy, deterministic, dh=None, workspace=None):
        self.calls.append(("bwd", tuple(h.shape), deterministic, dh is not None))
        return h, w

    def status(self, ws=None):
        pass


@pytest.mark.parametrize("spec, want, n", [
    ("bwd_det:256:4:24x256_pages", ("bwd", (4, 24, 256), True, False), 3),
    ("bwd_nondet:64:5:res", ("bwd", (5, 64), False, True), 3),
    ("fwd:64:3:plain:fp32", ("fwd", (3, 64), False), 4),  # the setup forward gives rstd
])
def test_profile_case_runs_the_named_call_three_times(spec, want, n):
    api = _FakeApi()
    bench.profile_case(spec, torch, api, torch.device("cpu"))
    assert api.calls.count(want) == n


def test_profile_case_rejects_unknown_op_and_form():
    with pytest.raises(SystemExit):
        bench.profile_case("bwd:64:3", torch, _FakeApi(), torch.device("cpu"))
    with pytest.raises(SystemExit):
        bench.profile_case("fwd:64:3:diag", torch, _FakeApi(), torch.device("cpu"))


def test_clock_sampler_without_a_gpu_reports_nothing():
    """No driver here: the sampler must report no clock rather than raise (the sweep records
    its result per group)."""
    s = bench.ClockSampler(0)
    s.start()
    c = s.stop()
    if not s.ok:
        assert c["sm_mhz"] is None and c["reasons"] == []
