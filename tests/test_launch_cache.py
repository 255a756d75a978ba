"""The library's per-device launch caches (kernel shared-memory grants and occupancy), checked
on the host without a GPU: a small C++ driver over the same header the kernels' launchers use,
compiled with g++ and run here."""

from __future__ import annotations

import os
import subprocess

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_launch_caches_are_keyed_by_device(tmp_path):
    exe = tmp_path / "launch_cache_check"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-pthread",
                           "-I", os.path.join(ROOT, "bwd_rmsnorm_fwd_b200", "csrc"),
                           os.path.join(ROOT, "tests", "native", "launch_cache_check.cpp"),
                           "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
