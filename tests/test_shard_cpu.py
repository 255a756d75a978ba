"""Row-sharded deterministic dw on CPU ranks (gloo, world sizes 2 and 4): every rank takes the
rows the library's shard plan gives it, computes its FP64 segment sums with the IEEE
emulation of the fixed order, the package's all-gather brings every rank the [16, H] table in
rank order, and the folded dw equals the single-process deterministic order bit for bit.
This covers the host side of the sharded path (plan, exchange, fold order); the GPU tests
run the kernels of each rank on one device."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bwd_rmsnorm_fwd_b200 import api, synth

from det_order import (emulate_chunk_partials, emulate_det_dw, emulate_fold_table,
                       emulate_segment_sums)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(T, H):
    x = synth.rows(50, "x", T, H, "F3")
    dy = synth.rows(50, "dy", T, H, "F3")
    rstd = (1.0 + 0.01 * np.random.default_rng(T).standard_normal(T)).astype(np.float32)
    return x, dy, rstd


def _rank_main(rank, world, port, T, H, out):
    import sys
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, dy, rstd = _problem(T, H)
        B, L, S = api.det_plan(T, 1, H)
        n_chunks = -(-T // (B * L))
        seg_len = -(-n_chunks // S)
        b, e, _ = api.shard_rows(T, H, rank, world)
        assert (b == T or b % (B * L) == 0) and (e == T or e % (B * L) == 0)
        if e > b:
            chunks = emulate_chunk_partials(x[b:e], dy[b:e], rstd[b:e], B, L)
        else:
            chunks = np.zeros((0, H))
        seg = emulate_segment_sums(chunks, seg_len, S // world)
        table = api.gather_segments(torch.from_numpy(seg))
        assert tuple(table.shape) == (S, H)
        dw = emulate_fold_table(table.numpy(), -(-n_chunks // seg_len))
        out[rank] = (b, e, dw.view(np.uint32).tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,T,H", [(2, 5000, 256), (4, 3000, 512), (2, 100, 512),
                                       (4, 2100, 1536)])
def test_sharded_fold_equals_single_process_order(world, T, H):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, T, H, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
            assert p.exitcode == 0
        res = dict(out)
    # the ranks' rows tile [0, T) in rank order
    spans = [res[r][:2] for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == T
    for (b0, e0), (b1, e1) in zip(spans, spans[1:]):
        assert e0 == b1
    x, dy, rstd = _problem(T, H)
    B, L, S = api.det_plan(T, 1, H)
    want = emulate_det_dw(x, dy, rstd, B, L, S).view(np.uint32)
    for r in range(world):
        assert np.array_equal(np.array(res[r][2], np.uint32), want), r


def test_shard_plan_rejects_bad_arguments():
    from bwd_rmsnorm_fwd_b200 import _lib
    for rank, world in ((0, 3), (2, 2), (-1, 4), (0, 32)):
        with pytest.raises(_lib.RmsError):
            api.shard_rows(1000, 512, rank, world)
    L = _lib.lib()
    import ctypes
    b = ctypes.c_int64()
    rc = L.rms_det_shard_plan(_lib.shape(100, 4, 256), 0, 2, ctypes.byref(b), None, None)
    assert rc == _lib.RMS_EINVAL  # heads > 1 is not sharded
