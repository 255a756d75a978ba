"""Row-sharded deterministic backward on one GPU: the shard call of every rank runs in turn
(no kernel waits on another rank's), their segment sums are put side by side in rank order
and folded, and the result equals the single-GPU deterministic dw of all rows bit for bit,
with each rank's dx equal to those rows of the single-GPU dx.  Also through
torch.distributed with a one-rank NCCL group (the all-gather path), and against the oracle."""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch

import oracle
from bwd_rmsnorm_fwd_b200 import api, synth

from gpu_common import assert_dw, assert_dx, dev_rows, dev_weight, host_bits

pytestmark = pytest.mark.gpu


def _full(T, H, wdt, seed, residual):
    x = synth.rows(seed, "x", T, H, "F3")
    dy = synth.rows(seed, "dy", T, H, "F3")
    w = synth.weight(seed, H, wdt)
    dh = synth.rows(seed, "dh", T, H) if residual else None
    _, rstd = oracle.train_fwd(x, w)
    return x, dy, w, dh, rstd


@pytest.mark.parametrize("world", [2, 4, 16])
@pytest.mark.parametrize("T,H,wdt,residual", [(70001, 2048, "bf16", False),
                                              (9000, 6144, "fp32", False),
                                              (40000, 256, "bf16", False),
                                              (5000, 6144, "bf16", True),
                                              (300, 512, "fp32", False)])
def test_shards_fold_to_the_single_gpu_bits(T, H, wdt, residual, world):
    x, dy, w, dh, rstd = _full(T, H, wdt, 60 + world, residual)
    xd, dyd, wd = dev_rows(x), dev_rows(dy), dev_weight(w)
    dhd = dev_rows(dh) if residual else None
    rs = torch.from_numpy(rstd).cuda()
    dx_ref, dw_ref = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=True, dh=dhd)
    # the shards run the pipelined pair; where the single-GPU call does too, dx agrees bit
    # for bit, else (the single-launch program rounds dx its own way) within the dx budget
    same_program = api.bwd_path(T, 1, H, True) == 2
    dx_oracle = oracle.train_bwd(x, w, rstd, dy, dh=dh, want_dw=False)[0]
    segs = []
    for rank in range(world):
        b, e, _ = api.shard_rows(T, H, rank, world)
        dx, seg = api.rmsnorm_train_bwd_det_shard(
            xd[b:e], wd, rs[b:e], dyd[b:e], T, rank, world,
            dh=dhd[b:e] if residual else None)
        if e > b:
            if same_program:
                assert np.array_equal(host_bits(dx), host_bits(dx_ref[b:e])), rank
            assert_dx(host_bits(dx), dx_oracle[b:e], f"shard dx rank {rank}")
        segs.append(seg)
    table = torch.cat(segs).contiguous()
    dw = api.fold_segments(table, T, H)
    api.status()
    assert np.array_equal(dw.cpu().numpy().view(np.uint32),
                          dw_ref.cpu().numpy().view(np.uint32))
    # accumulate mode of the fold: FP32(prev + dw)
    prev = torch.linspace(-3, 3, H, device="cuda")
    acc = prev.clone()
    api.fold_segments(table, T, H, dw=acc, accumulate=True)
    want = (prev.cpu().numpy() + dw_ref.cpu().numpy()).astype(np.float32)
    assert np.array_equal(acc.cpu().numpy().view(np.uint32), want.view(np.uint32))
    _, dw64 = oracle.train_bwd(x, w, rstd, dy, dh=dh, want_dx=False)
    assert_dw(dw.cpu().numpy(), dw64, f"sharded dw world={world}")


def test_sharded_api_through_a_one_rank_process_group():
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        T, H = 20000, 1536
        x, dy, w, _, rstd = _full(T, H, "bf16", 70, False)
        xd, dyd, wd = dev_rows(x), dev_rows(dy), dev_weight(w)
        rs = torch.from_numpy(rstd).cuda()
        dx, dw = api.rmsnorm_train_bwd_sharded(xd, wd, rs, dyd, T)
        dx_ref, dw_ref = api.rmsnorm_train_bwd(xd, wd, rs, dyd, deterministic=True)
        torch.cuda.synchronize()
        assert np.array_equal(host_bits(dx), host_bits(dx_ref))
        assert np.array_equal(dw.cpu().numpy().view(np.uint32),
                              dw_ref.cpu().numpy().view(np.uint32))
    finally:
        dist.destroy_process_group()
