"""Multi-rank host logic of bench.py on CPU: gloo, world size 2."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (10 + r) ms per step and (30 - r) ms end to end
        ms, e2e = bench.reduce_max([10.0 + rank, 30.0 - rank], dist)
        out[rank] = (ms, e2e, bench.aggregate(2.0e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_slowest_rank_decides_and_work_adds_up():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        ms, e2e, val = res[r]
        assert ms == 11.0 and e2e == 30.0
        assert val == pytest.approx(2 * 2.0e12 / 11e-3 / 1e12)


def test_reference_arm_exits_on_other_ranks(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    class A:  # minimal args
        warmup, steps, gpus, sparsity, ref_budget = 3, 1, 2, None, 0.1
    from block_sparse_video_rf_b200 import synth
    assert bench.run_reference(A, synth.workload("tiny")) == 0
