"""World-size-2 gloo test (CPU) of the multi-rank host logic of bench.py: every
rank runs its own independent batches (no data-path collective); the job's time
is the max over ranks and the throughput counts the work of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        ms_local = [3.0, 5.0][rank]                 # rank 1 is the slow one
        ms = bench.max_over_ranks(ms_local, ws, device="cpu")
        value = bench.weak_scaling_value(1000, 10, ms, ws)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_two_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(2):
        ms, value = out[r]
        assert ms == 5.0                            # every rank reports the slowest time
        assert value == pytest.approx(2 * 1000 * 10 / 5e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.weak_scaling_value(100, 4, 2.0, 1) == pytest.approx(100 * 4 / 2e-3)
