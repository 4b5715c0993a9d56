"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The layer's (sequence, head) units are independent, so N GPUs run N
independent batches with no collective on the data path (weak scaling); the
only cross-rank steps are the barrier and the max-over-ranks of the timing,
which these tests exercise with the gloo backend.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench.barrier(world)
        ms = 1.0 + rank  # rank 1 is the slow one
        m = bench.max_over_ranks(ms, world)
        value = bench.weak_scaling_value(10240, m, world)
        out[rank] = (m, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, PORT, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    m, value = res[0]
    assert m == 2.0
    assert value == pytest.approx(2 * 10240 / 2e-3)


PORT = _free_port()


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(100, 2.0, 1) == pytest.approx(50000.0)
