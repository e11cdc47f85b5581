"""bench.py's multi-rank aggregation on CPU: two gloo ranks, the timing is the max
over ranks and the value counts every rank's units (weak scaling)."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(own_ms, torch.device("cpu"), world)
        value = bench.whole_job_value(1000, world, ms)
        q.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 5.0                        # the slower rank's time, on every rank
        assert value == pytest.approx(2 * 1000 / 0.005)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    assert bench.max_over_ranks(2.5, torch.device("cpu"), 1) == 2.5
    assert bench.whole_job_value(500, 1, 2.0) == pytest.approx(250000.0)
