"""The multi-rank logic of bench.py (barrier, max over ranks, whole-job rate) on 2 gloo ranks (CPU)."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    try:
        bench.dist_init(world, backend="gloo")
        assert bench.dist_env() == (rank, rank, world)
        bench.barrier()
        m = bench.reduce_max(1.5 + rank, torch.device("cpu"))
        # every rank did 10 units; rank 1 was slower (3 s): the job rate is 2 * 10 / 3
        rate = bench.whole_job_rate(10.0, 2.0 + rank, torch.device("cpu"))
        q.put((rank, m, rate))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, m, rate in res:
        assert m == 2.5
        assert rate == pytest.approx(20.0 / 3.0)


def test_single_process_is_identity():
    import bench
    assert bench.reduce_max(3.25, torch.device("cpu")) == 3.25
    assert bench.whole_job_rate(8.0, 2.0, torch.device("cpu")) == 4.0
