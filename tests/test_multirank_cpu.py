"""The multi-process plumbing of bench.py on CPU: two gloo ranks (127.0.0.1)
reduce their timings with MAX and compute the whole-job (weak-scaling)
throughput.  Replicas share no data, so the timing reduction is the only
collective."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local = [10.0 + rank, 5.0 - rank, 7.0 * (rank + 1)]
        got = bench.max_over_ranks(local)
        ws, r, _ = bench.dist_env()
        q.put((rank, got, ws, r))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_with_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, ws, r in res:
        assert got == [11.0, 5.0, 14.0]
        assert ws == 2 and r == rank


def test_job_throughput_is_weak_scaling():
    import bench
    assert bench.job_throughput(1, 10, 5.0, 1000.0) == 50.0
    assert bench.job_throughput(4, 10, 5.0, 1000.0) == 200.0


def test_max_over_ranks_without_process_group_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
