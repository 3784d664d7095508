"""The multi-GPU plumbing of bench.py (replicas only: no data-path collective)
on two CPU ranks over gloo: the barrier, the max over ranks and the
whole-job throughput, which divides the units of all ranks by the slowest
rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(world)
        slowest = bench.max_over_ranks(1.0 + rank, world)      # rank 1 is slower
        value = bench.job_throughput(10.0, 2.0 + 3.0 * rank, world)
        bench.barrier(world)
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_replicas_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get() for _ in range(world))
    for rank, slowest, value in got:
        assert slowest == 2.0                       # max over ranks, seen by every rank
        assert value == pytest.approx(10.0 * 2 / 5.0)   # all ranks' units / slowest time


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(8.0, 2.0, 1) == 4.0
