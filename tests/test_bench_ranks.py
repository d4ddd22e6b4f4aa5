"""bench.py's multi-rank timing on CPU: two gloo ranks, each with its own
elapsed time; the job's time is the slowest rank's and the throughput counts
the layer's tokens once (the ranks share one layer: strong scaling)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench.barrier(world)
        ms_rank = [400.0, 500.0][rank]          # rank 1 is the slower one
        tps, ms_step = bench.job_throughput(131072, 10, ms_rank, world)
        out.put((rank, bench.max_over_ranks(float(rank), world), tps, ms_step))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, tps, ms_step in res:
        assert mx == 1.0
        assert ms_step == pytest.approx(50.0)
        assert tps == pytest.approx(131072 * 10 / 0.5)
