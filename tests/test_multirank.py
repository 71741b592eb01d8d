"""Host logic of the multi-GPU bench on CPU: two gloo ranks with different
device times and byte counts.  The job's time is the slowest rank's and its
throughput is all ranks' bytes over that time (weak scaling, no collective on
the data path: the only collectives are these scalar reductions)."""
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [10.0, 12.5][rank]
        nbytes = [1e9, 3e9][rank]
        v, t = bench.job_throughput(nbytes, ms, world)
        out.put((rank, v, t, bench.max_over_ranks(float(rank), world), bench.sum_over_ranks(1.0, world),
                 bench.decode_config(world)["parallelism"]))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_bench():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, v, t, mx, sm, par in res:
        assert t == 12.5                            # slowest rank
        assert v == pytest.approx(4e9 / 12.5e-3 / 1e9)  # all bytes / slowest time, GB/s
        assert mx == 1.0 and sm == 2.0
        assert par == "replicas2"


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.sum_over_ranks(3.0, 1) == 3.0
    v, t = bench.job_throughput(2e9, 4.0, 1)
    assert t == 4.0 and v == pytest.approx(500.0)
