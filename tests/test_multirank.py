"""The N > 1 path of bench.py on CPU: two gloo ranks run the reduction and the
whole-job aggregation that the benchmark uses under torchrun."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        # rank 1 is the slow one for the first entry, rank 0 for the second
        got = bench.max_over_ranks([10.0 + rank, 7.0 - rank], world, "cpu")
        value = bench.job_ms_per_layer(got[0], 5, 3, world)
        # a device condition on rank 1 only: both ranks see it and raise together
        st = bench.status_over_ranks(8 if rank == 1 else 0, world, "cpu")
        clean = bench.status_over_ranks(0, world, "cpu")
        dist.barrier()
        q.put((rank, got, value, st, clean))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_reduce_like_the_benchmark():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, got, value, st, clean in out:
        assert got == [11.0, 7.0]                 # the max over ranks, on every rank
        assert value == pytest.approx(11.0 / 5 / (3 * world))
        assert st != 0 and clean == 0


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([1.5, 2], 1, "cpu") == [1.5, 2.0]
    assert bench.job_ms_per_layer(30.0, 10, 3, 1) == pytest.approx(1.0)
