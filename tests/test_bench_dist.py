"""The multi-rank logic of bench.py on CPU: two gloo ranks agree on the max-over-ranks time
and on the whole-job (weak-scaling) throughput."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, wsize, local = bench.dist_env()
    assert (r, wsize, local) == (rank, world, rank)
    dist = bench.init_dist(wsize, local, backend="gloo", timeout_s=60)
    my_ms = 10.0 + 5.0 * rank                     # rank 1 is the slow one
    mx = bench.max_over_ranks(my_ms, dist)
    value = bench.aggregate_throughput(1000.0, wsize, mx / 1e3)
    out[rank] = (mx, value)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_weak_scaling(world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1]
    mx, value = out[0]
    assert mx == 15.0                               # the slowest rank's time
    assert value == pytest.approx(1000.0 * world / 0.015)   # all ranks' units / slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_dist(1, 0) is None
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.aggregate_throughput(100.0, 1, 2.0) == 50.0
