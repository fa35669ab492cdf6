"""The multi-process path of bench.py on CPU: two ranks over gloo join through
the torchrun environment, agree on the step count and the slowest rank's time
(max over ranks), and report the whole job's rate.  No GPU."""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    r, w, local = bench.dist_init(world, backend="gloo")
    try:
        assert (r, w, local) == (rank, world, rank)
        # every rank times its own replica; the job uses the slowest
        assert bench.dist_max(1.5 + rank, w) == 1.5 + world - 1
        assert int(bench.dist_max(float(10 + rank), w)) == 10 + world - 1
        bench.barrier(w)
        value, ms_max = bench.job_rate(36, 100, 100.0 + 50.0 * rank, w)
        assert ms_max == 100.0 + 50.0 * (world - 1)
        assert abs(value - world * 36 * 100 / (ms_max / 1000.0)) < 1e-6
    finally:
        dist.destroy_process_group()


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.dist_init(1) == (0, 1, 0)
    assert bench.dist_max(3.0, 1) == 3.0
    value, ms = bench.job_rate(36, 10, 20.0, 1)
    assert ms == 20.0 and abs(value - 36 * 10 / 0.02) < 1e-9


@pytest.mark.parametrize("world", [2])
def test_two_ranks_over_gloo(world):
    import torch.multiprocessing as mp
    mp.spawn(_rank_main, args=(world, _free_port()), nprocs=world, join=True)
