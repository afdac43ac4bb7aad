"""The multi-rank path of bench.py on CPU with the gloo backend, world size 2:
each rank runs its own layer, timings are reduced with a max over ranks, and the
whole-job throughput counts every rank's tokens (weak scaling).  There is no
data-path collective to test: heads and layers shard with no exchange."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    import bench
    local = [10.0 + rank, 3.0 * (1 + rank), 1.0]  # this rank's timings
    red = bench.reduce_max_over_ranks(local)
    rk, wd, _ = bench.dist_env()
    out[rank] = (red, rk, wd, bench.whole_job_tokens_per_s(1000, wd, red[0]))
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        red, rk, wd, val = res[rank]
        assert red == [11.0, 6.0, 1.0]
        assert rk == rank and wd == world
        assert val == pytest.approx(1000 * world / 11.0e-3)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_tokens_per_s(32768, 1, 10.0) == pytest.approx(3276800.0)
