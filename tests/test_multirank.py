"""Multi-process host path of bench.py on CPU (gloo, world size 2).

The hot path shards by batch with no data-path collective: each rank runs its
own batch and only the timing is combined (max over ranks). These tests run
that host logic as two gloo processes on the CPU.
"""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    r, w, local = bench.dist_setup(world, backend="gloo")
    assert (r, w, local) == (rank, world, rank)
    bench.barrier(w)
    elapsed = 10.0 + 5.0 * rank                       # rank 1 is the slow one
    slowest = bench.max_over_ranks(elapsed, w, "cpu")
    out[rank] = (slowest, bench.whole_job_rate(w, 16392, 100, slowest), bench.rank_seed(rank, 0))
    dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_batches():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    assert res[0][1] == pytest.approx(2 * 16392 * 100 / 0.015)
    assert res[0][2] != res[1][2]


def test_world_size_must_match():
    os.environ.pop("WORLD_SIZE", None)
    with pytest.raises(SystemExit):
        bench.dist_setup(2)
