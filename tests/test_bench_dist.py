"""Multi-rank host logic of bench.py on CPU: two gloo ranks, as torchrun would launch them.
The whole-job value divides the sum of all ranks' work by the max of their timed regions."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench

    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    d = bench.init_group(w, "gloo")
    elapsed = [12.5, 17.0][rank]  # rank 1 is the slow one
    units = [3.0e13, 3.0e13][rank]
    mx, tot = bench.aggregate(d, elapsed, units)
    out[rank] = (mx, tot)
    d.barrier()
    d.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_aggregation_takes_max_time_and_sum_of_work():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0] == res[1] == (17.0, 6.0e13)


def test_single_rank_needs_no_group():
    import bench

    assert bench.init_group(1, "gloo") is None
    assert bench.aggregate(None, 5.0, 7.0) == (5.0, 7.0)
