"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): every rank
runs an independent problem (distinct seeds, no data-path collective); the
job's time is the slowest rank's, its value all ranks' work over that time,
and collapse counts add up over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms = bench.reduce_max(10.0 + 5.0 * rank, world, dev)
        counts = bench.reduce_sum([100 + rank, 7 * rank], world, dev)
        out[rank] = (ms, counts, bench.rank_seed(rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    (ms0, c0, s0), (ms1, c1, s1) = out[0], out[1]
    assert ms0 == ms1 == 15.0                       # the slowest rank
    assert c0 == c1 == [201, 7]
    assert s0 != s1                                 # independent problems per rank
    import bench
    flops = bench.algorithmic_flops(1, 32, 32768, 128, True)
    assert bench.job_tflops(flops, 2, 15.0) == pytest.approx(2 * flops / 15e-3 / 1e12)
