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


def _shard_worker(rank, world, port, out):
    import datetime
    import sys

    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import oracle
    import workload
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        g0, g1 = bench.head_shard(rank, world, 4)
        W = workload.make_sink_workload(1, 8, 4, 256, 32, 4, 9.0, seed=77, kv_heads=(g0, g1))
        Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
        _, cr, tot = oracle.attn_emulate(Q8, K8, V8, W.B, W.H, W.Hkv, W.N, W.d, 1, W.scale, 1.0,
                                         0, 64, 4)
        out[rank] = bench.reduce_sum([int(tot[0]), int(tot[1])], world, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_head_sharded_problem_sums_to_the_whole():
    """Strong scaling by kv heads: each rank builds and runs only its heads; the
    all-reduced collapse counts equal those of the whole problem on one process."""
    import numpy as np

    import bench
    import oracle
    import workload
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
    W = workload.make_sink_workload(1, 8, 4, 256, 32, 4, 9.0, seed=77)
    Q8, K8, V8 = (oracle.e4m3_encode(x) for x in (W.q, W.k, W.v))
    _, _, tot = oracle.attn_emulate(Q8, K8, V8, 1, 8, 4, 256, 32, 1, W.scale, 1.0, 0, 64, 4)
    assert out[0] == out[1] == [int(tot[0]), int(tot[1])]
    assert int(np.sum(tot)) > 0
    assert bench.head_shard(1, 4, 8) == (2, 4)
    with pytest.raises(ValueError):
        bench.head_shard(0, 3, 8)
