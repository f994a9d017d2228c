"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by (b, h) with no data-path collective; the only
cross-rank steps are the timing reductions.  These tests run them on two
gloo ranks: the job time is the slowest rank's, the work is all ranks' work,
and every rank draws its own inputs.
"""
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


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    t = bench.max_over_ranks(10.0 + 5.0 * rank, dist)
    s = bench.sum_over_ranks(100.0 * (rank + 1), dist)
    r = bench.whole_job_rate(1e9, 2.0 + rank, dist)
    out[rank] = (t, s, r, bench.rank_seed(1002, rank))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t, s, r, seed = res[rank]
        assert t == 15.0              # slowest rank's time
        assert s == 300.0             # all ranks' work
        assert r == pytest.approx(2e9 / 3e-3)  # 2 ranks x 1e9 units over the slowest 3 ms
    assert res[0][3] != res[1][3]     # distinct inputs per rank
