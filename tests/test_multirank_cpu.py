"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

Each rank runs an independent batch of the same shape (weak scaling, no
collective on the data path); the step time is the max over ranks and the
reported value counts every rank's tokens.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys

    import numpy as np
    import torch.distributed as dist

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import oracle
    import workloads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        cfg = dict(workloads.CONFIGS["tiny"], T=64)
        cfg_r = bench.rank_config(cfg, rank)
        q, k, v = workloads.make_inputs(cfg_r)
        # each rank's work is self-contained: its own oracle output, no exchange
        o = oracle.direct(q, k, v)
        step_ms = [1.0 + rank, 5.0 - rank]
        mx = bench.reduce_max(step_ms, world)
        value = bench.aggregate_value(cfg["B"] * cfg["T"], world, mx[0])
        out[rank] = (cfg_r["seed"], float(q.sum()), mx, value, float(o[0, 0, 0, 0] - v[0, 0, 0, 0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (s0, q0, mx0, v0, e0), (s1, q1, mx1, v1, e1) = res[0], res[1]
    assert s0 != s1 and q0 != q1              # independent batches per rank
    assert mx0 == mx1 == [2.0, 5.0]           # element-wise max over ranks
    assert v0 == v1 == pytest.approx(2 * 64 / 2.0e-3)
    assert abs(e0) < 1e-12 and abs(e1) < 1e-12  # o_1 = v_1 on each rank


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max([3.0, 4.0], 1) == [3.0, 4.0]
    assert bench.aggregate_value(1000, 1, 2.0) == pytest.approx(5e5)
