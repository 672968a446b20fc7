"""The multi-GPU path of bench.py without GPUs: two gloo ranks on the CPU.

bench.py --gpus N runs one independent replica of the workload per rank (the
path partitions into independent problems; no data-path collective) and
reports the whole job's rate over the slowest rank's time.  Checked here: the
max-over-ranks reduction every rank agrees on, the weak-scaling aggregate, and
that the ranks' replicas are distinct seeded inputs of the same shape.
"""
import os
import socket
import sys

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_decode_flash_b200 import inputs as gen
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # per-rank times (ms per step): rank 1 is the slow one
        t = bench.max_over_ranks([3.0, 5.0][rank], dist, "cpu")
        case = gen.CONFIGS["tiny"](seed=rank)  # the rank's replica, as bench.py draws it
        kv = gen.visible_kv_bytes(case)
        dist.barrier()
        out[rank] = (t, bench.job_gbs(kv, world, t * 1e-3), kv, float(case.q.astype(np.float64).sum()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_weak_scaling_aggregate():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    (t0, v0, kv0, q0), (t1, v1, kv1, q1) = res[0], res[1]
    assert t0 == t1 == 5.0                       # every rank reports the slowest rank's time
    assert kv0 == kv1 == 1024 * 2 * 512          # the same workload on every rank
    assert v0 == v1 == pytest.approx(2 * kv0 / 5e-3 / 1e9)
    assert q0 != q1                              # independent seeded replicas


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, None, "cpu") == 7.5
    assert bench.job_gbs(1e9, 1, 1.0) == pytest.approx(1.0)
