"""Context-parallel decode across ranks, on the CPU: two and three gloo ranks
each own a contiguous run of a sequence's KV blocks, compute the partials
(O, lse) of every query row over their keys (here with the fp64 oracle in
place of the GPU kernel), exchange them with one all-gather (the product's
exchange()), and merge (oracle_merge).  The merged result equals the
one-pass oracle within 1e-12, on every rank."""
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


def _cases():
    from paged_kv_decode_flash_b200 import inputs as gen
    return [gen.make_case(seed=200, context_lens=(1000,), n_query=4, num_q_heads=8,
                          num_kv_heads=2, causal=1, spike_frac=0.01),
            gen.make_case(seed=201, context_lens=(700,), n_query=8, num_q_heads=4,
                          num_kv_heads=1, causal=0, window=300, block_size=32),
            gen.make_case(seed=202, context_lens=(333,), n_query=3, num_q_heads=6,
                          num_kv_heads=3, causal=1, window=100, kv_dtype=gen.KV_Q8_0)]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import oracle
    from paged_kv_decode_flash_b200 import context_parallel as cp
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        orc = oracle.load()
        res = []
        for case in _cases():
            L = int(case.context_lens[0])
            k0, kc = cp.partition(L, case.block_size, world, rank)
            rows = case.n_query * case.num_q_heads
            po = np.zeros((rows, case.head_dim))
            pl = np.full(rows, -np.inf)
            r = 0
            for i in range(case.n_query):
                for h in range(case.num_q_heads):
                    po[r], pl[r] = orc.attend_row_range(case, 0, i, h, k0, k0 + kc)
                    r += 1
            go, gl = cp.exchange(torch.from_numpy(po), torch.from_numpy(pl), dist)
            assert go.shape == (world, rows, case.head_dim)
            merged, lse = orc.merge(go.numpy(), gl.numpy())
            ref, ref_lse = orc.attend(case)
            res.append((float(np.max(np.abs(merged - ref.reshape(rows, -1)))),
                        float(np.max(np.abs(lse - ref_lse.reshape(rows)))), kc))
        out[rank] = res
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_merge_equals_one_pass(world):
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        for err, lerr, kc in res[rank]:
            assert err < 1e-12 and lerr < 1e-12, (rank, err, lerr)
    # the ranks' key ranges cover each sequence exactly once
    for c, case in enumerate(_cases()):
        assert sum(res[r][c][2] for r in range(world)) == int(case.context_lens[0])


def test_partition_whole_blocks():
    sys.path.insert(0, ROOT)
    from paged_kv_decode_flash_b200 import context_parallel as cp
    for L in (1, 15, 16, 17, 1000, 196608):
        for bs in (16, 32):
            for world in (1, 2, 3, 8):
                spans = [cp.partition(L, bs, world, r) for r in range(world)]
                pos = 0
                for k0, kc in spans:
                    assert k0 % bs == 0 and (kc == 0 or k0 == pos)
                    pos = k0 + kc if kc else pos
                assert sum(kc for _, kc in spans) == L
