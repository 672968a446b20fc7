"""Context-parallel decode of long sequences over several GPUs.

"Dual MI50, part 2" (sbm-labs blog), section "Decode: a new kernel for the
shape MTP actually runs": the decode work is split along the context and the
partial results are merged at the end.  Across GPUs the same split becomes:
every rank holds a contiguous run of each sequence's KV blocks (its own
cache pool and block table), computes with paged_attn_decode_partial the
fp32 partial (O, lse) of every query row over its keys only, one all-gather
exchanges the partials (rows x (head_dim + 1) fp32 per rank: about 16.5 KB
per GPU for one 200k-token sequence with 32 query heads), and every rank
merges them with paged_attn_merge.  The KV bytes never cross NVLink; only
the partials do.

The host logic here (partition, exchange, merge) is the same whether the
partials come from the CUDA library (on GPUs, over NCCL) or from another
source (the CPU tests use the fp64 oracle over gloo).
"""
from __future__ import annotations

import numpy as np


def partition(context_len: int, block_size: int, world: int, rank: int) -> tuple[int, int]:
    """Keys [key_begin, key_begin + key_count) of a sequence of length
    context_len that rank `rank` of `world` holds: whole KV blocks, as even
    as whole blocks allow (the first rank gets the first blocks)."""
    nb = -(-int(context_len) // block_size)
    b0 = rank * nb // world
    b1 = (rank + 1) * nb // world
    k0 = b0 * block_size
    k1 = min(int(context_len), b1 * block_size)
    return k0, max(0, k1 - k0)


def local_block_table(block_table_row: np.ndarray, key_begin: int, key_count: int,
                      block_size: int) -> np.ndarray:
    """The rank's block-table row: local block b holds global block
    key_begin / block_size + b."""
    b0 = key_begin // block_size
    nb = -(-key_count // block_size)
    return np.ascontiguousarray(block_table_row[b0: b0 + nb])


def exchange(part_out, part_lse, dist):
    """All-gather of every rank's partials: part_out [rows][D] and part_lse
    [rows] (torch tensors) -> ([world][rows][D], [world][rows]), rank order.
    One collective for both: the log-sum-exps ride as one more column."""
    import torch
    world = dist.get_world_size()
    rows, D = part_out.shape
    packed = torch.cat([part_out, part_lse.reshape(rows, 1)], dim=1).contiguous()
    gathered = torch.empty((world, rows, D + 1), dtype=packed.dtype, device=packed.device)
    if hasattr(dist, "all_gather_into_tensor") and packed.is_cuda:
        dist.all_gather_into_tensor(gathered, packed)
    else:
        parts = list(gathered.unbind(0))
        dist.all_gather(parts, packed)
        gathered = torch.stack(parts, 0)
    return gathered[:, :, :D].contiguous(), gathered[:, :, D].contiguous()


class ContextParallelDecode:
    """One rank's share of a context-parallel decode on the GPU: its local
    KV shard through paged_attn_decode_partial, the all-gather, the merge.

    The local cache pool, block table and key range describe only this
    rank's blocks; context_lens are the sequences' full (global) lengths, so
    that the query positions and masks are the global ones."""

    def __init__(self, *, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                 max_blocks_per_seq, num_blocks, n_query, device=None):
        from . import binding as B
        self.B = B
        self.dec = B.PagedDecode(num_seqs=num_seqs, num_q_heads=num_q_heads,
                                 num_kv_heads=num_kv_heads, head_dim=head_dim,
                                 block_size=block_size, max_blocks_per_seq=max_blocks_per_seq,
                                 num_blocks=num_blocks, n_query=n_query, device=device)

    def partial(self, q, k_cache, v_cache, block_table, context_lens, key_begin, key_count, *,
                causal, window, scale, kv_dtype, stream=None):
        return self.dec.partial(q, k_cache, v_cache, block_table, context_lens, key_begin,
                                key_count, causal=causal, window=window, scale=scale,
                                kv_dtype=kv_dtype, stream=stream)

    def __call__(self, dist, q, k_cache, v_cache, block_table, context_lens, key_begin,
                 key_count, *, causal, window, scale, kv_dtype, stream=None):
        """The full-context output, fp16 [B][nq][Hq][D], on every rank."""
        po, pl = self.partial(q, k_cache, v_cache, block_table, context_lens, key_begin,
                              key_count, causal=causal, window=window, scale=scale,
                              kv_dtype=kv_dtype, stream=stream)
        rows = po.numel() // po.shape[-1]
        go, gl = exchange(po.reshape(rows, -1), pl.reshape(rows), dist)
        out, _ = self.B.merge(go, gl, stream=stream)
        return out.reshape(q.shape)


def bench(args, rank, world, dist):
    """bench.py --split context: the 200k-context decode cut along the
    context over the ranks (each rank holds 1/world of the KV blocks in its
    own HBM), one all-gather of the partials, the merge on every rank.
    Value: the whole sequence's KV bytes over the slowest rank's time per
    step (strong scaling: the total work is fixed)."""
    import os
    import statistics
    import time

    import torch

    from . import inputs as gen
    dev_index = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(dev_index)
    device = torch.device("cuda", dev_index)
    full = gen.decode_200k(0)
    L = int(full.context_lens[0])
    k0, kc = partition(L, full.block_size, world, rank)
    bt_local = local_block_table(full.block_table[0], k0, kc, full.block_size)
    used = bt_local.astype(np.int64)
    # the rank's own pool: only its blocks (compacted), its own table
    k_local = np.ascontiguousarray(full.k_cache[used])
    v_local = np.ascontiguousarray(full.v_cache[used])
    table = np.arange(len(used), dtype=np.int32).reshape(1, -1)
    cp = ContextParallelDecode(num_seqs=1, num_q_heads=full.num_q_heads,
                               num_kv_heads=full.num_kv_heads, head_dim=full.head_dim,
                               block_size=full.block_size, max_blocks_per_seq=table.shape[1],
                               num_blocks=len(used), n_query=full.n_query, device=device)
    t = lambda a: torch.from_numpy(a).to(device)
    q, kc_, vc_, bt = t(full.q), t(k_local), t(v_local), t(table)
    cl = t(full.context_lens)
    kb = torch.tensor([k0], dtype=torch.int32, device=device)
    kn = torch.tensor([kc], dtype=torch.int32, device=device)
    kw = dict(causal=full.causal, window=full.window, scale=full.scale, kv_dtype=full.kv_dtype)
    for _ in range(args.warmup):
        cp(dist, q, kc_, vc_, bt, cl, kb, kn, **kw)
    torch.cuda.synchronize()
    times = []
    for _ in range(max(3, args.reps)):
        dist.barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            cp(dist, q, kc_, vc_, bt, cl, kb, kn, **kw)
        b.record()
        torch.cuda.synchronize()
        dist.barrier()
        x = torch.tensor([a.elapsed_time(b)], dtype=torch.float64, device=device)
        dist.all_reduce(x, op=dist.ReduceOp.MAX)
        times.append(float(x.item()))
    ms = times[0] / args.steps
    kv = gen.visible_kv_bytes(full)
    if rank != 0:
        return None
    return {
        "metric": "µs/call and KV-read HBM GB/s (% of B200 peak) at 61k and 200k context",
        "value": round(kv / (ms * 1e-3) / 1e9, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "us_per_call": round(ms * 1e3, 2), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "ours",
        "config": {"workload": "200k-context decode cut along the context over the ranks: B=1, "
                               "1 query token, Hq/Hkv=32/4, L=196608, fp16; each rank holds "
                               "1/N of the KV blocks, one all-gather of the partials",
                   "kv_bytes_per_step": kv, "parallelism": f"context x{world}"},
        "repeats_us": [round(x * 1e3 / args.steps, 2) for x in times],
        "spread_pct": round(100 * (max(times) - min(times)) / statistics.median(times), 2),
        "gpu_launches": 2 * args.steps,
    }
