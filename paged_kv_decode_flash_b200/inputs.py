"""Seeded synthetic inputs for paged-KV decode attention.

This module only makes data: shapes, random values, block tables, NaN
poisoning and the q8_0 *quantiser* that turns N(0,1) samples into a q8_0
cache.  It holds none of the attention arithmetic (no scores, softmax, masks
evaluated per key, dequantisation or merging), so that both the CUDA path and
the fp64 oracle can be fed from it without sharing any of the method.

Workload recipes follow the shapes the pages describe:
  * "Dual MI50, part 2: from 10 to 74 tokens/s, a 200k-token context, and two
    attention kernels" -- section "Decode: a new kernel for the shape MTP
    actually runs" (several query tokens per verify step, several query heads
    per KV head, ~61k-token context), "Bug 2: the drafter read freed memory"
    (2048-token sliding window, non-causal drafter, out-of-window blocks
    filled with NaN in the regression test), "200k context for coding agents"
    (int8 KV to reach 200k tokens).
  * "tps-maxxing on amd gpu" -- section "Baseline" (paged attention is the
    costliest decode kernel and grows with the cache).

Layouts (contiguous, row-major):
  q, out           fp16 [num_seqs][n_query][num_q_heads][head_dim]
  fp16 cache       fp16 [num_blocks][num_kv_heads][block_size][head_dim]
  q8_0 cache       uint8 [num_blocks][num_kv_heads][tile]; tile =
                   int8 qs[block_size][head_dim] then
                   fp16 d[block_size][head_dim // 32]
  int8-row cache   uint8 [num_blocks][num_kv_heads][tile]; tile =
                   int8 qs[block_size][head_dim] then fp32 s[block_size]
  block_table      int32 [num_seqs][max_blocks_per_seq]
  context_lens     int32 [num_seqs]  (includes the n_query new tokens)
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

KV_FP16 = 0
KV_Q8_0 = 1
KV_INT8_ROW = 2


@dataclasses.dataclass
class Case:
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    max_blocks_per_seq: int
    num_blocks: int
    n_query: int
    causal: int
    window: int
    kv_dtype: int
    scale: float  # a float32 value (the C ABI takes float)
    q: np.ndarray
    k_cache: np.ndarray
    v_cache: np.ndarray
    block_table: np.ndarray
    context_lens: np.ndarray

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def rows(self) -> int:
        return self.num_seqs * self.n_query * self.num_q_heads

    def kv_bytes_per_key_head(self) -> int:
        """Bytes of K plus V one key of one KV head occupies in the cache."""
        if self.kv_dtype == KV_FP16:
            return 2 * 2 * self.head_dim
        if self.kv_dtype == KV_Q8_0:
            return 2 * (self.head_dim + 2 * (self.head_dim // 32))
        return 2 * (self.head_dim + 4)


def q8_0_tile_bytes(block_size: int, head_dim: int) -> int:
    return block_size * head_dim + block_size * (head_dim // 32) * 2


def int8_row_tile_bytes(block_size: int, head_dim: int) -> int:
    return block_size * head_dim + block_size * 4


def cache_tile_bytes(kv_dtype: int, block_size: int, head_dim: int) -> int:
    """Bytes per (block, KV head) of a quantised cache."""
    if kv_dtype == KV_Q8_0:
        return q8_0_tile_bytes(block_size, head_dim)
    return int8_row_tile_bytes(block_size, head_dim)


def quantise_q8_0(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantise the last axis (a multiple of 32) in groups of 32.

    d = fp16(amax / 127); q = clamp(round_half_away(x / d), -127, 127);
    an all-zero group gets d = 0, q = 0.  Returns (int8 q, float16 d).
    """
    shp = x.shape
    g = x.astype(np.float64).reshape(shp[:-1] + (shp[-1] // 32, 32))
    amax = np.abs(g).max(axis=-1)
    d16 = (amax / 127.0).astype(np.float16)
    d = d16.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(d > 0, g / np.where(d > 0, d, 1.0), 0.0)
    qv = np.sign(r) * np.floor(np.abs(r) + 0.5)
    qv = np.clip(qv, -127, 127).astype(np.int8).reshape(shp)
    return qv, d16


def quantise_rows(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantise each row (last axis) with one scale: s = fp32(amax / 127);
    q = clamp(round_half_away(x / s), -127, 127); an all-zero row gets s = 0,
    q = 0.  Returns (int8 q, float32 s)."""
    g = x.astype(np.float64)
    amax = np.abs(g).max(axis=-1)
    s32 = (amax / 127.0).astype(np.float32)
    sc = s32.astype(np.float64)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(sc > 0, g / np.where(sc > 0, sc, 1.0), 0.0)
    qv = np.clip(np.sign(r) * np.floor(np.abs(r) + 0.5), -127, 127).astype(np.int8)
    return qv, s32


def pack_int8_rows(qs: np.ndarray, sc: np.ndarray) -> np.ndarray:
    """qs int8 [NB][H][bs][D], sc fp32 [NB][H][bs] -> uint8 tiles."""
    nb, h, bs, dim = qs.shape
    out = np.empty((nb, h, int8_row_tile_bytes(bs, dim)), dtype=np.uint8)
    out[:, :, : bs * dim] = qs.reshape(nb, h, bs * dim).view(np.uint8)
    out[:, :, bs * dim:] = np.ascontiguousarray(sc, dtype=np.float32).reshape(nb, h, bs).view(np.uint8)
    return out


def pack_q8_0(qs: np.ndarray, d: np.ndarray) -> np.ndarray:
    """qs int8 [NB][H][bs][D], d fp16 [NB][H][bs][D/32] -> uint8 tiles."""
    nb, h, bs, dim = qs.shape
    tile = q8_0_tile_bytes(bs, dim)
    out = np.empty((nb, h, tile), dtype=np.uint8)
    out[:, :, : bs * dim] = qs.reshape(nb, h, bs * dim).view(np.uint8)
    out[:, :, bs * dim:] = np.ascontiguousarray(d).reshape(nb, h, -1).view(np.uint8)
    return out


def _normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def make_case(
    *,
    name: str = "custom",
    seed: int = 0,
    context_lens=(64,),
    n_query: int = 1,
    num_q_heads: int = 8,
    num_kv_heads: int = 2,
    head_dim: int = 128,
    block_size: int = 16,
    causal: int = 1,
    window: int = 0,
    kv_dtype: int = KV_FP16,
    scale: float | None = None,
    max_blocks_per_seq: int | None = None,
    spare_blocks: int = 0,
    poison: bool = True,
    nan_below: list[int] | None = None,
    nan_keys_below: list[int] | None = None,
    spike_frac: float = 0.0,
    spike_gain: float = 8.0,
    q_std: float = 1.0,
) -> Case:
    """Build one seeded decode problem.

    Every sequence owns ceil(L/bs) blocks of one shared pool; the pool is a
    seeded random permutation, so logically adjacent blocks are physically
    scattered.  With ``poison`` the spare blocks, the padding slots after L
    in each last block, and one guard block that every unused block_table
    entry points to are filled with NaN: a kernel that reads any of them
    produces NaN.  ``nan_below[s]`` additionally NaN-fills every block of
    sequence s whose keys all lie below that position (used for sliding
    windows).  ``nan_keys_below[s]`` NaN-fills every key of sequence s below
    that position, key by key (also inside a block that holds visible keys).
    ``spike_frac`` scales round(frac * L) seeded key rows per
    (sequence, KV head) by ``spike_gain`` before rounding to fp16.
    """
    rng = np.random.default_rng(seed)
    L = np.asarray(context_lens, dtype=np.int64)
    B = int(L.size)
    bs, D, Hkv, Hq = block_size, head_dim, num_kv_heads, num_q_heads
    nblk = [(int(l) + bs - 1) // bs for l in L]
    if max_blocks_per_seq is None:
        max_blocks_per_seq = max(max(nblk), 1)
    used = int(sum(nblk))
    guard = 1 if poison else 0
    num_blocks = used + spare_blocks + guard
    perm = rng.permutation(used + spare_blocks).astype(np.int32)
    guard_block = num_blocks - 1 if poison else 0
    table = np.full((B, max_blocks_per_seq), guard_block, dtype=np.int32)
    off = 0
    for s in range(B):
        table[s, : nblk[s]] = perm[off: off + nblk[s]]
        off += nblk[s]
    spare = perm[used:]

    if scale is None:
        scale = 1.0 / math.sqrt(D)
    scale = float(np.float32(scale))

    q = (_normal_f32(rng, (B, n_query, Hq, D)) * np.float32(q_std)).astype(np.float16)
    k32 = _normal_f32(rng, (num_blocks, Hkv, bs, D))
    v32 = _normal_f32(rng, (num_blocks, Hkv, bs, D))

    if spike_frac > 0.0:
        for s in range(B):
            n_spk = int(round(spike_frac * int(L[s])))
            for h in range(Hkv):
                pos = rng.choice(int(L[s]), size=n_spk, replace=False)
                blk = table[s, pos // bs]
                k32[blk, h, pos % bs, :] *= np.float32(spike_gain)

    # Positions that must never be read: NaN.
    bad = np.zeros((num_blocks, bs), dtype=bool)
    if poison:
        bad[guard_block, :] = True
        bad[spare, :] = True
        for s in range(B):
            tail = int(L[s]) - (nblk[s] - 1) * bs
            if nblk[s] > 0 and tail < bs:
                bad[table[s, nblk[s] - 1], tail:] = True
    if nan_below is not None:
        for s in range(B):
            lo = int(nan_below[s])
            full = lo // bs  # logical blocks [0, full) end at or below lo - 1
            if full > 0:
                bad[table[s, :full], :] = True
    if nan_keys_below is not None:
        for s in range(B):
            for j in range(min(int(nan_keys_below[s]), int(L[s]))):
                bad[table[s, j // bs], j % bs] = True

    if kv_dtype == KV_FP16:
        k = np.ascontiguousarray(k32.astype(np.float16).transpose(0, 2, 1, 3))  # [NB][bs][H][D]
        v = np.ascontiguousarray(v32.astype(np.float16).transpose(0, 2, 1, 3))
        k[bad] = np.float16(np.nan)  # bad is [NB][bs]: every head, every d
        v[bad] = np.float16(np.nan)
        k = np.ascontiguousarray(k.transpose(0, 2, 1, 3))  # back to [NB][H][bs][D]
        v = np.ascontiguousarray(v.transpose(0, 2, 1, 3))
    elif kv_dtype == KV_INT8_ROW:
        kq, ks = quantise_rows(k32)   # [NB][H][bs][D], [NB][H][bs]
        vq, vs = quantise_rows(v32)
        ks = ks.transpose(0, 2, 1).copy()
        vs = vs.transpose(0, 2, 1).copy()
        ks[bad] = np.float32(np.nan)  # a NaN scale poisons the whole row
        vs[bad] = np.float32(np.nan)
        k = pack_int8_rows(kq, np.ascontiguousarray(ks.transpose(0, 2, 1)))
        v = pack_int8_rows(vq, np.ascontiguousarray(vs.transpose(0, 2, 1)))
    else:
        kq, kd = quantise_q8_0(k32)
        vq, vd = quantise_q8_0(v32)
        # A NaN scale poisons the whole group of 32 values.
        kd = kd.transpose(0, 2, 1, 3).copy()
        vd = vd.transpose(0, 2, 1, 3).copy()
        kd[bad] = np.float16(np.nan)
        vd[bad] = np.float16(np.nan)
        kd = np.ascontiguousarray(kd.transpose(0, 2, 1, 3))
        vd = np.ascontiguousarray(vd.transpose(0, 2, 1, 3))
        k = pack_q8_0(kq, kd)
        v = pack_q8_0(vq, vd)

    return Case(
        name=name, num_seqs=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
        block_size=bs, max_blocks_per_seq=int(max_blocks_per_seq),
        num_blocks=int(num_blocks), n_query=n_query, causal=int(causal),
        window=int(window), kv_dtype=int(kv_dtype), scale=scale, q=q,
        k_cache=k, v_cache=v, block_table=table,
        context_lens=L.astype(np.int32),
    )


def tiny(seed: int = 0) -> Case:
    """batch 1, 1 query token, 8/2 heads, d128, context 1024, bs 16; the
    block_table is the first 64 entries of a seeded permutation of a
    128-block pool whose other 64 blocks are NaN."""
    return make_case(name="tiny", seed=seed, context_lens=(1024,), n_query=1,
                     num_q_heads=8, num_kv_heads=2, spare_blocks=63,
                     poison=True, causal=1)


def spec_verify_61k(seed: int = 0) -> Case:
    """batch 1, 8 causal query tokens after 61440 cached tokens (L = 61448),
    32/8 heads, d128, bs 16, N(0,1)."""
    return make_case(name="spec_verify_61k", seed=seed, context_lens=(61448,),
                     n_query=8, num_q_heads=32, num_kv_heads=8, causal=1)


def sliding_window(seed: int = 0) -> Case:
    """batch 1, 8 non-causal query tokens, window 2048 over 24576 tokens,
    32/8 heads; every block wholly older than the most recent 2048 tokens
    is NaN."""
    L, W = 24576, 2048
    return make_case(name="sliding_window", seed=seed, context_lens=(L,),
                     n_query=8, num_q_heads=32, num_kv_heads=8, causal=0,
                     window=W, nan_below=[L - W])


def decode_200k(seed: int = 0) -> Case:
    """batch 1, 1 query token, 32/4 heads, context 196608, N(0,1) with 1% of
    key rows per KV head scaled x8 before fp16 rounding."""
    return make_case(name="decode_200k", seed=seed, context_lens=(196608,),
                     n_query=1, num_q_heads=32, num_kv_heads=4, causal=1,
                     spike_frac=0.01, spike_gain=8.0)


def mixed_q8_0(seed: int = 0) -> Case:
    """batch 8, 4 causal query tokens each, context lengths uniform in
    [4096, 65536] from the seed, 32/8 heads, q8_0 K/V quantised from N(0,1)."""
    rng = np.random.default_rng(seed + 1_000_003)
    lens = rng.integers(4096, 65536, size=8, endpoint=True)
    return make_case(name="mixed_q8_0", seed=seed, context_lens=tuple(int(x) for x in lens),
                     n_query=4, num_q_heads=32, num_kv_heads=8, causal=1,
                     kv_dtype=KV_Q8_0, max_blocks_per_seq=65536 // 16)


CONFIGS = {
    "tiny": tiny,
    "spec_verify_61k": spec_verify_61k,
    "sliding_window": sliding_window,
    "decode_200k": decode_200k,
    "mixed_q8_0": mixed_q8_0,
}


def visible_kv_bytes(case: Case) -> int:
    """Algorithmic KV bytes: for each sequence and KV head, every key that at
    least one of its queries can see, once, times the bytes per key.  The
    visible span per sequence is [lowest window edge, L); derived from the
    workload description (last n_query positions are the queries)."""
    total = 0
    for L in case.context_lens.tolist():
        if case.window > 0:
            lo = max(0, L - case.n_query - case.window + 1) if case.causal else max(0, L - case.window)
        else:
            lo = 0
        total += (L - lo) * case.num_kv_heads * case.kv_bytes_per_key_head()
    return total
