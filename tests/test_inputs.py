"""The seeded input generators (paged_kv_decode_flash_b200/inputs.py) follow
the recipe stated for the configurations: the q8_0 quantisation rule, NaN in
every position no query may read, the sliding window's out-of-window blocks,
the key spikes of the 200k decode, one permuted pool shared by a batch, and
the algorithmic byte count the metric divides by.  CPU only, small shapes
(the recipe code is the same at full size)."""
import dataclasses

import numpy as np
import pytest

from paged_kv_decode_flash_b200 import inputs as gen


def test_q8_0_rule_exactly():
    # d = fp16(amax / 127); q = clamp(round_half_away(x / d), -127, 127)
    g = np.zeros((3, 32), dtype=np.float32)
    g[0, :4] = [127.0, 2.5, -2.5, 0.49]          # amax 127 -> d = 1: ties go away from zero
    g[1, :3] = [-254.0, 3.0, 1.0]                # amax 254 -> d = 2: 3/2 = 1.5 -> 2, 1/2 -> 1
    q, d = gen.quantise_q8_0(g.reshape(1, 96))   # row 2 stays zero: d = 0, q = 0
    q, d = q.reshape(3, 32), d.reshape(3)
    assert d.dtype == np.float16 and q.dtype == np.int8
    assert d.tolist() == [1.0, 2.0, 0.0]
    assert q[0, :4].tolist() == [127, 3, -3, 0]
    assert q[1, :3].tolist() == [-127, 2, 1]
    assert not q[2].any()


def test_q8_0_scale_is_rounded_to_fp16_before_quantising():
    x = np.linspace(-1.0, 1.3, 32, dtype=np.float32)[None]
    q, d = gen.quantise_q8_0(x)
    d64 = float(d.astype(np.float64)[0, 0])
    assert d64 == float(np.float16(1.3 / 127.0))
    expect = np.clip(np.sign(x / d64) * np.floor(np.abs(x / d64) + 0.5), -127, 127)
    assert np.array_equal(q.astype(np.float64), expect)


def test_padding_after_the_context_and_unused_entries_are_nan():
    c = gen.make_case(seed=3, context_lens=(37, 16, 5), n_query=2, num_q_heads=4,
                      num_kv_heads=2, max_blocks_per_seq=4, spare_blocks=2)
    bs = c.block_size
    guard = c.num_blocks - 1
    assert np.isnan(c.k_cache[guard]).all() and np.isnan(c.v_cache[guard]).all()
    for s, L in enumerate(c.context_lens.tolist()):
        nblk = -(-L // bs)
        assert (c.block_table[s, nblk:] == guard).all()      # unused entries -> guard
        for j in range(nblk * bs):
            blk, slot = c.block_table[s, j // bs], j % bs
            row = c.k_cache[blk, :, slot]
            assert np.isnan(row).all() == (j >= L)           # NaN exactly after L
    used = set(c.block_table[c.block_table != guard].tolist())
    assert len(used) == sum(-(-L // bs) for L in c.context_lens.tolist())   # each block once
    spare = [b for b in range(c.num_blocks - 1) if b not in used]
    assert len(spare) == 2 and all(np.isnan(c.k_cache[b]).all() for b in spare)


def test_q8_0_poison_is_a_nan_scale():
    c = gen.make_case(seed=4, context_lens=(20,), n_query=1, num_q_heads=2, num_kv_heads=1,
                      kv_dtype=gen.KV_Q8_0)
    bs = c.block_size
    d = c.k_cache[:, :, bs * 128:].view(np.float16).reshape(c.num_blocks, 1, bs, 4)
    last = c.block_table[0, 1]
    assert np.isfinite(d[last, 0, :4]).all() and np.isnan(d[last, 0, 4:]).all()


def test_sliding_window_blocks_wholly_outside_are_nan():
    L, W = 24 * 16, 64  # the same recipe as the 24576 / 2048 configuration
    c = gen.make_case(seed=5, context_lens=(L,), n_query=8, num_q_heads=4, num_kv_heads=1,
                      causal=0, window=W, nan_below=[L - W])
    table = c.block_table[0]
    n_out = (L - W) // c.block_size
    assert all(np.isnan(c.k_cache[b]).all() for b in table[:n_out])
    assert all(np.isfinite(c.k_cache[b]).all() for b in table[n_out:])


def test_spikes_are_exactly_a_fraction_of_key_rows_per_head():
    L, frac, gain = 2000, 0.01, 8.0
    base = gen.make_case(seed=6, context_lens=(L,), n_query=1, num_q_heads=4, num_kv_heads=2)
    spk = gen.make_case(seed=6, context_lens=(L,), n_query=1, num_q_heads=4, num_kv_heads=2,
                        spike_frac=frac, spike_gain=gain)
    bs = base.block_size
    # draw order: q, K, V, then the spike positions -- q, K and V are the same draws
    assert np.array_equal(base.q.view(np.uint16), spk.q.view(np.uint16))
    for h in range(2):
        scaled = 0
        for j in range(L):
            blk = base.block_table[0, j // bs]
            a = base.k_cache[blk, h, j % bs].astype(np.float64)
            b = spk.k_cache[blk, h, j % bs].astype(np.float64)
            if not np.array_equal(a, b):
                # the whole row x gain before rounding to fp16
                assert np.allclose(b, a * gain, rtol=2e-3, atol=1e-2)
                scaled += 1
        assert scaled == round(frac * L)


def test_mixed_batch_lengths_and_shared_pool():
    rng = np.random.default_rng(0 + 1_000_003)
    lens = rng.integers(4096, 65536, size=8, endpoint=True)
    assert np.all((lens >= 4096) & (lens <= 65536))
    c = gen.make_case(seed=0, context_lens=(300, 17, 129), n_query=4, num_q_heads=8,
                      num_kv_heads=2, kv_dtype=gen.KV_Q8_0, max_blocks_per_seq=30)
    guard = c.num_blocks - 1
    ids = c.block_table[c.block_table != guard]
    assert len(ids) == len(set(ids.tolist()))   # one pool, each block owned once


@pytest.mark.parametrize("causal,window,nq", [(1, 0, 8), (0, 0, 8), (0, 100, 8), (1, 100, 4),
                                              (1, 1, 1)])
def test_visible_kv_bytes_counts_keys_some_query_sees(causal, window, nq):
    c = gen.make_case(seed=7, context_lens=(450, 37), n_query=nq, num_q_heads=4,
                      num_kv_heads=2, causal=causal, window=window)
    total = 0
    for L in c.context_lens.tolist():
        seen = set()
        for i in range(nq):
            p = L - nq + i
            hi = p if causal else L - 1
            lo = max(0, hi - window + 1) if window > 0 else 0
            seen.update(range(lo, hi + 1))
        total += len(seen) * c.num_kv_heads * 2 * c.head_dim * 2
    assert gen.visible_kv_bytes(c) == total


def test_headline_byte_counts():
    def light(**kw):  # the configurations' shapes without building caches
        z = np.zeros(1)
        base = dict(name="x", num_seqs=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
                    block_size=16, max_blocks_per_seq=1, num_blocks=1, n_query=8, causal=1,
                    window=0, kv_dtype=gen.KV_FP16, scale=0.088, q=z, k_cache=z, v_cache=z,
                    block_table=z, context_lens=np.array([1], dtype=np.int32))
        base.update(kw)
        return gen.Case(**base)
    assert gen.visible_kv_bytes(light(context_lens=np.array([61448]))) == 251_691_008
    assert gen.visible_kv_bytes(light(context_lens=np.array([196608]), num_kv_heads=4,
                                      n_query=1)) == 402_653_184
    assert gen.visible_kv_bytes(light(context_lens=np.array([24576]), causal=0,
                                      window=2048)) == 8_388_608
    assert gen.visible_kv_bytes(light(context_lens=np.array([1024]), num_q_heads=8,
                                      num_kv_heads=2, n_query=1)) == 1_048_576
