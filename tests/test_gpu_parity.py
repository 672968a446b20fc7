"""GPU parity: libpagedattn (through its C ABI) against the fp64 oracle on the
same seeded inputs, plus bit-exact invariants of the GPU path itself.

Tolerance (tests/parity.py): max-abs 2e-3 and max-rel 1e-2 against
max(|oracle|, 1e-3), on the fp16 output.  Block-index resolution and masking
are checked bit-exactly through the decode kernel's own key-resolution record
(paged_attn_trace), through NaN poisoning of never-visible keys (whole blocks
and key by key) and through closed forms.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
from parity import assert_parity
from paged_kv_decode_flash_b200 import inputs as gen

pytestmark = pytest.mark.gpu

DTYPES = (gen.KV_FP16, gen.KV_Q8_0, gen.KV_INT8_ROW)


@pytest.fixture(scope="module")
def orc():
    return oracle.load()


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_decode_flash_b200 import binding, build
    build.build()  # no-op when the in-tree library is up to date
    binding.lib()
    return binding


def run(B, case):
    out, dec = B.decode_case(case)
    torch.cuda.synchronize()
    assert dec.get_error() == 0
    return out.cpu().numpy(), dec


def zero_nans(case):
    import pins
    return pins.zero_nans(case)


def _args(B, case):
    dev = B.case_to_device(case)
    kw = dict(causal=case.causal, window=case.window, scale=case.scale, kv_dtype=case.kv_dtype)
    return dev, (dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                 dev["context_lens"]), kw


# ---------------------------------------------------------------------------
# small problems, every row against the oracle
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("seed", range(3))
def test_tiny_config(B, orc, seed):
    case = gen.tiny(seed)
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, f"tiny seed {seed}")


def _sweep_cases():
    rng = np.random.default_rng(2024)
    for t in range(48):
        nq = int(rng.choice([1, 2, 3, 4, 5, 8, 12, 16]))
        G = int(rng.choice([1, 2, 4, 6, 8]))
        while nq * G > 64:
            G = max(1, G // 2) if G > 1 else G
            if nq * G > 64:
                nq //= 2
        Hkv = int(rng.choice([1, 2, 3]))
        bs = int(rng.choice([16, 32, 64]))
        causal = int(rng.integers(0, 2))
        window = int(rng.choice([0, 0, 1, 7, 100, 513]))
        dt = DTYPES[t % 3]
        nseq = int(rng.integers(1, 4))
        lens = [int(x) for x in rng.integers(nq, 1500, size=nseq)]
        if t % 7 == 0:
            lens[0] = nq  # the shortest legal context
        extra = int(rng.integers(0, 3))
        mbps = max((l + bs - 1) // bs for l in lens) + extra
        yield gen.make_case(seed=5000 + t, context_lens=tuple(lens), n_query=nq,
                            num_q_heads=Hkv * G, num_kv_heads=Hkv, block_size=bs,
                            causal=causal, window=window, kv_dtype=dt, spare_blocks=3,
                            max_blocks_per_seq=mbps)


def _case_id(c):
    return (f"B{c.num_seqs}_nq{c.n_query}_G{c.group}_Hkv{c.num_kv_heads}"
            f"_bs{c.block_size}_c{c.causal}_w{c.window}_dt{c.kv_dtype}")


@pytest.mark.parametrize("case", list(_sweep_cases()), ids=_case_id)
def test_random_sweep(B, orc, case):
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, "sweep")


@pytest.mark.parametrize("tiles,dt,nq,G", [(2, gen.KV_FP16, 8, 4), (3, gen.KV_FP16, 1, 8),
                                          (5, gen.KV_FP16, 4, 4), (2, gen.KV_Q8_0, 4, 4),
                                          (4, gen.KV_Q8_0, 1, 8), (3, gen.KV_INT8_ROW, 2, 8)])
def test_several_tiles_per_cta(B, orc, tiles, dt, nq, G):
    """One long sequence over a few KV heads: every CTA's range holds several
    128-key tiles and, as the KV heads are laid end to end, some ranges run
    from one KV head into the next (two segments in one pipeline).  Key
    spikes make rows raise their running maximum after the first tile (the
    accumulated output is rescaled in place).  Every row against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    Hkv = 3
    L = (sms * 128 * tiles) // Hkv - 37  # about `tiles` tiles per CTA, ragged ends
    case = gen.make_case(seed=40 + tiles, context_lens=(L,), n_query=nq, num_q_heads=G * Hkv,
                         num_kv_heads=Hkv, causal=1, kv_dtype=dt, spike_frac=0.003,
                         spike_gain=6.0, max_blocks_per_seq=(L + 15) // 16)
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, f"{tiles} tiles per CTA")


@pytest.mark.parametrize("dt", DTYPES)
def test_pages_mtp_shape_and_wide_verify(B, orc, dt):
    """The pages' decode shape: 4 query tokens x 6 query heads per KV head =
    24 rows over an int8 cache ("Decode: a new kernel for the shape MTP
    actually runs"), and an 8-token verify at GQA 8 (64 rows), at a context
    of several tiles per CTA; every row against the oracle."""
    for nq, G, L in ((4, 6, 20000), (8, 8, 12000)):
        case = gen.make_case(seed=90 + nq, context_lens=(L,), n_query=nq, num_q_heads=4 * G,
                             num_kv_heads=4, causal=1, kv_dtype=dt, spike_frac=0.002)
        dec = B.PagedDecode.for_case(case)
        assert dec.launches_per_call(dt) == 1
        out, _ = run(B, case)
        ref, _ = orc.attend(case)
        assert_parity(out, ref, f"{nq} tokens x GQA {G}, dt {dt}")


def test_sixteen_token_verify(B, orc):
    """n_query = 16 (a 15-token draft verified in one step), GQA 4: 64 rows
    per KV head, causal among themselves, with and without a window."""
    for window in (0, 300):
        for dt in DTYPES:
            case = gen.make_case(seed=95, context_lens=(5000, 777), n_query=16, num_q_heads=16,
                                 num_kv_heads=4, causal=1, window=window, kv_dtype=dt)
            out, _ = run(B, case)
            ref, _ = orc.attend(case)
            assert_parity(out, ref, f"nq 16 window {window} dt {dt}")


@pytest.mark.parametrize("dt", DTYPES)
def test_chunked_prefill_of_many_tokens(B, orc, dt):
    """A chunk of 64 new tokens appended to the cache (chunked prefill),
    GQA 4: 256 rows per KV head in 8 (fp16) or 16 (int8) row parts, each
    over the keys its tokens see, causal, with and without a window; and
    128 tokens x 8 query heads per KV head (1024 rows, the most) on a short
    context.  Every row against the oracle."""
    for nq, Hq, Hkv, lens, window in ((64, 16, 4, (2500, 300), 0), (64, 16, 4, (2500, 300), 700),
                                      (128, 8, 1, (400,), 0)):
        case = gen.make_case(seed=170 + nq + window, context_lens=lens, n_query=nq,
                             num_q_heads=Hq, num_kv_heads=Hkv, causal=1, window=window,
                             kv_dtype=dt)
        out, _ = run(B, case)
        ref, _ = orc.attend(case)
        assert_parity(out, ref, f"nq {nq} rows {nq * Hq // Hkv} window {window} dt {dt}")


@pytest.mark.parametrize("bs,dt", [(48, gen.KV_FP16), (80, gen.KV_Q8_0), (112, gen.KV_FP16),
                                   (96, gen.KV_INT8_ROW)])
def test_block_sizes_that_do_not_divide_a_tile(B, orc, bs, dt):
    """Blocks of 48-112 keys: a 128-key tile spans parts of two blocks;
    every row against the oracle."""
    case = gen.make_case(seed=80 + bs, context_lens=(bs * 100 - 5,), n_query=4, num_q_heads=8,
                         num_kv_heads=1, block_size=bs, causal=1, window=bs * 37, kv_dtype=dt,
                         spare_blocks=3)
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, f"block_size {bs}")


def test_sliding_window_config_and_nan_invariance(B, orc):
    case = gen.sliding_window(0)
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, "sliding window")
    # the 1408 out-of-window blocks hold NaN; zeroing them changes no bit
    out2, _ = run(B, zero_nans(case))
    assert np.array_equal(out.view(np.uint16), out2.view(np.uint16))


@pytest.mark.parametrize("dt", DTYPES)
@pytest.mark.parametrize("causal", [0, 1])
def test_key_granular_nan_poisoning(B, orc, dt, causal):
    """Every key no query may see is NaN -- key by key, also inside the
    block that holds the first visible key (the pages' regression test fills
    out-of-window memory with NaN; "Bug 2: the drafter read freed memory").
    The output is finite, matches the oracle and is bit-identical to a run
    with those keys zeroed."""
    W, nq = 300, 8
    lens = (2000, 1337, 555)
    lo = [(L - W) if not causal else (L - nq - W + 1) for L in lens]
    case = gen.make_case(seed=120 + dt, context_lens=lens, n_query=nq, num_q_heads=16,
                         num_kv_heads=4, causal=causal, window=W, kv_dtype=dt,
                         nan_keys_below=lo, spare_blocks=2)
    assert all(l % 16 != 0 for l in lo)  # the edge falls inside a 16-key chunk
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, "key-granular NaN")
    out2, _ = run(B, zero_nans(case))
    assert np.array_equal(out.view(np.uint16), out2.view(np.uint16))


def test_single_key_is_bit_exact(B):
    import pins
    for dt in DTYPES:
        case = gen.make_case(seed=7, context_lens=(1, 1), n_query=1, num_q_heads=8,
                             num_kv_heads=2, kv_dtype=dt, spare_blocks=4)
        out, _ = run(B, case)
        for s in range(2):
            V = pins.dense_kv(case, s, "v")
            for h in range(8):
                want = V[h // 4, 0].astype(np.float16)  # the value rounded once to fp16
                assert np.array_equal(out[s, 0, h].view(np.uint16), want.view(np.uint16)), dt


def test_window_one_returns_own_value(B):
    import pins
    case = gen.make_case(seed=8, context_lens=(300,), n_query=4, num_q_heads=4,
                         num_kv_heads=1, causal=1, window=1)
    out, _ = run(B, case)
    V = pins.dense_kv(case, 0, "v")[0]
    for i in range(4):
        for h in range(4):
            assert np.array_equal(out[0, i, h].view(np.uint16),
                                  V[300 - 4 + i].astype(np.float16).view(np.uint16))


@pytest.mark.parametrize("dt", DTYPES)
def test_block_permutation_bit_identical(B, dt):
    case = gen.make_case(seed=9, context_lens=(2000, 777), n_query=4, num_q_heads=16,
                         num_kv_heads=4, causal=1, window=900, spare_blocks=10, kv_dtype=dt)
    out, _ = run(B, case)
    perm = np.random.default_rng(1).permutation(case.num_blocks)
    k2 = np.empty_like(case.k_cache); k2[perm] = case.k_cache
    v2 = np.empty_like(case.v_cache); v2[perm] = case.v_cache
    c2 = gen.Case(**{**case.__dict__, "k_cache": k2, "v_cache": v2,
                     "block_table": perm[case.block_table].astype(np.int32)})
    out2, _ = run(B, c2)
    assert np.array_equal(out.view(np.uint16), out2.view(np.uint16))


def test_sequence_independent_of_neighbours(B):
    """Each sequence's output depends only on its own data (the varlen
    indexing bug in 'Flash-Next (vLLM)' on the gfx1030 wiki reused a global
    chunk index): change the other sequences' lengths and values, keep the
    shapes, and sequence 1 must not change by a bit."""
    a = gen.make_case(seed=10, context_lens=(500, 1200, 64), n_query=3, num_q_heads=8,
                      num_kv_heads=2, causal=1, max_blocks_per_seq=80)
    out_a, _ = run(B, a)
    b = gen.Case(**a.__dict__)
    b.context_lens = a.context_lens.copy()
    b.context_lens[0], b.context_lens[2] = 3, 1279
    b.q = a.q.copy(); b.q[0] = -a.q[0]; b.q[2] = a.q[2] * 2
    rows_other = [bb for s in (0, 2) for bb in a.block_table[s] if bb != a.num_blocks - 1]
    b.k_cache = a.k_cache.copy(); b.v_cache = a.v_cache.copy()
    b.k_cache[rows_other] = 0.5; b.v_cache[rows_other] = -0.25
    b.block_table = a.block_table.copy()
    out_b, _ = run(B, b)
    assert np.array_equal(out_a[1].view(np.uint16), out_b[1].view(np.uint16))


@pytest.mark.parametrize("dt", DTYPES)
def test_batched_items_every_row(B, orc, dt):
    """Many (sequence, KV head) groups: each group's tiles are cut into items
    taken from a queue (the last item of a group in smaller pieces), and the
    CTA that completes a group merges it.  Ragged lengths (one shorter than a
    tile, one with an item boundary inside), every row against the oracle."""
    lens = (3000, 77, 2049, 1, 2500, 640, 4100)
    case = gen.make_case(seed=60 + dt, context_lens=tuple(max(l, 2) for l in lens), n_query=2,
                         num_q_heads=32, num_kv_heads=8, causal=1, kv_dtype=dt, spike_frac=0.002,
                         spike_gain=5.0)
    dec = B.PagedDecode.for_case(case)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert case.num_seqs * case.num_kv_heads * 4 > sms  # the work queue
    assert dec.num_splits(dt) > 1
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    assert_parity(out, ref, f"batched items dt={dt}")


def test_batched_items_sequence_independent_of_neighbours(B):
    """The item size comes from the shapes alone: other sequences' lengths
    and data do not change a sequence's output by a bit."""
    a = gen.make_case(seed=61, context_lens=(2500, 3900, 300, 4000, 10), n_query=4,
                      num_q_heads=32, num_kv_heads=8, causal=1, max_blocks_per_seq=260)
    out_a, _ = run(B, a)
    b = gen.Case(**a.__dict__)
    b.context_lens = a.context_lens.copy()
    b.context_lens[0], b.context_lens[2], b.context_lens[4] = 4100, 9, 3333
    b.q = a.q.copy(); b.q[3] = -a.q[3]
    out_b, _ = run(B, b)
    assert np.array_equal(out_a[1].view(np.uint16), out_b[1].view(np.uint16))


def test_large_batch_several_queue_launches(B, orc):
    """More sequences than one work-queue launch takes (256): the call makes
    one launch per 256 sequences, each with its own counters; every row of
    a sample of sequences against the oracle, the rest finite."""
    lens = tuple(int(x) for x in np.random.default_rng(62).integers(20, 400, size=300))
    case = gen.make_case(seed=62, context_lens=lens, n_query=1, num_q_heads=8, num_kv_heads=2,
                         causal=1)
    dec = B.PagedDecode.for_case(case)
    assert dec.launches_per_call(0) == 2
    out, _ = run(B, case)
    rows = np.array([r for s in (0, 1, 255, 256, 299) for r in range(s * 8, s * 8 + 8)])
    ref, _ = orc.attend_rows(case, rows)
    assert_parity(out.reshape(-1, 128)[rows], ref, "two queue launches")
    assert np.all(np.isfinite(out))


def _q8_scales(cache, bs):
    """The fp16 scales [NB][Hkv][bs][4] of a q8_0 cache held as bytes
    [NB][Hkv][bs * 136] (a view: writing it edits the cache)."""
    nb, h = cache.shape[0], cache.shape[1]
    return cache[:, :, bs * 128:].view(np.float16).reshape(nb, h, bs, 4)


def test_q8_0_extreme_scales(B, orc):
    """q8_0 scales across the range the kernel supports: V groups scaled to
    scales up to 512 (values up to 127 * 512 = 65024), 2^-10 (subnormal
    scales), 3 and 1; K groups by 1, 2^5, 2^-6 and 1.5.  Every row against
    the oracle, each V group's output dims rescaled back by the same factor
    on both sides before the comparison."""
    case = gen.make_case(seed=70, context_lens=(1500, 333, 2600), n_query=4, num_q_heads=16,
                         num_kv_heads=4, causal=1, kv_dtype=gen.KV_Q8_0, spare_blocks=2)
    vf = np.array([2.0 ** 14, 2.0 ** -10, 3.0, 1.0])
    kf = np.array([1.0, 2.0 ** 5, 2.0 ** -6, 1.5])
    for cache, f in ((case.k_cache, kf), (case.v_cache, vf)):
        d = _q8_scales(cache, case.block_size)
        d[...] = (d.astype(np.float64) * f).astype(np.float16)
    dv = _q8_scales(case.v_cache, case.block_size)
    dv[..., 0] = np.minimum(dv[..., 0].astype(np.float64), 512.0).astype(np.float16)
    dv64 = dv.astype(np.float64)
    assert np.nanmax(np.abs(dv64)) <= 512 and np.nanmax(np.abs(dv64[..., 0])) > 256
    assert np.nanmin(np.abs(dv64[..., 1][dv64[..., 1] != 0])) < 2.0 ** -14  # subnormal scales
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    # Back to unit size; the subnormal group only by 2^4, since outputs below
    # fp16's normal range carry a rounding error that a larger factor would
    # blow past the relative tolerance.
    back = np.repeat([2.0 ** -14, 2.0 ** 4, 1.0 / 3.0, 1.0], 32)  # per head_dim element
    assert_parity(out.astype(np.float64) * back, ref * back, "q8_0 extreme scales")


def test_int8_row_scales_across_range(B, orc):
    """int8 with fp32 row scales from 2^-12 to 512 (values up to 65024):
    every row against the oracle after scaling both sides back per row of
    V's scale class."""
    case = gen.make_case(seed=71, context_lens=(1800, 900), n_query=4, num_q_heads=16,
                         num_kv_heads=4, causal=1, kv_dtype=gen.KV_INT8_ROW, spare_blocks=2)
    bs = case.block_size
    for name, f in (("k_cache", 2.0 ** -3), ("v_cache", 0.0)):
        c = getattr(case, name)
        sc = c[:, :, bs * 128:].view(np.float32).reshape(c.shape[0], c.shape[1], bs)
        if name == "k_cache":
            sc[...] = sc * np.float32(f)
        else:  # every KV head a different scale class
            for h, m in enumerate([2.0 ** 14, 2.0 ** -8, 3.0, 1.0]):
                sc[:, h] = np.minimum(sc[:, h].astype(np.float64) * m, 512.0).astype(np.float32)
    out, _ = run(B, case)
    ref, _ = orc.attend(case)
    back = np.repeat([2.0 ** -14, 2.0 ** 8, 1.0 / 3.0, 1.0], 4)  # per query head (GQA 4)
    assert_parity(out.astype(np.float64) * back[None, None, :, None],
                  ref * back[None, None, :, None], "int8 row scales")


def test_batch_matches_each_sequence_alone(B, orc):
    case = gen.make_case(seed=11, context_lens=(900, 33, 2500, 8), n_query=2,
                         num_q_heads=8, num_kv_heads=2, causal=1)
    out, _ = run(B, case)
    for s in range(4):
        c1 = gen.Case(**{**case.__dict__, "num_seqs": 1, "q": case.q[s:s + 1].copy(),
                         "block_table": case.block_table[s:s + 1].copy(),
                         "context_lens": case.context_lens[s:s + 1].copy()})
        o1, _ = run(B, c1)
        ref, _ = orc.attend(c1)
        assert_parity(out[s:s + 1], ref, f"batch seq {s}")
        assert_parity(o1, ref, f"alone seq {s}")


def _trace_cases():
    yield gen.tiny(0)
    yield gen.sliding_window(0)
    yield from list(_sweep_cases())[:24]
    # the work queue (many groups), row parts, key-granular NaN below the window
    yield gen.make_case(seed=130, context_lens=(3000, 77, 2049, 1200, 640), n_query=2,
                        num_q_heads=32, num_kv_heads=8, causal=1, kv_dtype=gen.KV_Q8_0)
    yield gen.make_case(seed=131, context_lens=(9000,), n_query=8, num_q_heads=32,
                        num_kv_heads=4, causal=1, window=2500, kv_dtype=gen.KV_INT8_ROW)
    yield gen.make_case(seed=132, context_lens=(6000, 333), n_query=16, num_q_heads=16,
                        num_kv_heads=4, causal=0, window=1000, nan_keys_below=[5000, 0])
    # a prefill chunk: 40 tokens x 4 heads = 160 rows in five parts
    yield gen.make_case(seed=133, context_lens=(1500,), n_query=40, num_q_heads=8,
                        num_kv_heads=2, causal=1, window=600)


def test_decode_kernel_trace_is_bit_exact(B, orc):
    """The decode kernel's own record of every (row, key) pair it scored and
    the physical slot it copied that key's K row from -- count, first and
    last key, xor and sum of the slot ids -- equals the oracle's, bit for
    bit, over both kernels (the per-head split kernel: fp16, few groups, up
    to 8 tokens and 32 rows; the segment kernel: the rest) and every
    configuration (fp16 / q8_0 / int8 rows, few groups / work queue, one or
    several row parts).  The traced call's output is bit-identical to the
    plain call's."""
    for case in _trace_cases():
        dev, args, kw = _args(B, case)
        dec = B.PagedDecode.for_case(case)
        out_t, t = dec.trace(*args, **kw)
        out = dec(*args, **kw)
        torch.cuda.synchronize()
        assert dec.get_error() == 0
        got = t.cpu().numpy().reshape(-1, 5)
        assert np.array_equal(got, orc.trace(case)), _case_id(case)
        assert torch.equal(out_t.view(torch.int16), out.view(torch.int16)), _case_id(case)


def test_merge_entry_point(B, orc):
    rng = np.random.default_rng(12)
    for S, rows in ((1, 5), (7, 33), (148, 64)):
        po = rng.standard_normal((S, rows, 128)).astype(np.float32)
        pl = (rng.standard_normal((S, rows)) * 20).astype(np.float32)
        pl[rng.random((S, rows)) < 0.2] = -np.inf  # empty splits
        if rows > 1:
            pl[:, 1] = -np.inf  # a row no split saw
        po[pl == -np.inf] = np.nan  # an empty split's output is never read
        out, lse = B.merge(torch.from_numpy(po).cuda(), torch.from_numpy(pl).cuda())
        ref, ref_lse = orc.merge(np.nan_to_num(po, nan=0.0).astype(np.float64), pl.astype(np.float64))
        assert_parity(out.cpu().numpy(), ref, f"merge S={S}")
        l = lse.cpu().numpy()
        fin = np.isfinite(ref_lse)
        assert np.array_equal(np.isfinite(l), fin)
        assert np.max(np.abs(l[fin] - ref_lse[fin])) < 1e-4


@pytest.mark.parametrize("dt", DTYPES)
def test_bad_block_index_is_flagged(B, dt):
    case = gen.make_case(seed=13, context_lens=(200, 300), n_query=1, num_q_heads=4,
                         num_kv_heads=1, kv_dtype=dt)
    case.block_table[0, 3] = case.num_blocks + 5
    out, dec = B.decode_case(case)
    assert dec.get_error() == B.PA_ERR_BAD_BLOCK_INDEX
    assert dec.get_error() == 0  # cleared by the read
    o = out.cpu().numpy()
    assert np.all(o[0] == 0)  # the rows that reached the bad block
    assert np.all(np.isfinite(o))


def test_bad_context_len_is_flagged_and_rows_zeroed(B):
    case = gen.make_case(seed=14, context_lens=(100, 50), n_query=4, num_q_heads=4,
                         num_kv_heads=1, max_blocks_per_seq=7)
    case.context_lens[1] = 7 * 16 + 1  # beyond the table's capacity
    out, dec = B.decode_case(case)
    assert dec.get_error() == B.PA_ERR_BAD_CONTEXT_LEN
    o = out.cpu().numpy()
    assert np.all(o[1] == 0)
    case.context_lens[1] = 3  # fewer keys than query tokens
    out, dec = B.decode_case(case)
    assert dec.get_error() == B.PA_ERR_BAD_CONTEXT_LEN


def test_cuda_graph_replay_matches_eager(B):
    case = gen.make_case(seed=15, context_lens=(3000,), n_query=8, num_q_heads=32,
                         num_kv_heads=8, causal=1)
    dev, args, kw = _args(B, case)
    dec = B.PagedDecode.for_case(case)
    eager = dec(*args, **kw)
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        dec(*args, out=out, stream=s, **kw)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dec(*args, out=out, stream=torch.cuda.current_stream(), **kw)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))


def test_split_kernel_gives_every_kv_head_the_same_ctas(B):
    """fp16 calls with few (sequence, KV head) groups run the per-head split
    kernel with the same number of CTAs for every group -- SMs // groups,
    at least one, at most one per 128-key tile of a full table -- so that no
    head with one CTA fewer finishes last while the others idle."""
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    # (B, Hq, Hkv, max_blocks_per_seq, n_query) at block size 16: the 61k
    # verify, the 200k decode, the tiny and sliding-window calls, two
    # sequences with short tables
    for nseq, hq, hkv, mbps, nq in ((1, 32, 8, 3841, 8), (1, 32, 4, 12288, 1), (1, 8, 2, 64, 1),
                                    (1, 32, 8, 1536, 8), (2, 16, 4, 100, 4)):
        groups = nseq * hkv
        dec = B.PagedDecode(num_seqs=nseq, num_q_heads=hq, num_kv_heads=hkv, head_dim=128,
                            block_size=16, max_blocks_per_seq=mbps, num_blocks=nseq * mbps,
                            n_query=nq)
        max_tiles = -(-mbps // 8)
        assert dec.num_splits(B.KV_FP16) == max(1, min(sms // groups, max_tiles)), \
            (nseq, hq, hkv, mbps, nq)


@pytest.mark.parametrize("name", ["spec_verify_61k", "mixed_q8_0"])
def test_waits_that_time_out_leave_the_workspace_usable(B, orc, name):
    """A wait limit the pipeline cannot meet (1 ns): every kernel gives up
    through its bounded waits -- no fault, no hang -- the call reports
    PA_ERR_TIMEOUT, and the next call on the same workspace, with the
    default limit back, matches the oracle (sampled rows)."""
    case = gen.CONFIGS[name](0)
    dev, args, kw = _args(B, case)
    dec = B.PagedDecode.for_case(case)
    prev = B.set_wait_limit(1)
    try:
        dec(*args, **kw)
        torch.cuda.synchronize()
    finally:
        B.set_wait_limit(prev)
    assert dec.get_error() == B.PA_ERR_TIMEOUT
    for _ in range(2):  # and again, to see the counters were left consistent
        out = dec(*args, **kw)
        torch.cuda.synchronize()
        assert dec.get_error() == 0
    rows = np.arange(0, case.rows, max(1, case.rows // 48))
    ref, _ = orc.attend_rows(case, rows)
    assert_parity(out.cpu().numpy().reshape(-1, 128)[rows], ref, "after a timeout")


@pytest.mark.parametrize("dt", DTYPES)
def test_cache_write_is_bit_exact(B, orc, dt):
    """Writing the newest tokens' K and V into the paged cache (quantised on
    the way for the int8 caches) gives byte for byte the oracle's cache, for
    rows whose magnitudes span 1e-3 to 30; decode on a cache written with
    N(0,1) rows then matches the oracle (outputs of order one, where the
    fp16 output itself can meet the absolute tolerance)."""
    case = gen.make_case(seed=140 + dt, context_lens=(700, 129, 16), n_query=4, num_q_heads=16,
                         num_kv_heads=4, kv_dtype=dt, spare_blocks=3, causal=1)
    rng = np.random.default_rng(141)
    dec = B.PagedDecode.for_case(case)
    for scaled in (True, False):
        scale = rng.choice([1e-3, 1.0, 30.0], size=(3, 4, 4, 1)) if scaled else 1.0
        kn = (rng.standard_normal((3, 4, 4, 128)) * scale).astype(np.float16)
        vn = (rng.standard_normal((3, 4, 4, 128)) * scale).astype(np.float16)
        kc_ref, vc_ref, rc = orc.cache_write(case, kn, vn)
        assert rc == 0
        dev, args, kw = _args(B, case)
        dec.cache_write(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                        dev["block_table"], dev["context_lens"], kv_dtype=dt,
                        k_cache=dev["k_cache"], v_cache=dev["v_cache"])
        torch.cuda.synchronize()
        assert dec.get_error() == 0
        kc, vc = dev["k_cache"].cpu().numpy(), dev["v_cache"].cpu().numpy()
        assert np.array_equal(kc.view(np.uint8), kc_ref.view(np.uint8))
        assert np.array_equal(vc.view(np.uint8), vc_ref.view(np.uint8))
    written = gen.Case(**{**case.__dict__, "k_cache": kc_ref, "v_cache": vc_ref})
    out = dec(*args, **kw)
    torch.cuda.synchronize()
    ref, _ = orc.attend(written)
    assert_parity(out.cpu().numpy(), ref, "decode after the write")
    # a block index out of range: that row is not written, the flag is raised
    case.block_table[1, 128 // 16] = case.num_blocks + 1
    dev2 = B.case_to_device(case)
    dec.cache_write(torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                    dev2["block_table"], dev2["context_lens"], kv_dtype=dt,
                    k_cache=dev2["k_cache"], v_cache=dev2["v_cache"])
    assert dec.get_error() == B.PA_ERR_BAD_BLOCK_INDEX


# ---------------------------------------------------------------------------
# full-size workloads: every row against the oracle
# ---------------------------------------------------------------------------
@pytest.mark.slow
@pytest.mark.parametrize("name", ["spec_verify_61k", "decode_200k", "mixed_q8_0",
                                  "sliding_window"])
def test_full_size_every_row(B, orc, name):
    """The workloads at their full sizes, in the launch configuration the
    benchmark times: every output row against the oracle (OpenMP over the
    host cores), and a repeated call bit-identical."""
    case = gen.CONFIGS[name](0)
    dev, args, kw = _args(B, case)
    dec = B.PagedDecode.for_case(case)
    first = dec(*args, **kw)
    second = dec(*args, **kw)
    torch.cuda.synchronize()
    assert dec.get_error() == 0
    assert torch.equal(first.view(torch.int16), second.view(torch.int16))
    out = first.cpu().numpy()
    ref, _ = orc.attend(case)
    assert_parity(out, ref, name)


@pytest.mark.parametrize("dt", DTYPES)
def test_context_parallel_partials_merge_to_the_full_result(B, orc, dt):
    """Context-parallel decode on one GPU: the sequence's KV blocks are cut
    into 2 or 3 contiguous shares, each held in its own cache pool with its
    own block table (as on separate GPUs); paged_attn_decode_partial gives
    each share's fp32 (O, lse) and paged_attn_merge combines them.  The
    merged rows match the one-pass oracle, each share's partial matches the
    oracle restricted to its keys, and a share no query sees (outside the
    window) contributes O = 0, lse = -inf."""
    from paged_kv_decode_flash_b200 import context_parallel as cp
    import torch
    for world, window, L in ((2, 0, 9000), (3, 2500, 7777)):
        full = gen.make_case(seed=150 + world, context_lens=(L,), n_query=4, num_q_heads=16,
                             num_kv_heads=4, causal=1, window=window, kv_dtype=dt,
                             spike_frac=0.003)
        po_all, pl_all = [], []
        for r in range(world):
            k0, kc = cp.partition(L, full.block_size, world, r)
            used = cp.local_block_table(full.block_table[0], k0, kc, full.block_size).astype(np.int64)
            local = gen.Case(**{**full.__dict__, "k_cache": np.ascontiguousarray(full.k_cache[used]),
                                "v_cache": np.ascontiguousarray(full.v_cache[used]),
                                "num_blocks": len(used),
                                "block_table": np.arange(len(used), dtype=np.int32).reshape(1, -1),
                                "max_blocks_per_seq": len(used)})
            dev = B.case_to_device(local)
            dec = B.PagedDecode.for_case(local)
            kb = torch.tensor([k0], dtype=torch.int32, device="cuda")
            kn = torch.tensor([kc], dtype=torch.int32, device="cuda")
            po, pl = dec.partial(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
                                 dev["context_lens"], kb, kn, causal=full.causal,
                                 window=full.window, scale=full.scale, kv_dtype=dt)
            torch.cuda.synchronize()
            assert dec.get_error() == 0
            rows = full.n_query * full.num_q_heads
            ref_o = np.zeros((rows, 128))
            ref_l = np.zeros(rows)
            for i in range(full.n_query):
                for h in range(full.num_q_heads):
                    ref_o[i * full.num_q_heads + h], ref_l[i * full.num_q_heads + h] = \
                        orc.attend_row_range(full, 0, i, h, k0, k0 + kc)
            got_o = po.cpu().numpy().reshape(rows, 128)
            got_l = pl.cpu().numpy().reshape(rows)
            empty = ref_l == -np.inf
            assert np.array_equal(got_l == -np.inf, empty)
            assert np.all(got_o[empty] == 0)
            if (~empty).any():
                assert_parity(got_o[~empty], ref_o[~empty], f"share {r} of {world}")
                assert np.max(np.abs(got_l[~empty] - ref_l[~empty])) < 1e-4
            else:  # a share wholly below the first key any query's window reaches
                assert window > 0 and k0 + kc <= L - full.n_query - window + 1
            po_all.append(po.reshape(rows, 128))
            pl_all.append(pl.reshape(rows))
        out, lse = B.merge(torch.stack(po_all), torch.stack(pl_all))
        ref, ref_lse = orc.attend(full)
        assert_parity(out.cpu().numpy(), ref.reshape(-1, 128), f"merged over {world}")
