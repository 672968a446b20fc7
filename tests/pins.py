"""Checks that pin the fp64 oracle to things other than itself.

Each ``check_*(orc)`` raises AssertionError on a mismatch.  They are run on
the real oracle by test_oracle_pins.py and, by test_oracle_mutations.py, on
variants of the oracle with one planted mistake each, to show that every
planted mistake trips at least one of them.

What pins what:
  * closed forms -- one visible key returns its value; identical keys or
    scale 0 return the mean of the visible values; two keys weigh their values
    by a logistic function of the score difference; a hand-worked example
    (tests/golden/worked_small.json);
  * an independent dense float64 computation in numpy with an explicit mask
    matrix built from triangular matrices (textbook attention) on tiny random
    paged problems, fp16 and q8_0, every causal/window combination;
  * invariants -- physical block permutation, NaN in never-visible memory,
    batch versus each sequence alone, causal == non-causal at one query token,
    merge of arbitrary key splits == one pass;
  * exact decoding -- all 65536 fp16 bit patterns against numpy's float16;
  * quantise on write -- fp32 -> fp16 conversion against numpy on every
    exponent and on exact ties; hand-worked q8_0 groups and int8 rows, the
    half-step error bound, the generator's float64 rule away from fp32
    near-ties; a cache write read back through a one-key window.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from paged_kv_decode_flash_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# independent dense reference (numpy float64)
# ---------------------------------------------------------------------------
def dense_kv(case, s: int, which: str) -> np.ndarray:
    """Gather the logical [Hkv][L][D] float64 K or V of sequence s by walking
    the block table with numpy fancy indexing."""
    L = int(case.context_lens[s])
    bs, D, H = case.block_size, case.head_dim, case.num_kv_heads
    j = np.arange(L)
    phys = case.block_table[s, j // bs]
    slot = j % bs
    cache = case.k_cache if which == "k" else case.v_cache
    if case.kv_dtype == gen.KV_FP16:
        x = cache[phys, :, slot, :].astype(np.float64)  # [L][H][D]
    elif case.kv_dtype == gen.KV_INT8_ROW:
        nt = cache[phys]  # [L][H][tile]
        qs = nt[:, :, : bs * D].view(np.int8).reshape(L, H, bs, D)
        qs = qs[np.arange(L), :, slot, :].astype(np.float64)  # [L][H][D]
        sc = np.ascontiguousarray(nt[:, :, bs * D:]).view(np.float32).reshape(L, H, bs)
        sc = sc[np.arange(L), :, slot].astype(np.float64)  # [L][H]
        x = qs * sc[:, :, None]
    else:
        nt = cache[phys]  # [L][H][tile]
        qs = nt[:, :, : bs * D].view(np.int8).reshape(L, H, bs, D)
        qs = qs[np.arange(L), :, slot, :].astype(np.float64)  # [L][H][D]
        dd = np.ascontiguousarray(nt[:, :, bs * D:]).view(np.float16).reshape(L, H, bs, D // 32)
        dd = dd[np.arange(L), :, slot, :].astype(np.float64)  # [L][H][D/32]
        x = qs * np.repeat(dd, 32, axis=-1)
    return np.ascontiguousarray(x.transpose(1, 0, 2))


def dense_mask(L: int, nq: int, causal: int, window: int) -> np.ndarray:
    """Boolean [nq][L]: built from shifted triangular matrices."""
    m = np.ones((nq, L), dtype=bool)
    if causal:
        m &= np.tril(np.ones((nq, L), dtype=bool), k=L - nq)
        if window > 0:
            m &= ~np.tril(np.ones((nq, L), dtype=bool), k=L - nq - window)
    elif window > 0:
        m[:, : max(0, L - window)] = False
    return m


def dense_attention(case):
    B, nq, Hq, D = case.num_seqs, case.n_query, case.num_q_heads, case.head_dim
    out = np.zeros((B, nq, Hq, D))
    lse = np.full((B, nq, Hq), -np.inf)
    G = case.group
    for s in range(B):
        L = int(case.context_lens[s])
        K, V = dense_kv(case, s, "k"), dense_kv(case, s, "v")
        mask = dense_mask(L, nq, case.causal, case.window)
        for h in range(Hq):
            q = case.q[s, :, h, :].astype(np.float64)  # [nq][D]
            z = case.scale * (q @ K[h // G].T)  # [nq][L]
            z = np.where(mask, z, -np.inf)
            m = z.max(axis=1, keepdims=True)
            w = np.where(mask, np.exp(z - m), 0.0)
            l = w.sum(axis=1, keepdims=True)
            out[s, :, h, :] = (w @ np.where(mask.any(0)[:, None], V[h // G], 0.0)) / l
            lse[s, :, h] = (m + np.log(l))[:, 0]
    return out, lse


def _close(a, b, tol, what):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert a.shape == b.shape and err <= tol, f"{what}: max abs err {err} > {tol}"


# ---------------------------------------------------------------------------
# the checks
# ---------------------------------------------------------------------------
def check_half_decode(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan), "NaN patterns differ"
    assert np.array_equal(got[~nan], ref[~nan]), "fp16 decode differs from numpy"


def check_golden_worked_example(orc):
    with open(os.path.join(GOLDEN, "worked_small.json")) as f:
        g = json.load(f)
    bs, D = g["block_size"], g["head_dim"]
    keys = np.array(g["keys"], dtype=np.float16)
    vals = np.array(g["values"], dtype=np.float16)
    table = np.array(g["block_table"], dtype=np.int32)
    kc = np.full((g["num_blocks"], 1, bs, D), np.nan, dtype=np.float16)
    vc = kc.copy()
    for j in range(len(keys)):
        kc[table[0, j // bs], 0, j % bs] = keys[j]
        vc[table[0, j // bs], 0, j % bs] = vals[j]
    for c in g["cases"]:
        case = gen.Case("golden", 1, 1, 1, D, bs, table.shape[1], g["num_blocks"],
                        g["n_query"], c["causal"], c["window"], gen.KV_FP16,
                        g["scale"], np.array(g["q"], dtype=np.float16).reshape(1, 2, 1, D),
                        kc, vc, table, np.array(g["context_lens"], dtype=np.int32))
        out, lse = orc.attend(case)
        _close(out[0, :, 0, :], c["out"], 1e-14, f"golden out {c}")
        _close(lse[0, :, 0], c["lse"], 1e-14, f"golden lse {c}")


def check_single_key(orc):
    for dt in (gen.KV_FP16, gen.KV_Q8_0, gen.KV_INT8_ROW):
        # L = 1: the only key is visible; output must equal its value exactly.
        case = gen.make_case(seed=11, context_lens=(1,), n_query=1, num_q_heads=4,
                             num_kv_heads=2, kv_dtype=dt, spare_blocks=3)
        out, lse = orc.attend(case)
        V = dense_kv(case, 0, "v")
        K = dense_kv(case, 0, "k")
        for h in range(4):
            assert np.array_equal(out[0, 0, h], V[h // 2, 0]), "single key != its value"
            z = case.scale * float(case.q[0, 0, h].astype(np.float64) @ K[h // 2, 0])
            assert abs(lse[0, 0, h] - z) <= 1e-12 * max(1.0, abs(z)), "lse of one key"
        # window 1: each query sees only the key at its own position.
        case = gen.make_case(seed=12, context_lens=(37,), n_query=3, num_q_heads=2,
                             num_kv_heads=1, window=1, causal=1, kv_dtype=dt)
        out, _ = orc.attend(case)
        V = dense_kv(case, 0, "v")
        for i in range(3):
            assert np.array_equal(out[0, i, 0], V[0, 37 - 3 + i]), "window 1 != own value"


def check_mean_forms(orc):
    # scale 0: every visible key has the same weight -> mean of visible values.
    case = gen.make_case(seed=13, context_lens=(45,), n_query=2, num_q_heads=2,
                         num_kv_heads=1, scale=0.0, causal=1, window=20)
    out, lse = orc.attend(case)
    V = dense_kv(case, 0, "v")[0]
    for i in range(2):
        p = 45 - 2 + i
        vis = V[p - 20 + 1: p + 1]
        _close(out[0, i, 0], vis.mean(axis=0), 1e-13, "scale 0 mean")
        _close(lse[0, i, 0], math.log(20), 1e-13, "scale 0 lse = log n")
    # identical keys (one row copied everywhere) -> mean of values.
    case = gen.make_case(seed=14, context_lens=(33,), n_query=1, num_q_heads=2,
                         num_kv_heads=1, causal=1)
    row = case.k_cache[case.block_table[0, 0], 0, 0].copy()
    for j in range(33):
        case.k_cache[case.block_table[0, j // 16], 0, j % 16] = row
    out, _ = orc.attend(case)
    _close(out[0, 0, 0], dense_kv(case, 0, "v")[0].mean(axis=0), 1e-13, "identical keys")


def check_two_keys_logistic(orc):
    case = gen.make_case(seed=15, context_lens=(2,), n_query=1, num_q_heads=3,
                         num_kv_heads=1, causal=1)
    out, _ = orc.attend(case)
    K, V = dense_kv(case, 0, "k")[0], dense_kv(case, 0, "v")[0]
    for h in range(3):
        q = case.q[0, 0, h].astype(np.float64)
        dz = case.scale * float(q @ (K[0] - K[1]))
        w0 = 1.0 / (1.0 + math.exp(-dz))
        _close(out[0, 0, h], w0 * V[0] + (1.0 - w0) * V[1], 1e-13, "two-key logistic")


def _random_cases(seed_base=100):
    rng = np.random.default_rng(seed_base)
    for t in range(18):
        causal = t % 2
        window = [0, 1, 5, 17][(t // 2) % 4]
        nq = [1, 2, 3, 4][t % 4]
        Hkv = [1, 2][t % 2]
        G = [1, 2, 4][t % 3]
        bs = [16, 32][t % 2]
        dt = gen.KV_Q8_0 if t % 5 == 4 else gen.KV_INT8_ROW if t % 5 == 2 else gen.KV_FP16
        lens = tuple(int(x) for x in rng.integers(nq, 64, size=1 + t % 3))
        yield gen.make_case(seed=seed_base + t, context_lens=lens, n_query=nq,
                            num_q_heads=Hkv * G, num_kv_heads=Hkv, block_size=bs,
                            causal=causal, window=window, kv_dtype=dt,
                            spare_blocks=2, head_dim=64 if t % 3 == 0 else 128)


def check_dense_bruteforce(orc):
    for case in _random_cases():
        out, lse = orc.attend(case)
        ref_out, ref_lse = dense_attention(case)
        _close(out, ref_out, 1e-12, f"dense brute force ({case.causal=}, {case.window=})")
        _close(lse, ref_lse, 1e-12, "dense brute force lse")


def check_trace_bruteforce(orc):
    for case in _random_cases(300):
        t = orc.trace(case)
        r = 0
        for s in range(case.num_seqs):
            L = int(case.context_lens[s])
            mask = dense_mask(L, case.n_query, case.causal, case.window)
            j = np.arange(L)
            phys = (case.block_table[s, j // case.block_size].astype(np.int64)
                    * case.block_size + j % case.block_size)
            for i in range(case.n_query):
                vis = j[mask[i]]
                ph = phys[mask[i]].astype(np.uint32)
                exp = [vis.size, vis.min() if vis.size else -1, vis.max() if vis.size else -1,
                       int(np.bitwise_xor.reduce(ph)) if ph.size else 0,
                       int(ph.sum(dtype=np.uint64) & 0xFFFFFFFF)]
                exp = np.array(exp, dtype=np.int64).astype(np.uint32).view(np.int32)
                for h in range(case.num_q_heads):
                    assert np.array_equal(t[r], exp), f"trace row {r}: {t[r]} vs {exp}"
                    r += 1


def check_block_permutation(orc):
    case = gen.make_case(seed=16, context_lens=(70, 33), n_query=2, num_q_heads=4,
                         num_kv_heads=2, causal=1, window=30, spare_blocks=4)
    out, lse = orc.attend(case)
    rng = np.random.default_rng(5)
    perm = rng.permutation(case.num_blocks)  # new id of old block b = perm[b]
    k2 = np.empty_like(case.k_cache)
    v2 = np.empty_like(case.v_cache)
    k2[perm] = case.k_cache
    v2[perm] = case.v_cache
    c2 = gen.Case(**{**case.__dict__, "k_cache": k2, "v_cache": v2,
                     "block_table": perm[case.block_table].astype(np.int32)})
    out2, lse2 = orc.attend(c2)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2), "block permutation changed result"


def zero_nans(case):
    """The case with every NaN of its caches replaced by 0 (fp16 values; the
    scales of the int8 caches)."""
    clean = gen.Case(**case.__dict__)
    if case.kv_dtype == gen.KV_FP16:
        clean.k_cache = np.nan_to_num(case.k_cache, nan=0.0)
        clean.v_cache = np.nan_to_num(case.v_cache, nan=0.0)
        return clean
    sdt = np.float16 if case.kv_dtype == gen.KV_Q8_0 else np.float32
    for name in ("k_cache", "v_cache"):
        c = getattr(case, name).copy()
        d = c[:, :, case.block_size * case.head_dim:].view(sdt)
        d[np.isnan(d)] = 0.0
        setattr(clean, name, c)
    return clean


def check_nan_invariance(orc):
    for dt in (gen.KV_FP16, gen.KV_Q8_0, gen.KV_INT8_ROW):
        # whole out-of-window blocks (non-causal window) and, key by key, every
        # key below the window edge of the earliest query (causal window)
        for causal, kw in ((0, dict(nan_below=[100 - 40, 57 - 40])),
                           (1, dict(nan_keys_below=[100 - 3 - 40 + 1, 57 - 3 - 40 + 1]))):
            case = gen.make_case(seed=17, context_lens=(100, 57), n_query=3, num_q_heads=4,
                                 num_kv_heads=2, causal=causal, window=40, kv_dtype=dt,
                                 spare_blocks=3, **kw)
            out, lse = orc.attend(case)
            assert np.all(np.isfinite(out)), "NaN leaked from never-visible memory"
            out2, lse2 = orc.attend(zero_nans(case))
            assert np.array_equal(out, out2) and np.array_equal(lse, lse2), "NaN-poisoned != zeroed"


# ---------------------------------------------------------------------------
# quantise on write
# ---------------------------------------------------------------------------
def _half_midpoint(v32: np.float32) -> bool:
    """Is the fp32 value exactly halfway between two adjacent fp16 values?"""
    h = np.float16(v32)
    if not np.isfinite(h):
        return False
    a = np.float64(h)
    nb = np.nextafter(h, np.float16(np.inf) if np.float64(v32) > a else np.float16(-np.inf))
    return np.float64(v32) * 2 == a + np.float64(nb)


def check_float_to_half(orc):
    """fp32 -> fp16 round to nearest even, against numpy's conversion: every
    exponent (normal, subnormal, overflow), random mantissas, exact ties."""
    rng = np.random.default_rng(40)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    exps = rng.integers(100, 145, size=20000).astype(np.uint32)  # around fp16's range
    bits2 = (bits & np.uint32(0x807FFFFF)) | (exps << np.uint32(23))
    ties = []
    for e in range(-26, 17):  # fp16 value k * 2^(e-10) plus half an ulp
        for k in (1024, 1025, 1500, 2047):
            ties.append(np.float32((k + 0.5) * 2.0 ** (e - 10)))
    vals = np.concatenate([bits.view(np.float32), bits2.view(np.float32), np.array(ties, np.float32),
                           np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 2 ** -24, 2 ** -25,
                                     3 * 2 ** -26, np.inf, -np.inf], dtype=np.float32)])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = np.array([v], dtype=np.float32).astype(np.float16).view(np.uint16)[0]
        got = orc.float_to_half(v)
        if np.isnan(v):
            assert (got & 0x7c00) == 0x7c00 and (got & 0x3ff) != 0, "NaN"
        else:
            assert got == ref, f"float_to_half({v!r}) = {got:#06x}, numpy {ref:#06x}"


def check_quantize_q8_0(orc):
    """q8_0 on write: hand-worked groups, the error bound, and agreement with
    the float64 rule of the data generator except where fp32 and fp64 may
    legitimately differ (an fp32 quotient on an fp16 tie, or x / d within
    fp32 rounding of a half-integer)."""
    x = np.zeros(32, np.float32)
    x[:5] = [127.0, 2.5, -2.5, 0.49, -0.5]  # amax 127 -> d = 1; ties go away from zero
    q, d = orc.quantize_q8_0(x)
    assert d == 0x3C00 and q[:5].tolist() == [127, 3, -3, 0, -1], (q[:5], hex(d))
    x[:] = 0
    x[:3] = [-254.0, 3.0, 1.0]  # d = 2: 3/2 = 1.5 -> 2, 1/2 -> 1
    q, d = orc.quantize_q8_0(x)
    assert d == 0x4000 and q[:3].tolist() == [-127, 2, 1]
    q, d = orc.quantize_q8_0(np.zeros(32, np.float32))
    assert d == 0 and not q.any()
    rng = np.random.default_rng(41)
    xs = (rng.standard_normal((400, 32)) * rng.choice([1e-3, 1.0, 50.0], size=(400, 1))
          ).astype(np.float16).astype(np.float32)
    gq, gd = gen.quantise_q8_0(xs)
    for r in range(xs.shape[0]):
        q, d = orc.quantize_q8_0(xs[r])
        dv = np.float64(np.array([d], np.uint16).view(np.float16)[0])
        rec = q.astype(np.float64) * dv
        assert np.all(np.abs(rec - xs[r]) <= 0.5 * dv * (1 + 1e-5) + (np.abs(xs[r]) - 127 * dv).clip(0)), "error bound"
        if d != gd[r, 0].view(np.uint16):
            assert _half_midpoint(np.float32(np.abs(xs[r]).max()) / np.float32(127)), f"scale {r}"
            continue
        ratio = xs[r].astype(np.float64) / dv
        near = np.abs(np.abs(ratio) - np.floor(np.abs(ratio)) - 0.5) < 1e-5
        assert np.array_equal(q[~near], gq[r][~near]), f"codes of group {r}"


def check_quantize_row(orc):
    """int8 rows on write: hand-worked row, the error bound, the generator's
    float64 rule away from fp32 near-ties."""
    x = np.zeros(128, np.float32)
    x[:5] = [127.0, -63.5, 0.5, -0.5, 2.4999]  # s = 1
    q, sc = orc.quantize_row(x)
    assert sc == 1.0 and q[:5].tolist() == [127, -64, 1, -1, 2]
    q, sc = orc.quantize_row(np.zeros(128, np.float32))
    assert sc == 0.0 and not q.any()
    rng = np.random.default_rng(42)
    xs = (rng.standard_normal((200, 128)) * 3).astype(np.float16).astype(np.float32)
    gq, gs = gen.quantise_rows(xs)
    for r in range(xs.shape[0]):
        q, sc = orc.quantize_row(xs[r])
        assert np.float32(sc) == gs[r] or abs(sc - gs[r]) <= 1.2e-7 * sc, f"scale of row {r}"
        rec = q.astype(np.float64) * sc
        assert np.all(np.abs(rec - xs[r]) <= 0.5 * sc * (1 + 1e-5) +
                      (np.abs(xs[r]) - 127 * np.float64(sc)).clip(0)), "error bound"
        ratio = xs[r].astype(np.float64) / np.float64(sc)
        near = np.abs(np.abs(ratio) - np.floor(np.abs(ratio)) - 0.5) < 1e-5
        assert np.array_equal(q[~near], gq[r][~near]), f"codes of row {r}"


def check_cache_write(orc):
    """Writing the newest tokens: exactly their slots change, and attention
    with a window of one key returns, for each new token, the value just
    written (fp16: bit for bit; int8: its quantisation, within half a step)."""
    for dt in (gen.KV_FP16, gen.KV_Q8_0, gen.KV_INT8_ROW):
        case = gen.make_case(seed=43, context_lens=(70, 33), n_query=3, num_q_heads=4,
                             num_kv_heads=2, kv_dtype=dt, spare_blocks=2, causal=1, window=1)
        rng = np.random.default_rng(44)
        kn = rng.standard_normal((2, 3, 2, 128)).astype(np.float16)
        vn = rng.standard_normal((2, 3, 2, 128)).astype(np.float16)
        kc, vc, rc = orc.cache_write(case, kn, vn)
        assert rc == 0
        changed = np.zeros(case.num_blocks, dtype=bool)
        for s, L in enumerate(case.context_lens.tolist()):
            for i in range(3):
                changed[case.block_table[s, (L - 3 + i) // case.block_size]] = True
        for new_c, old_c in ((kc, case.k_cache), (vc, case.v_cache)):  # bytes: NaN-safe
            assert np.array_equal(new_c[~changed].view(np.uint8), old_c[~changed].view(np.uint8)), \
                "other blocks written"
        w = gen.Case(**{**case.__dict__, "k_cache": kc, "v_cache": vc})
        out, _ = orc.attend(w)  # window 1: each query returns its own position's value
        for s in range(2):
            V = dense_kv(w, s, "v")
            for i in range(3):
                for h in range(4):
                    new = vn[s, i, h // 2].astype(np.float64)
                    got = out[s, i, h]
                    assert np.array_equal(got, V[h // 2, int(w.context_lens[s]) - 3 + i])
                    if dt == gen.KV_FP16:
                        assert np.array_equal(got, new), "fp16 write not exact"
                    else:
                        step = np.abs(new).max() / 127 * (1 + 2 ** -10)
                        assert np.all(np.abs(got - new) <= 0.5 * step), "int8 write error"
        bad = gen.Case(**{**case.__dict__, "block_table": case.block_table.copy()})
        bad.block_table[0, (70 - 1) // case.block_size] = case.num_blocks + 3
        assert orc.cache_write(bad, kn, vn)[2] != 0, "bad block not reported"


def check_batch_equals_alone(orc):
    case = gen.make_case(seed=18, context_lens=(40, 90, 17), n_query=2, num_q_heads=4,
                         num_kv_heads=2, causal=1, spare_blocks=2)
    out, lse = orc.attend(case)
    for s in range(3):
        c1 = gen.Case(**{**case.__dict__, "num_seqs": 1, "q": case.q[s:s + 1].copy(),
                         "block_table": case.block_table[s:s + 1].copy(),
                         "context_lens": case.context_lens[s:s + 1].copy()})
        o1, l1 = orc.attend(c1)
        assert np.array_equal(o1[0], out[s]) and np.array_equal(l1[0], lse[s]), "batch != alone"


def check_causal_single_query(orc):
    a = gen.make_case(seed=19, context_lens=(50,), n_query=1, num_q_heads=2,
                      num_kv_heads=1, causal=1, window=12)
    b = gen.Case(**{**a.__dict__, "causal": 0})
    oa, la = orc.attend(a)
    ob, lb = orc.attend(b)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb), "causal nq=1 != non-causal"


def check_merge_of_splits(orc):
    case = gen.make_case(seed=20, context_lens=(150,), n_query=2, num_q_heads=2,
                         num_kv_heads=1, causal=1, window=90)
    ref, ref_lse = orc.attend(case)
    rng = np.random.default_rng(3)
    for _ in range(4):
        cuts = np.sort(rng.choice(np.arange(1, 150), size=5, replace=False))
        edges = [0, *cuts.tolist(), 150]
        S = len(edges) - 1
        po = np.zeros((S, 4, case.head_dim))
        pl = np.zeros((S, 4))
        for si in range(S):
            r = 0
            for i in range(2):
                for h in range(2):
                    o, l = orc.attend_row_range(case, 0, i, h, edges[si], edges[si + 1])
                    po[si, r], pl[si, r] = o, l
                    r += 1
        mo, ml = orc.merge(po, pl)
        _close(mo, ref.reshape(4, -1), 1e-12, "merge of splits")
        _close(ml, ref_lse.reshape(4), 1e-12, "merge lse")


def check_error_codes(orc):
    import oracle as O
    case = gen.make_case(seed=21, context_lens=(20,), n_query=1, num_q_heads=2,
                         num_kv_heads=1)
    bad = gen.Case(**{**case.__dict__, "block_table": case.block_table.copy()})
    bad.block_table[0, 1] = case.num_blocks  # out of range
    try:
        orc.attend(bad)
        raise AssertionError("bad block index not reported")
    except O.OracleError as e:
        assert e.code == O.ERR_BAD_BLOCK_INDEX
    for L in (case.max_blocks_per_seq * case.block_size + 1, 0):
        c = gen.Case(**{**case.__dict__, "context_lens": np.array([L], dtype=np.int32)})
        try:
            orc.attend(c)
            raise AssertionError("bad context length not reported")
        except O.OracleError as e:
            assert e.code == O.ERR_BAD_CONTEXT_LEN


ALL_CHECKS = [
    check_half_decode, check_golden_worked_example, check_single_key,
    check_mean_forms, check_two_keys_logistic, check_dense_bruteforce,
    check_trace_bruteforce, check_block_permutation, check_nan_invariance,
    check_batch_equals_alone, check_causal_single_query, check_merge_of_splits,
    check_error_codes, check_float_to_half, check_quantize_q8_0, check_quantize_row,
    check_cache_write,
]
