"""The fp64 oracle against closed forms, invariants and an independent dense
numpy computation (CPU only)."""
import numpy as np
import pytest

import oracle
import pins
from paged_kv_decode_flash_b200 import inputs as gen


@pytest.fixture(scope="module")
def orc():
    return oracle.load()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pin(orc, check):
    check(orc)


def test_dense_reference_agrees_with_textbook_single_query(orc):
    """G = 1, n_query = 1: plain single-query softmax attention over a
    contiguous key list (the textbook form), here written with scipy's
    logsumexp as a second, library-backed route."""
    from scipy.special import logsumexp, softmax
    for seed in range(4):
        case = gen.make_case(seed=seed, context_lens=(29 + 7 * seed,), n_query=1,
                             num_q_heads=1, num_kv_heads=1, head_dim=32, spare_blocks=2)
        out, lse = orc.attend(case)
        K = pins.dense_kv(case, 0, "k")[0]
        V = pins.dense_kv(case, 0, "v")[0]
        z = case.scale * (K @ case.q[0, 0, 0].astype(np.float64))
        assert np.max(np.abs(out[0, 0, 0] - softmax(z) @ V)) < 1e-12
        assert abs(lse[0, 0, 0] - logsumexp(z)) < 1e-12


def test_generator_shapes_and_poison():
    c = gen.tiny(0)
    assert c.num_blocks == 128 and c.block_table.shape == (1, 64)
    assert len(set(c.block_table[0].tolist())) == 64
    used = set(c.block_table[0].tolist())
    unused = [b for b in range(128) if b not in used]
    assert all(np.isnan(c.k_cache[b]).all() for b in unused)
    assert np.isfinite(c.k_cache[c.block_table[0]]).all()


def test_q8_0_quantiser_round_trip():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    q, d = gen.quantise_q8_0(x)
    rec = q.astype(np.float64) * np.repeat(d.astype(np.float64), 32, axis=-1)
    # error at most half a step of the group's scale (plus fp16 scale rounding)
    step = np.repeat(d.astype(np.float64), 32, axis=-1)
    assert np.all(np.abs(rec - x) <= 0.5 * step + 1e-3 * np.abs(x) + 1e-12)
    assert np.abs(q).max() <= 127
