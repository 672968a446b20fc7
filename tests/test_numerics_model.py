"""An executable model of the tensor-core kernel's arithmetic for the q8_0
cache, against the fp64 oracle: it shows that the scheme the kernel uses
meets the tolerance and that each of the two roundings it avoids does not.

The kernel (csrc/decode_tc.cu) keeps the int8 values exact on the tensor
core: per 32-element scale group g, S_g = sum_k q_k qs_jk (fp16 inputs, fp32
accumulation) and the score is sum_g dK_g S_g in fp32; V's operand is
qs * 2^e with d = m * 2^e, and the weights p (scaled by 2^13) times V's
mantissa m are split into an fp16 high part (11 significant bits) and an fp16
residual.  The two shortcuts it avoids: rounding qs * d to fp16 for K and V,
and rounding the weights to fp16 once.  Rows of one (sequence, KV head) are
modelled with a single reference maximum (the kernel's lazily rescaled one
differs only by exact powers of two).  CPU only; numpy float32 stands for the
fp32 arithmetic (summation order differs from the hardware's, which the
tolerance absorbs).
"""
import numpy as np
import pytest

import oracle
from parity import ABS_TOL, REL_TOL, parity_errors
from paged_kv_decode_flash_b200 import inputs as gen

f32, f16 = np.float32, np.float16


def _raw_q8(case, s, which):
    """int8 qs [Hkv][L][D] and fp16 scales [Hkv][L][D/32] of sequence s."""
    L = int(case.context_lens[s])
    bs, D, H = case.block_size, case.head_dim, case.num_kv_heads
    j = np.arange(L)
    nt = (case.k_cache if which == "k" else case.v_cache)[case.block_table[s, j // bs]]
    qs = nt[:, :, : bs * D].view(np.int8).reshape(L, H, bs, D)[j, :, j % bs, :]
    d = np.ascontiguousarray(nt[:, :, bs * D:]).view(f16).reshape(L, H, bs, D // 32)[j, :, j % bs, :]
    return qs.transpose(1, 0, 2), d.transpose(1, 0, 2)


def _visible(L, nq, causal, window):
    m = np.zeros((nq, L), bool)
    for i in range(nq):
        hi = L - nq + i if causal else L - 1
        m[i, (max(0, hi - window + 1) if window > 0 else 0): hi + 1] = True
    return m


def _trunc11(x):
    return (x.view(np.uint32) & np.uint32(0xFFFFE000)).view(f32)


def model(case, round_values=False, round_p_once=False):
    out = np.zeros((case.num_seqs, case.n_query, case.num_q_heads, case.head_dim))
    G, cs = case.group, f32(case.scale * 1.4426950408889634)
    for s in range(case.num_seqs):
        L = int(case.context_lens[s])
        vis = np.repeat(_visible(L, case.n_query, case.causal, case.window), G, axis=0)
        kq, kd = _raw_q8(case, s, "k")
        vq, vd = _raw_q8(case, s, "v")
        for h in range(case.num_kv_heads):
            q = case.q[s, :, h * G:(h + 1) * G].reshape(-1, 128).astype(f32)
            if round_values:  # K = fp16(qs * d)
                K = (kq[h] * np.repeat(kd[h].astype(f32), 32, -1)).astype(f16).astype(f32)
                sv = (q @ K.T).astype(f32)
            else:  # one partial product per scale group, combined in fp32
                sv = np.zeros((q.shape[0], L), f32)
                for g in range(4):
                    Sg = (q[:, 32 * g:32 * g + 32] @ kq[h][:, 32 * g:32 * g + 32].astype(f32).T)
                    sv = (sv + kd[h][:, g].astype(f32)[None, :] * Sg.astype(f32)).astype(f32)
            sv = np.where(vis, sv, -np.inf).astype(f32)
            p = np.exp2(((sv - sv.max(axis=1, keepdims=True)) * cs + f32(13)).astype(f32))
            l = p.sum(axis=1, dtype=f32)
            O = np.zeros((q.shape[0], 128))
            for g in range(4):
                cols = slice(32 * g, 32 * g + 32)
                if round_values:  # V = fp16(qs * d), weights unscaled by d
                    Vop = (vq[h][:, cols] * vd[h][:, g].astype(f32)[:, None]).astype(f16)
                    w = p
                else:  # V = qs * 2^e exactly, weights times the mantissa m
                    E = np.maximum((vd[h][:, g].view(np.uint16) >> 10) & 31, 1).astype(np.int64)
                    p2 = np.exp2(E - 15.0)
                    Vop = (vq[h][:, cols] * p2[:, None]).astype(f16)
                    w = (p * (vd[h][:, g].astype(np.float64) / p2).astype(f32)[None, :]).astype(f32)
                if round_p_once:
                    W = w.astype(f16).astype(np.float64)
                else:
                    hi = _trunc11(w)
                    W = hi.astype(f16).astype(np.float64) + (w - hi).astype(f16).astype(np.float64)
                O[:, cols] = (W @ Vop.astype(np.float64)).astype(f32)
            o = (O / l[:, None].astype(np.float64)).astype(f32).astype(f16).astype(np.float64)
            out[s, :, h * G:(h + 1) * G] = o.reshape(case.n_query, G, 128)
    return out


def _out_of_tolerance(got, ref):
    err, rel = parity_errors(got, ref)
    return int(((err > ABS_TOL) | (rel > REL_TOL)).sum())


@pytest.mark.parametrize("seed,gain", [(1, 8.0), (2, 12.0)])
def test_kernel_scheme_meets_tolerance_and_each_shortcut_does_not(seed, gain):
    case = gen.make_case(seed=seed, context_lens=(3000, 1777), n_query=4, num_q_heads=16,
                         num_kv_heads=4, causal=1, kv_dtype=gen.KV_Q8_0, spike_frac=0.01,
                         spike_gain=gain)
    ref, _ = oracle.load().attend(case)
    assert _out_of_tolerance(model(case), ref) == 0
    assert _out_of_tolerance(model(case, round_values=True), ref) > 0
    assert _out_of_tolerance(model(case, round_p_once=True), ref) > 0
