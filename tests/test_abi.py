"""The C-ABI library without a GPU: it builds, loads, exports every symbol
include/pagedattn.h declares, and its host-side logic (argument checks,
workspace sizing) behaves.  No call here reaches the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from paged_kv_decode_flash_b200 import build
    build.build()
    from paged_kv_decode_flash_b200 import binding
    return binding.lib()


def declared_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(paged_attn_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("paged_attn_decode", "paged_attn_merge", "paged_attn_workspace_size",
                 "paged_attn_get_error"):
        assert must in names


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), f"{name} declared but not exported"


def dims(**kw):
    from paged_kv_decode_flash_b200.binding import Dims
    d = dict(num_seqs=1, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
             max_blocks_per_seq=3841, num_blocks=3841, workspace=None, workspace_bytes=0)
    d.update(kw)
    return Dims(**d)


def test_workspace_size_host_only(L):
    d = dims()
    n = L.paged_attn_workspace_size(ctypes.byref(d), 8)
    assert n > 256 and n % 256 == 0
    # more query tokens need at least as much
    assert L.paged_attn_workspace_size(ctypes.byref(d), 8) >= L.paged_attn_workspace_size(ctypes.byref(d), 1)
    # invalid shapes -> 0
    for bad in (dims(num_q_heads=30), dims(block_size=8), dims(head_dim=64), dims(num_seqs=0)):
        assert L.paged_attn_workspace_size(ctypes.byref(bad), 8) == 0
    assert L.paged_attn_workspace_size(ctypes.byref(d), 0) == 0
    assert L.paged_attn_workspace_size(ctypes.byref(d), 129) == 0
    assert L.paged_attn_workspace_size(None, 1) == 0


def test_decode_rejects_bad_arguments_on_host(L):
    from paged_kv_decode_flash_b200 import binding as b
    d = dims(workspace=4096, workspace_bytes=1 << 30)
    p = ctypes.c_void_p(1 << 20)  # never dereferenced: checks fail first
    args = lambda **kw: dict(dict(q=p, k=p, v=p, bt=p, cl=p, nq=8, causal=1, window=0,
                                  scale=0.088, dt=0, out=p), **kw)

    def call(dd, a):
        return L.paged_attn_decode(ctypes.byref(dd) if dd is not None else None, a["q"], a["k"],
                                   a["v"], a["bt"], a["cl"], a["nq"], a["causal"], a["window"],
                                   a["scale"], a["dt"], a["out"], None)

    assert call(None, args()) == b.PA_ERR_INVALID_ARG
    assert call(d, args(q=None)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(nq=0)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(nq=129)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(causal=2)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(window=-1)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(dt=7)) == b.PA_ERR_INVALID_ARG
    assert call(d, args(scale=float("nan"))) == b.PA_ERR_INVALID_ARG
    assert call(d, args(q=ctypes.c_void_p((1 << 20) + 2))) == b.PA_ERR_INVALID_ARG  # misaligned
    assert call(dims(head_dim=64, workspace=4096, workspace_bytes=1 << 30), args()) == b.PA_ERR_UNSUPPORTED
    assert call(dims(num_q_heads=8 * 129, num_kv_heads=8, workspace=4096, workspace_bytes=1 << 30),
                args()) == b.PA_ERR_UNSUPPORTED  # 8 tokens x 129 heads per KV head > 1024 rows
    assert call(dims(workspace=None), args()) == b.PA_ERR_WORKSPACE
    assert call(dims(workspace=4100, workspace_bytes=1 << 30), args()) == b.PA_ERR_WORKSPACE


def test_merge_rejects_bad_arguments_on_host(L):
    from paged_kv_decode_flash_b200 import binding as b
    p = ctypes.c_void_p(1 << 20)
    assert L.paged_attn_merge(None, p, 2, 4, 128, p, None, None) == b.PA_ERR_INVALID_ARG
    assert L.paged_attn_merge(p, p, 0, 4, 128, p, None, None) == b.PA_ERR_INVALID_ARG
    assert L.paged_attn_merge(p, p, 2, -1, 128, p, None, None) == b.PA_ERR_INVALID_ARG
    assert L.paged_attn_merge(p, p, 2, 4, 96, p, None, None) == b.PA_ERR_UNSUPPORTED


def test_status_strings(L):
    from paged_kv_decode_flash_b200 import binding as b
    for code in range(-7, 1):
        assert L.paged_attn_status_string(code)
    assert b.status_string(b.PA_ERR_BAD_BLOCK_INDEX) == "block_table entry out of range"


def test_binding_refuses_to_run_without_library(monkeypatch, tmp_path):
    from paged_kv_decode_flash_b200 import binding as b
    monkeypatch.setattr(b, "_LIB", None)
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        b.lib()


def _ceil(a, b):
    return -(-a // b)


def _align(x):
    return (x + 255) & ~255


MAX_PARTS = 1024 // 16  # counters cover the most row parts any call uses (1024 rows in parts of 16)


def _plan(B, Hq, Hkv, bs, mbps, nq, kv_dtype, sms):
    """(partial slots, rows per part) of the plan paged_attn_decode makes on
    a device with `sms` SMs (the planner in csrc/dispatch.cu, restated): the
    rows of a KV head in parts of at most 32 (fp16) or 16 (int8 caches);
    few groups: an equal share of the SMs per (sequence, part), the same
    number of CTAs for every KV head (at least one, at most one per tile of a
    full table), plus one slot per KV head; a batch: items of up to 16
    tiles, the last cut into up to 4."""
    R = nq * (Hq // Hkv)
    H = _ceil(R, 32 if kv_dtype == 0 else 16)
    RH = _ceil(R, H)
    groups = B * Hkv * H
    max_chunks = mbps * bs // 16
    max_tiles = _ceil(max_chunks, 8)
    if groups * 4 <= sms:
        ch = Hkv * max(1, min(sms // (B * H) // Hkv, max_tiles))
        return B * H * (ch + Hkv), RH
    T = min(16, max_tiles)
    return groups * (_ceil(max_chunks, 8 * T) - 1 + 4), RH


def _ws_needed(B, Hq, Hkv, bs, mbps, nq, kv_dtype, sms):
    slots, RH = _plan(B, Hq, Hkv, bs, mbps, nq, kv_dtype, sms)
    prefix = 256 + _align(B * Hkv * MAX_PARTS * 2 * 4) + _align(_ceil(B, 256) * 4)
    return prefix + _align(slots * RH * 128 * 4) + _align(slots * RH * 4)


def test_workspace_size_covers_every_plan(L):
    """paged_attn_workspace_size needs no device, so it must cover the plan
    of any device and any cache type: every SM count up to 1024, every
    block size (a multiple of 16 up to 128), 1 to 128 query tokens: row
    counts that need one to 64 row parts."""
    import numpy as np
    rng = np.random.default_rng(7)
    shapes = [(1, 32, 8, 16, 3841, 8), (1, 32, 4, 16, 12288, 1), (8, 32, 8, 16, 4096, 4),
              (1, 8, 1, 48, 100, 4), (1, 8, 1, 112, 100, 4), (64, 64, 8, 16, 4096, 8),
              (300, 32, 8, 16, 64, 16), (2, 48, 8, 16, 500, 8)]
    for _ in range(60):
        Hkv = int(rng.choice([1, 2, 4, 8]))
        shapes.append((int(rng.integers(1, 40)), Hkv * int(rng.choice([1, 2, 4, 8])), Hkv,
                       16 * int(rng.integers(1, 9)), int(rng.integers(1, 5000)),
                       int(rng.choice([1, 2, 4, 8, 16, 33, 64, 128]))))
    for B, Hq, Hkv, bs, mbps, nq in shapes:
        if nq * (Hq // Hkv) > 1024:
            continue
        d = dims(num_seqs=B, num_q_heads=Hq, num_kv_heads=Hkv, block_size=bs,
                 max_blocks_per_seq=mbps, num_blocks=mbps * B + 1)
        have = L.paged_attn_workspace_size(ctypes.byref(d), nq)
        assert have > 0
        for kv_dtype in (0, 1, 2):
            for sms in list(range(1, 300)) + [512, 1024]:
                need = _ws_needed(B, Hq, Hkv, bs, mbps, nq, kv_dtype, sms)
                assert have >= need, (B, Hq, Hkv, bs, mbps, nq, kv_dtype, sms, have, need)


def test_wait_limit_setter(L):
    """paged_attn_set_wait_limit returns the previous limit; 0 restores the
    default of one second (host state only)."""
    first = L.paged_attn_set_wait_limit(12345)
    assert first == 10 ** 9
    assert L.paged_attn_set_wait_limit(0) == 12345
    assert L.paged_attn_set_wait_limit(0) == 10 ** 9


def test_mode0_partition_formulas():
    """The static partition's closed forms (csrc/decode_tc.cu: cta_holding,
    cta_ending_from) against brute force over the CTA ranges
    [k W / Ce, (k+1) W / Ce): the CTA holding each chunk, the first CTA whose
    range ends at or after each chunk."""
    for W in range(1, 80):
        for Ce in range(1, min(W, 30) + 1):
            b = [k * W // Ce for k in range(Ce + 1)]
            for x in range(W):
                k = next(k for k in range(Ce) if b[k] <= x < b[k + 1])
                assert ((x + 1) * Ce - 1) // W == k
                first_end = next(k for k in range(Ce) if b[k + 1] - 1 >= x)
                assert ((x + 1) * Ce + W - 1) // W - 1 == first_end


def test_binding_refuses_tensors_the_kernel_would_read_out_of_bounds():
    """The C ABI takes bare pointers, so the binding checks dtype, shape and
    device of every tensor against the configuration before a call."""
    import torch
    from paged_kv_decode_flash_b200 import binding as b
    dec = object.__new__(b.PagedDecode)  # no device: the checks only
    dec.n_query = 4
    dec.dims = b.Dims(2, 16, 4, 128, 16, 10, 25, None, 0)
    dec.workspace = torch.empty(1024, dtype=torch.uint8)
    f16, i32 = torch.float16, torch.int32
    good = dict(q=torch.empty(2, 4, 16, 128, dtype=f16),
                k_cache=torch.empty(25, 4, 16, 128, dtype=f16),
                v_cache=torch.empty(25, 4, 16, 128, dtype=f16),
                block_table=torch.empty(2, 10, dtype=i32),
                context_lens=torch.empty(2, dtype=i32))
    dec.check_args(kv_dtype=b.KV_FP16, out=None, **good)
    q8 = torch.empty(25, 4, 16 * 136, dtype=torch.uint8)
    dec.check_args(kv_dtype=b.KV_Q8_0, out=None, **{**good, "k_cache": q8, "v_cache": q8})
    bad = [("q", torch.empty(2, 4, 16, 64, dtype=f16)),              # wrong head_dim
           ("q", torch.empty(2, 4, 16, 128, dtype=torch.float32)),   # wrong dtype
           ("k_cache", torch.empty(24, 4, 16, 128, dtype=f16)),      # fewer blocks than num_blocks
           ("v_cache", q8),                                          # q8_0 bytes given as fp16
           ("block_table", torch.empty(2, 9, dtype=i32)),            # short rows
           ("block_table", torch.empty(2, 10, dtype=torch.int64)),
           ("context_lens", torch.empty(3, dtype=i32))]
    for name, t in bad:
        with pytest.raises(ValueError, match=name):
            dec.check_args(kv_dtype=b.KV_FP16, out=None, **{**good, name: t})
    with pytest.raises(ValueError, match="out"):
        dec.check_args(kv_dtype=b.KV_FP16, out=torch.empty(2, 4, 16, 127, dtype=f16), **good)
    with pytest.raises(ValueError, match="kv_dtype"):
        dec.check_args(kv_dtype=7, out=None, **good)
