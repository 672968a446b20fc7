"""Thin ctypes binding of libpagedattn (include/pagedattn.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  torch supplies device memory and streams.  There is no fallback:
if libpagedattn.so is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import inputs as _inputs

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_WORKSPACE = -3
PA_ERR_CUDA = -4
PA_ERR_BAD_BLOCK_INDEX = -5
PA_ERR_BAD_CONTEXT_LEN = -6
PA_ERR_TIMEOUT = -7

KV_FP16 = _inputs.KV_FP16
KV_Q8_0 = _inputs.KV_Q8_0
KV_INT8_ROW = _inputs.KV_INT8_ROW


class PagedAttnError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: libpagedattn status {code} ({status_string(code)})")


class Dims(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


_lock = threading.Lock()
_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libpagedattn.so (raises if it has not been built)."""
    global _LIB
    with _lock:
        if _LIB is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m paged_kv_decode_flash_b200.build` (no fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            P = ctypes.POINTER(Dims)
            vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
            L.paged_attn_workspace_size.argtypes = [P, i32]
            L.paged_attn_workspace_size.restype = ctypes.c_size_t
            L.paged_attn_workspace_init.argtypes = [P, vp]
            L.paged_attn_workspace_init.restype = ctypes.c_int
            L.paged_attn_decode.argtypes = [P, vp, vp, vp, vp, vp, i32, i32, i32, f32, i32, vp, vp]
            L.paged_attn_decode.restype = ctypes.c_int
            L.paged_attn_merge.argtypes = [vp, vp, i32, i32, i32, vp, vp, vp]
            L.paged_attn_merge.restype = ctypes.c_int
            L.paged_attn_get_error.argtypes = [P, vp]
            L.paged_attn_get_error.restype = ctypes.c_int
            L.paged_attn_trace.argtypes = [P, vp, vp, vp, vp, vp, i32, i32, i32, f32, i32, vp, vp, vp]
            L.paged_attn_trace.restype = ctypes.c_int
            L.paged_attn_decode_partial.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                                    f32, i32, vp, vp, vp]
            L.paged_attn_decode_partial.restype = ctypes.c_int
            L.paged_attn_set_wait_limit.argtypes = [ctypes.c_uint64]
            L.paged_attn_set_wait_limit.restype = ctypes.c_uint64
            L.paged_attn_cache_write.argtypes = [P, vp, vp, vp, vp, i32, i32, vp, vp, vp]
            L.paged_attn_cache_write.restype = ctypes.c_int
            L.paged_attn_num_splits.argtypes = [P, i32, i32]
            L.paged_attn_num_splits.restype = ctypes.c_int32
            L.paged_attn_launches_per_call.argtypes = [P, i32, i32]
            L.paged_attn_launches_per_call.restype = ctypes.c_int32
            L.paged_attn_status_string.argtypes = [i32]
            L.paged_attn_status_string.restype = ctypes.c_char_p
            _LIB = L
        return _LIB


def status_string(code: int) -> str:
    try:
        return lib().paged_attn_status_string(code).decode()
    except Exception:  # the library itself may be what is missing
        return "?"


def _check(code: int, what: str) -> None:
    if code != PA_OK:
        raise PagedAttnError(code, what)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libpagedattn takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libpagedattn takes contiguous tensors")
    return t.data_ptr()


def _expect(t: torch.Tensor, name: str, dtype, shape) -> None:
    """The C ABI takes bare pointers: a tensor of the wrong type or size
    would be read out of bounds, so it is refused here."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")


def set_wait_limit(nanoseconds: int) -> int:
    """Time after which device-side pipeline waits give up (PA_ERR_TIMEOUT)
    for later calls of this process; 0 restores the default (1 s).  Returns
    the previous value."""
    return int(lib().paged_attn_set_wait_limit(int(nanoseconds)))


def cache_shape(kv_dtype: int, num_blocks: int, num_kv_heads: int, block_size: int, head_dim: int):
    """(torch dtype, shape) of one cache tensor (include/pagedattn.h layouts)."""
    if int(kv_dtype) == KV_FP16:
        return torch.float16, (num_blocks, num_kv_heads, block_size, head_dim)
    if int(kv_dtype) == KV_Q8_0:
        return torch.uint8, (num_blocks, num_kv_heads, block_size * (head_dim + 2 * (head_dim // 32)))
    if int(kv_dtype) == KV_INT8_ROW:
        return torch.uint8, (num_blocks, num_kv_heads, block_size * (head_dim + 4))
    raise ValueError(f"kv_dtype {kv_dtype}: expected {KV_FP16} (fp16), {KV_Q8_0} (q8_0) "
                     f"or {KV_INT8_ROW} (int8 rows)")


class PagedDecode:
    """Owns the shapes and the workspace of one decode configuration.

    ``q`` fp16 [B][nq][Hq][D]; caches as described in include/pagedattn.h
    (fp16 [NB][Hkv][bs][D] or uint8 q8_0 tiles [NB][Hkv][tile]);
    ``block_table`` int32 [B][max_blocks_per_seq]; ``context_lens`` int32 [B].
    """

    def __init__(self, *, num_seqs: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, max_blocks_per_seq: int,
                 num_blocks: int, n_query: int, device=None, workspace=None):
        self.n_query = n_query
        self.dims = Dims(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                         max_blocks_per_seq, num_blocks, None, 0)
        need = lib().paged_attn_workspace_size(ctypes.byref(self.dims), n_query)
        if need == 0:
            raise PagedAttnError(PA_ERR_INVALID_ARG, "workspace_size (bad shapes)")
        self.workspace_bytes = int(need)
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=device or "cuda")
        elif workspace.numel() * workspace.element_size() < need:
            raise PagedAttnError(PA_ERR_WORKSPACE, "workspace too small")
        self.workspace = workspace
        self.dims.workspace = _dptr(workspace)
        self.dims.workspace_bytes = workspace.numel() * workspace.element_size()
        _check(lib().paged_attn_workspace_init(ctypes.byref(self.dims), _stream_ptr(None)),
               "workspace_init")

    @classmethod
    def for_case(cls, case, device=None):
        return cls(num_seqs=case.num_seqs, num_q_heads=case.num_q_heads,
                   num_kv_heads=case.num_kv_heads, head_dim=case.head_dim,
                   block_size=case.block_size, max_blocks_per_seq=case.max_blocks_per_seq,
                   num_blocks=case.num_blocks, n_query=case.n_query, device=device)

    def num_splits(self, kv_dtype: int = KV_FP16) -> int:
        n = lib().paged_attn_num_splits(ctypes.byref(self.dims), self.n_query, int(kv_dtype))
        if n < 0:
            raise PagedAttnError(n, "num_splits")
        return n

    def launches_per_call(self, kv_dtype: int = KV_FP16) -> int:
        n = lib().paged_attn_launches_per_call(ctypes.byref(self.dims), self.n_query, int(kv_dtype))
        if n < 0:
            raise PagedAttnError(n, "launches_per_call")
        return n

    def check_args(self, q, k_cache, v_cache, block_table, context_lens, kv_dtype, out=None):
        """dtype, shape and device of every tensor a decode call reads or
        writes, against this configuration (include/pagedattn.h layouts)."""
        d = self.dims
        B, nq, Hq, Hkv, D = d.num_seqs, self.n_query, d.num_q_heads, d.num_kv_heads, d.head_dim
        _expect(q, "q", torch.float16, (B, nq, Hq, D))
        if out is not None:
            _expect(out, "out", torch.float16, (B, nq, Hq, D))
        _expect(block_table, "block_table", torch.int32, (B, d.max_blocks_per_seq))
        _expect(context_lens, "context_lens", torch.int32, (B,))
        cache = cache_shape(kv_dtype, d.num_blocks, Hkv, d.block_size, D)
        _expect(k_cache, "k_cache", *cache)
        _expect(v_cache, "v_cache", *cache)
        dev = self.workspace.device
        for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                        ("block_table", block_table), ("context_lens", context_lens),
                        ("out", out)):
            if t is not None and t.device != dev:
                raise ValueError(f"{name} is on {t.device}, the workspace on {dev}")

    def __call__(self, q, k_cache, v_cache, block_table, context_lens, *, causal: int,
                 window: int, scale: float, kv_dtype: int, out=None, stream=None):
        self.check_args(q, k_cache, v_cache, block_table, context_lens, kv_dtype, out)
        if out is None:
            out = torch.empty_like(q)
        rc = lib().paged_attn_decode(
            ctypes.byref(self.dims), _dptr(q), _dptr(k_cache), _dptr(v_cache),
            _dptr(block_table), _dptr(context_lens), self.n_query, int(causal), int(window),
            float(scale), int(kv_dtype), _dptr(out), _stream_ptr(stream))
        _check(rc, "paged_attn_decode")
        return out

    def partial(self, q, k_cache, v_cache, block_table, context_lens, key_begin, key_count, *,
                causal: int, window: int, scale: float, kv_dtype: int, out=None, out_lse=None,
                stream=None):
        """paged_attn_decode_partial: this call's share of each sequence's
        keys, [key_begin, key_begin + key_count), with block_table mapping
        local blocks.  Returns (out fp32 [B][nq][Hq][D], out_lse fp32
        [B][nq][Hq])."""
        self.check_args(q, k_cache, v_cache, block_table, context_lens, kv_dtype, None)
        B = self.dims.num_seqs
        _expect(key_begin, "key_begin", torch.int32, (B,))
        _expect(key_count, "key_count", torch.int32, (B,))
        shp = tuple(q.shape)
        if out is None:
            out = torch.empty(shp, dtype=torch.float32, device=q.device)
        if out_lse is None:
            out_lse = torch.empty(shp[:-1], dtype=torch.float32, device=q.device)
        _expect(out, "out", torch.float32, shp)
        _expect(out_lse, "out_lse", torch.float32, shp[:-1])
        rc = lib().paged_attn_decode_partial(
            ctypes.byref(self.dims), _dptr(q), _dptr(k_cache), _dptr(v_cache),
            _dptr(block_table), _dptr(context_lens), _dptr(key_begin), _dptr(key_count),
            self.n_query, int(causal), int(window), float(scale), int(kv_dtype), _dptr(out),
            _dptr(out_lse), _stream_ptr(stream))
        _check(rc, "paged_attn_decode_partial")
        return out, out_lse

    def get_error(self, stream=None) -> int:
        """Synchronises and returns (and clears) the device data-error status."""
        return lib().paged_attn_get_error(ctypes.byref(self.dims), _stream_ptr(stream))

    def trace(self, q, k_cache, v_cache, block_table, context_lens, *, causal: int,
              window: int, scale: float, kv_dtype: int, out=None, stream=None):
        """paged_attn_trace: the decode plus the key-resolution record of the
        kernel that read the cache.  Returns (out, trace int32 [B][nq][Hq][5])."""
        self.check_args(q, k_cache, v_cache, block_table, context_lens, kv_dtype, out)
        if out is None:
            out = torch.empty_like(q)
        B, nq, Hq = self.dims.num_seqs, self.n_query, self.dims.num_q_heads
        t = torch.empty((B, nq, Hq, 5), dtype=torch.int32, device=q.device)
        rc = lib().paged_attn_trace(
            ctypes.byref(self.dims), _dptr(q), _dptr(k_cache), _dptr(v_cache),
            _dptr(block_table), _dptr(context_lens), nq, int(causal), int(window),
            float(scale), int(kv_dtype), _dptr(out), _dptr(t), _stream_ptr(stream))
        _check(rc, "paged_attn_trace")
        return out, t

    def cache_write(self, k_new, v_new, block_table, context_lens, *, kv_dtype: int, k_cache,
                    v_cache, stream=None):
        """paged_attn_cache_write: the n_query newest tokens' K/V (fp16
        [B][n_query][Hkv][D]) into the paged cache, quantised for the int8
        caches.  Data errors go to this decoder's workspace (get_error)."""
        d = self.dims
        shp = (d.num_seqs, self.n_query, d.num_kv_heads, d.head_dim)
        _expect(k_new, "k_new", torch.float16, shp)
        _expect(v_new, "v_new", torch.float16, shp)
        _expect(block_table, "block_table", torch.int32, (d.num_seqs, d.max_blocks_per_seq))
        _expect(context_lens, "context_lens", torch.int32, (d.num_seqs,))
        cache = cache_shape(kv_dtype, d.num_blocks, d.num_kv_heads, d.block_size, d.head_dim)
        _expect(k_cache, "k_cache", *cache)
        _expect(v_cache, "v_cache", *cache)
        rc = lib().paged_attn_cache_write(
            ctypes.byref(d), _dptr(k_new), _dptr(v_new), _dptr(block_table),
            _dptr(context_lens), self.n_query, int(kv_dtype), _dptr(k_cache), _dptr(v_cache),
            _stream_ptr(stream))
        _check(rc, "paged_attn_cache_write")


def merge(partial_out: torch.Tensor, partial_lse: torch.Tensor, out=None, out_lse=None,
          stream=None):
    """partial_out fp32 [S][rows][D], partial_lse fp32 [S][rows] ->
    (out fp16 [rows][D], out_lse fp32 [rows])."""
    S, rows, D = partial_out.shape
    _expect(partial_out, "partial_out", torch.float32, (S, rows, D))
    _expect(partial_lse, "partial_lse", torch.float32, (S, rows))
    if out is not None:
        _expect(out, "out", torch.float16, (rows, D))
    if out_lse is not None:
        _expect(out_lse, "out_lse", torch.float32, (rows,))
    if out is None:
        out = torch.empty((rows, D), dtype=torch.float16, device=partial_out.device)
    if out_lse is None:
        out_lse = torch.empty((rows,), dtype=torch.float32, device=partial_out.device)
    rc = lib().paged_attn_merge(_dptr(partial_out), _dptr(partial_lse), S, rows, D,
                                _dptr(out), _dptr(out_lse), _stream_ptr(stream))
    _check(rc, "paged_attn_merge")
    return out, out_lse


def case_to_device(case, device="cuda"):
    """Upload a generated Case's arrays (no arithmetic, copies only)."""
    t = lambda a: torch.from_numpy(a).to(device)
    return dict(q=t(case.q), k_cache=t(case.k_cache), v_cache=t(case.v_cache),
                block_table=t(case.block_table), context_lens=t(case.context_lens))


def decode_case(case, device="cuda", dec: PagedDecode | None = None, out=None):
    """Run paged_attn_decode on a generated Case; returns (out tensor, decoder)."""
    dev = case_to_device(case, device)
    dec = dec or PagedDecode.for_case(case, device=device)
    out = dec(dev["q"], dev["k_cache"], dev["v_cache"], dev["block_table"],
              dev["context_lens"], causal=case.causal, window=case.window,
              scale=case.scale, kv_dtype=case.kv_dtype, out=out)
    return out, dec
