"""ctypes front end of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this package; the product path never
does.  ``build()`` compiles oracle.c with gcc (plain C, -O2, OpenMP, no fast
math) into liboracle.so next to this file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
HDR = os.path.join(HERE, "oracle.h")
LIB = os.path.join(HERE, "liboracle.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_BAD_BLOCK_INDEX = -2
ERR_BAD_CONTEXT_LEN = -3


def build(plant: int = 0, out: str | None = None, openmp: bool = True) -> str:
    """Compile the oracle.  ``plant`` > 0 builds a variant with one planted
    mistake (only for the test that shows the pins catch mistakes)."""
    out = out or LIB
    if plant == 0 and out == LIB and os.path.exists(LIB):
        newest = max(os.path.getmtime(SRC), os.path.getmtime(HDR))
        if os.path.getmtime(LIB) >= newest:
            return LIB
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-Wno-unknown-pragmas", f"-DORACLE_PLANT={plant}", SRC, "-o", out, "-lm"]
    if openmp:
        cmd.insert(1, "-fopenmp")
    tmp = out + f".tmp{os.getpid()}"
    cmd[cmd.index(out)] = tmp
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    os.replace(tmp, out)
    return out


class _Problem(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32), ("max_blocks_per_seq", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32), ("n_query", ctypes.c_int32),
        ("causal", ctypes.c_int32), ("window", ctypes.c_int32),
        ("kv_dtype", ctypes.c_int32), ("scale", ctypes.c_double),
        ("q", ctypes.c_void_p), ("k_cache", ctypes.c_void_p),
        ("v_cache", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
        ("context_lens", ctypes.c_void_p),
    ]


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__(f"oracle returned {code}")
        self.code = code


class Oracle:
    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(_Problem)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        lib.oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_half_to_double.restype = ctypes.c_double
        lib.oracle_key_visible.argtypes = [i64, i32, i32, i32, i32, i64]
        lib.oracle_key_visible.restype = ctypes.c_int
        lib.oracle_attend_row.argtypes = [P, i32, i32, i32, i64, i64, vp, vp]
        lib.oracle_attend_row.restype = ctypes.c_int
        lib.oracle_paged_attn.argtypes = [P, vp, vp]
        lib.oracle_paged_attn.restype = ctypes.c_int
        lib.oracle_paged_attn_rows.argtypes = [P, vp, i64, vp, vp]
        lib.oracle_paged_attn_rows.restype = ctypes.c_int
        lib.oracle_trace.argtypes = [P, vp]
        lib.oracle_trace.restype = ctypes.c_int
        lib.oracle_merge.argtypes = [vp, vp, i32, i64, i32, vp, vp]
        lib.oracle_merge.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_num_threads.restype = None
        lib.oracle_float_to_half.argtypes = [ctypes.c_float]
        lib.oracle_float_to_half.restype = ctypes.c_uint16
        lib.oracle_quantize_q8_0.argtypes = [vp, vp, vp]
        lib.oracle_quantize_q8_0.restype = None
        lib.oracle_quantize_row.argtypes = [vp, i32, vp, vp]
        lib.oracle_quantize_row.restype = None
        lib.oracle_cache_write.argtypes = [P, vp, vp, vp, vp]
        lib.oracle_cache_write.restype = ctypes.c_int
        self.lib = lib

    # -- helpers -----------------------------------------------------------
    @staticmethod
    def _problem(case, keep: list) -> _Problem:
        arrs = [np.ascontiguousarray(case.q).view(np.uint16),
                np.ascontiguousarray(case.k_cache), np.ascontiguousarray(case.v_cache),
                np.ascontiguousarray(case.block_table, dtype=np.int32),
                np.ascontiguousarray(case.context_lens, dtype=np.int32)]
        keep.extend(arrs)
        return _Problem(
            case.num_seqs, case.num_q_heads, case.num_kv_heads, case.head_dim,
            case.block_size, case.max_blocks_per_seq, case.num_blocks,
            case.n_query, case.causal, case.window, case.kv_dtype,
            float(case.scale), *[_ptr(a) for a in arrs])

    def half_to_double(self, bits: int) -> float:
        return self.lib.oracle_half_to_double(bits)

    def key_visible(self, L, n_query, i, causal, window, j) -> bool:
        return bool(self.lib.oracle_key_visible(L, n_query, i, causal, window, j))

    def num_threads(self) -> int:
        return self.lib.oracle_num_threads()

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    # -- quantise on write ---------------------------------------------------
    def float_to_half(self, f) -> int:
        """fp16 bits of an fp32 value, round to nearest even."""
        return int(self.lib.oracle_float_to_half(float(np.float32(f))))

    def quantize_q8_0(self, x32: np.ndarray):
        """32 fp32 values -> (int8 q[32], fp16 scale bits)."""
        x = np.ascontiguousarray(x32, dtype=np.float32)
        assert x.size == 32
        q = np.zeros(32, dtype=np.int8)
        d = np.zeros(1, dtype=np.uint16)
        self.lib.oracle_quantize_q8_0(_ptr(x), _ptr(q), _ptr(d))
        return q, int(d[0])

    def quantize_row(self, x: np.ndarray):
        """n fp32 values -> (int8 q[n], fp32 scale)."""
        xx = np.ascontiguousarray(x, dtype=np.float32)
        q = np.zeros(xx.size, dtype=np.int8)
        sc = np.zeros(1, dtype=np.float32)
        self.lib.oracle_quantize_row(_ptr(xx), xx.size, _ptr(q), _ptr(sc))
        return q, float(sc[0])

    def cache_write(self, case, k_new: np.ndarray, v_new: np.ndarray):
        """The case's caches after writing k_new/v_new (fp16 [B][n_new][Hkv][D],
        n_new = case.n_query) for the last n_new positions of every sequence.
        Returns (k_cache, v_cache, status)."""
        keep: list = []
        p = self._problem(case, keep)
        kc = np.ascontiguousarray(case.k_cache).copy()
        vc = np.ascontiguousarray(case.v_cache).copy()
        kn = np.ascontiguousarray(k_new, dtype=np.float16).view(np.uint16)
        vn = np.ascontiguousarray(v_new, dtype=np.float16).view(np.uint16)
        rc = self.lib.oracle_cache_write(ctypes.byref(p), _ptr(kn), _ptr(vn), _ptr(kc), _ptr(vc))
        return kc, vc, int(rc)

    # -- the computation ---------------------------------------------------
    def attend(self, case):
        """All rows: (out [B][nq][Hq][D] float64, lse [B][nq][Hq] float64)."""
        keep: list = []
        p = self._problem(case, keep)
        out = np.zeros((case.num_seqs, case.n_query, case.num_q_heads, case.head_dim))
        lse = np.zeros((case.num_seqs, case.n_query, case.num_q_heads))
        rc = self.lib.oracle_paged_attn(ctypes.byref(p), _ptr(out), _ptr(lse))
        if rc:
            raise OracleError(rc)
        return out, lse

    def attend_rows(self, case, row_ids):
        """Selected rows (row id = (s*nq + i)*Hq + h): (out [n][D], lse [n])."""
        keep: list = []
        p = self._problem(case, keep)
        ids = np.ascontiguousarray(row_ids, dtype=np.int64)
        out = np.zeros((ids.size, case.head_dim))
        lse = np.zeros(ids.size)
        rc = self.lib.oracle_paged_attn_rows(ctypes.byref(p), _ptr(ids), ids.size,
                                             _ptr(out), _ptr(lse))
        if rc:
            raise OracleError(rc)
        return out, lse

    def attend_row_range(self, case, s, i, h, j_begin, j_end):
        keep: list = []
        p = self._problem(case, keep)
        out = np.zeros(case.head_dim)
        lse = np.zeros(1)
        rc = self.lib.oracle_attend_row(ctypes.byref(p), s, i, h, j_begin, j_end,
                                        _ptr(out), _ptr(lse))
        if rc:
            raise OracleError(rc)
        return out, float(lse[0])

    def trace(self, case) -> np.ndarray:
        keep: list = []
        p = self._problem(case, keep)
        t = np.zeros((case.rows, 5), dtype=np.int32)
        rc = self.lib.oracle_trace(ctypes.byref(p), _ptr(t))
        if rc:
            raise OracleError(rc)
        return t

    def merge(self, part_out: np.ndarray, part_lse: np.ndarray):
        """part_out [S][rows][D], part_lse [S][rows] -> (out, lse)."""
        po = np.ascontiguousarray(part_out, dtype=np.float64)
        pl = np.ascontiguousarray(part_lse, dtype=np.float64)
        S, rows, D = po.shape
        out = np.zeros((rows, D))
        lse = np.zeros(rows)
        self.lib.oracle_merge(_ptr(po), _ptr(pl), S, rows, D, _ptr(out), _ptr(lse))
        return out, lse


_lock = threading.Lock()
_default: Oracle | None = None


def load(path: str | None = None) -> Oracle:
    """The default oracle (built on first use), or the library at ``path``."""
    global _default
    if path is not None:
        return Oracle(path)
    with _lock:
        if _default is None:
            _default = Oracle(build())
        return _default
