"""paged_attn_decode_noalloc: the decode entry point for callers that cannot
give the library device memory (a host program that owns every byte of the
GPU's memory in one pre-planned pool, a plug-in host without an allocator, or
a hot path that must not call cudaMalloc because it can synchronise the
device).  Its split partials live in one fixed array inside the library.

Checked here through the C ABI: calls in a row (different shapes, cache
types and work decompositions, so each call runs over the previous one's
leftovers in the shared array) each give bit for bit what paged_attn_decode
gives -- the same plan and kernel, so any difference would be a bug in the
shared array's handling -- and shapes too large for the array are refused
before anything is enqueued.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from paged_kv_decode_flash_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from paged_kv_decode_flash_b200 import binding, build
    build.build()  # no-op when the in-tree library is up to date
    L = binding.lib()
    f = L.paged_attn_decode_noalloc
    vp, i32 = ctypes.c_void_p, ctypes.c_int32
    f.argtypes = [ctypes.POINTER(binding.Dims), vp, vp, vp, vp, vp, i32, i32, i32,
                  ctypes.c_float, i32, vp, vp]
    f.restype = ctypes.c_int
    return binding


def call_noalloc(B, case, dev, out):
    dims = B.Dims(case.num_seqs, case.num_q_heads, case.num_kv_heads, case.head_dim,
                  case.block_size, case.max_blocks_per_seq, case.num_blocks, None, 0)
    rc = B.lib().paged_attn_decode_noalloc(
        ctypes.byref(dims), dev["q"].data_ptr(), dev["k_cache"].data_ptr(),
        dev["v_cache"].data_ptr(), dev["block_table"].data_ptr(),
        dev["context_lens"].data_ptr(), case.n_query, case.causal, case.window,
        case.scale, case.kv_dtype, out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    return rc


def test_noalloc_matches_decode_on_consecutive_calls(B):
    a = gen.make_case(seed=31, context_lens=(5000,), n_query=8, num_q_heads=32,
                      num_kv_heads=8, causal=1)
    b = gen.make_case(seed=32, context_lens=(700, 2100, 64), n_query=4, num_q_heads=16,
                      num_kv_heads=4, causal=1, window=300, kv_dtype=gen.KV_Q8_0)
    c = gen.make_case(seed=33, context_lens=tuple(range(300, 4300, 100)), n_query=2,
                      num_q_heads=32, num_kv_heads=8, causal=1, kv_dtype=gen.KV_INT8_ROW)
    results = []
    for case in (a, b, c, a):
        dev = B.case_to_device(case)
        ref, dec = B.decode_case(case)
        out = torch.full_like(dev["q"], float("nan"))
        assert call_noalloc(B, case, dev, out) == B.PA_OK
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert np.array_equal(got.view(np.uint16), ref.cpu().numpy().view(np.uint16)), \
            "noalloc differs from paged_attn_decode"
        results.append(got)
    assert np.array_equal(results[0].view(np.uint16), results[3].view(np.uint16))


def test_noalloc_refuses_shapes_beyond_its_scratch(B):
    small = torch.zeros(64, dtype=torch.float16, device="cuda")
    ints = torch.zeros(64, dtype=torch.int32, device="cuda")
    # 64 sequences x 8 query tokens x 64 query heads need more than 16 MiB of
    # split partials.
    dims = B.Dims(64, 64, 8, 128, 16, 4096, 4096, None, 0)
    p, ip = small.data_ptr(), ints.data_ptr()
    rc = B.lib().paged_attn_decode_noalloc(ctypes.byref(dims), p, p, p, ip, ip, 8, 1, 0,
                                           0.088, 0, p, torch.cuda.current_stream().cuda_stream)
    assert rc == B.PA_ERR_WORKSPACE
