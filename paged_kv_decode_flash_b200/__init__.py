"""libpagedattn: decode attention over a paged KV cache on B200 (sm_100a).

The computation lives in the CUDA library libpagedattn.so (C ABI in
include/pagedattn.h); ``paged_kv_decode_flash_b200.binding`` is a thin ctypes
layer over it and ``paged_kv_decode_flash_b200.inputs`` makes seeded
synthetic workloads.
"""
