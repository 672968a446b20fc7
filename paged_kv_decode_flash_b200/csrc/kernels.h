// kernels.h -- launchers of the libpagedattn kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace pa {

// Plain split-KV decode on CUDA cores (any block_size % 16 == 0, fp16/q8_0).
size_t decode_simt_smem_bytes(int rows);
cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t stream);

// Split-KV decode on the tensor cores (tcgen05/TMEM, TMA-staged fp16 tiles).
// One CTA per SM; fp16 cache, rows = n_query * group <= 32.  Also merges the
// split partials into p.out (the last CTA of each (sequence, KV head)).
bool decode_tc_supported(int kv_dtype, int rows, int num_blocks, int num_kv_heads, int block_size);
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream);

// Log-sum-exp merge of split partials into fp16 rows.
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);

// Per-row key-resolution record (debug / tests).
cudaError_t launch_trace(const DecodeParams& p, int32_t* trace, cudaStream_t stream);

}  // namespace pa
