// kernels.h -- launchers of the libpagedattn kernels (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include "common.cuh"

namespace pa {

// Split-KV paged decode on the tensor cores (tcgen05/TMEM, TMA / bulk-copy
// staged KV tiles), merge included: one launch per call (per kMaxQueueSeqs
// sequences in work-queue mode).  Records the key-resolution trace when
// p.trace is set.
cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream);
// Most query rows one CTA handles per KV head for a cache type.
int max_rows_per_part(int kv_dtype);

// The per-head split kernel (decode_split.cu): fp16 cache, few (sequence,
// KV head) groups, up to 8 query tokens and 32 rows per KV head, every key
// of the context.  Each group's 128-key tiles are cut into contiguous runs
// over its share of `ctas` CTAs; partial slots are CTA-indexed (rows
// [cta * rows, cta * rows + rows)); merge included; records the trace when
// p.trace is set.  Only p's fields of a mode-0 plan are read.
bool split_decode_supported(int kv_dtype, int n_query, int rows, int num_blocks,
                            int num_kv_heads, int block_size);
cudaError_t launch_split_decode(const DecodeParams& p, int ctas, cudaStream_t stream);

// Log-sum-exp merge of split partials into fp16 rows.
cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream);

// Key-resolution record: set every row to {0, INT32_MAX, -1, 0, 0} before
// a traced decode, and rows no key reached to {0, -1, -1, 0, 0} after it.
cudaError_t launch_trace_init(int32_t* trace, long long rows, cudaStream_t stream);
cudaError_t launch_trace_finish(int32_t* trace, long long rows, cudaStream_t stream);

// Quantise new keys/values and write them into the paged cache.
struct CacheWriteParams {
  const __half* k_new;         // [B][n_new][Hkv][D]
  const __half* v_new;
  void* k_cache;
  void* v_cache;
  const int32_t* block_table;  // [B][mbps]
  const int32_t* context_lens; // [B]: the new tokens are the last n_new positions
  int num_seqs, num_kv_heads, block_size, max_blocks_per_seq, num_blocks, n_new, kv_dtype;
  unsigned* flags;             // data-error flags (a workspace status word)
};
cudaError_t launch_cache_write(const CacheWriteParams& p, cudaStream_t stream);

}  // namespace pa
