// api.cu -- the C ABI of libpagedattn (declared in include/pagedattn.h).
// Host code only: argument checks and the calls into dispatch.cu.
#include <cuda_runtime.h>

#include <cstdint>

#include "common.cuh"
#include "dispatch.h"
#include "kernels.h"
#include "pagedattn.h"

using namespace pa;

namespace {
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Checks shared by decode and its traced variant; on success *plan is the
// call's plan on the current device.
int prepare_decode(const pa_dims* dims, const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, const int32_t* context_lens, int32_t n_query,
                   int32_t causal, int32_t window, float scale, int32_t kv_dtype, const void* out,
                   Plan* plan) {
  int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  rc = check_decode_args(q, k_cache, v_cache, block_table, context_lens, causal, window, scale,
                         kv_dtype, out);
  if (rc != PA_OK) return rc;
  if (dims->workspace == nullptr || !aligned(dims->workspace, 256)) return PA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  *plan = make_plan(dims, n_query, kv_dtype, sms);
  if (dims->workspace_bytes < ws_layout(dims, n_query, *plan).total) return PA_ERR_WORKSPACE;
  return PA_OK;
}
}  // namespace

extern "C" {

size_t paged_attn_workspace_size(const pa_dims* dims, int32_t n_query) {
  if (check_dims(dims, n_query) != PA_OK) return 0;
  return ws_size_any_device(dims, n_query);
}

int32_t paged_attn_num_splits(const pa_dims* dims, int32_t n_query, int32_t kv_dtype) {
  const int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0 && kv_dtype != PA_KV_INT8_ROW)
    return PA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const Plan pl = make_plan(dims, n_query, kv_dtype, sms);
  if (pl.mode == 1) return pl.slots_per_group;
  if (pl.split_ctas > 0) {  // the per-head split kernel: CTAs per (sequence, KV head)
    const int groups = dims->num_seqs * dims->num_kv_heads;
    return (pl.split_ctas + groups - 1) / groups;
  }
  // A KV head's chunks span ceil(Ce / Hkv) ranges, plus one where they start
  // inside a range.
  return (pl.ctas_per_set + dims->num_kv_heads - 1) / dims->num_kv_heads + 1;
}

int32_t paged_attn_launches_per_call(const pa_dims* dims, int32_t n_query, int32_t kv_dtype) {
  const int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0 && kv_dtype != PA_KV_INT8_ROW)
    return PA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  return make_plan(dims, n_query, kv_dtype, sms).launches;
}

int paged_attn_workspace_init(const pa_dims* dims, void* stream) {
  if (dims == nullptr || dims->workspace == nullptr) return PA_ERR_WORKSPACE;
  if (check_dims(dims, 1) == PA_ERR_INVALID_ARG) return PA_ERR_INVALID_ARG;
  const size_t n = ws_zero_prefix(dims);
  if (dims->workspace_bytes < n) return PA_ERR_WORKSPACE;
  if (cudaMemsetAsync(dims->workspace, 0, n, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}

int paged_attn_decode(const pa_dims* dims, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_table,
                      const int32_t* context_lens, int32_t n_query, int32_t causal,
                      int32_t window, float scale, int32_t kv_dtype, void* out,
                      void* stream) {
  Plan plan;
  const int rc = prepare_decode(dims, q, k_cache, v_cache, block_table, context_lens, n_query,
                                causal, window, scale, kv_dtype, out, &plan);
  if (rc != PA_OK) return rc;
  return enqueue_decode(dims, plan, q, k_cache, v_cache, block_table, context_lens, n_query,
                        causal, window, scale, kv_dtype, out, dims->workspace, nullptr,
                        static_cast<cudaStream_t>(stream));
}

int paged_attn_decode_partial(const pa_dims* dims, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_table,
                              const int32_t* context_lens, const int32_t* key_begin,
                              const int32_t* key_count, int32_t n_query, int32_t causal,
                              int32_t window, float scale, int32_t kv_dtype, float* out,
                              float* out_lse, void* stream) {
  if (!key_begin || !key_count || !out_lse || !aligned(key_begin, 4) || !aligned(key_count, 4) ||
      !aligned(out_lse, 4))
    return PA_ERR_INVALID_ARG;
  Plan plan;
  const int rc = prepare_decode(dims, q, k_cache, v_cache, block_table, context_lens, n_query,
                                causal, window, scale, kv_dtype, out, &plan);
  if (rc != PA_OK) return rc;
  PartialArgs pa_args;
  pa_args.key_begin = key_begin;
  pa_args.key_count = key_count;
  pa_args.out = out;
  pa_args.out_lse = out_lse;
  return enqueue_decode(dims, plan, q, k_cache, v_cache, block_table, context_lens, n_query,
                        causal, window, scale, kv_dtype, nullptr, dims->workspace, nullptr,
                        static_cast<cudaStream_t>(stream), pa_args);
}

int paged_attn_trace(const pa_dims* dims, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_table,
                     const int32_t* context_lens, int32_t n_query, int32_t causal,
                     int32_t window, float scale, int32_t kv_dtype, void* out,
                     int32_t* trace, void* stream) {
  Plan plan;
  const int rc = prepare_decode(dims, q, k_cache, v_cache, block_table, context_lens, n_query,
                                causal, window, scale, kv_dtype, out, &plan);
  if (rc != PA_OK) return rc;
  if (trace == nullptr || !aligned(trace, 4)) return PA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long rows = (long long)dims->num_seqs * n_query * dims->num_q_heads;
  if (launch_trace_init(trace, rows, st) != cudaSuccess) return PA_ERR_CUDA;
  const int r = enqueue_decode(dims, plan, q, k_cache, v_cache, block_table, context_lens, n_query,
                               causal, window, scale, kv_dtype, out, dims->workspace, trace, st);
  if (r != PA_OK) return r;
  return launch_trace_finish(trace, rows, st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int paged_attn_merge(const float* partial_out, const float* partial_lse, int32_t num_splits,
                     int32_t rows, int32_t head_dim, void* out, float* out_lse, void* stream) {
  if (!partial_out || !partial_lse || !out) return PA_ERR_INVALID_ARG;
  if (num_splits < 1 || rows < 0) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (!aligned(partial_out, 16) || !aligned(partial_lse, 4) || !aligned(out, 8) ||
      (out_lse && !aligned(out_lse, 4)))
    return PA_ERR_INVALID_ARG;
  MergeParams m{};
  m.part_out = partial_out;
  m.part_lse = partial_lse;
  m.num_seqs = 1;
  m.num_splits = num_splits;
  m.rows_per_seq = rows;
  m.head_dim = head_dim;
  m.out = static_cast<__half*>(out);
  m.out_lse = out_lse;
  if (launch_merge(m, static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}

int paged_attn_get_error(const pa_dims* dims, void* stream) {
  if (dims == nullptr || dims->workspace == nullptr || dims->workspace_bytes < kWsHeader)
    return PA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  unsigned flags = 0;
  if (cudaMemcpyAsync(&flags, dims->workspace, sizeof(flags), cudaMemcpyDeviceToHost, st) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  // Clear the flag; after a timeout clear the counters too (a safety net:
  // the kernels keep them consistent on that path as well).
  size_t n = sizeof(flags);
  if ((flags & kFlagTimeout) && check_dims(dims, 1) != PA_ERR_INVALID_ARG &&
      dims->workspace_bytes >= ws_zero_prefix(dims))
    n = ws_zero_prefix(dims);
  if (cudaMemsetAsync(dims->workspace, 0, n, st) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  if (flags & kFlagTimeout) return PA_ERR_TIMEOUT;
  if (flags & kFlagBadBlock) return PA_ERR_BAD_BLOCK_INDEX;
  if (flags & kFlagBadLen) return PA_ERR_BAD_CONTEXT_LEN;
  return PA_OK;
}

uint64_t paged_attn_set_wait_limit(uint64_t nanoseconds) {
  return set_wait_limit_ns(nanoseconds);
}

int paged_attn_cache_write(const pa_dims* dims, const void* k_new, const void* v_new,
                           const int32_t* block_table, const int32_t* context_lens,
                           int32_t n_new, int32_t kv_dtype, void* k_cache, void* v_cache,
                           void* stream) {
  const int rc = check_dims(dims, n_new);
  if (rc != PA_OK && rc != PA_ERR_UNSUPPORTED) return rc;
  if (dims->head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if (!k_new || !v_new || !block_table || !context_lens || !k_cache || !v_cache)
    return PA_ERR_INVALID_ARG;
  if (!aligned(k_new, 8) || !aligned(v_new, 8) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_table, 4) || !aligned(context_lens, 4))
    return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0 && kv_dtype != PA_KV_INT8_ROW)
    return PA_ERR_INVALID_ARG;
  if (dims->workspace == nullptr || dims->workspace_bytes < kWsHeader) return PA_ERR_WORKSPACE;
  CacheWriteParams p{};
  p.k_new = static_cast<const __half*>(k_new);
  p.v_new = static_cast<const __half*>(v_new);
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.block_table = block_table;
  p.context_lens = context_lens;
  p.num_seqs = dims->num_seqs;
  p.num_kv_heads = dims->num_kv_heads;
  p.block_size = dims->block_size;
  p.max_blocks_per_seq = dims->max_blocks_per_seq;
  p.num_blocks = dims->num_blocks;
  p.n_new = n_new;
  p.kv_dtype = kv_dtype;
  p.flags = static_cast<unsigned*>(dims->workspace);
  return launch_cache_write(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PA_OK
                                                                                 : PA_ERR_CUDA;
}

const char* paged_attn_status_string(int32_t status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_INVALID_ARG: return "invalid argument";
    case PA_ERR_UNSUPPORTED: return "unsupported shape or type";
    case PA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PA_ERR_CUDA: return "CUDA runtime error";
    case PA_ERR_BAD_BLOCK_INDEX: return "block_table entry out of range";
    case PA_ERR_BAD_CONTEXT_LEN: return "context length out of range";
    case PA_ERR_TIMEOUT: return "a device-side wait timed out; output invalid";
    default: return "unknown status";
  }
}

}  // extern "C"
