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
}  // namespace

extern "C" {

size_t paged_attn_workspace_size(const pa_dims* dims, int32_t n_query) {
  if (check_dims(dims, n_query) != PA_OK) return 0;
  return ws_layout(dims, n_query, max_plan(dims).splits).total;
}

int32_t paged_attn_num_splits(const pa_dims* dims, int32_t n_query, int32_t kv_dtype) {
  const int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  return make_plan(dims, n_query, kv_dtype, sms).splits;
}

int32_t paged_attn_launches_per_call(const pa_dims* dims, int32_t n_query, int32_t kv_dtype) {
  const int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  // tensor-core kernel: merges in its last CTAs; CUDA-core kernel: + merge kernel
  return make_plan(dims, n_query, kv_dtype, sms).tensor_cores ? 1 : 2;
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
  int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  rc = check_decode_args(q, k_cache, v_cache, block_table, context_lens, causal, window, scale,
                         kv_dtype, out);
  if (rc != PA_OK) return rc;
  if (dims->workspace == nullptr || !aligned(dims->workspace, 256)) return PA_ERR_WORKSPACE;
  const int sms = device_sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const Plan plan = make_plan(dims, n_query, kv_dtype, sms);
  if (dims->workspace_bytes < ws_layout(dims, n_query, plan.splits).total) return PA_ERR_WORKSPACE;
  return enqueue_decode(dims, plan, q, k_cache, v_cache, block_table, context_lens, n_query,
                        causal, window, scale, kv_dtype, out, dims->workspace,
                        static_cast<cudaStream_t>(stream));
}

int paged_attn_merge(const float* partial_out, const float* partial_lse, int32_t num_splits,
                     int32_t rows, int32_t head_dim, void* out, float* out_lse, void* stream) {
  if (!partial_out || !partial_lse || !out) return PA_ERR_INVALID_ARG;
  if (num_splits < 1 || rows < 0) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return PA_ERR_UNSUPPORTED;
  if (!aligned(partial_out, 4) || !aligned(partial_lse, 4) || !aligned(out, 2) ||
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
  if (cudaMemsetAsync(dims->workspace, 0, sizeof(flags), st) != cudaSuccess) return PA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PA_ERR_CUDA;
  if (flags & kFlagTimeout) return PA_ERR_TIMEOUT;
  if (flags & kFlagBadBlock) return PA_ERR_BAD_BLOCK_INDEX;
  if (flags & kFlagBadLen) return PA_ERR_BAD_CONTEXT_LEN;
  return PA_OK;
}

int paged_attn_trace(const pa_dims* dims, const int32_t* block_table,
                     const int32_t* context_lens, int32_t n_query, int32_t causal,
                     int32_t window, int32_t* trace, void* stream) {
  if (dims == nullptr || n_query < 1 || n_query > kMaxQuery) return PA_ERR_INVALID_ARG;
  if (dims->num_seqs < 1 || dims->num_q_heads < 1 || dims->block_size < 1 ||
      dims->max_blocks_per_seq < 1 || dims->num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (!block_table || !context_lens || !trace) return PA_ERR_INVALID_ARG;
  if ((causal != 0 && causal != 1) || window < 0) return PA_ERR_INVALID_ARG;
  if (dims->workspace == nullptr || dims->workspace_bytes < kWsHeader) return PA_ERR_WORKSPACE;
  DecodeParams p{};
  p.block_table = block_table;
  p.context_lens = context_lens;
  p.num_seqs = dims->num_seqs;
  p.num_q_heads = dims->num_q_heads;
  p.num_kv_heads = dims->num_kv_heads;
  p.block_size = dims->block_size;
  p.max_blocks_per_seq = dims->max_blocks_per_seq;
  p.num_blocks = dims->num_blocks;
  p.n_query = n_query;
  p.causal = causal;
  p.window = window;
  p.flags = static_cast<unsigned*>(dims->workspace);
  if (launch_trace(p, trace, static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
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
