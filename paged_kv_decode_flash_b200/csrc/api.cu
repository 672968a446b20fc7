// api.cu -- the C ABI of libpagedattn (declared in include/pagedattn.h):
// argument checks, the split planner and the launches.  Host code only.
//
// Split planner ("Dual MI50, part 2", section "Decode: a new kernel for the
// shape MTP actually runs": the work is split along the context so that all
// compute units stay busy at batch 1).  The number of splits depends only on
// host integers (shapes and the SM count), never on context_lens, which stay
// on the device: the call needs no host synchronisation and can be captured
// in a CUDA graph.  Each split owns a contiguous run of logical blocks; a
// CTA (split, KV head, sequence) intersects its run with the sequence's
// visible key range on the device and exits early when that is empty.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "pagedattn.h"

namespace {

using namespace pa;

constexpr int kCtasPerSm = 2;           // resident decode CTAs per SM the plan aims for
constexpr int kMaxTargetCtas = 4096;    // device-independent bound used to size workspaces
constexpr int kMinKeysPerSplit = 128;   // a split below this is all overhead

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_dims(const pa_dims* d, int n_query) {
  if (d == nullptr) return PA_ERR_INVALID_ARG;
  if (d->num_seqs < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->head_dim < 1 ||
      d->block_size < 1 || d->max_blocks_per_seq < 1 || d->num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (n_query < 1 || n_query > kMaxQuery) return PA_ERR_INVALID_ARG;
  if (d->block_size % kChunk != 0) return PA_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if ((long long)n_query * (d->num_q_heads / d->num_kv_heads) > kMaxRows) return PA_ERR_UNSUPPORTED;
  if ((long long)d->max_blocks_per_seq * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if ((long long)d->num_blocks * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

// splits = target CTAs / (sequences x KV heads), at least 128 keys per
// split.  `fill` rounds up (the CUDA-core kernel, several CTAs per SM) or
// down (the tensor-core kernel, one CTA per SM: a second wave would double
// the time).
int plan_splits(const pa_dims* d, long long target_ctas, bool round_up, int* blocks_per_split) {
  const long long min_blocks = ceil_div(kMinKeysPerSplit, d->block_size);
  const long long max_splits = std::max(1LL, ceil_div(d->max_blocks_per_seq, min_blocks));
  const long long per_split = (long long)d->num_seqs * d->num_kv_heads;
  long long splits = round_up ? ceil_div(target_ctas, per_split) : target_ctas / per_split;
  splits = std::max(1LL, std::min(splits, max_splits));
  const long long bps = ceil_div(d->max_blocks_per_seq, splits);
  *blocks_per_split = (int)bps;
  return (int)ceil_div(d->max_blocks_per_seq, bps);
}

// Which kernel a call uses, and its split plan.
struct Plan {
  bool tensor_cores;
  int splits, blocks_per_split;
};

Plan make_plan(const pa_dims* d, int n_query, int kv_dtype, int sms) {
  Plan pl{};
  const int rows = n_query * (d->num_q_heads / d->num_kv_heads);
  pl.tensor_cores = decode_tc_supported(kv_dtype, rows, d->num_blocks, d->num_kv_heads,
                                        d->block_size);
  pl.splits = pl.tensor_cores ? plan_splits(d, sms, false, &pl.blocks_per_split)
                              : plan_splits(d, (long long)sms * kCtasPerSm, true,
                                            &pl.blocks_per_split);
  return pl;
}

struct WsLayout {
  size_t part_out, part_lse, total;
};

WsLayout ws_layout(const pa_dims* d, int n_query, int splits) {
  const size_t rows = (size_t)d->num_seqs * splits * n_query * d->num_q_heads;
  WsLayout w;
  w.part_out = kWsHeader;
  w.part_lse = w.part_out + align256(rows * d->head_dim * sizeof(float));
  w.total = w.part_lse + align256(rows * sizeof(float));
  return w;
}

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" {

size_t paged_attn_workspace_size(const pa_dims* dims, int32_t n_query) {
  if (check_dims(dims, n_query) != PA_OK) return 0;
  int bps = 0;
  const int splits = plan_splits(dims, kMaxTargetCtas, true, &bps);
  return ws_layout(dims, n_query, splits).total;
}

int32_t paged_attn_num_splits(const pa_dims* dims, int32_t n_query, int32_t kv_dtype) {
  const int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  return make_plan(dims, n_query, kv_dtype, sms).splits;
}

int paged_attn_workspace_init(const pa_dims* dims, void* stream) {
  if (dims == nullptr || dims->workspace == nullptr || dims->workspace_bytes < kWsHeader)
    return PA_ERR_WORKSPACE;
  if (cudaMemsetAsync(dims->workspace, 0, kWsHeader, (cudaStream_t)stream) != cudaSuccess)
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
  if (!q || !k_cache || !v_cache || !block_table || !context_lens || !out)
    return PA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(out, 16) ||
      !aligned(block_table, 4) || !aligned(context_lens, 4))
    return PA_ERR_INVALID_ARG;
  if ((causal != 0 && causal != 1) || window < 0) return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (dims->workspace == nullptr || !aligned(dims->workspace, 256)) return PA_ERR_WORKSPACE;

  const int sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const Plan plan = make_plan(dims, n_query, kv_dtype, sms);
  const int splits = plan.splits, bps = plan.blocks_per_split;
  const WsLayout w = ws_layout(dims, n_query, splits);
  if (dims->workspace_bytes < w.total) return PA_ERR_WORKSPACE;

  char* ws = static_cast<char*>(dims->workspace);
  DecodeParams p{};
  p.q = static_cast<const __half*>(q);
  p.k = k_cache;
  p.v = v_cache;
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
  p.kv_dtype = kv_dtype;
  p.group = dims->num_q_heads / dims->num_kv_heads;
  p.rows = n_query * p.group;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_splits = splits;
  p.blocks_per_split = bps;
  p.part_out = reinterpret_cast<float*>(ws + w.part_out);
  p.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  p.flags = reinterpret_cast<unsigned*>(ws);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = plan.tensor_cores ? launch_decode_tc(p, st) : launch_decode_simt(p, st);
  if (e != cudaSuccess) return PA_ERR_CUDA;

  MergeParams m{};
  m.part_out = p.part_out;
  m.part_lse = p.part_lse;
  m.num_seqs = dims->num_seqs;
  m.num_splits = splits;
  m.rows_per_seq = n_query * dims->num_q_heads;
  m.head_dim = kHeadDim;
  m.out = static_cast<__half*>(out);
  m.out_lse = nullptr;
  if (launch_merge(m, st) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
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
