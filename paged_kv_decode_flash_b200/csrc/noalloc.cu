// noalloc.cu -- paged_attn_decode_noalloc: the decode entry point for
// callers that cannot hand the library any device memory of its own.
//
// Who needs it: code that runs inside a host program which owns every byte
// of device memory (a serving engine that carves one fixed pool at start-up
// and hands out no scratch buffers, or a plug-in whose host exposes no
// allocator), and code that must not call cudaMalloc on its hot path because
// that call can implicitly synchronise the device and stall other work.
// Such callers still pass their inputs and output; the split partials and
// the status word that paged_attn_decode keeps in a caller-provided
// workspace live here in one fixed array in the library's own device image.
//
// Limits and sharing:
//   * The array holds kNoAllocScratchBytes (16 MiB); every GPU that loads the
//     library keeps it until the process exits.  Shapes whose split partials
//     need more are rejected with PA_ERR_WORKSPACE before anything is
//     enqueued.
//   * All calls on a device share the one array, which keeps the previous
//     call's contents.  Calls whose work overlaps on the GPU (on different
//     streams without ordering between them) race on it and corrupt each
//     other's results; order them on one stream or with events.
//   * The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture is in progress.
//   * The status word is cleared at the start of every call, so device-side
//     data errors (block index or context length out of range) are handled
//     exactly as in paged_attn_decode (masked keys, zeroed rows) but cannot be
//     read back: this variant has no paged_attn_get_error counterpart.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "common.cuh"
#include "kernels.h"
#include "pagedattn.h"

namespace {

using namespace pa;

constexpr size_t kNoAllocScratchBytes = PA_NOALLOC_SCRATCH_BYTES;
constexpr int kNoAllocCtasPerSm = 2;
constexpr int kNoAllocMinKeysPerSplit = 128;

// The scratch itself.  In host code this name is only a stand-in for the
// device object: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }
size_t round256(size_t x) { return (x + 255) & ~size_t(255); }
bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Once per device, with that device current: the scratch array's device
// address and the SM count.
int setup_device(void** scratch, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return PA_ERR_CUDA;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      return PA_ERR_CUDA;
    g_sm_count[dev] = n;
    g_scratch_addr[dev] = p;
  }
  *scratch = g_scratch_addr[dev];
  *sms = g_sm_count[dev];
  return PA_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(const pa_dims* dims, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_table,
                                         const int32_t* context_lens, int32_t n_query,
                                         int32_t causal, int32_t window, float scale,
                                         int32_t kv_dtype, void* out, void* stream) {
  // Shape and argument checks: the same rules as paged_attn_decode.
  if (dims == nullptr) return PA_ERR_INVALID_ARG;
  const pa_dims& d = *dims;
  if (d.num_seqs < 1 || d.num_q_heads < 1 || d.num_kv_heads < 1 || d.head_dim < 1 ||
      d.block_size < 1 || d.max_blocks_per_seq < 1 || d.num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (d.num_q_heads % d.num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (n_query < 1 || n_query > kMaxQuery || d.block_size % kChunk != 0) return PA_ERR_INVALID_ARG;
  if (d.head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  const int group = d.num_q_heads / d.num_kv_heads;
  if ((long long)n_query * group > kMaxRows) return PA_ERR_UNSUPPORTED;
  if ((long long)d.max_blocks_per_seq * d.block_size > INT32_MAX ||
      (long long)d.num_blocks * d.block_size > INT32_MAX)
    return PA_ERR_UNSUPPORTED;
  if (!q || !k_cache || !v_cache || !block_table || !context_lens || !out) return PA_ERR_INVALID_ARG;
  if (!is_aligned(q, 16) || !is_aligned(k_cache, 16) || !is_aligned(v_cache, 16) ||
      !is_aligned(out, 16) || !is_aligned(block_table, 4) || !is_aligned(context_lens, 4))
    return PA_ERR_INVALID_ARG;
  if ((causal != 0 && causal != 1) || window < 0) return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;

  void* scratch = nullptr;
  int sms = 0;
  const int rc = setup_device(&scratch, &sms);
  if (rc != PA_OK) return rc;

  // The split plan of paged_attn_decode, sized for the scratch array.
  const long long min_blocks = cdiv(kNoAllocMinKeysPerSplit, d.block_size);
  const long long max_splits = std::max(1LL, cdiv(d.max_blocks_per_seq, min_blocks));
  long long splits = std::max(1LL, cdiv((long long)sms * kNoAllocCtasPerSm,
                                        (long long)d.num_seqs * d.num_kv_heads));
  splits = std::min(splits, max_splits);
  const long long bps = cdiv(d.max_blocks_per_seq, splits);
  splits = cdiv(d.max_blocks_per_seq, bps);

  const size_t rows = (size_t)d.num_seqs * splits * n_query * d.num_q_heads;
  const size_t off_out = kWsHeader;
  const size_t off_lse = off_out + round256(rows * kHeadDim * sizeof(float));
  const size_t need = off_lse + round256(rows * sizeof(float));
  if (need > kNoAllocScratchBytes) return PA_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(scratch);
  // The status word must start at zero; the partials are fully overwritten.
  if (cudaMemsetAsync(ws, 0, kWsHeader, st) != cudaSuccess) return PA_ERR_CUDA;

  DecodeParams p{};
  p.q = static_cast<const __half*>(q);
  p.k = k_cache;
  p.v = v_cache;
  p.block_table = block_table;
  p.context_lens = context_lens;
  p.num_seqs = d.num_seqs;
  p.num_q_heads = d.num_q_heads;
  p.num_kv_heads = d.num_kv_heads;
  p.block_size = d.block_size;
  p.max_blocks_per_seq = d.max_blocks_per_seq;
  p.num_blocks = d.num_blocks;
  p.n_query = n_query;
  p.causal = causal;
  p.window = window;
  p.kv_dtype = kv_dtype;
  p.group = group;
  p.rows = n_query * group;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_splits = (int)splits;
  p.blocks_per_split = (int)bps;
  p.part_out = reinterpret_cast<float*>(ws + off_out);
  p.part_lse = reinterpret_cast<float*>(ws + off_lse);
  p.flags = reinterpret_cast<unsigned*>(ws);
  if (launch_decode_simt(p, st) != cudaSuccess) return PA_ERR_CUDA;

  MergeParams m{};
  m.part_out = p.part_out;
  m.part_lse = p.part_lse;
  m.num_seqs = d.num_seqs;
  m.num_splits = (int)splits;
  m.rows_per_seq = n_query * d.num_q_heads;
  m.head_dim = kHeadDim;
  m.out = static_cast<__half*>(out);
  m.out_lse = nullptr;
  if (launch_merge(m, st) != cudaSuccess) return PA_ERR_CUDA;
  return PA_OK;
}
