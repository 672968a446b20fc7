// noalloc.cu -- paged_attn_decode_noalloc: the decode entry point for
// callers that cannot hand the library any device memory of its own.
//
// Who needs it: code that runs inside a host program which owns every byte
// of device memory (a serving engine that carves one fixed pool at start-up
// and hands out no scratch buffers, or a plug-in whose host exposes no
// allocator), and code that must not call cudaMalloc on its hot path because
// that call can implicitly synchronise the device and stall other work.
// Such callers still pass their inputs and output; the split partials, the
// counters and the status word that paged_attn_decode keeps in a
// caller-provided workspace live here in one fixed array in the library's
// own device image.
//
// Limits and sharing:
//   * The array holds kNoAllocScratchBytes (16 MiB); every GPU that loads the
//     library keeps it until the process exits.  Shapes whose workspace
//     needs more are rejected with PA_ERR_WORKSPACE before anything is
//     enqueued.
//   * All calls on a device share the one array, which keeps the previous
//     call's contents.  Calls whose work overlaps on the GPU (on different
//     streams without ordering between them) race on it and corrupt each
//     other's results; order them on one stream or with events.
//   * The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; the
//     look-up is serialised by a mutex, so first calls from several host
//     threads are safe.  Make that first call before any stream capture is
//     in progress.
//   * The status word and the counters are cleared at the start of every
//     call, so device-side data errors (block index or context length out of
//     range) are handled exactly as in paged_attn_decode (masked keys,
//     zeroed rows) but cannot be read back, and neither can a device-side
//     wait that timed out: such a call leaves its output undefined.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "common.cuh"
#include "dispatch.h"
#include "kernels.h"
#include "pagedattn.h"

namespace {

using namespace pa;

constexpr size_t kNoAllocScratchBytes = PA_NOALLOC_SCRATCH_BYTES;

// The scratch itself.  In host code this name is only a stand-in for the
// device object: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_addr[kMaxDevices];
std::atomic<int> g_sm_count[kMaxDevices];
std::mutex g_setup_mutex;

// Once per device, with that device current: the scratch array's device
// address and the SM count (published after both are known).
int setup_device(void** scratch, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  void* addr = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (addr == nullptr) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    addr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (addr == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return PA_ERR_CUDA;
      int n = 0;
      if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return PA_ERR_CUDA;
      g_sm_count[dev].store(n, std::memory_order_relaxed);
      g_scratch_addr[dev].store(p, std::memory_order_release);
      addr = p;
    }
  }
  *scratch = addr;
  *sms = g_sm_count[dev].load(std::memory_order_relaxed);
  return PA_OK;
}

}  // namespace

extern "C" int paged_attn_decode_noalloc(const pa_dims* dims, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_table,
                                         const int32_t* context_lens, int32_t n_query,
                                         int32_t causal, int32_t window, float scale,
                                         int32_t kv_dtype, void* out, void* stream) {
  // The same argument rules, plan and kernels as paged_attn_decode.
  int rc = check_dims(dims, n_query);
  if (rc != PA_OK) return rc;
  rc = check_decode_args(q, k_cache, v_cache, block_table, context_lens, causal, window, scale,
                         kv_dtype, out);
  if (rc != PA_OK) return rc;

  void* scratch = nullptr;
  int sms = 0;
  rc = setup_device(&scratch, &sms);
  if (rc != PA_OK) return rc;

  const Plan plan = make_plan(dims, n_query, kv_dtype, sms);
  if (ws_layout(dims, n_query, plan).total > kNoAllocScratchBytes) return PA_ERR_WORKSPACE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The status word and counters must start at zero; the partials are fully
  // overwritten by every call.
  if (cudaMemsetAsync(scratch, 0, ws_zero_prefix(dims), st) != cudaSuccess) return PA_ERR_CUDA;
  return enqueue_decode(dims, plan, q, k_cache, v_cache, block_table, context_lens, n_query,
                        causal, window, scale, kv_dtype, out, scratch, nullptr, st);
}
