// probe.cu -- paged_attn_stream_read: a read-only HBM streaming kernel that
// moves data the way the decode kernel does (untiled bulk copies of 4 KB
// pieces into a ring of 32 KB shared-memory slots, completion on mbarriers,
// one CTA per SM), with no arithmetic.  It measures the read ceiling the
// decode kernel's rate is compared with; it is not part of the attention.
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "pagedattn.h"
#include "sm100.cuh"

namespace pa {
namespace {

constexpr int kSlots = 6;                 // 6 x 32 KB in flight per SM
constexpr uint32_t kSlotBytes = 32768;
constexpr uint32_t kPiece = 4096;         // one bulk copy (a 16-key fp16 chunk)

__global__ void __launch_bounds__(32, 1) stream_read_kernel(const uint8_t* src, long long tiles,
                                                            unsigned* sink) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (sm100::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = sm100::smem_u32(smem);
  __shared__ uint64_t bars[kSlots];
  __shared__ int abort_flag;
  const int lane = threadIdx.x;
  auto bar = [&](int i) { return sm100::smem_u32(&bars[i]); };
  if (lane == 0) {
    for (int i = 0; i < kSlots; ++i) sm100::mbar_init(bar(i), 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncwarp();
  // CTA c reads tiles c, c + C, c + 2C, ... of 32 KB.
  const long long C = gridDim.x;
  const long long n = tiles > blockIdx.x ? (tiles - blockIdx.x + C - 1) / C : 0;
  unsigned acc = 0;
  long long issued = 0, consumed = 0;
  auto issue = [&](long long k) {  // lane 0: tile k of this CTA into slot k % kSlots
    const uint32_t slot = sbase + (uint32_t)(k % kSlots) * kSlotBytes;
    const uint8_t* g = src + (blockIdx.x + k * C) * (long long)kSlotBytes;
    sm100::mbar_arrive_expect_tx(bar((int)(k % kSlots)), kSlotBytes);
    for (uint32_t o = 0; o < kSlotBytes; o += kPiece)
      sm100::bulk_load(slot + o, g + o, kPiece, bar((int)(k % kSlots)));
  };
  if (lane == 0)
    for (; issued < n && issued < kSlots; ++issued) issue(issued);
  issued = __shfl_sync(0xffffffffu, issued, 0);
  bool ok = true;
  for (long long k = 0; k < n; ++k) {
    int w = 1;
    if (lane == 0) w = sm100::mbar_wait(bar((int)(k % kSlots)), (uint32_t)((k / kSlots) & 1), &abort_flag);
    ok = __shfl_sync(0xffffffffu, w, 0) != 0;
    if (!ok) break;
    consumed = k + 1;
    // touch one word per lane so that the data is used
    acc ^= *reinterpret_cast<const unsigned*>(smem + (k % kSlots) * kSlotBytes + lane * 1024);
    __syncwarp();
    if (lane == 0 && issued < n) issue(issued);
    issued = __shfl_sync(0xffffffffu, issued < n ? issued + 1 : issued, 0);
  }
  if (lane == 0) {  // drain copies still in flight (abort path only)
    volatile int no_abort = 0;
    for (long long u = consumed; u < issued; ++u)
      sm100::mbar_wait(bar((int)(u % kSlots)), (uint32_t)((u / kSlots) & 1), &no_abort);
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if (lane == 0) sink[blockIdx.x] = ok ? acc : 0xdeadbeefu;
}

}  // namespace
}  // namespace pa

extern "C" int paged_attn_stream_read(const void* src, size_t bytes, uint32_t* sink, int32_t ctas,
                                      void* stream) {
  using namespace pa;
  if (src == nullptr || sink == nullptr || ctas < 1) return PA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(src) & 15) != 0) return PA_ERR_INVALID_ARG;
  const long long tiles = (long long)(bytes / kSlotBytes);
  const size_t smem = (size_t)kSlots * kSlotBytes + 1024;
  static std::atomic<bool> configured[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
  if (!configured[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(stream_read_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return PA_ERR_CUDA;
    configured[dev].store(true, std::memory_order_release);
  }
  stream_read_kernel<<<ctas, 32, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(src), tiles, sink);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
