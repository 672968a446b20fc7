// cache_write.cu -- write the new tokens' keys and values into the paged KV
// cache: scatter through the block table, quantising on the way for the
// int8 caches.  This is the step before decode attention in a decode or
// verify step ("Dual MI50, part 2: from 10 to 74 tokens/s, a 200k-token
// context, and two attention kernels", section "Bug 2: the drafter read
// freed memory": vLLM's cache manager hands out the blocks a sequence's
// tokens live in; section "200k context for coding agents": an int8 cache
// makes the long context fit).
//
// Quantisation rules, all arithmetic in fp32 with IEEE rounding (the inputs
// are fp16, so amax and every x are exact in fp32):
//   q8_0, per group of 32 head_dim elements:
//     d = fp16_rn(amax / 127);  q = d > 0 ? clamp(roundf(x / d), -127, 127) : 0
//   int8 with row scales, per (token, KV head) row of 128 elements:
//     s = amax / 127 (fp32);     q = s > 0 ? clamp(roundf(x / s), -127, 127) : 0
// roundf rounds halves away from zero.
//
// One warp per (sequence, new token, KV head): lane l holds head_dim
// elements 4l .. 4l+3 of the key row and of the value row.
#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

// Quantise four fp32 values with the scale `d` (as fp32): packed int8.
__device__ __forceinline__ uint32_t quant4(const float (&x)[4], float d) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float r = d > 0.f ? roundf(__fdiv_rn(x[e], d)) : 0.f;
    r = fminf(fmaxf(r, -127.f), 127.f);
    w |= ((uint32_t)(int)r & 0xffu) << (8 * e);
  }
  return w;
}

__device__ __forceinline__ void load4(const __half* src, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(src);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
}

// One row (key or value) of 128 elements into its cache slot.
__device__ __forceinline__ void write_row(const CacheWriteParams& p, const __half* src, void* cache,
                                          long long phys, int kvh, int slot, int lane) {
  if (p.kv_dtype == kKvFp16) {
    const long long row = (phys * p.num_kv_heads + kvh) * p.block_size + slot;
    *reinterpret_cast<uint2*>(static_cast<__half*>(cache) + row * kHeadDim + lane * 4) =
        *reinterpret_cast<const uint2*>(src + lane * 4);
    return;
  }
  float x[4];
  load4(src + lane * 4, x);
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  uint8_t* tile = static_cast<uint8_t*>(cache) +
                  (phys * p.num_kv_heads + kvh) * quant_tile_bytes(p.kv_dtype, p.block_size);
  uint8_t* scales = tile + (long long)p.block_size * kHeadDim;
  if (p.kv_dtype == kKvQ8_0) {
    // max over the 8 lanes of this lane's group of 32 elements
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const __half dh = __float2half_rn(__fdiv_rn(amax, 127.f));
    const uint32_t w = quant4(x, __half2float(dh));
    *reinterpret_cast<uint32_t*>(tile + (long long)slot * kHeadDim + lane * 4) = w;
    if (lane % 8 == 0)
      *reinterpret_cast<__half*>(scales + (long long)slot * 8 + (lane / 8) * 2) = dh;
  } else {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = __fdiv_rn(amax, 127.f);
    const uint32_t w = quant4(x, s);
    *reinterpret_cast<uint32_t*>(tile + (long long)slot * kHeadDim + lane * 4) = w;
    if (lane == 0) *reinterpret_cast<float*>(scales + (long long)slot * 4) = s;
  }
}

__global__ void __launch_bounds__(128) cache_write_kernel(const CacheWriteParams p) {
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  const long long rows = (long long)p.num_seqs * p.n_new * p.num_kv_heads;
  if (row >= rows) return;  // uniform per warp
  const int kvh = (int)(row % p.num_kv_heads);
  const int i = (int)((row / p.num_kv_heads) % p.n_new);
  const int s = (int)(row / ((long long)p.num_kv_heads * p.n_new));
  const int L = p.context_lens[s];
  if (!context_len_ok(L, p.n_new, p.max_blocks_per_seq, p.block_size)) {
    if (lane == 0 && i == 0 && kvh == 0) atomicOr(p.flags, kFlagBadLen);
    return;
  }
  const int pos = L - p.n_new + i;
  const long long phys = p.block_table[(long long)s * p.max_blocks_per_seq + pos / p.block_size];
  if (phys < 0 || phys >= p.num_blocks) {
    if (lane == 0) atomicOr(p.flags, kFlagBadBlock);
    return;
  }
  const long long src = row * kHeadDim;
  write_row(p, p.k_new + src, p.k_cache, phys, kvh, pos % p.block_size, lane);
  write_row(p, p.v_new + src, p.v_cache, phys, kvh, pos % p.block_size, lane);
}

}  // namespace

cudaError_t launch_cache_write(const CacheWriteParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.num_seqs * p.n_new * p.num_kv_heads;
  if (rows == 0) return cudaSuccess;
  cache_write_kernel<<<(unsigned)((rows * 32 + 127) / 128), 128, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
