// merge.cu -- log-sum-exp merge of split-KV partials.
//
// "Dual MI50, part 2" (sbm-labs blog), section "Decode: a new kernel for the
// shape MTP actually runs": the decode work is split along the context and
// the partial results are merged at the end.  Each split s of a row carries
// its normalised output O_s and the natural-log sum of its exponentiated
// scores lse_s; the exact combination is
//   M = max_s lse_s,  w_s = exp(lse_s - M),  out = sum_s w_s O_s / sum_s w_s,
//   lse = M + log(sum_s w_s),
// with splits that saw no key (lse_s = -inf) weighted by exactly zero (their
// O_s is never multiplied).
//
// One warp per output row.  The lanes first take the maximum of the split
// log-sum-exps together; then every lane owns head_dim/32 consecutive
// elements and walks the splits with one vector load per split, unrolled so
// that many loads are in flight (the merge is latency-bound: it reads data
// the decode kernel has just written).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace pa {
namespace {

constexpr int kWarpsPerCta = 4;

template <int D>
__global__ void __launch_bounds__(32 * kWarpsPerCta) merge_kernel(const MergeParams p) {
  // Launched as a programmatic dependent of the decode kernel: wait for its
  // partials (returns at once when launched normally).
  sm100::griddep_wait();
  constexpr int E = D / 32;  // elements per lane: 2, 4 or 8
  const int lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kWarpsPerCta + threadIdx.x / 32;
  if (row >= (long long)p.num_seqs * p.rows_per_seq) return;
  const int s = (int)(row / p.rows_per_seq), r = (int)(row % p.rows_per_seq);
  const long long rps = p.rows_per_seq;
  const long long b0 = (long long)s * p.num_splits * rps + r;  // split 0 of this row

  float M = -INFINITY;
  for (int k = lane; k < p.num_splits; k += 32) M = fmaxf(M, __ldcg(p.part_lse + b0 + k * rps));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
#pragma unroll 4
    for (int k = 0; k < p.num_splits; ++k) {
      const long long pk = b0 + k * rps;
      const float l = __ldcg(p.part_lse + pk);
      float o[E];
      const float* src = p.part_out + pk * D + lane * E;
      if constexpr (E == 2) {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
        o[0] = v.x; o[1] = v.y;
      } else {
#pragma unroll
        for (int q = 0; q < E / 4; ++q) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(src) + q);
          o[4 * q] = v.x; o[4 * q + 1] = v.y; o[4 * q + 2] = v.z; o[4 * q + 3] = v.w;
        }
      }
      const float w = (l == -INFINITY) ? 0.f : expf(l - M);  // empty split: weight 0
      wsum += w;
      if (w > 0.f) {
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = fmaf(w, o[e], acc[e]);
      }
    }
  }
  const float inv = (M == -INFINITY) ? 0.f : 1.f / wsum;
  __half2 h[E / 2];
#pragma unroll
  for (int e = 0; e < E; e += 2) h[e / 2] = __floats2half2_rn(acc[e] * inv, acc[e + 1] * inv);
  __half* dst = p.out + row * D + lane * E;
  if constexpr (E == 2) {
    *reinterpret_cast<__half2*>(dst) = h[0];
  } else {
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&h[2 * q]);
      u.y = *reinterpret_cast<const uint32_t*>(&h[2 * q + 1]);
      reinterpret_cast<uint2*>(dst)[q] = u;
    }
  }
  if (p.out_lse != nullptr && lane == 0)
    p.out_lse[row] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
}

template <int D>
cudaError_t launch_d(const MergeParams& p, long long rows, cudaStream_t stream) {
  // Programmatic stream serialization: the merge grid may be scheduled while
  // the preceding decode kernel still runs and starts the moment it ends.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((rows + kWarpsPerCta - 1) / kWarpsPerCta));
  cfg.blockDim = dim3(32 * kWarpsPerCta);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel<D>, p);
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.num_seqs * p.rows_per_seq;
  if (rows == 0) return cudaSuccess;
  switch (p.head_dim) {
    case 64: return launch_d<64>(p, rows, stream);
    case 128: return launch_d<128>(p, rows, stream);
    case 256: return launch_d<256>(p, rows, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pa
