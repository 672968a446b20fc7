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
// O_s is never multiplied).  One CTA per row, one thread per head_dim
// element; reads are coalesced along head_dim.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace pa {
namespace {

__global__ void merge_kernel(const MergeParams p) {
  // Launched as a programmatic dependent of the decode kernel: wait for its
  // partials (returns at once when launched normally).
  sm100::griddep_wait();
  const long long row = blockIdx.x;               // over num_seqs * rows_per_seq
  const int s = (int)(row / p.rows_per_seq);
  const int r = (int)(row % p.rows_per_seq);
  const int d = threadIdx.x;
  const long long base = (long long)s * p.num_splits * p.rows_per_seq + r;  // split 0
  const long long stride = p.rows_per_seq;

  float M = -INFINITY;
  for (int k = 0; k < p.num_splits; ++k) M = fmaxf(M, p.part_lse[base + k * stride]);

  float acc = 0.f, wsum = 0.f;
  if (M != -INFINITY) {
    for (int k = 0; k < p.num_splits; ++k) {
      const float l = p.part_lse[base + k * stride];
      if (l == -INFINITY) continue;
      const float w = expf(l - M);
      wsum += w;
      acc = fmaf(w, p.part_out[(base + k * stride) * p.head_dim + d], acc);
    }
  }
  const float o = (M == -INFINITY) ? 0.f : acc / wsum;
  p.out[row * p.head_dim + d] = __float2half_rn(o);
  if (p.out_lse != nullptr && d == 0)
    p.out_lse[row] = (M == -INFINITY) ? -INFINITY : M + logf(wsum);
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, cudaStream_t stream) {
  const long long rows = (long long)p.num_seqs * p.rows_per_seq;
  if (rows == 0) return cudaSuccess;
  // Programmatic stream serialization: the merge grid may be scheduled while
  // the preceding decode kernel still runs and starts the moment it ends.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows);
  cfg.blockDim = dim3(p.head_dim);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel, p);
}

}  // namespace pa
