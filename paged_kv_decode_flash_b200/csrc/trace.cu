// trace.cu -- per-row key-resolution record, for bit-exact checks of the
// masking and block-table code the decode kernels use (key_range,
// context_len_ok and the block lookup below are the same functions and the
// same arithmetic).  One thread walks one row's visible keys; tests only.
#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

__global__ void trace_kernel(const DecodeParams p, int32_t* trace) {
  const long long rows = (long long)p.num_seqs * p.n_query * p.num_q_heads;
  const long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (id >= rows) return;
  const int i = (int)((id / p.num_q_heads) % p.n_query);
  const int s = (int)(id / ((long long)p.num_q_heads * p.n_query));
  int32_t* t = trace + id * 5;
  const int L = p.context_lens[s];
  if (!context_len_ok(L, p.n_query, p.max_blocks_per_seq, p.block_size)) {
    atomicOr(p.flags, kFlagBadLen);
    t[0] = 0; t[1] = -1; t[2] = -1; t[3] = 0; t[4] = 0;
    return;
  }
  int lo, hi;
  key_range(L, p.n_query, i, p.causal, p.window, lo, hi);
  const int* table = p.block_table + (long long)s * p.max_blocks_per_seq;
  int count = 0, jmin = -1, jmax = -1;
  unsigned x = 0, sum = 0;
  for (int j = lo; j <= hi; ++j) {
    const long long phys = table[j / p.block_size];
    if (phys < 0 || phys >= p.num_blocks) {  // masked, flagged: as in decode
      atomicOr(p.flags, kFlagBadBlock);
      continue;
    }
    const unsigned id_phys = (unsigned)(phys * p.block_size + j % p.block_size);
    if (count == 0) jmin = j;
    jmax = j;
    ++count;
    x ^= id_phys;
    sum += id_phys;
  }
  t[0] = count; t[1] = jmin; t[2] = jmax; t[3] = (int32_t)x; t[4] = (int32_t)sum;
}

}  // namespace

cudaError_t launch_trace(const DecodeParams& p, int32_t* trace, cudaStream_t stream) {
  const long long rows = (long long)p.num_seqs * p.n_query * p.num_q_heads;
  if (rows == 0) return cudaSuccess;
  trace_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, stream>>>(p, trace);
  return cudaGetLastError();
}

}  // namespace pa
