// split_common.cuh -- definitions of the per-head split decode kernel
// (decode_split.cu), in their own namespace.
//
// Paged decode attention: "Dual MI50, part 2: from 10 to 74 tokens/s, a
// 200k-token context, and two attention kernels" (sbm-labs blog), sections
// "Bug 2: the drafter read freed memory" (block table, sliding-window mask,
// non-causal drafter) and "Decode: a new kernel for the shape MTP actually
// runs" (multi-token verify, grouped-query heads, split along the context,
// merged partials).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

namespace pa {
namespace split {

constexpr int kHeadDim = 128;          // the only head_dim the decode kernels take
constexpr int kMaxRows = 64;           // n_query * (Hq / Hkv) rows per KV head
constexpr int kMaxQuery = 8;
constexpr size_t kWsHeader = 256;      // status header at the start of the workspace
constexpr int kChunk = 16;             // keys per gather unit (block_size % 16 == 0)

// Device-side data-error flags (bits of the first uint32 of the workspace).
enum : unsigned { kFlagBadBlock = 1u, kFlagBadLen = 2u, kFlagTimeout = 4u };

enum KvDtype : int { kKvFp16 = 0, kKvQ8_0 = 1 };

// Everything a decode launch needs, passed by value.
struct DecodeParams {
  const __half* q;            // [B][nq][Hq][D]
  const void* k;              // cache, see pagedattn.h
  const void* v;
  const int32_t* block_table; // [B][mbps]
  const int32_t* context_lens;// [B]
  int num_seqs, num_q_heads, num_kv_heads, block_size, max_blocks_per_seq;
  int num_blocks, n_query, causal, window, kv_dtype, group, rows;
  float scale_log2;           // scale * log2(e): scores live in the log2 domain
  int num_splits;             // key splits per (seq, kv head) (CUDA-core kernel;
                              // tensor-core kernel: ceil(num_ctas / groups))
  int num_ctas;               // tensor-core kernel: CTAs of the (1-D) grid
  int tiles_per_item;         // tensor-core kernel: 0 = the CTAs are shared
                              // evenly among the (sequence, KV head) groups
                              // (one wave); T > 0 = each group's 128-key tiles
                              // are cut into items of T tiles, CTA c taking
                              // item c % num_splits of group c / num_splits
  int blocks_per_split;       // logical blocks per split
  float* part_out;            // [B][S][nq*Hq][D]
  float* part_lse;            // [B][S][nq*Hq], natural log
  unsigned* flags;            // workspace status word
  int* arrivals;              // [B][Hkv][2] per (sequence, KV head): CTAs that
                              // finished their split / finished merging in
                              // this call; zero between calls
  __half* out;                // [B][nq][Hq][D], written by the fused merge
  int coop;                   // every CTA of the grid is resident at once
                              // (cooperative launch): groups merge together
  int32_t* trace;             // null, or [B][nq][Hq][5] key-resolution record
  unsigned long long wait_limit_ns;  // bound of every pipeline and group wait
};

struct MergeParams {
  const float* part_out;      // [B][S][rps][D]
  const float* part_lse;      // [B][S][rps]
  int num_seqs, num_splits, rows_per_seq, head_dim;
  __half* out;                // [B][rps][D]
  float* out_lse;             // [B][rps] or null
};

// Visible keys of query token i: the inclusive range [lo, hi]; empty when
// lo > hi.  The n_query new tokens are the last positions of the context.
__host__ __device__ __forceinline__ void key_range(int L, int nq, int i, int causal,
                                                   int window, int& lo, int& hi) {
  const int p = L - nq + i;          // position of query token i
  hi = causal ? p : L - 1;           // the window anchor, too
  lo = window > 0 ? (hi - window + 1 > 0 ? hi - window + 1 : 0) : 0;
}

// Union of the visible ranges of all n_query tokens of a sequence.
__host__ __device__ __forceinline__ void union_range(int L, int nq, int causal, int window,
                                                     int& lo, int& hi) {
  int lo0, hi0, lo1, hi1;
  key_range(L, nq, 0, causal, window, lo0, hi0);
  key_range(L, nq, nq - 1, causal, window, lo1, hi1);
  lo = lo0 < lo1 ? lo0 : lo1;
  hi = hi0 > hi1 ? hi0 : hi1;
}

__host__ __device__ __forceinline__ bool context_len_ok(int L, int nq, int mbps, int bs) {
  return L >= nq && (long long)L <= (long long)mbps * bs;
}

__host__ __device__ __forceinline__ long long q8_0_tile_bytes(int bs, int d) {
  return (long long)bs * d + (long long)bs * (d / 32) * 2;
}

}  // namespace split
}  // namespace pa
