// common.cuh -- definitions shared by the libpagedattn kernels and host code.
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

constexpr int kHeadDim = 128;          // the only head_dim the decode kernels take
constexpr int kMaxRows = 1024;         // n_query * (Hq / Hkv) rows per KV head
constexpr int kMaxQuery = 128;        // new tokens per call (chunked verify / prefill)
constexpr size_t kWsHeader = 256;      // status header at the start of the workspace
constexpr int kChunk = 16;             // keys per gather unit (block_size % 16 == 0)
constexpr int kTileKeys = 128;         // keys per pipeline tile
constexpr int kChunksPerTile = kTileKeys / kChunk;
// A batch is handled by one work-queue launch per kMaxQueueSeqs sequences.
constexpr int kMaxQueueSeqs = 256;
// Default time after which a device-side wait gives up.
constexpr unsigned long long kDefaultWaitLimitNs = 1000000000ull;  // 1 s

// Device-side data-error flags (bits of the first uint32 of the workspace).
enum : unsigned { kFlagBadBlock = 1u, kFlagBadLen = 2u, kFlagTimeout = 4u };

enum KvDtype : int { kKvFp16 = 0, kKvQ8_0 = 1, kKvInt8Row = 2 };

// Bytes of one (block, KV head) tile of a quantised cache: int8 values
// [bs][128], then q8_0: fp16 scales [bs][4]; int8 with row scales: fp32
// scales [bs].
__host__ __device__ __forceinline__ long long quant_tile_bytes(int kv_dtype, int bs) {
  return (long long)bs * kHeadDim + (long long)bs * (kv_dtype == kKvQ8_0 ? 8 : 4);
}
// Bytes of the scales of one key (row) in such a tile.
__host__ __device__ __forceinline__ int quant_scale_bytes(int kv_dtype) {
  return kv_dtype == kKvQ8_0 ? 8 : 4;
}

// Everything a decode launch needs, passed by value.
//
// Work decomposition (tensor-core kernel).  The rows that share one KV head
// (n_query tokens x the query heads of the group) are cut into `halves`
// equal parts of at most rows_half rows; a (sequence, KV head, part) is a
// *group*.  Its visible keys, from the union of its tokens' ranges rounded
// down to a 16-key chunk, are numbered in 16-key chunks.  A CTA streams
// *segments* (a run of chunks of one group) through one pipeline and writes
// one fp32 partial (O, lse) per segment into a partial slot:
//   mode 0 (few groups, batch 1 typically): the sequences share the grid
//     evenly; within a sequence, each of its `halves` CTA sets cuts the
//     chunks of all KV heads, laid end to end, into ctas_per_set equal
//     ranges (a range may run into the next KV head: two segments).  The
//     CTAs are resident together (cooperative launch) and the CTAs whose
//     range ends in a KV head merge that head's partials;
//   mode 1 (a batch): every group's chunks are cut into items of
//     item_tiles tiles (the last item into up to four smaller ones), and the
//     CTAs take items from a queue, the big items first; the CTA whose
//     partial completes a group merges that group at the end.
// The cut depends only on the shapes and the sequence's own length, so a
// sequence's output does not depend on its batch neighbours, and, as each
// segment's partial is merged in a fixed order whoever computed it, results
// are bit-reproducible.
struct DecodeParams {
  const __half* q;            // [B][nq][Hq][D]
  const void* k;              // cache, see pagedattn.h
  const void* v;
  const int32_t* block_table; // [B][mbps]
  const int32_t* context_lens;// [B]
  int num_seqs, num_q_heads, num_kv_heads, block_size, max_blocks_per_seq;
  int num_blocks, n_query, causal, window, kv_dtype, group, rows;
  float scale_log2;           // scale * log2(e): scores live in the log2 domain
  int halves, rows_half;      // row parts per KV head, rows per part
  int mode;                   // 0: static partition, 1: work queue
  int num_ctas;               // CTAs of the (1-D) grid
  int ctas_per_set;           // mode 0: CTAs per (sequence, part)
  int item_tiles;             // mode 1: tiles per big item
  int slots_per_group;        // mode 1: partial slots per group
  unsigned long long wait_limit_ns;  // pipeline waits give up after this long
  float* part_out;            // [slots][rows_half][D]
  float* part_lse;            // [slots][rows_half], natural log
  unsigned* flags;            // workspace status word
  int* arrivals;              // [B][Hkv][halves][2] per group; zero between calls
  int* queue;                 // mode 1: item counter of this launch; zero between calls
  __half* out;                // [B][nq][Hq][D]
  // Partial mode (context-parallel decode): the keys of sequence s are
  // limited to [key_begin[s], key_begin[s] + key_count[s]) (whole blocks;
  // block_table row s maps local block b to key_begin[s] / block_size + b),
  // and the merged result is written as fp32 out_f32 [B][nq][Hq][D] and
  // out_lse [B][nq][Hq] (natural log) instead of fp16 out.
  const int32_t* key_begin;   // null: every key of the context
  const int32_t* key_count;
  float* out_f32;
  float* out_lse;
  int32_t* trace;             // null, or [B][nq][Hq][5] key-resolution record
  int coop;                   // every CTA of the grid is resident at once
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

// The query tokens that see key j form one contiguous run [i_lo, i_hi]
// (empty when i_lo > i_hi): causal keeps tokens whose position is >= j, a
// window keeps tokens whose anchor is < j + W.
__host__ __device__ __forceinline__ void tokens_seeing(int L, int nq, int causal, int window,
                                                       int j, int& i_lo, int& i_hi) {
  const int p0 = L - nq;             // position of token 0
  i_lo = 0;
  i_hi = nq - 1;
  if (j < 0 || j >= L) {
    i_lo = 1;
    i_hi = 0;
    return;
  }
  if (causal) {
    if (j - p0 > i_lo) i_lo = j - p0;
    if (window > 0 && j + window - 1 - p0 < i_hi) i_hi = j + window - 1 - p0;
  } else if (window > 0 && j < L - window) {
    i_lo = 1;
    i_hi = 0;
  }
}

__host__ __device__ __forceinline__ bool context_len_ok(int L, int nq, int mbps, int bs) {
  return L >= nq && (long long)L <= (long long)mbps * bs;
}

}  // namespace pa
