// decode_tc.cu -- split-KV paged decode attention on the sm_100a tensor
// cores (tcgen05 + TMEM), with TMA / bulk-copy staging of the paged KV tiles.
//
// What it computes is the decode step of "Dual MI50, part 2: from 10 to 74
// tokens/s, a 200k-token context, and two attention kernels" (sbm-labs
// blog), section "Decode: a new kernel for the shape MTP actually runs": all
// query rows that share one KV head (n_query tokens x the query heads of the
// group) are scored against the same keys, the context is split so that
// every SM is busy at batch 1, and one fp32 partial (O, lse) per split is
// merged by log-sum-exp weights.  Masks and block-table resolution follow
// section "Bug 2: the drafter read freed memory"; the int8 caches follow
// sections "200k context for coding agents" and "Prefill: teach the fork's
// fast kernel to read the int8 cache" (per-row scales, fp32 scale products).
//
// Work: a CTA streams *segments* -- runs of 16-key chunks of one group (a
// sequence, a KV head and a part of its query rows) -- through one
// pipeline, 128-key tiles at a time, and writes one partial per segment
// (DecodeParams in common.cuh describes the two ways the work is cut).
//
// Roles (one CTA per SM; 11 warps for fp16, 19 for the int8 caches):
//   warp 0      K producer: takes the CTA's segments (a static range, or
//               items from a queue), resolves the block table one tile
//               ahead, bounds-checks every block, publishes each tile's
//               description and copies its 16-key chunks into the K ring
//               (fp16: 4-D TMA boxes in the 128-byte-swizzled operand
//               layout; int8: untiled bulk copies of the raw chunk into the
//               upper half of a slot); it also stages each segment's Q rows.
//   warp 1      MMA issuer (one thread): QK(0), QK(1), then PV(t), QK(t+2):
//               S^T = K Q^T (M = 128 keys, N = query rows) double-buffered
//               in TMEM, O^T += V^T [P_hi | P_lo]^T (M = 128 head_dim lanes)
//               into one of two O accumulators (a segment's O stays put
//               while the next segment's accumulates).
//   warps 2..   softmax warpgroups (rows split between two): thread = key
//               for S; lazy per-row reference maximum in the log2 domain;
//               O rescaled in TMEM when it rises; P split into an fp16 high
//               part and residual; at a segment's last tile the partial
//               (O / l, lse) is written.
//   next warp   V producer: follows the published tiles.
//   last 8      (int8 caches) converters, four for K and four for V.
//
// Exactness: Q, K and V reach the tensor core as exact fp16 values.  Softmax
// weights are scaled by 2^14 and split into two fp16 parts (error ~2^-22).
// Both int8 caches: K's operand is qs itself (q8_0: S^T gets one accumulator
// per 32-element scale group and the softmax adds the groups times K's fp16
// scales in fp32; int8 rows: the score is multiplied by K's fp32 row scale).
// V's operand is the pair V_hi = fp16(qs * d), V_lo = fp16(qs * d - V_hi),
// multiplied as V_hi [P_hi | P_lo] + V_lo P_hi: exact for q8_0 (qs * d has
// at most 19 significant bits), within 2^-22 for an fp32 row scale.  Keys
// that no row of a part can see are never multiplied: wholly invisible
// chunks are not loaded, their scores are selected to -inf and their V rows
// are written as zeros before PV (NaN-poisoned memory cannot leak).
//
// Every wait is bounded (DecodeParams::wait_limit_ns): on a timeout the
// kernel raises kFlagTimeout, stops issuing work, drains its own copies and
// MMAs with a fixed one-second bound, frees TMEM, and keeps the workspace
// counters consistent for the next call (every segment it owns is counted
// in, with an invalid partial).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstring>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace pa {
namespace {

using namespace sm100;

constexpr int kMaxStages = 3;
// A K or V tile of 128 keys in shared memory: [key group of 8][half][8 keys]
// [64 fp16] with the 128-byte swizzle (1 KB atoms; the two 64-column halves
// of a key group 1 KB apart, key groups 2 KB apart).  One 16-key chunk is a
// single TMA box of 4 KB.
constexpr uint32_t kAtomBytes = 1024;
constexpr uint32_t kGroupBytes = 2 * kAtomBytes;
constexpr uint32_t kKVBytes = kTileKeys / 8 * kGroupBytes;  // 32 KB
constexpr uint32_t kChunkBytes = kChunk * 256;
constexpr uint32_t kRawOff = kKVBytes / 2;       // in-place K slots: raw int8 in the upper half
constexpr uint32_t kQsChunk = kChunk * kHeadDim; // 2 KB of int8 per 16-key chunk
constexpr uint32_t kRawScales = kQsChunk * kChunksPerTile;  // raw V slot: scales after the qs
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kBarSetup = 1;   // named barrier: set-up done
constexpr uint32_t kBarGroup0 = 2;  // named barriers 2, 3: softmax warpgroups
constexpr uint32_t kBarConv0 = 4;   // named barriers 4, 5: K / V converters
// A row's reference maximum is raised only when a score passes it by more
// than kLazy (log2 units); weights scaled by 2^kPShift then stay below
// 2^(kPShift + kLazy), inside the fp16 range.
constexpr float kLazy = 1.5f;
constexpr int kPShift = 14;
constexpr int kInfoSlots = 8;
constexpr int kSegSlots = 8;
constexpr int kMergeListLen = 64;
constexpr unsigned kInvalidLse = 0x7fc00000u;  // NaN: a partial that must not be used

enum : int {
  BAR_KFULL = 0,     // [3] K chunks landed (int8: raw)
  BAR_KEMPTY = 3,    // [3] K slot read by QK^T
  BAR_VFULL = 6,     // [3] V chunks landed (int8: in a raw slot)
  BAR_VEMPTY = 9,    // [3] V slot free again
  BAR_CKFULL = 12,   // [3] int8: K slot converted
  BAR_CVFULL = 15,   // [3] int8: a converted half-tile of V (hi | lo) ready
  BAR_CVEMPTY = 18,  // [3] int8: a converted half-tile read by PV
  BAR_SFULL = 21,    // [2] S^T in TMEM
  BAR_SEMPTY = 23,   // [2] S^T read by the softmax
  BAR_PFULL = 25,    // [2] P of a tile in shared memory
  BAR_OFULL = 27,    // PV of one more tile accumulated
  BAR_OEMPTY = 28,   // [2] a segment's O accumulator read out
  BAR_QFULL = 30,    // [2] a segment's Q staged
  BAR_QEMPTY = 32,   // [2] Q buffer free
  BAR_DONE = 34,     // every MMA finished
  BAR_INFO = 35,     // [8] a tile's description published
  BAR_COUNT = 43
};
constexpr int kBarSlots = 44;
// int8: converted V lives in a ring of three half-tile slots (64 keys: the hi
// tile, then the lo tile), so that the converters run ahead of PV.
constexpr int kVCSlots = 3;
constexpr uint32_t kVCSlot = kKVBytes;           // 64 keys x (hi + lo)
constexpr uint32_t kVCLo = kKVBytes / 2;         // offset of the lo half-tile

// A tile as the K producer publishes it.
struct TileInfo {
  int seg;       // segment number within this CTA (-1: end of the stream)
  int flags;     // 1: first tile of its segment, 2: last tile
  int key0;      // key of the tile's first chunk
  int vis_lo;    // keys of the segment that some row of its part can see
  int vis_hi;
  uint32_t mask; // 16-key chunks copied
  int row8[kChunksPerTile];  // fp16: TMA row coordinate / 8; int8: (block, head) tile
  int pad[2];
};
static_assert(sizeof(TileInfo) == 64, "TileInfo layout");

struct SegInfo {
  int s, kvh, h, slot;  // sequence (of this launch), KV head, row part, partial slot
  int L;                // the sequence's context length
  int rows;             // valid rows of the part
  int group;            // (s * Hkv + kvh) * halves + h
  int first;            // this segment makes the group's designated first arrival
  int expect;           // arrivals the group expects (segments x softmax warpgroups)
  int bad;              // a block index out of range was replaced by block 0
  int key_first;        // key of the segment's first tile
  int ntile;            // the segment's tiles
  int vis_lo, vis_hi;   // the keys of the segment that some row sees
  int pad[2];
};
static_assert(sizeof(SegInfo) == 64, "SegInfo layout");

// Finished partials a softmax warpgroup has yet to count in (group, expected
// arrivals, designated first): counted in at the end of its loop, or when
// the list is full.
constexpr int kPendLen = 8;

struct Misc {
  uint32_t tmem_base;
  int abort;
  int nqk, npv;                // QK and PV products issued (drains)
  int k_conv, v_conv;          // int8: tiles converted (drains)
  int n_merge;                 // mode 1: groups this CTA merges at the end
  int own_group;               // mode 0: the KV head whose merge this CTA shares (-1: none)
  int own_phase;               // ... its barrier phase before this call's arrivals
  int own_first, own_count;    // ... its partials: CTAs [first, first + count) of the set
  int own_slice, own_slices;   // ... this CTA's share of the merge
  int own_s, own_h, own_rows;
  int segs_published;          // segments whose description was published
  int segs_done[2];            // segments each softmax warpgroup counted in
  int last;
  int pad[11];
};
static_assert(sizeof(Misc) <= 128, "Misc layout");

template <int RW, int NG, int KV>
struct Cfg {
  static constexpr bool kQuant = KV != kKvFp16;
  static constexpr bool kQ8 = KV == kKvQ8_0;
  static constexpr int kVWarp = 2 + NG * 4;      // the V producer's warp
  static constexpr int kConvWarp = kVWarp + 1;   // int8: first converter warp
  static constexpr int kConvWarps = 4;           // converter warps per stream (K, V)
  static constexpr int kThreads = 32 * (kVWarp + 1 + (kQuant ? 2 * kConvWarps : 0));
  static constexpr int NR = (NG * RW < 16) ? 16 : NG * RW;  // MMA N of QK^T
  static constexpr int kSG = kQ8 ? kHeadDim / 32 : 1;      // S^T accumulators per tile
  static constexpr int KS = kQuant ? 2 : 3;
  static constexpr int VS = kQuant ? 2 : (NR > 16 ? 2 : 3);
  static constexpr uint32_t kKSlot = kKVBytes;
  // int8: raw V slots (16 KB of qs, then the tile's scales) feeding a ring of
  // kVCSlots converted half-tiles.
  static constexpr uint32_t kVSlot = kQuant ? kRawScales + 1024 : kKVBytes;
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = KS * kKSlot;
  static constexpr uint32_t kVC = kV + VS * kVSlot;
  static constexpr uint32_t kVCBytes = kQuant ? kVCSlots * kVCSlot : 0;
  static constexpr uint32_t kQ = kVC + kVCBytes;
  static constexpr uint32_t kQHalf = NR * 128;       // one 64-column half of Q
  static constexpr uint32_t kQBuf = 2 * kQHalf;      // Q of one segment
  static constexpr int kPN = 2 * NR;                 // N of the PV product
  static constexpr int PB = 2;
  static constexpr uint32_t kP = kQ + 2 * kQBuf;
  static constexpr uint32_t kPBytes = kTileKeys * kPN * 2;
  static constexpr uint32_t kRed = kP + PB * kPBytes;                 // float [NG][2][4][32]
  static constexpr uint32_t kLsum = kRed + NG * 2 * 4 * 32 * 4;       // float [NG][4][32]
  static constexpr uint32_t kBars = kLsum + NG * 4 * 32 * 4;          // uint64 [kBarSlots]
  static constexpr uint32_t kInfo = kBars + kBarSlots * 8;
  static constexpr uint32_t kSeg = kInfo + kInfoSlots * sizeof(TileInfo);
  static constexpr uint32_t kMisc = kSeg + kSegSlots * sizeof(SegInfo);
  static constexpr uint32_t kQueueArr = kMisc + 128;   // mode 1: int [3][kMaxQueueSeqs + 1]
  static constexpr uint32_t kMergeList = kQueueArr + 3 * (kMaxQueueSeqs + 1) * 4;
  static constexpr uint32_t kPend = kMergeList + kMergeListLen * 4;  // int [NG][kPendLen][3]
  static constexpr uint32_t kTotal = kPend + NG * kPendLen * 3 * 4;
  // TMEM: S^T[2] (kSG accumulators of NR columns), then O^T[2] (2 NR: the
  // high parts' products, then the residuals').
  static constexpr uint32_t kTmemS = 2 * kSG * NR;
  static constexpr uint32_t kTmemO = 2 * NR;
  static constexpr uint32_t kTmemUsed = kTmemS + 2 * kTmemO;
  static constexpr uint32_t kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64
                                        : kTmemUsed <= 128 ? 128 : kTmemUsed <= 256 ? 256 : 512;
  static_assert(KS <= kMaxStages && VS <= kMaxStages, "ring depth");
  static_assert(kTotal + 1024 <= 232448, "shared memory per CTA");
  static_assert(kV % 1024 == 0 && kVSlot % 1024 == 0 && kVC % 1024 == 0 && kQ % 1024 == 0,
                "tiles sit on 1 KB swizzle atoms");
  static_assert(kTmemUsed <= 512, "TMEM columns");
  static_assert(NG == 2 && NG * RW <= 32 && RW % 4 == 0, "rows per part");
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ int ld_nc_s32(const int* p) {
  int r;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ uint32_t ldg_nc_u32(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}
__device__ __forceinline__ uint16_t lds_u16(uint32_t addr) {
  uint16_t r;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr));
  return r;
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}
__device__ __forceinline__ void sts_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<const uint32_t*>(&h); }

// Four signed bytes -> four exact fp16 values, two per half2: byte b
// becomes the low mantissa byte of the fp16 1024 + (b + 128) (bits 0x6400 |
// (b ^ 0x80)), minus 1152; every integer below 2048 is exact in fp16.
__device__ __forceinline__ void q8_to_half4(uint32_t q, __half2& lo, __half2& hi) {
  const uint32_t w = q ^ 0x80808080u;
  const uint32_t a = __byte_perm(w, 0x64646464u, 0x5140), b = __byte_perm(w, 0x64646464u, 0x7362);
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
  lo = __hsub2(*reinterpret_cast<const __half2*>(&a), off);
  hi = __hsub2(*reinterpret_cast<const __half2*>(&b), off);
}

// Warp transpose-reduction over the 32 lanes (= 32 keys): lane l ends with
// the reduction of row (l % RW) in the return value.
template <int RW, bool kMax>
__device__ __forceinline__ float warp_row_reduce(float (&v)[RW], int lane) {
#pragma unroll
  for (int n = RW, o = RW / 2; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
#pragma unroll
  for (int o = RW; o < 32; o <<= 1) {
    const float got = __shfl_xor_sync(0xffffffffu, v[0], o);
    v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
  }
  return v[0];
}

// ----------------------------------------------------- the work decomposition
// Visible keys of a sequence (all its tokens; in partial mode only those in
// its key range) cut into 16-key chunks from `base` (the first visible key
// rounded down to a chunk).  bad: a context length outside [n_query,
// max_blocks_per_seq * block_size], or a key range that is not whole blocks
// inside the context and the table; nch = 0 then, and also for a valid key
// range that no query sees.
struct SeqVis {
  int lo, hi, base, nch, kb;
  bool bad;
};
__device__ __forceinline__ SeqVis seq_vis(const DecodeParams& p, int s, int L) {
  SeqVis v{0, -1, 0, 0, 0, false};
  int kb = 0, kc = 0;
  bool ok;
  if (p.key_begin != nullptr) {
    kb = ld_nc_s32(p.key_begin + s);
    kc = ld_nc_s32(p.key_count + s);
    ok = L >= p.n_query && kb >= 0 && kb % p.block_size == 0 && kc >= 0 &&
         (long long)kb + kc <= L && (long long)kc <= (long long)p.max_blocks_per_seq * p.block_size;
  } else {
    ok = context_len_ok(L, p.n_query, p.max_blocks_per_seq, p.block_size);
  }
  if (!ok) {
    v.bad = true;
    return v;
  }
  union_range(L, p.n_query, p.causal, p.window, v.lo, v.hi);
  if (p.key_begin != nullptr) {
    v.lo = max(v.lo, kb);
    v.hi = min(v.hi, kb + kc - 1);
  }
  v.kb = kb;
  v.base = (v.lo / kChunk) * kChunk;
  if (v.hi >= v.lo) v.nch = (v.hi + 1 - v.base + kChunk - 1) / kChunk;
  return v;
}
__device__ __forceinline__ int part_rows(const DecodeParams& p, int h) {
  return min(p.rows, (h + 1) * p.rows_half) - h * p.rows_half;
}
// Keys that some row of part h can see: the union over the part's tokens
// (consecutive tokens' ranges overlap, so the union is one range).
__device__ __forceinline__ void part_range(const DecodeParams& p, int L, int h, int& lo, int& hi) {
  const int r0 = h * p.rows_half;
  const int r1 = r0 + part_rows(p, h) - 1;
  int lo0, hi0, lo1, hi1;
  key_range(L, p.n_query, r0 / p.group, p.causal, p.window, lo0, hi0);
  key_range(L, p.n_query, r1 / p.group, p.causal, p.window, lo1, hi1);
  lo = min(lo0, lo1);
  hi = max(hi0, hi1);
}
// a / b for a >= 0, b > 0, with 32-bit division when both fit (the usual
// case: far cheaper than the 64-bit sequence).
__device__ __forceinline__ long long div64(long long a, long long b) {
  if (((unsigned long long)a | (unsigned long long)b) <= 0xffffffffull)
    return (long long)((unsigned)a / (unsigned)b);
  return a / b;
}
// Mode 0: the CTA of Ce whose chunk range [k W / Ce, (k+1) W / Ce) holds
// chunk x, and the first CTA whose range ends at or after chunk y.
__device__ __forceinline__ int cta_holding(long long x, int Ce, long long W) {
  return (int)div64((x + 1) * Ce - 1, W);
}
__device__ __forceinline__ int cta_ending_from(long long y, int Ce, long long W) {
  return (int)div64((y + 1) * Ce + W - 1, W) - 1;
}
// Mode 1: a group's chunks are items of 8T chunks, the last of which is cut
// into up to four sub-items (processed after every big item).
__device__ __forceinline__ void seq_items(int nch, int T, int& n_big, int& n_sub) {
  if (nch <= 0) {  // a sequence with a bad length: one item that writes its rows as 0
    n_big = 0;
    n_sub = 1;
    return;
  }
  n_big = (nch + 8 * T - 1) / (8 * T) - 1;
  const int last = nch - n_big * 8 * T;
  n_sub = min(4, (last + kChunksPerTile - 1) / kChunksPerTile);
}

// What the K producer knows of the segment it streams (kb: the sequence's
// first key in this call's block table, 0 outside partial mode).
struct SegDesc {
  int s, kvh, h, c0, c1, slot, L, base, kb, lo, hi, vis_lo, vis_hi, expect, first;
};

// Output row of local row r of part h of (sequence s, KV head kvh).
__device__ __forceinline__ long long out_row(const DecodeParams& p, int s, int kvh, int h, int r) {
  const int gr = h * p.rows_half + r;
  return ((long long)s * p.n_query + gr / p.group) * p.num_q_heads + kvh * p.group + gr % p.group;
}

// A group's arrival counter pair: [0] mode 0 barrier, [1] mode 1 count.
__device__ __forceinline__ int* group_counter(const DecodeParams& p, int group) {
  return p.arrivals + (long long)group * 2;
}

// Count `n` arrivals of a segment into its group (the designated first
// arrival adds 2^31 minus the others, so that the top bit flips once every
// arrival is in and the low bits return to zero).  Mode 1: the arrival that
// completes the group resets the counter and returns true.
__device__ __forceinline__ bool arrive(const DecodeParams& p, int group, int expect, bool first,
                                       int n) {
  int* cnt = group_counter(p, group);
  if (p.mode == 0) {
    red_release_add_gpu(cnt, first ? 0x80000000u - (unsigned)(expect - n) : (unsigned)n);
    return false;
  }
  const int old = atomicAdd(cnt + 1, n);
  if (old + n == expect) {
    atomicExch(cnt + 1, 0);
    return true;
  }
  return false;
}

// ------------------------------------------------------------------ merges
// Merge of S consecutive partial slots [slot0, slot0 + S) of one group into
// its output rows, the (row, float4 column) pairs [pa, pb) of it: M = max_k
// lse_k, w_k = exp(lse_k - M) (0 for an empty split), out = sum_k w_k O_k /
// sum_k w_k, splits added in slot order with a fixed lane split, so results
// are reproducible.  A NaN log-sum-exp marks a partial that read a
// stand-in for an out-of-range block: the group's rows are written as 0.
// The partial columns are staged with 16-byte asynchronous copies, all of a
// round in flight at once.
template <int kThreads>
__device__ __forceinline__ void merge_pairs(const DecodeParams& p, long long slot0, int S, int rows,
                                            int s, int kvh, int h, int pa, int pb, uint8_t* smem,
                                            uint32_t sbase, uint32_t smem_cap) {
  constexpr int kRowF4 = kHeadDim / 4;
  constexpr int kWarps = kThreads / 32;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long RHs = p.rows_half;  // partial rows per slot
  while (pa < pb) {
    const int r_lo = pa / kRowF4;
    int np = pb - pa;  // as many pairs per round as the staging area holds
    for (;;) {
      const int nr = (pa + np - 1) / kRowF4 - r_lo + 1;
      const uint32_t stage_off = ((uint32_t)(nr * S + nr) * 4u + 1023u) & ~1023u;
      if (stage_off + (uint32_t)(S * np) * 16u <= smem_cap || np == 1) break;
      np = max(1, np / 2);
    }
    const int nr = (pa + np - 1) / kRowF4 - r_lo + 1;
    float* w = reinterpret_cast<float*>(smem);  // [nr][S]
    float* inv = w + nr * S;                    // [nr]
    const uint32_t stage_off = ((uint32_t)(nr * S + nr) * 4u + 1023u) & ~1023u;
    const float4* stage4 = reinterpret_cast<const float4*>(smem + stage_off);  // [S][np]
    for (int e = threadIdx.x; e < S * np; e += kThreads) {
      const int k = e / np, pr = pa + e % np;
      const float* src =
          p.part_out + ((slot0 + k) * RHs + pr / kRowF4) * kHeadDim + (pr % kRowF4) * 4;
      cp_async_16(sbase + stage_off + (uint32_t)e * 16u, src);
    }
    for (int e = threadIdx.x; e < nr * S; e += kThreads)
      w[e] = __ldcg(p.part_lse + (slot0 + e % S) * RHs + r_lo + e / S);
    __syncthreads();
    for (int j = warp; j < nr; j += kWarps) {
      float M = -INFINITY;
      bool bad = false;
      for (int k = lane; k < S; k += 32) {
        M = fmaxf(M, w[j * S + k]);
        bad |= isnan(w[j * S + k]);
      }
      bad = __any_sync(0xffffffffu, bad);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      float sum = 0.f;
      for (int k = lane; k < S; k += 32) {
        const float l = w[j * S + k];
        const float wk = (bad || l == -INFINITY) ? 0.f : expf(l - M);
        w[j * S + k] = wk;
        sum += wk;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        inv[j] = sum > 0.f ? 1.f / sum : 0.f;
        // partial mode: the row's log-sum-exp, written by the share that
        // holds the row's first column
        const int r = r_lo + j;
        if (p.out_lse != nullptr && r < rows && r * kRowF4 >= pa && r * kRowF4 < pb)
          p.out_lse[out_row(p, s, kvh, h, r)] = sum > 0.f ? M + logf(sum) : -INFINITY;
      }
    }
    cp_async_wait_all();
    __syncthreads();
    // tp lanes of one warp per pair, each adding every tp-th split, then a
    // fixed butterfly; loop bounds are uniform per warp.
    int tp = 1;
    while (tp < 32 && 2 * tp * np <= kThreads) tp *= 2;
    const int per_warp = 32 / tp, sub = lane % tp;
    for (int q0 = warp * per_warp; q0 < np; q0 += kWarps * per_warp) {
      const int q = q0 + lane / tp;
      const bool valid = q < np;
      const int pr = pa + (valid ? q : 0), r = pr / kRowF4, c4 = pr % kRowF4, j = r - r_lo;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (valid) {
        for (int k = sub; k < S; k += tp) {
          const float wk = w[j * S + k];
          const float4 v = stage4[k * np + q];
          acc.x = fmaf(wk, v.x, acc.x);
          acc.y = fmaf(wk, v.y, acc.y);
          acc.z = fmaf(wk, v.z, acc.z);
          acc.w = fmaf(wk, v.w, acc.w);
        }
      }
      for (int o = tp / 2; o > 0; o >>= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
      }
      if (valid && sub == 0 && r < rows) {
        const float iv = inv[j];
        if (p.out_f32 != nullptr) {
          *reinterpret_cast<float4*>(p.out_f32 + out_row(p, s, kvh, h, r) * kHeadDim + c4 * 4) =
              make_float4(acc.x * iv, acc.y * iv, acc.z * iv, acc.w * iv);
        } else {
          uint2 u;
          u.x = h2_bits(__floats2half2_rn(acc.x * iv, acc.y * iv));
          u.y = h2_bits(__floats2half2_rn(acc.z * iv, acc.w * iv));
          *reinterpret_cast<uint2*>(p.out + out_row(p, s, kvh, h, r) * kHeadDim + c4 * 4) = u;
        }
      }
    }
    __syncthreads();  // the staging area is reused by the next round
    pa += np;
  }
}

// Output rows of part h of (s, kvh) that see no key (a bad length, or in
// partial mode a key range no query sees): 0 (partial mode: O = 0,
// lse = -inf).
__device__ __forceinline__ void zero_rows(const DecodeParams& p, int s, int kvh, int h, int lane) {
  const int rows = part_rows(p, h);
  for (int e = lane; e < rows * (kHeadDim / 8); e += 32) {
    const int r = e / (kHeadDim / 8), c = e % (kHeadDim / 8);
    const long long row = out_row(p, s, kvh, h, r);
    if (p.out_f32 != nullptr) {
      float4* o = reinterpret_cast<float4*>(p.out_f32 + row * kHeadDim + c * 8);
      o[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      o[1] = o[0];
      if (c == 0) p.out_lse[row] = -INFINITY;
    } else {
      *reinterpret_cast<uint4*>(p.out + row * kHeadDim + c * 8) = make_uint4(0, 0, 0, 0);
    }
  }
}

template <int RW, int NG, int KV, bool TR>
__global__ void __launch_bounds__(Cfg<RW, NG, KV>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using C = Cfg<RW, NG, KV>;
  constexpr bool kQuant = C::kQuant, kQ8 = C::kQ8;
  constexpr int kThreads = C::kThreads, kVWarp = C::kVWarp;
  constexpr int NR = C::NR, KS = C::KS, VS = C::VS, PB = C::PB;
  constexpr int kScaleBytes = KV == kKvQ8_0 ? 8 : 4;  // scales of one key (int8 caches)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by pointer
  // arithmetic so that accesses through it stay shared-space loads/stores.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kMisc);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + C::kInfo);
  SegInfo* seginfo = reinterpret_cast<SegInfo*>(smem + C::kSeg);
  int* merge_list = reinterpret_cast<int*>(smem + C::kMergeList);
  volatile int* abort = &misc->abort;
  const unsigned long long wl = p.wait_limit_ns;
  auto bar = [&](int i) { return sbase + C::kBars + 8u * i; };
  auto wait = [&](int b, int parity) { return mbar_wait(bar(b), (uint32_t)parity, abort, wl); };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int Hkv = p.num_kv_heads, H = p.halves;
  const uint32_t sK = sbase + C::kK, sV = sbase + C::kV, sVC = sbase + C::kVC;
  const uint32_t sQ = sbase + C::kQ, sP = sbase + C::kP;

  // Launched as a programmatic dependent of whatever precedes it on the
  // stream: nothing global is read before that grid has completed.
  griddep_wait();
  griddep_launch_dependents();

  if (warp == 0) {
    // =========================== K producer ===================================
    if (lane == 0) {
      for (int i = 0; i < kMaxStages; ++i) {
        mbar_init(bar(BAR_KFULL + i), 1);
        mbar_init(bar(BAR_KEMPTY + i), 1);
        mbar_init(bar(BAR_VFULL + i), 1);
        // int8 raw V slots are freed by the converter warps, fp16 ones by a commit
        mbar_init(bar(BAR_VEMPTY + i), kQuant ? C::kConvWarps : 1);
        mbar_init(bar(BAR_CKFULL + i), C::kConvWarps);
        mbar_init(bar(BAR_CVFULL + i), C::kConvWarps);
        mbar_init(bar(BAR_CVEMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(BAR_SFULL + i), 1);
        mbar_init(bar(BAR_SEMPTY + i), 4 * NG);
        mbar_init(bar(BAR_PFULL + i), 4 * NG);
        mbar_init(bar(BAR_OEMPTY + i), 4 * NG);
        mbar_init(bar(BAR_QFULL + i), 32);  // one per lane of the K producer
        mbar_init(bar(BAR_QEMPTY + i), 1);
      }
      mbar_init(bar(BAR_OFULL), 1);
      mbar_init(bar(BAR_DONE), 1);
      for (int i = 0; i < kInfoSlots; ++i) mbar_init(bar(BAR_INFO + i), 1);
      misc->abort = 0;
      misc->nqk = misc->npv = misc->k_conv = misc->v_conv = 0;
      misc->n_merge = 0;
      misc->own_group = -1;
      misc->segs_published = 0;
      misc->segs_done[0] = misc->segs_done[1] = 0;
      fence_mbar_init();
    }
    __syncwarp();
    named_bar_arrive(kBarSetup, kThreads);

    const int c = lane;  // lane c < 8 owns chunk c of every tile
    const int cta = blockIdx.x, Cgrid = gridDim.x;
    // The cache is streamed once: its lines go first when L2 needs room.
    const uint64_t pol = l2_evict_first_policy();
    int* qarr = reinterpret_cast<int*>(smem + C::kQueueArr);  // mode 1: Ls, P1, P2
    int* Ls = qarr;
    int* P1 = Ls + (kMaxQueueSeqs + 1);
    int* P2 = P1 + (kMaxQueueSeqs + 1);
    const int nseq = p.num_seqs;
    int total_items = 0, p1_total = 0;
    int next_q = 0;  // mode 1: the next item index, taken one segment ahead

    // -- mode 0: this CTA's chunk range of its (sequence, part) set ---------
    constexpr long long kNone = -(1LL << 40);
    int m0_s = 0, m0_h = 0, m0_k = 0, m0_L = 0, m0_Ce = 0, m0_nseg = 0, m0_next = 0;
    SeqVis m0_v{0, -1, 0, 0, 0, false};
    long long m0_a = 0, m0_b = 0, m0_W = 0;
    int own_g = -1, own_phase_raw = 0;
    // Speculation (mode 0, no window, every key of the context): the range
    // this CTA gets if the sequence fills its whole table, whose first
    // tile's table entries are read while the context length is in flight;
    // they are used when the real range starts at the same chunk.
    long long spec_raw = kNone;
    int spec_kvh = -1, spec_c0 = -1;
    if (p.mode == 0) {
      const int sigma = cta / p.ctas_per_set;
      m0_k = cta % p.ctas_per_set;
      m0_s = sigma / H;
      m0_h = sigma % H;
      m0_L = ld_nc_s32(p.context_lens + m0_s);
      if (p.window == 0 && p.key_begin == nullptr) {
        const long long nch_s = (long long)p.max_blocks_per_seq * p.block_size / kChunk;
        const long long Ws = (long long)Hkv * nch_s;
        const int Ces = (int)(Ws < (long long)p.ctas_per_set ? Ws : (long long)p.ctas_per_set);
        if (m0_k < Ces) {
          const long long a = div64((long long)m0_k * Ws, Ces);
          spec_kvh = (int)div64(a, nch_s);
          spec_c0 = (int)(a - (long long)spec_kvh * nch_s);
          const long long ch = spec_c0 + c;
          if (c < kChunksPerTile && ch < nch_s)
            spec_raw = ld_nc_s32(p.block_table + (long long)m0_s * p.max_blocks_per_seq +
                                 ch * kChunk / p.block_size);
        }
      }
      m0_v = seq_vis(p, m0_s, m0_L);
      m0_W = (long long)Hkv * m0_v.nch;
      m0_Ce = (int)(m0_W < (long long)p.ctas_per_set ? m0_W : (long long)p.ctas_per_set);
      if (m0_W == 0) {
        // No key (a bad length, or a key range no query sees): the set's
        // first CTA writes the part's rows.
        if (m0_k == 0) {
          for (int g = 0; g < Hkv; ++g) zero_rows(p, m0_s, g, m0_h, lane);
          if (lane == 0 && m0_h == 0 && m0_v.bad) atomicOr(p.flags, kFlagBadLen);
        }
      } else if (m0_k < m0_Ce) {
        m0_a = div64((long long)m0_k * m0_W, m0_Ce);
        m0_b = div64((long long)(m0_k + 1) * m0_W, m0_Ce);
        const int kvh0 = (int)div64(m0_a, m0_v.nch);
        m0_nseg = (m0_b > (long long)(kvh0 + 1) * m0_v.nch) ? 2 : 1;
        // Merge duty: the KV head of this CTA's last chunk, shared with the
        // other CTAs whose range ends in it.  Its barrier phase is read now,
        // before this CTA can arrive (relaxed: the load stays in flight).
        own_g = (int)div64(m0_b - 1, m0_v.nch);
        if (lane == 0)
          own_phase_raw = ld_relaxed_gpu(group_counter(p, (m0_s * Hkv + own_g) * H + m0_h));
      }
    } else {
      // -- mode 1: per-sequence item counts and their prefix sums ----------    } else {
      // -- mode 1: per-sequence item counts and their prefix sums ----------
      const int GH = Hkv * H;
      int run1 = 0, run2 = 0;
      if (lane == 0) {
        P1[0] = 0;
        P2[0] = 0;
      }
      for (int s0 = 0; s0 < nseq; s0 += 32) {
        const int s = s0 + lane;
        int nb = 0, ns = 0;
        if (s < nseq) {
          const int L = ld_nc_s32(p.context_lens + s);
          seq_items(seq_vis(p, s, L).nch, p.item_tiles, nb, ns);
          Ls[s] = L;
        }
        int a = nb * GH, b = ns * GH;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {  // inclusive scans
          const int ya = __shfl_up_sync(0xffffffffu, a, o), yb = __shfl_up_sync(0xffffffffu, b, o);
          if (lane >= o) {
            a += ya;
            b += yb;
          }
        }
        if (s < nseq) {
          P1[s + 1] = run1 + a;
          P2[s + 1] = run2 + b;
        }
        run1 += __shfl_sync(0xffffffffu, a, 31);
        run2 += __shfl_sync(0xffffffffu, b, 31);
      }
      p1_total = run1;
      total_items = run1 + run2;
      __syncwarp();
      if (lane == 0) next_q = atomicAdd(p.queue, 1);
      next_q = __shfl_sync(0xffffffffu, next_q, 0);
    }

    // The next segment of this CTA (false: none left).  Mode 1 takes items
    // off the queue until one with keys comes up; every CTA makes exactly one
    // take past the end, and the last of all takes resets the counter.
    auto next_segment = [&](SegDesc& d) -> bool {
      if (p.mode == 0) {
        if (m0_next >= m0_nseg) return false;
        d.kvh = (int)div64(m0_a, m0_v.nch) + m0_next;
        const long long g0 = (long long)d.kvh * m0_v.nch;
        d.c0 = (int)max(0LL, m0_a - g0);
        d.c1 = (int)min((long long)m0_v.nch, m0_b - g0);
        d.s = m0_s;
        d.h = m0_h;
        d.L = m0_L;
        d.base = m0_v.base;
        d.kb = m0_v.kb;
        d.lo = m0_v.lo;
        d.hi = m0_v.hi;
        d.slot = (m0_s * H + m0_h) * (p.ctas_per_set + Hkv) + m0_k + d.kvh;
        const int kf = cta_holding(g0, m0_Ce, m0_W);
        const int kl = cta_holding(g0 + m0_v.nch - 1, m0_Ce, m0_W);
        d.expect = (kl - kf + 1) * NG;
        d.first = d.c0 == 0;
        ++m0_next;
      } else {
        for (;;) {
          int q = next_q;
          if (q >= total_items) {
            if (q == total_items + Cgrid - 1 && lane == 0) atomicExch(p.queue, 0);
            return false;
          }
          if (lane == 0) next_q = atomicAdd(p.queue, 1);  // the one after, in flight
          next_q = __shfl_sync(0xffffffffu, next_q, 0);
          const bool phase1 = q < p1_total;
          const int* P = phase1 ? P1 : P2;
          if (!phase1) q -= p1_total;
          int lo = 0, hi = nseq - 1;  // the last s with P[s] <= q
          while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (P[mid] <= q) lo = mid; else hi = mid - 1;
          }
          const int s = lo;
          int rem = q - P[s];
          d.h = rem % H;
          rem /= H;
          d.kvh = rem % Hkv;
          const int i = rem / Hkv;
          d.s = s;
          d.L = Ls[s];
          const SeqVis v = seq_vis(p, s, d.L);
          int nb, ns;
          seq_items(v.nch, p.item_tiles, nb, ns);
          if (v.nch == 0) {  // no key: write the part's rows
            zero_rows(p, s, d.kvh, d.h, lane);
            if (lane == 0 && d.kvh == 0 && d.h == 0 && v.bad) atomicOr(p.flags, kFlagBadLen);
            continue;
          }
          const int g = (s * Hkv + d.kvh) * H + d.h;
          d.base = v.base;
          d.kb = v.kb;
          d.lo = v.lo;
          d.hi = v.hi;
          if (phase1) {
            d.c0 = i * 8 * p.item_tiles;
            d.c1 = d.c0 + 8 * p.item_tiles;
            d.slot = g * p.slots_per_group + i;
          } else {
            const int start = nb * 8 * p.item_tiles, last = v.nch - start;
            d.c0 = start + (int)((long long)i * last / ns);
            d.c1 = start + (int)((long long)(i + 1) * last / ns);
            d.slot = g * p.slots_per_group + nb + i;
          }
          d.expect = (nb + ns) * NG;
          d.first = 0;
          break;
        }
      }
      int plo, phi;
      part_range(p, d.L, d.h, plo, phi);
      d.vis_lo = max(max(plo, d.lo), d.base + d.c0 * kChunk);
      d.vis_hi = min(min(phi, d.hi), d.base + d.c1 * kChunk - 1);
      return true;
    };

    // Q rows of a segment -> shared memory by asynchronous 16-byte copies
    // (lane-strided pieces), K-major with the 128-byte swizzle: row n, piece
    // cc of half cc / 8 at half * kQHalf + n * 128 + ((cc % 8) ^ (n % 8)) * 16.
    // Rows past the part's valid rows are zero-filled.  Each lane's copies
    // count one arrival on QFULL when they have landed; the MMA issuer makes
    // them visible to the tensor cores with a proxy fence.
    constexpr int kQPer = NR * 16 / 32;  // 16-byte pieces per lane
    auto stage_q = [&](const SegDesc& d, int qb) {
      const int rows = part_rows(p, d.h);
      const uint32_t dst = sQ + qb * C::kQBuf;
      // Row n = 2k + lane / 16 of the part is token qi, head qg of the KV
      // head's group (as out_row), stepped by two rows per piece.
      const int cc = lane % 16, gr0 = d.h * p.rows_half + lane / 16;
      int qi = gr0 / p.group, qg = gr0 - qi * p.group;
      const __half* base =
          p.q + ((long long)d.s * p.n_query * p.num_q_heads + (long long)d.kvh * p.group) * kHeadDim +
          cc * 8;
#pragma unroll
      for (int k = 0; k < kQPer; ++k) {
        const int n = 2 * k + lane / 16;
        const bool in = n < rows;
        const __half* src = in ? base + ((long long)qi * p.num_q_heads + qg) * kHeadDim : p.q;
        cp_async_16_zfill(dst + (cc / 8) * C::kQHalf + n * 128 + (((cc % 8) ^ (n & 7)) * 16), src,
                          in ? 16u : 0u);
        qg += 2;
        while (qg >= p.group) {
          qg -= p.group;
          ++qi;
        }
      }
      cp_async_mbar_arrive_noinc(bar(BAR_QFULL + qb));
    };

    // Block-table entry of chunk c of the tile that starts at chunk tc0
    // (kNone: not copied).
    auto lookup = [&](const SegDesc& d, int tc0) -> long long {
      const int ci = tc0 + c;
      if (c >= kChunksPerTile || ci >= d.c1) return kNone;
      const int key0 = d.base + ci * kChunk;
      if (key0 > d.vis_hi || key0 + kChunk - 1 < d.vis_lo) return kNone;
      return ld_nc_s32(p.block_table + (long long)d.s * p.max_blocks_per_seq +
                       (key0 - d.kb) / p.block_size);
    };
    // TMA row coordinate / 8 (fp16) or (block, head) tile (int8) of that
    // chunk; -1 if not copied.  An out-of-range block is never dereferenced:
    // block 0 stands in for it, the error flag is raised and the segment is
    // marked, so that the merge writes the group's rows as 0.
    auto to_row8 = [&](long long phys, const SegDesc& d, int tc0, int segslot) -> int {
      if (phys == kNone) return -1;
      if (phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.flags, kFlagBadBlock);
        seginfo[segslot].bad = 1;
        phys = 0;
      }
      if (kQuant) return (int)(phys * Hkv + d.kvh);
      const int key0 = d.base + (tc0 + c) * kChunk;
      return (int)(((phys * Hkv + d.kvh) * p.block_size + key0 % p.block_size) / 8);
    };
    // A segment this CTA owns but will not compute (abort path): an invalid
    // partial, counted in for every softmax warpgroup.
    auto give_up = [&](const SegDesc& d) {
      const int rows = part_rows(p, d.h);
      for (int r = lane; r < rows; r += 32)
        p.part_lse[(long long)d.slot * p.rows_half + r] = __uint_as_float(kInvalidLse);
      __threadfence();
      __syncwarp();
      if (lane == 0) arrive(p, (d.s * Hkv + d.kvh) * H + d.h, d.expect, d.first, NG);
    };

    int t = 0, seg_n = 0, seg_written = 0;
    SegDesc cur{}, nxt{};
    bool have = next_segment(cur);
    // The segment after the current one is taken at the current one's first
    // tile, so that its first block-table entries are in flight for a whole
    // segment (a load issued behind the stream takes microseconds).
    bool have_nxt = false, planned = false;
    long long raw_first_nxt = kNone;
    long long raw_cur = kNone;
    if (have) {
      if (cur.kvh == spec_kvh && cur.c0 == spec_c0 && cur.base == 0) {
        // the speculated entries, for the chunks the real range keeps
        const int ci = cur.c0 + c, key0 = cur.base + ci * kChunk;
        raw_cur = (c < kChunksPerTile && ci < cur.c1 && key0 <= cur.vis_hi &&
                   key0 + kChunk - 1 >= cur.vis_lo) ? spec_raw : kNone;
      } else {
        raw_cur = lookup(cur, cur.c0);
      }
    }
    bool ok = true;
    while (have && ok) {
      const int segslot = seg_n % kSegSlots, qb = seg_n % 2;
      if (lane == 0) {
        SegInfo& si = seginfo[segslot];
        si.s = cur.s; si.kvh = cur.kvh; si.h = cur.h; si.slot = cur.slot;
        si.L = cur.L; si.rows = part_rows(p, cur.h);
        si.group = (cur.s * Hkv + cur.kvh) * H + cur.h;
        si.first = cur.first; si.expect = cur.expect; si.bad = 0;
        si.key_first = cur.base + cur.c0 * kChunk;
        si.ntile = (cur.c1 - cur.c0 + kChunksPerTile - 1) / kChunksPerTile;
        si.vis_lo = cur.vis_lo; si.vis_hi = cur.vis_hi;
      }
      seg_written = seg_n + 1;
      __syncwarp();
      // The Q buffer of this segment is free once QK of segment seg_n - 2 ended.
      int w = 1;
      if (lane == 0) w = wait(BAR_QEMPTY + qb, ((seg_n / 2) & 1) ^ 1);
      ok = __shfl_sync(0xffffffffu, w, 0) != 0;
      if (!ok) break;
      const int ntile = (cur.c1 - cur.c0 + kChunksPerTile - 1) / kChunksPerTile;
      planned = false;
      for (int tau = 0; tau < ntile; ++tau) {
        const int tc0 = cur.c0 + tau * kChunksPerTile;
        const int row_cur = to_row8(raw_cur, cur, tc0, segslot);
        // The next tile's block-table entries, in flight during this one.
        const bool more = tau + 1 < ntile;
        long long raw_nxt = more ? lookup(cur, tc0 + kChunksPerTile) : kNone;
        const uint32_t mask = __ballot_sync(0xffffffffu, row_cur >= 0);
        TileInfo& ti = info[t % kInfoSlots];
        if (lane < kChunksPerTile) ti.row8[lane] = row_cur;
        if (lane == 0) {
          ti.seg = seg_n;
          ti.flags = (tau == 0 ? 1 : 0) | (tau == ntile - 1 ? 2 : 0);
          ti.key0 = cur.base + tc0 * kChunk;
          ti.vis_lo = cur.vis_lo;
          ti.vis_hi = cur.vis_hi;
          ti.mask = mask;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(BAR_INFO + t % kInfoSlots));
        const int st = t % KS;
        if (lane == 0) w = wait(BAR_KEMPTY + st, ((t / KS) & 1) ^ 1);
        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
        if (!ok) break;
        const uint32_t fb = bar(BAR_KFULL + st);
        if (lane == 0) mbar_arrive_expect_tx(fb, __popc(mask) * (kQuant ? kQsChunk : kChunkBytes));
        __syncwarp();
        if (row_cur >= 0) {
          if constexpr (kQuant) {
            const long long tb = quant_tile_bytes(KV, p.block_size);
            const int slot0 = (cur.base + (tc0 + c) * kChunk) % p.block_size;
            const long long off = (long long)row_cur * tb + (long long)slot0 * kHeadDim;
            const long long soff = (long long)row_cur * tb + (long long)p.block_size * kHeadDim +
                                   (long long)slot0 * kScaleBytes;
            const uint8_t* kc = static_cast<const uint8_t*>(p.k);
            const uint8_t* vc = static_cast<const uint8_t*>(p.v);
            bulk_load_hint(sK + st * C::kKSlot + kRawOff + c * kQsChunk, kc + off, kQsChunk, fb, pol);
            // K scales (the softmax reads them) and the V tile, into L2
            bulk_prefetch_l2_hint(kc + soff, kChunk * kScaleBytes, pol);
            bulk_prefetch_l2_hint(vc + off, kQsChunk, pol);
            bulk_prefetch_l2_hint(vc + soff, kChunk * kScaleBytes, pol);
          } else {
            tma_load_4d_hint(sK + st * C::kKSlot + c * kChunkBytes, &tmap_k, 0, 0, 0, row_cur, fb, pol);
            tma_prefetch_4d_hint(&tmap_v, 0, 0, 0, row_cur, pol);
          }
        }
        __syncwarp();
        if (tau == 0) {
          // The segment's Q rows, behind its first K copies (QK(first) waits
          // for both).
          stage_q(cur, qb);
          have_nxt = next_segment(nxt);
          planned = true;
          if (have_nxt) raw_first_nxt = lookup(nxt, nxt.c0);
        }
        ++t;
        if (!more) {
          ++seg_n;
          raw_nxt = raw_first_nxt;
        }
        raw_cur = raw_nxt;
      }
      if (!ok) break;
      cur = nxt;
      have = have_nxt;
    }
    if (ok) {  // end of the stream
      if (lane == 0) {
        TileInfo& ti = info[t % kInfoSlots];
        ti.seg = -1;
        ti.flags = 0;
        mbar_arrive(bar(BAR_INFO + t % kInfoSlots));
      }
    } else {
      // Abort: count in every segment this CTA owns but did not publish, and
      // (mode 1) take the remaining items off the queue the same way (the
      // queue is taken from until it first reports its end, never after).
      if (planned && have_nxt) give_up(nxt);
      if (!planned || have_nxt) {
        SegDesc d{};
        while (next_segment(d)) give_up(d);
      }
    }
    cp_async_wait_all();  // no Q copy outlives the producer
    if (lane == 0) misc->segs_published = seg_written;
    if (own_g >= 0 && lane == 0) {
      // mode 0 merge duty (see above): the KV head's partials are CTAs
      // [kf, kl] of the set, its owners [ko_lo, ko_hi]
      const long long g0 = (long long)own_g * m0_v.nch;
      const int ko_lo = cta_ending_from(g0, m0_Ce, m0_W);
      const int ko_hi =
          own_g + 1 < Hkv ? cta_ending_from(g0 + m0_v.nch, m0_Ce, m0_W) - 1 : m0_Ce - 1;
      const int kf = cta_holding(g0, m0_Ce, m0_W);
      const int kl = cta_holding(g0 + m0_v.nch - 1, m0_Ce, m0_W);
      misc->own_phase = (int)((unsigned)own_phase_raw & 0x80000000u);
      misc->own_group = own_g;
      misc->own_first = kf;
      misc->own_count = kl - kf + 1;
      misc->own_slice = m0_k - ko_lo;
      misc->own_slices = ko_hi - ko_lo + 1;
      misc->own_s = m0_s;
      misc->own_h = m0_h;
      misc->own_rows = part_rows(p, m0_h);
    }
    __syncwarp();
    __syncthreads();  // (A) every role finished its loop
    if (lane == 0) {  // drain copies that no consumer waited for (abort path only)
      volatile int no_abort = 0;
      for (int u = kQuant ? misc->k_conv : misc->nqk; u < t; ++u)
        mbar_wait(bar(BAR_KFULL + u % KS), (u / KS) & 1, &no_abort);
    }
  } else {
    // ---- set-up of the other roles ----------------------------------------
    if (warp == 1) {
      tmem_alloc(sbase + C::kMisc + offsetof(Misc, tmem_base), C::kTmemCols);
      tmem_relinquish();
    }
    if (warp == kVWarp) {
      // P buffers start at zero: the columns of padding rows are never written.
      for (uint32_t off = lane * 16; off < PB * C::kPBytes; off += 32 * 16)
        sts_v4(sP + off, make_uint4(0, 0, 0, 0));
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_bar_sync(kBarSetup, kThreads);  // barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kVWarp) {
      // ===================== V producer ======================================
      const int c = lane;
      const uint64_t pol = l2_evict_first_policy();
      int issued = 0;
      for (int t = 0;; ++t) {
        int w = 1;
        if (lane == 0) w = wait(BAR_INFO + t % kInfoSlots, (t / kInfoSlots) & 1);
        w = __shfl_sync(0xffffffffu, w, 0);
        __syncwarp();
        if (!w) break;
        const TileInfo& ti = info[t % kInfoSlots];
        if (ti.seg < 0) break;
        const uint32_t mask = ti.mask;
        const int row8 = c < kChunksPerTile ? ti.row8[c] : 0;
        const int key0 = ti.key0 + c * kChunk;
        const int st = t % VS;
        if (lane == 0) w = wait(BAR_VEMPTY + st, ((t / VS) & 1) ^ 1);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) break;
        const uint32_t fb = bar(BAR_VFULL + st);
        if (lane == 0)
          mbar_arrive_expect_tx(fb, __popc(mask) * (kQuant ? kQsChunk + kChunk * kScaleBytes
                                                           : kChunkBytes));
        __syncwarp();
        if (c < kChunksPerTile && ((mask >> c) & 1u)) {
          if constexpr (kQuant) {
            const long long tb = quant_tile_bytes(KV, p.block_size);
            const int slot0 = key0 % p.block_size;
            const uint8_t* src = static_cast<const uint8_t*>(p.v) + (long long)row8 * tb;
            const uint32_t dst = sV + st * C::kVSlot;
            bulk_load_hint(dst + c * kQsChunk, src + (long long)slot0 * kHeadDim, kQsChunk, fb, pol);
            bulk_load_hint(dst + kRawScales + c * (kChunk * kScaleBytes),
                           src + (long long)p.block_size * kHeadDim + (long long)slot0 * kScaleBytes,
                           kChunk * kScaleBytes, fb, pol);
          } else {
            tma_load_4d_hint(sV + st * C::kVSlot + c * kChunkBytes, &tmap_v, 0, 0, 0, row8, fb, pol);
          }
        }
        __syncwarp();
        issued = t + 1;
      }
      __syncthreads();  // (A)
      if (lane == 0) {  // drain copies that no consumer waited for (abort path only)
        volatile int no_abort = 0;
        for (int u = kQuant ? misc->v_conv : misc->npv; u < issued; ++u)
          mbar_wait(bar(BAR_VFULL + u % VS), (u / VS) & 1, &no_abort);
      }
    } else if (warp == 1) {
      // ===================== MMA issuer ======================================
      if (lane == 0) {
        constexpr int kSG = C::kSG;
        const uint32_t id_qk = idesc_f16_f32(128, NR, false, false);
        const uint32_t id_pv = idesc_f16_f32(128, C::kPN, true, true);
        const uint32_t id_pv_lo = idesc_f16_f32(128, NR, true, true);
        // Descriptors at offset 0; a byte offset o is added as o >> 4.
        const uint64_t dK = smem_desc(sK, 16, kGroupBytes, kSwizzle128B);
        const uint64_t dQ = smem_desc(sQ, 16, 1024, kSwizzle128B);
        const uint64_t dV = smem_desc(kQuant ? sVC : sV, kAtomBytes, kGroupBytes, kSwizzle128B);
        const uint64_t dP = smem_desc(sP, C::kPN * 16, 128, kSwizzleNone);
        int t_end = 0x7fffffff, nqk = 0, npv = 0;
        // QK(u) once tile u is described, K(u) is ready and the softmax took
        // S(u-2) from its buffer; returns 0 ok, 1 end of stream, -1 abort.
        auto issue_qk = [&](int u) -> int {
          if (!wait(BAR_INFO + u % kInfoSlots, (u / kInfoSlots) & 1)) return -1;
          const TileInfo& ti = info[u % kInfoSlots];
          const int seg = ti.seg, flags = ti.flags;
          if (seg < 0) return 1;
          if (flags & 1) {
            if (!wait(BAR_QFULL + seg % 2, (seg / 2) & 1)) return -1;
            fence_proxy_async_smem();  // Q arrived by cp.async (generic proxy)
          }
          if (!wait((kQuant ? BAR_CKFULL : BAR_KFULL) + u % KS, (u / KS) & 1)) return -1;
          if (!wait(BAR_SEMPTY + u % 2, ((u / 2) & 1) ^ 1)) return -1;
          tc_fence_after();
          const uint64_t so = (uint64_t)((u % KS) * C::kKSlot) >> 4;
          const uint64_t qo0 = (uint64_t)((seg % 2) * C::kQBuf) >> 4;
          const uint32_t d = tmem + (u % 2) * kSG * NR;
          constexpr int kSteps = kHeadDim / 16 / kSG;  // steps of 16 per accumulator
#pragma unroll
          for (int k = 0; k < kHeadDim / 16; ++k) {
            const uint64_t ko = ((k / 4) * kAtomBytes + (k % 4) * 32) >> 4;
            const uint64_t qo = ((k / 4) * C::kQHalf + (k % 4) * 32) >> 4;
            tc_mma_f16_ss(d + (k / kSteps) * NR, dK + so + ko, dQ + qo0 + qo, id_qk, k % kSteps != 0);
          }
          tc_commit(bar(BAR_SFULL + u % 2));
          tc_commit(bar(BAR_KEMPTY + u % KS));
          if (flags & 2) tc_commit(bar(BAR_QEMPTY + seg % 2));
          return 0;
        };
        bool ok = true;
        for (int u = 0; u < 2 && ok; ++u) {
          const int r = issue_qk(u);
          if (r == 1) {
            t_end = u;
            break;
          }
          ok = r == 0;
          if (ok) nqk = u + 1;
        }
        for (int t = 0; ok && t < t_end; ++t) {
          const TileInfo& ti = info[t % kInfoSlots];  // described before QK(t)
          const int seg = ti.seg, flags = ti.flags, ob = seg % 2;
          ok = wait(BAR_PFULL + t % PB, (t / PB) & 1) &&
               (kQuant || wait(BAR_VFULL + t % VS, (t / VS) & 1)) &&
               (!(flags & 1) || wait(BAR_OEMPTY + ob, ((seg / 2) & 1) ^ 1));
          if (!ok) break;
          tc_fence_after();
          const uint64_t pb = (uint64_t)((t % PB) * C::kPBytes) >> 4;
          const uint32_t d = tmem + C::kTmemS + ob * C::kTmemO;
          if constexpr (kQuant) {
            // Two half-tiles of 64 keys, each from its converted slot:
            // V_hi [P_hi | P_lo], then V_lo times the high parts of P (the
            // first NR columns).
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int hx = 2 * t + hf;
              if (!wait(BAR_CVFULL + hx % kVCSlots, (hx / kVCSlots) & 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t so = (uint32_t)(hx % kVCSlots) * kVCSlot;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t vo = (so + k * 2 * kGroupBytes) >> 4;
                const uint64_t po = ((hf * 4 + k) * 2 * C::kPN * 16) >> 4;
                tc_mma_f16_ss(d, dV + vo, dP + pb + po, id_pv, !(flags & 1) || hf > 0 || k > 0);
                tc_mma_f16_ss(d, dV + vo + (kVCLo >> 4), dP + pb + po, id_pv_lo, 1);
              }
              tc_commit(bar(BAR_CVEMPTY + hx % kVCSlots));
            }
            if (!ok) break;
          } else {
            const uint64_t so = (uint64_t)((t % VS) * C::kVSlot) >> 4;
#pragma unroll
            for (int k = 0; k < kTileKeys / 16; ++k) {
              const uint64_t vo = (k * 2 * kGroupBytes) >> 4;
              const uint64_t po = (k * 2 * C::kPN * 16) >> 4;
              tc_mma_f16_ss(d, dV + so + vo, dP + pb + po, id_pv, !(flags & 1) || k > 0);
            }
            tc_commit(bar(BAR_VEMPTY + t % VS));
          }
          tc_commit(bar(BAR_OFULL));
          npv = t + 1;
          if (t_end == 0x7fffffff) {
            const int r = issue_qk(t + 2);
            if (r == 1) t_end = t + 2;
            ok = r >= 0;
            if (r == 0) nqk = t + 3;
          }
        }
        misc->nqk = nqk;
        misc->npv = npv;
        tc_commit(bar(BAR_DONE));  // completes once every MMA above has finished
        volatile int no_abort = 0;
        mbar_wait(bar(BAR_DONE), 0, &no_abort);
      }
      __syncwarp();
      __syncthreads();  // (A)
    } else if (kQuant && warp >= C::kConvWarp) {
      // ===================== int8 converters =================================
      // Layout of a converted tile as the fp16 TMA boxes: [key/8][half]
      // [key%8][64 dims], 128-byte swizzle.  Thread ct of a stream's 128
      // takes the 16-byte column chunk c16 = ct % 8 (head_dim 16 c16 .. +15,
      // half of one q8_0 scale group) of keys r0 + 16 k, k = 0..7: one
      // 16-byte load and two 16-byte stores per key and operand, no bank
      // conflicts on either side.
      // K: in place, the raw int8 tile in the upper half of its slot; keys
      // 0..63 are written below it, keys 64..127 only after every thread of
      // the stream has read its raw rows (named barrier); the operand is qs.
      // V: raw slot -> the converted slot's hi and lo tiles (qs * d split
      // into two fp16 parts); rows of keys no row of the part sees are
      // written as zeros.
      constexpr int kCT = 32 * C::kConvWarps;
      constexpr int kRS = kCT / 8;               // key stride between a thread's keys (16)
      constexpr int kKeysPer = kTileKeys / kRS;  // keys per thread per tile (8)
      constexpr int kHalfKeys = kKeysPer / 2;
      const int kv = (warp - C::kConvWarp) / C::kConvWarps;  // 0: K, 1: V
      const int ct = threadIdx.x - 32 * (C::kConvWarp + C::kConvWarps * kv);
      const int c16 = ct & 7, r0 = ct >> 3;
      const int r08 = r0 & 7;
      const uint32_t dst_a = (r0 >> 3) * kGroupBytes + ((2 * c16) >> 3) * kAtomBytes + r08 * 128 +
                             ((((2 * c16) & 7) ^ r08) << 4);
      const uint32_t dst_b = (r0 >> 3) * kGroupBytes + ((2 * c16 + 1) >> 3) * kAtomBytes +
                             r08 * 128 + ((((2 * c16 + 1) & 7) ^ r08) << 4);
      const int NSl = kv == 0 ? KS : VS;
      int t = 0;
      for (;; ++t) {
        // The tile's description (end of the stream, V's visible keys), then
        // the data; the stream's threads decide together so that all of them
        // reach the named barriers.
        bool live = wait(BAR_INFO + t % kInfoSlots, (t / kInfoSlots) & 1);
        const TileInfo& ti = info[t % kInfoSlots];
        live = live && ti.seg >= 0;
        const int rs = t % NSl;
        if (live) live = wait((kv == 0 ? BAR_KFULL : BAR_VFULL) + rs, (t / NSl) & 1);
        if (!named_bar_and(kBarConv0 + kv, kCT, __all_sync(0xffffffffu, live))) break;
        const int key_t = ti.key0, vlo = ti.vis_lo, vhi = ti.vis_hi;
        if (kv == 1) {
         const uint32_t slot = sV + rs * C::kVSlot;
         bool vok = true;
#pragma unroll 1
         for (int hf = 0; hf < 2; ++hf) {
          // half-tile hx = keys 64 hf .. 64 hf + 63 of tile t, into converted
          // slot hx % kVCSlots once PV has read that slot's previous half-tile
          const int hx = 2 * t + hf;
          vok = __all_sync(0xffffffffu, vok && wait(BAR_CVEMPTY + hx % kVCSlots, ((hx / kVCSlots) & 1) ^ 1));
          const uint32_t dslot = sVC + (uint32_t)(hx % kVCSlots) * kVCSlot;
          const uint32_t src = slot + (hf * 64 + r0) * kHeadDim + c16 * 16;
#pragma unroll 2
          for (int k = 0; k < kKeysPer / 2; ++k) {
            const int r = hf * 64 + k * kRS + r0;
            const uint4 qv = lds_v4(src + k * kRS * kHeadDim);
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) hi[e] = lo[e] = 0u;
            if (key_t + r >= vlo && key_t + r <= vhi) {
              __half2 x[8];
              q8_to_half4(qv.x, x[0], x[1]);
              q8_to_half4(qv.y, x[2], x[3]);
              q8_to_half4(qv.z, x[4], x[5]);
              q8_to_half4(qv.w, x[6], x[7]);
              if constexpr (kQ8) {
                // d: the fp16 scale of this 32-element group; qs * d split
                // exactly into fp16(qs * d) and the (exact) residual.
                const __half d = __ushort_as_half(
                    lds_u16(slot + kRawScales + r * kScaleBytes + (c16 >> 1) * 2));
                const __half2 d2 = __halves2half2(d, d);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const __half2 yh = __hmul2(x[e], d2);
                  hi[e] = h2_bits(yh);
                  lo[e] = h2_bits(__hfma2(x[e], d2, __hneg2(yh)));
                }
              } else {
                // s: the fp32 scale of this row; qs * s in fp32, split into
                // two fp16 parts.
                const float sc = __uint_as_float(lds_u32(slot + kRawScales + r * kScaleBytes));
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  const float2 f = __half22float2(x[e]);
                  const float a = f.x * sc, b = f.y * sc;
                  const __half2 yh = __floats2half2_rn(a, b);
                  const float2 g2 = __half22float2(yh);
                  hi[e] = h2_bits(yh);
                  lo[e] = h2_bits(__floats2half2_rn(a - g2.x, b - g2.y));
                }
              }
            }
            const uint32_t g8 = k * (kRS / 8) * kGroupBytes;
            if (vok) {
              sts_v4(dslot + g8 + dst_a, make_uint4(hi[0], hi[1], hi[2], hi[3]));
              sts_v4(dslot + g8 + dst_b, make_uint4(hi[4], hi[5], hi[6], hi[7]));
              sts_v4(dslot + kVCLo + g8 + dst_a, make_uint4(lo[0], lo[1], lo[2], lo[3]));
              sts_v4(dslot + kVCLo + g8 + dst_b, make_uint4(lo[4], lo[5], lo[6], lo[7]));
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && vok) mbar_arrive(bar(BAR_CVFULL + hx % kVCSlots));
         }
         __syncwarp();
         if (lane == 0) mbar_arrive(bar(BAR_VEMPTY + rs));  // the raw slot may be refilled
        } else {
          const uint32_t slot = sK + rs * C::kKSlot;
          const uint32_t src = slot + kRawOff + r0 * kHeadDim + c16 * 16;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint4 xa[kHalfKeys], xb[kHalfKeys];
#pragma unroll
            for (int i = 0; i < kHalfKeys; ++i) {
              const int k = hh * kHalfKeys + i;
              const uint4 qv = lds_v4(src + k * kRS * kHeadDim);
              __half2 a0, a1, a2, a3;
              q8_to_half4(qv.x, a0, a1);
              q8_to_half4(qv.y, a2, a3);
              xa[i] = make_uint4(h2_bits(a0), h2_bits(a1), h2_bits(a2), h2_bits(a3));
              q8_to_half4(qv.z, a0, a1);
              q8_to_half4(qv.w, a2, a3);
              xb[i] = make_uint4(h2_bits(a0), h2_bits(a1), h2_bits(a2), h2_bits(a3));
            }
            // The upper keys overwrite raw rows: every thread of the stream
            // has read all of its rows once it is past this barrier.
            if (hh == 1) named_bar_sync(kBarConv0 + kv, kCT);
#pragma unroll
            for (int i = 0; i < kHalfKeys; ++i) {
              const uint32_t g8 = (hh * kHalfKeys + i) * (kRS / 8) * kGroupBytes;
              sts_v4(slot + g8 + dst_a, xa[i]);
              sts_v4(slot + g8 + dst_b, xb[i]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_CKFULL + rs));
        }
        (void)key_t;
      }
      if (ct == 0) {
        if (kv == 0) misc->k_conv = t; else misc->v_conv = t;
      }
      __syncthreads();  // (A)
    } else {
      // ===================== softmax + correction ============================
      // Warpgroup g handles rows [g*RW, g*RW + RW) of the part; its warps
      // cover the four TMEM lane quarters: keys (for S), head_dim (for O).
      const int g = (warp - 2) / 4, widx = (warp - 2) % 4;
      const int row0 = g * RW;
      const int q4 = warp & 3;
      const int j = q4 * 32 + lane;  // this thread's key within a tile / head_dim lane of O
      const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
      float* red = reinterpret_cast<float*>(smem + C::kRed) + g * 2 * 4 * 32;  // [2][4][32]
      float* lsum = reinterpret_cast<float*>(smem + C::kLsum) + g * 4 * 32;    // [4][32]
      const uint32_t bar_id = kBarGroup0 + g;
      // Scores are scaled by cs >= 0 (log2 domain); a negative scale is an
      // exact sign flip of every score, taken as the score is read.
      const float cs = fabsf(p.scale_log2);
      const float sgn = p.scale_log2 < 0.f ? -1.f : 1.f;
      constexpr int kSG = C::kSG;

      float lpart[RW], bias[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        lpart[r] = 0.f;
        bias[r] = INFINITY;
      }
      float m_lane = -INFINITY;  // reference max (raw score) of row row0 + lane % RW
      int seg_cur = -1, seg_rows = 0, seg_L = 0, seg_h = 0, lo_all = 0, hi_all = -1;
      uint32_t all_rows = 0, part_rows_mask = 0;
      bool ok = true;
      int o_seen = 0;  // PV phases known to be complete
      // Wait until PV(k) has finished: exact while phases < k are complete
      // and phase k + 1 cannot be (P(k+1) not yet published).
      auto wait_o_done = [&](int k) -> bool {
        if (o_seen > k) return true;
        if (!wait(BAR_OFULL, k & 1)) return false;
        o_seen = k + 1;
        return true;
      };
      // int8 caches: K's scales of this thread's key (q8_0: four fp16 group
      // scales; int8 rows: the fp32 row scale), read from the cache (an L2
      // hit: the K producer prefetched them) one tile ahead; zero for a key
      // that is not copied.
      auto fetch_scales = [&](int u) -> uint2 {
        uint2 sc = make_uint2(0, 0);
        if constexpr (kQuant) {
          const TileInfo& ti = info[u % kInfoSlots];
          const int key = ti.key0 + j;
          const int tix = ti.row8[j / kChunk];
          if (tix >= 0 && key >= ti.vis_lo && key <= ti.vis_hi) {
            const long long off = (long long)tix * quant_tile_bytes(KV, p.block_size) +
                                  (long long)p.block_size * kHeadDim +
                                  (long long)(key % p.block_size) * kScaleBytes;
            const uint8_t* src = static_cast<const uint8_t*>(p.k) + off;
            if constexpr (kQ8) sc = ldg_nc_v2(src);
            else sc.x = ldg_nc_u32(src);
          }
        }
        return sc;
      };
      auto info_wait = [&](int u) -> bool {
        int r = 1;
        if (lane == 0) r = wait(BAR_INFO + u % kInfoSlots, (u / kInfoSlots) & 1);
        r = __shfl_sync(0xffffffffu, r, 0);
        __syncwarp();
        return r != 0;
      };
      int* pend = reinterpret_cast<int*>(smem + C::kPend) + g * kPendLen * 3;
      int npend = 0, pend_last = -1;
      // Count the listed partials in (the warpgroup's leader, after a barrier
      // that follows every thread's stores).  Mode 0 arrives with a release
      // reduction, which publishes the warpgroup's stores (ordered before it
      // by the barrier); mode 1's arrivals return a value: a fence first.
      auto flush = [&]() {
        if (widx == 0 && lane == 0 && npend > 0) {
          if (p.mode != 0) __threadfence();
          for (int i = 0; i < npend; ++i) {
            const int* pe = pend + i * 3;
            if (arrive(p, pe[0], pe[1], pe[2] != 0, 1)) {
              const int k = atomicAdd(&misc->n_merge, 1);  // complete: merge it at the end
              if (k < kMergeListLen) merge_list[k] = pe[0];
            }
          }
          misc->segs_done[g] = pend_last + 1;
        }
        npend = 0;
      };
      uint2 sc_next = make_uint2(0, 0);
      bool next_known = false;  // INFO(t) already waited for (scale prefetch)
      // fp16 without the trace: a tile's description is read only at the
      // first tile of a segment; the others follow from the segment's.
      constexpr bool kSegDriven = !kQuant && !TR;
      int seg_left = 0, seg_key = 0, seg_vlo = 1, seg_vhi = 0;
      for (int t = 0;; ++t) {
        // This warp's view of tile t: live unless the stream ended or a wait
        // gave up.  The warpgroup learns at its one barrier per tile (below)
        // whether any warp is not live, and then stops together.
        const TileInfo& ti = info[t % kInfoSlots];
        bool live;
        int seg, flags, key0, vlo, vhi;
        if (kSegDriven && seg_left > 0) {
          live = ok;
          seg = seg_cur;
          flags = seg_left == 1 ? 2 : 0;
          key0 = seg_key;
          vlo = seg_vlo;
          vhi = seg_vhi;
        } else {
          live = ok && (next_known || info_wait(t));
          live = live && ti.seg >= 0;
          seg = live ? ti.seg : 0;
          flags = live ? ti.flags : 0;
          key0 = ti.key0;
          vlo = live ? ti.vis_lo : 1;
          vhi = live ? ti.vis_hi : 0;
        }
        ok = ok && live;
        const int sb = t % 2, st = t % VS, ob = seg % 2;
        if (live && seg != seg_cur) {
          // A new segment: its rows, its context and a fresh softmax state.
          const SegInfo& si = seginfo[seg % kSegSlots];
          seg_cur = seg;
          seg_rows = si.rows;
          seg_L = si.L;
          seg_h = si.h;
          seg_left = si.ntile;
          seg_key = si.key_first;
          seg_vlo = si.vis_lo;
          seg_vhi = si.vis_hi;
          const int vr = min(RW, max(0, seg_rows - row0));
          all_rows = vr >= 32 ? 0xffffffffu : ((1u << vr) - 1u);
          part_rows_mask = seg_rows >= 32 ? 0xffffffffu : ((1u << seg_rows) - 1u);
          // The keys every row of the part sees (tokens i_first .. i_last):
          // [lo_all, hi_all], where the row mask is the whole part.
          {
            const int off = seg_h * p.rows_half;
            const int i_first = off / p.group, i_last = (off + seg_rows - 1) / p.group;
            const int p0 = seg_L - p.n_query;
            if (p.causal) {
              lo_all = p.window > 0 ? max(0, p0 + i_last - p.window + 1) : 0;
              hi_all = min(seg_L - 1, p0 + i_first);
            } else {
              lo_all = p.window > 0 ? max(0, seg_L - p.window) : 0;
              hi_all = seg_L - 1;
            }
          }
          m_lane = -INFINITY;
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            lpart[r] = 0.f;
            bias[r] = INFINITY;  // no reference yet: the row's first key forces one
          }
        }
        uint2 sc = make_uint2(0, 0);
        if constexpr (kQuant) {
          if (live) {
            sc = next_known ? sc_next : fetch_scales(t);
            next_known = false;
            if (info_wait(t + 1)) {  // prefetch the next tile's scales
              next_known = true;
              if (info[(t + 1) % kInfoSlots].seg >= 0) sc_next = fetch_scales(t + 1);
            } else {
              ok = false;
            }
          }
        }
        float sv[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) sv[r] = 0.f;
        ok = __all_sync(0xffffffffu, ok && wait(BAR_SFULL + sb, (t / 2) & 1));
        if (ok) {
          tc_fence_after();
          if constexpr (kQ8) {
            // Score = sum over the scale groups of K's scale times the
            // group's partial product (fp32, groups in order).
            float sg[kSG][RW];
#pragma unroll
            for (int q = 0; q < kSG; ++q) tmem_ld<RW>(tmem + lane_off + sb * kSG * NR + q * NR + row0, sg[q]);
            tmem_ld_wait();
            const uint32_t kw[2] = {sc.x, sc.y};
#pragma unroll
            for (int q = 0; q < kSG; ++q) {
              const float dk = sgn * __half2float(__ushort_as_half((uint16_t)(kw[q / 2] >> (16 * (q % 2)))));
#pragma unroll
              for (int r = 0; r < RW; ++r) sv[r] = q == 0 ? dk * sg[0][r] : fmaf(dk, sg[q][r], sv[r]);
            }
          } else {
            tmem_ld<RW>(tmem + lane_off + sb * NR + row0, sv);
            tmem_ld_wait();
            if constexpr (kQuant) {  // int8 rows: K's row scale
              const float dk = sgn * __uint_as_float(sc.x);
#pragma unroll
              for (int r = 0; r < RW; ++r) sv[r] *= dk;
            } else if (sgn < 0.f) {
#pragma unroll
              for (int r = 0; r < RW; ++r) sv[r] = -sv[r];
            }
          }
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(BAR_SEMPTY + sb));

        // Which rows of the part see this key: the tokens that see it form a
        // contiguous run, whose rows are a contiguous run of bits.
        const int key = key0 + j;
        uint32_t rmask = 0;
        if (ok && key >= vlo && key <= vhi && key >= lo_all && key <= hi_all) {
          rmask = part_rows_mask;  // the interior: every row of the part
        } else if (ok && key >= vlo && key <= vhi) {
          int i_lo, i_hi;
          tokens_seeing(seg_L, p.n_query, p.causal, p.window, key, i_lo, i_hi);
          const int off = seg_h * p.rows_half;
          const int b = min(max(i_lo * p.group - off, 0), seg_rows);
          const int e = min(max((i_hi + 1) * p.group - off, 0), seg_rows);
          if (e > b) rmask = (e >= 32 ? 0xffffffffu : ((1u << e) - 1u)) & ~((1u << b) - 1u);
        }
        const uint32_t rm_g = rmask >> row0;  // this warpgroup's rows
        const bool all_vis = __all_sync(0xffffffffu, all_rows != 0 && (rm_g & all_rows) == all_rows);
        if constexpr (TR) {
          // Key-resolution record: every (row, key) pair this kernel scores,
          // with the physical slot its K row was copied from.
          if (ok && rm_g != 0) {
            const int row8 = ti.row8[j / kChunk];
            long long phys;
            if constexpr (kQuant) {
              phys = row8 / Hkv;
            } else {
              const long long row = (long long)row8 * 8 + (key % kChunk);
              phys = row / p.block_size / Hkv;
            }
            const unsigned id = (unsigned)(phys * p.block_size + key % p.block_size);
            const SegInfo& si = seginfo[seg % kSegSlots];
#pragma unroll
            for (int r = 0; r < RW; ++r) {
              if ((rm_g >> r) & 1u) {
                int32_t* tr = p.trace + out_row(p, si.s, si.kvh, si.h, row0 + r) * 5;
                atomicAdd(tr + 0, 1);
                atomicMin(tr + 1, key);
                atomicMax(tr + 2, key);
                atomicXor(reinterpret_cast<unsigned*>(tr + 3), id);
                atomicAdd(reinterpret_cast<unsigned*>(tr + 4), id);
              }
            }
          }
        }
        // x = cs * s + bias, the log2 of the scaled weight; -inf for a row
        // that does not see this key: its weight is exactly 0 and it cannot
        // raise the row's reference.
        float x[RW];
        float xmax = -INFINITY;
        if (all_vis) {
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            x[r] = fmaf(sv[r], cs, bias[r]);
            xmax = fmaxf(xmax, x[r]);
          }
        } else {
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            x[r] = ((rm_g >> r) & 1u) ? fmaf(sv[r], cs, bias[r]) : -INFINITY;
            xmax = fmaxf(xmax, x[r]);
          }
        }
        const bool exceed = xmax > (float)kPShift + kLazy;
        // Reconverge before the group barrier (a diverged arrival makes the
        // barrier several times slower).
        __syncwarp();
        // One barrier per tile: orders the group's shared-memory traffic and
        // counts the threads that are not live or saw a score pass their
        // row's reference; only then (rarely) a second one tells the two
        // apart, so that the whole warpgroup leaves the loop together.
        const uint32_t flagged = named_bar_popc(bar_id, kSoftmaxThreads, !live || exceed);
        if (flagged != 0 && named_bar_or(bar_id, kSoftmaxThreads, !live)) break;
        const bool rescale = flagged != 0;
        if (rescale) {
          const uint32_t rm = all_vis ? 0xffffffffu : rm_g;
          float tmp[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) tmp[r] = ((rm >> r) & 1u) ? sv[r] : -INFINITY;
          const float wmax = warp_row_reduce<RW, true>(tmp, lane);
          if (lane < RW) red[(sb * 4 + widx) * 32 + lane] = wmax;
          __syncwarp();
          named_bar_sync(bar_id, kSoftmaxThreads);
          const int rl = lane % RW;
          float tmax = red[(sb * 4 + 0) * 32 + rl];
          tmax = fmaxf(tmax, red[(sb * 4 + 1) * 32 + rl]);
          tmax = fmaxf(tmax, red[(sb * 4 + 2) * 32 + rl]);
          tmax = fmaxf(tmax, red[(sb * 4 + 3) * 32 + rl]);
          const float m_new = fmaxf(m_lane, tmax);
          // alpha = 2^(cs (m_old - m_new)); bias makes 2^(cs s + bias) =
          // 2^(cs (s - m_new) + kPShift).
          const float alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(cs * (m_lane - m_new));
          const float bias_l = (m_new == -INFINITY) ? INFINITY : fmaf(-cs, m_new, (float)kPShift);
          m_lane = m_new;
          float av[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            bias[r] = __shfl_sync(0xffffffffu, bias_l, r);
            av[r] = __shfl_sync(0xffffffffu, alpha, r);
            x[r] = ((rm >> r) & 1u) ? fmaf(sv[r], cs, bias[r]) : -INFINITY;
            lpart[r] *= av[r];
          }
          if (!(flags & 1)) {  // rescale this segment's accumulated O columns
            ok = __all_sync(0xffffffffu, ok && wait_o_done(t - 1));
            if (ok) {
              tc_fence_after();
              const uint32_t o_hi = tmem + lane_off + C::kTmemS + ob * C::kTmemO + row0;
              float oh[RW], ol[RW];
              tmem_ld<RW>(o_hi, oh);
              tmem_ld<RW>(o_hi + NR, ol);
              tmem_ld_wait();
#pragma unroll
              for (int r = 0; r < RW; ++r) {
                oh[r] *= av[r];
                ol[r] *= av[r];
              }
              tmem_st<RW>(o_hi, oh);
              tmem_st<RW>(o_hi + NR, ol);
              tmem_st_wait();
              tc_fence_before();  // ordered before the PFULL arrive below
            }
          }
        }

        // Scaled weights (2^-inf = 0 for keys a row does not see).
        float pw[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          pw[r] = fast_exp2(x[r]);
          lpart[r] += pw[r];
        }

        // fp16 cache: a key no row of the part sees must not reach the PV
        // product: zero its V row once the V tile has landed (the int8
        // converters write such rows as zeros themselves).
        if (!kQuant && g == 0 && !all_vis && __any_sync(0xffffffffu, ok && rmask == 0)) {
          ok = __all_sync(0xffffffffu, ok && wait(BAR_VFULL + st, (t / VS) & 1));
          if (ok && rmask == 0) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            const uint32_t vrow = sV + st * C::kVSlot + (j / 8) * kGroupBytes + (j % 8) * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              sts_v4(vrow + cc * 16, z);
              sts_v4(vrow + kAtomBytes + cc * 16, z);
            }
          }
        }
        // A segment's last P goes out only after PV(t-1), so that the wait
        // for PV(t) below is for one phase only.
        if ((flags & 2) && t > 0) {
          ok = __all_sync(0xffffffffu, ok && wait_o_done(t - 1));
          if (ok) tc_fence_after();
        }
        if (ok) {
          // P^T as no-swizzle MN-major core matrices [key/8][n/8][key%8][n%8]:
          // n < NR the high parts of the rows, n >= NR their residuals.  Each
          // weight is split into an fp16 high part (truncated to 11
          // significant bits) and a residual.
          const uint32_t kb = (j >> 3) * (C::kPN / 8) * 128 + (j & 7) * 16;
          constexpr uint32_t lo_off = (NR / 8) * 128;
          const uint32_t pbuf = sP + (t % PB) * C::kPBytes;
          uint32_t phi[RW / 2], plo[RW / 2];
#pragma unroll
          for (int r = 0; r < RW; r += 2) {
            const float h0 = __uint_as_float(__float_as_uint(pw[r]) & 0xffffe000u);
            const float h1 = __uint_as_float(__float_as_uint(pw[r + 1]) & 0xffffe000u);
            phi[r / 2] = h2_bits(__floats2half2_rn(h0, h1));
            plo[r / 2] = h2_bits(__floats2half2_rn(pw[r] - h0, pw[r + 1] - h1));
          }
          if constexpr (RW >= 8) {
#pragma unroll
            for (int r8 = 0; r8 < RW / 8; ++r8) {
              const uint32_t off = kb + ((row0 / 8) + r8) * 128;
              sts_v4(pbuf + off, make_uint4(phi[r8 * 4], phi[r8 * 4 + 1], phi[r8 * 4 + 2], phi[r8 * 4 + 3]));
              sts_v4(pbuf + lo_off + off,
                     make_uint4(plo[r8 * 4], plo[r8 * 4 + 1], plo[r8 * 4 + 2], plo[r8 * 4 + 3]));
            }
          } else {  // four rows: half of one 16-byte core-matrix row
            const uint32_t off = kb + (row0 / 8) * 128 + (row0 % 8) * 2;
            sts_v2(pbuf + off, phi[0], phi[1]);
            sts_v2(pbuf + lo_off + off, plo[0], plo[1]);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(BAR_PFULL + t % PB));

        if (flags & 2) {
          // ---- the segment's partial: O once PV(t) has finished ------------
          const SegInfo& si = seginfo[seg % kSegSlots];
          float acc[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) acc[r] = 0.f;
          ok = __all_sync(0xffffffffu, ok && wait_o_done(t));
          if (ok) {
            tc_fence_after();
            const uint32_t o_hi = tmem + lane_off + C::kTmemS + ob * C::kTmemO + row0;
            float oh[RW], ol[RW];
            tmem_ld<RW>(o_hi, oh);
            tmem_ld<RW>(o_hi + NR, ol);
            tmem_ld_wait();
#pragma unroll
            for (int r = 0; r < RW; ++r) acc[r] = oh[r] + ol[r];
            tc_fence_before();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(BAR_OEMPTY + ob));  // the accumulator may be reused
          // Row sums: per-thread partials -> per warp (lane r) -> across warps.
          float lp[RW];
#pragma unroll
          for (int r = 0; r < RW; ++r) lp[r] = lpart[r];
          const float wsum = warp_row_reduce<RW, false>(lp, lane);
          if (lane < RW) lsum[widx * 32 + lane] = wsum;
          __syncwarp();
          named_bar_sync(bar_id, kSoftmaxThreads);
          const bool bad = si.bad != 0;
          const long long pbase = (long long)si.slot * p.rows_half;
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            if (row0 + r < seg_rows) {
              const float l = lsum[r] + lsum[32 + r] + lsum[64 + r] + lsum[96 + r];
              p.part_out[(pbase + row0 + r) * kHeadDim + j] = (ok && !bad && l > 0.f) ? acc[r] / l : 0.f;
            }
          }
          if (widx == 0 && lane < RW && row0 + lane < seg_rows) {
            // lse = ln sum_j e^{z_j}: log2 sum_j 2^{cs s_j} = log2 l' + cs m - kPShift.
            // NaN marks a partial that must not be used (a stand-in block, a timeout).
            const float l = lsum[lane] + lsum[32 + lane] + lsum[64 + lane] + lsum[96 + lane];
            p.part_lse[pbase + row0 + lane] =
                (bad || !ok) ? __uint_as_float(kInvalidLse)
                : l > 0.f ? (fmaf(cs, m_lane, -(float)kPShift) + log2f(l)) * 0.69314718055994531f
                          : -INFINITY;
          }
          // Counted in later: a fence here would wait for these stores to
          // drain behind the stream.  The warpgroup's barriers order every
          // thread's stores before the leader's fence at the flush.
          if (widx == 0 && lane == 0) {
            int* pe = pend + npend * 3;
            pe[0] = si.group;
            pe[1] = si.expect;
            pe[2] = (si.first && g == 0) ? 1 : 0;
          }
          ++npend;
          pend_last = seg;
          if (npend == kPendLen) {
            named_bar_sync(bar_id, kSoftmaxThreads);
            flush();
          }
        }
        --seg_left;
        seg_key += kTileKeys;
      }
      flush();          // the loop's exit barrier ordered the last stores
      __syncthreads();  // (A)
    }
    // ---- tear-down (every thread passed (A)) ---------------------------------
    tc_fence_after();
    if (warp == 1) {
      __syncwarp();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  }

  // ---- unfinished segments, abort flag, merges ---------------------------------
  __syncthreads();  // (B) partials written, copies drained, TMEM freed
  if (threadIdx.x == 0) {
    if (misc->abort) atomicOr(p.flags, kFlagTimeout);
    // Segments published but not counted in by a softmax warpgroup (abort
    // path): an invalid partial, counted in for that warpgroup.
    for (int g = 0; g < NG; ++g) {
      for (int sg = misc->segs_done[g]; sg < misc->segs_published; ++sg) {
        const SegInfo& si = seginfo[sg % kSegSlots];
        for (int r = 0; r < si.rows; ++r)
          p.part_lse[(long long)si.slot * p.rows_half + r] = __uint_as_float(kInvalidLse);
        __threadfence();
        if (arrive(p, si.group, si.expect, si.first && g == 0, 1)) {
          const int i = atomicAdd(&misc->n_merge, 1);
          if (i < kMergeListLen) merge_list[i] = si.group;
        }
      }
    }
  }
  __syncthreads();
  if (p.mode == 0) {
    // The CTAs whose range ends in a KV head merge its partials, each a
    // share, once all of the head's partials are in (a bounded wait on the
    // group's barrier: every CTA of the grid is resident).
    if (misc->own_group < 0) return;
    if (threadIdx.x == 0) {
      const int grp = (misc->own_s * Hkv + misc->own_group) * H + misc->own_h;
      const int* cnt = group_counter(p, grp);
      const unsigned phase = (unsigned)misc->own_phase;
      const unsigned long long t0 = globaltimer();
      int ok = 1;
      while (((unsigned)ld_acquire_gpu(cnt) & 0x80000000u) == phase) {
        if (globaltimer() - t0 > p.wait_limit_ns) {
          ok = 0;
          break;
        }
      }
      misc->last = ok;
      if (!ok) atomicOr(p.flags, kFlagTimeout);
    }
    __syncthreads();
    if (!misc->last) return;
    const int P = misc->own_rows * (kHeadDim / 4);
    const int sl = misc->own_slice, ns = misc->own_slices;
    const int pa = sl * P / ns, pb = (sl + 1) * P / ns;  // P <= 64 * 32, sl < 4096: no overflow
    const long long slot0 = (long long)(misc->own_s * H + misc->own_h) * (p.ctas_per_set + Hkv) +
                            misc->own_first + misc->own_group;
    merge_pairs<kThreads>(p, slot0, misc->own_count, misc->own_rows, misc->own_s, misc->own_group,
                          misc->own_h, pa, pb, smem, sbase, C::kRed);
  } else {
    // Groups this CTA completed: merge each, whole.
    const int n = min(misc->n_merge, kMergeListLen);
    if (n > 0) __threadfence();  // the other CTAs' partials, published before their counts
    for (int i = 0; i < n; ++i) {
      const int grp = merge_list[i];
      const int h = grp % H, kvh = (grp / H) % Hkv, s = grp / (H * Hkv);
      const int L = ld_nc_s32(p.context_lens + s);
      int nb, ns;
      seq_items(seq_vis(p, s, L).nch, p.item_tiles, nb, ns);
      const int rows = part_rows(p, h);
      merge_pairs<kThreads>(p, (long long)grp * p.slots_per_group, nb + ns, rows, s, kvh, h, 0,
                            rows * (kHeadDim / 4), smem, sbase, C::kRed);
    }
  }
}

// ---- host side ----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};
  PFN_cuTensorMapEncodeTiled_v12000 f = fn.load(std::memory_order_acquire);
  if (f == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
      fn.store(f, std::memory_order_release);
    }
  }
  return f;
}

// The fp16 cache viewed as a 4-D tensor {64 columns, 8 rows, 2 halves,
// rows/8 groups} (row = one key of one KV head, 256 bytes): one box
// {64, 8, 2, 2} is a 16-row chunk, stored in shared memory as
// [group][half][8 rows][64 columns] with the 128-byte swizzle the tcgen05
// descriptors expect.
bool encode_cache_map(CUtensorMap* m, const void* cache, long long rows) {
  auto fn = encode_fn();
  if (fn == nullptr || rows % 8 != 0) return false;
  cuuint64_t dims[4] = {64, 8, 2, (cuuint64_t)(rows / 8)};
  cuuint64_t strides[3] = {(cuuint64_t)kHeadDim * 2, 128, 8 * (cuuint64_t)kHeadDim * 2};
  cuuint32_t box[4] = {64, 8, 2, 2};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(cache), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kMaxDevices = 64;

template <int RW, int NG, int KV, bool TR>
cudaError_t launch_cfg(DecodeParams p, const CUtensorMap& mk, const CUtensorMap& mv,
                       cudaStream_t stream) {
  using Cf = Cfg<RW, NG, KV>;
  auto kern = decode_tc_kernel<RW, NG, KV, TR>;
  const size_t smem = Cf::kTotal + 1024;
  // CTAs of this kernel the device holds at once (0: not yet known).
  static std::atomic<int> resident[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  int res = resident[dev].load(std::memory_order_acquire);
  if (res == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cf::kThreads, smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    res = per_sm * sms;
    if (res <= 0) return cudaErrorInvalidConfiguration;
    resident[dev].store(res, std::memory_order_release);
  }
  // Mode 0 waits on other CTAs: every CTA must be resident at once, which a
  // cooperative launch guarantees; the plan never asks for more CTAs than
  // the device holds.
  if (p.num_ctas > res) return cudaErrorCooperativeLaunchTooLarge;
  p.coop = p.mode == 0 ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_ctas);
  cfg.blockDim = dim3(Cf::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.coop ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, mk, mv, p);
}

template <bool TR>
cudaError_t launch_any(const DecodeParams& p, cudaStream_t stream) {
  if (p.kv_dtype != kKvFp16) {
    // Raw int8 tiles arrive by untiled bulk copies: no tensor maps.
    CUtensorMap none;
    memset(&none, 0, sizeof(none));
    if (p.kv_dtype == kKvQ8_0) {
      if (p.rows_half <= 8) return launch_cfg<4, 2, kKvQ8_0, TR>(p, none, none, stream);
      return launch_cfg<8, 2, kKvQ8_0, TR>(p, none, none, stream);
    }
    if (p.rows_half <= 8) return launch_cfg<4, 2, kKvInt8Row, TR>(p, none, none, stream);
    return launch_cfg<8, 2, kKvInt8Row, TR>(p, none, none, stream);
  }
  CUtensorMap mk, mv;
  const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
  if (!encode_cache_map(&mk, p.k, rows) || !encode_cache_map(&mv, p.v, rows))
    return cudaErrorInvalidValue;
  if (p.rows_half <= 8) return launch_cfg<4, 2, kKvFp16, TR>(p, mk, mv, stream);
  if (p.rows_half <= 16) return launch_cfg<8, 2, kKvFp16, TR>(p, mk, mv, stream);
  return launch_cfg<16, 2, kKvFp16, TR>(p, mk, mv, stream);
}

}  // namespace

int max_rows_per_part(int kv_dtype) { return kv_dtype == kKvFp16 ? 32 : 16; }

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream) {
  return p.trace != nullptr ? launch_any<true>(p, stream) : launch_any<false>(p, stream);
}

}  // namespace pa
