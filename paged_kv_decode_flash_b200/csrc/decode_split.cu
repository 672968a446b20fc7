// decode_split.cu -- the per-head split kernel: split-KV paged decode
// attention on the sm_100a tensor cores (tcgen05 + TMEM), with TMA staging of
// the paged KV tiles, for an fp16 cache with few (sequence, KV head) groups
// (batch 1 typically), up to 8 query tokens and up to 32 query rows per KV
// head.  Every other call (int8 caches, more rows, batches, the key ranges of
// context-parallel shares) runs the segment kernel of decode_tc.cu.  This
// file's kernel is instantiated for the fp16 cache only (its int8 paths are
// not built into the library).
//
// What it computes is the decode step of "Dual MI50, part 2: from 10 to 74
// tokens/s, a 200k-token context, and two attention kernels" (sbm-labs
// blog), section "Decode: a new kernel for the shape MTP actually runs": all
// query rows that share one KV head (n_query tokens x the query heads of the
// group) are scored against the same keys, the context is split so that
// every SM is busy at batch 1, and one fp32 partial (O, lse) per split is
// left for the log-sum-exp merge.  Masks and block-table resolution follow
// section "Bug 2: the drafter read freed memory".
//
// Hardware mapping (one CTA per SM, 11 warps; 19 for the q8_0 cache):
//   warps 0, 10 TMA producers for K and for V: resolve the block table and
//               load whole 16-key chunks into separate rings of 128-key tiles
//               (fp16: 4-D boxes of two 64-column halves with the 128-byte
//               swizzle, 2-3 slots; q8_0: untiled bulk copies of the raw
//               chunk into the upper half of a slot, 2 K and 3 V slots).  K
//               slots are released as soon as QK^T has read them, so K runs
//               ahead.  With each K copy the same chunk of V is prefetched
//               into L2, so that V's own copy a tile later is short.
//   warp 1      MMA issuer (one thread), fixed order QK(0), QK(1), then
//               PV(t), QK(t+2): S^T = K Q^T with M = 128 keys and N = the
//               query rows (double-buffered in TMEM), O^T += V^T
//               [P_hi | P_lo]^T with M = 128 head_dim lanes (one TMEM
//               accumulator over all tiles); P is double-buffered in shared
//               memory (fp16) so that the softmax of tile t+1 overlaps PV(t).
//   warps 2-9   two softmax warpgroups, each owning half of the query rows:
//               thread = key for S (row max by a warp transpose-reduction
//               plus one named barrier per group); when a row's reference
//               maximum rises, its O column is rescaled in TMEM in place
//               (thread = head_dim lane) before the tile's P is published.
//   warps 11-18 (q8_0 cache only) converters, four for K and four for V:
//               each raw int8 tile is expanded in place into its exact fp16
//               operand tile (see below).
// Putting keys and head_dim on the MMA's M side keeps the tensor core free of
// padding even at 4-32 query rows.
//
// Exactness: Q, K and V are fed to the tensor core as the exact fp16 inputs.
// The softmax weights are scaled by 2^14 (2^13 for q8_0, so that weights
// down to ~4e-12 of the row maximum stay representable) and split into an fp16 high part and
// an fp16 residual; both are multiplied with V and accumulated in fp32, which
// keeps the weights to about 2^-22 relative.  Keys no query row can see are
// never multiplied: their chunks are not loaded when wholly outside the
// visible range, their scores are selected to -inf, and their V rows are
// zero-filled in shared memory before the PV product (the NaN-poisoned
// out-of-window blocks of the pages' regression test must not leak).
//
// The template keeps a q8_0 variant (scales kept out of the operands: K's
// applied to the per-group scores, V's power of two folded into the operand
// and its mantissa into one P copy per scale group), which the library does
// not instantiate: int8 caches run the segment kernel (decode_tc.cu).
// (The kernel can also cut every group's tiles into fixed-size items, one CTA
// each, over several waves; the library uses it only with few groups, one
// wave, where each group's CTAs take contiguous runs of its tiles.)
//
// Merge: every CTA writes its fp32 partial (O, lse).  With a cooperative
// launch (every CTA resident) the CTAs of one (sequence, KV head) meet at a
// bounded counter barrier and each merges a slice of the group's rows;
// otherwise the last CTA of the group to arrive merges all of it.  Splits
// are added in a fixed order (log-sum-exp weights), so results are
// bit-reproducible.  A call is one launch.
//
// Every wait is bounded (sm100::mbar_wait and the group barrier): on a
// timeout the kernel raises kFlagTimeout, drains its own copies and MMAs,
// frees TMEM and still takes part in the merge (its rows count as empty).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "split_common.cuh"
#include "sm100.cuh"

namespace pa {
namespace split {
namespace {

using namespace sm100;

constexpr int kTileKeys = 128;                 // keys per pipeline tile (M of S^T)
constexpr int kChunksPerTile = kTileKeys / kChunk;
constexpr int kMaxStages = 3;                  // slots per K ring and per V ring (at most)
// A K or V tile of 128 keys in shared memory: [key group of 8][half][8 keys]
// [64 fp16] with the 128-byte swizzle, i.e. 1 KB swizzle atoms; the atoms of
// one 64-column half sit 2 KB apart, the two halves of a key group 1 KB apart.
// One 16-key chunk (a contiguous 4 KB (block, head) tile in the cache for
// block_size 16) is a single TMA box.
constexpr uint32_t kAtomBytes = 1024;              // 8 keys x 128 bytes
constexpr uint32_t kGroupBytes = 2 * kAtomBytes;   // both halves of 8 keys
constexpr uint32_t kKVBytes = kTileKeys / 8 * kGroupBytes;  // one K (or V) tile
constexpr uint32_t kChunkBytes = kChunk * 256;     // one 16-key chunk (TMA box)
// q8_0: a raw 128-key tile in shared memory is qs [128 keys][128 int8] then
// d [128 keys][4 fp16]; a 16-key chunk arrives as two bulk copies (2048 B of
// qs, 128 B of scales).
constexpr uint32_t kRawOff = kKVBytes / 2;          // q8_0: raw qs in the slot's upper half
constexpr uint32_t kQ8QsChunk = kChunk * kHeadDim;    // 2048 B of qs per 16-key chunk
constexpr uint32_t kQ8DChunk = kChunk * 8;            // 128 B of scales per 16-key chunk
constexpr int kSoftmaxThreads = 128;           // per softmax warpgroup
constexpr uint32_t kBarSetup = 1;              // named barrier: set-up done
constexpr uint32_t kBarGroup0 = 2;             // named barriers 2, 3: softmax groups
constexpr uint32_t kBarConv0 = 4;              // named barriers 4, 5: q8_0 K / V converters
// A row's reference max is only raised when a score passes it by more than
// kLazy (log2 units); weights scaled by 2^kPShift (see Cfg) then stay below
// 2^(kPShift + kLazy), inside fp16 range.
constexpr float kLazy = 1.5f;

enum : int {
  BAR_KFULL = 0,    // [3] K tile landed
  BAR_KEMPTY = 3,   // [3] K tile read by QK^T
  BAR_VFULL = 6,    // [3] V tile landed
  BAR_VEMPTY = 9,   // [3] V tile read by PV
  BAR_SFULL = 12,   // [2] S^T in TMEM
  BAR_SEMPTY = 14,  // [2] S^T read by the softmax warps
  BAR_PFULL = 16,   // [2] P of one tile written to shared memory
  BAR_OFULL = 18,   // PV of one more tile accumulated into O^T
  BAR_DONE = 22,    // every MMA finished
  BAR_INFO = 23,    // [8] a tile's number, chunk mask and cache rows published
  BAR_CKFULL = 31,  // [3] q8_0: K slot converted to fp16
  BAR_CVFULL = 34,  // [3] q8_0: V slot converted to fp16
  BAR_COUNT = 37
};
constexpr int kBarSlots = 40;
constexpr int kInfoSlots = 8;  // depth of the tile-information ring

// NG softmax warpgroups of RW query rows each; NR = the MMA's N for S
// (>= 16).  Warps: 0 K producer, 1 MMA issuer, 2 .. 4*NG+1 softmax, then the
// V producer (and, q8_0 only, four converter warps).
// KS / VS slots in the K / V rings, PB buffers for P.  fp16: two P buffers,
// so that the softmax of tile t+1 never waits for PV(t); at 32 rows they take
// 32 KB and the V ring keeps two slots (measured: three V slots with one P
// buffer is slower).  q8_0: a slot is the fp16 operand tile; the raw int8
// tile lands in its upper half and the converters expand it in place (a V
// slot also keeps the raw scales after the tile); two K slots, three V
// slots, one P buffer that holds a P per scale group (the softmax of tile t
// waits for PV(t-1) before it stores P(t)).
template <int RW, int NG, bool Q8>
struct Cfg {
  static constexpr int kGroups = NG;
  static constexpr int kVWarp = 2 + NG * 4;      // the V producer's warp
  static constexpr int kConvWarp = kVWarp + 1;   // q8_0: first converter warp
  static constexpr int kConvWarps = 4;           // q8_0: converter warps per stream (K, V)
  static constexpr int kThreads = 32 * (kVWarp + 1 + (Q8 ? 2 * kConvWarps : 0));
  static constexpr int NR = (kGroups * RW < 16) ? 16 : kGroups * RW;
  // q8_0: one S^T accumulator, one P and one O^T accumulator per group of 32
  // head_dim elements that shares a scale; fp16: one of each.
  static constexpr int kSG = Q8 ? kHeadDim / 32 : 1;
  static constexpr int KS = Q8 ? 2 : 3;
  static constexpr int VS = Q8 ? 3 : (NR > 16 ? 2 : 3);
  static constexpr int PB = Q8 ? 1 : 2;  // q8_0 measured: two V slots and two P buffers are slower
  // Weights are scaled by 2^kPShift before they are split into fp16 parts.
  // q8_0 multiplies them by a scale mantissa in [1, 2) as well, so it keeps
  // one bit of headroom more.
  static constexpr int kPShift = Q8 ? 13 : 14;
  static constexpr uint32_t kKSlot = kKVBytes;                           // K slot
  static constexpr uint32_t kVSlot = kKVBytes + (Q8 ? kTileKeys * 8 : 0);  // V slot (+ scales)
  static constexpr uint32_t kK = 0;                                      // K ring
  static constexpr uint32_t kV = KS * kKSlot;                            // V ring
  static constexpr uint32_t kQ = kV + VS * kVSlot;
  static constexpr uint32_t kQHalf = NR * 128;
  // P^T of one tile: per scale group 2*NR "rows" (the fp16 high parts of the
  // NR query rows, then their residuals), the groups side by side, so that
  // one MMA with N = kSG * 2 * NR multiplies all of them with each V step
  // (V is read once).  Tile t uses buffer t % PB.
  static constexpr int kPN = kSG * 2 * NR;  // N of the PV product
  static constexpr uint32_t kP = kQ + 2 * kQHalf;
  static constexpr uint32_t kPBytes = kTileKeys * kPN * 2;
  static constexpr uint32_t kRed = kP + PB * kPBytes;               // float [2 grp][2][4][32]
  static constexpr uint32_t kAlpha = kRed + kGroups * 2 * 4 * 32 * 4;  // float [4 tiles][32 rows]
  static constexpr uint32_t kLsum = kAlpha + 4 * 32 * 4;            // float [2 grp][4][32]
  static constexpr uint32_t kBcast = kLsum + kGroups * 4 * 32 * 4;  // float [4*NG warps][2][32]
  static constexpr uint32_t kBars = kBcast + kGroups * 4 * 2 * 32 * 4;  // uint64 [kBarSlots]
  static constexpr uint32_t kInfo = kBars + kBarSlots * 8;          // TileInfo [8]
  static constexpr uint32_t kMisc = kInfo + kInfoSlots * 48;        // small ints
  static constexpr uint32_t kTotal = kMisc + 64;
  // TMEM columns: S^T[2] (kSG accumulators of NR columns each), then O^T
  // from column kTmemS (kSG accumulators of 2*NR: high | residual).
  static constexpr uint32_t kTmemS = 2 * kSG * NR;
  static constexpr uint32_t kTmemUsed = kTmemS + kSG * 2 * NR;
  static constexpr uint32_t kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64
                                        : kTmemUsed <= 128 ? 128 : kTmemUsed <= 256 ? 256 : 512;
  static_assert(KS <= kMaxStages && VS <= kMaxStages, "ring depth");
  static_assert(kTotal + 1024 <= 232448, "shared memory per CTA");
  static_assert(kV % 1024 == 0 && kVSlot % 1024 == 0, "tiles sit on 1 KB swizzle atoms");
  static_assert(kTmemUsed <= 512, "TMEM columns");
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int k_consumed, v_consumed;
  int last;  // this CTA arrived last in its (sequence, KV head): it merges
  int bad;   // a block index of this CTA's keys was out of range
};

// What the K producer publishes for each local tile of a CTA: the tile's
// number in the head's key space (-1: no more tiles), which of its 16-key
// chunks were loaded, and each loaded chunk's TMA row coordinate (row / 8).
struct TileInfo {
  int tile;
  uint32_t mask;
  int row8[kChunksPerTile];
  int pad[2];
};
static_assert(sizeof(TileInfo) == 48, "TileInfo layout");

// 32-bit load through the non-coherent path, issued in program order with
// the other volatile loads (so that two independent loads are in flight).
__device__ __forceinline__ int ld_nc_s32(const int* p) {
  int r;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}
__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}
__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
// Shared-memory loads by 32-bit shared address (issued in program order with
// the other volatile shared-memory accesses).
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
__device__ __forceinline__ void sts_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}

// Visible 128-key tiles of a sequence of context length L (0 for a length
// outside [n_query, max_blocks_per_seq * block_size]); also its first key
// rounded down to a 16-key chunk and its visible range.
struct SeqTiles {
  int lo, hi, base, tiles;
};
__device__ __forceinline__ SeqTiles seq_tiles(const DecodeParams& p, int L) {
  SeqTiles t{0, -1, 0, 0};
  if (context_len_ok(L, p.n_query, p.max_blocks_per_seq, p.block_size)) {
    union_range(L, p.n_query, p.causal, p.window, t.lo, t.hi);
    t.base = (t.lo / kChunk) * kChunk;
    if (t.hi >= t.lo) t.tiles = (t.hi + 1 - t.base + kTileKeys - 1) / kTileKeys;
  }
  return t;
}

// Which (sequence, KV head) group CTA c of the C CTAs works for.  Each of the
// G = num_seqs * num_kv_heads groups gets C / G CTAs, as even as whole CTAs
// allow: group g owns CTAs [cum(g), cum(g+1)) with cum(g) = g + floor((C -
// G) g / G), in blockIdx order.  The grid and this mapping depend on the
// shapes alone, never on the context lengths, so a sequence's splits, and
// with them every bit of its output, do not depend on the other sequences
// of the batch.
struct GroupOf {
  int s, kvh, split, splits, first;  // first: the group's first CTA
};
__device__ __forceinline__ GroupOf group_of(const DecodeParams& p, int c, int C) {
  GroupOf r;
  if (p.tiles_per_item > 0) {  // items: num_splits consecutive CTAs per group
    const int g = c / p.num_splits;
    r.s = g / p.num_kv_heads;
    r.kvh = g % p.num_kv_heads;
    r.splits = p.num_splits;
    r.first = g * p.num_splits;
    r.split = c - r.first;
    return r;
  }
  const int G = p.num_seqs * p.num_kv_heads;
  const long long E = (long long)C - G;
  auto cum = [&](int g) { return g + (int)(E * g / G); };
  int g = (int)((long long)c * G / C);
  while (g > 0 && cum(g) > c) --g;
  while (g + 1 < G && cum(g + 1) <= c) ++g;
  r.s = g / p.num_kv_heads;
  r.kvh = g % p.num_kv_heads;
  r.first = cum(g);
  r.splits = cum(g + 1) - r.first;
  r.split = c - r.first;
  return r;
}

// q8_0 cache: byte offset of the qs rows of the 16-key chunk that starts at
// key key0 of (block, head) tile `tile` (tiles are block_size * (128 + 8)
// bytes: qs [block_size][128] then fp16 d [block_size][4]).
__device__ __forceinline__ long long q8_chunk_offset(const DecodeParams& p, int tile, int key0) {
  return (long long)tile * p.block_size * (kHeadDim + 8) + (long long)(key0 % p.block_size) * kHeadDim;
}
// ... and from there to the chunk's scales.
__device__ __forceinline__ long long q8_scale_offset(const DecodeParams& p, int key0) {
  const int slot = key0 % p.block_size;
  return (long long)(p.block_size - slot) * kHeadDim + slot * 8;
}

// ... and of the four scales of one key (slot `slot` of its block) of q8_0
// (block, head) tile `tile`.
__device__ __forceinline__ long long q8_key_scales_offset(const DecodeParams& p, int tile, int slot) {
  return (long long)tile * p.block_size * (kHeadDim + 8) + (long long)p.block_size * kHeadDim +
         (long long)slot * 8;
}

// A q8_0 scale d (fp16 bits) as d = m * 2^e with 2^e the power of two of its
// exponent field (2^-14 for zero and subnormal scales): 2^e as fp16 bits, and
// the factor 2^-e that turns d into m (|m| in [1, 2), below 1 for subnormal
// scales).  Both are exact.
__device__ __forceinline__ uint16_t q8_scale_pow2_bits(uint16_t d) {
  const uint16_t e = d & 0x7C00u;
  return e != 0 ? e : (uint16_t)0x0400u;
}
__device__ __forceinline__ float q8_scale_mantissa(uint16_t d) {
  const int E = max((int)((d >> 10) & 31u), 1);
  return __half2float(__ushort_as_half(d)) * __int_as_float((127 + 15 - E) << 23);
}

// Eight signed bytes -> eight exact fp16 values, two per half2: byte b
// becomes the low mantissa byte of the fp16 1024 + (b + 128) (bits 0x6400 |
// (b ^ 0x80)), minus 1152; every integer below 2048 is exact in fp16.
__device__ __forceinline__ void q8_to_half8(uint2 q, __half2 (&x)[4]) {
  const uint32_t w0 = q.x ^ 0x80808080u, w1 = q.y ^ 0x80808080u;
  const uint32_t u[4] = {__byte_perm(w0, 0x64646464u, 0x5140), __byte_perm(w0, 0x64646464u, 0x7362),
                         __byte_perm(w1, 0x64646464u, 0x5140), __byte_perm(w1, 0x64646464u, 0x7362)};
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));  // 1152
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = __hsub2(*reinterpret_cast<const __half2*>(&u[e]), off);
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

// The last CTA of a (sequence, KV head) merges the group's split partials
// into the output rows: M = max_k lse_k, w_k = exp(lse_k - M) (0 for an
// empty split), out = sum_k w_k O_k / sum_k w_k, splits added in index
// order.  The group's partial rows are staged in shared memory with 16-byte
// asynchronous copies, as many splits per round as fit, all of a round in
// flight at once, so that the merge costs a few memory latencies rather than
// one per split.
template <int RW, int NG, bool Q8>
__device__ __forceinline__ void merge_group(const DecodeParams& p, int s, int kvh, int S, int first,
                                            uint8_t* smem, uint32_t sbase) {
  using C = Cfg<RW, NG, Q8>;
  constexpr int kThreads = C::kThreads;
  constexpr int kRowF4 = kHeadDim / 4;  // float4 per partial row
  constexpr int kWarps = kThreads / 32;
  constexpr int kPairsMax = (NG * RW * kRowF4 + kThreads - 1) / kThreads;  // rows <= NG * RW
  const int R = p.rows, G = p.group, Hq = p.num_q_heads;
  const long long rps = (long long)p.n_query * Hq;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  float* w = reinterpret_cast<float*>(smem);  // [S][R]
  float* inv = w + S * R;                     // [R]
  const uint32_t stage_off = ((uint32_t)(S * R + R) * 4u + 1023u) & ~1023u;
  const uint32_t stage = sbase + stage_off;
  const float4* stage4 = reinterpret_cast<const float4*>(smem + stage_off);
  const int per_round = max(1, (int)((C::kRed - stage_off) / (uint32_t)(R * kHeadDim * 4)));
  auto row_index = [&](int r) { return (long long)(r / G) * Hq + kvh * G + (r % G); };
  const long long split0 = (long long)first * R;  // partial row of (split 0, row 0) of the group

  // Raw log-sum-exps, all loads in flight together.
  for (int i0 = 0; i0 < S * R; i0 += 8 * kThreads) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kThreads + threadIdx.x;
      v[u] = i < S * R ? __ldcg(p.part_lse + split0 + i) : 0.f;  // [split][row]
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * kThreads + threadIdx.x;
      if (i < S * R) w[i] = v[u];
    }
  }
  __syncthreads();
  for (int r = warp; r < R; r += kWarps) {
    float M = -INFINITY;
    bool bad = false;  // a split read a stand-in for an out-of-range block
    for (int k = lane; k < S; k += 32) {
      M = fmaxf(M, w[k * R + r]);
      bad |= isnan(w[k * R + r]);
    }
    bad = __any_sync(0xffffffffu, bad);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float sum = 0.f;
    for (int k = lane; k < S; k += 32) {
      const float l = w[k * R + r];
      const float wk = (bad || l == -INFINITY) ? 0.f : expf(l - M);
      w[k * R + r] = wk;
      sum += wk;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) inv[r] = sum > 0.f ? 1.f / sum : 0.f;
  }

  // Thread = (row, 4 consecutive head_dim elements), up to kPairsMax pairs;
  // empty splits carry weight 0 and a zero partial.
  float4 acc[kPairsMax];
#pragma unroll
  for (int q = 0; q < kPairsMax; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k0 = 0; k0 < S; k0 += per_round) {
    const int k1 = min(S, k0 + per_round);
    __syncthreads();  // weights ready / the previous round's reads done
    // Staged row q = (k - k0) * R + r; lane = its float4 column (kThreads is
    // a multiple of 32, so every copy of this thread has column `lane`).
    const int nrows = (k1 - k0) * R;
    for (int q = warp; q < nrows; q += kWarps) {
      const int k = k0 + q / R, r = q % R;
      const float* src = p.part_out + (split0 + (long long)k * R + r) * kHeadDim + lane * 4;
      cp_async_16(stage + (uint32_t)(q * kRowF4 + lane) * 16u, src);
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPairsMax; ++q) {
      const int pr = threadIdx.x + q * kThreads;
      if (pr < R * kRowF4) {
        const int r = pr / kRowF4, c4 = pr % kRowF4;
        for (int k = k0; k < k1; ++k) {
          const float wk = w[k * R + r];
          const float4 v = stage4[((k - k0) * R + r) * kRowF4 + c4];
          acc[q].x = fmaf(wk, v.x, acc[q].x);
          acc[q].y = fmaf(wk, v.y, acc[q].y);
          acc[q].z = fmaf(wk, v.z, acc[q].z);
          acc[q].w = fmaf(wk, v.w, acc[q].w);
        }
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kPairsMax; ++q) {
    const int pr = threadIdx.x + q * kThreads;
    if (pr < R * kRowF4) {
      const int r = pr / kRowF4, c4 = pr % kRowF4;
      const float iv = inv[r];
      const __half2 h0 = __floats2half2_rn(acc[q].x * iv, acc[q].y * iv);
      const __half2 h1 = __floats2half2_rn(acc[q].z * iv, acc[q].w * iv);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&h0);
      u.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(p.out + ((long long)s * rps + row_index(r)) * kHeadDim + c4 * 4) = u;
    }
  }
}

// Cooperative merge (every CTA of the grid resident): once its whole group
// has written its partials, split k of a (sequence, KV head) merges pairs
// [k*P/S, (k+1)*P/S) of the group's P = R*32 (row, float4 column) pairs.
// The log-sum-exp weights of merge_group, spread over all S CTAs of the
// group so that each stages only a few kilobytes of partials with one round
// of 16-byte asynchronous copies; the weighted partials of a pair are added
// in a fixed order (lane i of a pair's lanes takes splits i, i + tp, ...,
// then a butterfly), so results stay reproducible.
template <int RW, int NG, bool Q8>
__device__ __forceinline__ void merge_slice(const DecodeParams& p, int s, int kvh, int split, int S,
                                            int first, uint8_t* smem, uint32_t sbase) {
  constexpr int kThreads = Cfg<RW, NG, Q8>::kThreads;
  constexpr int kRowF4 = kHeadDim / 4;
  constexpr int kWarps = kThreads / 32;
  const int R = p.rows, G = p.group, Hq = p.num_q_heads;
  const long long rps = (long long)p.n_query * Hq;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int P = R * kRowF4;
  const int pa = (int)((long long)split * P / S), pb = (int)((long long)(split + 1) * P / S);
  if (pa >= pb) return;  // uniform across the CTA
  const int r_lo = pa / kRowF4, nr = (pb - 1) / kRowF4 - r_lo + 1, np = pb - pa;
  auto row_index = [&](int r) { return (long long)(r / G) * Hq + kvh * G + (r % G); };
  const long long split0 = (long long)first * R;  // partial row of (split 0, row 0) of the group
  float* w = reinterpret_cast<float*>(smem);  // [nr][S]
  float* inv = w + nr * S;                    // [nr]
  const uint32_t stage_off = ((uint32_t)(nr * S + nr) * 4u + 1023u) & ~1023u;
  const float4* stage4 = reinterpret_cast<const float4*>(smem + stage_off);  // [S][np]

  // The partial columns first (the longest wait), then the log-sum-exps.
  for (int e = threadIdx.x; e < S * np; e += kThreads) {
    const int k = e / np, pr = pa + e % np;
    const float* src =
        p.part_out + (split0 + (long long)k * R + pr / kRowF4) * kHeadDim + (pr % kRowF4) * 4;
    cp_async_16(sbase + stage_off + (uint32_t)e * 16u, src);
  }
  for (int e = threadIdx.x; e < nr * S; e += kThreads)
    w[e] = __ldcg(p.part_lse + split0 + (long long)(e % S) * R + r_lo + e / S);
  __syncthreads();
  for (int j = warp; j < nr; j += kWarps) {
    float M = -INFINITY;
    bool bad = false;  // a split read a stand-in for an out-of-range block
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
    if (lane == 0) inv[j] = sum > 0.f ? 1.f / sum : 0.f;
  }
  cp_async_wait_all();
  __syncthreads();
  // tp threads (lanes of one warp) per pair, each adding every tp-th split;
  // then a fixed butterfly over the tp lanes.  Loop bounds are uniform per
  // warp, so every lane takes part in the shuffles.
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
    if (valid && sub == 0) {
      const float iv = inv[j];
      const __half2 h0 = __floats2half2_rn(acc.x * iv, acc.y * iv);
      const __half2 h1 = __floats2half2_rn(acc.z * iv, acc.w * iv);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&h0);
      u.y = *reinterpret_cast<const uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(p.out + ((long long)s * rps + row_index(r)) * kHeadDim + c4 * 4) = u;
    }
  }
}

template <int RW, int NG, bool Q8, bool TR>
__global__ void __launch_bounds__(Cfg<RW, NG, Q8>::kThreads, 1)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using C = Cfg<RW, NG, Q8>;
  constexpr int kThreads = C::kThreads, kGroups = NG, kVWarp = C::kVWarp;
  constexpr int NR = C::NR, KS = C::KS, VS = C::VS, PB = C::PB;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by pointer
  // arithmetic so that accesses through it stay shared-space loads/stores.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kMisc);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + C::kInfo);
  volatile int* abort = &misc->abort;
  const unsigned long long wl = p.wait_limit_ns;  // bound of every pipeline wait
  auto bar = [&](int i) { return sbase + C::kBars + 8u * i; };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nq = p.n_query, G = p.group, Hq = p.num_q_heads, R = p.rows;
  const int C_all = gridDim.x, cta = blockIdx.x;

  // Launched as a programmatic dependent of whatever precedes it on the
  // stream: set-up above touched only registers; nothing global is read
  // before that grid has completed and flushed.  Dependents of this grid
  // may launch at once (they wait the same way).
  griddep_wait();
  griddep_launch_dependents();
  // Which (sequence, KV head) this CTA works for: every thread computes it
  // (arithmetic only), so that no barrier stands between the grid
  // dependency and the first memory reads.  The context length is read at
  // once; with one sequence, the K producer lanes read the block-table
  // entries of this CTA's first tile at the same time, on the guess that the
  // whole table is visible (no window, full length), used below only if the
  // guess held.  Both latencies overlap.
  const GroupOf go = group_of(p, cta, C_all);
  const int s = go.s, kvh = go.kvh, split = go.split, S = go.splits, first = go.first;
  const int L = ld_nc_s32(p.context_lens + s);
  int spec_key0 = -1, spec_phys = 0;
  if (warp == 0 && p.num_seqs == 1 && p.tiles_per_item == 0 && lane < kChunksPerTile) {
    const int ntg =
        (int)(((long long)p.max_blocks_per_seq * p.block_size + kTileKeys - 1) / kTileKeys);
    const int tfg = go.split * (ntg / go.splits) + min(go.split, ntg % go.splits);
    const int key0 = tfg * kTileKeys + lane * kChunk;
    if (ntg / go.splits + (go.split < ntg % go.splits ? 1 : 0) > 0 &&
        key0 / p.block_size < p.max_blocks_per_seq) {
      spec_key0 = key0;
      spec_phys = ld_nc_s32(p.block_table + key0 / p.block_size);
    }
  }
  // Group barrier of the cooperative merge (below): its phase bit, read
  // before this CTA arrives (it cannot flip before then).  A relaxed load:
  // it stays in flight while this thread (the K producer's lane 0) goes on;
  // an acquire would hold back its every later access until it returns.
  int* cnt = p.arrivals + ((long long)s * p.num_kv_heads + kvh) * 2;
  unsigned int bar_phase = 0;
  if (p.coop && threadIdx.x == 0) bar_phase = (unsigned int)ld_relaxed_gpu(cnt) & 0x80000000u;
  // Partials: CTA c owns rows [c*R, c*R + R) of the partial outputs and
  // log-sum-exps; the CTAs of one group are consecutive.
  const long long part_base = (long long)cta * R;
  auto row_index = [&](int r) { return (r / G) * Hq + kvh * G + (r % G); };

  // ---- the head's visible keys and its tiles (uniform across the CTA) ------
  // The keys of (sequence s, KV head kvh) that any query token sees form
  // [lo_u, hi_u]; they are cut into 128-key tiles from `base`, and the S
  // splits take contiguous runs of them (as even as whole tiles allow, or
  // items of tiles_per_item tiles).  The partition depends only on the
  // sequence's own context length and the shapes, so every call on the same
  // inputs adds the same tiles in the same order: results are
  // bit-reproducible.
  const int* table = p.block_table + (long long)s * p.max_blocks_per_seq;
  const SeqTiles st_ = seq_tiles(p, L);
  const int lo_u = st_.lo, hi_u = st_.hi, base = st_.base, ntiles_h = st_.tiles;
  if (!context_len_ok(L, nq, p.max_blocks_per_seq, p.block_size) && split == 0 && kvh == 0 &&
      threadIdx.x == 0)
    atomicOr(p.flags, kFlagBadLen);
  int t_first, t_count;
  if (p.tiles_per_item > 0) {  // item `split` of T tiles
    t_first = split * p.tiles_per_item;
    t_count = max(0, min(p.tiles_per_item, ntiles_h - t_first));
  } else {  // the S CTAs of the group take contiguous runs, as even as whole tiles allow
    const int t_per = ntiles_h / S, t_rem = ntiles_h % S;
    t_first = split * t_per + min(split, t_rem);
    t_count = t_per + (split < t_rem ? 1 : 0);
  }

  const uint32_t sKr = sbase + C::kK, sVr = sbase + C::kV;
  const uint32_t sQ = sbase + C::kQ, sP = sbase + C::kP;

  if (t_count == 0) {
    // Every tile is another CTA's: an empty partial (weight 0 in the merge).
    for (int t = threadIdx.x; t < R * kHeadDim; t += kThreads) {
      const int r = t / kHeadDim;
      p.part_out[(part_base + r) * kHeadDim + t % kHeadDim] = 0.f;
      if (t % kHeadDim == 0) p.part_lse[part_base + r] = -INFINITY;
    }
  } else if (warp == 0) {
    // ======================= K producer (also sets up the barriers) ========
    if (lane == 0) {
      for (int i = 0; i < kMaxStages; ++i) {
        mbar_init(bar(BAR_KFULL + i), 1);
        mbar_init(bar(BAR_KEMPTY + i), 1);
        mbar_init(bar(BAR_VFULL + i), 1);
        mbar_init(bar(BAR_VEMPTY + i), 1);
        if (Q8) {  // q8_0: a slot's fp16 tile is ready once every converter warp arrived
          mbar_init(bar(BAR_CKFULL + i), C::kConvWarps);
          mbar_init(bar(BAR_CVFULL + i), C::kConvWarps);
        }
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(BAR_SFULL + i), 1);
        mbar_init(bar(BAR_SEMPTY + i), 4 * kGroups);
        mbar_init(bar(BAR_PFULL + i), 4 * kGroups);
      }
      mbar_init(bar(BAR_OFULL), 1);
      mbar_init(bar(BAR_DONE), 1);
      for (int i = 0; i < kInfoSlots; ++i) mbar_init(bar(BAR_INFO + i), 1);
      misc->abort = 0;
      misc->bad = 0;
      misc->k_consumed = misc->v_consumed = 0;
      fence_mbar_init();
    }
    __syncwarp();
    // The other roles wait for these barriers; this warp starts loading now.
    named_bar_arrive(kBarSetup, kThreads);

    // Lane c < 8 owns chunk c of every tile.  Its block-table entry for tile
    // t + 1 is read right after tile t's copy is issued and used one slot
    // wait later, so the load's latency hides behind that wait.
    const int c = lane;
    constexpr long long kNone = -(1LL << 40);
    auto tile_of = [&](int t) { return t < t_count ? t_first + t : -1; };
    // Physical block of chunk c of local tile t (kNone: not loaded).
    auto lookup_raw = [&](int t) -> long long {
      const int g = tile_of(t);
      if (g < 0 || c >= kChunksPerTile) return kNone;
      const int key0 = base + g * kTileKeys + c * kChunk;
      if (key0 > hi_u || key0 + kChunk - 1 < lo_u) return kNone;
      return table[key0 / p.block_size];
    };
    // TMA row coordinate (row / 8) of that chunk, -1 if it is not loaded.
    // An out-of-range block is never dereferenced: row 0 of the cache stands
    // in for it (so that every visible key has finite-or-not data the
    // softmax need not know about), the error flag is raised, and the CTA's
    // partial is marked invalid so that the merge writes the group's rows
    // as 0.
    auto to_row8 = [&](long long phys, int t) -> int {
      if (phys == kNone) return -1;
      if (phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.flags, kFlagBadBlock);
        misc->bad = 1;
        return 0;
      }
      if (Q8) return (int)(phys * p.num_kv_heads + kvh);  // q8_0: the (block, head) tile
      const int key0 = base + tile_of(t) * kTileKeys + c * kChunk;
      return (int)(((phys * p.num_kv_heads + kvh) * p.block_size + key0 % p.block_size) / 8);
    };
    long long raw0 = kNone;
    if (c < kChunksPerTile && t_count > 0) {
      const int key0 = base + t_first * kTileKeys + c * kChunk;
      if (key0 <= hi_u && key0 + kChunk - 1 >= lo_u)
        raw0 = key0 == spec_key0 ? (long long)spec_phys : (long long)table[key0 / p.block_size];
    }
    int row_cur = to_row8(raw0, 0);
    long long raw_nxt = lookup_raw(1);
    int issued = 0;
    for (int t = 0;; ++t) {
      const int g_cur = tile_of(t);
      const bool w_cur = row_cur >= 0;
      // Publish tile t for the V producer, the MMA issuer and the softmax.
      const uint32_t mask = __ballot_sync(0xffffffffu, w_cur);
      TileInfo& ti = info[t % kInfoSlots];
      if (lane < kChunksPerTile) ti.row8[lane] = row_cur;
      if (lane == 0) {
        ti.tile = g_cur;
        ti.mask = mask;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BAR_INFO + t % kInfoSlots));
      if (g_cur < 0) break;
      // Wait for the slot, then every lane issues its chunk's copy.
      const int st = t % KS;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar(BAR_KEMPTY + st), ((t / KS) & 1) ^ 1, abort, wl);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const uint32_t fb = bar(BAR_KFULL + st);
      if (lane == 0) mbar_arrive_expect_tx(fb, __popc(mask) * (Q8 ? kQ8QsChunk : kChunkBytes));
      __syncwarp();
      if (w_cur) {
        if constexpr (Q8) {
          // K's scales are read by the softmax (from L2), not staged here.
          const long long off = q8_chunk_offset(p, row_cur, base + g_cur * kTileKeys + c * kChunk);
          const uint8_t* src = static_cast<const uint8_t*>(p.k);
          bulk_load(sKr + st * C::kKSlot + kRawOff + c * kQ8QsChunk, src + off, kQ8QsChunk, fb);
          bulk_prefetch_l2(static_cast<const uint8_t*>(p.v) + off, kChunk * kHeadDim);
          bulk_prefetch_l2(static_cast<const uint8_t*>(p.v) + off +
                               q8_scale_offset(p, base + g_cur * kTileKeys + c * kChunk),
                           kChunk * 8);
        } else {
          tma_load_4d(sKr + st * kKVBytes + c * kChunkBytes, &tmap_k, 0, 0, 0, row_cur, fb);
          tma_prefetch_4d(&tmap_v, 0, 0, 0, row_cur);
        }
      }
      __syncwarp();
      issued = t + 1;
      row_cur = to_row8(raw_nxt, t + 1);
      raw_nxt = lookup_raw(t + 2);
    }
    __syncthreads();  // (A) every role finished its loop
    if (lane == 0) {  // drain copies that no MMA waited for (abort path only)
      volatile int no_abort = 0;
      for (int t = misc->k_consumed; t < issued; ++t)
        mbar_wait(bar(BAR_KFULL + t % KS), (t / KS) & 1, &no_abort);
    }
  } else {
    // ---- set-up of the other roles ----------------------------------------
    if (warp == 1) {
      tmem_alloc(sbase + C::kMisc + offsetof(Misc, tmem_base), C::kTmemCols);
      tmem_relinquish();
    }
    if (warp >= 2 && warp < kVWarp) {
      // Q rows of this KV head -> shared memory, K-major with 128-byte
      // swizzle: row n, 16-byte chunk c of half h at h*NR*128 + n*128 +
      // ((c ^ n%8) * 16).  Rows >= R are zero; so are P's padding rows (never
      // written later).  A negative scale is moved into Q (an exact sign
      // flip) so that the kernel only multiplies scores by a factor >= 0.
      const int t = threadIdx.x - 64;
      const uint32_t flip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
      for (int c = t; c < NR * 16; c += kGroups * kSoftmaxThreads) {
        const int n = c / 16, cc = c % 16, h = cc / 8, k8 = cc % 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < R) {
          const long long qrow = ((long long)s * nq + n / G) * Hq + kvh * G + (n % G);
          v = ldg_nc_v4(p.q + qrow * kHeadDim + cc * 8);
          v.x ^= flip; v.y ^= flip; v.z ^= flip; v.w ^= flip;
        }
        sts_v4(sQ + h * C::kQHalf + n * 128 + ((k8 ^ (n & 7)) * 16), v);
      }
      for (uint32_t off = t * 16; off < PB * C::kPBytes; off += kGroups * kSoftmaxThreads * 16)
        sts_v4(sP + off, make_uint4(0, 0, 0, 0));
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_bar_sync(kBarSetup, kThreads);  // barriers initialised, TMEM allocated, Q staged
    tc_fence_after();
    const uint32_t tmem = misc->tmem_base;

    if (warp == kVWarp) {
      // ===================== V producer ======================================
      // Follows the K producer's published tiles; lane c < 8 issues chunk c.
      const int c = lane;
      int issued = 0;
      for (int t = 0;; ++t) {
        int ok = 1;
        if (lane == 0)
          ok = mbar_wait(bar(BAR_INFO + t % kInfoSlots), (t / kInfoSlots) & 1, abort, wl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // lane 0's acquire orders the other lanes' reads below
        if (!ok) break;
        const TileInfo& ti = info[t % kInfoSlots];
        if (ti.tile < 0) break;
        const uint32_t mask = ti.mask;
        const int row8 = c < kChunksPerTile ? ti.row8[c] : 0;  // q8_0: the tile index
        const int st = t % VS;
        if (lane == 0) ok = mbar_wait(bar(BAR_VEMPTY + st), ((t / VS) & 1) ^ 1, abort, wl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const uint32_t fb = bar(BAR_VFULL + st);
        if (lane == 0)
          mbar_arrive_expect_tx(fb, __popc(mask) * (Q8 ? kQ8QsChunk + kQ8DChunk : kChunkBytes));
        __syncwarp();
        if (c < kChunksPerTile && ((mask >> c) & 1u)) {
          if constexpr (Q8) {
            const long long off = q8_chunk_offset(p, row8, base + ti.tile * kTileKeys + c * kChunk);
            const uint32_t dst = sVr + st * C::kVSlot;
            const uint8_t* src = static_cast<const uint8_t*>(p.v);
            bulk_load(dst + kRawOff + c * kQ8QsChunk, src + off, kQ8QsChunk, fb);
            bulk_load(dst + kKVBytes + c * kQ8DChunk,
                      src + off + q8_scale_offset(p, base + ti.tile * kTileKeys + c * kChunk),
                      kQ8DChunk, fb);
          } else {
            tma_load_4d(sVr + st * kKVBytes + c * kChunkBytes, &tmap_v, 0, 0, 0, row8, fb);
          }
        }
        __syncwarp();
        issued = t + 1;
      }
      __syncthreads();  // (A)
      if (lane == 0) {  // drain copies that no MMA waited for (abort path only)
        volatile int no_abort = 0;
        for (int t = misc->v_consumed; t < issued; ++t)
          mbar_wait(bar(BAR_VFULL + t % VS), (t / VS) & 1, &no_abort);
      }
    } else if (warp == 1) {
      // ===================== MMA issuer ======================================
      // One thread, in a fixed order: QK(0), QK(1), then PV(t), QK(t+2) for
      // t = 0, 1, ...  A commit completes once every MMA this thread issued
      // before it has finished, so S(t) in TMEM also means that O(t-2) is.
      // The number of tiles is t_count (uniform), so the issuer reads no
      // published tile information.
      if (lane == 0) {
        const uint32_t id_qk = idesc_f16_f32(128, NR, false, false);
        const uint32_t id_pv = idesc_f16_f32(128, C::kPN, true, true);
        // Descriptors at offset 0; a byte offset o is added as o >> 4 (the
        // start-address field is the low 14 bits, addresses stay < 256 KB).
        // q8_0: K and V are the converted slots (exact fp16 images of the
        // int8 values; V's rows also carry the power of two of their scales).
        // S^T gets one accumulator per scale group g (head_dim 32g .. 32g+31,
        // two steps of 16), which the softmax combines with K's scales; PV
        // multiplies V with each group's P (the weights times V's scale
        // mantissas) into that group's O^T accumulator.
        const uint64_t dK = smem_desc(sKr, 16, kGroupBytes, kSwizzle128B);
        const uint64_t dQ = smem_desc(sQ, 16, 1024, kSwizzle128B);
        const uint64_t dV = smem_desc(sVr, kAtomBytes, kGroupBytes, kSwizzle128B);
        const uint64_t dP = smem_desc(sP, C::kPN * 16, 128, kSwizzleNone);
        constexpr int kSG = C::kSG;
        // QK(u) once K(u) is ready and the softmax took S(u-2) from its buffer.
        auto issue_qk = [&](int u) -> bool {
          const bool ready =
              mbar_wait(bar((Q8 ? BAR_CKFULL : BAR_KFULL) + u % KS), (u / KS) & 1, abort, wl);
          if (!(ready && mbar_wait(bar(BAR_SEMPTY + u % 2), ((u / 2) & 1) ^ 1, abort, wl)))
            return false;
          tc_fence_after();
          const uint64_t so = (uint64_t)((u % KS) * C::kKSlot) >> 4;
          const uint32_t d = tmem + (u % 2) * kSG * NR;
          constexpr int kSteps = kHeadDim / 16 / kSG;  // steps of 16 per accumulator
#pragma unroll
          for (int k = 0; k < kHeadDim / 16; ++k) {
            const uint64_t ko = ((k / 4) * kAtomBytes + (k % 4) * 32) >> 4;
            const uint64_t qo = ((k / 4) * C::kQHalf + (k % 4) * 32) >> 4;
            tc_mma_f16_ss(d + (k / kSteps) * NR, dK + so + ko, dQ + qo, id_qk, k % kSteps != 0);
          }
          tc_commit(bar(BAR_SFULL + u % 2));
          tc_commit(bar(BAR_KEMPTY + u % KS));
          return true;
        };
        int nqk = 0, npv = 0;
        bool ok = true;
        for (int u = 0; u < 2 && u < t_count && ok; ++u) {
          ok = issue_qk(u);
          if (ok) nqk = u + 1;
        }
        for (int t = 0; ok && t < t_count; ++t) {
          // PV(t) once P(t), V(t) and the O buffer are ready, then QK(t+2).
          ok = mbar_wait(bar(BAR_PFULL + t % PB), (t / PB) & 1, abort, wl) &&
               mbar_wait(bar((Q8 ? BAR_CVFULL : BAR_VFULL) + t % VS), (t / VS) & 1, abort, wl);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = (uint64_t)((t % VS) * C::kVSlot) >> 4;
          const uint64_t pb = (uint64_t)((t % PB) * C::kPBytes) >> 4;
          // O^T accumulates over all tiles; q8_0: the kSG group accumulators
          // are the consecutive column ranges of one N = kPN product.
          const uint32_t d = tmem + C::kTmemS;
#pragma unroll
          for (int k = 0; k < kTileKeys / 16; ++k) {
            const uint64_t vo = (k * 2 * kGroupBytes) >> 4;
            const uint64_t po = (k * 2 * C::kPN * 16) >> 4;
            tc_mma_f16_ss(d, dV + so + vo, dP + pb + po, id_pv, t > 0 || k > 0);
          }
          tc_commit(bar(BAR_OFULL));
          tc_commit(bar(BAR_VEMPTY + t % VS));
          npv = t + 1;
          if (t + 2 < t_count) {
            ok = issue_qk(t + 2);
            if (ok) nqk = t + 3;
          }
        }
        misc->k_consumed = nqk;
        misc->v_consumed = npv;
        tc_commit(bar(BAR_DONE));  // completes once every MMA above has finished
        volatile int no_abort = 0;
        mbar_wait(bar(BAR_DONE), 0, &no_abort);
      }
      __syncwarp();
      __syncthreads();  // (A)
    } else if (Q8 && warp >= C::kConvWarp) {
      // ===================== q8_0 converters =================================
      // Raw tile t (int8 qs in the upper half of its slot; V: fp16 scales d
      // per 32 elements after the tile) -> the fp16 operand in the same slot,
      // exactly: K's operand is qs itself (every integer below 2048 is an
      // fp16 value; K's scales are applied to the per-group scores in the
      // softmax), V's is qs * 2^e with 2^e the power of two of the element's
      // scale d = m * 2^e (exact for |d| < 1024: at most 7 significant bits
      // above 2^-24); the mantissa m goes into that group's P.  The
      // arithmetic is packed fp16 (two elements per instruction).  Layout as
      // the fp16 TMA boxes: [key/8][half][key%8][64 dims], 128-byte swizzle.
      // V rows of keys outside [lo_u, hi_u] (masked or never loaded) are
      // written as zeros: they must not reach the PV product.
      // The first kConvWarps converter warps convert K, the next kConvWarps
      // V.  Thread ct of a stream's kCT takes the 16-byte column chunk
      // c16 = ct % 8 (head_dim 16*c16 .. +15, half of one scale group) of keys
      // r = ct / 8 + kRS*k: one 16-byte load and two 16-byte stores per key,
      // the swizzled destination offset constant up to the key group, no bank
      // conflicts on either side.  In place: keys 0 .. 63 land below the raw
      // data; keys 64 .. 127 are stored only after every thread of the stream
      // has read (and converted into registers) all its raw rows.
      constexpr int kCT = 32 * C::kConvWarps;   // threads per stream
      constexpr int kRS = kCT / 8;              // key stride between a thread's keys
      constexpr int kKeysPer = kTileKeys / kRS; // keys per thread per tile
      constexpr int kHalfKeys = kKeysPer / 2;   // per half tile
      static_assert(kKeysPer % 2 == 0 && (kTileKeys / 2) * 256 <= kRawOff,
                    "the lower half of the keys is stored below the raw tile");
      const int kv = (warp - C::kConvWarp) / C::kConvWarps;  // 0: K, 1: V
      const int ct = threadIdx.x - 32 * (C::kConvWarp + C::kConvWarps * kv);  // 0 .. kCT-1
      const int c16 = ct & 7, r0 = ct >> 3;      // column chunk, first key
      const int r08 = r0 & 7;                    // its row within a key group
      // destination of the two 8-element halves: chunk cc = 2*c16 + e of the
      // key's 256-byte row, i.e. half cc / 8, 16-byte slot (cc % 8) ^ (key % 8)
      const uint32_t dst_a = (r0 >> 3) * kGroupBytes + ((2 * c16) >> 3) * kAtomBytes + r08 * 128 +
                             ((((2 * c16) & 7) ^ r08) << 4);
      const uint32_t dst_b = (r0 >> 3) * kGroupBytes + ((2 * c16 + 1) >> 3) * kAtomBytes +
                             r08 * 128 + ((((2 * c16 + 1) & 7) ^ r08) << 4);
      const int NSl = kv == 0 ? KS : VS;
      const uint32_t bar_full = kv == 0 ? BAR_KFULL : BAR_VFULL;
      const uint32_t bar_conv = kv == 0 ? BAR_CKFULL : BAR_CVFULL;
      const uint32_t ring = sbase + (kv == 0 ? C::kK : C::kV);
      const uint32_t slot_bytes = kv == 0 ? C::kKSlot : C::kVSlot;
      bool ok = true;
      // Eight int8 -> eight fp16 values times the power of two p2 (1 for K).
      auto convert = [&](uint32_t w0, uint32_t w1, __half2 p2) -> uint4 {
        __half2 x[4];
        q8_to_half8(make_uint2(w0, w1), x);
        uint32_t h[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 y = kv == 0 ? x[e] : __hmul2(x[e], p2);
          h[e] = *reinterpret_cast<const uint32_t*>(&y);
        }
        return make_uint4(h[0], h[1], h[2], h[3]);
      };
      for (int t = 0; t < t_count && ok; ++t) {
        const int key_t = base + (t_first + t) * kTileKeys;  // first key of the tile
        const int rs = t % NSl;
        // The stream's threads decide together (one gave up: all stop), so
        // that every one of them reaches the named barrier below.
        ok = named_bar_and(kBarConv0 + kv, kCT,
                           __all_sync(0xffffffffu, mbar_wait(bar(bar_full + rs), (t / NSl) & 1, abort, wl)));
        if (!ok) break;
        const uint32_t slot = ring + rs * slot_bytes;
        const uint32_t src = slot + kRawOff + r0 * kHeadDim + c16 * 16;       // key r0, chunk c16
        const uint32_t srcd = slot + kKVBytes + r0 * 8 + (c16 >> 1) * 2;     // its scale (V)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 qv[kHalfKeys];
          uint16_t dv[kHalfKeys];
#pragma unroll
          for (int i = 0; i < kHalfKeys; ++i) {
            const int k = h * kHalfKeys + i;
            qv[i] = lds_v4(src + k * kRS * kHeadDim);
            dv[i] = kv == 0 ? (uint16_t)0 : lds_u16(srcd + k * kRS * 8);
          }
          uint4 xa[kHalfKeys], xb[kHalfKeys];
#pragma unroll
          for (int i = 0; i < kHalfKeys; ++i) {
            const int r = (h * kHalfKeys + i) * kRS + r0;
            xa[i] = make_uint4(0, 0, 0, 0);
            xb[i] = xa[i];
            if (kv == 0 || (key_t + r >= lo_u && key_t + r <= hi_u)) {
              const __half p2 = __ushort_as_half(q8_scale_pow2_bits(dv[i]));
              const __half2 p22 = __halves2half2(p2, p2);
              xa[i] = convert(qv[i].x, qv[i].y, p22);
              xb[i] = convert(qv[i].z, qv[i].w, p22);
            }
          }
          // The upper half overwrites raw rows: every thread of the stream
          // has read all of its rows once it is past this barrier.
          if (h == 1) named_bar_sync(kBarConv0 + kv, kCT);
#pragma unroll
          for (int i = 0; i < kHalfKeys; ++i) {
            const uint32_t g8 = (h * kHalfKeys + i) * (kRS / 8) * kGroupBytes;
            sts_v4(slot + g8 + dst_a, xa[i]);
            sts_v4(slot + g8 + dst_b, xb[i]);
          }
        }
        fence_proxy_async_smem();  // generic writes -> the tensor core's reads
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(bar_conv + rs));
      }
      __syncthreads();  // (A)
    } else {
      // ===================== softmax + correction ============================
      // Warpgroup g handles rows [g*RW, g*RW + RW); its warps cover the four
      // TMEM lane quarters, i.e. keys (for S) and head_dim elements (for O).
      const int g = (warp - 2) / 4, widx = (warp - 2) % 4;
      const int row0 = g * RW;
      const int q4 = warp & 3;
      const int j = q4 * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
      float* red = reinterpret_cast<float*>(smem + C::kRed) + g * 2 * 4 * 32;  // [2][4][32]
      float* lsum = reinterpret_cast<float*>(smem + C::kLsum) + g * 4 * 32;    // [4][32]
      float* bc = reinterpret_cast<float*>(smem + C::kBcast) + (warp - 2) * 64;  // [2][32]
      const uint32_t bar_id = kBarGroup0 + g;
      const float cs = fabsf(p.scale_log2);  // scores are scaled by cs >= 0 (log2 domain)

      // Per query token, the visible key range; keys inside every token's
      // range see all rows: the fast path of interior tiles.
      int tlo[kMaxQuery], thi[kMaxQuery];
      int lo_all = lo_u, hi_all = hi_u;
#pragma unroll
      for (int i = 0; i < kMaxQuery; ++i) {
        tlo[i] = 1;
        thi[i] = 0;
        if (i < nq) {
          key_range(L, nq, i, p.causal, p.window, tlo[i], thi[i]);
          lo_all = max(lo_all, tlo[i]);
          hi_all = min(hi_all, thi[i]);
        }
      }
      const uint32_t grp = G >= 32 ? 0xffffffffu : ((1u << G) - 1u);
      const uint32_t all_rows = R >= 32 ? 0xffffffffu : ((1u << R) - 1u);

      float lpart[RW], bias[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        lpart[r] = 0.f;
        bias[r] = INFINITY;  // no reference yet: the row's first key forces one
      }
      // Reference max (raw score) of row row0 + lane % RW; -inf until the
      // row sees a key.  bias[r] = kPShift - cs * (row r's reference max).
      float m_lane = -INFINITY;
      bool ok = true;
      const int end_t = t_count;  // tiles of this CTA (local t -> tile t_first + t)
      // O^T accumulates in TMEM over every tile (from column kTmemS: the
      // high parts of the rows, then their residuals).  When a row's
      // reference rises at tile t, its O column is scaled by alpha in place,
      // after PV(t-1) has finished and before P(t) is published.  fp16: S(t)
      // in TMEM implies that PV(t-2) has finished (the issuer commits S(t)
      // after issuing PV(t-2)), so P buffer t % 2 is free again; q8_0 (one P
      // buffer) waits for PV(t-1) before storing P(t).
      // q8_0: this thread's lanes of O^T are head_dim elements 32*q4 ..
      // 32*q4 + 31, i.e. scale group q4: only that group's accumulator is
      // read (and rescaled) here.
      const uint32_t o_hi = tmem + lane_off + C::kTmemS + (Q8 ? q4 * 2 * NR : 0) + row0;
      const uint32_t o_lo = o_hi + NR;
      constexpr int kSG = C::kSG;
      // q8_0: the K and V scales of this thread's key (4 fp16 each), read
      // from the cache (an L2 hit: the tile's bulk copies brought them) one
      // tile ahead; zeros for a key no row sees.
      auto fetch_scales = [&](int u) -> uint4 {
        uint4 sc = make_uint4(0, 0, 0, 0);
        ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_INFO + u % kInfoSlots),
                                                     (u / kInfoSlots) & 1, abort, wl));
        if (ok) {
          const int key = base + (t_first + u) * kTileKeys + j;
          const int tix = info[u % kInfoSlots].row8[j / kChunk];  // (block, head) tile, -1: not loaded
          if (tix >= 0 && key >= lo_u && key <= hi_u) {
            const long long off = q8_key_scales_offset(p, tix, key % p.block_size);
            const uint2 a = ldg_nc_v2(static_cast<const uint8_t*>(p.k) + off);
            const uint2 b = ldg_nc_v2(static_cast<const uint8_t*>(p.v) + off);
            sc = make_uint4(a.x, a.y, b.x, b.y);
          }
        }
        return sc;
      };
      // Wait until PV(k) has finished.  A parity wait for phase k of the
      // O barrier is exact only when phases < k have completed and phase k+1
      // cannot have (P(k+1) not yet published): k = t-1 before P(t) goes
      // out, where phases < t-1 are complete because S(t) implies PV(t-2).
      // A wait after the last P went out would not be exact for PV(end_t-2),
      // so that one is waited for before.  o_seen counts the phases known to
      // be complete.
      int o_seen = 0;
      auto wait_o_done = [&](int k) -> bool {
        if (o_seen > k) return true;
        if (!mbar_wait(bar(BAR_OFULL), k & 1, abort, wl)) return false;
        o_seen = k + 1;
        return true;
      };
      uint4 sc_next = make_uint4(0, 0, 0, 0);
      if constexpr (Q8) {
        if (end_t > 0) sc_next = fetch_scales(0);
      }
      for (int t = 0; t < end_t; ++t) {
        const int gt = t_first + t;  // tile number of local tile t
        const int sb = t % 2, st = t % VS;
        float mv[kSG];  // q8_0: V's scale mantissas of this key, per group
        float sv[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) sv[r] = 0.f;
        if constexpr (Q8) {
          const uint4 sc = sc_next;
          if (t + 1 < end_t) sc_next = fetch_scales(t + 1);
          ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_SFULL + sb), (t / 2) & 1, abort, wl));
          // Score = sum over the scale groups of K's scale times the group's
          // partial product (fp32, groups in order).
          float sg[kSG][RW];
#pragma unroll
          for (int q = 0; q < kSG; ++q)
#pragma unroll
            for (int r = 0; r < RW; ++r) sg[q][r] = 0.f;
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < kSG; ++q)
              tmem_ld<RW>(tmem + lane_off + sb * kSG * NR + q * NR + row0, sg[q]);
            tmem_ld_wait();
            tc_fence_before();
          }
          const uint32_t kw[2] = {sc.x, sc.y}, vw[2] = {sc.z, sc.w};
#pragma unroll
          for (int q = 0; q < kSG; ++q) {
            const uint16_t kd = (uint16_t)(kw[q / 2] >> (16 * (q % 2)));
            const uint16_t vd = (uint16_t)(vw[q / 2] >> (16 * (q % 2)));
            const float dk = __half2float(__ushort_as_half(kd));
            mv[q] = q8_scale_mantissa(vd);
#pragma unroll
            for (int r = 0; r < RW; ++r) sv[r] = q == 0 ? dk * sg[0][r] : fmaf(dk, sg[q][r], sv[r]);
          }
        } else {
          ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_SFULL + sb), (t / 2) & 1, abort, wl));
          mv[0] = 1.f;
          if (ok) {
            tc_fence_after();
            tmem_ld<RW>(tmem + lane_off + sb * NR + row0, sv);
            tmem_ld_wait();
            tc_fence_before();
          }
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(BAR_SEMPTY + sb));

        uint32_t rmask = 0;
        // Which rows see this key?  Chunks that were not loaded lie wholly
        // outside [lo_u, hi_u], so their keys see none.
        const int key = base + gt * kTileKeys + j;
        if (ok && key >= lo_u && key <= hi_u) {
          if (key >= lo_all && key <= hi_all) {
            rmask = all_rows;
          } else {
#pragma unroll
            for (int i = 0; i < kMaxQuery; ++i)
              if (i < nq && key >= tlo[i] && key <= thi[i]) rmask |= grp << (i * G);
          }
        }
        // every key of this warp is seen by every row: the interior fast path
        const bool all_vis = __all_sync(0xffffffffu, rmask == all_rows);
        if constexpr (TR) {
          // Key-resolution record: every (row, key) pair this kernel scores,
          // with the physical slot its K row was copied from (the tile's
          // published cache coordinates).
          ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_INFO + t % kInfoSlots),
                                                       (t / kInfoSlots) & 1, abort, wl));
          const uint32_t rm = rmask >> row0;
          if (ok && rm != 0) {
            const int row8 = info[t % kInfoSlots].row8[j / kChunk];
            const long long row = (long long)row8 * 8 + (key % kChunk);
            const long long phys = row / p.block_size / p.num_kv_heads;
            const unsigned id = (unsigned)(phys * p.block_size + key % p.block_size);
#pragma unroll
            for (int r = 0; r < RW; ++r) {
              if ((rm >> r) & 1u) {
                const int n = row0 + r;
                int32_t* tr = p.trace + (((long long)s * nq + n / G) * Hq + kvh * G + n % G) * 5;
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
          const uint32_t rm = rmask >> row0;
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            x[r] = ((rm >> r) & 1u) ? fmaf(sv[r], cs, bias[r]) : -INFINITY;
            xmax = fmaxf(xmax, x[r]);
          }
        }
        const bool exceed = xmax > (float)C::kPShift + kLazy;
        // Reconverge before the group barrier: a warp that arrives diverged
        // (after lane-predicated code) makes the barrier several times slower
        // (measured: 61k verify 122 -> 67 us per call).
        __syncwarp();
        // One barrier per tile: orders the shared-memory traffic of the group
        // and tells every thread whether any score passed its row's reference.
        const bool rescale = named_bar_or(bar_id, kSoftmaxThreads, exceed);
        if (rescale) {
          // New reference max per row: warp transpose-reduction, then
          // across the group's four warps.
          const uint32_t rm = all_vis ? 0xffffffffu : (rmask >> row0);
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
          const float bias_l =
              (m_new == -INFINITY) ? INFINITY : fmaf(-cs, m_new, (float)C::kPShift);
          m_lane = m_new;
          if (lane < RW) {
            bc[lane] = bias_l;
            bc[32 + lane] = alpha;
          }
          __syncwarp();
          float av[RW];
#pragma unroll
          for (int r = 0; r < RW; r += 4) {
            const float4 a4 = *reinterpret_cast<const float4*>(bc + r);
            const float4 b4 = *reinterpret_cast<const float4*>(bc + 32 + r);
            bias[r] = a4.x; bias[r + 1] = a4.y; bias[r + 2] = a4.z; bias[r + 3] = a4.w;
            av[r] = b4.x; av[r + 1] = b4.y; av[r + 2] = b4.z; av[r + 3] = b4.w;
          }
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            x[r] = ((rm >> r) & 1u) ? fmaf(sv[r], cs, bias[r]) : -INFINITY;
            lpart[r] *= av[r];
          }
          if (t > 0) {  // rescale the accumulated O columns of this group's rows
            ok = __all_sync(0xffffffffu, ok && wait_o_done(t - 1));
            if (ok) {
              tc_fence_after();
              float oh[RW], ol[RW];
              tmem_ld<RW>(o_hi, oh);
              tmem_ld<RW>(o_lo, ol);
              tmem_ld_wait();
#pragma unroll
              for (int r = 0; r < RW; ++r) {
                oh[r] *= av[r];
                ol[r] *= av[r];
              }
              tmem_st<RW>(o_hi, oh);
              tmem_st<RW>(o_lo, ol);
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

        // A key no row can see must not reach the PV product: zero its V
        // row (after its V tile has landed).  (q8_0: the converter does.)
        if (!Q8 && g == 0 && !all_vis && __any_sync(0xffffffffu, ok && rmask == 0)) {
          ok = __all_sync(0xffffffffu,
                          ok && mbar_wait(bar(BAR_VFULL + st), (t / VS) & 1, abort, wl));
          if (ok && rmask == 0) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            const uint32_t vrow = sVr + st * kKVBytes + (j / 8) * kGroupBytes + (j % 8) * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              sts_v4(vrow + c * 16, z);
              sts_v4(vrow + kAtomBytes + c * 16, z);
            }
          }
        }
        // One P buffer: PV(t-1) must have read it before P(t) goes in.  The
        // last tile waits for PV(t-1) in any case, so that the final wait
        // below is for one phase only.
        if ((PB == 1 || t == end_t - 1) && t > 0) {
          ok = __all_sync(0xffffffffu, ok && wait_o_done(t - 1));
          if (ok) tc_fence_after();
        }
        if (ok) {
          // P^T as no-swizzle MN-major core matrices [key/8][n/8][key%8]
          // [n%8], n = group * 2NR + row' with row' < NR the high parts and
          // row' >= NR the residuals, in P buffer t % PB.  Each weight (times
          // V's scale mantissa of the group, q8_0) is split into an fp16 high
          // part (truncated to 11 significant bits: exact in fp16 over the
          // weights' range) and an fp16 residual.
          const uint32_t kb = (j >> 3) * (C::kPN / 8) * 128 + (j & 7) * 16;
          constexpr uint32_t lo_off = (NR / 8) * 128;
#pragma unroll
          for (int q = 0; q < kSG; ++q) {
            const uint32_t pbuf = sP + (t % PB) * C::kPBytes + q * (2 * NR / 8) * 128;
            uint32_t phi[RW / 2], plo[RW / 2];
#pragma unroll
            for (int r = 0; r < RW; r += 2) {
              const float p0 = Q8 ? pw[r] * mv[q] : pw[r];
              const float p1 = Q8 ? pw[r + 1] * mv[q] : pw[r + 1];
              const float h0 = __uint_as_float(__float_as_uint(p0) & 0xffffe000u);
              const float h1 = __uint_as_float(__float_as_uint(p1) & 0xffffe000u);
              const __half2 h = __floats2half2_rn(h0, h1);
              const __half2 l2 = __floats2half2_rn(p0 - h0, p1 - h1);
              phi[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
              plo[r / 2] = *reinterpret_cast<const uint32_t*>(&l2);
            }
            if constexpr (RW >= 8) {
#pragma unroll
              for (int r8 = 0; r8 < RW / 8; ++r8) {
                const uint32_t off = kb + ((row0 / 8) + r8) * 128;
                sts_v4(pbuf + off,
                       make_uint4(phi[r8 * 4], phi[r8 * 4 + 1], phi[r8 * 4 + 2], phi[r8 * 4 + 3]));
                sts_v4(pbuf + lo_off + off,
                       make_uint4(plo[r8 * 4], plo[r8 * 4 + 1], plo[r8 * 4 + 2], plo[r8 * 4 + 3]));
              }
            } else {  // four rows: half of one 16-byte core-matrix row
              const uint32_t off = kb + (row0 / 8) * 128 + (row0 % 8) * 2;
              sts_v2(pbuf + off, phi[0], phi[1]);
              sts_v2(pbuf + lo_off + off, plo[0], plo[1]);
            }
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(BAR_PFULL + t % PB));
      }

      // The accumulated O^T once PV(end_t - 1) has finished: high + residual
      // (PV(end_t - 2) was waited for before the last P went out).
      float acc[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) acc[r] = 0.f;
      if (end_t >= 1) ok = __all_sync(0xffffffffu, ok && wait_o_done(end_t - 1));
      if (ok) {
        tc_fence_after();
        float oh[RW], ol[RW];
        tmem_ld<RW>(o_hi, oh);
        tmem_ld<RW>(o_lo, ol);
        tmem_ld_wait();
#pragma unroll
        for (int r = 0; r < RW; ++r) acc[r] = oh[r] + ol[r];
        tc_fence_before();
      }

      // Row sums: per-thread partials -> per-warp (lane r) -> across warps.
      const float wl = warp_row_reduce<RW, false>(lpart, lane);
      if (lane < RW) lsum[widx * 32 + lane] = wl;
      __syncwarp();
      named_bar_sync(bar_id, kSoftmaxThreads);
      __syncthreads();  // (A): also makes the K producer's bad-block mark visible
      const bool aborted = *abort != 0;
      const bool bad = misc->bad != 0;
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        if (row0 + r < R) {
          const float l = lsum[r] + lsum[32 + r] + lsum[64 + r] + lsum[96 + r];
          const long long pr = part_base + row0 + r;
          p.part_out[pr * kHeadDim + j] = (!aborted && !bad && l > 0.f) ? acc[r] / l : 0.f;
        }
      }
      if (widx == 0 && lane < RW && row0 + lane < R) {
        // lse = ln sum_j e^{z_j}: log2 sum_j 2^{cs s_j} = log2 l' + cs m - kPShift.
        // NaN marks a partial that read a stand-in for an out-of-range block.
        const float l = lsum[lane] + lsum[32 + lane] + lsum[64 + lane] + lsum[96 + lane];
        p.part_lse[part_base + row0 + lane] =
            bad ? __int_as_float(0x7fc00000)
            : (!aborted && l > 0.f)
                ? (fmaf(cs, m_lane, -(float)C::kPShift) + log2f(l)) * 0.69314718055994531f
                : -INFINITY;
      }
    }
    // ---- tear-down (every thread passed (A)) ---------------------------------
    if (threadIdx.x == 32 && misc->abort) atomicOr(p.flags, kFlagTimeout);
    tc_fence_after();
    if (warp == 1) {
      __syncwarp();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  }

  // ---- arrival and merge --------------------------------------------------------
  if (t_count == 0 && threadIdx.x == 0) misc->abort = 0;  // set by the K producer otherwise
  __syncthreads();  // (B) partials written, copies drained, TMEM freed
  // Two counters per (sequence, KV head) group (cnt, above).  After (B), one
  // thread counts the CTA in with release semantics, which publish the
  // CTA's partials (the barrier ordered their stores before it).
  if (p.coop) {
    // Every CTA of the grid is resident: a barrier over the group's S CTAs,
    // then each merges its share of the group.  The barrier needs no reset:
    // the group's first CTA adds 2^31 - (S - 1) and the others 1, so the top
    // bit of counter 0 flips once all S have arrived and its low bits return
    // to their value (zero).  The arrival does not wait for a reply; the
    // wait (acquire loads) is bounded.
    if (threadIdx.x == 0) {
      const unsigned int add = split == 0 ? 0x80000000u - (unsigned int)(S - 1) : 1u;
      red_release_add_gpu(cnt, add);
      const unsigned long long t0 = globaltimer();
      int ok = 1;
      while (((unsigned int)ld_acquire_gpu(cnt) & 0x80000000u) == bar_phase) {
        if (globaltimer() - t0 > p.wait_limit_ns) {
          ok = 0;
          break;
        }
        __nanosleep(20);
      }
      misc->last = ok;
    }
    __syncthreads();
    if (misc->last) {
      merge_slice<RW, NG, Q8>(p, s, kvh, split, S, first, smem, sbase);
    } else if (threadIdx.x == 0) {
      atomicOr(p.flags, kFlagTimeout);
    }
    return;
  }
  // Otherwise the last CTA of the group to arrive (counter 1) merges all of
  // it and sets the counter back to zero.
  if (threadIdx.x == 0) {
    __threadfence();
    misc->last = (atomicAdd(cnt + 1, 1) == S - 1);
  }
  __syncthreads();
  if (!misc->last) return;
  __threadfence();  // the other CTAs' partials, published before their counts
  merge_group<RW, NG, Q8>(p, s, kvh, S, first, smem, sbase);
  if (threadIdx.x == 0) cnt[1] = 0;
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

template <int RW, bool TR>
cudaError_t launch_rw(DecodeParams p, const CUtensorMap& mk, const CUtensorMap& mv,
                      cudaStream_t stream) {
  constexpr int NG = 2;
  auto kern = decode_split_kernel<RW, NG, false, TR>;
  const size_t smem = Cfg<RW, NG, false>::kTotal + 1024;
  // CTAs of this kernel the device holds at once (0: unknown), per device
  static std::atomic<int> resident[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int res = (dev >= 0 && dev < 64) ? resident[dev].load(std::memory_order_acquire) : 0;
  if (res == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0, sms = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Cfg<RW, NG, false>::kThreads,
                                                      smem);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    res = per_sm * sms;
    if (dev >= 0 && dev < 64) resident[dev].store(res, std::memory_order_release);
  }
  // A cooperative launch guarantees that every CTA is resident at once, which
  // the group-wide merge waits rely on; larger grids merge in their last CTA.
  p.coop = p.num_ctas <= res ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.num_ctas);
  cfg.blockDim = dim3(Cfg<RW, NG, false>::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // Programmatic stream serialization lets this grid's CTAs be scheduled
  // while the previous kernel drains (they wait in griddepcontrol.wait).
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
  CUtensorMap mk, mv;
  const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
  if (!encode_cache_map(&mk, p.k, rows) || !encode_cache_map(&mv, p.v, rows))
    return cudaErrorInvalidValue;
  // Two softmax warpgroups of RW rows each.
  if (p.rows <= 8) return launch_rw<4, TR>(p, mk, mv, stream);
  if (p.rows <= 16) return launch_rw<8, TR>(p, mk, mv, stream);
  return launch_rw<16, TR>(p, mk, mv, stream);
}

}  // namespace
}  // namespace split

bool split_decode_supported(int kv_dtype, int n_query, int rows, int num_blocks,
                            int num_kv_heads, int block_size) {
  return kv_dtype == kKvFp16 && n_query >= 1 && n_query <= split::kMaxQuery && rows >= 1 &&
         rows <= 32 && block_size % kChunk == 0 &&
         (long long)num_blocks * num_kv_heads * block_size <= INT32_MAX;
}

cudaError_t launch_split_decode(const DecodeParams& c, int ctas, cudaStream_t stream) {
  split::DecodeParams p{};
  p.q = c.q;
  p.k = c.k;
  p.v = c.v;
  p.block_table = c.block_table;
  p.context_lens = c.context_lens;
  p.num_seqs = c.num_seqs;
  p.num_q_heads = c.num_q_heads;
  p.num_kv_heads = c.num_kv_heads;
  p.block_size = c.block_size;
  p.max_blocks_per_seq = c.max_blocks_per_seq;
  p.num_blocks = c.num_blocks;
  p.n_query = c.n_query;
  p.causal = c.causal;
  p.window = c.window;
  p.kv_dtype = split::kKvFp16;
  p.group = c.group;
  p.rows = c.rows;
  p.scale_log2 = c.scale_log2;
  const int groups = c.num_seqs * c.num_kv_heads;
  p.num_splits = (ctas + groups - 1) / groups;
  p.num_ctas = ctas;
  p.tiles_per_item = 0;
  p.blocks_per_split = (c.max_blocks_per_seq + p.num_splits - 1) / p.num_splits;
  p.part_out = c.part_out;
  p.part_lse = c.part_lse;
  p.flags = c.flags;
  p.arrivals = c.arrivals;
  p.out = c.out;
  p.trace = c.trace;
  p.wait_limit_ns = c.wait_limit_ns;
  return c.trace != nullptr ? split::launch_any<true>(p, stream)
                            : split::launch_any<false>(p, stream);
}

}  // namespace pa
