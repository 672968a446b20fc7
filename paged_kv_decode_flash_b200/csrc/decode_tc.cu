// decode_tc.cu -- split-KV paged decode attention on the sm_100a tensor
// cores (tcgen05 + TMEM), with TMA staging of the paged KV tiles.
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
// Hardware mapping (one CTA per SM, 11 warps):
//   warps 0, 10 TMA producers for K and for V: resolve the block table and
//               load whole 16-key chunks (two 64-column halves each, 128-byte
//               swizzle) into separate 3-slot rings of 128-key tiles; K slots
//               are released as soon as QK^T has read them, so K runs ahead.
//   warp 1      MMA issuer (one thread): S^T = K Q^T with M = 128 keys and
//               N = the query rows, then O^T = V^T [P_hi | P_lo]^T with
//               M = 128 head_dim lanes; accumulators live in TMEM.
//   warps 2-9   two softmax warpgroups, each owning half of the query rows:
//               thread = key for S (row max by a warp transpose-reduction
//               plus one named barrier per group), thread = head_dim element
//               for O (running accumulators in registers).
// Putting keys and head_dim on the MMA's M side keeps the tensor core free of
// padding even at 4-32 query rows.
//
// Exactness: Q, K and V are fed to the tensor core as the exact fp16 inputs.
// The softmax weights are scaled by 2^14 (so that weights down to ~4e-12 of
// the row maximum stay representable) and split into an fp16 high part and
// an fp16 residual; both are multiplied with V and accumulated in fp32, which
// keeps the weights to about 2^-22 relative.  Keys no query row can see are
// never multiplied: their chunks are not loaded when wholly outside the
// visible range, their scores are selected to -inf, and their V rows are
// zero-filled in shared memory before the PV product (the NaN-poisoned
// out-of-window blocks of the pages' regression test must not leak).
//
// Every wait is bounded (sm100::mbar_wait): on a timeout the kernel raises
// kFlagTimeout, drains its own copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace pa {
namespace {

using namespace sm100;

constexpr int kTileKeys = 128;                 // keys per pipeline tile (M of S^T)
constexpr int kChunksPerTile = kTileKeys / kChunk;
constexpr int kStages = 3;                     // slots per K ring and per V ring
// A K or V tile of 128 keys in shared memory: [key group of 8][half][8 keys]
// [64 fp16] with the 128-byte swizzle, i.e. 1 KB swizzle atoms; the atoms of
// one 64-column half sit 2 KB apart, the two halves of a key group 1 KB apart.
// One 16-key chunk (a contiguous 4 KB (block, head) tile in the cache for
// block_size 16) is a single TMA box.
constexpr uint32_t kAtomBytes = 1024;              // 8 keys x 128 bytes
constexpr uint32_t kGroupBytes = 2 * kAtomBytes;   // both halves of 8 keys
constexpr uint32_t kKVBytes = kTileKeys / 8 * kGroupBytes;  // one K (or V) tile
constexpr uint32_t kChunkBytes = kChunk * 256;     // one 16-key chunk (TMA box)
constexpr int kGroups = 2;                     // softmax warpgroups (split the rows)
constexpr int kSoftmaxThreads = 128;           // per warpgroup
constexpr int kVWarp = 2 + kGroups * 4;        // the V producer's warp
constexpr int kThreads = 32 * (kVWarp + 1);
constexpr int kPShift = 14;                    // weights scaled by 2^14 before fp16
// A row's reference max is only raised when a score passes it by more than
// kLazy (log2 units); scaled weights then stay below 2^(kPShift + kLazy),
// inside fp16 range.
constexpr float kLazy = 1.5f;

enum : int {
  BAR_KFULL = 0,    // [3] K tile landed
  BAR_KEMPTY = 3,   // [3] K tile read by QK^T
  BAR_VFULL = 6,    // [3] V tile landed
  BAR_VEMPTY = 9,   // [3] V tile read by PV
  BAR_SFULL = 12,   // [2] S^T in TMEM
  BAR_SEMPTY = 14,  // [2] S^T read by the softmax warps
  BAR_PFULL = 16,   // P written to shared memory
  BAR_PEMPTY = 17,  // P consumed by the PV product
  BAR_OFULL = 18,   // [2] O^T of one tile in TMEM
  BAR_OEMPTY = 20,  // [2] O^T read by the softmax warps
  BAR_DONE = 22,    // every MMA finished
  BAR_INFO = 23,    // [8] a tile's number, chunk mask and cache rows published
  BAR_COUNT = 31
};
constexpr int kInfoSlots = 8;  // depth of the tile-information ring

// RW query rows per softmax warpgroup; NR = the MMA's N for S (>= 16).
template <int RW>
struct Cfg {
  static constexpr int NR = (kGroups * RW < 16) ? 16 : kGroups * RW;
  static constexpr uint32_t kK = 0;                                 // K ring
  static constexpr uint32_t kV = kStages * kKVBytes;                // V ring
  static constexpr uint32_t kQ = 2 * kStages * kKVBytes;
  static constexpr uint32_t kQHalf = NR * 128;
  // P^T of one tile: 2*NR "rows" (the fp16 high parts of the NR query rows,
  // then their residuals), so one MMA with N = 2*NR multiplies both.
  static constexpr uint32_t kP = kQ + 2 * kQHalf;
  static constexpr uint32_t kPBytes = kTileKeys * 2 * NR * 2;
  static constexpr uint32_t kRed = kP + kPBytes;                    // float [2 grp][2][4][32]
  static constexpr uint32_t kAlpha = kRed + kGroups * 2 * 4 * 32 * 4;  // float [4][32]
  static constexpr uint32_t kLsum = kAlpha + 4 * 32 * 4;            // float [2 grp][4][32]
  static constexpr uint32_t kBcast = kLsum + kGroups * 4 * 32 * 4;  // float [8 warps][2][32]
  static constexpr uint32_t kBars = kBcast + kGroups * 4 * 2 * 32 * 4;  // uint64 [32]
  static constexpr uint32_t kInfo = kBars + 32 * 8;                 // TileInfo [8]
  static constexpr uint32_t kMisc = kInfo + kInfoSlots * 48;        // small ints
  static constexpr uint32_t kTotal = kMisc + 64;
  // TMEM columns: S^T[2] (NR each) then O^T[2] (2*NR each: high | residual).
  static constexpr uint32_t kTmemUsed = 6 * NR;
  static constexpr uint32_t kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64
                                        : kTmemUsed <= 128 ? 128 : 256;
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  int k_consumed, v_consumed;
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

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
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

template <int RW>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using C = Cfg<RW>;
  constexpr int NR = C::NR;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, derived from the __shared__ array by pointer
  // arithmetic so that accesses through it stay shared-space loads/stores.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + C::kMisc);
  TileInfo* info = reinterpret_cast<TileInfo*>(smem + C::kInfo);
  volatile int* abort = &misc->abort;
  auto bar = [&](int i) { return sbase + C::kBars + 8u * i; };

  const int split = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int S = p.num_splits;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nq = p.n_query, G = p.group, Hq = p.num_q_heads, R = p.rows;
  const int rps = nq * Hq;
  const long long part_base = ((long long)s * S + split) * rps;
  auto row_index = [&](int r) { return (r / G) * Hq + kvh * G + (r % G); };

  // ---- the head's visible keys and its tiles (uniform across the CTA) ------
  // The keys of (sequence s, KV head kvh) that any query token sees form
  // [lo_u, hi_u]; they are cut into 128-key tiles from `base`, and the S
  // splits take contiguous runs of them, as even as whole tiles allow.  The
  // partition depends only on the context length and S, so every call on the
  // same inputs adds the same tiles in the same order: results are
  // bit-reproducible.
  const int L = p.context_lens[s];
  int lo_u = 0, hi_u = -1;
  if (context_len_ok(L, nq, p.max_blocks_per_seq, p.block_size)) {
    union_range(L, nq, p.causal, p.window, lo_u, hi_u);
  } else if (split == 0 && kvh == 0 && threadIdx.x == 0) {
    atomicOr(p.flags, kFlagBadLen);
  }
  const int base = (lo_u / kChunk) * kChunk;
  const int ntiles_h = hi_u >= lo_u ? (hi_u + 1 - base + kTileKeys - 1) / kTileKeys : 0;
  const int t_per = ntiles_h / S, t_rem = ntiles_h % S;
  const int t_first = split * t_per + min(split, t_rem);
  const int t_count = t_per + (split < t_rem ? 1 : 0);
  if (t_count == 0) {  // every tile is another CTA's: an empty partial
    for (int t = threadIdx.x; t < R * kHeadDim; t += kThreads) {
      const int r = t / kHeadDim;
      p.part_out[(part_base + row_index(r)) * kHeadDim + t % kHeadDim] = 0.f;
      if (t % kHeadDim == 0) p.part_lse[part_base + row_index(r)] = -INFINITY;
    }
    griddep_launch_dependents();
    return;
  }
  const int* table = p.block_table + (long long)s * p.max_blocks_per_seq;

  const uint32_t sKr = sbase + C::kK, sVr = sbase + C::kV;
  const uint32_t sQ = sbase + C::kQ, sP = sbase + C::kP;

  if (warp == 0) {
    // ======================= K producer (also sets up the barriers) ========
    if (lane == 0) {
      for (int i = 0; i < kStages; ++i) {
        mbar_init(bar(BAR_KFULL + i), 1);
        mbar_init(bar(BAR_KEMPTY + i), 1);
        mbar_init(bar(BAR_VFULL + i), 1);
        mbar_init(bar(BAR_VEMPTY + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(BAR_SFULL + i), 1);
        mbar_init(bar(BAR_SEMPTY + i), 4 * kGroups);
        mbar_init(bar(BAR_OFULL + i), 1);
        mbar_init(bar(BAR_OEMPTY + i), 4 * kGroups);
      }
      mbar_init(bar(BAR_PFULL), 4 * kGroups);
      mbar_init(bar(BAR_PEMPTY), 1);
      mbar_init(bar(BAR_DONE), 1);
      for (int i = 0; i < kInfoSlots; ++i) mbar_init(bar(BAR_INFO + i), 1);
      misc->abort = 0;
      misc->k_consumed = misc->v_consumed = 0;
      fence_mbar_init();
    }
    __syncwarp();
    // The other roles wait for these barriers; this warp starts loading now.
    named_bar_arrive(3, kThreads);

    // Lane c < 8 owns chunk c of every tile and reads its block-table entry
    // one tile ahead.
    const int c = lane;
    auto lookup = [&](int g, int& row8) -> bool {
      if (g < 0 || c >= kChunksPerTile) return false;
      const int key0 = base + g * kTileKeys + c * kChunk;
      if (key0 > hi_u || key0 + kChunk - 1 < lo_u) return false;
      const long long phys = table[key0 / p.block_size];
      if (phys < 0 || phys >= p.num_blocks) {
        atomicOr(p.flags, kFlagBadBlock);  // masked, never dereferenced
        return false;
      }
      row8 = (int)(((phys * p.num_kv_heads + kvh) * p.block_size + key0 % p.block_size) / 8);
      return true;
    };
    auto tile_of = [&](int t) { return t < t_count ? t_first + t : -1; };
    int g_cur = tile_of(0);
    int row_cur = 0, row_nxt = 0;
    bool w_cur = lookup(g_cur, row_cur);
    int issued = 0;
    for (int t = 0;; ++t) {
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
      // Tile t + 1's block-table entries, read while tile t's slot frees up.
      const int g_nxt = tile_of(t + 1);
      const bool w_nxt = lookup(g_nxt, row_nxt);
      // Wait for the slot, then every lane issues its chunk's copy.
      const int st = t % kStages;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar(BAR_KEMPTY + st), ((t / kStages) & 1) ^ 1, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const uint32_t fb = bar(BAR_KFULL + st);
      if (lane == 0) mbar_arrive_expect_tx(fb, __popc(mask) * kChunkBytes);
      __syncwarp();
      if (w_cur) tma_load_4d(sKr + st * kKVBytes + c * kChunkBytes, &tmap_k, 0, 0, 0, row_cur, fb);
      __syncwarp();
      issued = t + 1;
      g_cur = g_nxt;
      w_cur = w_nxt;
      row_cur = row_nxt;
    }
    __syncthreads();  // (A) every role finished its loop
    if (lane == 0) {  // drain copies that no MMA waited for (abort path only)
      volatile int no_abort = 0;
      for (int t = misc->k_consumed; t < issued; ++t)
        mbar_wait(bar(BAR_KFULL + t % kStages), (t / kStages) & 1, &no_abort);
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
      for (uint32_t off = t * 16; off < C::kPBytes; off += kGroups * kSoftmaxThreads * 16)
        sts_v4(sP + off, make_uint4(0, 0, 0, 0));
      fence_proxy_async_smem();
    }
    tc_fence_before();
    named_bar_sync(3, kThreads);  // barriers initialised, TMEM allocated, Q staged
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
          ok = mbar_wait(bar(BAR_INFO + t % kInfoSlots), (t / kInfoSlots) & 1, abort);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // lane 0's acquire orders the other lanes' reads below
        if (!ok) break;
        const TileInfo& ti = info[t % kInfoSlots];
        if (ti.tile < 0) break;
        const uint32_t mask = ti.mask;
        const int row8 = c < kChunksPerTile ? ti.row8[c] : 0;
        const int st = t % kStages;
        if (lane == 0) ok = mbar_wait(bar(BAR_VEMPTY + st), ((t / kStages) & 1) ^ 1, abort);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const uint32_t fb = bar(BAR_VFULL + st);
        if (lane == 0) mbar_arrive_expect_tx(fb, __popc(mask) * kChunkBytes);
        __syncwarp();
        if (c < kChunksPerTile && ((mask >> c) & 1u))
          tma_load_4d(sVr + st * kKVBytes + c * kChunkBytes, &tmap_v, 0, 0, 0, row8, fb);
        __syncwarp();
        issued = t + 1;
      }
      __syncthreads();  // (A)
      if (lane == 0) {  // drain copies that no MMA waited for (abort path only)
        volatile int no_abort = 0;
        for (int t = misc->v_consumed; t < issued; ++t)
          mbar_wait(bar(BAR_VFULL + t % kStages), (t / kStages) & 1, &no_abort);
      }
    } else if (warp == 1) {
      // ===================== MMA issuer ======================================
      if (lane == 0) {
        const uint32_t id_qk = idesc_f16_f32(128, NR, false, false);
        const uint32_t id_pv = idesc_f16_f32(128, 2 * NR, true, true);
        // Descriptors at offset 0; a byte offset o is added as o >> 4 (the
        // start-address field is the low 14 bits, addresses stay < 256 KB).
        const uint64_t dK = smem_desc(sKr, 16, kGroupBytes, kSwizzle128B);
        const uint64_t dQ = smem_desc(sQ, 16, 1024, kSwizzle128B);
        const uint64_t dV = smem_desc(sVr, kAtomBytes, kGroupBytes, kSwizzle128B);
        const uint64_t dP = smem_desc(sP, 2 * NR * 16, 128, kSwizzleNone);
        int nqk = 0;              // QK^T products issued
        int end_t = 0x7fffffff;   // number of tiles, once the producer said so
        // Issue QK^T of tile nqk if it exists and its K tile and S buffer are
        // ready (or wait for them when `block`).  1 = issued, 0 = not ready or
        // no such tile, -1 = gave up.
        auto try_qk = [&](bool block) -> int {
          if (nqk >= end_t) return 0;
          const uint32_t ib = bar(BAR_INFO + nqk % kInfoSlots), ip = (nqk / kInfoSlots) & 1;
          if (block) {
            if (!mbar_wait(ib, ip, abort)) return -1;
          } else if (!mbar_test_wait(ib, ip)) {
            return 0;
          }
          if (info[nqk % kInfoSlots].tile < 0) {
            end_t = nqk;
            return 0;
          }
          const uint32_t f = bar(BAR_KFULL + nqk % kStages), e = bar(BAR_SEMPTY + nqk % 2);
          const uint32_t pf = (nqk / kStages) & 1, pe = ((nqk / 2) & 1) ^ 1;
          if (block) {
            if (!(mbar_wait(f, pf, abort) && mbar_wait(e, pe, abort))) return -1;
          } else if (!(mbar_test_wait(f, pf) && mbar_test_wait(e, pe))) {
            return 0;
          }
          tc_fence_after();
          const uint64_t so = (uint64_t)((nqk % kStages) * kKVBytes) >> 4;
          const uint32_t d = tmem + (nqk % 2) * NR;
#pragma unroll
          for (int k = 0; k < kHeadDim / 16; ++k) {
            const uint64_t ko = ((k / 4) * kAtomBytes + (k % 4) * 32) >> 4;
            const uint64_t qo = ((k / 4) * C::kQHalf + (k % 4) * 32) >> 4;
            tc_mma_f16_ss(d, dK + so + ko, dQ + qo, id_qk, k > 0);
          }
          tc_commit(bar(BAR_SFULL + nqk % 2));
          tc_commit(bar(BAR_KEMPTY + nqk % kStages));
          ++nqk;
          return 1;
        };
        int npv = 0;
        bool ok = true;
        for (int t = 0; ok; ++t) {
          if (nqk <= t && try_qk(true) < 0) { ok = false; break; }  // QK(t) comes first
          if (t >= end_t) break;                                     // no tile t
          if (nqk == t + 1) try_qk(false);
          // Wait for P(t), issuing QK(t+1) as soon as its K tile lands.
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait_ns(bar(BAR_PFULL), t & 1, 200)) {
            if (nqk == t + 1) try_qk(false);
            if (*abort || globaltimer() - t0 > kWaitLimitNs) { *abort = 1; ok = false; break; }
          }
          if (!ok) break;
          ok = mbar_wait(bar(BAR_VFULL + t % kStages), (t / kStages) & 1, abort) &&
               mbar_wait(bar(BAR_OEMPTY + t % 2), ((t / 2) & 1) ^ 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint64_t so = (uint64_t)((t % kStages) * kKVBytes) >> 4;
          const uint32_t d = tmem + 2 * NR + (t % 2) * 2 * NR;
#pragma unroll
          for (int k = 0; k < kTileKeys / 16; ++k) {
            const uint64_t vo = (k * 2 * kGroupBytes) >> 4;
            const uint64_t po = (k * 2 * 2 * NR * 16) >> 4;
            tc_mma_f16_ss(d, dV + so + vo, dP + po, id_pv, k > 0);
          }
          tc_commit(bar(BAR_OFULL + t % 2));
          tc_commit(bar(BAR_PEMPTY));
          tc_commit(bar(BAR_VEMPTY + t % kStages));
          npv = t + 1;
          if (nqk == t + 1) try_qk(false);
        }
        misc->k_consumed = nqk;
        misc->v_consumed = npv;
        tc_commit(bar(BAR_DONE));  // completes once every MMA above has finished
        volatile int no_abort = 0;
        mbar_wait(bar(BAR_DONE), 0, &no_abort);
      }
      __syncwarp();
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
      float* alpha_s = reinterpret_cast<float*>(smem + C::kAlpha);             // [4][32]
      float* lsum = reinterpret_cast<float*>(smem + C::kLsum) + g * 4 * 32;    // [4][32]
      float* bc = reinterpret_cast<float*>(smem + C::kBcast) + (warp - 2) * 64;  // [2][32]
      const uint32_t bar_id = 1 + g;
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

      float acc[RW], lpart[RW], bias[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        acc[r] = lpart[r] = 0.f;
        bias[r] = INFINITY;  // no reference yet: the row's first key forces one
      }
      // Reference max (raw score) of row row0 + lane % RW; -inf until the
      // row sees a key.  bias[r] = kPShift - cs * (row r's reference max).
      float m_lane = -INFINITY;
      bool ok = true;
      int end_t = 0x7fffffff;  // number of tiles, once published

      // Iteration t scores tile t and folds tile t-2's O^T (finished long
      // ago) into the register accumulators; the two iterations after the
      // last tile only fold.  Tile u's rescale factors live in alpha_s[u % 4].
      for (int t = 0;; ++t) {
        int gt = -1;  // tile number of local tile t
        if (t < end_t) {
          ok = __all_sync(0xffffffffu,
                          ok && mbar_wait(bar(BAR_INFO + t % kInfoSlots),
                                          (t / kInfoSlots) & 1, abort));
          gt = ok ? info[t % kInfoSlots].tile : -1;
          if (gt < 0) end_t = t;
        }
        if (t - 2 >= end_t) break;  // the last tile (end_t - 1) was folded at end_t + 1
        const bool has_s = t < end_t, has_o = t >= 2;
        const int sb = t % 2, st = t % kStages, ob = t % 2;  // O of tile t-2 sits in buffer t%2
        if (has_o)
          ok = __all_sync(0xffffffffu,
                          ok && mbar_wait(bar(BAR_OFULL + ob), ((t - 2) / 2) & 1, abort));
        if (has_s)
          ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_SFULL + sb), (t / 2) & 1, abort));
        float sv[RW], oh[RW], ol[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) sv[r] = oh[r] = ol[r] = 0.f;
        if (ok) {
          tc_fence_after();
          if (has_o) {
            tmem_ld<RW>(tmem + lane_off + 2 * NR + ob * 2 * NR + row0, oh);
            tmem_ld<RW>(tmem + lane_off + 2 * NR + ob * 2 * NR + NR + row0, ol);
          }
          if (has_s) tmem_ld<RW>(tmem + lane_off + sb * NR + row0, sv);
          tmem_ld_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) {
          if (has_o) mbar_arrive(bar(BAR_OEMPTY + ob));
          if (has_s) mbar_arrive(bar(BAR_SEMPTY + sb));
        }

        uint32_t rmask = 0;
        bool all_vis = false;  // every key of this warp is seen by every row
        float x[RW];           // cs * s + bias: log2 of the scaled weight
        bool exceed = false;
        if (has_s) {
          // Which rows see this key?  Keys of chunks that were not loaded
          // (outside the visible range or an out-of-range block) see none.
          const int key = base + gt * kTileKeys + j;
          if (ok && ((info[t % kInfoSlots].mask >> (j / kChunk)) & 1u) && key >= lo_u &&
              key <= hi_u) {
            if (key >= lo_all && key <= hi_all) {
              rmask = all_rows;
            } else {
#pragma unroll
              for (int i = 0; i < kMaxQuery; ++i)
                if (i < nq && key >= tlo[i] && key <= thi[i]) rmask |= grp << (i * G);
            }
          }
          all_vis = __all_sync(0xffffffffu, rmask == all_rows);
          const uint32_t rm = rmask >> row0;
#pragma unroll
          for (int r = 0; r < RW; ++r) {
            x[r] = fmaf(sv[r], cs, bias[r]);
            const bool vis = all_vis || ((rm >> r) & 1u);
            exceed |= vis && x[r] > (float)kPShift + kLazy;
          }
        }
        // Reconverge before the group barrier: a warp that arrives diverged
        // (after lane-predicated code) makes the barrier several times slower
        // (measured: 61k verify 122 -> 67 us per call).
        __syncwarp();
        // One barrier per tile: orders the shared-memory traffic of the group
        // and tells every thread whether any score passed its row's reference.
        const bool rescale = named_bar_or(bar_id, kSoftmaxThreads, exceed);
        if (has_o && ok) {  // acc = acc * alpha_{t-2} + O_{t-2} (high + residual)
          const float* al = alpha_s + ((t - 2) % 4) * 32 + row0;
#pragma unroll
          for (int r = 0; r < RW; ++r) acc[r] = fmaf(acc[r], al[r], oh[r] + ol[r]);
        }
        if (has_s) {
          const uint32_t rm = rmask >> row0;
          float alpha = 1.f;
          if (rescale) {
            // New reference max per row: warp transpose-reduction, then
            // across the group's four warps.
            float tmp[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r)
              tmp[r] = (all_vis || ((rm >> r) & 1u)) ? sv[r] : -INFINITY;
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
            alpha = (m_new == -INFINITY) ? 1.f : fast_exp2(cs * (m_lane - m_new));
            const float bias_l =
                (m_new == -INFINITY) ? INFINITY : fmaf(-cs, m_new, (float)kPShift);
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
              x[r] = fmaf(sv[r], cs, bias[r]);
              lpart[r] *= av[r];
            }
          }
          if (widx == 0 && lane < RW) alpha_s[(t % 4) * 32 + row0 + lane] = alpha;

          // Scaled weights, split into an fp16 high part and an fp16 residual.
          uint32_t phi[RW / 2], plo[RW / 2];
#pragma unroll
          for (int r = 0; r < RW; r += 2) {
            float pr[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const bool vis = all_vis || ((rm >> (r + e)) & 1u);
              pr[e] = vis ? fast_exp2(x[r + e]) : 0.f;
              lpart[r + e] += pr[e];
            }
            const __half2 h = __floats2half2_rn(pr[0], pr[1]);
            const float2 hf = __half22float2(h);
            const __half2 l2 = __floats2half2_rn(pr[0] - hf.x, pr[1] - hf.y);
            phi[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
            plo[r / 2] = *reinterpret_cast<const uint32_t*>(&l2);
          }

          // A key no row can see must not reach the PV product: zero its V
          // row (after its V tile has landed).
          if (g == 0 && __any_sync(0xffffffffu, ok && rmask == 0)) {
            ok = __all_sync(0xffffffffu,
                            ok && mbar_wait(bar(BAR_VFULL + st), (t / kStages) & 1, abort));
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
          ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_PEMPTY), (t & 1) ^ 1, abort));
          if (ok) {
            // P^T as no-swizzle MN-major core matrices [key/8][row'/8][key%8]
            // [row'%8] with row' < NR the high parts and row' >= NR the
            // residuals.
            const uint32_t kb = (j >> 3) * (2 * NR / 8) * 128 + (j & 7) * 16;
            constexpr uint32_t lo_off = (NR / 8) * 128;
            if constexpr (RW >= 8) {
#pragma unroll
              for (int r8 = 0; r8 < RW / 8; ++r8) {
                const uint32_t off = kb + ((row0 / 8) + r8) * 128;
                sts_v4(sP + off,
                       make_uint4(phi[r8 * 4], phi[r8 * 4 + 1], phi[r8 * 4 + 2], phi[r8 * 4 + 3]));
                sts_v4(sP + lo_off + off,
                       make_uint4(plo[r8 * 4], plo[r8 * 4 + 1], plo[r8 * 4 + 2], plo[r8 * 4 + 3]));
              }
            } else {  // four rows: half of one 16-byte core-matrix row
              const uint32_t off = kb + (row0 / 8) * 128 + (row0 % 8) * 2;
              sts_v2(sP + off, phi[0], phi[1]);
              sts_v2(sP + lo_off + off, plo[0], plo[1]);
            }
            fence_proxy_async_smem();
          }
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(bar(BAR_PFULL));
        }
      }

      // Row sums: per-thread partials -> per-warp (lane r) -> across warps.
      const float wl = warp_row_reduce<RW, false>(lpart, lane);
      if (lane < RW) lsum[widx * 32 + lane] = wl;
      __syncwarp();
      named_bar_sync(bar_id, kSoftmaxThreads);
      const bool aborted = *abort != 0;
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        if (row0 + r < R) {
          const float l = lsum[r] + lsum[32 + r] + lsum[64 + r] + lsum[96 + r];
          const long long pr = part_base + row_index(row0 + r);
          p.part_out[pr * kHeadDim + j] = (!aborted && l > 0.f) ? acc[r] / l : 0.f;
        }
      }
      if (widx == 0 && lane < RW && row0 + lane < R) {
        // lse = ln sum_j e^{z_j}: log2 sum_j 2^{cs s_j} = log2 l' + cs m - kPShift.
        const float l = lsum[lane] + lsum[32 + lane] + lsum[64 + lane] + lsum[96 + lane];
        p.part_lse[part_base + row_index(row0 + lane)] =
            (!aborted && l > 0.f)
                ? (fmaf(cs, m_lane, -(float)kPShift) + log2f(l)) * 0.69314718055994531f
                : -INFINITY;
      }
      __syncthreads();  // (A)
    }
    // ---- tear-down (every thread passed (A)) ---------------------------------
    if (threadIdx.x == 32 && misc->abort) atomicOr(p.flags, kFlagTimeout);
    tc_fence_after();
    if (warp == 1) {
      __syncwarp();
      tmem_dealloc(tmem, C::kTmemCols);
    }
  }
  // This CTA's partial is written: the merge kernel that follows on the
  // stream may be scheduled (it waits for the whole grid before reading).
  // Triggering any earlier lets idle merge CTAs share the SMs with the
  // decode and slows it (measured: 61k verify 64 -> 70 us per call).
  griddep_launch_dependents();
}

// ---- host side ----------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
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

template <int RW>
cudaError_t launch_rw(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                      cudaStream_t stream) {
  const size_t smem = Cfg<RW>::kTotal + 1024;
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel<RW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const dim3 grid(p.num_splits, p.num_kv_heads, p.num_seqs);
  decode_tc_kernel<RW><<<grid, kThreads, smem, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(int kv_dtype, int rows, int num_blocks, int num_kv_heads, int block_size) {
  return kv_dtype == kKvFp16 && rows >= 1 && rows <= 2 * 16 &&
         (long long)num_blocks * num_kv_heads * block_size <= INT32_MAX;
}

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream) {
  CUtensorMap mk, mv;
  const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
  if (!encode_cache_map(&mk, p.k, rows) || !encode_cache_map(&mv, p.v, rows))
    return cudaErrorInvalidValue;
  if (p.rows <= 8) return launch_rw<4>(p, mk, mv, stream);
  if (p.rows <= 16) return launch_rw<8>(p, mk, mv, stream);
  return launch_rw<16>(p, mk, mv, stream);
}

}  // namespace pa
