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
// Hardware mapping (one CTA per SM, 6 warps):
//   warp 0      TMA producer: resolves the block table, loads whole 16-key
//               chunks of K and V (two 64-column halves each, 128-byte
//               swizzle) into a 3-stage ring of 128-key tiles.
//   warp 1      MMA issuer (one thread): S^T = K Q^T with M = 128 keys and
//               N = the query rows (16 or 32), then O^T = V^T P^T with
//               M = 128 head_dim lanes; accumulators live in TMEM.
//   warps 2-5   softmax and correction: thread = key for S (row max by a
//               warp transpose-reduction plus one named barrier), thread =
//               head_dim element for O (running accumulators in registers).
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
constexpr int kStages = 3;
constexpr uint32_t kHalfBytes = kTileKeys * 128;   // 64 fp16 columns of 128 keys
constexpr uint32_t kKVBytes = 2 * kHalfBytes;      // one K (or V) tile
constexpr uint32_t kStageBytes = 2 * kKVBytes;     // K then V
constexpr uint32_t kChunkBytes = kChunk * 128;     // one 16-key half-chunk (TMA box)
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr int kPShift = 14;                    // weights scaled by 2^14 before fp16

enum : int {
  BAR_FULL = 0,     // [3] TMA tile landed
  BAR_EMPTY = 3,    // [3] stage consumed (PV done)
  BAR_SFULL = 6,    // [2] S^T in TMEM
  BAR_SEMPTY = 8,   // [2] S^T read by the softmax warps
  BAR_PFULL = 10,   // P written to shared memory
  BAR_PEMPTY = 11,  // P consumed by the PV product
  BAR_OFULL = 12,   // [2] O^T of one tile in TMEM
  BAR_OEMPTY = 14,  // [2] O^T read by the correction
  BAR_DONE = 16,    // every MMA finished
  BAR_COUNT = 17
};

template <int NR>
struct Layout {
  static constexpr uint32_t kQ = kStages * kStageBytes;
  static constexpr uint32_t kQHalf = NR * 128;
  static constexpr uint32_t kPHi = kQ + 2 * kQHalf;
  static constexpr uint32_t kPBytes = kTileKeys * NR * 2;
  static constexpr uint32_t kPLo = kPHi + kPBytes;
  static constexpr uint32_t kRed = kPLo + kPBytes;            // float [2][4][32]
  static constexpr uint32_t kAlpha = kRed + 2 * 4 * 32 * 4;   // float [2][32]
  static constexpr uint32_t kLsum = kAlpha + 2 * 32 * 4;      // float [4][32]
  static constexpr uint32_t kBars = kLsum + 4 * 32 * 4;       // uint64 [24]
  static constexpr uint32_t kMisc = kBars + 24 * 8;           // small ints
  static constexpr uint32_t kTotal = kMisc + 64;
  static constexpr uint32_t kTmemCols = 4 * NR;              // S[2], O[2]
};

struct Misc {
  uint32_t tmem_base;
  int abort;
  uint32_t chunk_mask[kStages];
  int n_consumed;
};

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

// Warp transpose-reduction: lane l ends with op over all 32 lanes of row
// (l % NR) in v[0].
template <int NR, bool kMax>
__device__ __forceinline__ float warp_row_reduce(float (&v)[NR], int lane) {
#pragma unroll
  for (int n = NR, o = NR / 2; n > 1; n >>= 1, o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  if constexpr (NR == 16) {
    const float got = __shfl_xor_sync(0xffffffffu, v[0], 16);
    v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
  }
  return v[0];
}

template <int NR>
__global__ void __launch_bounds__(kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
  using Lay = Layout<NR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  Misc* misc = reinterpret_cast<Misc*>(smem + Lay::kMisc);
  volatile int* abort = &misc->abort;
  auto bar = [&](int i) { return sbase + Lay::kBars + 8u * i; };

  const int split = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int nq = p.n_query, G = p.group, Hq = p.num_q_heads, R = p.rows;
  const int rps = nq * Hq;
  const long long part_base = ((long long)s * p.num_splits + split) * rps;
  auto row_index = [&](int r) { return (r / G) * Hq + kvh * G + (r % G); };

  // ---- the CTA's key range (uniform across the CTA) -----------------------
  const int L = p.context_lens[s];
  int k0 = 0, k1 = -1;
  const bool len_ok = context_len_ok(L, nq, p.max_blocks_per_seq, p.block_size);
  if (len_ok) {
    int lo_u, hi_u;
    union_range(L, nq, p.causal, p.window, lo_u, hi_u);
    const long long sk0 = (long long)split * p.blocks_per_split * p.block_size;
    const long long sk1 = sk0 + (long long)p.blocks_per_split * p.block_size - 1;
    k0 = (int)max((long long)lo_u, sk0);
    k1 = (int)min((long long)hi_u, sk1);
  } else if (split == 0 && kvh == 0 && threadIdx.x == 0) {
    atomicOr(p.flags, kFlagBadLen);
  }
  if (k0 > k1) {  // nothing visible here: an empty partial
    for (int t = threadIdx.x; t < R * kHeadDim; t += kThreads) {
      const int r = t / kHeadDim;
      p.part_out[(part_base + row_index(r)) * kHeadDim + t % kHeadDim] = 0.f;
      if (t % kHeadDim == 0) p.part_lse[part_base + row_index(r)] = -INFINITY;
    }
    return;
  }
  const int base = (k0 / kChunk) * kChunk;
  const int ntiles = (k1 + 1 - base + kTileKeys - 1) / kTileKeys;

  // ---- set-up ---------------------------------------------------------------
  if (warp == 1) {
    tmem_alloc(sbase + Lay::kMisc + offsetof(Misc, tmem_base), Lay::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(BAR_FULL + i), 1);
      mbar_init(bar(BAR_EMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BAR_SFULL + i), 1);
      mbar_init(bar(BAR_SEMPTY + i), 4);
      mbar_init(bar(BAR_OFULL + i), 1);
      mbar_init(bar(BAR_OEMPTY + i), 4);
    }
    mbar_init(bar(BAR_PFULL), 4);
    mbar_init(bar(BAR_PEMPTY), 1);
    mbar_init(bar(BAR_DONE), 1);
    misc->abort = 0;
    misc->n_consumed = 0;
    fence_mbar_init();
  }
  if (warp >= 2) {
    // Q rows of this KV head -> shared memory, K-major with 128-byte swizzle:
    // row n, 16-byte chunk c of half h at h*NR*128 + n*128 + ((c ^ n%8) * 16).
    const int t = threadIdx.x - 64;
    for (int c = t; c < NR * 16; c += kSoftmaxThreads) {
      const int n = c / 16, cc = c % 16, h = cc / 8, k8 = cc % 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n < R) {
        const long long qrow = ((long long)s * nq + n / G) * Hq + kvh * G + (n % G);
        v = ldg_nc_v4(p.q + qrow * kHeadDim + cc * 8);
      }
      sts_v4(sbase + Lay::kQ + h * Lay::kQHalf + n * 128 + ((k8 ^ (n & 7)) * 16), v);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc->tmem_base;

  const uint32_t sQ = sbase + Lay::kQ;
  const uint32_t sPhi = sbase + Lay::kPHi, sPlo = sbase + Lay::kPLo;
  auto sK = [&](int st) { return sbase + st * kStageBytes; };
  auto sV = [&](int st) { return sbase + st * kStageBytes + kKVBytes; };

  if (warp == 0) {
    // ======================= TMA producer ==================================
    const int* table = p.block_table + (long long)s * p.max_blocks_per_seq;
    int issued = 0;
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % kStages;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(bar(BAR_EMPTY + st), ((t / kStages) & 1) ^ 1, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const int c = lane;
      const int key0 = base + t * kTileKeys + c * kChunk;
      bool want = c < kChunksPerTile && key0 <= k1 && key0 + kChunk - 1 >= k0;
      long long phys = 0;
      if (want) {
        phys = table[key0 / p.block_size];
        if (phys < 0 || phys >= p.num_blocks) {
          atomicOr(p.flags, kFlagBadBlock);
          want = false;
        }
      }
      const uint32_t mask = __ballot_sync(0xffffffffu, want);
      const int row = want ? (int)((phys * p.num_kv_heads + kvh) * p.block_size +
                                   key0 % p.block_size)
                           : 0;
      int rows[kChunksPerTile];
#pragma unroll
      for (int cc = 0; cc < kChunksPerTile; ++cc) rows[cc] = __shfl_sync(0xffffffffu, row, cc);
      if (lane == 0) {  // the thread that saw the stage free issues its copies
        misc->chunk_mask[st] = mask;
        mbar_arrive_expect_tx(bar(BAR_FULL + st), __popc(mask) * 4 * kChunkBytes);
        const uint32_t fb = bar(BAR_FULL + st);
#pragma unroll
        for (int cc = 0; cc < kChunksPerTile; ++cc) {
          if (!((mask >> cc) & 1u)) continue;
          tma_load_2d(sK(st) + cc * kChunkBytes, &tmap_k, 0, rows[cc], fb);
          tma_load_2d(sK(st) + kHalfBytes + cc * kChunkBytes, &tmap_k, 64, rows[cc], fb);
          tma_load_2d(sV(st) + cc * kChunkBytes, &tmap_v, 0, rows[cc], fb);
          tma_load_2d(sV(st) + kHalfBytes + cc * kChunkBytes, &tmap_v, 64, rows[cc], fb);
        }
      }
      __syncwarp();
      issued = t + 1;
    }
    __syncthreads();  // (A) every role finished its loop
    if (lane == 0) {  // drain copies that no MMA waited for (abort path only)
      volatile int no_abort = 0;
      for (int t = misc->n_consumed; t < issued; ++t)
        mbar_wait(bar(BAR_FULL + t % kStages), (t / kStages) & 1, &no_abort);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer ====================================
    if (lane == 0) {
      const uint32_t id_qk = idesc_f16_f32(128, NR, false, false);
      const uint32_t id_pv = idesc_f16_f32(128, NR, true, true);
      auto issue_qk = [&](int t) {
        const int st = t % kStages;
        const uint32_t d = tmem + (t % 2) * NR;
#pragma unroll
        for (int k = 0; k < kHeadDim / 16; ++k) {
          const uint64_t a = smem_desc(sK(st) + (k / 4) * kHalfBytes + (k % 4) * 32, 16, 1024,
                                       kSwizzle128B);
          const uint64_t b = smem_desc(sQ + (k / 4) * Lay::kQHalf + (k % 4) * 32, 16, 1024,
                                       kSwizzle128B);
          tc_mma_f16_ss(d, a, b, id_qk, k > 0);
        }
      };
      auto issue_pv = [&](int t) {
        const int st = t % kStages;
        const uint32_t d = tmem + 2 * NR + (t % 2) * NR;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t sp = half == 0 ? sPhi : sPlo;
#pragma unroll
          for (int k = 0; k < kTileKeys / 16; ++k) {
            const uint64_t a = smem_desc(sV(st) + k * 2048, kHalfBytes, 1024, kSwizzle128B);
            const uint64_t b = smem_desc(sp + k * 2 * NR * 16, NR * 16, 128, kSwizzleNone);
            tc_mma_f16_ss(d, a, b, id_pv, (half | k) != 0);
          }
        }
      };
      auto qk_ready = [&](int t, bool block) {
        const uint32_t f = bar(BAR_FULL + t % kStages), e = bar(BAR_SEMPTY + t % 2);
        const uint32_t pf = (t / kStages) & 1, pe = ((t / 2) & 1) ^ 1;
        if (!block) return mbar_test_wait(f, pf) && mbar_test_wait(e, pe);
        return mbar_wait(f, pf, abort) && mbar_wait(e, pe, abort);
      };
      int consumed = 0;
      bool ok = ntiles > 0 && qk_ready(0, true);
      if (ok) {
        tc_fence_after();
        issue_qk(0);
        tc_commit(bar(BAR_SFULL + 0));
        consumed = 1;
      }
      for (int t = 0; ok && t < ntiles; ++t) {
        bool next_done = false;
        if (t + 1 < ntiles && qk_ready(t + 1, false)) {
          tc_fence_after();
          issue_qk(t + 1);
          tc_commit(bar(BAR_SFULL + (t + 1) % 2));
          consumed = t + 2;
          next_done = true;
        }
        ok = mbar_wait(bar(BAR_PFULL), t & 1, abort) &&
             mbar_wait(bar(BAR_OEMPTY + t % 2), ((t / 2) & 1) ^ 1, abort);
        if (!ok) break;
        tc_fence_after();
        issue_pv(t);
        tc_commit(bar(BAR_OFULL + t % 2));
        tc_commit(bar(BAR_PEMPTY));
        tc_commit(bar(BAR_EMPTY + t % kStages));
        if (t + 1 < ntiles && !next_done) {
          ok = qk_ready(t + 1, true);
          if (!ok) break;
          tc_fence_after();
          issue_qk(t + 1);
          tc_commit(bar(BAR_SFULL + (t + 1) % 2));
          consumed = t + 2;
        }
      }
      misc->n_consumed = consumed;
      tc_commit(bar(BAR_DONE));  // completes once every MMA above has finished
      volatile int no_abort = 0;
      mbar_wait(bar(BAR_DONE), 0, &no_abort);
    }
    __syncwarp();
    __syncthreads();  // (A)
  } else {
    // ======================= softmax + correction ==========================
    const int q4 = warp & 3;             // TMEM lane quarter of this warp
    const int j = q4 * 32 + lane;        // key within the tile / head_dim element
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    float* red = reinterpret_cast<float*>(smem + Lay::kRed);      // [2][4][32]
    float* alpha_s = reinterpret_cast<float*>(smem + Lay::kAlpha);  // [2][32]
    float* lsum = reinterpret_cast<float*>(smem + Lay::kLsum);      // [4][32]
    const int widx = warp - 2;

    int tlo[kMaxQuery], thi[kMaxQuery];
#pragma unroll
    for (int i = 0; i < kMaxQuery; ++i) {
      tlo[i] = 1;
      thi[i] = 0;
      if (i < nq) key_range(L, nq, i, p.causal, p.window, tlo[i], thi[i]);
    }
    const uint32_t grp = G >= 32 ? 0xffffffffu : ((1u << G) - 1u);

    float acc[NR], lpart[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = lpart[r] = 0.f;
    float m_lane = -INFINITY;  // running max of row lane % NR (log2 domain)
    bool ok = true;

    // Iteration t scores tile t and folds tile t-1's O^T into the registers;
    // the extra last iteration only folds.
    for (int t = 0; t <= ntiles; ++t) {
     if (t < ntiles) {
      const int sb = t % 2, st = t % kStages;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_SFULL + sb), (t / 2) & 1, abort));
      float sv[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) sv[r] = 0.f;
      if (ok) {
        tc_fence_after();
        tmem_ld16<0>(tmem + lane_off + sb * NR, sv);
        if constexpr (NR == 32) tmem_ld16<16 % NR>(tmem + lane_off + sb * NR + 16, sv);
        tmem_ld_wait();
        tc_fence_before();
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(bar(BAR_SEMPTY + sb));
      ok = __all_sync(0xffffffffu,
                      ok && mbar_wait(bar(BAR_FULL + st), (t / kStages) & 1, abort));  // complete

      // Which rows see this key?  (Only keys of loaded chunks inside the
      // CTA's range; the per-token ranges are the ones key_range gives.)
      const int key = base + t * kTileKeys + j;
      const uint32_t cmask = ok ? misc->chunk_mask[st] : 0u;
      uint32_t rmask = 0;
      if (((cmask >> (j / kChunk)) & 1u) && key >= k0 && key <= k1) {
#pragma unroll
        for (int i = 0; i < kMaxQuery; ++i)
          if (i < nq && key >= tlo[i] && key <= thi[i]) rmask |= grp << (i * G);
      }
      float sc[NR], red_in[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        sc[r] = ((rmask >> r) & 1u) ? sv[r] * p.scale_log2 : -INFINITY;
        red_in[r] = sc[r];
      }
      const float wmax = warp_row_reduce<NR, true>(red_in, lane);
      if (lane < NR) red[(sb * 4 + widx) * 32 + lane] = wmax;
      named_bar_sync(1, kSoftmaxThreads);
      const int rl = lane % NR;
      float tmax = red[(sb * 4 + 0) * 32 + rl];
      tmax = fmaxf(tmax, red[(sb * 4 + 1) * 32 + rl]);
      tmax = fmaxf(tmax, red[(sb * 4 + 2) * 32 + rl]);
      tmax = fmaxf(tmax, red[(sb * 4 + 3) * 32 + rl]);
      const float m_new = fmaxf(m_lane, tmax);
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_lane - m_new);
      m_lane = m_new;
      if (widx == 0 && lane < NR) alpha_s[sb * 32 + lane] = alpha;

      // Scaled weights, split into fp16 high part + fp16 residual.
      uint32_t phi[NR / 2], plo[NR / 2];
#pragma unroll
      for (int r = 0; r < NR; r += 2) {
        float pr[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float mr = __shfl_sync(0xffffffffu, m_new, r + e);
          const float ar = __shfl_sync(0xffffffffu, alpha, r + e);
          const float x = sc[r + e];
          pr[e] = (x == -INFINITY) ? 0.f : exp2f(x - mr + (float)kPShift);
          lpart[r + e] = fmaf(lpart[r + e], ar, pr[e]);
        }
        const __half2 h = __floats2half2_rn(pr[0], pr[1]);
        const float2 hf = __half22float2(h);
        const __half2 l2 = __floats2half2_rn(pr[0] - hf.x, pr[1] - hf.y);
        phi[r / 2] = *reinterpret_cast<const uint32_t*>(&h);
        plo[r / 2] = *reinterpret_cast<const uint32_t*>(&l2);
      }

      // A key no row can see must not reach the PV product: zero its V row.
      if (ok && rmask == 0) {
        const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          sts_v4(sV(st) + j * 128 + c * 16, z);
          sts_v4(sV(st) + kHalfBytes + j * 128 + c * 16, z);
        }
      }
      ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_PEMPTY), (t & 1) ^ 1, abort));
      if (ok) {
        // P^T as no-swizzle MN-major core matrices: [key/8][row/8][key%8][row%8].
#pragma unroll
        for (int rg = 0; rg < NR / 8; ++rg) {
          const uint32_t off = ((j >> 3) * (NR / 8) + rg) * 128 + (j & 7) * 16;
          sts_v4(sPhi + off, make_uint4(phi[rg * 4], phi[rg * 4 + 1], phi[rg * 4 + 2], phi[rg * 4 + 3]));
          sts_v4(sPlo + off, make_uint4(plo[rg * 4], plo[rg * 4 + 1], plo[rg * 4 + 2], plo[rg * 4 + 3]));
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(bar(BAR_PFULL));
     } else {
      named_bar_sync(1, kSoftmaxThreads);  // alpha of the last tile visible to all
     }
      if (t > 0) {  // O^T of tile u = t-1: acc = acc * alpha_u + O_u
        const int u = t - 1, ob = u % 2;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(bar(BAR_OFULL + ob), (u / 2) & 1, abort));
        float ov[NR];
#pragma unroll
        for (int r = 0; r < NR; ++r) ov[r] = 0.f;
        if (ok) {
          tc_fence_after();
          tmem_ld16<0>(tmem + lane_off + 2 * NR + ob * NR, ov);
          if constexpr (NR == 32) tmem_ld16<16 % NR>(tmem + lane_off + 2 * NR + ob * NR + 16, ov);
          tmem_ld_wait();
          tc_fence_before();
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(bar(BAR_OEMPTY + ob));
        if (ok) {
#pragma unroll
          for (int r = 0; r < NR; ++r) acc[r] = fmaf(acc[r], alpha_s[ob * 32 + r], ov[r]);
        }
      }
    }

    // Row sums: per-thread partials -> per-warp (lane r) -> across warps.
    const float wl = warp_row_reduce<NR, false>(lpart, lane);
    if (lane < NR) lsum[widx * 32 + lane] = wl;
    named_bar_sync(1, kSoftmaxThreads);
    const bool aborted = *abort != 0;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      if (r < R) {
        const float l = lsum[r] + lsum[32 + r] + lsum[64 + r] + lsum[96 + r];
        const long long pr = part_base + row_index(r);
        p.part_out[pr * kHeadDim + j] = (!aborted && l > 0.f) ? acc[r] / l : 0.f;
      }
    }
    if (widx == 0 && lane < R) {
      const float l = lsum[lane] + lsum[32 + lane] + lsum[64 + lane] + lsum[96 + lane];
      p.part_lse[part_base + row_index(lane)] =
          (!aborted && l > 0.f) ? ((m_lane - (float)kPShift) + log2f(l)) * 0.69314718055994531f
                                : -INFINITY;
    }
    __syncthreads();  // (A)
  }

  // ---- tear-down (every thread passed (A)) -----------------------------------
  if (threadIdx.x == 0 && misc->abort) atomicOr(p.flags, kFlagTimeout);
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
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

// The fp16 cache viewed as a 2-D tensor: 128 columns (head_dim) by
// num_blocks * Hkv * block_size rows; one TMA box = 16 rows x 64 columns,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).
bool encode_cache_map(CUtensorMap* m, const void* cache, long long rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kChunk};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(cache), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NR>
cudaError_t launch_nr(const DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                      cudaStream_t stream) {
  const size_t smem = Layout<NR>::kTotal + 1024;
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(decode_tc_kernel<NR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const dim3 grid(p.num_splits, p.num_kv_heads, p.num_seqs);
  decode_tc_kernel<NR><<<grid, kThreads, smem, stream>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool decode_tc_supported(int kv_dtype, int rows, int num_blocks, int num_kv_heads, int block_size) {
  return kv_dtype == kKvFp16 && rows >= 1 && rows <= 32 &&
         (long long)num_blocks * num_kv_heads * block_size <= INT32_MAX;
}

cudaError_t launch_decode_tc(const DecodeParams& p, cudaStream_t stream) {
  CUtensorMap mk, mv;
  const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
  if (!encode_cache_map(&mk, p.k, rows) || !encode_cache_map(&mv, p.v, rows))
    return cudaErrorInvalidValue;
  if (p.rows <= 16) return launch_nr<16>(p, mk, mv, stream);
  return launch_nr<32>(p, mk, mv, stream);
}

}  // namespace pa
