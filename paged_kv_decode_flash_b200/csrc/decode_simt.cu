// decode_simt.cu -- the plain split-KV decode kernel on CUDA cores, fp32.
//
// One CTA per (key split, KV head, sequence).  It walks its share of the
// sequence's KV blocks 16 keys at a time, gathers K and V through the block
// table into shared memory (fp16 or q8_0, converted exactly to fp32), scores
// all n_query * G query rows that share the KV head, keeps a running
// (max, sum) per row in the log2 domain, and writes one fp32 partial output
// and log-sum-exp per row for the merge ("Dual MI50, part 2", section
// "Decode: a new kernel for the shape MTP actually runs": split along the
// context, partial results merged at the end; all query rows of one KV head
// read the same keys).
//
// This is the general path: any block_size multiple of 16, any row count up
// to 64, both cache types.  Keys that no row can see are never multiplied:
// their V rows are zero-filled when staged, their scores are selected to
// -inf, and whole chunks outside the visible range are not loaded at all
// ("Bug 2: the drafter read freed memory": out-of-window blocks may hold
// anything, and the regression test fills them with NaN).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace pa {
namespace {

constexpr int kThreads = 128;
constexpr int kKStride = kHeadDim + 4;  // fp32 row pitch of staged K (bank skew)

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}
__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

// Stage keys [c0, c0+16) of one chunk (all in physical block `phys`, slots
// slot0..slot0+15) for KV head kvh into ks/vs as fp32.  Keys outside
// [lo_u, hi_u] are written as 0 without reading memory.
__device__ void stage_chunk(const DecodeParams& p, long long phys, int kvh, int slot0, int c0,
                            int lo_u, int hi_u, float* ks, float* vs) {
  for (int t = threadIdx.x; t < kChunk * (kHeadDim / 8); t += kThreads) {
    const int key = t / (kHeadDim / 8);
    const int d0 = (t % (kHeadDim / 8)) * 8;
    const int j = c0 + key;
    const bool live = j >= lo_u && j <= hi_u;
    float kf[8], vf[8];
    if (!live) {
#pragma unroll
      for (int e = 0; e < 8; ++e) kf[e] = vf[e] = 0.f;
    } else if (p.kv_dtype == kKvFp16) {
      const long long row = ((phys * p.num_kv_heads + kvh) * p.block_size + slot0 + key);
      const uint4 kr = ldg_nc_v4((const __half*)p.k + row * kHeadDim + d0);
      const uint4 vr = ldg_nc_v4((const __half*)p.v + row * kHeadDim + d0);
      const __half2* kh = reinterpret_cast<const __half2*>(&kr);
      const __half2* vh = reinterpret_cast<const __half2*>(&vr);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = __half22float2(kh[e]);
        const float2 b = __half22float2(vh[e]);
        kf[2 * e] = a.x; kf[2 * e + 1] = a.y;
        vf[2 * e] = b.x; vf[2 * e + 1] = b.y;
      }
    } else {
      const long long tb = q8_0_tile_bytes(p.block_size, kHeadDim);
      const long long tile = (phys * p.num_kv_heads + kvh) * tb;
      const int slot = slot0 + key;
      const long long qoff = tile + (long long)slot * kHeadDim + d0;
      const long long doff = tile + (long long)p.block_size * kHeadDim +
                             ((long long)slot * (kHeadDim / 32) + d0 / 32) * 2;
      const uint2 kq = ldg_nc_v2((const char*)p.k + qoff);
      const uint2 vq = ldg_nc_v2((const char*)p.v + qoff);
      const float kd = __half2float(*reinterpret_cast<const __half*>((const char*)p.k + doff));
      const float vd = __half2float(*reinterpret_cast<const __half*>((const char*)p.v + doff));
      const signed char* kb = reinterpret_cast<const signed char*>(&kq);
      const signed char* vb = reinterpret_cast<const signed char*>(&vq);
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // int8 * fp16 scale: exact in fp32
        kf[e] = (float)kb[e] * kd;
        vf[e] = (float)vb[e] * vd;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ks[key * kKStride + d0 + e] = kf[e];
      vs[key * kHeadDim + d0 + e] = vf[e];
    }
  }
}

__global__ void __launch_bounds__(kThreads) decode_simt_kernel(const DecodeParams p) {
  extern __shared__ float4 smem_f4[];
  float* smem = reinterpret_cast<float*>(smem_f4);
  const int R = p.rows;
  float* qs = smem;                           // [R][D], pre-scaled by scale*log2(e)
  float* ks = qs + R * kHeadDim;              // [16][D+4]
  float* vs = ks + kChunk * kKStride;         // [16][D]
  float* ps = vs + kChunk * kHeadDim;         // [R][16]
  float* m_s = ps + R * kChunk;               // [R] running max (log2 domain)
  float* l_s = m_s + R;                       // [R] running sum
  float* a_s = l_s + R;                       // [R] rescale factor of this chunk

  const int split = blockIdx.x, kvh = blockIdx.y, s = blockIdx.z;
  const int tid = threadIdx.x;
  const int nq = p.n_query, G = p.group, Hq = p.num_q_heads;
  const int rps = nq * Hq;
  const long long part_base = ((long long)s * p.num_splits + split) * rps;

  // Row r of this CTA is query token r / G, query head kvh * G + r % G.
  auto row_index = [&](int r) { return (r / G) * Hq + kvh * G + (r % G); };
  auto write_empty = [&]() {
    for (int r = 0; r < R; ++r) {
      const long long pr = part_base + row_index(r);
      p.part_out[pr * kHeadDim + tid] = 0.f;
      if (tid == 0) p.part_lse[pr] = -INFINITY;
    }
    sm100::griddep_launch_dependents();  // partial written: the merge may be scheduled
  };

  const int L = p.context_lens[s];
  if (!context_len_ok(L, nq, p.max_blocks_per_seq, p.block_size)) {
    if (split == 0 && kvh == 0 && tid == 0) atomicOr(p.flags, kFlagBadLen);
    write_empty();
    return;
  }
  int lo_u, hi_u;
  union_range(L, nq, p.causal, p.window, lo_u, hi_u);
  const long long split_k0 = (long long)split * p.blocks_per_split * p.block_size;
  const long long split_k1 = split_k0 + (long long)p.blocks_per_split * p.block_size - 1;
  const int k0 = (int)max((long long)lo_u, split_k0);
  const int k1 = (int)min((long long)hi_u, split_k1);
  if (k0 > k1) {
    write_empty();
    return;
  }

  for (int t = tid; t < R * kHeadDim; t += kThreads) {
    const int r = t / kHeadDim, d = t % kHeadDim;
    const int i = r / G;
    const long long qrow = ((long long)s * nq + i) * Hq + kvh * G + (r % G);
    qs[t] = __half2float(p.q[qrow * kHeadDim + d]) * p.scale_log2;
  }
  for (int r = tid; r < R; r += kThreads) {
    m_s[r] = -INFINITY;
    l_s[r] = 0.f;
  }

  float acc[kMaxRows];
#pragma unroll
  for (int r = 0; r < kMaxRows; ++r) acc[r] = 0.f;

  const int jj = tid & (kChunk - 1);   // key within the chunk (score phase)
  const int rg = tid / kChunk;         // first row of this thread (score phase)
  const int* table = p.block_table + (long long)s * p.max_blocks_per_seq;

  for (int c0 = (k0 / kChunk) * kChunk; c0 <= k1; c0 += kChunk) {
    const int lb = c0 / p.block_size;
    const int slot0 = c0 % p.block_size;
    const long long phys = table[lb];
    const bool bad = phys < 0 || phys >= p.num_blocks;
    __syncthreads();  // previous chunk fully consumed
    if (bad) {
      if (tid == 0) atomicOr(p.flags, kFlagBadBlock);
      continue;  // keys of an out-of-range block are treated as masked
    }
    stage_chunk(p, phys, kvh, slot0, c0, k0, k1, ks, vs);
    __syncthreads();

    // Scores, masked online softmax: 16 lanes per row, one key each.  Every
    // half-warp runs the same number of iterations (rows padded to 8) so the
    // shuffles always see all 32 lanes.
    const int j = c0 + jj;
    const int R8 = (R + 7) & ~7;
    for (int r = rg; r < R8; r += kThreads / kChunk) {
      const bool row_ok = r < R;
      int lo = 0, hi = -1;
      if (row_ok) key_range(L, nq, r / G, p.causal, p.window, lo, hi);
      const bool vis = row_ok && j >= lo && j <= hi && j >= k0 && j <= k1;
      float sc = -INFINITY;
      if (vis) {
        const float4* qv = reinterpret_cast<const float4*>(qs + r * kHeadDim);
        const float4* kv = reinterpret_cast<const float4*>(ks + jj * kKStride);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
        for (int d4 = 0; d4 < kHeadDim / 4; ++d4) {
          const float4 x = qv[d4], y = kv[d4];
          a0 = fmaf(x.x, y.x, a0);
          a1 = fmaf(x.y, y.y, a1);
          a2 = fmaf(x.z, y.z, a2);
          a3 = fmaf(x.w, y.w, a3);
        }
        sc = (a0 + a1) + (a2 + a3);
      }
      float mx = sc;
#pragma unroll
      for (int o = kChunk / 2; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = row_ok ? m_s[r] : -INFINITY;
      const float m_new = fmaxf(m_old, mx);
      const float pr = (vis && m_new != -INFINITY) ? exp2f(sc - m_new) : 0.f;
      float sum = pr;
#pragma unroll
      for (int o = kChunk / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (row_ok) ps[r * kChunk + jj] = pr;
      __syncwarp();
      if (row_ok && jj == 0) {
        const float alpha = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
        a_s[r] = alpha;
        m_s[r] = m_new;
        l_s[r] = l_s[r] * alpha + sum;
      }
    }
    __syncthreads();

    // acc[r][d = tid] = acc * alpha + sum_k P[r][k] V[k][d]
    float vcol[kChunk];
#pragma unroll
    for (int k = 0; k < kChunk; ++k) vcol[k] = vs[k * kHeadDim + tid];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r) {
      if (r < R) {
        float a = acc[r] * a_s[r];
        const float4* pv = reinterpret_cast<const float4*>(ps + r * kChunk);
#pragma unroll
        for (int k4 = 0; k4 < kChunk / 4; ++k4) {
          const float4 w = pv[k4];
          a = fmaf(w.x, vcol[4 * k4 + 0], a);
          a = fmaf(w.y, vcol[4 * k4 + 1], a);
          a = fmaf(w.z, vcol[4 * k4 + 2], a);
          a = fmaf(w.w, vcol[4 * k4 + 3], a);
        }
        acc[r] = a;
      }
    }
  }
  __syncthreads();

#pragma unroll
  for (int r = 0; r < kMaxRows; ++r) {
    if (r < R) {
      const float l = l_s[r];
      const long long pr = part_base + row_index(r);
      p.part_out[pr * kHeadDim + tid] = l > 0.f ? acc[r] / l : 0.f;
      if (tid == 0) p.part_lse[pr] = l > 0.f ? (m_s[r] + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }
  sm100::griddep_launch_dependents();  // partial written: the merge may be scheduled
}

}  // namespace

size_t decode_simt_smem_bytes(int rows) {
  return sizeof(float) * ((size_t)rows * kHeadDim + kChunk * kKStride + kChunk * kHeadDim +
                          (size_t)rows * kChunk + 3 * (size_t)rows);
}

cudaError_t launch_decode_simt(const DecodeParams& p, cudaStream_t stream) {
  const size_t smem = decode_simt_smem_bytes(p.rows);
  // Opt in to the largest dynamic shared memory any row count needs, once per
  // device (not per launch, so captured launches make no attribute calls).
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || !configured[dev]) {
    e = cudaFuncSetAttribute(decode_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)decode_simt_smem_bytes(kMaxRows));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = true;
  }
  const dim3 grid(p.num_splits, p.num_kv_heads, p.num_seqs);
  decode_simt_kernel<<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pa
