// dispatch.cu -- argument checks, the split planner, the workspace layout and
// the launches behind every decode entry point.  Host code only.
//
// Split planner ("Dual MI50, part 2", section "Decode: a new kernel for the
// shape MTP actually runs": the work is split along the context so that all
// compute units stay busy at batch 1).  The number of splits depends only on
// host integers (shapes and the SM count), never on context_lens, which stay
// on the device: a call needs no host synchronisation and can be captured in
// a CUDA graph.  Each split owns a contiguous run of logical blocks; a CTA
// (split, KV head, sequence) intersects its run with the sequence's visible
// key range on the device and leaves early when that is empty.
#include "dispatch.h"

#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr int kCtasPerSm = 2;           // CUDA-core kernel: resident CTAs per SM aimed for
constexpr int kMaxTargetCtas = 4096;    // device-independent bound used to size workspaces
constexpr int kMinKeysPerSplit = 128;   // a split below this is all overhead
// Tensor-core kernel, many (sequence, KV head) groups: items of at least this
// many 128-key tiles, sized for about kItemWaves waves of CTAs.
constexpr int kMinItemTiles = 16;
constexpr int kItemWaves = 4;

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// splits = target CTAs / (sequences x KV heads), at least 128 keys per split;
// rounded up for the CUDA-core kernel (several CTAs per SM) and down for the
// tensor-core kernel (one CTA per SM: a second wave would double the time).
int plan_splits(const pa_dims* d, long long target_ctas, bool round_up, int* blocks_per_split) {
  const long long min_blocks = ceil_div(kMinKeysPerSplit, d->block_size);
  const long long max_splits = std::max(1LL, ceil_div(d->max_blocks_per_seq, min_blocks));
  const long long per_split = (long long)d->num_seqs * d->num_kv_heads;
  long long splits = round_up ? ceil_div(target_ctas, per_split) : target_ctas / per_split;
  splits = std::max(1LL, std::min(splits, max_splits));
  const long long bps = ceil_div(d->max_blocks_per_seq, splits);
  *blocks_per_split = (int)bps;
  return (int)ceil_div(d->max_blocks_per_seq, bps);
}

}  // namespace

int check_dims(const pa_dims* d, int n_query) {
  if (d == nullptr) return PA_ERR_INVALID_ARG;
  if (d->num_seqs < 1 || d->num_q_heads < 1 || d->num_kv_heads < 1 || d->head_dim < 1 ||
      d->block_size < 1 || d->max_blocks_per_seq < 1 || d->num_blocks < 1)
    return PA_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (n_query < 1 || n_query > kMaxQuery) return PA_ERR_INVALID_ARG;
  if (d->block_size % kChunk != 0) return PA_ERR_INVALID_ARG;
  if (d->head_dim != kHeadDim) return PA_ERR_UNSUPPORTED;
  if ((long long)n_query * (d->num_q_heads / d->num_kv_heads) > kMaxRows) return PA_ERR_UNSUPPORTED;
  if ((long long)d->max_blocks_per_seq * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if ((long long)d->num_blocks * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}

int check_decode_args(const void* q, const void* k, const void* v, const int32_t* bt,
                      const int32_t* cl, int causal, int window, float scale, int kv_dtype,
                      const void* out) {
  if (!q || !k || !v || !bt || !cl || !out) return PA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(bt, 4) || !aligned(cl, 4))
    return PA_ERR_INVALID_ARG;
  if ((causal != 0 && causal != 1) || window < 0) return PA_ERR_INVALID_ARG;
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

Plan make_plan(const pa_dims* d, int n_query, int kv_dtype, int sms) {
  Plan pl{};
  const int rows = n_query * (d->num_q_heads / d->num_kv_heads);
  pl.tensor_cores =
      decode_tc_supported(kv_dtype, rows, d->num_blocks, d->num_kv_heads, d->block_size);
  if (pl.tensor_cores) {
    const long long groups = (long long)d->num_seqs * d->num_kv_heads;
    const long long max_split = ceil_div((long long)d->max_blocks_per_seq * d->block_size, 128);
    if (groups * 4 > sms) {
      // Many groups (a batch): an even share of the SMs would give a long
      // sequence no more CTAs than a short one.  Instead every group's tiles
      // are cut into items of T tiles, T from the shapes alone (so that a
      // sequence's split, and every bit of its output, depends only on its
      // own length), one CTA per item over about kItemWaves waves; the
      // hardware hands each free SM the next item, and a group's items past
      // its length leave at once.
      const long long T = std::max<long long>(
          kMinItemTiles, ceil_div(max_split * groups, (long long)kItemWaves * sms));
      pl.splits = (int)ceil_div(max_split, T);
      pl.ctas = (int)(groups * pl.splits);
      pl.tiles_per_item = (int)T;
    } else {
      // One CTA per SM (one per group at least, and no more than the
      // table's 128-key tiles could keep busy); the kernel shares them out
      // evenly among the (sequence, KV head) groups.
      pl.ctas = (int)std::max(groups, std::min<long long>(sms, groups * max_split));
      pl.splits = (int)ceil_div(pl.ctas, groups);
      pl.tiles_per_item = 0;
    }
    pl.blocks_per_split = (int)ceil_div(d->max_blocks_per_seq, pl.splits);
  } else {
    pl.splits = plan_splits(d, (long long)sms * kCtasPerSm, true, &pl.blocks_per_split);
    pl.ctas = pl.splits * d->num_kv_heads * d->num_seqs;
  }
  return pl;
}

Plan max_plan(const pa_dims* d) {
  Plan pl{};
  pl.tensor_cores = false;
  pl.splits = plan_splits(d, kMaxTargetCtas, true, &pl.blocks_per_split);
  // The tensor-core planner cuts the table into 128-key tiles, which for a
  // block_size that does not divide 128 allows more splits than whole
  // blocks do: at most one per tile, and no more than kMaxTargetCtas CTAs
  // over the groups (one wave, or items of >= 16 tiles over a few waves).
  const long long groups = (long long)d->num_seqs * d->num_kv_heads;
  const long long tiles = ceil_div((long long)d->max_blocks_per_seq * d->block_size, 128);
  const long long tc = std::min(tiles, std::max(1LL, ceil_div(kMaxTargetCtas, groups)));
  pl.splits = std::max<int>(pl.splits, (int)tc);
  return pl;
}

// Status header, then two arrival counters per (sequence, KV head).
size_t ws_zero_prefix(const pa_dims* d) {
  return kWsHeader + align256((size_t)d->num_seqs * d->num_kv_heads * 2 * sizeof(int));
}

WsLayout ws_layout(const pa_dims* d, int n_query, int splits) {
  const size_t rows = (size_t)d->num_seqs * splits * n_query * d->num_q_heads;
  WsLayout w;
  w.part_out = ws_zero_prefix(d);
  w.part_lse = w.part_out + align256(rows * d->head_dim * sizeof(float));
  w.total = w.part_lse + align256(rows * sizeof(float));
  return w;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

int enqueue_decode(const pa_dims* d, const Plan& plan, const void* q, const void* k_cache,
                   const void* v_cache, const int32_t* block_table, const int32_t* context_lens,
                   int n_query, int causal, int window, float scale, int kv_dtype, void* out,
                   void* ws_ptr, cudaStream_t st) {
  const WsLayout w = ws_layout(d, n_query, plan.splits);
  char* ws = static_cast<char*>(ws_ptr);
  DecodeParams p{};
  p.q = static_cast<const __half*>(q);
  p.k = k_cache;
  p.v = v_cache;
  p.block_table = block_table;
  p.context_lens = context_lens;
  p.num_seqs = d->num_seqs;
  p.num_q_heads = d->num_q_heads;
  p.num_kv_heads = d->num_kv_heads;
  p.block_size = d->block_size;
  p.max_blocks_per_seq = d->max_blocks_per_seq;
  p.num_blocks = d->num_blocks;
  p.n_query = n_query;
  p.causal = causal;
  p.window = window;
  p.kv_dtype = kv_dtype;
  p.group = d->num_q_heads / d->num_kv_heads;
  p.rows = n_query * p.group;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.num_splits = plan.splits;
  p.num_ctas = plan.ctas;
  p.tiles_per_item = plan.tiles_per_item;
  p.blocks_per_split = plan.blocks_per_split;
  p.part_out = reinterpret_cast<float*>(ws + w.part_out);
  p.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  p.flags = reinterpret_cast<unsigned*>(ws);
  p.arrivals = reinterpret_cast<int*>(ws + kWsHeader);
  p.out = static_cast<__half*>(out);

  if (plan.tensor_cores)  // one launch: the last CTA of each group merges
    return launch_decode_tc(p, st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  if (launch_decode_simt(p, st) != cudaSuccess) return PA_ERR_CUDA;
  MergeParams m{};
  m.part_out = p.part_out;
  m.part_lse = p.part_lse;
  m.num_seqs = d->num_seqs;
  m.num_splits = plan.splits;
  m.rows_per_seq = n_query * d->num_q_heads;
  m.head_dim = kHeadDim;
  m.out = static_cast<__half*>(out);
  m.out_lse = nullptr;
  return launch_merge(m, st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
