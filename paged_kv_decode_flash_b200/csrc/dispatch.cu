// dispatch.cu -- argument checks, the work planner, the workspace layout and
// the launches behind every decode entry point.  Host code only.
//
// Planner ("Dual MI50, part 2", section "Decode: a new kernel for the shape
// MTP actually runs": the work is split along the context so that all
// compute units stay busy at batch 1).  The plan depends only on host
// integers (shapes, cache type and the SM count), never on context_lens,
// which stay on the device: a call needs no host synchronisation and can be
// captured in a CUDA graph.  Within the plan, the device cuts each
// sequence's visible keys from its own length (common.cuh, DecodeParams).
#include "dispatch.h"

#include <algorithm>
#include <atomic>
#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace pa {
namespace {

constexpr int kMaxSmsAnyDevice = 4096;  // bound used to size workspaces without a device
constexpr int kMaxItemTiles = 16;       // mode 1: tiles per big item
constexpr int kMaxSubItems = 4;         // mode 1: the last item of a group is cut into up to 4

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};

int rows_of(const pa_dims* d, int n_query) { return n_query * (d->num_q_heads / d->num_kv_heads); }
long long max_chunks(const pa_dims* d) { return (long long)d->max_blocks_per_seq * d->block_size / kChunk; }

// Row parts: the rows of a KV head are cut into equal parts of at most
// max_rows_per_part rows (32 for fp16, 16 for the int8 caches, whose
// converter warps leave fewer registers to the softmax).
void row_parts(const pa_dims* d, int n_query, int kv_dtype, int* halves, int* rows_half) {
  const int R = rows_of(d, n_query);
  const int maxr = max_rows_per_part(kv_dtype);
  *halves = (int)ceil_div(R, maxr);
  *rows_half = (int)ceil_div(R, *halves);
}

int launches_of(const pa_dims* d) { return (int)ceil_div(d->num_seqs, kMaxQueueSeqs); }

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
  if ((long long)rows_of(d, n_query) > kMaxRows) return PA_ERR_UNSUPPORTED;
  if ((long long)d->max_blocks_per_seq * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if ((long long)d->num_blocks * d->block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
  // TMA row coordinates (rows / 8) and int8 tile indices are 32-bit.
  if ((long long)d->num_blocks * d->num_kv_heads * d->block_size / 8 > INT32_MAX) return PA_ERR_UNSUPPORTED;
  if ((long long)d->num_seqs * d->num_kv_heads * kMaxRows > INT32_MAX) return PA_ERR_UNSUPPORTED;
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
  if (kv_dtype != PA_KV_FP16 && kv_dtype != PA_KV_Q8_0 && kv_dtype != PA_KV_INT8_ROW)
    return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  return PA_OK;
}

Plan make_plan(const pa_dims* d, int n_query, int kv_dtype, int sms) {
  Plan pl{};
  row_parts(d, n_query, kv_dtype, &pl.halves, &pl.rows_half);
  const long long groups = (long long)d->num_seqs * d->num_kv_heads * pl.halves;
  const long long max_tiles = ceil_div(max_chunks(d), kChunksPerTile);
  if (groups * 4 <= sms) {
    // Few groups: each (sequence, part) gets an equal share of the SMs, the
    // same number of CTAs for every KV head (so that a full table's cut
    // falls on head boundaries and no CTA switches heads mid-stream), at
    // least one and at most one per tile of a full table.
    const long long share = sms / ((long long)d->num_seqs * pl.halves);
    const long long per_head =
        std::max<long long>(1, std::min<long long>(share / d->num_kv_heads, max_tiles));
    pl.mode = 0;
    pl.ctas_per_set = (int)(d->num_kv_heads * per_head);
    pl.ctas = (int)((long long)d->num_seqs * pl.halves * pl.ctas_per_set);
    pl.launches = 1;
    pl.slots = (long long)d->num_seqs * pl.halves * (pl.ctas_per_set + d->num_kv_heads);
    // fp16, at most 8 tokens and 32 rows (one part): the per-head split
    // kernel, at most one CTA per SM and the same number for every
    // (sequence, KV head) group -- a head with one CTA fewer than the others
    // finishes last while they idle (61k verify: 18 per head on 144 SMs
    // measured 0.9 us faster per call than 18-19 on all 148) -- at least one
    // each and no more than a full table's tiles.  Its CTA-indexed partials
    // fit in the slots above: groups x (SMs / groups + 1) >= its CTAs.
    const long long kv_groups = (long long)d->num_seqs * d->num_kv_heads;
    if (pl.halves == 1 &&
        split_decode_supported(kv_dtype, n_query, n_query * (d->num_q_heads / d->num_kv_heads),
                               d->num_blocks, d->num_kv_heads, d->block_size))
      pl.split_ctas = (int)(kv_groups * std::max<long long>(
                                            1, std::min<long long>(sms / kv_groups, max_tiles)));
  } else {
    // A batch: items of T tiles (the last one of a group in up to four
    // pieces) from a queue, one CTA per SM; one launch per kMaxQueueSeqs
    // sequences.
    const long long T = std::min<long long>(kMaxItemTiles, max_tiles);
    pl.mode = 1;
    pl.item_tiles = (int)T;
    pl.slots_per_group = (int)(ceil_div(max_chunks(d), 8 * T) - 1 + kMaxSubItems);
    pl.launches = launches_of(d);
    const long long per_launch = (long long)std::min(d->num_seqs, kMaxQueueSeqs) *
                                 d->num_kv_heads * pl.halves * pl.slots_per_group;
    pl.ctas = (int)std::max<long long>(1, std::min<long long>(sms, per_launch));
    pl.slots = groups * pl.slots_per_group;
  }
  return pl;
}

// The counters cover the most row parts any call on these shapes uses (64
// rows in parts of 16), so that the zero prefix does not depend on the call.
constexpr int kMaxParts = kMaxRows / 16;

size_t ws_zero_prefix(const pa_dims* d) {
  const long long groups = (long long)d->num_seqs * d->num_kv_heads * kMaxParts;
  return kWsHeader + align256((size_t)groups * 2 * sizeof(int)) +
         align256((size_t)launches_of(d) * sizeof(int));
}

WsLayout ws_layout(const pa_dims* d, int n_query, const Plan& plan) {
  (void)n_query;
  const long long groups = (long long)d->num_seqs * d->num_kv_heads * kMaxParts;
  WsLayout w;
  w.arrivals = kWsHeader;
  w.queue = w.arrivals + align256((size_t)groups * 2 * sizeof(int));
  w.part_out = ws_zero_prefix(d);
  const size_t rows = (size_t)plan.slots * plan.rows_half;
  w.part_lse = w.part_out + align256(rows * kHeadDim * sizeof(float));
  w.total = w.part_lse + align256(rows * sizeof(float));
  return w;
}

size_t ws_size_any_device(const pa_dims* d, int n_query) {
  size_t need = 0;
  for (int kv : {PA_KV_FP16, PA_KV_Q8_0, PA_KV_INT8_ROW}) {
    // The most partial slots any SM count gives: mode 1 (few SMs) or mode 0
    // at the largest SM count.
    Plan a = make_plan(d, n_query, kv, 1);
    Plan b = make_plan(d, n_query, kv, kMaxSmsAnyDevice);
    need = std::max(need, ws_layout(d, n_query, a.slots >= b.slots ? a : b).total);
  }
  return need;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  static std::atomic<int> cache[64];
  if (dev >= 0 && dev < 64) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
unsigned long long set_wait_limit_ns(unsigned long long ns) {
  return g_wait_limit_ns.exchange(ns == 0 ? kDefaultWaitLimitNs : ns);
}

int enqueue_decode(const pa_dims* d, const Plan& plan, const void* q, const void* k_cache,
                   const void* v_cache, const int32_t* block_table, const int32_t* context_lens,
                   int n_query, int causal, int window, float scale, int kv_dtype, void* out,
                   void* ws_ptr, int32_t* trace, cudaStream_t st, const PartialArgs& partial) {
  const WsLayout w = ws_layout(d, n_query, plan);
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
  p.halves = plan.halves;
  p.rows_half = plan.rows_half;
  p.mode = plan.mode;
  p.num_ctas = plan.ctas;
  p.ctas_per_set = plan.ctas_per_set;
  p.item_tiles = plan.item_tiles;
  p.slots_per_group = plan.slots_per_group;
  p.wait_limit_ns = wait_limit_ns();
  p.part_out = reinterpret_cast<float*>(ws + w.part_out);
  p.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  p.flags = reinterpret_cast<unsigned*>(ws);
  p.arrivals = reinterpret_cast<int*>(ws + w.arrivals);
  p.queue = reinterpret_cast<int*>(ws + w.queue);
  p.out = static_cast<__half*>(out);
  p.trace = trace;
  p.key_begin = partial.key_begin;
  p.key_count = partial.key_count;
  p.out_f32 = partial.out;
  p.out_lse = partial.out_lse;
  if (plan.mode == 0) {
    // Every key of the context (no context-parallel key range): the per-head
    // split kernel where the plan chose it.
    if (plan.split_ctas > 0 && partial.key_begin == nullptr)
      return launch_split_decode(p, plan.split_ctas, st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    return launch_decode_tc(p, st) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
  }
  // Mode 1: one launch per kMaxQueueSeqs sequences, each with its own
  // counters and partial slots.
  const long long rows_per_seq = (long long)n_query * d->num_q_heads;
  const long long groups_per_seq = (long long)d->num_kv_heads * plan.halves;
  for (int l = 0; l < plan.launches; ++l) {
    const int s0 = l * kMaxQueueSeqs;
    DecodeParams pl = p;
    pl.num_seqs = std::min(kMaxQueueSeqs, d->num_seqs - s0);
    pl.q = p.q + (long long)s0 * rows_per_seq * kHeadDim;
    pl.out = p.out + (long long)s0 * rows_per_seq * kHeadDim;
    pl.block_table = p.block_table + (long long)s0 * d->max_blocks_per_seq;
    pl.context_lens = p.context_lens + s0;
    if (p.key_begin != nullptr) {
      pl.key_begin = p.key_begin + s0;
      pl.key_count = p.key_count + s0;
      pl.out_f32 = p.out_f32 + (long long)s0 * rows_per_seq * kHeadDim;
      pl.out_lse = p.out_lse + (long long)s0 * rows_per_seq;
    }
    pl.arrivals = p.arrivals + (long long)s0 * groups_per_seq * 2;
    pl.queue = p.queue + l;
    const long long slot0 = (long long)s0 * groups_per_seq * plan.slots_per_group;
    pl.part_out = p.part_out + slot0 * plan.rows_half * kHeadDim;
    pl.part_lse = p.part_lse + slot0 * plan.rows_half;
    if (trace != nullptr) pl.trace = trace + (long long)s0 * rows_per_seq * 5;
    if (launch_decode_tc(pl, st) != cudaSuccess) return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace pa
