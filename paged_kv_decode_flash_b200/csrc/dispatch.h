// dispatch.h -- host-side planning and launch shared by the C entry points
// (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "pagedattn.h"

namespace pa {

// Which kernel a call uses, and how the context is split.
struct Plan {
  bool tensor_cores;
  int splits, blocks_per_split;
  int ctas;  // tensor-core kernel: CTAs of the grid (the device shares them out
             // among the (sequence, KV head) groups); splits = ceil(ctas / groups)
  int tiles_per_item;  // tensor-core kernel: 0, or the item size of a batched grid
};

// Workspace: status header | arrival counters | split partial outputs |
// split partial log-sum-exps.  Header and counters (the zero prefix) must be
// zero before the first call; every call leaves the counters at zero.
struct WsLayout {
  size_t part_out, part_lse, total;
};

int check_dims(const pa_dims* d, int n_query);
int check_decode_args(const void* q, const void* k, const void* v, const int32_t* bt,
                      const int32_t* cl, int causal, int window, float scale, int kv_dtype,
                      const void* out);
Plan make_plan(const pa_dims* d, int n_query, int kv_dtype, int sms);
// The largest plan any device can choose (sizes workspaces without a device).
Plan max_plan(const pa_dims* d);
WsLayout ws_layout(const pa_dims* d, int n_query, int splits);
size_t ws_zero_prefix(const pa_dims* d);
int device_sm_count();

// Enqueue one decode with a prepared plan on `ws` (>= ws_layout(...).total
// bytes, 256-byte aligned, zero prefix).  Returns a pa_status.
int enqueue_decode(const pa_dims* d, const Plan& plan, const void* q, const void* k_cache,
                   const void* v_cache, const int32_t* block_table, const int32_t* context_lens,
                   int n_query, int causal, int window, float scale, int kv_dtype, void* out,
                   void* ws, cudaStream_t stream);

}  // namespace pa
