// dispatch.h -- host-side planning and launch shared by the C entry points
// (internal to the library).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "pagedattn.h"

namespace pa {

// How one call's work is cut (the work decomposition is described with
// DecodeParams in common.cuh).
struct Plan {
  int mode;             // 0: static partition (few groups), 1: work queue (a batch)
  int halves;           // row parts per KV head
  int rows_half;        // rows per part
  int ctas;             // CTAs per launch
  int ctas_per_set;     // mode 0: CTAs per (sequence, part)
  int item_tiles;       // mode 1: 128-key tiles per big item
  int slots_per_group;  // mode 1: partial slots per group
  int launches;         // kernel launches of the call
  long long slots;      // partial slots of the whole call
  int split_ctas;       // > 0: the call runs the per-head split kernel on this many CTAs
};

// Workspace: status header | arrival counters (two per group) | queue
// counters (one per launch) | split partial outputs | split partial
// log-sum-exps.  The header and the counters (the zero prefix) must be zero
// before the first call; every call leaves the counters at zero.
struct WsLayout {
  size_t arrivals, queue, part_out, part_lse, total;
};

int check_dims(const pa_dims* d, int n_query);
int check_decode_args(const void* q, const void* k, const void* v, const int32_t* bt,
                      const int32_t* cl, int causal, int window, float scale, int kv_dtype,
                      const void* out);
Plan make_plan(const pa_dims* d, int n_query, int kv_dtype, int sms);
size_t ws_zero_prefix(const pa_dims* d);
WsLayout ws_layout(const pa_dims* d, int n_query, const Plan& plan);
// Bytes a workspace needs for any cache type on any device.
size_t ws_size_any_device(const pa_dims* d, int n_query);
int device_sm_count();
// Wait limit of device-side pipeline waits for calls enqueued from now on.
unsigned long long wait_limit_ns();
unsigned long long set_wait_limit_ns(unsigned long long ns);

// Partial mode (context-parallel decode): every pointer null, or the key
// range of each sequence and the fp32 outputs (see DecodeParams).
struct PartialArgs {
  const int32_t* key_begin = nullptr;
  const int32_t* key_count = nullptr;
  float* out = nullptr;
  float* out_lse = nullptr;
};

// Enqueue one decode with a prepared plan on `ws` (>= ws_layout(...).total
// bytes, 256-byte aligned, zero prefix).  trace: null, or the key-resolution
// record (set up by the caller).  Returns a pa_status.
int enqueue_decode(const pa_dims* d, const Plan& plan, const void* q, const void* k_cache,
                   const void* v_cache, const int32_t* block_table, const int32_t* context_lens,
                   int n_query, int causal, int window, float scale, int kv_dtype, void* out,
                   void* ws, int32_t* trace, cudaStream_t stream,
                   const PartialArgs& partial = PartialArgs());

}  // namespace pa
