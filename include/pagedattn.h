/*
 * pagedattn.h -- C ABI of libpagedattn: decode attention over a paged KV
 * cache on NVIDIA B200 (sm_100a).
 *
 * The operation ("Dual MI50, part 2: from 10 to 74 tokens/s, a 200k-token
 * context, and two attention kernels", sbm-labs blog):
 *   - section "Decode: a new kernel for the shape MTP actually runs": one
 *     decode or speculative-verify step checks several query tokens per
 *     sequence, several query heads share one KV head (grouped-query
 *     attention), the work is split along the context so every compute unit
 *     is busy, and the split partial results are merged at the end; the
 *     kernel allocates nothing and never waits on the CPU, so it can run
 *     inside captured GPU graphs;
 *   - section "Bug 2: the drafter read freed memory": KV lives in fixed-size
 *     blocks reached through a block table; an optional sliding window keeps
 *     only the most recent W tokens visible and is expressed as a mask; the
 *     drafter uses a non-causal path;
 *   - sections "200k context for coding agents" and "Prefill: teach the
 *     fork's fast kernel to read the int8 cache": an int8 KV cache with
 *     scales (vLLM's has one scale per row) is what makes a 200k-token
 *     context fit; scale products and accumulators are fp32.
 *
 * For every sequence s, query token i < n_query and query head h the call
 * computes softmax(scale * q K^T) V over the keys j of sequence s that are
 * visible to (s, i):
 *   p_i = L_s - n_query + i        (the new tokens are the last n_query
 *                                    positions; L_s = context_lens[s]
 *                                    includes them and their K/V are
 *                                    already in the cache)
 *   causal:      j <= p_i          non-causal: j <= L_s - 1
 *   window W>0:  j >= anchor - W + 1, anchor = p_i (causal) or L_s - 1
 *   always       0 <= j < L_s
 * Key j of sequence s is row (j % block_size) of physical block
 * block_table[s * max_blocks_per_seq + j / block_size].  Query head h reads
 * KV head h / (num_q_heads / num_kv_heads).
 *
 * Layouts (all contiguous, row-major, device memory unless stated):
 *   q, out        fp16 [num_seqs][n_query][num_q_heads][head_dim]
 *   k/v cache     PA_KV_FP16: fp16 [num_blocks][num_kv_heads][block_size][head_dim]
 *                 PA_KV_Q8_0: bytes [num_blocks][num_kv_heads][tile], one tile =
 *                   int8 qs[block_size][head_dim] followed by
 *                   fp16 d[block_size][head_dim/32]; element value = qs * d of
 *                   its group of 32 consecutive head_dim elements; scales of
 *                   keys a query can see must be finite with |d| <= 512
 *                   (true of any cache quantised from fp16 data whose
 *                   magnitudes stay below 65024, d = amax / 127)
 *                 PA_KV_INT8_ROW: bytes [num_blocks][num_kv_heads][tile], one
 *                   tile = int8 qs[block_size][head_dim] followed by
 *                   fp32 s[block_size]; element value = qs * s of its row;
 *                   scales of visible keys must be finite with |s| <= 512
 *                   (each value reaches the tensor core as two fp16 parts:
 *                   relative error below 2^-21, absolute below 2^-25)
 *   block_table   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens  int32 [num_seqs]
 * Supported: head_dim 128; block_size a multiple of 16 (the kernels work in
 * 16-key chunks; sizes 16 to 112 are exercised by the tests); n_query
 * 1..128; num_q_heads a multiple of num_kv_heads with
 * n_query * num_q_heads / num_kv_heads <= 1024.  A KV head's rows are cut
 * into parts of at most 32 (fp16) or 16 (int8 caches) rows, each of which
 * reads the keys its tokens see: a chunk of many tokens (a long verify, a
 * prefill chunk appended to the cache) costs one pass over its visible KV
 * per part.
 *
 * Ownership and synchronisation: the caller owns every buffer, including the
 * workspace.  Calls allocate nothing, never synchronise the host with the
 * device (except paged_attn_get_error, which says so) and only enqueue work
 * on `stream` (a cudaStream_t passed as void*; NULL = the legacy default
 * stream).  Pointers are read during the call only where noted "host".
 *
 * Errors: every call returns 0 (PA_OK) or a negative pa_status.  Argument
 * errors are found on the host before anything is enqueued.  Data errors
 * that only the device can see (a block index outside [0, num_blocks), a
 * context length outside [n_query, max_blocks_per_seq * block_size]) do not
 * trap and never dereference the bad index: the rows of a sequence with a
 * bad length are written as 0, and so are the rows of a (sequence, KV head)
 * whose visible keys reach an out-of-range block; either way a flag is
 * raised in the workspace that paged_attn_get_error reports.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_KV_FP16 = 0, PA_KV_Q8_0 = 1, PA_KV_INT8_ROW = 2 } pa_kv_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = -1,    /* null pointer, bad shape or flag */
  PA_ERR_UNSUPPORTED = -2,    /* valid but not implemented (e.g. head_dim) */
  PA_ERR_WORKSPACE = -3,      /* workspace missing, misaligned or too small */
  PA_ERR_CUDA = -4,           /* a CUDA runtime call or launch failed */
  PA_ERR_BAD_BLOCK_INDEX = -5,/* device saw block_table entry out of range */
  PA_ERR_BAD_CONTEXT_LEN = -6,/* device saw context_lens out of range */
  PA_ERR_TIMEOUT = -7         /* a device-side wait gave up (kernel left early) */
} pa_status;

/* Static shapes of one call.  Host memory, read during the call only. */
typedef struct {
  int32_t num_seqs;           /* batch; >= 1 */
  int32_t num_q_heads;        /* Hq */
  int32_t num_kv_heads;       /* Hkv; Hq % Hkv == 0 */
  int32_t head_dim;           /* 128 */
  int32_t block_size;         /* tokens per KV block; a multiple of 16 */
  int32_t max_blocks_per_seq; /* row stride of block_table */
  int32_t num_blocks;         /* physical blocks in the pool (bounds check) */
  void* workspace;            /* device, caller-owned, 256-byte aligned */
  size_t workspace_bytes;     /* >= paged_attn_workspace_size(dims, n_query) */
} pa_dims;

/* Bytes of workspace paged_attn_decode needs for these shapes, any cache
 * type, any device: a 256-byte status header, arrival and queue counters
 * and the split partials.  Host only, no device access.  Returns 0 for
 * invalid shapes. */
size_t paged_attn_workspace_size(const pa_dims* dims, int32_t n_query);

/* Zero the workspace status header and counters (enqueued on `stream`).
 * Call once after allocating a workspace, before its first
 * paged_attn_decode; every decode call leaves the counters ready for the
 * next, a timed-out one included. */
int paged_attn_workspace_init(const pa_dims* dims, void* stream);

/* Decode attention (see the header comment for the exact definition).
 * q, k_cache, v_cache, block_table, context_lens, out: device pointers,
 * 16-byte aligned.  n_query in 1..128; causal 0 or 1; window >= 0 (0 = no
 * window); scale multiplies q.k (usually 1/sqrt(head_dim)); kv_dtype a
 * pa_kv_dtype.  Enqueues the split-KV kernel, whose CTAs also merge the
 * split partials, on `stream` (see paged_attn_launches_per_call).  Calls
 * that share a workspace must not overlap on the GPU (order them on one
 * stream).  A sequence's result depends only on its own inputs, and
 * repeated calls give bit-identical results. */
int paged_attn_decode(const pa_dims* dims, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_table,
                      const int32_t* context_lens, int32_t n_query,
                      int32_t causal, int32_t window, float scale,
                      int32_t kv_dtype, void* out, void* stream);

/* Partial decode of a share of each sequence's keys, for context-parallel
 * decode across GPUs ("Dual MI50, part 2", section "Decode: a new kernel
 * for the shape MTP actually runs": the work is split along the context
 * and the partial results are merged at the end).  The same computation as
 * paged_attn_decode, restricted for sequence s to the keys j in
 * [key_begin[s], key_begin[s] + key_count[s]) (device int32 [num_seqs]);
 * context_lens are the full lengths, so query positions and masks are the
 * global ones.  key_begin[s] must be a multiple of block_size, the range
 * must lie inside [0, L_s), and block_table row s maps the LOCAL block b
 * (keys key_begin[s] + b * block_size ...) to a physical block of this
 * call's cache pool.  Instead of fp16 rows it writes, per row,
 *   out      fp32 [num_seqs][n_query][num_q_heads][head_dim]: the softmax-
 *            weighted mean of V over the row's visible keys in the range
 *   out_lse  fp32 [num_seqs][n_query][num_q_heads]: the natural log of
 *            sum exp(scale q.k) over them
 * (0 and -inf for a row that sees none of them).  paged_attn_merge over the
 * ranks' (out, out_lse) gives the full-context result.  A range that is not
 * whole blocks inside the context and the table is a data error
 * (PA_ERR_BAD_CONTEXT_LEN from paged_attn_get_error). */
int paged_attn_decode_partial(const pa_dims* dims, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_table,
                              const int32_t* context_lens, const int32_t* key_begin,
                              const int32_t* key_count, int32_t n_query, int32_t causal,
                              int32_t window, float scale, int32_t kv_dtype, float* out,
                              float* out_lse, void* stream);

/* Log-sum-exp merge of split partials ("Dual MI50, part 2", section
 * "Decode: a new kernel for the shape MTP actually runs": partial results
 * are merged at the end).  For each row r:
 *   M = max_s lse[s][r];  w_s = exp(lse[s][r] - M)  (0 for lse = -inf)
 *   out[r] = sum_s w_s partial_out[s][r] / sum_s w_s   (fp16, round to
 *   nearest even);  out_lse[r] = M + log(sum_s w_s)
 * A row whose every split has lse = -inf gets out = 0, out_lse = -inf.
 *   partial_out  fp32 [num_splits][rows][head_dim]   (device)
 *   partial_lse  fp32 [num_splits][rows], natural log (device)
 *   out          fp16 [rows][head_dim]               (device)
 *   out_lse      fp32 [rows] or NULL                 (device)
 * num_splits >= 1, rows >= 0, head_dim in {64, 128, 256}. */
int paged_attn_merge(const float* partial_out, const float* partial_lse,
                     int32_t num_splits, int32_t rows, int32_t head_dim,
                     void* out, float* out_lse, void* stream);

/* Synchronises `stream`, then returns and clears the device-side data-error
 * flag of the workspace: PA_OK, PA_ERR_TIMEOUT, PA_ERR_BAD_BLOCK_INDEX or
 * PA_ERR_BAD_CONTEXT_LEN (the first of these that was raised, in that order),
 * or PA_ERR_CUDA if the stream reports an error.  PA_ERR_TIMEOUT means a
 * pipeline wait inside a kernel passed its time limit: the kernel released
 * its resources and returned and its output is not valid; the workspace
 * stays usable (this call also clears its counters, as a safety net). */
int paged_attn_get_error(const pa_dims* dims, void* stream);

/* Sets the time after which a device-side pipeline wait gives up (raising
 * PA_ERR_TIMEOUT) for calls enqueued afterwards by this process, and
 * returns the previous value.  0 restores the default of one second.  A
 * test aid: a limit the pipeline cannot meet makes the kernels exercise
 * their give-up path without faulting or hanging the GPU. */
uint64_t paged_attn_set_wait_limit(uint64_t nanoseconds);

/* Debug: paged_attn_decode (same arguments and output) that also records,
 * for every output row, which keys the decode kernel scored and where it
 * read them: trace is device int32 [num_seqs][n_query][num_q_heads][5] =
 *   {visible key count, min j, max j, xor of physical slot ids,
 *    sum of physical slot ids mod 2^32},
 * physical slot id = block * block_size + slot of the K row the kernel
 * copied; rows without keys get {0, -1, -1, 0, 0}.  Slower (atomics per
 * scored pair): tests only. */
int paged_attn_trace(const pa_dims* dims, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_table,
                     const int32_t* context_lens, int32_t n_query, int32_t causal,
                     int32_t window, float scale, int32_t kv_dtype, void* out,
                     int32_t* trace, void* stream);

/* Writes the keys and values of the n_new newest tokens of every sequence
 * into the paged cache: token i < n_new of sequence s sits at position
 * L_s - n_new + i (L_s = context_lens[s], which includes them), in slot
 * position % block_size of block block_table[s][position / block_size].
 *   k_new, v_new  fp16 [num_seqs][n_new][num_kv_heads][head_dim] (device)
 *   k/v cache     the layouts above (device, written)
 * The int8 caches are quantised on the way, in fp32 with IEEE rounding:
 *   PA_KV_Q8_0, per 32 elements: d = fp16(amax / 127),
 *     q = d > 0 ? clamp(round_half_away(x / d), -127, 127) : 0;
 *   PA_KV_INT8_ROW, per row: s = amax / 127, q as above with s.
 * Uses the status word of dims->workspace (>= 256 bytes) for data errors (a
 * block index or context length out of range: that row is not written),
 * which paged_attn_get_error reports.  n_new in 1..16. */
int paged_attn_cache_write(const pa_dims* dims, const void* k_new, const void* v_new,
                           const int32_t* block_table, const int32_t* context_lens,
                           int32_t n_new, int32_t kv_dtype, void* k_cache, void* v_cache,
                           void* stream);

/* The most split partials one (sequence, KV head, row part) of a call with
 * these shapes and cache type is merged from on the current device (host
 * only; negative pa_status on error). */
int paged_attn_num_splits(const pa_dims* dims, int32_t n_query, int32_t kv_dtype);

/* Allocation-free variant of paged_attn_decode.  The paper has no
 * counterpart: it exists for callers that cannot give the library device
 * memory of its own -- programs whose host owns every byte of device memory
 * (a serving engine with one fixed pool planned at start-up, a plug-in host
 * without an allocator) or hot paths that must not call cudaMalloc, which can
 * implicitly synchronise the device.  Same arguments, layouts and results as
 * paged_attn_decode (bit-identical); the workspace fields of *dims are
 * ignored.  The split partials live in one array of PA_NOALLOC_SCRATCH_BYTES
 * inside the library's device image, held by every GPU that loads the
 * library until exit; shapes that need more return PA_ERR_WORKSPACE before
 * anything is enqueued.  All calls on a device share that array: calls whose
 * work overlaps on the GPU race and corrupt each other, so order them (one
 * stream, or events).  The first call on a device looks up the array's
 * device address and caches it (safe from several host threads); make it
 * before any stream capture begins.  The array's counters and status word
 * are cleared at the start of every call, so device-side data errors are
 * handled as in paged_attn_decode (masked keys, zeroed rows) but are not
 * reported, and neither is a timeout of a device-side wait: such a call
 * leaves its output undefined and cannot be detected. */
#define PA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int paged_attn_decode_noalloc(const pa_dims* dims, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_table,
                              const int32_t* context_lens, int32_t n_query,
                              int32_t causal, int32_t window, float scale,
                              int32_t kv_dtype, void* out, void* stream);

/* Measurement aid, not part of the attention: streams `bytes` (rounded
 * down to 32 KB) of device memory at `src` (16-byte aligned) into shared
 * memory the way the decode kernel moves KV tiles (4 KB bulk copies into a
 * ring of 32 KB slots, completion on mbarriers, six slots in flight) on
 * `ctas` CTAs, and writes one word per CTA to sink (device uint32
 * [ctas]; 0xdeadbeef from a CTA whose wait timed out).  Timing it gives the
 * read-only HBM ceiling of that access pattern. */
int paged_attn_stream_read(const void* src, size_t bytes, uint32_t* sink, int32_t ctas,
                           void* stream);

/* Kernel launches one paged_attn_decode call makes for these shapes and
 * cache type on the current device: 1, or, for a batch large enough to use
 * the work queue, one per 256 sequences.  Host only; negative pa_status on
 * error. */
int32_t paged_attn_launches_per_call(const pa_dims* dims, int32_t n_query, int32_t kv_dtype);

/* Static string for a pa_status. */
const char* paged_attn_status_string(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H */
