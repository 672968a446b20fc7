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
 *     scales is what makes a 200k-token context fit.
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
 *                 PA_KV_Q8_0: bytes [num_blocks][num_kv_heads][tile] with one
 *                   tile = int8 qs[block_size][head_dim] followed by
 *                   fp16 d[block_size][head_dim/32]; element value = qs * d of
 *                   its group of 32 consecutive head_dim elements; scales of
 *                   keys that a query can see must be finite with |d| < 1024
 *                   (true of any cache quantised from fp16 data, where
 *                   d = amax / 127 <= 516): larger ones give non-finite rows
 *   block_table   int32 [num_seqs][max_blocks_per_seq]
 *   context_lens  int32 [num_seqs]
 * Supported: head_dim 128; block_size a multiple of 16 (the kernels work in
 * 16-key chunks; sizes 16 to 112 are exercised by the tests); n_query 1..8;
 * num_q_heads a multiple of num_kv_heads with
 * n_query * num_q_heads / num_kv_heads <= 64.
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
 * bad length are written as 0; rows whose visible keys reach an out-of-range
 * block get finite values that are otherwise unspecified (the tensor-core
 * kernel writes the rows of that (sequence, KV head) as 0, the CUDA-core
 * kernel leaves the block's keys out); either way a flag is raised in the
 * workspace that paged_attn_get_error reports.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_KV_FP16 = 0, PA_KV_Q8_0 = 1 } pa_kv_dtype;

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

/* Bytes of workspace paged_attn_decode needs for these shapes: a 256-byte
 * status header, two int32 arrival counters per (sequence, KV head) and the
 * split partials.  Host only, no device access.  Returns 0 for invalid
 * shapes. */
size_t paged_attn_workspace_size(const pa_dims* dims, int32_t n_query);

/* Zero the workspace status header and arrival counters (enqueued on
 * `stream`).  Call once after allocating a workspace, before its first
 * paged_attn_decode; every decode call leaves the counters ready for the
 * next (their low 31 bits at zero). */
int paged_attn_workspace_init(const pa_dims* dims, void* stream);

/* Decode attention (see the header comment for the exact definition).
 * q, k_cache, v_cache, block_table, context_lens, out: device pointers,
 * 16-byte aligned.  n_query in 1..8; causal 0 or 1; window >= 0 (0 = no
 * window); scale multiplies q.k (usually 1/sqrt(head_dim)); kv_dtype a
 * pa_kv_dtype.  Enqueues the split-KV kernel and the merge of its partials
 * on `stream` (see paged_attn_launches_per_call).  Calls that share a
 * workspace must not overlap on the GPU (order them on one stream). */
int paged_attn_decode(const pa_dims* dims, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* block_table,
                      const int32_t* context_lens, int32_t n_query,
                      int32_t causal, int32_t window, float scale,
                      int32_t kv_dtype, void* out, void* stream);

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
 * pipeline wait inside a kernel passed its time limit (about a second): the
 * kernel released its resources and returned, and its output is not valid. */
int paged_attn_get_error(const pa_dims* dims, void* stream);

/* Debug: the key-resolution record of every row, computed on the device
 * with the same range, mask and block-table code the decode kernels use.
 * trace: device int32 [num_seqs][n_query][num_q_heads][5] =
 *   {visible key count, min j, max j, xor of physical slot ids,
 *    sum of physical slot ids mod 2^32}, physical slot id =
 *   block * block_size + slot; empty rows {0, -1, -1, 0, 0}.
 * Cost grows with the context (one thread walks each row): tests only. */
int paged_attn_trace(const pa_dims* dims, const int32_t* block_table,
                     const int32_t* context_lens, int32_t n_query,
                     int32_t causal, int32_t window, int32_t* trace,
                     void* stream);

/* Number of key splits paged_attn_decode uses for these shapes and cache
 * type on the current device (host only; negative pa_status on error). */
int32_t paged_attn_num_splits(const pa_dims* dims, int32_t n_query, int32_t kv_dtype);

/* Allocation-free variant of paged_attn_decode.  The paper has no
 * counterpart: it exists for callers that cannot give the library device
 * memory of its own -- programs whose host owns every byte of device memory
 * (a serving engine with one fixed pool planned at start-up, a plug-in host
 * without an allocator) or hot paths that must not call cudaMalloc, which can
 * implicitly synchronise the device.  Same arguments, layouts and results as
 * paged_attn_decode; the workspace fields of *dims are ignored.  The split
 * partials live in one array of PA_NOALLOC_SCRATCH_BYTES inside the
 * library's device image, held by every GPU that loads the library until
 * exit; shapes that need more return PA_ERR_WORKSPACE before anything is
 * enqueued.  All calls on a device share that array: calls whose work
 * overlaps on the GPU race and corrupt each other, so order them (one
 * stream, or events).  The first call on a device looks up the array's
 * device address and caches it; make it before any stream capture begins.
 * Device-side data errors are handled as in paged_attn_decode (masked keys,
 * zeroed rows) but are not reported: the status word is cleared per call. */
#define PA_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int paged_attn_decode_noalloc(const pa_dims* dims, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_table,
                              const int32_t* context_lens, int32_t n_query,
                              int32_t causal, int32_t window, float scale,
                              int32_t kv_dtype, void* out, void* stream);

/* Kernel launches one paged_attn_decode call makes for these shapes and
 * cache type on the current device: 1 where the tensor-core kernel runs (its
 * CTAs also merge the split partials of each (sequence, KV head)), 2 for
 * the CUDA-core kernel followed by the merge kernel (launched as a
 * programmatic dependent so that it starts as soon as the split-KV kernel
 * ends).  Host only; negative pa_status on error. */
int32_t paged_attn_launches_per_call(const pa_dims* dims, int32_t n_query, int32_t kv_dtype);

/* Static string for a pa_status. */
const char* paged_attn_status_string(int32_t status);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDATTN_H */
