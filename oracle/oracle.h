/*
 * oracle.h -- plain fp64 CPU reference for paged-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load or call this code; the product
 * path (the CUDA library) never does, and the two share no source.
 *
 * What it computes: for every sequence s, query token i and query head h,
 * exact softmax attention of that query over the keys/values of sequence s,
 * where key j lives in physical KV block block_table[s][j / block_size] at
 * slot j % block_size (paged KV cache; "Dual MI50, part 2", section "Bug 2:
 * the drafter read freed memory": vLLM's cache manager hands out fixed-size
 * KV blocks and frees/reuses them).  Everything is fp64; the fp16 and q8_0
 * inputs are decoded exactly ("Dual MI50, part 2", section "Did quality
 * change?": both attention kernels were checked against a float64
 * reference).
 */
#ifndef PAGEDATTN_ORACLE_H
#define PAGEDATTN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORACLE_KV_FP16 = 0, ORACLE_KV_Q8_0 = 1, ORACLE_KV_INT8_ROW = 2 };

enum {
  ORACLE_OK = 0,
  ORACLE_ERR_INVALID_ARG = -1,
  ORACLE_ERR_BAD_BLOCK_INDEX = -2,
  ORACLE_ERR_BAD_CONTEXT_LEN = -3,
  ORACLE_ERR_NOMEM = -4
};

/* One decode problem.  All pointers are host memory owned by the caller.
 *   q            fp16 bits  [num_seqs][n_query][num_q_heads][head_dim]
 *   k/v_cache    fp16:  fp16 bits [num_blocks][num_kv_heads][block_size][head_dim]
 *                q8_0:  bytes [num_blocks][num_kv_heads][tile], one tile =
 *                       int8 qs[block_size][head_dim] followed by
 *                       fp16 d[block_size][head_dim/32]
 *                int8 rows: bytes [num_blocks][num_kv_heads][tile], one tile =
 *                       int8 qs[block_size][head_dim] followed by
 *                       fp32 s[block_size]
 *   block_table  int32 [num_seqs][max_blocks_per_seq]
 *   context_lens int32 [num_seqs]; includes the n_query new tokens
 */
typedef struct {
  int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, block_size;
  int32_t max_blocks_per_seq, num_blocks;
  int32_t n_query, causal, window, kv_dtype;
  double scale;
  const uint16_t* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_table;
  const int32_t* context_lens;
} oracle_problem;

/* Exact fp16 -> fp64 decode (bit manipulation). */
double oracle_half_to_double(uint16_t h);

/* Is key j visible to query token i of a sequence of length L? */
int oracle_key_visible(int64_t L, int32_t n_query, int32_t i, int32_t causal,
                       int32_t window, int64_t j);

/* Attention of one row (s, i, h) restricted to keys j in [j_begin, j_end).
 * out_row gets head_dim fp64 values, *lse the natural-log sum of exp of the
 * scaled scores.  No visible key: out_row = 0, *lse = -inf. */
int oracle_attend_row(const oracle_problem* p, int32_t s, int32_t i, int32_t h,
                      int64_t j_begin, int64_t j_end, double* out_row,
                      double* lse);

/* All rows.  out [num_seqs][n_query][num_q_heads][head_dim],
 * lse [num_seqs][n_query][num_q_heads] (nullable).  OpenMP over rows when
 * compiled with it. */
int oracle_paged_attn(const oracle_problem* p, double* out, double* lse);

/* A subset of rows; row id r = (s * n_query + i) * num_q_heads + h.
 * out [n_rows][head_dim], lse [n_rows] (nullable). */
int oracle_paged_attn_rows(const oracle_problem* p, const int64_t* row_ids,
                           int64_t n_rows, double* out, double* lse);

/* Key resolution record per row: {visible count, min j, max j,
 * xor of physical slot ids, sum of physical slot ids mod 2^32}, with the
 * physical slot id of key j = block * block_size + slot.  Empty rows give
 * {0, -1, -1, 0, 0}.  trace is int32 [rows][5] in row-id order. */
int oracle_trace(const oracle_problem* p, int32_t* trace);

/* Log-sum-exp merge of split partials: part_out [S][rows][D],
 * part_lse [S][rows] -> out [rows][D], out_lse [rows] (nullable). */
void oracle_merge(const double* part_out, const double* part_lse, int32_t S,
                  int64_t rows, int32_t D, double* out, double* out_lse);

/* Threads an oracle_paged_attn call will use; oracle_set_num_threads
 * changes it (n >= 1). */
int oracle_num_threads(void);
void oracle_set_num_threads(int n);

/* Quantise-on-write, fp32 arithmetic with IEEE rounding:
 *   oracle_float_to_half: fp32 -> fp16 bits, round to nearest even;
 *   oracle_quantize_q8_0: 32 values -> int8 q[32] and the fp16 scale
 *     d = fp16(amax / 127), q = clamp(round_half_away(x / d), -127, 127)
 *     (all zero when d = 0);
 *   oracle_quantize_row: n values -> int8 q[n] and the fp32 scale
 *     s = amax / 127, q likewise with s.
 * oracle_cache_write: for every sequence s, new token i < p->n_query (the
 * last n_query positions of context_lens[s]) and KV head h, write row
 * k_new/v_new [s][i][h][:] (fp16 bits, [num_seqs][n_query][Hkv][head_dim])
 * into its slot of k_cache / v_cache (p->kv_dtype layout), quantised as
 * above.  Rows with a bad context length or block index are skipped and the
 * first such error is returned. */
uint16_t oracle_float_to_half(float f);
void oracle_quantize_q8_0(const float* x, int8_t* q, uint16_t* d_bits);
void oracle_quantize_row(const float* x, int32_t n, int8_t* q, float* s);
int oracle_cache_write(const oracle_problem* p, const uint16_t* k_new, const uint16_t* v_new,
                       void* k_cache, void* v_cache);

#ifdef __cplusplus
}
#endif
#endif
