/*
 * oracle.c -- plain, slow, obviously correct fp64 CPU reference for
 * paged-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the test suite, the smoke check and
 * the benchmark's CPU-baseline leg, never by the product path.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section):
 *  - "Dual MI50, part 2: from 10 to 74 tokens/s, a 200k-token context, and
 *    two attention kernels" (sbm-labs blog)
 *      * "Bug 2: the drafter read freed memory": KV lives in fixed-size
 *        blocks handed out and reused by vLLM's cache manager; a sliding
 *        window keeps only the most recent W tokens visible, expressed as a
 *        mask; a non-causal drafter path exists.
 *      * "Decode: a new kernel for the shape MTP actually runs": several
 *        query tokens per step (speculative verify), several query heads
 *        sharing one KV head (grouped-query attention), split along the
 *        context with the partial results merged at the end.
 *      * "Prefill: teach the fork's fast kernel to read the int8 cache" and
 *        "Did quality change?": int8 KV with scales, checked against a
 *        float64 reference.
 *  The method computes exact attention, softmax(scale * q K^T) V over the
 *  visible keys, so this file is that definition written out in fp64, one
 *  row at a time, with no blocking, splitting or reordering.
 *
 * Readings where the pages are silent (stated once here, used throughout):
 *  - the n_query new tokens are the last n_query positions of the context:
 *    query i sits at position p_i = L - n_query + i;
 *  - causal: key j is visible to query i iff j <= p_i; non-causal: every
 *    j < L is visible;
 *  - window W > 0 keeps exactly W keys ending at the anchor, j >= anchor-W+1,
 *    where the anchor is p_i (causal) or L-1 (non-causal);
 *  - query head h reads KV head h / (num_q_heads / num_kv_heads);
 *  - q8_0: value = int8 q times the fp16 scale d of its group of 32
 *    consecutive head_dim elements (exact in fp64);
 *  - int8 with row scales ("Prefill: teach the fork's fast kernel to read
 *    the int8 cache": vLLM's int8 cache has per-row scales): value = int8 q
 *    times the fp32 scale of its (token, head) row (exact in fp64);
 *  - writing new tokens into the cache (the step before attention; "Bug 2":
 *    vLLM's cache manager assigns the blocks) quantises in fp32 with IEEE
 *    rounding, the precision the kernel decides in: q8_0 d = fp16(amax/127)
 *    per 32 elements, int8 rows s = amax/127 per row, q = round half away
 *    from zero of x / d (or x / s), clamped to [-127, 127];
 *  - lse is the natural log of sum_j exp(scale * q.k_j).
 *
 * Building with -DORACLE_PLANT=n plants one deliberate mistake (used only by
 * the test that shows the pins catch such mistakes); the default build has
 * none.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

double oracle_half_to_double(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1f;
  const int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* zero or subnormal: m * 2^-24 */
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(m | 0x400), e - 25); /* (1 + m/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

int oracle_key_visible(int64_t L, int32_t n_query, int32_t i, int32_t causal,
                       int32_t window, int64_t j) {
  if (j < 0 || j >= L) return 0;
  int64_t p = L - n_query + i; /* position of query token i */
#if ORACLE_PLANT == 2
  p += 1; /* planted: causal edge off by one */
#endif
  if (causal && j > p) return 0;
  if (window > 0) {
    const int64_t anchor = causal ? p : L - 1;
#if ORACLE_PLANT == 1
    if (j < anchor - window) return 0; /* planted: window one key too wide */
#else
    if (j < anchor - window + 1) return 0;
#endif
  }
  return 1;
}

/* Physical location of logical key j of sequence s: block id and slot.
 * Returns 0, or ORACLE_ERR_BAD_BLOCK_INDEX. */
static int resolve_key(const oracle_problem* p, int32_t s, int64_t j,
                       int64_t* block, int32_t* slot) {
  const int64_t logical_block = j / p->block_size;
  const int64_t b =
      p->block_table[(int64_t)s * p->max_blocks_per_seq + logical_block];
  if (b < 0 || b >= p->num_blocks) return ORACLE_ERR_BAD_BLOCK_INDEX;
  *block = b;
  *slot = (int32_t)(j % p->block_size);
  return ORACLE_OK;
}

/* Element d of the key (or value) row at (block, kv head, slot), in fp64. */
static double cache_value(const oracle_problem* p, const void* cache,
                          int64_t block, int32_t kvh, int32_t slot, int32_t d) {
  const int64_t D = p->head_dim, bs = p->block_size, H = p->num_kv_heads;
  if (p->kv_dtype == ORACLE_KV_FP16) {
    const uint16_t* c = (const uint16_t*)cache;
#if ORACLE_PLANT == 4
    /* planted: block and head axes swapped */
    const int64_t row = ((int64_t)kvh * p->num_blocks + block) * bs + slot;
#else
    const int64_t row = (block * H + kvh) * bs + slot;
#endif
    return oracle_half_to_double(c[row * D + d]);
  } else if (p->kv_dtype == ORACLE_KV_INT8_ROW) {
    /* int8 with one fp32 scale per (token, head) row: value = q * s */
    const int64_t tile_bytes = bs * D + bs * 4;
    const uint8_t* tile = (const uint8_t*)cache + (block * H + kvh) * tile_bytes;
    const int8_t q = (int8_t)tile[(int64_t)slot * D + d];
    float s;
#if ORACLE_PLANT == 9
    memcpy(&s, tile + bs * D + (int64_t)((slot + 1) % bs) * 4, 4); /* planted: neighbour's scale */
#else
    memcpy(&s, tile + bs * D + (int64_t)slot * 4, 4);
#endif
    return (double)q * (double)s;
  } else {
    const int64_t groups = D / 32;
    const int64_t tile_bytes = bs * D + bs * groups * 2;
    const uint8_t* tile = (const uint8_t*)cache + (block * H + kvh) * tile_bytes;
    const int8_t q = (int8_t)tile[(int64_t)slot * D + d];
    uint16_t dbits;
#if ORACLE_PLANT == 7
    /* planted: scale of the wrong group */
    memcpy(&dbits, tile + bs * D + ((int64_t)slot * groups + 0) * 2, 2);
#else
    memcpy(&dbits, tile + bs * D + ((int64_t)slot * groups + d / 32) * 2, 2);
#endif
    return (double)q * oracle_half_to_double(dbits);
  }
}

static int check_problem(const oracle_problem* p) {
  if (!p || !p->q || !p->k_cache || !p->v_cache || !p->block_table ||
      !p->context_lens)
    return ORACLE_ERR_INVALID_ARG;
  if (p->num_seqs < 0 || p->num_q_heads <= 0 || p->num_kv_heads <= 0 ||
      p->head_dim <= 0 || p->block_size <= 0 || p->max_blocks_per_seq <= 0 ||
      p->num_blocks <= 0 || p->n_query <= 0 || p->window < 0)
    return ORACLE_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return ORACLE_ERR_INVALID_ARG;
  if (p->kv_dtype != ORACLE_KV_FP16 && p->kv_dtype != ORACLE_KV_Q8_0 &&
      p->kv_dtype != ORACLE_KV_INT8_ROW)
    return ORACLE_ERR_INVALID_ARG;
  if (p->kv_dtype == ORACLE_KV_Q8_0 && p->head_dim % 32 != 0)
    return ORACLE_ERR_INVALID_ARG;
  return ORACLE_OK;
}

int oracle_attend_row(const oracle_problem* p, int32_t s, int32_t i, int32_t h,
                      int64_t j_begin, int64_t j_end, double* out_row,
                      double* lse) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (s < 0 || s >= p->num_seqs || i < 0 || i >= p->n_query || h < 0 ||
      h >= p->num_q_heads)
    return ORACLE_ERR_INVALID_ARG;
  const int64_t L = p->context_lens[s];
  const int64_t cap = (int64_t)p->max_blocks_per_seq * p->block_size;
  if (L < p->n_query || L > cap) return ORACLE_ERR_BAD_CONTEXT_LEN;

  const int32_t D = p->head_dim;
  const int32_t group = p->num_q_heads / p->num_kv_heads;
#if ORACLE_PLANT == 3
  const int32_t kvh = h % p->num_kv_heads; /* planted: strided head mapping */
#else
  const int32_t kvh = h / group;
#endif
  const uint16_t* qbits =
      p->q + (((int64_t)s * p->n_query + i) * p->num_q_heads + h) * D;

  double* qd = (double*)malloc(sizeof(double) * D);
  const int64_t jb = j_begin < 0 ? 0 : j_begin;
  const int64_t je = j_end > L ? L : j_end;
  const int64_t nkeys = je > jb ? je - jb : 0;
  double* z = (double*)malloc(sizeof(double) * (nkeys ? nkeys : 1));
  int64_t* kb = (int64_t*)malloc(sizeof(int64_t) * (nkeys ? nkeys : 1));
  int32_t* ks = (int32_t*)malloc(sizeof(int32_t) * (nkeys ? nkeys : 1));
  if (!qd || !z || !kb || !ks) {
    free(qd); free(z); free(kb); free(ks);
    return ORACLE_ERR_NOMEM;
  }
  for (int32_t d = 0; d < D; ++d) qd[d] = oracle_half_to_double(qbits[d]);

  /* Scores z_j = scale * sum_d q[d] k_j[d] over the visible keys. */
  int64_t n = 0;
  for (int64_t j = jb; j < je; ++j) {
    if (!oracle_key_visible(L, p->n_query, i, p->causal, p->window, j)) continue;
    int64_t b;
    int32_t slot;
    rc = resolve_key(p, s, j, &b, &slot);
    if (rc) break;
    double dot = 0.0;
    for (int32_t d = 0; d < D; ++d)
      dot += qd[d] * cache_value(p, p->k_cache, b, kvh, slot, d);
#if ORACLE_PLANT == 5
    z[n] = dot; /* planted: scale dropped */
#else
    z[n] = p->scale * dot;
#endif
    kb[n] = b;
    ks[n] = slot;
    ++n;
  }

  if (rc == ORACLE_OK) {
    for (int32_t d = 0; d < D; ++d) out_row[d] = 0.0;
    if (n == 0) {
      if (lse) *lse = -INFINITY;
    } else {
      double m = z[0];
      for (int64_t t = 1; t < n; ++t)
        if (z[t] > m) m = z[t];
      double sum = 0.0;
      for (int64_t t = 0; t < n; ++t) {
#if ORACLE_PLANT == 6
        const double w = exp(m - z[t]); /* planted: sign error */
#else
        const double w = exp(z[t] - m);
#endif
        sum += w;
        for (int32_t d = 0; d < D; ++d)
          out_row[d] += w * cache_value(p, p->v_cache, kb[t], kvh, ks[t], d);
      }
      for (int32_t d = 0; d < D; ++d) out_row[d] /= sum;
#if ORACLE_PLANT == 8
      if (lse) *lse = log(sum); /* planted: max term dropped */
#else
      if (lse) *lse = m + log(sum);
#endif
    }
  }
  free(qd); free(z); free(kb); free(ks);
  return rc;
}

static int64_t num_rows(const oracle_problem* p) {
  return (int64_t)p->num_seqs * p->n_query * p->num_q_heads;
}

int oracle_paged_attn_rows(const oracle_problem* p, const int64_t* row_ids,
                           int64_t n_rows, double* out, double* lse) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int64_t total = num_rows(p);
  for (int64_t r = 0; r < n_rows; ++r)
    if (row_ids[r] < 0 || row_ids[r] >= total) return ORACLE_ERR_INVALID_ARG;
  int first_err = ORACLE_OK;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (int64_t r = 0; r < n_rows; ++r) {
    const int64_t id = row_ids[r];
    const int32_t h = (int32_t)(id % p->num_q_heads);
    const int32_t i = (int32_t)((id / p->num_q_heads) % p->n_query);
    const int32_t s = (int32_t)(id / ((int64_t)p->num_q_heads * p->n_query));
    double l;
    const int e = oracle_attend_row(p, s, i, h, 0, INT64_MAX,
                                    out + r * p->head_dim, &l);
    if (lse) lse[r] = l;
    if (e) {
#ifdef _OPENMP
#pragma omp critical
#endif
      if (first_err == ORACLE_OK) first_err = e;
    }
  }
  return first_err;
}

int oracle_paged_attn(const oracle_problem* p, double* out, double* lse) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int64_t total = num_rows(p);
  int64_t* ids = (int64_t*)malloc(sizeof(int64_t) * (total ? total : 1));
  double* l = (double*)malloc(sizeof(double) * (total ? total : 1));
  if (!ids || !l) {
    free(ids); free(l);
    return ORACLE_ERR_NOMEM;
  }
  for (int64_t r = 0; r < total; ++r) ids[r] = r;
  rc = oracle_paged_attn_rows(p, ids, total, out, l);
  if (lse)
    for (int64_t r = 0; r < total; ++r) lse[r] = l[r];
  free(ids);
  free(l);
  return rc;
}

int oracle_trace(const oracle_problem* p, int32_t* trace) {
  int rc = check_problem(p);
  if (rc) return rc;
  const int64_t total = num_rows(p);
  for (int64_t id = 0; id < total; ++id) {
    const int32_t i = (int32_t)((id / p->num_q_heads) % p->n_query);
    const int32_t s = (int32_t)(id / ((int64_t)p->num_q_heads * p->n_query));
    const int64_t L = p->context_lens[s];
    const int64_t cap = (int64_t)p->max_blocks_per_seq * p->block_size;
    if (L < p->n_query || L > cap) return ORACLE_ERR_BAD_CONTEXT_LEN;
    int32_t count = 0, jmin = -1, jmax = -1;
    uint32_t x = 0, sum = 0;
    for (int64_t j = 0; j < L; ++j) {
      if (!oracle_key_visible(L, p->n_query, i, p->causal, p->window, j))
        continue;
      int64_t b;
      int32_t slot;
      rc = resolve_key(p, s, j, &b, &slot);
      if (rc) return rc;
      const uint32_t phys = (uint32_t)(b * p->block_size + slot);
      if (count == 0) jmin = (int32_t)j;
      jmax = (int32_t)j;
      ++count;
      x ^= phys;
      sum += phys;
    }
    int32_t* t = trace + id * 5;
    t[0] = count;
    t[1] = jmin;
    t[2] = jmax;
    t[3] = (int32_t)x;
    t[4] = (int32_t)sum;
  }
  return ORACLE_OK;
}

void oracle_merge(const double* part_out, const double* part_lse, int32_t S,
                  int64_t rows, int32_t D, double* out, double* out_lse) {
  for (int64_t r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int32_t s = 0; s < S; ++s)
      if (part_lse[(int64_t)s * rows + r] > M) M = part_lse[(int64_t)s * rows + r];
    double* o = out + r * D;
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    if (M == -INFINITY) { /* no split saw a visible key */
      if (out_lse) out_lse[r] = -INFINITY;
      continue;
    }
    double wsum = 0.0;
    for (int32_t s = 0; s < S; ++s) {
      const double ls = part_lse[(int64_t)s * rows + r];
      if (ls == -INFINITY) continue; /* empty split: weight exactly zero */
      const double w = exp(ls - M);
      wsum += w;
      const double* po = part_out + ((int64_t)s * rows + r) * D;
      for (int32_t d = 0; d < D; ++d) o[d] += w * po[d];
    }
    for (int32_t d = 0; d < D; ++d) o[d] /= wsum;
    if (out_lse) out_lse[r] = M + log(wsum);
  }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* ---------------------------------------------------------------------------
 * Writing new tokens into the cache (quantise on write).
 * -------------------------------------------------------------------------*/

/* fp32 -> fp16 bits, round to nearest, ties to even (IEEE 754 binary16),
 * from the bit patterns.  A finite fp32 value is sig * 2^(E - 23) with sig
 * its 24-bit significand (implicit bit included) and E its unbiased
 * exponent.  In fp16 it becomes q units of 2^(E - 10) (normal range,
 * E >= -14) or of 2^-24 (subnormal), q = sig rounded to the shift that
 * drops the bits below that unit; the fp16 bits are then (E + 14) * 2^10 + q
 * (normal: q in [2^10, 2^11], where q = 2^11 carries into the exponent) or
 * q itself (subnormal: q = 2^10 is the smallest normal), infinity from
 * 0x7c00 up. */
uint16_t oracle_float_to_half(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const int32_t exp = (int32_t)((u >> 23) & 0xffu);
  const uint32_t mant = u & 0x7fffffu;
  if (exp == 0xff) return (uint16_t)(sign | 0x7c00u | (mant ? 0x200u : 0u)); /* inf, NaN */
  const uint32_t sig = exp ? (mant | 0x800000u) : mant;
  const int32_t E = (exp ? exp : 1) - 127;
  int32_t shift;
  uint32_t base;
  if (E >= -14) {
    shift = 13;
    base = (uint32_t)(E + 14) << 10;
  } else {
    shift = 13 + (-14 - E);
    base = 0;
  }
  uint32_t q = 0;
  if (shift < 25) { /* otherwise sig < 2^24 <= half a unit: rounds to 0 */
    q = sig >> shift;
    const uint32_t rem = sig & ((1u << shift) - 1u), half = 1u << (shift - 1);
#if ORACLE_PLANT == 12
    (void)rem; (void)half; /* planted: truncation instead of rounding */
#else
    if (rem > half || (rem == half && (q & 1u))) q += 1u;
#endif
  }
  uint32_t bits = base + q;
  if (bits >= 0x7c00u) bits = 0x7c00u;
  return (uint16_t)(sign | bits);
}

static float half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

static int8_t quant_one(float x, float d) {
  if (!(d > 0.0f)) return 0;
#if ORACLE_PLANT == 10
  float r = truncf(x / d); /* planted: rounding toward zero */
#else
  float r = roundf(x / d); /* round half away from zero */
#endif
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int8_t)r;
}

void oracle_quantize_q8_0(const float* x, int8_t* q, uint16_t* d_bits) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) {
    const float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  const uint16_t dh = oracle_float_to_half(amax / 127.0f);
  const float d = half_to_float(dh);
  for (int i = 0; i < 32; ++i) q[i] = quant_one(x[i], d);
  *d_bits = dh;
}

void oracle_quantize_row(const float* x, int32_t n, int8_t* q, float* s_out) {
  float amax = 0.0f;
  for (int32_t i = 0; i < n; ++i) {
    const float a = fabsf(x[i]);
    if (a > amax) amax = a;
  }
  const float s = amax / 127.0f;
  for (int32_t i = 0; i < n; ++i) q[i] = quant_one(x[i], s);
  *s_out = s;
}

int oracle_cache_write(const oracle_problem* p, const uint16_t* k_new, const uint16_t* v_new,
                       void* k_cache, void* v_cache) {
  if (!p || !k_new || !v_new || !k_cache || !v_cache || !p->block_table || !p->context_lens)
    return ORACLE_ERR_INVALID_ARG;
  if (p->num_kv_heads <= 0 || p->head_dim <= 0 || p->head_dim % 32 != 0 || p->block_size <= 0 ||
      p->n_query <= 0)
    return ORACLE_ERR_INVALID_ARG;
  const int64_t D = p->head_dim, bs = p->block_size, H = p->num_kv_heads;
  int first_err = ORACLE_OK;
  float* x = (float*)malloc(sizeof(float) * D);
  int8_t* q = (int8_t*)malloc((size_t)D);
  if (!x || !q) {
    free(x); free(q);
    return ORACLE_ERR_NOMEM;
  }
  for (int32_t s = 0; s < p->num_seqs; ++s) {
    const int64_t L = p->context_lens[s];
    if (L < p->n_query || L > (int64_t)p->max_blocks_per_seq * bs) {
      if (!first_err) first_err = ORACLE_ERR_BAD_CONTEXT_LEN;
      continue;
    }
    for (int32_t i = 0; i < p->n_query; ++i) {
#if ORACLE_PLANT == 11
      const int64_t pos = L - p->n_query + i - (i > 0); /* planted: positions off by one */
#else
      const int64_t pos = L - p->n_query + i;
#endif
      int64_t b;
      int32_t slot;
      if (resolve_key(p, s, pos, &b, &slot)) {
        if (!first_err) first_err = ORACLE_ERR_BAD_BLOCK_INDEX;
        continue;
      }
      for (int32_t h = 0; h < H; ++h) {
        for (int kv = 0; kv < 2; ++kv) {
          const uint16_t* src = (kv ? v_new : k_new) + (((int64_t)s * p->n_query + i) * H + h) * D;
          void* cache = kv ? v_cache : k_cache;
          if (p->kv_dtype == ORACLE_KV_FP16) {
            uint16_t* c = (uint16_t*)cache + ((b * H + h) * bs + slot) * D;
            memcpy(c, src, (size_t)D * 2);
            continue;
          }
          for (int64_t e = 0; e < D; ++e) x[e] = half_to_float(src[e]);
          if (p->kv_dtype == ORACLE_KV_Q8_0) {
            const int64_t tb = bs * D + bs * (D / 32) * 2;
            uint8_t* tile = (uint8_t*)cache + (b * H + h) * tb;
            for (int64_t g = 0; g < D / 32; ++g) {
              uint16_t dh;
              oracle_quantize_q8_0(x + 32 * g, q + 32 * g, &dh);
              memcpy(tile + bs * D + ((int64_t)slot * (D / 32) + g) * 2, &dh, 2);
            }
            memcpy(tile + (int64_t)slot * D, q, (size_t)D);
          } else {
            const int64_t tb = bs * D + bs * 4;
            uint8_t* tile = (uint8_t*)cache + (b * H + h) * tb;
            float sc;
            oracle_quantize_row(x, (int32_t)D, q, &sc);
            memcpy(tile + (int64_t)slot * D, q, (size_t)D);
            memcpy(tile + bs * D + (int64_t)slot * 4, &sc, 4);
          }
        }
      }
    }
  }
  free(x);
  free(q);
  return first_err;
}
