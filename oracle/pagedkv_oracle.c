/*
 * pagedkv_oracle.c -- plain fp64 CPU oracle for attention over a block-paged KV cache.
 *
 * TEST INFRASTRUCTURE. Only the test-suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. The CUDA library
 * never calls it, and the two share no code, header, table or helper: the only
 * thing both sides see is the same seeded input tensors.
 *
 * What it computes (and where the pages state it):
 *   - The KV cache is cut into fixed-size blocks ("pages"); a per-sequence
 *     mapping table turns a logical position into a physical block
 *     ("从零构建CUDA推理引擎：Tiny-Infer项目的技术深度解析", section
 *     "分页KV缓存：借鉴操作系统的内存管理").
 *   - Attention itself is exact softmax attention.  FlashAttention only changes
 *     how the work is tiled and where partial softmax state lives (running
 *     max / running sum in SRAM); the result is the plain definition
 *     (same Tiny-Infer page, section "Flash Attention：内存与计算的重平衡";
 *     "5 Fun Projects for LLM Inference Engineering", section 2).
 *   So the oracle gathers the keys of each sequence through its block table and
 *   applies naive two-pass softmax attention in fp64.  There is no tiling, no
 *   online softmax and no reordering beyond that definition.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - cache layout [num_blocks][num_kv_heads][block_size][head_dim] (bf16);
 *   - grouped-query mapping: query head h reads kv head h / (Hq / Hkv);
 *   - slot = physical_block * block_size + offset; a negative slot is skipped;
 *   - context_lens counts every valid key, including the tokens just written;
 *   - a query chunk is the LAST Q_b positions of its sequence (bottom-right causal):
 *     query i of Q_b sees keys 0 .. L_b - Q_b + i;
 *   - L_b = 0 gives an all-zero output row.
 *
 * bf16 inputs arrive as their 16-bit patterns and are widened exactly
 * (bf16 -> f32 by a 16-bit left shift, then f32 -> f64).
 *
 * Return codes: 0 = ok, 1 = invalid argument, 5 = out-of-range index
 * (a slot or block id outside the pool).  These follow the library's status
 * numbering only so the tests can print one vocabulary.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC pagedkv_oracle.c -lm
 * (no -ffast-math: fp64 semantics are the point).
 *
 * PKV_ORACLE_MUTANT: compile-time switch that plants one deliberate mistake.
 * Only the test that proves the pins can tell a wrong oracle from a right one
 * builds with it; the default build has none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef PKV_ORACLE_MUTANT
#define PKV_ORACLE_MUTANT 0
#endif

#define ORC_OK 0
#define ORC_INVALID 1
#define ORC_BOUNDS 5

static double bf16_bits_to_f64(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

int ref_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Threads the next parallel loops use (timing on one core or all). */
void ref_set_num_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n > 0 ? n : 1);
#else
  (void)n;
#endif
}

int ref_mutant_id(void) { return PKV_ORACLE_MUTANT; }

/* ------------------------------------------------------------------------- */
/* Cache write: scatter new K/V rows into their physical slots.               */
/* key/value: [T][Hkv][D], token stride given in elements, head stride = D.   */
/* k_cache/v_cache: [NB][Hkv][bs][D].                                         */
/* ------------------------------------------------------------------------- */
int ref_kv_cache_write(const uint16_t* key, const uint16_t* value,
                       int64_t key_stride_tok, int64_t value_stride_tok,
                       uint16_t* k_cache, uint16_t* v_cache,
                       const int64_t* slot_mapping, int32_t T, int32_t Hkv,
                       int32_t D, int32_t NB, int32_t bs) {
  if (T < 0 || Hkv <= 0 || D <= 0 || NB < 0 || bs <= 0) return ORC_INVALID;
  int status = ORC_OK;
  const int64_t pool_slots = (int64_t)NB * bs;
  for (int32_t t = 0; t < T; ++t) {
    int64_t slot = slot_mapping[t];
#if PKV_ORACLE_MUTANT == 8
    slot += 1; /* planted: off-by-one slot */
#endif
    if (slot < 0) continue; /* padding token: nothing to write */
    if (slot >= pool_slots) {
      status = ORC_BOUNDS;
      continue;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    for (int32_t h = 0; h < Hkv; ++h) {
      const int64_t dst = ((blk * Hkv + h) * bs + off) * (int64_t)D;
      memcpy(k_cache + dst, key + t * key_stride_tok + (int64_t)h * D,
             (size_t)D * sizeof(uint16_t));
      memcpy(v_cache + dst, value + t * value_stride_tok + (int64_t)h * D,
             (size_t)D * sizeof(uint16_t));
    }
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* Softmax attention of one query row over n keys, given as row pointers.     */
/* Two passes: scores and their max, then exp / sum / weighted V.             */
/* Returns the natural-log normaliser lse = max + log(sum) (or -inf if n=0).  */
/* s is caller scratch of n doubles.                                          */
/* ------------------------------------------------------------------------- */
static double attend_row(double* out, const double* q, int32_t D, double scale,
                         const uint16_t* const* krows,
                         const uint16_t* const* vrows, int64_t n, double* s) {
  for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
  if (n <= 0) return -INFINITY;
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double dot = 0.0;
#if PKV_ORACLE_MUTANT == 9
    const uint16_t* kr = vrows[j]; /* planted: scores against V instead of K */
#else
    const uint16_t* kr = krows[j];
#endif
    for (int32_t d = 0; d < D; ++d) dot += q[d] * bf16_bits_to_f64(kr[d]);
#if PKV_ORACLE_MUTANT == 3
    s[j] = dot; /* planted: scale dropped */
#elif PKV_ORACLE_MUTANT == 18
    s[j] = fabs(scale) * dot; /* planted: sign of the scale dropped */
#else
    s[j] = scale * dot;
#endif
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    s[j] = exp(s[j] - m);
    l += s[j];
  }
  for (int64_t j = 0; j < n; ++j) {
    const uint16_t* vr = vrows[j];
    for (int32_t d = 0; d < D; ++d) out[d] += s[j] * bf16_bits_to_f64(vr[d]);
  }
#if PKV_ORACLE_MUTANT != 6 /* planted (6): normalisation by l dropped */
  for (int32_t d = 0; d < D; ++d) out[d] /= l;
#endif
  return m + log(l);
}

/* kv head read by query head h under grouped-query attention */
static int32_t kv_head_of(int32_t h, int32_t Hq, int32_t Hkv) {
#if PKV_ORACLE_MUTANT == 1
  (void)Hq;
  return h % Hkv; /* planted: interleaved instead of consecutive groups */
#else
  return h / (Hq / Hkv);
#endif
}

/* Pointer to K (or V) row of logical key j of sequence b, kv head g.
 * Returns NULL if the block-table entry is outside the pool. */
static const uint16_t* paged_row(const uint16_t* cache,
                                 const int32_t* block_tables, int32_t MB,
                                 int32_t b, int64_t j, int32_t g, int32_t Hkv,
                                 int32_t D, int32_t NB, int32_t bs) {
#if PKV_ORACLE_MUTANT == 2
  const int64_t page = j % bs, row = j / bs; /* planted: page/row swapped */
#else
  const int64_t page = j / bs, row = j % bs;
#endif
  const int32_t blk = block_tables[(int64_t)b * MB + page];
  if (blk < 0 || blk >= NB) return NULL;
#if PKV_ORACLE_MUTANT == 7
  /* planted: token-major page layout [NB][bs][Hkv][D] */
  return cache + (((int64_t)blk * bs + row) * Hkv + g) * (int64_t)D;
#else
  return cache + (((int64_t)blk * Hkv + g) * bs + row) * (int64_t)D;
#endif
}

/* widen a bf16 query row to fp64 */
static void widen_row(double* dst, const uint16_t* src, int32_t D) {
  for (int32_t d = 0; d < D; ++d) dst[d] = bf16_bits_to_f64(src[d]);
}

/* ------------------------------------------------------------------------- */
/* Decode: one query token per sequence.                                      */
/* out [B][Hq][D] fp64; q [B][Hq][D] bf16 bits; block_tables [B][MB] int32;   */
/* context_lens [B] int32.                                                    */
/* ------------------------------------------------------------------------- */
int ref_paged_attention(double* out, const uint16_t* q, const uint16_t* k_cache,
                        const uint16_t* v_cache, const int32_t* block_tables,
                        int32_t MB, const int32_t* context_lens, int32_t B,
                        int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                        int32_t bs, float scale) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || MB < 0 ||
      Hq % Hkv != 0)
    return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b)
    if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs)
      return ORC_INVALID;
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int32_t b = (int32_t)(bh / Hq), h = (int32_t)(bh % Hq);
    int64_t n = context_lens[b];
#if PKV_ORACLE_MUTANT == 5
    if (n > 0) n -= 1; /* planted: newest key dropped */
#endif
    const int32_t g = kv_head_of(h, Hq, Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      kr[j] = paged_row(k_cache, block_tables, MB, b, j, g, Hkv, D, NB, bs);
      vr[j] = paged_row(v_cache, block_tables, MB, b, j, g, Hkv, D, NB, bs);
      if (!kr[j] || !vr[j]) bad = 1;
    }
    double* o = out + bh * D;
    if (bad) {
      for (int32_t d = 0; d < D; ++d) o[d] = NAN;
#pragma omp atomic write
      status = ORC_BOUNDS;
    } else {
      widen_row(qd, q + bh * D, D);
      attend_row(o, qd, D, (double)scale, kr, vr, n, s);
    }
    free(kr); free(vr); free(s); free(qd);
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* Static (contiguous) cache form used as the layout-equivalence check.       */
/* k, v: [B][Lmax][Hkv][D]; q [B][Hq][D]; out [B][Hq][D].                     */
/* Same row routine, so paged == contiguous must hold bit for bit.            */
/* ------------------------------------------------------------------------- */
int ref_contiguous_attention(double* out, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, const int32_t* context_lens,
                             int32_t B, int32_t Lmax, int32_t Hq, int32_t Hkv,
                             int32_t D, float scale) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax < 0 || Hq % Hkv != 0)
    return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b)
    if (context_lens[b] < 0 || context_lens[b] > Lmax) return ORC_INVALID;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int32_t b = (int32_t)(bh / Hq), h = (int32_t)(bh % Hq);
    const int64_t n = context_lens[b];
    const int32_t g = h / (Hq / Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    for (int64_t j = 0; j < n; ++j) {
      const int64_t off = (((int64_t)b * Lmax + j) * Hkv + g) * (int64_t)D;
      kr[j] = k + off;
      vr[j] = v + off;
    }
    widen_row(qd, q + bh * D, D);
    attend_row(out + bh * D, qd, D, (double)scale, kr, vr, n, s);
    free(kr); free(vr); free(s); free(qd);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Chunked causal prefill over the paged cache.                               */
/* q [sumQ][Hq][D]; query_start_loc [B+1] (cu_seqlens of the chunk);          */
/* context_lens [B] INCLUDE the chunk, whose K/V are already in the cache.    */
/* Query i of sequence b sits at absolute position L_b - Q_b + i and sees     */
/* keys 0 .. that position.                                                   */
/* ------------------------------------------------------------------------- */
int ref_paged_attention_prefill(double* out, const uint16_t* q,
                                const int32_t* query_start_loc,
                                const uint16_t* k_cache, const uint16_t* v_cache,
                                const int32_t* block_tables, int32_t MB,
                                const int32_t* context_lens, int32_t B,
                                int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                int32_t bs, float scale) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || MB < 0 ||
      Hq % Hkv != 0)
    return ORC_INVALID;
  if (query_start_loc[0] != 0) return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b) {
    const int32_t Qb = query_start_loc[b + 1] - query_start_loc[b];
    if (Qb < 0 || context_lens[b] < Qb ||
        (int64_t)context_lens[b] > (int64_t)MB * bs)
      return ORC_INVALID;
  }
  const int64_t sumQ = query_start_loc[B];
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t th = 0; th < sumQ * Hq; ++th) {
    const int64_t t = th / Hq;
    const int32_t h = (int32_t)(th % Hq);
    int32_t b = 0;
    while (query_start_loc[b + 1] <= t) ++b;
    const int64_t i = t - query_start_loc[b];
    const int64_t Qb = query_start_loc[b + 1] - query_start_loc[b];
    const int64_t L = context_lens[b];
#if PKV_ORACLE_MUTANT == 4
    const int64_t n = L - Qb + i; /* planted: query cannot see itself */
#else
    const int64_t n = L - Qb + i + 1;
#endif
    const int32_t g = kv_head_of(h, Hq, Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      kr[j] = paged_row(k_cache, block_tables, MB, b, j, g, Hkv, D, NB, bs);
      vr[j] = paged_row(v_cache, block_tables, MB, b, j, g, Hkv, D, NB, bs);
      if (!kr[j] || !vr[j]) bad = 1;
    }
    double* o = out + th * D;
    if (bad) {
      for (int32_t d = 0; d < D; ++d) o[d] = NAN;
#pragma omp atomic write
      status = ORC_BOUNDS;
    } else {
      widen_row(qd, q + th * D, D);
      attend_row(o, qd, D, (double)scale, kr, vr, n, s);
    }
    free(kr); free(vr); free(s); free(qd);
  }
  return status;
}

/* ------------------------------------------------------------------------- */
/* Split-KV partials (flash-decoding form, for checking the merge algebra and */
/* a GPU kernel's intermediate results).  Split c covers logical keys         */
/* [c*S, min((c+1)*S, L_b)).  Each split's o_c is its own normalised          */
/* attention output and lse_c = max_c + log(sum_c) in natural log; an empty   */
/* split has o_c = 0 and lse_c = -inf.                                        */
/* o_part [B][Hq][C][D], lse [B][Hq][C].                                      */
/* ------------------------------------------------------------------------- */
int ref_decode_partials(double* o_part, double* lse, const uint16_t* q,
                        const uint16_t* k_cache, const uint16_t* v_cache,
                        const int32_t* block_tables, int32_t MB,
                        const int32_t* context_lens, int32_t B, int32_t Hq,
                        int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                        float scale, int32_t split_tokens, int32_t C) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || split_tokens <= 0 ||
      C <= 0 || Hq % Hkv != 0)
    return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b)
    if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs ||
        (int64_t)context_lens[b] > (int64_t)C * split_tokens)
      return ORC_INVALID;
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bhc = 0; bhc < (int64_t)B * Hq * C; ++bhc) {
    const int32_t c = (int32_t)(bhc % C);
    const int64_t bh = bhc / C;
    const int32_t b = (int32_t)(bh / Hq), h = (int32_t)(bh % Hq);
    const int64_t L = context_lens[b];
    const int64_t j0 = (int64_t)c * split_tokens;
    int64_t j1 = j0 + split_tokens;
    if (j1 > L) j1 = L;
    const int64_t n = j1 > j0 ? j1 - j0 : 0;
    const int32_t g = h / (Hq / Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      kr[j] = paged_row(k_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      vr[j] = paged_row(v_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      if (!kr[j] || !vr[j]) bad = 1;
    }
    if (bad) {
#pragma omp atomic write
      status = ORC_BOUNDS;
      lse[bhc] = NAN;
    } else {
      widen_row(qd, q + bh * D, D);
      lse[bhc] = attend_row(o_part + bhc * D, qd, D, (double)scale, kr, vr, n, s);
    }
    free(kr); free(vr); free(s); free(qd);
  }
  return status;
}

/* Log-sum-exp merge of split partials: M = max_c lse_c,
 * out = sum_c e^{lse_c - M} o_c / sum_c e^{lse_c - M}; all-empty gives 0. */
int ref_lse_merge(double* out, const double* o_part, const double* lse,
                  int64_t rows, int32_t C, int32_t D) {
  if (rows < 0 || C <= 0 || D <= 0) return ORC_INVALID;
  for (int64_t r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int32_t c = 0; c < C; ++c)
      if (lse[r * C + c] > M) M = lse[r * C + c];
    double* o = out + r * D;
    for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
    if (M == -INFINITY) continue;
    double wsum = 0.0;
    for (int32_t c = 0; c < C; ++c) {
      const double lc = lse[r * C + c];
      if (lc == -INFINITY) continue;
#if PKV_ORACLE_MUTANT == 10
      const double w = exp(M - lc); /* planted: weight exponent sign flipped */
#else
      const double w = exp(lc - M);
#endif
      wsum += w;
      for (int32_t d = 0; d < D; ++d) o[d] += w * o_part[(r * C + c) * D + d];
    }
    for (int32_t d = 0; d < D; ++d) o[d] /= wsum;
  }
  return ORC_OK;
}

/* ========================================================================= */
/* INT8 KV cache with one fp32 scale per (token, kv head).                    */
/*                                                                            */
/* The pages name an INT8 KV cache as the way to halve its memory            */
/* (Tiny-Infer page, section "推测性解码与INT8量化"); they fix neither the     */
/* scale granularity nor the rounding.  Reading taken here: symmetric, one    */
/* scale per written row (a token's D values of one kv head), the only        */
/* granularity an incremental cache write can fix when the row is written;    */
/*   amax = max_d |x_d|;  scale = amax / 127;  inv = 127 / amax;              */
/*   code_d = clamp(round_half_even(x_d * inv), -127, 127);                   */
/* all in fp32 (x is bf16 widened exactly), so the codes are one exact        */
/* function of the row; amax = 0 gives codes 0 and scale 0.  The row's value  */
/* is code_d * scale, exact in fp64, and attention is the plain definition    */
/* over those values.                                                         */
/* Pools: k_cache/v_cache int8 [NB][Hkv][bs][D]; k_scale/v_scale fp32         */
/* [NB][Hkv][bs].                                                             */
/* ========================================================================= */

static float bf16_bits_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* quantise one row of D bf16 values */
static void quantize_row_int8(int8_t* codes, float* scale_out, const uint16_t* x, int32_t D) {
  float amax = 0.0f;
  for (int32_t d = 0; d < D; ++d) {
    const float a = fabsf(bf16_bits_to_f32(x[d]));
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) {
    for (int32_t d = 0; d < D; ++d) codes[d] = 0;
    *scale_out = 0.0f;
    return;
  }
#if PKV_ORACLE_MUTANT == 11
  const float inv = 128.0f / amax; /* planted: wrong code range */
#else
  const float inv = 127.0f / amax;
#endif
  for (int32_t d = 0; d < D; ++d) {
    const float y = bf16_bits_to_f32(x[d]) * inv;
#if PKV_ORACLE_MUTANT == 12
    float r = truncf(y); /* planted: rounds toward zero */
#else
    float r = rintf(y); /* round half to even (default rounding mode) */
#endif
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    codes[d] = (int8_t)r;
  }
  *scale_out = amax / 127.0f;
}

/* Quantise new K/V rows into their slots (see ref_kv_cache_write for the
 * scatter itself).  key/value [T][Hkv][D] bf16 bits, token stride in
 * elements. */
int ref_kv_cache_write_int8(const uint16_t* key, const uint16_t* value,
                            int64_t key_stride_tok, int64_t value_stride_tok,
                            int8_t* k_cache, int8_t* v_cache, float* k_scale,
                            float* v_scale, const int64_t* slot_mapping,
                            int32_t T, int32_t Hkv, int32_t D, int32_t NB,
                            int32_t bs) {
  if (T < 0 || Hkv <= 0 || D <= 0 || NB < 0 || bs <= 0) return ORC_INVALID;
  const int64_t pool_slots = (int64_t)NB * bs;
  int status = ORC_OK;
  for (int64_t t = 0; t < T; ++t) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= pool_slots) {
      status = ORC_BOUNDS;
      continue;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    for (int32_t h = 0; h < Hkv; ++h) {
      const int64_t row = (blk * Hkv + h) * bs + off;
      quantize_row_int8(k_cache + row * D, k_scale + row, key + t * key_stride_tok + (int64_t)h * D, D);
      quantize_row_int8(v_cache + row * D, v_scale + row, value + t * value_stride_tok + (int64_t)h * D, D);
    }
  }
  return status;
}

/* Attention of one query row over n int8 rows with their scales; same two
 * passes as attend_row. */
static void attend_row_int8(double* out, const double* q, int32_t D, double scale,
                            const int8_t* const* krows, const float* ks,
                            const int8_t* const* vrows, const float* vs, int64_t n,
                            double* s) {
  for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
  if (n <= 0) return;
  double m = -INFINITY;
  for (int64_t j = 0; j < n; ++j) {
    double dot = 0.0;
    for (int32_t d = 0; d < D; ++d) dot += q[d] * ((double)krows[j][d] * (double)ks[j]);
    s[j] = scale * dot;
    if (s[j] > m) m = s[j];
  }
  double l = 0.0;
  for (int64_t j = 0; j < n; ++j) {
    s[j] = exp(s[j] - m);
    l += s[j];
  }
  for (int64_t j = 0; j < n; ++j) {
#if PKV_ORACLE_MUTANT == 13
    const double vscale = (double)ks[j]; /* planted: V rows scaled by the K scale */
#else
    const double vscale = (double)vs[j];
#endif
    for (int32_t d = 0; d < D; ++d) out[d] += s[j] * ((double)vrows[j][d] * vscale);
  }
  for (int32_t d = 0; d < D; ++d) out[d] /= l;
}

static int64_t window_start(int64_t p, int32_t W);

/* Decode over the int8 pool; same gather and grouped-query mapping as
 * ref_paged_attention.  window > 0: only the keys of the query's sliding
 * window (see the sliding-window section below) are gathered. */
static int paged_attention_int8(double* out, const uint16_t* q, const int8_t* k_cache,
                                const int8_t* v_cache, const float* k_scale,
                                const float* v_scale, const int32_t* block_tables,
                                int32_t MB, const int32_t* context_lens, int32_t B,
                                int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                int32_t bs, float scale, int32_t window) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || MB < 0 ||
      Hq % Hkv != 0 || window < 0)
    return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b)
    if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs)
      return ORC_INVALID;
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int32_t b = (int32_t)(bh / Hq), h = (int32_t)(bh % Hq);
    const int64_t L = context_lens[b];
    const int64_t j0 = (window > 0 && L > 0) ? window_start(L - 1, window) : 0;
    const int64_t n = L - j0;
    const int32_t g = kv_head_of(h, Hq, Hkv);
    const int8_t** kr = (const int8_t**)malloc(sizeof(void*) * (n + 1));
    const int8_t** vr = (const int8_t**)malloc(sizeof(void*) * (n + 1));
    float* ks = (float*)malloc(sizeof(float) * (n + 1));
    float* vs = (float*)malloc(sizeof(float) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      const int64_t page = (j0 + j) / bs, row = (j0 + j) % bs;
      const int32_t blk = block_tables[(int64_t)b * MB + page];
      if (blk < 0 || blk >= NB) {
        bad = 1;
        break;
      }
      const int64_t r = ((int64_t)blk * Hkv + g) * bs + row;
      kr[j] = k_cache + r * D;
      vr[j] = v_cache + r * D;
      ks[j] = k_scale[r];
      vs[j] = v_scale[r];
    }
    double* o = out + bh * D;
    if (bad) {
      for (int32_t d = 0; d < D; ++d) o[d] = NAN;
#pragma omp atomic write
      status = ORC_BOUNDS;
    } else {
      widen_row(qd, q + bh * D, D);
      attend_row_int8(o, qd, D, (double)scale, kr, ks, vr, vs, n, s);
    }
    free(kr); free(vr); free(ks); free(vs); free(s); free(qd);
  }
  return status;
}

int ref_paged_attention_int8(double* out, const uint16_t* q, const int8_t* k_cache,
                             const int8_t* v_cache, const float* k_scale,
                             const float* v_scale, const int32_t* block_tables,
                             int32_t MB, const int32_t* context_lens, int32_t B,
                             int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                             int32_t bs, float scale) {
  return paged_attention_int8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, MB,
                              context_lens, B, Hq, Hkv, D, NB, bs, scale, 0);
}

/* Sliding-window decode over the int8 pool (window >= 1). */
int ref_paged_attention_int8_window(double* out, const uint16_t* q, const int8_t* k_cache,
                                    const int8_t* v_cache, const float* k_scale,
                                    const float* v_scale, const int32_t* block_tables,
                                    int32_t MB, const int32_t* context_lens, int32_t B,
                                    int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                    int32_t bs, float scale, int32_t window) {
  if (window < 1) return ORC_INVALID;
  return paged_attention_int8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, MB,
                              context_lens, B, Hq, Hkv, D, NB, bs, scale, window);
}

/* ========================================================================= */
/* Sliding-window attention over the paged cache.                             */
/*                                                                            */
/* A sliding-window cache is one of the KV cache variants the inference-lab  */
/* page lists, an approximation for tight memory ("从零开始的LLM推理优化实验  */
/* 室：从PyTorch基线到Triton内核的完整实践", section "KV缓存实验与长上下文   */
/* 优化").  It gives no semantics; reading taken: a query at absolute         */
/* position p sees the W keys p - W < j <= p (all of them if fewer exist).    */
/* The result is plain attention over that key range, so the oracle gathers  */
/* exactly those keys.                                                        */
/* ========================================================================= */

/* first key a query at absolute position p sees under window W (W >= 1) */
static int64_t window_start(int64_t p, int32_t W) {
#if PKV_ORACLE_MUTANT == 14
  const int64_t j0 = p - W; /* planted: one key too many */
#else
  const int64_t j0 = p - W + 1;
#endif
  return j0 > 0 ? j0 : 0;
}

/* Decode: the query sits at position L_b - 1; out [B][Hq][D]. */
int ref_paged_attention_window(double* out, const uint16_t* q, const uint16_t* k_cache,
                               const uint16_t* v_cache, const int32_t* block_tables,
                               int32_t MB, const int32_t* context_lens, int32_t B,
                               int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                               int32_t bs, float scale, int32_t window) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || MB < 0 ||
      Hq % Hkv != 0 || window < 1)
    return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b)
    if (context_lens[b] < 0 || (int64_t)context_lens[b] > (int64_t)MB * bs)
      return ORC_INVALID;
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < (int64_t)B * Hq; ++bh) {
    const int32_t b = (int32_t)(bh / Hq), h = (int32_t)(bh % Hq);
    const int64_t L = context_lens[b];
    const int64_t j0 = L > 0 ? window_start(L - 1, window) : 0;
    const int64_t n = L - j0;
    const int32_t g = kv_head_of(h, Hq, Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      kr[j] = paged_row(k_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      vr[j] = paged_row(v_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      if (!kr[j] || !vr[j]) bad = 1;
    }
    double* o = out + bh * D;
    if (bad) {
      for (int32_t d = 0; d < D; ++d) o[d] = NAN;
#pragma omp atomic write
      status = ORC_BOUNDS;
    } else {
      widen_row(qd, q + bh * D, D);
      attend_row(o, qd, D, (double)scale, kr, vr, n, s);
    }
    free(kr); free(vr); free(s); free(qd);
  }
  return status;
}

/* Chunked prefill: query i of sequence b sits at p = L_b - Q_b + i and sees
 * keys window_start(p, W) .. p. */
int ref_paged_attention_prefill_window(double* out, const uint16_t* q,
                                       const int32_t* query_start_loc,
                                       const uint16_t* k_cache, const uint16_t* v_cache,
                                       const int32_t* block_tables, int32_t MB,
                                       const int32_t* context_lens, int32_t B,
                                       int32_t Hq, int32_t Hkv, int32_t D, int32_t NB,
                                       int32_t bs, float scale, int32_t window) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || MB < 0 ||
      Hq % Hkv != 0 || window < 1)
    return ORC_INVALID;
  if (query_start_loc[0] != 0) return ORC_INVALID;
  for (int32_t b = 0; b < B; ++b) {
    const int32_t Qb = query_start_loc[b + 1] - query_start_loc[b];
    if (Qb < 0 || context_lens[b] < Qb ||
        (int64_t)context_lens[b] > (int64_t)MB * bs)
      return ORC_INVALID;
  }
  const int64_t sumQ = query_start_loc[B];
  int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t th = 0; th < sumQ * Hq; ++th) {
    const int64_t t = th / Hq;
    const int32_t h = (int32_t)(th % Hq);
    int32_t b = 0;
    while (query_start_loc[b + 1] <= t) ++b;
    const int64_t i = t - query_start_loc[b];
    const int64_t Qb = query_start_loc[b + 1] - query_start_loc[b];
    const int64_t p = context_lens[b] - Qb + i;
    const int64_t j0 = window_start(p, window);
    const int64_t n = p + 1 - j0;
    const int32_t g = kv_head_of(h, Hq, Hkv);
    const uint16_t** kr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    const uint16_t** vr = (const uint16_t**)malloc(sizeof(void*) * (n + 1));
    double* s = (double*)malloc(sizeof(double) * (n + 1));
    double* qd = (double*)malloc(sizeof(double) * D);
    int bad = 0;
    for (int64_t j = 0; j < n; ++j) {
      kr[j] = paged_row(k_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      vr[j] = paged_row(v_cache, block_tables, MB, b, j0 + j, g, Hkv, D, NB, bs);
      if (!kr[j] || !vr[j]) bad = 1;
    }
    double* o = out + th * D;
    if (bad) {
      for (int32_t d = 0; d < D; ++d) o[d] = NAN;
#pragma omp atomic write
      status = ORC_BOUNDS;
    } else {
      widen_row(qd, q + th * D, D);
      attend_row(o, qd, D, (double)scale, kr, vr, n, s);
    }
    free(kr); free(vr); free(s); free(qd);
  }
  return status;
}

/* ========================================================================= */
/* Rotary position embedding applied to K as it is written into the cache.    */
/*                                                                            */
/* The fused-ops page fuses RoPE with the step before it so the rotated rows  */
/* make one trip through memory ("Triton融合算子优化：LLM推理性能提升3倍的工  */
/* 程实践", section 3.1); the Tiny-Infer page lists RoPE among Llama's       */
/* operators.  Neither prints the formula.  Reading taken: Llama's form as   */
/* the HuggingFace implementation the Tiny-Infer page checks against uses    */
/* it: element i < D/2 pairs with i + D/2, angle pos * base^(-2i/D),          */
/*   y[i]       = x[i] cos - x[i + D/2] sin                                  */
/*   y[i + D/2] = x[i + D/2] cos + x[i] sin                                  */
/* in fp64 here (exact cos/sin of the exact angle up to fp64 rounding).      */
/* ========================================================================= */

static void rope_row(double* y, const uint16_t* x, int64_t pos, int32_t D, double base) {
  const int32_t half = D / 2;
  for (int32_t i = 0; i < half; ++i) {
#if PKV_ORACLE_MUTANT == 17
    const double inv_freq = pow(base, -(double)i / (double)D); /* planted: exponent halved */
#else
    const double inv_freq = pow(base, -2.0 * (double)i / (double)D);
#endif
    const double a = (double)pos * inv_freq;
    const double c = cos(a);
#if PKV_ORACLE_MUTANT == 16
    const double s = -sin(a); /* planted: rotation the other way */
#else
    const double s = sin(a);
#endif
#if PKV_ORACLE_MUTANT == 15
    const int32_t i1 = 2 * i, i2 = 2 * i + 1; /* planted: adjacent pairs */
#else
    const int32_t i1 = i, i2 = i + half;
#endif
    const double x1 = bf16_bits_to_f64(x[i1]), x2 = bf16_bits_to_f64(x[i2]);
    y[i1] = x1 * c - x2 * s;
    y[i2] = x2 * c + x1 * s;
  }
}

/* Rotated rows in fp64: x [T][H][D] bf16 bits (token stride in elements),
 * positions [T]; out [T][H][D].  D even. */
int ref_rope_rows(double* out, const uint16_t* x, int64_t x_stride_tok, const int64_t* positions,
                  int64_t T, int32_t H, int32_t D, double base) {
  if (T < 0 || H <= 0 || D <= 0 || D % 2 != 0 || !(base > 0.0)) return ORC_INVALID;
  for (int64_t t = 0; t < T; ++t)
    for (int32_t h = 0; h < H; ++h)
      rope_row(out + (t * H + h) * D, x + t * x_stride_tok + (int64_t)h * D, positions[t], D, base);
  return ORC_OK;
}

/* fp64 -> bf16 bits, round to nearest even on the value itself (no double
 * rounding through fp32): 8 significant bits for normal values. */
static uint16_t f64_to_bf16_bits(double v) {
  float f;
  if (v == 0.0 || !isfinite(v)) {
    f = (float)v;
  } else {
    int e;
    const double m = frexp(v, &e);              /* v = m * 2^e, 0.5 <= |m| < 1 */
    const double r = nearbyint(ldexp(m, 8));    /* 8 significant bits, ties to even */
    f = (float)ldexp(r, e - 8);                 /* exact in fp32 */
  }
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* Cache write with K rotated at its position: K rows become bf16(rope(K)),
 * V rows are copied; slots < 0 are skipped. */
int ref_kv_cache_write_rope(const uint16_t* key, const uint16_t* value,
                            int64_t key_stride_tok, int64_t value_stride_tok,
                            uint16_t* k_cache, uint16_t* v_cache,
                            const int64_t* slot_mapping, const int64_t* positions,
                            int32_t T, int32_t Hkv, int32_t D, int32_t NB, int32_t bs,
                            double base) {
  if (T < 0 || Hkv <= 0 || D <= 0 || D % 2 != 0 || NB < 0 || bs <= 0 || !(base > 0.0))
    return ORC_INVALID;
  const int64_t pool_slots = (int64_t)NB * bs;
  int status = ORC_OK;
  double* y = (double*)malloc(sizeof(double) * D);
  for (int64_t t = 0; t < T; ++t) {
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= pool_slots) {
      status = ORC_BOUNDS;
      continue;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    for (int32_t h = 0; h < Hkv; ++h) {
      const int64_t dst = ((blk * Hkv + h) * bs + off) * (int64_t)D;
      rope_row(y, key + t * key_stride_tok + (int64_t)h * D, positions[t], D, base);
      for (int32_t d = 0; d < D; ++d) k_cache[dst + d] = f64_to_bf16_bits(y[d]);
      memcpy(v_cache + dst, value + t * value_stride_tok + (int64_t)h * D, (size_t)D * sizeof(uint16_t));
    }
  }
  free(y);
  return status;
}
