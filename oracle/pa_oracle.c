/*
 * Paged KV-cache decode attention: the CPU oracle (plain C, fp64).
 *
 * TEST INFRASTRUCTURE ONLY.  The product (the CUDA library and its Python binding) never
 * links, imports or calls this file.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA path: it is written from the definition of the operations, slowly and plainly, so that
 * a reader can check it against the sources by eye.
 *
 * Sources (web tutorials on vLLM, cited by page and section):
 *   [P1] "vLLM architecture and core features: PagedAttention principle, continuous batching,
 *        quantization support", section 3.1 (KV cache cut into fixed-size pages allocated on
 *        demand; requests with a common prefix share pages).
 *   [P2] "vLLM core features: PagedAttention, Continuous Batching, quantization support,
 *        distributed inference", section 4.1 (the block table maps each logical block to a
 *        physical block; generating a token appends one mapping; sequences may share physical
 *        blocks, e.g. in parallel sampling).
 *   [P3] "Core inference engine (part 1): vLLM architecture, PagedAttention principle,
 *        Continuous Batching mechanism", section 2.2 (pages of a fixed size such as 16 tokens;
 *        pages need not be contiguous; shared prompt pages).
 *   [P4] "vLLM core architecture: model loading, PagedAttention principle, KV cache
 *        management", section 2.2.1 table (logical block of a fixed number of tokens, physical
 *        block of the same size, block table) and section 2.2.2 (attention has to assemble the
 *        complete KV sequence from the block table; the per-block loop shown there only states
 *        the principle).
 *
 * Readings where the sources are silent (each is also listed with the design notes):
 *   - Cache layout: key_cache and value_cache are each [num_blocks][num_kv_heads][block_size]
 *     [head_dim], row-major.  The sources fix only that the cache is indexed by physical block
 *     first ([P4] 2.2.2 reads "physical_kv_cache[physical_block_id]").
 *   - The per-block loop of [P4] 2.2.2 adds per-block attention outputs; read literally that is
 *     not attention over the context.  The oracle computes the full-context softmax that
 *     [P4] 2.2.2 says the loop stands for: out = softmax(scale * q K^T) V over positions
 *     0 .. context_len-1 of the assembled sequence.
 *   - Grouped query heads: query head h reads kv head h / (num_heads / num_kv_heads).
 *   - A context length of 0 gives an all-zero output row.
 *   - A negative slot in slot_mapping means "store nothing" (a padding token).
 *
 * Element types: 0 = fp32, 1 = bf16 (upper half of an fp32), 2 = IEEE binary16, 3 = FP8 E4M3
 * (cache only).  Elements are widened exactly to double before any arithmetic; all arithmetic
 * is in double, except the quantisation to FP8, which divides in fp32 (the precision the write
 * kernel decides the code in).
 *
 * FP8 KV cache ([P2] 4.3 lists FP8 E4M3, 8-bit floating point, ~50 % memory, as a supported
 * storage format; applying it to the KV cache with one fp32 scale per kv head is a reading of
 * that passage, which states no scaling): the cache holds code(x / scale[h]) and the attention
 * reads decode(code) * scale[h].
 * E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 is subnormal
 * (m * 2^-9); S.1111.111 is NaN; no infinities; the largest finite magnitude is 448.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { PAO_F32 = 0, PAO_BF16 = 1, PAO_F16 = 2, PAO_FP8 = 3 };

enum {
  PAO_OK = 0,
  PAO_BAD_BLOCK_ID = -1,    /* a block-table entry needed for the context is outside the pool */
  PAO_BAD_CONTEXT_LEN = -2, /* context_len larger than the block table can describe */
  PAO_BAD_ARG = -3,
  PAO_NO_MEMORY = -4
};

static size_t elt_size(int dtype) { return dtype == PAO_F32 ? 4u : (dtype == PAO_FP8 ? 1u : 2u); }

/* Value of one FP8 E4M3 code. */
static double fp8_to_double(uint8_t c) {
  const int sign = c >> 7, e = (c >> 3) & 0xf, m = c & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
  else
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return sign ? -v : v;
}

/* The E4M3 code nearest to x, ties to the even code, magnitudes of 448 and above saturated to
 * 448, NaN to the NaN code 0x7f. */
static uint8_t double_to_fp8(double x) {
  if (isnan(x)) return 0x7f;
  const uint8_t sign = signbit(x) ? 0x80 : 0;
  const double a = fabs(x);
  if (a >= 448.0) return sign | 0x7e;
  int code;
  if (a < ldexp(1.0, -6)) {
    code = (int)rint(a * 512.0); /* subnormal lattice m * 2^-9; 8 is the smallest normal */
  } else {
    int ex;
    frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1): exponent of the leading bit ex - 1 */
    const int e = ex - 1;
    int m = (int)rint((ldexp(a, -e) - 1.0) * 8.0);
    int be = e + 7;
    if (m == 8) {
      m = 0;
      ++be;
    }
    code = (be << 3) | m; /* at most 0x7e: a < 448 */
  }
  return sign | (uint8_t)code;
}

/* Widen element idx of a buffer of the given element type to double (exact for all three). */
static double elt_to_double(const void *base, size_t idx, int dtype) {
  if (dtype == PAO_F32) {
    float f;
    memcpy(&f, (const char *)base + idx * 4u, 4u);
    return (double)f;
  }
  if (dtype == PAO_FP8) return fp8_to_double(((const uint8_t *)base)[idx]);
  uint16_t h;
  memcpy(&h, (const char *)base + idx * 2u, 2u);
  if (dtype == PAO_BF16) {
    /* bf16 is the upper 16 bits of an IEEE binary32. */
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4u);
    return (double)f;
  }
  /* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
  int sign = (h >> 15) & 1, e = (h >> 10) & 0x1f, m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m | 0x400), e - 25); /* 1.m * 2^(e-15) */
  return sign ? -v : v;
}

/*
 * Write side: store each new token's key and value rows into the slot the scheduler gave it.
 * [P2] 4.1: generating a token appends one logical->physical mapping; the token's K/V then
 * lives at offset slot % block_size of physical block slot / block_size.
 *
 * key, value: [num_tokens][num_kv_heads][head_dim].  Caches as in the file header.
 * Returns the number of tokens skipped because their slot lies outside the pool (0 = all good).
 */
int pao_reshape_and_cache(const void *key, const void *value, void *key_cache, void *value_cache,
                          const int64_t *slot_mapping, int64_t num_tokens, int64_t num_blocks,
                          int num_kv_heads, int block_size, int head_dim, int dtype) {
  if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
    return PAO_BAD_ARG;
  const size_t row = (size_t)head_dim * elt_size(dtype);
  const int64_t num_slots = num_blocks * (int64_t)block_size;
  int skipped = 0;
  for (int64_t i = 0; i < num_tokens; ++i) {
    const int64_t slot = slot_mapping[i];
    if (slot < 0) continue; /* padding token */
    if (slot >= num_slots) {
      ++skipped;
      continue;
    }
    const int64_t block = slot / block_size;
    const int64_t offset = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      const size_t src = ((size_t)i * (size_t)num_kv_heads + (size_t)h) * row;
      const size_t dst =
          (((size_t)block * (size_t)num_kv_heads + (size_t)h) * (size_t)block_size + (size_t)offset) *
          row;
      memcpy((char *)key_cache + dst, (const char *)key + src, row);
      memcpy((char *)value_cache + dst, (const char *)value + src, row);
    }
  }
  return skipped;
}

/*
 * FP8 codes of n elements of src (element type src_dtype), each divided by `scale` in fp32
 * first: out[i] = code((float)src[i] / scale).
 */
void pao_fp8_encode(const void *src, int src_dtype, int64_t n, float scale, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) {
    const float x = (float)elt_to_double(src, (size_t)i, src_dtype);
    const float q = x / scale;
    out[i] = double_to_fp8((double)q);
  }
}

/* The values of n FP8 codes. */
void pao_fp8_decode(const uint8_t *codes, int64_t n, double *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = fp8_to_double(codes[i]);
}

/*
 * Write side of an FP8 cache: like pao_reshape_and_cache, the rows of kv head h quantised
 * with k_scale[h] (keys) and v_scale[h] (values) on the way in.  key, value have element type
 * src_dtype; the caches hold one code per element.
 */
int pao_reshape_and_cache_fp8(const void *key, const void *value, int src_dtype, uint8_t *key_cache,
                              uint8_t *value_cache, const int64_t *slot_mapping, int64_t num_tokens,
                              int64_t num_blocks, int num_kv_heads, int block_size, int head_dim,
                              const float *k_scale, const float *v_scale) {
  if (num_tokens < 0 || num_blocks < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
    return PAO_BAD_ARG;
  const size_t es = elt_size(src_dtype);
  int skipped = 0;
  for (int64_t i = 0; i < num_tokens; ++i) {
    const int64_t slot = slot_mapping[i];
    if (slot < 0) continue; /* a padding token stores nothing */
    if (slot >= num_blocks * (int64_t)block_size) {
      ++skipped;
      continue;
    }
    const int64_t blk = slot / block_size, off = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      const size_t srow = ((size_t)i * (size_t)num_kv_heads + (size_t)h) * (size_t)head_dim;
      const size_t drow =
          (((size_t)blk * (size_t)num_kv_heads + (size_t)h) * (size_t)block_size + (size_t)off) *
          (size_t)head_dim;
      pao_fp8_encode((const char *)key + srow * es, src_dtype, head_dim, k_scale[h], key_cache + drow);
      pao_fp8_encode((const char *)value + srow * es, src_dtype, head_dim, v_scale[h],
                     value_cache + drow);
    }
  }
  return skipped;
}

/*
 * Copy whole physical blocks (all kv heads, all slots) of both caches: dst <- src for each
 * (src, dst) pair of block_mapping [num_pairs][2].  This is the copy a shared block needs when
 * one of its sharers is about to write into it ([P2] 4.1 and [P3] 2.2: sequences may share a
 * physical block; [P4] 2.2.1 lists beam search as a sharer).
 * Returns the number of pairs skipped because an id lies outside the pool.
 */
int pao_copy_blocks(void *key_cache, void *value_cache, const int64_t *block_mapping,
                    int64_t num_pairs, int64_t num_blocks, int num_kv_heads, int block_size,
                    int head_dim, int dtype) {
  if (num_pairs < 0 || num_blocks < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
    return PAO_BAD_ARG;
  const size_t block_bytes =
      (size_t)num_kv_heads * (size_t)block_size * (size_t)head_dim * elt_size(dtype);
  int skipped = 0;
  for (int64_t p = 0; p < num_pairs; ++p) {
    const int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      ++skipped;
      continue;
    }
    memcpy((char *)key_cache + (size_t)dst * block_bytes,
           (const char *)key_cache + (size_t)src * block_bytes, block_bytes);
    memcpy((char *)value_cache + (size_t)dst * block_bytes,
           (const char *)value_cache + (size_t)src * block_bytes, block_bytes);
  }
  return skipped;
}

/*
 * Move whole physical blocks between two pools of the same block shape: dst pool block dst <-
 * src pool block src, keys and values, for each (src, dst) pair ([P4] 2.3.2: the scheduler
 * swaps KV cache out block by block, to CPU memory, and back in).  src_blocks and dst_blocks
 * are the two pools' block counts.  Returns the number of pairs skipped because an id lies
 * outside its pool.
 */
int pao_swap_blocks(const void *src_key, const void *src_value, int64_t src_blocks,
                    void *dst_key, void *dst_value, int64_t dst_blocks,
                    const int64_t *block_mapping, int64_t num_pairs, int num_kv_heads,
                    int block_size, int head_dim, int dtype) {
  if (num_pairs < 0 || src_blocks < 0 || dst_blocks < 0 || num_kv_heads <= 0 || block_size <= 0 ||
      head_dim <= 0)
    return PAO_BAD_ARG;
  const size_t block_bytes =
      (size_t)num_kv_heads * (size_t)block_size * (size_t)head_dim * elt_size(dtype);
  int skipped = 0;
  for (int64_t p = 0; p < num_pairs; ++p) {
    const int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      ++skipped;
      continue;
    }
    memcpy((char *)dst_key + (size_t)dst * block_bytes,
           (const char *)src_key + (size_t)src * block_bytes, block_bytes);
    memcpy((char *)dst_value + (size_t)dst * block_bytes,
           (const char *)src_value + (size_t)src * block_bytes, block_bytes);
  }
  return skipped;
}

/*
 * Assemble the first `len` tokens of one sequence's keys and values for kv head g into
 * contiguous rows kc[t][d], vc[t][d] ([P4] 2.2.2: look up the physical block of each logical
 * block in the block table, then read K/V from the physical cache).
 */
static int assemble_context(double *kc, double *vc, const void *key_cache,
                            const void *value_cache, int kv_dtype, const int32_t *table_row,
                            int64_t num_blocks, int num_kv_heads, int block_size, int head_dim,
                            int g, int64_t len) {
  for (int64_t t = 0; t < len; ++t) {
    const int64_t logical_block = t / block_size;
    const int64_t offset = t % block_size;
    const int64_t physical_block = table_row[logical_block];
    if (physical_block < 0 || physical_block >= num_blocks) return PAO_BAD_BLOCK_ID;
    const size_t row =
        (((size_t)physical_block * (size_t)num_kv_heads + (size_t)g) * (size_t)block_size +
         (size_t)offset) *
        (size_t)head_dim;
    for (int d = 0; d < head_dim; ++d) {
      kc[(size_t)t * (size_t)head_dim + (size_t)d] = elt_to_double(key_cache, row + (size_t)d, kv_dtype);
      vc[(size_t)t * (size_t)head_dim + (size_t)d] =
          elt_to_double(value_cache, row + (size_t)d, kv_dtype);
    }
  }
  return PAO_OK;
}

/*
 * Softmax attention of one query row over rows [t0, t1) of the assembled context:
 *   z_t = scale * sum_d q[d] k_t[d],   m = max_t z_t,   w_t = exp(z_t - m),
 *   l = sum_t w_t,                     o = sum_t w_t v_t / l.
 * Also returns m and l so that results over disjoint ranges can be merged (pao_lse_combine).
 * An empty range gives o = 0, m = -inf, l = 0.
 */
static void attend_rows(double *o, double *m_out, double *l_out, const double *q, const double *kc,
                        const double *vc, int64_t t0, int64_t t1, int head_dim, double scale,
                        double *z) {
  for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
  if (t1 <= t0) {
    *m_out = -INFINITY;
    *l_out = 0.0;
    return;
  }
  double m = -INFINITY;
  for (int64_t t = t0; t < t1; ++t) {
    double dot = 0.0;
    for (int d = 0; d < head_dim; ++d) dot += q[d] * kc[(size_t)t * (size_t)head_dim + (size_t)d];
    z[t - t0] = scale * dot;
    if (z[t - t0] > m) m = z[t - t0];
  }
  double l = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    const double w = exp(z[t - t0] - m);
    l += w;
    for (int d = 0; d < head_dim; ++d) o[d] += w * vc[(size_t)t * (size_t)head_dim + (size_t)d];
  }
  for (int d = 0; d < head_dim; ++d) o[d] /= l;
  *m_out = m;
  *l_out = l;
}

/*
 * Decode attention over a paged cache, restricted to context positions [t_begin, t_end)
 * (clipped to [0, context_len)).  With t_begin = 0 and t_end >= context_len this is the whole
 * decode step; a narrower range gives one partition's partial result.
 *
 *   out      [num_seqs][num_heads][head_dim]  double
 *   m_out    [num_seqs][num_heads]            double (may be NULL)  max of the scaled logits
 *   l_out    [num_seqs][num_heads]            double (may be NULL)  sum of exp(z - m)
 *   query    [num_seqs][num_heads][head_dim]  q_dtype
 *   block_tables [num_seqs][max_blocks] int32, context_lens [num_seqs] int32
 */
/*
 * As pao_decode_range, with the keys and values of kv head g multiplied by k_scale[g] and
 * v_scale[g] (either may be NULL: 1) after they are read: the attention of an FP8 cache.
 */
int pao_decode_range_scaled(double *out, double *m_out, double *l_out, const void *query,
                            int q_dtype, const void *key_cache, const void *value_cache,
                            int kv_dtype, const int32_t *block_tables, int64_t max_blocks,
                            const int32_t *context_lens, int64_t num_seqs, int num_heads,
                            int num_kv_heads, int head_dim, int block_size, int64_t num_blocks,
                            double scale, int64_t t_begin, int64_t t_end, int num_threads,
                            const float *k_scale, const float *v_scale) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks < 0 || num_heads % num_kv_heads != 0)
    return PAO_BAD_ARG;
  for (int64_t s = 0; s < num_seqs; ++s)
    if (context_lens[s] > max_blocks * (int64_t)block_size) return PAO_BAD_CONTEXT_LEN;
  const int group = num_heads / num_kv_heads;
  int status = PAO_OK;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for collapse(2) schedule(dynamic, 1) num_threads(num_threads)
#endif
  for (int64_t s = 0; s < num_seqs; ++s) {
    for (int h = 0; h < num_heads; ++h) {
      double *o = out + ((size_t)s * (size_t)num_heads + (size_t)h) * (size_t)head_dim;
      double m = -INFINITY, l = 0.0;
      const int64_t len = context_lens[s] > 0 ? context_lens[s] : 0;
      const int64_t t0 = t_begin < 0 ? 0 : (t_begin > len ? len : t_begin);
      const int64_t t1 = t_end > len ? len : (t_end < t0 ? t0 : t_end);
      if (t1 <= t0) {
        for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
      } else {
        const int g = h / group;
        double *kc = (double *)malloc((size_t)t1 * (size_t)head_dim * sizeof(double));
        double *vc = (double *)malloc((size_t)t1 * (size_t)head_dim * sizeof(double));
        double *q = (double *)malloc((size_t)head_dim * sizeof(double));
        double *z = (double *)malloc((size_t)(t1 - t0) * sizeof(double));
        if (!kc || !vc || !q || !z) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
          status = PAO_NO_MEMORY;
        } else {
          const int rc = assemble_context(kc, vc, key_cache, value_cache, kv_dtype,
                                          block_tables + (size_t)s * (size_t)max_blocks,
                                          num_blocks, num_kv_heads, block_size, head_dim, g, t1);
          if (rc != PAO_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = rc;
            for (int d = 0; d < head_dim; ++d) o[d] = NAN;
          } else {
            const double ks = k_scale ? (double)k_scale[g] : 1.0;
            const double vs = v_scale ? (double)v_scale[g] : 1.0;
            for (size_t i = 0; i < (size_t)t1 * (size_t)head_dim; ++i) {
              kc[i] *= ks;
              vc[i] *= vs;
            }
            const size_t qrow = ((size_t)s * (size_t)num_heads + (size_t)h) * (size_t)head_dim;
            for (int d = 0; d < head_dim; ++d) q[d] = elt_to_double(query, qrow + (size_t)d, q_dtype);
            attend_rows(o, &m, &l, q, kc, vc, t0, t1, head_dim, scale, z);
          }
        }
        free(kc);
        free(vc);
        free(q);
        free(z);
      }
      if (m_out) m_out[(size_t)s * (size_t)num_heads + (size_t)h] = m;
      if (l_out) l_out[(size_t)s * (size_t)num_heads + (size_t)h] = l;
    }
  }
  return status;
}

/*
 * Prefill (several new tokens per sequence) over a paged cache.  [P2] 4.2: at each iteration
 * requests join the running batch; a joining request's prompt tokens (or a chunk of them) are
 * the step's new tokens, already written into the sequence's blocks.  Sequence s has
 * q_len = query_start[s+1] - query_start[s] new tokens, the last q_len of its context_len
 * positions; new token j (position p = context_len - q_len + j) attends causally, to positions
 * 0 .. p of the context assembled through the block table ([P4] 2.2.2).
 *
 *   out    [total new tokens][num_heads][head_dim] double, row query_start[s] + j
 *   query  [total new tokens][num_heads][head_dim] q_dtype
 * A sequence with q_len > context_len is an error (PAO_BAD_ARG).
 */
int pao_prefill(double *out, const void *query, int q_dtype, const void *key_cache,
                const void *value_cache, int kv_dtype, const int32_t *block_tables,
                int64_t max_blocks, const int32_t *context_lens, const int32_t *query_start,
                int64_t num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                int64_t num_blocks, double scale, int num_threads) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks < 0 || num_heads % num_kv_heads != 0)
    return PAO_BAD_ARG;
  for (int64_t s = 0; s < num_seqs; ++s) {
    const int64_t q_len = (int64_t)query_start[s + 1] - query_start[s];
    if (q_len < 0 || q_len > context_lens[s]) return PAO_BAD_ARG;
    if (context_lens[s] > max_blocks * (int64_t)block_size) return PAO_BAD_CONTEXT_LEN;
  }
  const int group = num_heads / num_kv_heads;
  int status = PAO_OK;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for collapse(2) schedule(dynamic, 1) num_threads(num_threads)
#endif
  for (int64_t s = 0; s < num_seqs; ++s) {
    for (int h = 0; h < num_heads; ++h) {
      const int64_t len = context_lens[s];
      const int64_t q0 = query_start[s], q_len = (int64_t)query_start[s + 1] - q0;
      if (q_len == 0) continue;
      const int kvh = h / group; /* the kv head query head h reads */
      double *kc = (double *)malloc((size_t)len * (size_t)head_dim * sizeof(double));
      double *vc = (double *)malloc((size_t)len * (size_t)head_dim * sizeof(double));
      double *q = (double *)malloc((size_t)head_dim * sizeof(double));
      double *z = (double *)malloc((size_t)len * sizeof(double));
      int rc = (!kc || !vc || !q || !z) ? PAO_NO_MEMORY : PAO_OK;
      if (rc == PAO_OK)
        rc = assemble_context(kc, vc, key_cache, value_cache, kv_dtype,
                              block_tables + (size_t)s * (size_t)max_blocks, num_blocks,
                              num_kv_heads, block_size, head_dim, kvh, len);
      for (int64_t j = 0; j < q_len; ++j) {
        double *o = out + ((size_t)(q0 + j) * (size_t)num_heads + (size_t)h) * (size_t)head_dim;
        if (rc != PAO_OK) {
          for (int d = 0; d < head_dim; ++d) o[d] = NAN;
          continue;
        }
        const int64_t p = len - q_len + j; /* this token's position: it sees 0 .. p */
        const size_t qrow = ((size_t)(q0 + j) * (size_t)num_heads + (size_t)h) * (size_t)head_dim;
        for (int d = 0; d < head_dim; ++d) q[d] = elt_to_double(query, qrow + (size_t)d, q_dtype);
        double m, l;
        attend_rows(o, &m, &l, q, kc, vc, 0, p + 1, head_dim, scale, z);
      }
      if (rc != PAO_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
        status = rc;
      }
      free(kc);
      free(vc);
      free(q);
      free(z);
    }
  }
  return status;
}

int pao_decode_range(double *out, double *m_out, double *l_out, const void *query, int q_dtype,
                     const void *key_cache, const void *value_cache, int kv_dtype,
                     const int32_t *block_tables, int64_t max_blocks, const int32_t *context_lens,
                     int64_t num_seqs, int num_heads, int num_kv_heads, int head_dim,
                     int block_size, int64_t num_blocks, double scale, int64_t t_begin,
                     int64_t t_end, int num_threads) {
  return pao_decode_range_scaled(out, m_out, l_out, query, q_dtype, key_cache, value_cache,
                                 kv_dtype, block_tables, max_blocks, context_lens, num_seqs,
                                 num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale,
                                 t_begin, t_end, num_threads, NULL, NULL);
}

/* The whole decode step: softmax(scale * q K^T) V over each sequence's full context. */
int pao_decode(double *out, const void *query, int q_dtype, const void *key_cache,
               const void *value_cache, int kv_dtype, const int32_t *block_tables,
               int64_t max_blocks, const int32_t *context_lens, int64_t num_seqs, int num_heads,
               int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, double scale,
               int num_threads) {
  return pao_decode_range(out, NULL, NULL, query, q_dtype, key_cache, value_cache, kv_dtype,
                          block_tables, max_blocks, context_lens, num_seqs, num_heads,
                          num_kv_heads, head_dim, block_size, num_blocks, scale, 0, INT64_MAX,
                          num_threads);
}

/*
 * Merge partial results of one query row over disjoint ranges of its context (the
 * split-context reduce): with M = max_p m_p and w_p = l_p * exp(m_p - M),
 *   out = sum_p w_p o_p / sum_p w_p.
 * o_parts [num_parts][head_dim]; m [num_parts]; l [num_parts].  Parts with l = 0 are empty.
 * If every part is empty, out = 0.
 */
void pao_lse_combine(double *out, const double *o_parts, const double *m, const double *l,
                     int64_t num_parts, int head_dim) {
  double big_m = -INFINITY;
  for (int64_t p = 0; p < num_parts; ++p)
    if (l[p] > 0.0 && m[p] > big_m) big_m = m[p];
  double denom = 0.0;
  for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
  if (big_m == -INFINITY) return;
  for (int64_t p = 0; p < num_parts; ++p) {
    if (!(l[p] > 0.0)) continue;
    const double w = l[p] * exp(m[p] - big_m);
    denom += w;
    for (int d = 0; d < head_dim; ++d) out[d] += w * o_parts[(size_t)p * (size_t)head_dim + (size_t)d];
  }
  for (int d = 0; d < head_dim; ++d) out[d] /= denom;
}

/* Number of threads an OpenMP region of this library would use by default (1 without OpenMP). */
int pao_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
