/*
 * pa_oracle.c -- plain, slow, fp64 CPU oracle for single-query decode
 * attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no source, header, table or
 * helper with the CUDA library; the two meet only through the seeded input
 * arrays the tests hand to both.
 *
 * What it computes follows the pages literally, with no blocking, fusion or
 * reordering beyond what they state:
 *
 *   - Address mapping (page "Implementing teaching PagedAttention: reading the
 *     historical KV cache from the block table", section "From logical token
 *     to physical block"): logical_block_id = t / block_size,
 *     block_offset = t % block_size, physical_block_id =
 *     block_table[logical_block_id]; the K/V row lives at
 *     key_cache[physical_block_id, block_offset].
 *   - Gather first, then attention (same page, sections "Teaching
 *     implementation: gather first, then attention", "Paged gather for a
 *     single Sequence" and "Extending to a batch"): for t in [0, context_len)
 *     copy K/V rows in logical order into a contiguous [context_len, Hkv, D]
 *     buffer, then run standard attention on it.
 *   - Standard attention (page "From correct to faster: the PagedAttention
 *     optimisation route", section "What the attention kernel really does"):
 *     score_t = dot(query, key_t) * scale with scale = 1/sqrt(head_dim)
 *     passed in by the caller, weights = softmax(scores),
 *     output = sum_t weight_t * value_t.  Two passes, all in double.
 *   - Cache write by slot (teaching page, section "Writing slots and reading
 *     the block table must agree"): the current token's K/V row is stored at
 *     (physical_block_id, block_offset); the slot is encoded as the flat
 *     integer physical_block_id * block_size + block_offset, negative = skip.
 *   - Per-partition partials (max, sum, normalised partial output) and their
 *     merge: the running-max / normaliser bookkeeping of the online softmax
 *     (optimisation-route page, section "What the attention kernel really
 *     does", blockwise softmax paragraph), applied to whole partitions.
 *   - Paged (chunked) prefill with the causal mask (teaching page, section
 *     "Where is the attention mask"): new token j of a chunk of n attends to
 *     positions 0 .. context_len - n + j, gathered through the block table.
 *   - FP8 pages (a reading: the pages name quantised KV as a later
 *     addition): E4M3 codes of the OCP 8-bit floating point format, value =
 *     code * per-tensor scale; the write rounds x / scale (IEEE single
 *     precision division) to the nearest code, ties to even, saturating.
 *
 * Readings where the pages are silent: query head hq uses KV head
 * hq / (Hq / Hkv) (contiguous GQA groups); bf16 values are widened exactly
 * (bits << 16) before any arithmetic; a sequence whose context length is
 * outside [0, max_blocks * block_size] or whose block table names a block
 * outside [0, num_blocks) is reported through the returned flags and its
 * output is all zeros; context_len == 0 gives a zero output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_DTYPE_F32 0
#define ORC_DTYPE_BF16 1
#define ORC_DTYPE_FP8_E4M3 2 /* cache codes; see orc_e4m3_value */
#define ORC_DTYPE_F64 3      /* already-widened values (e.g. dequantised pages) */

#define ORC_FLAG_BLOCK_ID 1
#define ORC_FLAG_CONTEXT_LEN 2
#define ORC_FLAG_SLOT 4

/* FP8 KV pages (a reading: the pages name quantised KV only as a later
 * addition).  Codes follow the OCP 8-bit floating point format E4M3 in its
 * "fn" form: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent 0 holds the subnormals m/8 * 2^-6; there are no infinities and
 * S.1111.111 is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.
 * A cache entry stands for code value * scale (one scale per tensor). */
static double orc_e4m3_value(uint8_t c) {
  const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  const double v = (e == 0) ? ldexp((double)m, -9) : ldexp(8.0 + m, e - 10);
  return sgn ? -v : v;
}

/* The E4M3 code nearest to x: ties go to the even mantissa, magnitudes at
 * or above 448 saturate to 448, NaN stays NaN (0x7F), the sign of zero is
 * kept.  Uses the default round-to-nearest-even mode of nearbyint. */
uint8_t orc_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sgn = signbit(x) ? 0x80 : 0;
  const double a = fabs(x);
  if (a >= 448.0) return sgn | 0x7E;
  if (a < ldexp(1.0, -6)) {
    /* subnormal range, quantum 2^-9; n == 8 is the smallest normal (0x08) */
    const double n = nearbyint(ldexp(a, 9));
    return sgn | (uint8_t)n;
  }
  int k;
  frexp(a, &k); /* a in [2^(k-1), 2^k) */
  int E = k - 1; /* -6 .. 8 */
  double n = nearbyint(ldexp(a, 3 - E)); /* a / 2^(E-3), in [8, 16] */
  if (n == 16.0) {
    E += 1;
    n = 8.0;
  }
  if (E > 8) return sgn | 0x7E;
  return sgn | (uint8_t)(((E + 7) << 3) | ((int)n - 8));
}

void orc_e4m3_encode_array(const double *x, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

/* Read element idx of a stored array and widen it exactly to double. */
static double orc_load(const void *base, int64_t idx, int dtype) {
  if (dtype == ORC_DTYPE_F32) {
    return (double)((const float *)base)[idx];
  }
  if (dtype == ORC_DTYPE_FP8_E4M3) {
    return orc_e4m3_value(((const uint8_t *)base)[idx]);
  }
  if (dtype == ORC_DTYPE_F64) {
    return ((const double *)base)[idx];
  }
  uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Widen n stored values to double (exposed so tests can pin the widening
 * against a library conversion). */
void orc_widen(const void *src, int dtype, int64_t n, double *dst) {
  for (int64_t i = 0; i < n; ++i) dst[i] = orc_load(src, i, dtype);
}

/* The address mapping of one logical token.  This is the definition the
 * teaching page gives (section "From logical token to physical block": the
 * logical block is the token index divided by the block size, the offset
 * its remainder, the physical block the table's entry), written out from
 * that statement in this file's own terms; the gather below applies it per
 * token in logical order.  Returns 0, or a flag if the logical block is
 * past max_blocks or the physical id is out of range. */
int orc_map_token(const int32_t *block_table, int32_t max_blocks,
                  int32_t num_blocks, int32_t block_size, int64_t token_index,
                  int32_t *physical_block_id, int32_t *block_offset) {
  int64_t logical_block_id = token_index / block_size;
  int64_t offset = token_index % block_size;
  if (logical_block_id >= max_blocks) return ORC_FLAG_CONTEXT_LEN;
  int32_t pb = block_table[logical_block_id];
  *physical_block_id = pb;
  *block_offset = (int32_t)offset;
  if (pb < 0 || pb >= num_blocks) return ORC_FLAG_BLOCK_ID;
  return 0;
}

/* Paged gather: K/V rows of tokens [0, context_len) in logical order, each
 * row Hkv*D values widened to double.  keys/values: [context_len, Hkv, D]. */
int orc_gather_kv(const void *key_cache, const void *value_cache, int dtype,
                  int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                  int32_t head_dim, const int32_t *block_table,
                  int32_t max_blocks, int32_t context_len, double *keys,
                  double *values) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  int flags = 0;
  for (int64_t t = 0; t < context_len; ++t) {
    int32_t pb = 0, off = 0;
    int f = orc_map_token(block_table, max_blocks, num_blocks, block_size, t,
                          &pb, &off);
    if (f) {
      flags |= f;
      continue;
    }
    const int64_t src = ((int64_t)pb * block_size + off) * row;
    for (int64_t e = 0; e < row; ++e) {
      keys[t * row + e] = orc_load(key_cache, src + e, dtype);
      values[t * row + e] = orc_load(value_cache, src + e, dtype);
    }
  }
  return flags;
}

/* Softmax attention of one query vector over tokens [t0, t1) of contiguous
 * K/V whose rows are row_stride doubles apart (keys/values already point at
 * the head's slice of row 0).  Writes the score maximum m, the normaliser
 * l = sum exp(s - m) and out = sum_t (exp(s_t - m) / l) * v_t. */
static void orc_attend_range(const double *qh, const double *keys,
                             const double *values, int64_t row_stride,
                             int64_t t0, int64_t t1, int32_t head_dim,
                             double scale, double *scores, double *m_out,
                             double *l_out, double *oh) {
  for (int32_t d = 0; d < head_dim; ++d) oh[d] = 0.0;
  double m = -INFINITY;
  for (int64_t t = t0; t < t1; ++t) {
    const double *k = keys + t * row_stride;
    double dot = 0.0;
    for (int32_t d = 0; d < head_dim; ++d) dot += qh[d] * k[d];
    scores[t - t0] = dot * scale;
    if (scores[t - t0] > m) m = scores[t - t0];
  }
  double denom = 0.0;
  for (int64_t t = t0; t < t1; ++t) denom += exp(scores[t - t0] - m);
  for (int64_t t = t0; t < t1; ++t) {
    const double w = exp(scores[t - t0] - m) / denom;
    const double *v = values + t * row_stride;
    for (int32_t d = 0; d < head_dim; ++d) oh[d] += w * v[d];
  }
  *m_out = m;
  *l_out = denom;
}

/* Standard single-query attention for one sequence on contiguous K/V.
 * q: [Hq, D]; keys/values: [context_len, Hkv, D]; out: [Hq, D].
 * A zero-length context gives zeros.  Query heads run in parallel. */
void orc_attention(const double *q, const double *keys, const double *values,
                   int32_t context_len, int32_t num_q_heads,
                   int32_t num_kv_heads, int32_t head_dim, double scale,
                   double *out) {
  const int32_t group = num_q_heads / num_kv_heads;
  const int64_t row = (int64_t)num_kv_heads * head_dim;
#pragma omp parallel for schedule(static)
  for (int32_t hq = 0; hq < num_q_heads; ++hq) {
    const int32_t h = hq / group;
    double *oh = out + (int64_t)hq * head_dim;
    if (context_len <= 0) {
      for (int32_t d = 0; d < head_dim; ++d) oh[d] = 0.0;
      continue;
    }
    double *scores = (double *)malloc(sizeof(double) * context_len);
    double m, l;
    orc_attend_range(q + (int64_t)hq * head_dim, keys + (int64_t)h * head_dim,
                     values + (int64_t)h * head_dim, row, 0, context_len,
                     head_dim, scale, scores, &m, &l, oh);
    free(scores);
  }
}

static int orc_check_len(int32_t context_len, int32_t max_blocks,
                         int32_t block_size) {
  if (context_len < 0) return ORC_FLAG_CONTEXT_LEN;
  if ((int64_t)context_len > (int64_t)max_blocks * block_size)
    return ORC_FLAG_CONTEXT_LEN;
  return 0;
}

/* Gather one sequence; on success returns 0 and hands back malloc'd
 * keys/values (caller frees), else flags and NULL buffers. */
static int orc_gather_seq(const void *key_cache, const void *value_cache,
                          int dtype, int32_t num_blocks, int32_t block_size,
                          int32_t num_kv_heads, int32_t head_dim,
                          const int32_t *block_table, int32_t max_blocks,
                          int32_t ctx, double **keys, double **values) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  *keys = NULL;
  *values = NULL;
  int flags = orc_check_len(ctx, max_blocks, block_size);
  if (flags || ctx == 0) return flags;
  *keys = (double *)malloc(sizeof(double) * ctx * row);
  *values = (double *)malloc(sizeof(double) * ctx * row);
  flags = orc_gather_kv(key_cache, value_cache, dtype, num_blocks, block_size,
                        num_kv_heads, head_dim, block_table, max_blocks, ctx,
                        *keys, *values);
  if (flags) {
    free(*keys);
    free(*values);
    *keys = NULL;
    *values = NULL;
  }
  return flags;
}

/* Batched decode: for each sequence gather its history through its block
 * table, then apply standard attention.  q: [B, Hq, D] stored in dtype;
 * out: [B, Hq, D] double; seq_flags (nullable): per-sequence flags.
 * Returns the OR of all flags. */
int orc_decode(const void *q, const void *key_cache, const void *value_cache,
               int dtype, int32_t num_blocks, int32_t block_size,
               int32_t num_kv_heads, int32_t head_dim,
               const int32_t *block_tables, const int32_t *context_lens,
               int32_t batch, int32_t num_q_heads, int32_t max_blocks,
               double scale, double *out, int32_t *seq_flags) {
  const int64_t qrow = (int64_t)num_q_heads * head_dim;
  double *qd = (double *)malloc(sizeof(double) * qrow);
  int all = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t ctx = context_lens[b];
    double *ob = out + (int64_t)b * qrow;
    double *keys, *values;
    int flags = orc_gather_seq(key_cache, value_cache, dtype, num_blocks,
                               block_size, num_kv_heads, head_dim,
                               block_tables + (int64_t)b * max_blocks,
                               max_blocks, ctx, &keys, &values);
    if (flags || ctx == 0) {
      for (int64_t e = 0; e < qrow; ++e) ob[e] = 0.0;
    } else {
      for (int64_t e = 0; e < qrow; ++e)
        qd[e] = orc_load(q, (int64_t)b * qrow + e, dtype);
      orc_attention(qd, keys, values, ctx, num_q_heads, num_kv_heads, head_dim,
                    scale, ob);
    }
    free(keys);
    free(values);
    if (seq_flags) seq_flags[b] = flags;
    all |= flags;
  }
  free(qd);
  return all;
}

/* Paged (chunked) prefill with the causal mask.  Teaching page, section
 * "Where is the attention mask": in prefill every prompt token sees only
 * itself and the tokens before it; route page, section "decode attention
 * and prefill attention are different": prefill processes a whole prompt
 * (or a chunk of it) at once.  Sequence b brings n_b = qstart[b+1] -
 * qstart[b] new tokens whose K/V rows are already stored at their slots;
 * its history is context_lens[b] tokens including them, so new token j sits
 * at position p = context_lens[b] - n_b + j and attends to positions
 * [0, p], read through the block table (gather first, then attention, as in
 * orc_decode).  q, out: [qstart[batch], Hq, D] (q stored in dtype, out
 * double).  n_b < 0 or n_b > context_lens[b], or bad metadata, flags the
 * sequence and its rows are zero.  Returns the OR of all flags. */
int orc_prefill(const void *q, const void *key_cache, const void *value_cache, int dtype,
                int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                int32_t head_dim, const int32_t *block_tables, const int32_t *context_lens,
                const int32_t *qstart, int32_t batch, int32_t num_q_heads, int32_t max_blocks,
                double scale, double *out, int32_t *seq_flags) {
  const int64_t qrow = (int64_t)num_q_heads * head_dim;
  const int64_t kvrow = (int64_t)num_kv_heads * head_dim;
  const int32_t group = num_q_heads / num_kv_heads;
  int all = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t n = qstart[b + 1] - qstart[b];
    const int32_t ctx = context_lens[b];
    double *rows = out + (int64_t)qstart[b] * qrow;
    double *keys = NULL, *values = NULL;
    int flags = 0;
    if (n < 0 || n > ctx) {
      flags = ORC_FLAG_CONTEXT_LEN;
    } else {
      flags = orc_gather_seq(key_cache, value_cache, dtype, num_blocks, block_size,
                             num_kv_heads, head_dim, block_tables + (int64_t)b * max_blocks,
                             max_blocks, ctx, &keys, &values);
    }
    if (flags || n <= 0) {
      for (int64_t e = 0; n > 0 && e < (int64_t)n * qrow; ++e) rows[e] = 0.0;
    } else {
      double *scores = (double *)malloc(sizeof(double) * ctx);
      double *qh = (double *)malloc(sizeof(double) * head_dim);
      for (int32_t j = 0; j < n; ++j) {
        const int64_t pos = (int64_t)ctx - n + j;
        for (int32_t hq = 0; hq < num_q_heads; ++hq) {
          const int32_t h = hq / group;
          const int64_t qi = ((int64_t)qstart[b] + j) * qrow + (int64_t)hq * head_dim;
          for (int32_t d = 0; d < head_dim; ++d) qh[d] = orc_load(q, qi + d, dtype);
          double m, l;
          orc_attend_range(qh, keys + (int64_t)h * head_dim, values + (int64_t)h * head_dim,
                           kvrow, 0, pos + 1, head_dim, scale, scores, &m, &l,
                           rows + (int64_t)j * qrow + (int64_t)hq * head_dim);
        }
      }
      free(scores);
      free(qh);
    }
    free(keys);
    free(values);
    if (seq_flags) seq_flags[b] = flags;
    all |= flags;
  }
  return all;
}

/* Per-partition partials.  Partition p of sequence b covers tokens
 * [p*P, min((p+1)*P, ctx)).  For every non-empty partition:
 *   part_max[b,hq,p] = max_t s_t,  part_sum[b,hq,p] = sum_t exp(s_t - max),
 *   part_out[b,hq,p,:] = sum_t exp(s_t - max) v_t / part_sum.
 * Empty partitions (p >= ceil(ctx/P)) and whole sequences with flags get
 * part_max = -inf, part_sum = 0, part_out = 0.
 * Shapes: part_max/part_sum [B, Hq, max_partitions], part_out [..., D]. */
int orc_partials(const void *q, const void *key_cache, const void *value_cache,
                 int dtype, int32_t num_blocks, int32_t block_size,
                 int32_t num_kv_heads, int32_t head_dim,
                 const int32_t *block_tables, const int32_t *context_lens,
                 int32_t batch, int32_t num_q_heads, int32_t max_blocks,
                 double scale, int32_t partition_tokens,
                 int32_t max_partitions, double *part_max, double *part_sum,
                 double *part_out) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  const int64_t qrow = (int64_t)num_q_heads * head_dim;
  const int32_t group = num_q_heads / num_kv_heads;
  int all = 0;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t ctx = context_lens[b];
    double *keys, *values;
    int flags = orc_gather_seq(key_cache, value_cache, dtype, num_blocks,
                               block_size, num_kv_heads, head_dim,
                               block_tables + (int64_t)b * max_blocks,
                               max_blocks, ctx, &keys, &values);
    const int64_t nparts =
        flags ? 0 : ((int64_t)ctx + partition_tokens - 1) / partition_tokens;
    if (nparts > max_partitions) flags |= ORC_FLAG_CONTEXT_LEN;
    all |= flags;
#pragma omp parallel for schedule(static)
    for (int32_t hq = 0; hq < num_q_heads; ++hq) {
      const int32_t h = hq / group;
      double *qh = (double *)malloc(sizeof(double) * head_dim);
      double *scores = (double *)malloc(sizeof(double) * partition_tokens);
      for (int32_t d = 0; d < head_dim; ++d)
        qh[d] = orc_load(q, (int64_t)b * qrow + (int64_t)hq * head_dim + d,
                         dtype);
      for (int64_t p = 0; p < max_partitions; ++p) {
        const int64_t ix = ((int64_t)b * num_q_heads + hq) * max_partitions + p;
        double *op = part_out + ix * head_dim;
        if (flags || p >= nparts) {
          part_max[ix] = -INFINITY;
          part_sum[ix] = 0.0;
          for (int32_t d = 0; d < head_dim; ++d) op[d] = 0.0;
          continue;
        }
        const int64_t t0 = p * partition_tokens;
        int64_t t1 = t0 + partition_tokens;
        if (t1 > ctx) t1 = ctx;
        orc_attend_range(qh, keys + (int64_t)h * head_dim,
                         values + (int64_t)h * head_dim, row, t0, t1, head_dim,
                         scale, scores, &part_max[ix], &part_sum[ix], op);
      }
      free(scores);
      free(qh);
    }
    free(keys);
    free(values);
  }
  return all;
}

/* Merge of per-partition partials into the output:
 *   M = max_p m_p over partitions with l_p > 0,  w_p = l_p * exp(m_p - M),
 *   out = sum_p w_p o_p / sum_p w_p;  no non-empty partition -> zeros. */
void orc_merge(const double *part_max, const double *part_sum,
               const double *part_out, int32_t batch, int32_t num_q_heads,
               int32_t head_dim, int32_t max_partitions, double *out) {
  for (int64_t bh = 0; bh < (int64_t)batch * num_q_heads; ++bh) {
    const double *mp = part_max + bh * max_partitions;
    const double *lp = part_sum + bh * max_partitions;
    double *o = out + bh * head_dim;
    for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    double M = -INFINITY;
    for (int32_t p = 0; p < max_partitions; ++p)
      if (lp[p] > 0.0 && mp[p] > M) M = mp[p];
    if (M == -INFINITY) continue;
    double wsum = 0.0;
    for (int32_t p = 0; p < max_partitions; ++p) {
      if (!(lp[p] > 0.0)) continue;
      const double w = lp[p] * exp(mp[p] - M);
      wsum += w;
      const double *op = part_out + (bh * max_partitions + p) * head_dim;
      for (int32_t d = 0; d < head_dim; ++d) o[d] += w * op[d];
    }
    for (int32_t d = 0; d < head_dim; ++d) o[d] /= wsum;
  }
}

/* Cache write into FP8 pages: the new rows arrive as bf16 (widened
 * exactly), each element is divided by its tensor's scale in IEEE single
 * precision and rounded to the nearest E4M3 code (orc_e4m3_encode) -- the
 * quantisation decision is taken in the precision the kernel takes it in.
 * Slots as in orc_write_kv_cache. */
int orc_write_kv_cache_fp8(uint8_t *key_cache, uint8_t *value_cache, const uint16_t *k_new,
                           const uint16_t *v_new, const int64_t *slot_mapping,
                           int32_t num_tokens, float k_scale, float v_scale,
                           int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                           int32_t head_dim) {
  const int64_t row = (int64_t)num_kv_heads * head_dim;
  int flags = 0;
  for (int32_t i = 0; i < num_tokens; ++i) {
    const int64_t s = slot_mapping[i];
    if (s < 0) continue;
    if (s >= (int64_t)num_blocks * block_size) {
      flags |= ORC_FLAG_SLOT;
      continue;
    }
    for (int64_t e = 0; e < row; ++e) {
      const volatile float kq = (float)orc_load(k_new, i * row + e, ORC_DTYPE_BF16) / k_scale;
      const volatile float vq = (float)orc_load(v_new, i * row + e, ORC_DTYPE_BF16) / v_scale;
      key_cache[s * row + e] = orc_e4m3_encode((double)kq);
      value_cache[s * row + e] = orc_e4m3_encode((double)vq);
    }
  }
  return flags;
}

/* Cache write by slot mapping: for each new token i with slot s >= 0 copy
 * its K row and V row (Hkv*D elements of elem_bytes each) byte for byte to
 * key_cache[s / block_size, s % block_size] and the same in value_cache.
 * A slot at or past num_blocks*block_size is flagged and skipped. */
int orc_write_kv_cache(void *key_cache, void *value_cache, const void *k_new,
                       const void *v_new, const int64_t *slot_mapping,
                       int32_t num_tokens, int32_t elem_bytes,
                       int32_t num_blocks, int32_t block_size,
                       int32_t num_kv_heads, int32_t head_dim) {
  const int64_t row_bytes = (int64_t)num_kv_heads * head_dim * elem_bytes;
  int flags = 0;
  for (int32_t i = 0; i < num_tokens; ++i) {
    const int64_t s = slot_mapping[i];
    if (s < 0) continue;
    if (s >= (int64_t)num_blocks * block_size) {
      flags |= ORC_FLAG_SLOT;
      continue;
    }
    const int64_t pb = s / block_size, off = s % block_size;
    const int64_t dst = (pb * block_size + off) * row_bytes;
    memcpy((char *)key_cache + dst, (const char *)k_new + i * row_bytes,
           row_bytes);
    memcpy((char *)value_cache + dst, (const char *)v_new + i * row_bytes,
           row_bytes);
  }
  return flags;
}

/* Threads of the OpenMP loops (query heads of a sequence, partitions):
 * set for timing runs, read back to report what a run used.  Without OpenMP
 * everything runs on one thread. */
#ifdef _OPENMP
#include <omp.h>
#endif
void orc_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
