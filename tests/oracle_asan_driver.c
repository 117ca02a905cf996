/* Runs every entry point of the C oracle (oracle/pa_oracle.c) on small inputs
 * held in heap buffers of exactly their size, including the edge cases the
 * oracle flags (empty and over-long contexts, block ids outside the pool,
 * slots past the pool, chunks longer than their history).  Built with
 * AddressSanitizer and UndefinedBehaviorSanitizer by tests/test_oracle_asan.py:
 * any read or write outside an array, use after free, leak or undefined
 * arithmetic aborts the run.  A few closed forms are checked on the way
 * (a one-token context gives V_0; split partials merge to the decode).
 * Test infrastructure only. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

int orc_map_token(const int32_t *, int32_t, int32_t, int32_t, int64_t, int32_t *, int32_t *);
int orc_gather_kv(const void *, const void *, int, int32_t, int32_t, int32_t, int32_t,
                  const int32_t *, int32_t, int32_t, double *, double *);
void orc_attention(const double *, const double *, const double *, int32_t, int32_t, int32_t,
                   int32_t, double, double *);
int orc_decode(const void *, const void *, const void *, int, int32_t, int32_t, int32_t, int32_t,
               const int32_t *, const int32_t *, int32_t, int32_t, int32_t, double, double *,
               int32_t *);
int orc_prefill(const void *, const void *, const void *, int, int32_t, int32_t, int32_t, int32_t,
                const int32_t *, const int32_t *, const int32_t *, int32_t, int32_t, int32_t,
                double, double *, int32_t *);
int orc_partials(const void *, const void *, const void *, int, int32_t, int32_t, int32_t,
                 int32_t, const int32_t *, const int32_t *, int32_t, int32_t, int32_t, double,
                 int32_t, int32_t, double *, double *, double *);
void orc_merge(const double *, const double *, const double *, int32_t, int32_t, int32_t,
               int32_t, double *);
int orc_write_kv_cache(void *, void *, const void *, const void *, const int64_t *, int32_t,
                       int32_t, int32_t, int32_t, int32_t, int32_t);
int orc_write_kv_cache_fp8(uint8_t *, uint8_t *, const uint16_t *, const uint16_t *,
                           const int64_t *, int32_t, float, float, int32_t, int32_t, int32_t,
                           int32_t);
uint8_t orc_e4m3_encode(double);
void orc_e4m3_encode_array(const double *, int64_t, uint8_t *);
void orc_widen(const void *, int, int64_t, double *);

enum { F32 = 0, BF16 = 1, FP8 = 2, F64 = 3 };
enum { NB = 10, BS = 4, HKV = 2, D = 8, HQ = 4, MB = 3, B = 6 };
#define ROW (HKV * D)
#define POOL ((int64_t)NB * BS * ROW)

static int failures = 0;
#define CHECK(c)                                                   \
  do {                                                             \
    if (!(c)) {                                                    \
      fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #c); \
      ++failures;                                                  \
    }                                                              \
  } while (0)

static uint64_t rng_state = 0x9e3779b97f4a7c15ull;
static double uniform(void) { /* splitmix64 -> [-1, 1) */
  uint64_t z = (rng_state += 0x9e3779b97f4a7c15ull);
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  z ^= z >> 31;
  return (double)(z >> 11) / (double)(1ull << 52) - 1.0;
}

static void *exact(size_t bytes) { /* a heap block of exactly `bytes` (>= 1) */
  void *p = malloc(bytes ? bytes : 1);
  if (!p) abort();
  return p;
}

static float *f32_array(int64_t n) {
  float *a = exact(sizeof(float) * n);
  for (int64_t i = 0; i < n; ++i) a[i] = (float)uniform();
  return a;
}

static uint16_t *bf16_of(const float *a, int64_t n) { /* truncation is enough here */
  uint16_t *o = exact(sizeof(uint16_t) * n);
  for (int64_t i = 0; i < n; ++i) {
    uint32_t u;
    memcpy(&u, &a[i], 4);
    o[i] = (uint16_t)(u >> 16);
  }
  return o;
}

int main(void) {
  /* pools and queries in every stored format */
  float *kc = f32_array(POOL), *vc = f32_array(POOL), *q = f32_array((int64_t)B * HQ * D);
  uint16_t *kc16 = bf16_of(kc, POOL), *vc16 = bf16_of(vc, POOL);
  uint16_t *q16 = bf16_of(q, (int64_t)B * HQ * D);
  double *kc64 = exact(sizeof(double) * POOL), *vc64 = exact(sizeof(double) * POOL);
  double *q64 = exact(sizeof(double) * B * HQ * D);
  orc_widen(kc, F32, POOL, kc64);
  orc_widen(vc, F32, POOL, vc64);
  orc_widen(q, F32, (int64_t)B * HQ * D, q64);
  double *tmp = exact(sizeof(double) * POOL);
  for (int64_t i = 0; i < POOL; ++i) tmp[i] = 300.0 * uniform();
  uint8_t *kc8 = exact(POOL), *vc8 = exact(POOL);
  orc_e4m3_encode_array(tmp, POOL, kc8);
  orc_e4m3_encode_array(tmp, POOL, vc8);

  /* tables: [B, MB]; contexts: empty, one token, full table, two pages,
   * a bad id inside the context, a bad id past it (never read) */
  const int32_t tables[B * MB] = {7, 2, 9, 3, 0, 1, 4, 5, 6, 8, 1, 0, 2, NB + 4, 3, 5, 6, -1};
  const int32_t ctx[B] = {0, 1, MB * BS, 2 * BS, 5, 2 * BS};
  const void *pools[4][2] = {{kc, vc}, {kc16, vc16}, {kc8, vc8}, {kc64, vc64}};
  const void *queries[4] = {q, q16, q16, q64}; /* FP8 pages take bf16 queries */
  for (int dt = 0; dt < 4; ++dt) {
    double *out = exact(sizeof(double) * B * HQ * D);
    int32_t flags[B];
    const int all = orc_decode(queries[dt], pools[dt][0], pools[dt][1], dt, NB, BS, HKV, D,
                               tables, ctx, B, HQ, MB, 0.3, out, flags);
    CHECK(all == 1);
    CHECK(flags[0] == 0 && flags[1] == 0 && flags[2] == 0 && flags[3] == 0);
    CHECK(flags[4] == 1 && flags[5] == 0);
    for (int e = 0; e < HQ * D; ++e) CHECK(out[e] == 0.0);         /* empty context */
    for (int e = 0; e < HQ * D; ++e) CHECK(out[4 * HQ * D + e] == 0.0); /* flagged */
    if (dt != FP8) {
      /* one token: the weight is 1 and the output is V_0 of the head, exactly */
      for (int hq = 0; hq < HQ; ++hq)
        for (int d = 0; d < D; ++d) {
          const int64_t at = ((int64_t)tables[MB] * BS * HKV + hq / (HQ / HKV)) * D + d;
          double want;
          orc_widen(pools[dt][1], dt, 1, &want); /* exercise the widening of element 0 */
          if (dt == F32) {
            want = (double)vc[at];
          } else if (dt == BF16) {
            const uint32_t u = (uint32_t)vc16[at] << 16;
            float f;
            memcpy(&f, &u, 4);
            want = f;
          } else {
            want = vc64[at];
          }
          CHECK(out[(int64_t)HQ * D + hq * D + d] == want);
        }
    }
    free(out);
  }
  {
    /* lengths the table cannot hold, negative lengths */
    const int32_t bad_ctx[2] = {MB * BS + 1, -3};
    double *out = exact(sizeof(double) * 2 * HQ * D);
    int32_t flags[2];
    CHECK(orc_decode(q, kc, vc, F32, NB, BS, HKV, D, tables, bad_ctx, 2, HQ, MB, 0.3, out,
                     flags) == 2);
    CHECK(flags[0] == 2 && flags[1] == 2);
    free(out);
  }
  {
    /* mapping and gather */
    int32_t pb = -7, off = -7;
    CHECK(orc_map_token(tables, MB, NB, BS, 5, &pb, &off) == 0 && pb == 2 && off == 1);
    CHECK(orc_map_token(tables, MB, NB, BS, MB * BS, &pb, &off) == 2);
    CHECK(orc_map_token(tables + 4 * MB, MB, NB, BS, BS, &pb, &off) == 1);
    const int32_t n = MB * BS;
    double *keys = exact(sizeof(double) * n * ROW), *values = exact(sizeof(double) * n * ROW);
    CHECK(orc_gather_kv(kc16, vc16, BF16, NB, BS, HKV, D, tables, MB, n, keys, values) == 0);
    double *att = exact(sizeof(double) * HQ * D);
    orc_attention(q64, keys, values, n, HQ, HKV, D, 0.3, att);
    orc_attention(q64, keys, values, 0, HQ, HKV, D, 0.3, att);
    for (int e = 0; e < HQ * D; ++e) CHECK(att[e] == 0.0);
    free(att);
    free(keys);
    free(values);
  }
  {
    /* split partials (4-token partitions) merged == decode */
    enum { P = 4, MP = 3 };
    double *pm = exact(sizeof(double) * B * HQ * MP), *ps = exact(sizeof(double) * B * HQ * MP);
    double *po = exact(sizeof(double) * B * HQ * MP * D);
    double *merged = exact(sizeof(double) * B * HQ * D), *dec = exact(sizeof(double) * B * HQ * D);
    orc_partials(q, kc, vc, F32, NB, BS, HKV, D, tables, ctx, B, HQ, MB, 0.3, P, MP, pm, ps, po);
    orc_merge(pm, ps, po, B, HQ, D, MP, merged);
    orc_decode(q, kc, vc, F32, NB, BS, HKV, D, tables, ctx, B, HQ, MB, 0.3, dec, NULL);
    for (int b = 0; b < B; ++b) {
      if (b == 4) continue; /* flagged: both give zeros, the partials empty ones */
      for (int e = 0; e < HQ * D; ++e)
        CHECK(fabs(merged[(int64_t)b * HQ * D + e] - dec[(int64_t)b * HQ * D + e]) < 1e-12);
    }
    /* too few partitions for a context */
    CHECK(orc_partials(q, kc, vc, F32, NB, BS, HKV, D, tables, ctx, B, HQ, MB, 0.3, P, 2, pm, ps,
                       po) & 2);
    free(pm);
    free(ps);
    free(po);
    free(merged);
    free(dec);
  }
  {
    /* prefill: chunks of 0, 1, a whole prompt, a later chunk, one over a
     * bad block, one longer than its history */
    const int32_t pctx[B] = {0, 1, MB * BS, 2 * BS, 5, 2 * BS};
    const int32_t n[B] = {0, 1, MB * BS, 3, 2, 2 * BS + 1};
    int32_t qstart[B + 1];
    qstart[0] = 0;
    for (int b = 0; b < B; ++b) qstart[b + 1] = qstart[b] + n[b];
    const int32_t T = qstart[B];
    float *pq = f32_array((int64_t)T * HQ * D);
    double *out = exact(sizeof(double) * T * HQ * D);
    int32_t flags[B];
    const int all = orc_prefill(pq, kc, vc, F32, NB, BS, HKV, D, tables, pctx, qstart, B, HQ, MB,
                                0.3, out, flags);
    CHECK(all == 3);
    CHECK(flags[0] == 0 && flags[1] == 0 && flags[2] == 0 && flags[3] == 0);
    CHECK(flags[4] == 1 && flags[5] == 2);
    for (int64_t e = (int64_t)qstart[4] * HQ * D; e < (int64_t)T * HQ * D; ++e)
      CHECK(out[e] == 0.0);
    free(pq);
    free(out);
  }
  {
    /* cache writes: a skipped token, a slot past the pool, the last slot */
    enum { N = 4 };
    const int64_t slots[N] = {9, -1, (int64_t)NB * BS, (int64_t)NB * BS - 1};
    float *kn = f32_array(N * ROW), *vn = f32_array(N * ROW);
    CHECK(orc_write_kv_cache(kc, vc, kn, vn, slots, N, 4, NB, BS, HKV, D) == 4);
    CHECK(memcmp(kc + 9 * ROW, kn, sizeof(float) * ROW) == 0);
    CHECK(memcmp(vc + ((int64_t)NB * BS - 1) * ROW, vn + 3 * ROW, sizeof(float) * ROW) == 0);
    uint16_t *kn16 = bf16_of(kn, N * ROW), *vn16 = bf16_of(vn, N * ROW);
    CHECK(orc_write_kv_cache(kc16, vc16, kn16, vn16, slots, N, 2, NB, BS, HKV, D) == 4);
    CHECK(orc_write_kv_cache_fp8(kc8, vc8, kn16, vn16, slots, N, 0.25f, 0.5f, NB, BS, HKV, D) ==
          4);
    CHECK(orc_write_kv_cache(kc, vc, kn, vn, slots, 0, 4, NB, BS, HKV, D) == 0);
    free(kn);
    free(vn);
    free(kn16);
    free(vn16);
  }
  {
    /* the E4M3 encoder at its special values */
    const double x[8] = {NAN, INFINITY, -INFINITY, 448.0, 1e9, 1e-30, -0.0, 0.0};
    uint8_t c[8];
    orc_e4m3_encode_array(x, 8, c);
    CHECK(c[0] == 0x7f && c[1] == 0x7e && c[2] == 0xfe);
    CHECK(c[3] == 0x7e && c[4] == 0x7e);
    CHECK(c[5] == 0 && c[6] == 0x80 && c[7] == 0);
    CHECK(orc_e4m3_encode(-448.0) == 0xfe);
  }
  free(kc);
  free(vc);
  free(q);
  free(kc16);
  free(vc16);
  free(q16);
  free(kc64);
  free(vc64);
  free(q64);
  free(tmp);
  free(kc8);
  free(vc8);
  if (failures) {
    fprintf(stderr, "%d checks failed\n", failures);
    return 1;
  }
  printf("oracle under sanitizers: ok\n");
  return 0;
}
