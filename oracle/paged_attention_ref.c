/*
 * Oracle for paged decode attention, in float64.  TEST INFRASTRUCTURE ONLY:
 * this file is compiled into liboracle.so, which only the tests, the smoke
 * check and the CPU-baseline leg of the benchmark load.  The product path
 * never calls it and shares no code, header or constant with it.
 *
 * What it follows:
 *  - "PagedAttention Internals" (wondering.app), section "The Block Table Map":
 *    a sequence's logical block n lives in whatever physical block the
 *    sequence's block table names; the attention step reads keys and values
 *    through that table, and the logical order of tokens is kept.
 *  - "pagedattention" glossary entry (chipfoundryservices.com), paragraph 3
 *    (block tables): fixed-size blocks (16 tokens as the example), one table
 *    per request, and the attention kernel gathers keys and values through it.
 *  - The attention itself is the textbook scaled dot-product decode step
 *    (the pages state no formula): for one query vector q and the keys and
 *    values of tokens 0..n-1,
 *        s_t   = scale * <q, k_t>
 *        out   = sum_t exp(s_t - max_s) v_t / sum_t exp(s_t - max_s)
 *    computed as a plain two-pass softmax, no partitions, no online rescale.
 *  - Grouped query heads: query head h reads KV head h / (Hq / Hkv)
 *    (contiguous groups; the pages are silent, this is the plainest reading).
 *
 * Cache layout (part of the call contract, not of the math):
 *   k_cache, v_cache : [num_blocks][Hkv][bs][D], element (blk, g, off, d) at
 *   ((blk * Hkv + g) * bs + off) * D + d.
 * Token t of sequence b is at blk = table[b][t / bs], off = t % bs.
 *
 * Element types: 0 = float32, 1 = bfloat16 (raw 16-bit patterns, the upper
 * half of a float32), 2 = float64.  Every value is widened to double before
 * any arithmetic.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

static double orc_load(const void *base, int dtype, int64_t i) {
  if (dtype == ORC_F32) return (double)((const float *)base)[i];
  if (dtype == ORC_BF16) {
    uint32_t u = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
  }
  return ((const double *)base)[i];
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Checks the shapes and every table entry a sequence uses. 0 = fine. */
static int orc_check(int64_t num_blocks, int Hkv, int bs, int D, const int32_t *tables,
                     int max_blocks, const int32_t *lens, int B, int Hq) {
  if (Hkv <= 0 || bs <= 0 || D <= 0 || B < 0 || Hq <= 0) return 1;
  if (Hq % Hkv != 0) return 2;
  for (int b = 0; b < B; ++b) {
    int n = lens[b];
    if (n < 0) return 3;
    int nblk = (n + bs - 1) / bs;
    if (nblk > max_blocks) return 4;
    for (int j = 0; j < nblk; ++j) {
      int32_t blk = tables[(int64_t)b * max_blocks + j];
      if (blk < 0 || blk >= num_blocks) return 5;
    }
  }
  return 0;
}

/* Offset of element (token t of sequence b, kv head g, dim 0) in a cache. */
static int64_t orc_row(const int32_t *tables, int max_blocks, int b, int t, int Hkv, int bs,
                       int D, int g) {
  int64_t blk = tables[(int64_t)b * max_blocks + t / bs];
  int off = t % bs;
  return ((blk * Hkv + g) * bs + off) * (int64_t)D;
}

/* One output row: query head h of sequence b over its whole context. */
static void orc_one_row(const void *q, const void *k_cache, const void *v_cache, int dtype,
                        int Hkv, int bs, int D, const int32_t *tables, int max_blocks,
                        const int32_t *lens, int Hq, double scale, int b, int h,
                        double *out_row) {
  int G = Hq / Hkv;
  int g = h / G;
  int n = lens[b];
  for (int d = 0; d < D; ++d) out_row[d] = 0.0;
  if (n == 0) return;
  double *s = (double *)malloc(sizeof(double) * (size_t)n);
  const int64_t qoff = ((int64_t)b * Hq + h) * D;
  /* pass 1: logits and their maximum */
  double m = -INFINITY;
  for (int t = 0; t < n; ++t) {
    int64_t kr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += orc_load(q, dtype, qoff + d) * orc_load(k_cache, dtype, kr + d);
    s[t] = scale * dot;
    if (s[t] > m) m = s[t];
  }
  /* pass 2: weights, their sum and the weighted sum of values */
  double denom = 0.0;
  for (int t = 0; t < n; ++t) {
    double p = exp(s[t] - m);
    denom += p;
    int64_t vr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
    for (int d = 0; d < D; ++d) out_row[d] += p * orc_load(v_cache, dtype, vr + d);
  }
  for (int d = 0; d < D; ++d) out_row[d] /= denom;
  free(s);
}

/*
 * Decode attention for every (b, h), or for the listed rows only.
 *   q   : [B][Hq][D] of `dtype`
 *   out : [B][Hq][D] float64 when rows == NULL, else [n_rows][D] with
 *         rows[2*i] = b, rows[2*i+1] = h.
 * Returns 0, or a nonzero code for malformed input (nothing written).
 */
int oracle_decode(const void *q, const void *k_cache, const void *v_cache, int dtype,
                  int64_t num_blocks, int Hkv, int bs, int D, const int32_t *tables,
                  int max_blocks, const int32_t *lens, int B, int Hq, double scale,
                  const int32_t *rows, int n_rows, double *out) {
  int rc = orc_check(num_blocks, Hkv, bs, D, tables, max_blocks, lens, B, Hq);
  if (rc) return rc;
  int64_t total = rows ? (int64_t)n_rows : (int64_t)B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < total; ++i) {
    int b, h;
    if (rows) {
      b = rows[2 * i];
      h = rows[2 * i + 1];
    } else {
      b = (int)(i / Hq);
      h = (int)(i % Hq);
    }
    orc_one_row(q, k_cache, v_cache, dtype, Hkv, bs, D, tables, max_blocks, lens, Hq, scale, b,
                h, out + i * D);
  }
  return 0;
}

/*
 * The split-context form: the context of each sequence is cut into
 * partitions of `part` tokens; partition p of row (b, h) holds tokens
 * [p*part, min((p+1)*part, n)).  For each it writes, over its own tokens,
 *   m_p = max s_t,   l_p = sum exp(s_t - m_p),   acc_p = sum exp(s_t - m_p) v_t
 * into m[(b*Hq+h)*P + p], l[...] and acc[((b*Hq+h)*P + p)*D + d], where
 * P = max_parts.  Partitions past the end of a sequence are left untouched.
 */
int oracle_decode_partials(const void *q, const void *k_cache, const void *v_cache, int dtype,
                           int64_t num_blocks, int Hkv, int bs, int D, const int32_t *tables,
                           int max_blocks, const int32_t *lens, int B, int Hq, double scale,
                           int part, int max_parts, double *m_out, double *l_out,
                           double *acc_out) {
  int rc = orc_check(num_blocks, Hkv, bs, D, tables, max_blocks, lens, B, Hq);
  if (rc) return rc;
  if (part <= 0) return 6;
  for (int b = 0; b < B; ++b)
    if ((lens[b] + part - 1) / part > max_parts) return 7;
  int G = Hq / Hkv;
  int64_t total = (int64_t)B * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < total; ++i) {
    int b = (int)(i / Hq), h = (int)(i % Hq), g = h / G;
    int n = lens[b];
    int np = (n + part - 1) / part;
    const int64_t qoff = ((int64_t)b * Hq + h) * D;
    for (int p = 0; p < np; ++p) {
      int t0 = p * part, t1 = t0 + part < n ? t0 + part : n;
      double *s = (double *)malloc(sizeof(double) * (size_t)(t1 - t0));
      double m = -INFINITY;
      for (int t = t0; t < t1; ++t) {
        int64_t kr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
          dot += orc_load(q, dtype, qoff + d) * orc_load(k_cache, dtype, kr + d);
        s[t - t0] = scale * dot;
        if (s[t - t0] > m) m = s[t - t0];
      }
      double l = 0.0;
      double *acc = acc_out + (i * max_parts + p) * D;
      for (int d = 0; d < D; ++d) acc[d] = 0.0;
      for (int t = t0; t < t1; ++t) {
        double w = exp(s[t - t0] - m);
        l += w;
        int64_t vr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
        for (int d = 0; d < D; ++d) acc[d] += w * orc_load(v_cache, dtype, vr + d);
      }
      m_out[i * max_parts + p] = m;
      l_out[i * max_parts + p] = l;
      free(s);
    }
  }
  return 0;
}

/*
 * Merges the partials of oracle_decode_partials (the log-sum-exp combine):
 *   M = max_p m_p,  L = sum_p l_p exp(m_p - M),  out = sum_p acc_p exp(m_p - M) / L
 * nparts[i] partitions are used for row i; a row with none gets zeros.
 */
void oracle_merge_partials(const double *m, const double *l, const double *acc,
                           const int32_t *nparts, int64_t n_rows, int max_parts, int D,
                           double *out) {
  for (int64_t i = 0; i < n_rows; ++i) {
    double *o = out + i * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    int np = nparts[i];
    if (np == 0) continue;
    double M = -INFINITY;
    for (int p = 0; p < np; ++p)
      if (m[i * max_parts + p] > M) M = m[i * max_parts + p];
    double L = 0.0;
    for (int p = 0; p < np; ++p) {
      double w = exp(m[i * max_parts + p] - M);
      L += l[i * max_parts + p] * w;
      for (int d = 0; d < D; ++d) o[d] += acc[(i * max_parts + p) * D + d] * w;
    }
    for (int d = 0; d < D; ++d) o[d] /= L;
  }
}

/*
 * Paged prefill (chunked-prefill) attention.  Sequence b holds lens[b]
 * tokens in the cache; the last n_b = qstart[b+1] - qstart[b] of them are
 * its new tokens, whose queries are rows qstart[b] .. qstart[b+1]-1 of q.
 * New token i sits at position p = lens[b] - n_b + i and attends to the
 * sequence's tokens 0..p only (causal), through the block table:
 *   s_t = scale * <q[qstart[b] + i, h], k_t>,   t = 0..p
 *   out[qstart[b] + i, h] = sum_t exp(s_t - max_s) v_t / sum_t exp(s_t - max_s)
 * the same textbook step as the decode, here for every new token (the decode
 * is the case n_b = 1).  Two-pass softmax in float64, no tiling.
 *   q   : [total][Hq][D] of `dtype`, total = qstart[B]
 *   out : [total][Hq][D] float64 when rows == NULL, else [n_rows][D] with
 *         rows[2*i] = query row j (0 <= j < total), rows[2*i+1] = h.
 * Returns 0, or a nonzero code for malformed input (nothing written).
 */
int oracle_prefill(const void *q, const void *k_cache, const void *v_cache, int dtype,
                   int64_t num_blocks, int Hkv, int bs, int D, const int32_t *tables,
                   int max_blocks, const int32_t *lens, const int32_t *qstart, int B, int Hq,
                   double scale, const int32_t *rows, int n_rows, double *out) {
  int rc = orc_check(num_blocks, Hkv, bs, D, tables, max_blocks, lens, B, Hq);
  if (rc) return rc;
  if (qstart[0] != 0) return 8;
  for (int b = 0; b < B; ++b) {
    int n = qstart[b + 1] - qstart[b];
    if (n < 0 || n > lens[b]) return 9;
  }
  const int64_t total_q = qstart[B];
  const int G = Hq / Hkv;
  int64_t total = rows ? (int64_t)n_rows : total_q * Hq;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < total; ++i) {
    int64_t j;
    int h;
    if (rows) {
      j = rows[2 * i];
      h = rows[2 * i + 1];
    } else {
      j = i / Hq;
      h = (int)(i % Hq);
    }
    double *o = out + i * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (j < 0 || j >= total_q || h < 0 || h >= Hq) continue;
    int b = 0;  /* the sequence whose query rows hold j */
    while (qstart[b + 1] <= j) ++b;
    const int n = qstart[b + 1] - qstart[b];
    const int p = lens[b] - n + (int)(j - qstart[b]);
    const int g = h / G;
    const int64_t qoff = (j * Hq + h) * D;
    double *s = (double *)malloc(sizeof(double) * (size_t)(p + 1));
    double m = -INFINITY;
    for (int t = 0; t <= p; ++t) {
      int64_t kr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += orc_load(q, dtype, qoff + d) * orc_load(k_cache, dtype, kr + d);
      s[t] = dot * scale;
      if (s[t] > m) m = s[t];
    }
    double denom = 0.0;
    for (int t = 0; t <= p; ++t) {
      double w = exp(s[t] - m);
      denom += w;
      int64_t vr = orc_row(tables, max_blocks, b, t, Hkv, bs, D, g);
      for (int d = 0; d < D; ++d) o[d] += w * orc_load(v_cache, dtype, vr + d);
    }
    for (int d = 0; d < D; ++d) o[d] /= denom;
    free(s);
  }
  return 0;
}
