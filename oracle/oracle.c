/*
 * Float64 CPU oracle for single-token decode attention over a per-layer KV
 * cache.  TEST INFRASTRUCTURE ONLY: the library never links, loads or calls this
 * file; only the tests, the package smoke check and the bench's CPU-baseline leg
 * do.  It shares no source with the CUDA path.
 *
 * What it computes is the plain definition, in the order the pages give it,
 * with no splitting, tiling or reordering:
 *
 *   kv   = h / (Hq / Hkv)                       contiguous GQA groups
 *   [lo, hi) = [max(0, L - w), L) for a sliding layer (w > 0), [0, L) otherwise
 *   slot = j mod C                              ring-buffer cache slot
 *   x_j  = scale * <q_h, k_{kv, slot}>
 *   s_j  = softcap * tanh(x_j / softcap)        when softcap > 0
 *   LSE  = log sum_j exp(s_j)                   natural log
 *   out  = sum_j exp(s_j - LSE) * v'_{kv, slot},   v' = K when K serves as V
 *
 * Sources: the window ("reads exactly w KV entries") and the ring cache
 * (RotatingKVCache) are from "Gemma 4 12B", serviceability join and item (6);
 * the two head geometries and key/value sharing on full layers are from
 * "Gemma4-26B-A4B ... NO-GO", section 3 Break 4, and the "Gemma support" PR
 * summary (K = V global attention, attention soft-capping, sliding-window
 * layers); the per-geometry 1/sqrt(head_dim) scale is that NO-GO note's section 5.
 * The soft-cap form cap*tanh(s/cap) applied to the scaled logit, and the
 * natural-log LSE, are the plainest readings where the pages are silent.
 *
 * Cache rows are bf16 bit patterns (uint16), widened exactly to double, or, in
 * oracle_decode_fp8, e4m3 codes times a float scale per row (the quantized
 * rotating cache of "Gemma 4 12B", serviceability join, item 6; the format and
 * scale layout are spelled out at e4m3_to_double and row_source).  q is bf16.
 *
 * Compile-time ORACLE_MUTATION=n plants one deliberate mistake (used only by the
 * test that shows the pins catch plausible mistakes); 0 (default) is the oracle.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTATION
#define ORACLE_MUTATION 0
#endif

static double bf16_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * An fp8 code in the OCP 8-bit floating point format E4M3 (the "e4m3" of the
 * fp8 KV caches the pages speak of): sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits; exponent field 0 holds the subnormals m/8 * 2^-6; no
 * infinities, and S.1111.111 is NaN (largest finite magnitude 448).
 */
static double e4m3_to_double(uint8_t code) {
  int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
  int bias = 7;
#if ORACLE_MUTATION == 9
  bias = 8; /* exponent bias off by one */
#endif
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp((double)m / 8.0, 1 - bias) : ldexp(1.0 + (double)m / 8.0, e - bias);
#if ORACLE_MUTATION == 17
  if (e == 0) mag = ldexp(1.0 + (double)m / 8.0, -bias); /* subnormals with a leading one */
#endif
  return sign ? -mag : mag;
}

int oracle_e4m3_to_double(uint8_t code, double *value) {
  *value = e4m3_to_double(code);
  return 0;
}

/*
 * Where the cache rows come from.  Layout of both caches: sequence b starts at
 * b * batch_stride elements; within it [C][Hkv][D] token-major, D contiguous.
 *  bf16: rows of bf16 bit patterns, widened exactly to double.
 *  fp8:  rows of e4m3 codes; row (b, kv, slot) has one float scale at
 *        scale[(b * Hkv + kv) * C + slot], and its values are code * scale
 *        (the per-row scales of a quantized rotating cache: "Gemma 4 12B",
 *        serviceability join, item 6).
 */
typedef struct row_source {
  int fp8;
  const uint16_t *k, *v;     /* bf16 */
  const uint8_t *kc, *vc;    /* fp8 codes */
  const float *ks, *vs;      /* fp8 per-row scales */
  int64_t batch_stride;
  int32_t Hkv, D, C, kv_shared;
} row_source;

/* The D values of row (b, slot, kv) of K (value == 0) or of the value tensor
 * (value == 1: V, or K when K serves as V). */
static void fetch_row(const row_source *src, int32_t b, int32_t slot, int32_t kv, int value,
                      double *row) {
  const int use_v = value && !src->kv_shared;
  const int64_t off = (int64_t)b * src->batch_stride + ((int64_t)slot * src->Hkv + kv) * src->D;
  if (!src->fp8) {
    const uint16_t *r = (use_v ? src->v : src->k) + off;
    for (int32_t d = 0; d < src->D; ++d) row[d] = bf16_to_double(r[d]);
    return;
  }
  const uint8_t *r = (use_v ? src->vc : src->kc) + off;
  const float *scales = use_v ? src->vs : src->ks;
#if ORACLE_MUTATION == 10
  scales = src->ks; /* V rows scaled by the K scales */
#endif
  int64_t si = ((int64_t)b * src->Hkv + kv) * src->C + slot;
#if ORACLE_MUTATION == 12
  si = ((int64_t)b * src->C + slot) * src->Hkv + kv; /* scales read token-major */
#endif
  double sc = (double)scales[si];
#if ORACLE_MUTATION == 11
  sc = sc * sc; /* scale applied twice */
#endif
  for (int32_t d = 0; d < src->D; ++d) row[d] = e4m3_to_double(r[d]) * sc;
}

int oracle_version(void) { return 1 + 1000 * ORACLE_MUTATION; }

/*
 * Attention of every query head over an explicit logical position range
 * [lo[b], hi[b]) per sequence, with cache rows from `src`.  An empty range
 * yields LSE = -inf and out = 0.  q: [B][Hq][D]; out: [B][Hq][D] doubles;
 * lse: [B][Hq] doubles.  Returns 0, or -1 on bad input.
 */
static int attend(const uint16_t *q, int32_t B, int32_t Hq, const int32_t *lo, const int32_t *hi,
                  double softcap, double scale, const row_source *src, double *out,
                  double *lse) {
  const int32_t Hkv = src->Hkv, D = src->D, C = src->C;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || C <= 0 || Hq % Hkv != 0) return -1;
  const int32_t G = Hq / Hkv;
  int value_tensor = 1;
#if ORACLE_MUTATION == 6
  value_tensor = 0; /* values taken from K even when a separate V exists */
#endif
  double *qd = (double *)malloc(sizeof(double) * (size_t)D);
  double *row = (double *)malloc(sizeof(double) * (size_t)D);
  if (!qd || !row) {
    free(qd);
    free(row);
    return -1;
  }
  for (int32_t b = 0; b < B; ++b) {
    const int32_t n = hi[b] - lo[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!s) {
      free(qd);
      free(row);
      return -1;
    }
    for (int32_t h = 0; h < Hq; ++h) {
      int32_t kv = h / G;
#if ORACLE_MUTATION == 2
      kv = h % Hkv; /* interleaved instead of contiguous GQA groups */
#endif
      const uint16_t *qh = q + ((int64_t)b * Hq + h) * D;
      for (int32_t d = 0; d < D; ++d) qd[d] = bf16_to_double(qh[d]);
      double *o = out + ((int64_t)b * Hq + h) * D;
      for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
      if (n <= 0) {
        lse[(int64_t)b * Hq + h] = -INFINITY;
        continue;
      }
      /* scores */
      double m = -INFINITY;
      for (int32_t j = lo[b]; j < hi[b]; ++j) {
        int32_t slot = j % C;
#if ORACLE_MUTATION == 7
        slot = (j + 1) % C; /* ring index off by one */
#endif
        fetch_row(src, b, slot, kv, 0, row);
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += qd[d] * row[d];
        double x = scale * dot;
#if ORACLE_MUTATION == 8
        x = dot; /* scale dropped */
#endif
        double sj = x;
        if (softcap > 0.0) {
          sj = softcap * tanh(x / softcap);
#if ORACLE_MUTATION == 3
          sj = scale * softcap * tanh(dot / softcap); /* cap before scale */
#endif
#if ORACLE_MUTATION == 16
          sj = tanh(x / softcap); /* outer factor cap dropped */
#endif
        }
        s[j - lo[b]] = sj;
        if (sj > m) m = sj;
      }
      /* normaliser */
      double z = 0.0;
      for (int32_t i = 0; i < n; ++i) z += exp(s[i] - m);
      double L = m + log(z);
#if ORACLE_MUTATION == 4
      L = m + log2(z); /* wrong log base */
#endif
      lse[(int64_t)b * Hq + h] = L;
      /* weighted values */
      for (int32_t j = lo[b]; j < hi[b]; ++j) {
        int32_t slot = j % C;
#if ORACLE_MUTATION == 7
        slot = (j + 1) % C;
#endif
        double p = exp(s[j - lo[b]] - L);
#if ORACLE_MUTATION == 5
        p = exp(s[j - lo[b]] - m); /* weights not normalised */
#endif
        fetch_row(src, b, slot, kv, value_tensor, row);
        for (int32_t d = 0; d < D; ++d) o[d] += p * row[d];
      }
    }
    free(s);
  }
  free(qd);
  free(row);
  return 0;
}

/* Position range [lo_b, hi_b) of one decode step: the last `window` positions
 * of the context L_b (window 0: all of it).  -1 when a range needs more slots
 * than the cache has, or L_b < 1. */
static int decode_ranges(const int32_t *seqlens, int32_t B, int32_t window, int32_t C,
                         int32_t *lo, int32_t *hi) {
  int rc = 0;
  for (int32_t b = 0; b < B; ++b) {
    int32_t L = seqlens[b];
    int32_t start = 0;
    if (window > 0 && L > window) start = L - window;
#if ORACLE_MUTATION == 1
    if (window > 0 && L > window) start = L - window + 1; /* window one short */
#endif
    lo[b] = start;
    hi[b] = L;
    if (L < 1 || L - start > C) rc = -1;
  }
  return rc;
}

static int decode_with(const int32_t *seqlens, const uint16_t *q, int32_t B, int32_t Hq,
                       int32_t window, double softcap, double scale, const row_source *src,
                       double *out, double *lse) {
  int32_t *lo = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  int32_t *hi = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  if (!lo || !hi) {
    free(lo);
    free(hi);
    return -1;
  }
  int rc = decode_ranges(seqlens, B, window, src->C, lo, hi);
  if (rc == 0) rc = attend(q, B, Hq, lo, hi, softcap, scale, src, out, lse);
  free(lo);
  free(hi);
  return rc;
}

/*
 * Attention over explicit ranges with a bf16 cache (k; v, or K as V when
 * kv_shared != 0).
 */
int oracle_attend(const uint16_t *q, const uint16_t *k, const uint16_t *v, int32_t B, int32_t Hq,
                  int32_t Hkv, int32_t D, int32_t C, int64_t batch_stride, const int32_t *lo,
                  const int32_t *hi, double softcap, double scale, int32_t kv_shared, double *out,
                  double *lse) {
  if (!kv_shared && v == NULL) return -1;
  row_source src = {0, k, v, NULL, NULL, NULL, NULL, batch_stride, Hkv, D, C, kv_shared};
  return attend(q, B, Hq, lo, hi, softcap, scale, &src, out, lse);
}

/*
 * Decode attention for one layer over a bf16 cache: the position range
 * follows from the context length L_b (current token included) and the
 * window.  window == 0 attends the whole context.  Returns -1 when a range
 * needs more slots than the cache has.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *seqlens,
                  int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t C, int64_t batch_stride,
                  int32_t window, double softcap, double scale, int32_t kv_shared, double *out,
                  double *lse) {
  if (!kv_shared && v == NULL) return -1;
  row_source src = {0, k, v, NULL, NULL, NULL, NULL, batch_stride, Hkv, D, C, kv_shared};
  return decode_with(seqlens, q, B, Hq, window, softcap, scale, &src, out, lse);
}

/*
 * oracle_decode over an fp8 cache: codes kc (vc) in e4m3 with per-row scales
 * ks (vs), [B][Hkv][C] floats; values are code * scale.  vc and vs are ignored
 * when kv_shared != 0 (K, with its scales, serves as V).
 */
int oracle_decode_fp8(const uint16_t *q, const uint8_t *kc, const uint8_t *vc, const float *ks,
                      const float *vs, const int32_t *seqlens, int32_t B, int32_t Hq, int32_t Hkv,
                      int32_t D, int32_t C, int64_t batch_stride, int32_t window, double softcap,
                      double scale, int32_t kv_shared, double *out, double *lse) {
  if (!kv_shared && (vc == NULL || vs == NULL)) return -1;
  row_source src = {1, NULL, NULL, kc, vc, ks, vs, batch_stride, Hkv, D, C, kv_shared};
  return decode_with(seqlens, q, B, Hq, window, softcap, scale, &src, out, lse);
}

/*
 * Multi-query decode over a bf16 cache: T query tokens per sequence, the
 * sequence's last T positions.  Query t of sequence b sits at position
 * p = L_b - T + t and attends [max(0, p + 1 - window), p + 1) (window 0: [0, p + 1)),
 * causally, as a speculative-decoding verify step does.  q: [T][B][Hq][D]; out:
 * [T][B][Hq][D]; lse: [T][B][Hq].  Returns -1 when a query's range is empty, or
 * reaches a position the ring no longer holds (older than L_b - C).
 */
int oracle_decode_multi(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *seqlens, int32_t T, int32_t B, int32_t Hq, int32_t Hkv,
                        int32_t D, int32_t C, int64_t batch_stride, int32_t window, double softcap,
                        double scale, int32_t kv_shared, double *out, double *lse) {
  if (T < 1 || B < 0) return -1;
  if (!kv_shared && v == NULL) return -1;
  int32_t *lo = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  int32_t *hi = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  if (!lo || !hi) {
    free(lo);
    free(hi);
    return -1;
  }
  row_source src = {0, k, v, NULL, NULL, NULL, NULL, batch_stride, Hkv, D, C, kv_shared};
  int rc = 0;
  for (int32_t t = 0; t < T && rc == 0; ++t) {
    for (int32_t b = 0; b < B; ++b) {
      const int32_t L = seqlens[b];
      int32_t end = L - T + t + 1; /* one past this query's position */
#if ORACLE_MUTATION == 13
      end = L; /* every query sees all T new tokens (not causal) */
#endif
      int32_t start = (window > 0 && end > window) ? end - window : 0;
#if ORACLE_MUTATION == 18
      if (window > 0 && end > window) start = end - window + 1; /* window one short */
#endif
      lo[b] = start;
      hi[b] = end;
      if (end < 1 || start < L - C) rc = -1;
    }
    if (rc == 0)
      rc = attend(q + (int64_t)t * B * Hq * D, B, Hq, lo, hi, softcap, scale, &src,
                  out + (int64_t)t * B * Hq * D, lse + (int64_t)t * B * Hq);
  }
  free(lo);
  free(hi);
  return rc;
}

/*
 * Merge n partial results of one query head, each normalised over its own part
 * of the position range: LSE = log sum_s exp(LSE_s), out = sum_s exp(LSE_s - LSE) o_s.
 * Parts with LSE_s = -inf contribute nothing; if all are -inf the result is
 * LSE = -inf, out = 0.  o_parts: [n][D]; out: [D].
 */
void oracle_combine(const double *o_parts, const double *lse_parts, int32_t n, int32_t D,
                    double *out, double *lse) {
  double m = -INFINITY;
  for (int32_t s = 0; s < n; ++s)
    if (lse_parts[s] > m) m = lse_parts[s];
  for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double z = 0.0;
  for (int32_t s = 0; s < n; ++s) z += exp(lse_parts[s] - m);
#if ORACLE_MUTATION == 14
  double L = m;
#else
  double L = m + log(z);
#endif
  *lse = L;
  for (int32_t s = 0; s < n; ++s) {
    if (lse_parts[s] == -INFINITY) continue;
#if ORACLE_MUTATION == 15
    double w = exp(lse_parts[s] - m);
#else
    double w = exp(lse_parts[s] - L);
#endif
    for (int32_t d = 0; d < D; ++d) out[d] += w * o_parts[(int64_t)s * D + d];
  }
}
