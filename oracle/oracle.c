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
 * All inputs are bf16 bit patterns (uint16), widened exactly to double.
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

/* Address of element d of KV head `kv` in cache slot `slot` of sequence b.
 * Cache layout: sequence b starts at b * batch_stride elements; within it
 * [C][Hkv][D] token-major, D contiguous. */
static const uint16_t *kv_row(const uint16_t *cache, int64_t batch_stride, int32_t Hkv, int32_t D,
                              int32_t b, int32_t slot, int32_t kv) {
  return cache + (int64_t)b * batch_stride + ((int64_t)slot * Hkv + kv) * D;
}

int oracle_version(void) { return 1 + 1000 * ORACLE_MUTATION; }

/*
 * Attention of every query head over an explicit logical position range
 * [lo[b], hi[b]) per sequence.  An empty range yields LSE = -inf and out = 0.
 * q: [B][Hq][D]; k, v: caches as above (v ignored when kv_shared != 0);
 * out: [B][Hq][D] doubles; lse: [B][Hq] doubles.  Returns 0, or -1 on bad input.
 */
int oracle_attend(const uint16_t *q, const uint16_t *k, const uint16_t *v, int32_t B, int32_t Hq,
                  int32_t Hkv, int32_t D, int32_t C, int64_t batch_stride, const int32_t *lo,
                  const int32_t *hi, double softcap, double scale, int32_t kv_shared, double *out,
                  double *lse) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || C <= 0 || Hq % Hkv != 0) return -1;
  if (!kv_shared && v == NULL) return -1;
  const int32_t G = Hq / Hkv;
  const uint16_t *vals = kv_shared ? k : v;
#if ORACLE_MUTATION == 6
  vals = k; /* values taken from K even when a separate V exists */
#endif
  for (int32_t b = 0; b < B; ++b) {
    const int32_t n = hi[b] - lo[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!s) return -1;
    for (int32_t h = 0; h < Hq; ++h) {
      int32_t kv = h / G;
#if ORACLE_MUTATION == 2
      kv = h % Hkv; /* interleaved instead of contiguous GQA groups */
#endif
      const uint16_t *qh = q + ((int64_t)b * Hq + h) * D;
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
        const uint16_t *kr = kv_row(k, batch_stride, Hkv, D, b, slot, kv);
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(kr[d]);
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
        const uint16_t *vr = kv_row(vals, batch_stride, Hkv, D, b, slot, kv);
        for (int32_t d = 0; d < D; ++d) o[d] += p * bf16_to_double(vr[d]);
      }
    }
    free(s);
  }
  return 0;
}

/*
 * Decode attention for one layer: the position range follows from the context
 * length L_b (current token included) and the window.  window == 0 attends the
 * whole context.  Returns -1 when a range needs more slots than the cache has.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const int32_t *seqlens,
                  int32_t B, int32_t Hq, int32_t Hkv, int32_t D, int32_t C, int64_t batch_stride,
                  int32_t window, double softcap, double scale, int32_t kv_shared, double *out,
                  double *lse) {
  int32_t *lo = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  int32_t *hi = (int32_t *)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1));
  if (!lo || !hi) {
    free(lo);
    free(hi);
    return -1;
  }
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
  if (rc == 0)
    rc = oracle_attend(q, k, v, B, Hq, Hkv, D, C, batch_stride, lo, hi, softcap, scale, kv_shared,
                       out, lse);
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
  double L = m + log(z);
  *lse = L;
  for (int32_t s = 0; s < n; ++s) {
    if (lse_parts[s] == -INFINITY) continue;
    double w = exp(lse_parts[s] - L);
    for (int32_t d = 0; d < D; ++d) out[d] += w * o_parts[(int64_t)s * D + d];
  }
}
