// Log-sum-exp merge of split-KV partial results.
//
// Each part s of a (sequence, head) holds o_s (normalised over its own
// positions) and lse_s; the merged result is
//   lse = log sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * o_s,
// with empty parts (lse_s = -inf) contributing nothing.
//
// One CTA per (unit or sequence, head); a thread owns one float4 column of D.
// The merge is a single pass over the parts with a running maximum; the
// parts' LSE and O loads do not depend on one another, so they are issued
// kBatch parts at a time and the cost after the decode kernel completes is a
// few L2 round trips.  Where the parts sit is worked out from seqlens before
// waiting on the decode kernel (programmatic dependent launch).
#pragma once

#include <cstdint>

#include "partition.cuh"
#include "ptx.cuh"

namespace gdattn {

struct CombineParams {
  const float *parts_o;
  const float *parts_lse;
  uint16_t *out;           // [B, Hq, D]
  float *lse;              // [B, Hq] or null
  int32_t n_q_heads;
  int32_t head_dim;
  // Internal (workspace) layout: parts of unit u in slots c_first+u .. c_last+u,
  // each slot [heads_per_unit][D]; the split is recomputed from geo.
  Geometry geo;
  int32_t heads_per_unit;
  // Caller layout: o [B, Hq, n_splits, D], lse [B, Hq, n_splits].
  int32_t n_splits;
  // Internal layout with units cut into split_k parts (> 1): unit u's parts are
  // in slots u * split_k + u .. + split_k - 1, empty ones with LSE -inf.
  int32_t split_k;
  // Internal layout of a multi-token step (> 0): row r of a unit is query token
  // r / (heads_per_unit / tokens) of head r % (heads_per_unit / tokens), and
  // out / lse are token-major [tokens][B][Hq].
  int32_t tokens;
};

// Threads per combine CTA: one float4 column of D each, whole warps.
__host__ __device__ constexpr int combine_threads(int head_dim) {
  return (head_dim / 4 + 31) / 32 * 32;
}

// Flattened start of unit (b, x) and the split chunk size, from seqlens.
__device__ void unit_position(const Geometry &g, int32_t b, int32_t x, int64_t &unit_start,
                              int32_t &n, int64_t &chunk) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  int64_t before = 0, total = 0;
  for (int32_t bb = lane; bb < g.batch; bb += 32) {
    const int64_t span =
        static_cast<int64_t>(attended_count(__ldg(g.seqlens + bb), g.window, g.capacity, bad)) *
        g.units_per_seq;
    total += span;
    if (bb < b) before += span;
  }
  total = warp_sum_i64(total);
  before = warp_sum_i64(before);
  n = attended_count(__ldg(g.seqlens + b), g.window, g.capacity, bad);
  unit_start = before + static_cast<int64_t>(x) * n;
  chunk = total > 0 ? ceil_div64(ceil_div64(total, geo_nchunks(g)), geo_align(g)) * geo_align(g)
                    : 1;
}

// Merges np parts for NC float4 columns at once: for column c, part s holds
// o at o_col[c] + s * o_stride (4 floats) and lse at l_col[c][s * l_stride].
// The loads of kBatch parts for all NC columns are issued together; a running
// maximum rescales the sums between batches.  res[c] is the normalised column;
// m[c] and z[c] end as the max and the sum of exp(lse_s - m), so lse = m + log z
// (m = -inf when every part is empty).  load_o = false skips the O loads.
template <int NC, int kBatch>
__device__ __forceinline__ void merge_columns(const float *const (&o_col)[NC],
                                              const float *const (&l_col)[NC], int64_t o_stride,
                                              int64_t l_stride, int32_t np, bool load_o,
                                              float4 (&res)[NC], float (&m)[NC], float (&z)[NC]) {
  float4 acc[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    m[c] = -INFINITY;
    z[c] = 0.f;
    acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int32_t s0 = 0; s0 < np; s0 += kBatch) {
    float lv[NC][kBatch];
    float4 ov[NC][kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const bool in = s0 + q < np;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        lv[c][q] = in ? __ldcg(l_col[c] + (s0 + q) * l_stride) : -INFINITY;
        ov[c][q] = (in && load_o)
                       ? __ldcg(reinterpret_cast<const float4 *>(o_col[c] + (s0 + q) * o_stride))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      float bm = m[c];
#pragma unroll
      for (int q = 0; q < kBatch; ++q) bm = fmaxf(bm, lv[c][q]);
      if (bm == -INFINITY) continue;  // only empty parts so far
      const float r = (m[c] == -INFINITY) ? 0.f : __expf(m[c] - bm);
      z[c] *= r;
      acc[c].x *= r;
      acc[c].y *= r;
      acc[c].z *= r;
      acc[c].w *= r;
#pragma unroll
      for (int q = 0; q < kBatch; ++q) {
        // an empty part has weight 0 and may hold anything: select, don't multiply
        if (lv[c][q] == -INFINITY) continue;
        const float w = __expf(lv[c][q] - bm);
        z[c] += w;
        acc[c].x = fmaf(w, ov[c][q].x, acc[c].x);
        acc[c].y = fmaf(w, ov[c][q].y, acc[c].y);
        acc[c].z = fmaf(w, ov[c][q].z, acc[c].z);
        acc[c].w = fmaf(w, ov[c][q].w, acc[c].w);
      }
      m[c] = bm;
    }
  }
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const float inv_z = (m[c] == -INFINITY) ? 0.f : __fdividef(1.f, z[c]);
    res[c] = make_float4(acc[c].x * inv_z, acc[c].y * inv_z, acc[c].z * inv_z, acc[c].w * inv_z);
  }
}

// One column (see merge_columns).
template <int kBatch>
__device__ __forceinline__ float4 merge_column(const float *o_base, int64_t o_stride,
                                               const float *l_base, int64_t l_stride, int32_t np,
                                               bool load_o, float &m, float &z) {
  const float *const o_col[1] = {o_base};
  const float *const l_col[1] = {l_base};
  float4 res[1];
  float mm[1], zz[1];
  merge_columns<1, kBatch>(o_col, l_col, o_stride, l_stride, np, load_o, res, mm, zz);
  m = mm[0];
  z = zz[0];
  return res[0];
}

__device__ __forceinline__ void store_bf16x4(uint16_t *dst, float4 v) {
  uint2 pk;
  pk.x = pack_bf16x2(v.x, v.y);
  pk.y = pack_bf16x2(v.z, v.w);
  *reinterpret_cast<uint2 *>(dst) = pk;
}

template <bool INTERNAL>
__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  constexpr int kBatch = 16;
  __shared__ int64_t sh_slot0;
  __shared__ int32_t sh_nparts;

  grid_launch_dependents();
  int32_t b, h;
  const int32_t hh = blockIdx.y;
  if (INTERNAL) {
    // seqlens do not change while the decode kernel runs: locate the parts first.
    const int32_t u = blockIdx.x;
    b = u / p.geo.units_per_seq;
    const int32_t x = u - b * p.geo.units_per_seq;
    h = x * p.heads_per_unit + hh;
    if (p.split_k > 1) {
      if (threadIdx.x == 0) {
        sh_nparts = p.split_k;
        sh_slot0 = static_cast<int64_t>(u) * p.split_k + u;
      }
    } else if (threadIdx.x < 32) {
      int64_t ustart, chunk;
      int32_t n;
      unit_position(p.geo, b, x, ustart, n, chunk);
      if (threadIdx.x == 0) {
        int32_t cf = 0, cl = 0;
        if (n > 0) unit_chunks(ustart, n, chunk, cf, cl);
        sh_nparts = (n > 0 && cl > cf) ? (cl - cf + 1) : 0;  // 0: written by the decode kernel
        sh_slot0 = static_cast<int64_t>(cf) + u;
      }
    }
    __syncthreads();
  } else {
    b = blockIdx.x;
    h = hh;
    if (threadIdx.x == 0) {
      sh_nparts = p.n_splits;
      sh_slot0 = 0;
    }
    __syncthreads();
  }
  const int32_t np = sh_nparts;
  if (np == 0) return;
  grid_dependency_wait();  // the parts come from the preceding kernel
  const int32_t D = p.head_dim;

  // Part s of this (b, h): o at o_base + s * o_stride, lse at l_base + s * l_stride.
  const float *o_base;
  const float *l_base;
  int64_t o_stride, l_stride;
  if (INTERNAL) {
    o_stride = static_cast<int64_t>(p.heads_per_unit) * D;
    l_stride = p.heads_per_unit;
    o_base = p.parts_o + (sh_slot0 * p.heads_per_unit + hh) * D;
    l_base = p.parts_lse + sh_slot0 * p.heads_per_unit + hh;
  } else {
    o_stride = D;
    l_stride = 1;
    o_base = p.parts_o + (static_cast<int64_t>(b) * p.n_q_heads + h) * np * D;
    l_base = p.parts_lse + (static_cast<int64_t>(b) * p.n_q_heads + h) * np;
  }

  int64_t orow = static_cast<int64_t>(b) * p.n_q_heads + h;  // output row of (b, h)
  if (INTERNAL && p.tokens > 0) {
    const int32_t gq = p.heads_per_unit / p.tokens;  // query heads of the unit
    const int32_t t = hh / gq;
    orow = (static_cast<int64_t>(t) * p.geo.batch + b) * p.n_q_heads + (h - hh) / p.heads_per_unit * gq +
           hh % gq;
  }
  uint16_t *dst = p.out + orow * D;
  const int d = 4 * threadIdx.x;
  const bool owner = d < D;
  float m, z;
  const float4 v = merge_column<kBatch>(o_base + (owner ? d : 0), o_stride, l_base, l_stride, np,
                                        owner, m, z);
  if (owner) store_bf16x4(dst + d, v);
  if (threadIdx.x == 0 && p.lse != nullptr)
    p.lse[orow] = (m == -INFINITY) ? -INFINITY : m + logf(z);
}

}  // namespace gdattn
