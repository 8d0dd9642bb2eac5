// Log-sum-exp merge of split-KV partial results.
//
// Each part s of a (sequence, head) holds o_s (normalised over its own
// positions) and lse_s; the merged result is
//   lse = log sum_s exp(lse_s),   out = sum_s exp(lse_s - lse) * o_s,
// with empty parts (lse_s = -inf) contributing nothing.  One CTA per
// (unit or sequence, head); a thread owns 4 consecutive elements of D.
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
};

constexpr int kCombineThreads = 128;

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
  chunk = total > 0 ? ceil_div64(total, g.nchunks) : 1;
}

template <bool INTERNAL>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  extern __shared__ __align__(16) float wts[];  // [n_parts] weights, then [NG][NC] float4
  __shared__ int64_t sh_slot0;
  __shared__ int32_t sh_nparts;

  grid_launch_dependents();
  grid_dependency_wait();

  int32_t b, h;
  const int32_t hh = blockIdx.y;
  if (INTERNAL) {
    const int32_t u = blockIdx.x;
    b = u / p.geo.units_per_seq;
    const int32_t x = u - b * p.geo.units_per_seq;
    h = x * p.heads_per_unit + hh;
    if (threadIdx.x < 32) {
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

  // Max of the parts' lse, then weights exp(lse_s - max) and their sum.
  float mx = -INFINITY;
  for (int32_t s = threadIdx.x; s < np; s += blockDim.x) {
    const float v = l_base[s * l_stride];
    wts[s] = v;
    mx = fmaxf(mx, v);
  }
  __shared__ float red[kCombineThreads / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int w = 1; w < kCombineThreads / 32; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float z = 0.f;
  for (int32_t s = threadIdx.x; s < np; s += blockDim.x) {
    const float v = wts[s];
    const float e = (v == -INFINITY) ? 0.f : __expf(v - mx);
    wts[s] = e;
    z += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = z;
  __syncthreads();
  z = 0.f;
  for (int w = 0; w < kCombineThreads / 32; ++w) z += red[w];
  const bool empty = (mx == -INFINITY);
  const float inv_z = empty ? 0.f : 1.f / z;

  // Thread t owns float4 column (t mod NC) and parts t / NC, t / NC + NG, ...;
  // loads are issued kUnroll at a time so each thread keeps several in flight.
  uint16_t *dst = p.out + (static_cast<int64_t>(b) * p.n_q_heads + h) * D;
  const int NC = D / 4;
  const int NG = NC >= kCombineThreads ? 1 : kCombineThreads / NC;
  const int grp = threadIdx.x / NC;
  float4 *part_acc = reinterpret_cast<float4 *>(wts + ((np + 3) & ~3));  // [NG][NC]
  for (int d4 = threadIdx.x % NC; d4 < NC; d4 += kCombineThreads) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (!empty && grp < NG) {
      constexpr int kUnroll = 8;
      int32_t s = grp;
      for (; s + (kUnroll - 1) * NG < np; s += kUnroll * NG) {
        float4 v[kUnroll];
        float wv[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          v[u] = *reinterpret_cast<const float4 *>(o_base + (s + u * NG) * o_stride + 4 * d4);
          wv[u] = wts[s + u * NG];
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          // an empty part has weight 0 and may hold anything: select, don't multiply
          if (wv[u] != 0.f) {
            acc.x = fmaf(wv[u], v[u].x, acc.x);
            acc.y = fmaf(wv[u], v[u].y, acc.y);
            acc.z = fmaf(wv[u], v[u].z, acc.z);
            acc.w = fmaf(wv[u], v[u].w, acc.w);
          }
        }
      }
      for (; s < np; s += NG) {
        const float w = wts[s];
        if (w != 0.f) {
          const float4 v = *reinterpret_cast<const float4 *>(o_base + s * o_stride + 4 * d4);
          acc.x = fmaf(w, v.x, acc.x);
          acc.y = fmaf(w, v.y, acc.y);
          acc.z = fmaf(w, v.z, acc.z);
          acc.w = fmaf(w, v.w, acc.w);
        }
      }
    }
    if (NG > 1) {
      if (grp < NG) part_acc[grp * NC + d4] = acc;
      __syncthreads();
      if (grp == 0) {
        for (int g2 = 1; g2 < NG; ++g2) {
          const float4 o = part_acc[g2 * NC + d4];
          acc.x += o.x;
          acc.y += o.y;
          acc.z += o.z;
          acc.w += o.w;
        }
      }
    }
    if (grp == 0) {
      uint2 pk;
      pk.x = pack_bf16x2(acc.x * inv_z, acc.y * inv_z);
      pk.y = pack_bf16x2(acc.z * inv_z, acc.w * inv_z);
      *reinterpret_cast<uint2 *>(dst + 4 * d4) = pk;
    }
  }
  if (threadIdx.x == 0 && p.lse != nullptr)
    p.lse[static_cast<int64_t>(b) * p.n_q_heads + h] = empty ? -INFINITY : mx + logf(z);
}

}  // namespace gdattn
