// Split-KV decode attention on CUDA cores, for small GQA groups (G = Hq/Hkv in
// {1, 2, 4}) such as Gemma-4 sliding layers (16 q heads over 8 KV heads, G = 2).
//
// With G <= 4 a KV row feeds at most 4 query heads, 1-2 flop per byte: not a
// dense contraction, so the products run as fp32 FMAs (packed two per
// instruction with Blackwell's fma.rn.f32x2) and the kernel is bound by HBM.
//
// CTA = 8 compute warps + 1 producer warp, one CTA per SM.  The producer streams
// whole token rows (all Hkv heads, contiguous in the token-major cache) with
// 1-D bulk copies into an NSTAGE-deep shared-memory ring, one mbarrier pair per
// stage.  Compute warp w owns KV head w % Hkv and, when Hkv < 8, every
// (8/Hkv)-th token of a stage.  A lane holds D/32 elements (16-byte chunks
// 256 * j + 8 * lane) of q, of the output accumulator and of each K/V row it
// reads, so shared-memory reads are conflict-free 16-byte vectors.
//
// Per stage a warp handles TPW tokens: it forms TPW*G partial dot products per
// lane, reduce-scatters them across the warp (each lane ends with one full
// score), applies scale / soft-cap, updates the running max and sum of the online
// softmax, broadcasts the weights and accumulates P.V.
#pragma once

#include <cstdint>

#include "partition.cuh"
#include "ptx.cuh"

namespace gdattn {

struct CoreParams {
  const uint16_t *q;      // [B, Hq, D]
  const uint16_t *k;      // cache
  const uint16_t *v;      // cache (== k when shared)
  int64_t batch_stride;   // elements
  uint16_t *out;          // [B, Hq, D]
  float *lse;             // [B, Hq] or null
  float *ws_o;            // partial outputs [slots][Hq][D]
  float *ws_lse;          // partial lse [slots][Hq]
  uint32_t *status;       // device status word
  // Current-token append (k_new non-null): the token row ([Hkv][D] of k_new /
  // v_new, [B][Hkv][D]) is copied into slot (L - 1) mod C before the stage
  // holding it is loaded.
  const uint16_t *k_new;
  const uint16_t *v_new;  // null when K serves as V
  Geometry geo;           // units_per_seq == 1
  int32_t n_q_heads;
  float qscale;           // folded into q: scale*log2(e), or scale/softcap
  float post;             // softcap*log2(e), or 0 when soft-cap is off
  // Test hook (GDATTN_FLAG_TEST_WITHHOLD_KV): every CTA leaves its first stage
  // unloaded, so the wait for it runs out and the timeout path runs.
  int32_t test_withhold;
};

template <int D, int G, int HKV, bool SHARED>
struct CoreConfig {
  static constexpr int NT = SHARED ? 1 : 2;
  static constexpr int MHDR = 8;                      // per-warp merge header (m[G], l[G])
  static constexpr int MSTRIDE = MHDR + G * D;        // floats per warp, 16-byte multiple
  // 16 compute warps (two or more per KV head) hide latency better; 8 when the
  // cross-warp merge area for 16 would not fit beside the ring.
  static constexpr int kComputeWarps = ((16 - HKV) * MSTRIDE * 4 <= 40 * 1024) ? 16 : 8;
  static constexpr int kThreads = (kComputeWarps + 1) * 32;
  static constexpr int TS = kComputeWarps / HKV;      // warps sharing one KV head
  static constexpr int ROWB = HKV * D * 2;            // bytes of one token row (one tensor)
  // Tokens per warp per stage: the largest of 8, 4, 2 that keeps a stage <= 64 KiB.
  static constexpr int TPW = (TS * 8 * ROWB * NT <= 65536) ? 8
                             : (TS * 4 * ROWB * NT <= 65536) ? 4 : 2;
  static constexpr int T = TS * TPW;                  // tokens per stage
  static constexpr int EPL = D / 32;                  // elements per lane
  static constexpr int CH = EPL / 8;                  // 16-byte chunks per lane
  static constexpr int STAGEB = T * ROWB * NT;
  static constexpr int MERGEB = TS > 1 ? (kComputeWarps - HKV) * MSTRIDE * 4 : 0;
  // Stages: up to 192 KiB of ring, within what the merge area leaves of the
  // 227 KiB a CTA may use (3 KiB kept for barriers, alignment and statics).
  static constexpr int RING = (224 * 1024 - MERGEB) < 196608 ? (224 * 1024 - MERGEB) : 196608;
  static constexpr int NSTAGE = (RING / STAGEB) < 2 ? 2 : (RING / STAGEB > 8 ? 8 : RING / STAGEB);
  static constexpr int NV = TPW * G;                  // scores per warp per stage
  static constexpr int LOGNV = NV == 2 ? 1 : NV == 4 ? 2 : (NV == 8 ? 3 : (NV == 16 ? 4 : 5));
  static constexpr int LOGG = G == 1 ? 0 : (G == 2 ? 1 : 2);
  static constexpr int LOGT = TPW == 2 ? 1 : (TPW == 4 ? 2 : 3);
  static constexpr int SMEM = NSTAGE * STAGEB + 2 * NSTAGE * 8 + 128 + MERGEB + 1024;
  static_assert(HKV == 1 || HKV == 2 || HKV == 4 || HKV == 8, "HKV");
  static_assert(G == 1 || G == 2 || G == 4, "G");
  static_assert(D == 256 || D == 512, "D");
  static_assert(NV >= 2 && NV <= 32, "one score per lane at most");
  static_assert(SMEM <= 226 * 1024, "shared memory");
};

template <int D, int G, int HKV, bool SHARED>
__global__ void __launch_bounds__(CoreConfig<D, G, HKV, SHARED>::kThreads, 1)
    core_decode_kernel(const CoreParams p) {
  using Cfg = CoreConfig<D, G, HKV, SHARED>;
  constexpr int NSTAGE = Cfg::NSTAGE, T = Cfg::T, CH = Cfg::CH;
  constexpr int ROWB = Cfg::ROWB, NV = Cfg::NV, LOGNV = Cfg::LOGNV, TPW = Cfg::TPW;
  constexpr int P2 = Cfg::EPL / 2;  // float2 pairs per lane

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stage_k = smem;
  uint8_t *stage_v = smem + NSTAGE * T * ROWB;  // unused when SHARED
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + NSTAGE * Cfg::STAGEB);
  uint64_t *empty = full + NSTAGE;
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(empty + NSTAGE);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(plan + 1);
  float *merge = reinterpret_cast<float *>(smem + NSTAGE * Cfg::STAGEB + 2 * NSTAGE * 8 + 128);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::kComputeWarps);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  grid_launch_dependents();
  // The split plan reads only seqlens, so it (and the producer's first KV
  // loads below) may run before the preceding kernel has completed; every other
  // global access waits for it (griddepcontrol.wait) in the role that makes it.
  if (warp == 0) plan_chunk(p.geo, c, plan);
  __syncthreads();

  if (c == 0 && warp == 0 && plan->bad) {
    grid_dependency_wait();
    if (lane == 0) atomicOr(p.status, kStatusSeqlen);
    // Sequences with nothing to attend get out = 0 and lse = -inf.
    for (int32_t b = 0; b < p.geo.batch; ++b) {
      bool dummy = false;
      if (attended_count(__ldg(p.geo.seqlens + b), p.geo.window, p.geo.capacity, dummy) != 0)
        continue;
      for (int i = lane; i < p.n_q_heads * D; i += 32)
        p.out[static_cast<int64_t>(b) * p.n_q_heads * D + i] = 0;
      if (p.lse != nullptr)
        for (int i = lane; i < p.n_q_heads; i += 32)
          p.lse[static_cast<int64_t>(b) * p.n_q_heads + i] = -INFINITY;
    }
  }

  const int32_t C = p.geo.capacity;

  if (warp == Cfg::kComputeWarps) {
    // ------------------------------------------------------------ producer
    // The whole warp walks the schedule and waits; one elected lane copies.
    const uint64_t pol = l2_evict_first_policy();
    uint32_t fills = 0;
    bool ok = true;
    // Until the preceding kernel completes, only cache rows of positions before
    // each sequence's newest one are read (earlier decode steps wrote them).
    bool waited = false;
    SegmentIter it;
    it.init(p.geo, *plan);
    Segment s;
    while (ok && it.next(s)) {
      const SlotRuns runs = segment_runs(s, C);
      for (int r = 0; ok && r < runs.count; ++r) {
        for (int32_t t0 = 0; t0 < runs.len(r); t0 += T) {
          const int ntok = min(T, runs.len(r) - t0);
          const int st = fills % NSTAGE;
          const bool newest = s.lo + (r == 1 ? runs.len0 : 0) + t0 + ntok == s.n;
          if (!waited && (fills >= NSTAGE || newest)) {
            grid_dependency_wait();
            waited = true;
          }
          if (fills >= NSTAGE &&
              !mbar_wait(&empty[st], ((fills / NSTAGE) - 1) & 1, abort_flag, p.status))
            ok = false;
          if (!__all_sync(0xffffffffu, ok)) {
            ok = false;
            break;
          }
          const uint32_t bytes = static_cast<uint32_t>(ntok * ROWB);
          const int64_t off = static_cast<int64_t>(cache_seq(p.geo, s.b)) * p.batch_stride +
                              static_cast<int64_t>(runs.start(r) + t0) * (HKV * D);
          if (p.k_new != nullptr && newest) {  // append the current token's rows first
            const int64_t row = static_cast<int64_t>(s.b) * p.batch_stride +
                                static_cast<int64_t>((s.first_pos + s.n - 1) % C) * (HKV * D);
            const int64_t src = static_cast<int64_t>(s.b) * (HKV * D);
            append_row(const_cast<uint16_t *>(p.k) + row, p.k_new + src, HKV * D, lane);
            if (!SHARED) append_row(const_cast<uint16_t *>(p.v) + row, p.v_new + src, HKV * D, lane);
          }
          if (!(p.test_withhold && fills == 0) && elect_one()) {
            mbar_arrive_expect_tx(&full[st], bytes * Cfg::NT);
            bulk_g2s(stage_k + st * T * ROWB, p.k + off, bytes, &full[st], pol);
            if (!SHARED) bulk_g2s(stage_v + st * T * ROWB, p.v + off, bytes, &full[st], pol);
          }
          __syncwarp();
          ++fills;
        }
      }
    }
    // Never leave with copies in flight into this CTA's shared memory.
    for (uint32_t f = fills > NSTAGE ? fills - NSTAGE : 0; f < fills; ++f) {
      volatile int no_abort = 0;
      if (!(p.test_withhold && f == 0))
        mbar_wait(&full[f % NSTAGE], (f / NSTAGE) & 1, &no_abort, p.status);
    }
  } else {
    // ------------------------------------------------------------- compute
    grid_dependency_wait();  // q, outputs and workspace
    const int kvh = warp % HKV;
    const int tp = warp / HKV;
    float2 q[G][P2];
    float2 o[G][P2];
    float m[G], l[G];
    uint32_t fills = 0;
    bool ok = true;
    SegmentIter it;
    it.init(p.geo, *plan);
    Segment s;
    while (it.next(s)) {
      // This sequence's query rows for the warp's heads, pre-scaled, as pairs.
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint16_t *qr = p.q + (static_cast<int64_t>(s.b) * p.n_q_heads + kvh * G + g) * D;
#pragma unroll
        for (int j = 0; j < CH; ++j) {
          const uint4 w = __ldg(reinterpret_cast<const uint4 *>(qr + 256 * j + 8 * lane));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            q[g][4 * j + e] = make_float2(bf16lo(ww[e]) * p.qscale, bf16hi(ww[e]) * p.qscale);
        }
#pragma unroll
        for (int e = 0; e < P2; ++e) o[g][e] = make_float2(0.f, 0.f);
        m[g] = -INFINITY;
        l[g] = 0.f;
      }

      const SlotRuns runs = segment_runs(s, C);
      for (int r = 0; r < runs.count; ++r) {
        for (int32_t t0 = 0; t0 < runs.len(r); t0 += T) {
          const int ntok = min(T, runs.len(r) - t0);
          const int st = fills % NSTAGE;
          if (ok && !mbar_wait(&full[st], (fills / NSTAGE) & 1, abort_flag, p.status)) ok = false;
          ok = __all_sync(0xffffffffu, ok);  // warp-uniform before warp-collective code
          ++fills;
          if (!ok) continue;
          const uint8_t *kst = stage_k + st * T * ROWB + kvh * D * 2;
          const uint8_t *vst = (SHARED ? stage_k : stage_v) + st * T * ROWB + kvh * D * 2;

          // Partial dot products part[i*G + g] over this lane's elements, two
          // elements per packed FMA.
          float part[NV];
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            const int t = tp + Cfg::TS * i;
            float2 acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = make_float2(0.f, 0.f);
            if (t < ntok) {
#pragma unroll
              for (int j = 0; j < CH; ++j) {
                const uint4 w =
                    *reinterpret_cast<const uint4 *>(kst + t * ROWB + 512 * j + 16 * lane);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 k2 = make_float2(bf16lo(ww[e]), bf16hi(ww[e]));
#pragma unroll
                  for (int g = 0; g < G; ++g) acc[g] = __ffma2_rn(q[g][4 * j + e], k2, acc[g]);
                }
              }
            }
#pragma unroll
            for (int g = 0; g < G; ++g) part[i * G + g] = acc[g].x + acc[g].y;
          }
          // Reduce-scatter: after log2(NV) halving steps a lane holds one score,
          // index bit k <-> lane bit (5 - LOGNV + k); lanes below bit
          // (5 - LOGNV) then sum their copies with the remaining xor steps.
          {
            int cnt = NV;
#pragma unroll
            for (int lev = 0; lev < LOGNV; ++lev) {
              const int off = 16 >> lev;
              const bool upper = (lane & off) != 0;
              const int half = cnt >> 1;
#pragma unroll
              for (int i2 = 0; i2 < NV / 2; ++i2) {
                if (i2 < half) {
                  const float send = upper ? part[i2] : part[i2 + half];
                  const float keep = upper ? part[i2 + half] : part[i2];
                  part[i2] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
              }
              cnt = half;
            }
#pragma unroll
            for (int off = 16 >> LOGNV; off > 0; off >>= 1)
              part[0] += __shfl_xor_sync(0xffffffffu, part[0], off);
          }
          const int idx = (lane >> (5 - LOGNV)) & (NV - 1);
          const int my_g = idx & (G - 1);
          const int my_t = tp + Cfg::TS * (idx >> Cfg::LOGG);
          float sc = part[0];
          if (p.post != 0.f) sc = p.post * tanhf(sc);
          if (my_t >= ntok) sc = -INFINITY;
          // Max over this stage's tokens for the lane's head: the token bits
          // are lane bits 5 - LOGT .. 4.
          float tmax = sc;
#pragma unroll
          for (int off = 16; off >= (1 << (5 - Cfg::LOGT)); off >>= 1)
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
          float mnew[G], alpha[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float mx = __shfl_sync(0xffffffffu, tmax, g << (5 - LOGNV));
            mnew[g] = fmaxf(m[g], mx);
            alpha[g] = (mnew[g] == -INFINITY) ? 1.f : exp2f(m[g] - mnew[g]);
          }
          float mine_m = mnew[0];
#pragma unroll
          for (int g = 1; g < G; ++g)
            if (my_g == g) mine_m = mnew[g];
          const float pe = (sc == -INFINITY) ? 0.f : exp2f(sc - mine_m);
          float psum = pe;
#pragma unroll
          for (int off = 16; off >= (1 << (5 - Cfg::LOGT)); off >>= 1)
            psum += __shfl_xor_sync(0xffffffffu, psum, off);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float ps = __shfl_sync(0xffffffffu, psum, g << (5 - LOGNV));
            l[g] = l[g] * alpha[g] + ps;
            m[g] = mnew[g];
            if (alpha[g] != 1.f) {  // warp-uniform: every lane holds the same alpha
              const float2 a2 = make_float2(alpha[g], alpha[g]);
#pragma unroll
              for (int e = 0; e < P2; ++e) o[g][e] = __fmul2_rn(o[g][e], a2);
            }
          }
          // P.V for this warp's tokens.
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            const int t = tp + Cfg::TS * i;
            float2 pw[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
              const float x = __shfl_sync(0xffffffffu, pe, (i * G + g) << (5 - LOGNV));
              pw[g] = make_float2(x, x);
            }
            if (t < ntok) {
#pragma unroll
              for (int j = 0; j < CH; ++j) {
                const uint4 w =
                    *reinterpret_cast<const uint4 *>(vst + t * ROWB + 512 * j + 16 * lane);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 v2 = make_float2(bf16lo(ww[e]), bf16hi(ww[e]));
#pragma unroll
                  for (int g = 0; g < G; ++g)
                    o[g][4 * j + e] = __ffma2_rn(pw[g], v2, o[g][4 * j + e]);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[st]);
        }
      }

      // ---------------------------------------------------- segment epilogue
      if (Cfg::TS > 1) {
        // Merge the TS warps that share a KV head: warps tp > 0 hand their state
        // to the tp == 0 warp through shared memory.
        if (tp > 0) {
          float *mine = merge + ((tp - 1) * HKV + kvh) * Cfg::MSTRIDE;
          if (lane == 0) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
              mine[g] = m[g];
              mine[4 + g] = l[g];
            }
          }
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              float4 *dst =
                  reinterpret_cast<float4 *>(mine + Cfg::MHDR + g * D + 256 * j + 8 * lane);
              dst[0] = make_float4(o[g][4 * j].x, o[g][4 * j].y, o[g][4 * j + 1].x,
                                   o[g][4 * j + 1].y);
              dst[1] = make_float4(o[g][4 * j + 2].x, o[g][4 * j + 2].y, o[g][4 * j + 3].x,
                                   o[g][4 * j + 3].y);
            }
        }
        named_bar_sync(1, Cfg::kComputeWarps * 32);
        if (tp == 0) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float M = m[g];
            for (int k = 1; k < Cfg::TS; ++k)
              M = fmaxf(M, merge[((k - 1) * HKV + kvh) * Cfg::MSTRIDE + g]);
            const float w0 = (m[g] == -INFINITY) ? 0.f : exp2f(m[g] - M);
            float Ls = l[g] * w0;
            const float2 w02 = make_float2(w0, w0);
#pragma unroll
            for (int e = 0; e < P2; ++e) o[g][e] = __fmul2_rn(o[g][e], w02);
#pragma unroll
            for (int k = 1; k < Cfg::TS; ++k) {
              const float *src = merge + ((k - 1) * HKV + kvh) * Cfg::MSTRIDE;
              const float wk = (src[g] == -INFINITY) ? 0.f : exp2f(src[g] - M);
              Ls += src[4 + g] * wk;
              const float2 w2 = make_float2(wk, wk);
              src += Cfg::MHDR + g * D;
#pragma unroll
              for (int j = 0; j < CH; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  o[g][4 * j + e] = __ffma2_rn(
                      w2, *reinterpret_cast<const float2 *>(src + 256 * j + 8 * lane + 2 * e),
                      o[g][4 * j + e]);
            }
            m[g] = M;
            l[g] = Ls;
          }
        }
        named_bar_sync(1, Cfg::kComputeWarps * 32);
      }
      if (tp == 0 && ok) {
        const bool single = s.whole();
        const int64_t slot = static_cast<int64_t>(c) + s.unit;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const int h = kvh * G + g;
          const float inv = __fdividef(1.f, l[g]);
          const float lse_v = (m[g] + log2f(l[g])) * 0.69314718055994530942f;
          if (single) {
            uint16_t *dst = p.out + (static_cast<int64_t>(s.b) * p.n_q_heads + h) * D;
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              uint4 w;
              w.x = pack_bf16x2(o[g][4 * j].x * inv, o[g][4 * j].y * inv);
              w.y = pack_bf16x2(o[g][4 * j + 1].x * inv, o[g][4 * j + 1].y * inv);
              w.z = pack_bf16x2(o[g][4 * j + 2].x * inv, o[g][4 * j + 2].y * inv);
              w.w = pack_bf16x2(o[g][4 * j + 3].x * inv, o[g][4 * j + 3].y * inv);
              *reinterpret_cast<uint4 *>(dst + 256 * j + 8 * lane) = w;
            }
            if (lane == 0 && p.lse != nullptr)
              p.lse[static_cast<int64_t>(s.b) * p.n_q_heads + h] = lse_v;
          } else {
            float *dst = p.ws_o + (slot * p.n_q_heads + h) * D;
#pragma unroll
            for (int j = 0; j < CH; ++j) {
              float4 *d4 = reinterpret_cast<float4 *>(dst + 256 * j + 8 * lane);
              d4[0] = make_float4(o[g][4 * j].x * inv, o[g][4 * j].y * inv,
                                  o[g][4 * j + 1].x * inv, o[g][4 * j + 1].y * inv);
              d4[1] = make_float4(o[g][4 * j + 2].x * inv, o[g][4 * j + 2].y * inv,
                                  o[g][4 * j + 3].x * inv, o[g][4 * j + 3].y * inv);
            }
            if (lane == 0) p.ws_lse[slot * p.n_q_heads + h] = lse_v;
          }
        }
      }
    }
  }
  __syncthreads();
}

}  // namespace gdattn
