// Split-KV decode attention on the 5th-generation tensor cores (tcgen05), for a
// GQA group of 16 query heads over one KV head with key == value, head_dim 512:
// Gemma-4 full-attention layers (attention_k_eq_v).
//
// With 16 query rows per KV row the products are a dense contraction (32 flop
// per KV byte), far beyond what CUDA-core FMAs sustain at HBM speed, so both
// products run on tcgen05 with the accumulators in tensor memory (TMEM):
//
//   S^T[64 tok x 16 h]  = K_tile[64 x 512] . Q^T[512 x 16]   (M=64, N=16, K=512)
//   O^T[512 d x 16 h]   = V_tile^T[512 x 64] . P^T[64 x 16]  (M=128 x4, N=16, K=64)
//
// K = V: the one 64-token tile in shared memory is the K-major A operand of the
// first product and the MN-major A operand of the second, so each cache byte
// crosses HBM once.  The tile arrives by TMA as eight 64x64 boxes with 128-byte
// swizzle, which is the canonical operand layout for both majors.
//
// Warp roles (192 threads): warp 0 issues TMA loads; warp 1 owns TMEM and issues
// MMAs (one elected lane); warps 2-5 read S from TMEM, run the online softmax
// (running max / sum per head), write P^T (bf16) to shared memory, and fold each
// tile's O^T into fp32 registers with the rescale factor.  S and O^T are double
// buffered in TMEM so the tensor core computes tile i+1 while tile i's softmax
// runs.  Every wait is bounded; on a timeout all roles fast-forward, drain
// their copies / MMAs and free TMEM.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "partition.cuh"
#include "ptx.cuh"

namespace gdattn {

struct TcParams {
  const uint16_t *q;      // [B, Hq, D] (through qmap; pointer kept for reference)
  uint16_t *out;          // [B, Hq, D]
  float *lse;             // [B, Hq] or null
  float *ws_o;            // partial outputs [slots][16][D]
  float *ws_lse;          // partial lse [slots][16]
  uint32_t *status;
  Geometry geo;           // units_per_seq == n_kv_heads
  int32_t n_q_heads;
  float qscale;           // multiplies raw scores: scale*log2(e), or scale/softcap
  float post;             // softcap*log2(e), or 0 when soft-cap is off
};

struct TcConfig {
  static constexpr int D = 512;
  static constexpr int G = 16;
  static constexpr int TILE = 64;                     // tokens per tile
  static constexpr int NST = 3;                       // KV stages
  static constexpr int BOXB = TILE * 128;             // one 64-token x 64-d box
  static constexpr int STAGEB = BOXB * (D / 64);      // 64 KiB
  static constexpr int QB = G * D * 2;                // 16 KiB
  static constexpr int PB = G * TILE * 2;             // 2 KiB per P buffer
  static constexpr int OFF_Q = NST * STAGEB;
  static constexpr int OFF_P = OFF_Q + QB;
  static constexpr int OFF_BAR = OFF_P + 2 * PB;
  static constexpr int OFF_RED = OFF_BAR + 256;
  static constexpr int SMEM = OFF_RED + 2 * 2 * 4 * G * 4 + 1024;
  static constexpr int kThreads = 192;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;                // 2 x 16 columns
  static constexpr uint32_t O_COL = 64;               // 2 x 64 columns
};

// Tiles of one CTA, in order, across its segments.
struct TileIter {
  SegmentIter seg_it;
  Segment seg;
  SlotRuns runs;
  int32_t run, t0;
  bool have_seg;
  int32_t seg_index;

  __device__ __forceinline__ void init(const Geometry &g, const ChunkPlan &p) {
    seg_it.init(g, p);
    have_seg = false;
    seg_index = -1;
  }
  // Yields the next tile: slot row of its first token, valid token count, and
  // whether it opens / closes its segment.
  __device__ __forceinline__ bool next(int32_t C, int32_t &row, int32_t &ntok, bool &first,
                                       bool &last) {
    first = false;
    if (!have_seg) {
      if (!seg_it.next(seg)) return false;
      runs = segment_runs(seg, C);
      run = 0;
      t0 = 0;
      have_seg = true;
      first = true;
      ++seg_index;
    }
    row = runs.start(run) + t0;
    ntok = min(TcConfig::TILE, runs.len(run) - t0);
    t0 += TcConfig::TILE;
    if (t0 >= runs.len(run)) {
      ++run;
      t0 = 0;
    }
    last = (run >= runs.count);
    if (last) have_seg = false;
    return true;
  }
};

__global__ void __launch_bounds__(TcConfig::kThreads, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  using Cfg = TcConfig;
  constexpr int G = Cfg::G, D = Cfg::D, NST = Cfg::NST;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint8_t *ps = smem + Cfg::OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *full = bars;            // [NST]  TMA -> MMA
  uint64_t *empty = bars + 3;       // [NST]  MMA -> TMA
  uint64_t *qfull = bars + 6;       // TMA -> MMA
  uint64_t *qempty = bars + 7;      // MMA -> TMA
  uint64_t *sfull = bars + 8;       // [2] MMA -> softmax
  uint64_t *sempty = bars + 10;     // [2] softmax -> MMA
  uint64_t *pfull = bars + 12;      // [2] softmax -> MMA
  uint64_t *ofull = bars + 14;      // [2] MMA -> softmax
  uint64_t *oempty = bars + 16;     // [2] softmax -> MMA
  uint64_t *drain = bars + 18;
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 19);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 20);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(bars + 21);  // 48 bytes, ends before +256
  float *red = reinterpret_cast<float *>(smem + Cfg::OFF_RED);  // [2 kinds][2 buf][4 warps][16]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
      mbar_init(&pfull[s], 4);
      mbar_init(&ofull[s], 1);
      mbar_init(&oempty[s], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  grid_launch_dependents();
  grid_dependency_wait();
  if (warp == 2) plan_chunk(p.geo, c, plan);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  if (c == 0 && warp == 2 && plan->bad) {
    if (lane == 0) atomicOr(p.status, kStatusSeqlen);
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

  if (warp == 0) {
    // -------------------------------------------------------------- TMA
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      bool ok = true;
      uint32_t i = 0, nseg = 0;
      TileIter it;
      it.init(p.geo, *plan);
      int32_t row, ntok;
      bool first, last;
      while (ok && it.next(C, row, ntok, first, last)) {
        if (first) {
          if (nseg > 0 && !mbar_wait(qempty, (nseg - 1) & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const int32_t qrow = it.seg.b * p.n_q_heads + it.seg.x * G;
          mbar_arrive_expect_tx(qfull, Cfg::QB);
#pragma unroll
          for (int j = 0; j < D / 64; ++j) tma_load_2d(qs + j * (G * 128), &qmap, 64 * j, qrow, qfull);
          ++nseg;
        }
        const int st = i % NST;
        if (i >= NST && !mbar_wait(&empty[st], ((i / NST) - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[st], Cfg::STAGEB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(stages + st * Cfg::STAGEB + j * Cfg::BOXB, &kmap, 64 * j, it.seg.x, row,
                      it.seg.b, &full[st], pol);
        ++i;
      }
      // Drain: never leave with copies in flight into shared memory.
      volatile int no_abort = 0;
      for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
        mbar_wait(&full[f % NST], (f / NST) & 1, &no_abort, p.status);
      if (nseg > 0) mbar_wait(qfull, (nseg - 1) & 1, &no_abort, p.status);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc_qk = idesc_bf16_f32(64, 16, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, 16, true, false);
      const uint32_t st_addr = smem_u32(stages);
      const uint32_t q_addr = smem_u32(qs);
      const uint32_t p_addr = smem_u32(ps);
      bool ok = true;
      uint32_t i = 0, nseg = 0;
      int32_t prev = -1;  // tile whose P.V is still to issue
      TileIter it;
      it.init(p.geo, *plan);
      int32_t row, ntok;
      bool first, last;
      auto issue_pv = [&](uint32_t t) -> bool {
        const int pb = t & 1, ob = t & 1;
        if (!mbar_wait(&pfull[pb], (t >> 1) & 1, abort_flag, p.status)) return false;
        if (t >= 2 && !mbar_wait(&oempty[ob], ((t >> 1) - 1) & 1, abort_flag, p.status))
          return false;
        tc_fence_after();
        const uint32_t a0 = st_addr + (t % NST) * Cfg::STAGEB;
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(a0 + (2 * jb) * Cfg::BOXB + kk * 2048, Cfg::BOXB, 1024);
            const uint64_t bd = smem_desc_sw128(p_addr + pb * Cfg::PB + kk * 32, 16, 1024);
            tc_mma_bf16(tmem + Cfg::O_COL + ob * 64 + jb * 16, ad, bd, idesc_pv, kk > 0);
          }
        }
        tc_commit(&ofull[ob]);
        tc_commit(&empty[t % NST]);
        return true;
      };
      while (ok && it.next(C, row, ntok, first, last)) {
        if (first) {
          if (!mbar_wait(qfull, nseg & 1, abort_flag, p.status)) {
            ok = false;
            break;
          }
          ++nseg;
        }
        const int st = i % NST, sb = i & 1;
        if (!mbar_wait(&full[st], (i / NST) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        if (i >= 2 && !mbar_wait(&sempty[sb], ((i >> 1) - 1) & 1, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = st_addr + st * Cfg::STAGEB;
#pragma unroll
        for (int j = 0; j < D / 64; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc_sw128(a0 + j * Cfg::BOXB + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(q_addr + j * (G * 128) + kk * 32, 16, 1024);
            tc_mma_bf16(tmem + Cfg::S_COL + sb * 16, ad, bd, idesc_qk, (j | kk) != 0);
          }
        }
        tc_commit(&sfull[sb]);
        if (last) tc_commit(qempty);
        if (prev >= 0 && !issue_pv(static_cast<uint32_t>(prev))) {
          ok = false;
          break;
        }
        prev = static_cast<int32_t>(i);
        ++i;
      }
      if (ok && prev >= 0) ok = issue_pv(static_cast<uint32_t>(prev));
      // Drain: wait until every issued MMA has completed before TMEM is freed.
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, p.status);
    }
  } else {
    // ---------------------------------------------------------- softmax
    const int qd = warp & 3;                 // TMEM sub-partition: lanes 32*qd ..
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 16 * qd + lane;          // tile token held by this lane (lane < 16)
    float acc[4][G];
    float m[G], l[G], alpha_prev[G], m_fin[G], l_fin[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
      m_fin[h] = -INFINITY;
      l_fin[h] = 1.f;
      alpha_prev[h] = 0.f;
#pragma unroll
      for (int jb = 0; jb < 4; ++jb) acc[jb][h] = 0.f;
    }
    bool ok = true;
    uint32_t i = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    bool prev_last = false;
    Segment prev_seg;
    prev_seg.b = 0;

    auto correction = [&](uint32_t t) {
      const int ob = t & 1;
      if (ok && !mbar_wait(&ofull[ob], (t >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          float v[16];
          tmem_ld16(tmem + lane_base + Cfg::O_COL + ob * 64 + jb * 16, v);
#pragma unroll
          for (int h = 0; h < G; ++h) acc[jb][h] = fmaf(acc[jb][h], alpha_prev[h], v[h]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&oempty[ob]);
      }
    };

    auto finalize = [&](const Segment &s) {
      if (!ok) return;
      int32_t cf, cl;
      unit_chunks(s.unit_start, s.n, plan->chunk, cf, cl);
      const bool single = (cf == cl);
      const int64_t slot = static_cast<int64_t>(c) + s.unit;
      const int h0 = s.x * G;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float inv = 1.f / l_fin[h];
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          const int d = 128 * jb + 32 * qd + lane;
          const float val = acc[jb][h] * inv;
          if (single)
            p.out[(static_cast<int64_t>(s.b) * p.n_q_heads + h0 + h) * D + d] = f32_to_bf16_rn(val);
          else
            p.ws_o[(slot * G + h) * D + d] = val;
        }
      }
      if (qd == 0 && lane < G) {
        float mf_l = m_fin[0], lf_l = l_fin[0];
#pragma unroll
        for (int h = 1; h < G; ++h)
          if (lane == h) {
            mf_l = m_fin[h];
            lf_l = l_fin[h];
          }
        const float lse_v = (mf_l + log2f(lf_l)) * 0.69314718055994530942f;
        if (single) {
          if (p.lse != nullptr) p.lse[static_cast<int64_t>(s.b) * p.n_q_heads + h0 + lane] = lse_v;
        } else {
          p.ws_lse[slot * G + lane] = lse_v;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) acc[jb][h] = 0.f;
    };

    while (it.next(C, row, ntok, first, last)) {
      const int sb = i & 1, pb = i & 1, buf = i & 1;
      if (first) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m[h] = -INFINITY;
          l[h] = 0.f;
        }
      }
      // --- scores of tile i
      float s[16];
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 16, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      const bool valid = ok && lane < 16 && tok < ntok;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float x = s[h] * p.qscale;
        if (p.post != 0.f) x = p.post * tanhf(x);
        s[h] = valid ? x : -INFINITY;
      }
      // --- per-head tile max: reduce-scatter over the warp, then across warps
      float r[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) r[h] = s[h];
#pragma unroll
      for (int lev = 0; lev < 4; ++lev) {
        const int off = 16 >> lev, half = 8 >> lev;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < half) {
            const float send = upper ? r[k] : r[k + half];
            const float keep = upper ? r[k + half] : r[k];
            r[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
          }
      }
      r[0] = fmaxf(r[0], __shfl_xor_sync(0xffffffffu, r[0], 1));
      float *redmax = red + (0 * 2 + buf) * 4 * G;
      float *redsum = red + (1 * 2 + buf) * 4 * G;
      if ((lane & 1) == 0) redmax[qd * G + (lane >> 1)] = r[0];
      named_bar_sync(1, 128);
      float mnew[G], alpha[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float tm = fmaxf(fmaxf(redmax[h], redmax[G + h]), fmaxf(redmax[2 * G + h], redmax[3 * G + h]));
        mnew[h] = fmaxf(m[h], tm);
        alpha[h] = (mnew[h] == -INFINITY) ? 1.f : exp2f(m[h] - mnew[h]);
        m[h] = mnew[h];
      }
      // --- probabilities, P^T (bf16, 128B-swizzled K-major) and row sums
      uint8_t *prow = ps + pb * Cfg::PB;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pe = (s[h] == -INFINITY) ? 0.f : exp2f(s[h] - mnew[h]);
        r[h] = pe;
        if (lane < 16) {
          const uint32_t off = h * 128 + ((((tok >> 3) ^ (h & 7)) & 7) << 4) + (tok & 7) * 2;
          *reinterpret_cast<uint16_t *>(prow + off) = f32_to_bf16_rn(pe);
        }
      }
      if (ok && ntok < Cfg::TILE) {
        // Rows past the attended range hold other cache contents (possibly
        // NaN); they get weight 0, but 0 * NaN would still reach O, so clear them.
        uint8_t *tile = stages + (i % NST) * Cfg::STAGEB;
        const int nchunk = (Cfg::TILE - ntok) * 8 * (D / 64);
        for (int e = threadIdx.x - 64; e < nchunk; e += 128) {
          const int box = e / ((Cfg::TILE - ntok) * 8);
          const int rem = e - box * ((Cfg::TILE - ntok) * 8);
          const int rrow = ntok + (rem >> 3);
          *reinterpret_cast<uint4 *>(tile + box * Cfg::BOXB + rrow * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
#pragma unroll
      for (int lev = 0; lev < 4; ++lev) {
        const int off = 16 >> lev, half = 8 >> lev;
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < half) {
            const float send = upper ? r[k] : r[k + half];
            const float keep = upper ? r[k + half] : r[k];
            r[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
      }
      r[0] += __shfl_xor_sync(0xffffffffu, r[0], 1);
      if ((lane & 1) == 0) redsum[qd * G + (lane >> 1)] = r[0];
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);
      named_bar_sync(1, 128);
#pragma unroll
      for (int h = 0; h < G; ++h)
        l[h] = l[h] * alpha[h] + ((redsum[h] + redsum[G + h]) + (redsum[2 * G + h] + redsum[3 * G + h]));

      // --- fold the previous tile's O^T, then close its segment if it ended
      if (i > 0) {
        correction(i - 1);
        if (prev_last) finalize(prev_seg);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
      prev_last = last;
      prev_seg = it.seg;
      if (last) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_fin[h] = m[h];
          l_fin[h] = l[h];
        }
      }
      ++i;
    }
    if (i > 0) {
      correction(i - 1);
      if (prev_last) finalize(prev_seg);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace gdattn
