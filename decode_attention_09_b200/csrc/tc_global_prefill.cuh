// Flash prefill on the global geometry (8 or 16 query heads per KV head,
// head_dim 512, one cache tensor serving as K and V): a multi-token step of more
// than 8 tokens, the head_dim-512 counterpart of tc_pair_prefill.cuh.  Token t
// of sequence b sits at position p = L_b - T + t and attends [max(0, p + 1 - w),
// p + 1) (w = 0: [0, p + 1)).
//
// A 64-row block is 64 / GU query tokens x GU heads (row GU tq + h), one M = 64
// MMA.  An O of 64 rows x 512 dims would take all 512 TMEM columns, so each
// block runs on two CTAs, one per half of the head dimension: both compute the
// full scores, each accumulates and writes its own 256 output dims.  Per 64-token
// KV tile (the tile is both the K-major B operand of QK and, its half of the
// dims, the MN-major B operand of P.V, so a tile crosses HBM once per CTA and
// mostly comes from L2 for the second):
//
//   S[64 x 64]    = Q[64 x 512] . K_tile^T[512 x 64]          (M=64, N=64,  K=512)
//   O[64 x 256]  += P_hi[64 x 64] . V_half[64 x 256]
//                 + P_lo[64 x 64] . V_half[64 x 256]           (M=64, N=256, K=64 x 2)
//
// An M = 64 accumulator puts row 16 s + i in lane i of TMEM sub-partition s, so
// softmax warp s owns rows 16 s .. 16 s + 15 in its lanes 0-15 (lanes 16-31 join
// the warp-wide TMEM loads and stores and own nothing).  Each row's thread keeps
// its running maximum (moved lazily by 2^8), row sum and the rescale of its O row,
// as in the head_dim-256 kernel; the weights are split into bf16 parts by
// truncation (2^-14 relative), written as the K-major A operand in shared memory
// (double-buffered).
//
// Shared memory (1 CTA per SM): the block's Q (64 KiB), two 64 KiB KV stages,
// two P buffers (16 KiB each): 224 KiB.  TMEM: S double buffered (2 x 64
// columns) and O (256 columns).  Warp roles as in the head_dim-256 kernel: warp
// 0 loads Q and the KV tiles, warp 1 issues QK and owns TMEM, warp 2 issues P.V,
// warps 4-7 run the softmax.  Every wait is bounded.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "partition.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"
#include "tc_pair_prefill.cuh"

namespace gdattn {

struct TcGlobalPrefillConfig {
  static constexpr int D = 512;
  static constexpr int DH = 256;                  // output dims per CTA
  static constexpr int M = 64;                    // query rows per block
  static constexpr int TILE = 64;                 // KV tokens per tile
  static constexpr int NST = 2;                   // KV stages
  static constexpr int BOXB = TILE * 128;         // 64 KV rows x 64 d: 8 KiB
  static constexpr int KB = BOXB * (D / 64);      // 64 KiB
  static constexpr int QBOXB = M * 128;           // 64 rows x 64 d: 8 KiB
  static constexpr int QB = QBOXB * (D / 64);     // 64 KiB
  static constexpr int PHB = M * 128;             // one P part: 64 rows x 64 KV bf16, 8 KiB
  static constexpr int PB = 2 * PHB;              // weights then remainders
  static constexpr int OFF_Q = NST * KB;
  static constexpr int OFF_P = OFF_Q + QB;
  static constexpr int OFF_BAR = OFF_P + 2 * PB;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int kThreads = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;            // 2 buffers x 64 columns
  static constexpr uint32_t O_COL = 256;          // 256 columns
};
static_assert(TcGlobalPrefillConfig::SMEM <= 227 * 1024, "shared memory budget");

// Block c -> (sequence b, KV head x, query block qb, dimension half dh),
// heaviest causal blocks first.
__device__ __forceinline__ void global_prefill_block(const PrefillParams &p, int32_t c,
                                                     int32_t &b, int32_t &x, int32_t &qb,
                                                     int32_t &dh) {
  dh = c & 1;
  const int32_t cb = c >> 1;
  const int32_t nb = p.nblocks;
  const int32_t u = cb / nb;
  qb = nb - 1 - (cb - u * nb);
  b = u / p.n_kv_heads;
  x = u - b * p.n_kv_heads;
}

template <int GU>
__global__ void __launch_bounds__(TcGlobalPrefillConfig::kThreads, 1)
    tc_global_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                             const __grid_constant__ CUtensorMap qmap, const PrefillParams p) {
  using Cfg = TcGlobalPrefillConfig;
  constexpr int D = Cfg::D, DH = Cfg::DH, NST = Cfg::NST, TILE = Cfg::TILE;
  constexpr int QT = Cfg::M / GU;  // query tokens per block
  static_assert(GU == 16 || GU == 8, "query heads per KV head");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *kv = smem;                // KV ring
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint8_t *ps = smem + Cfg::OFF_P;   // [2] x (weights, remainders)
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *full = bars;           // [NST] TMA -> QK (and the softmax, for partial tiles)
  uint64_t *empty = bars + 2;      // [NST] P.V (after the tile's QK) -> TMA
  uint64_t *sfull = bars + 4;      // [2] QK -> softmax
  uint64_t *sempty = bars + 6;     // [2] softmax -> QK
  uint64_t *qfull = bars + 8;      // Q TMA -> QK
  uint64_t *pfull = bars + 9;      // [2] softmax -> P.V, per P buffer
  uint64_t *odone = bars + 11;     // [2] P.V -> softmax, per P buffer
  uint64_t *drain = bars + 13;     // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 15);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 16);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int32_t b, x, qb, dh;
  global_prefill_block(p, static_cast<int32_t>(blockIdx.x), b, x, qb, dh);
  const int32_t T = p.tokens;
  const int32_t L = __ldg(p.seqlens + b);
  const int32_t P0 = L - T + qb * QT;  // position of the block's first token
  const int32_t nq = min(QT, T - qb * QT);
  int32_t lo = p.window > 0 ? P0 + 1 - p.window : 0;
  if (lo < 0) lo = 0;
  const int32_t hi = P0 + nq;
  const bool bad = L < T || (hi > lo && lo < L - p.capacity);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
      mbar_init(&pfull[s], 4);
      mbar_init(&odone[s], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;
  const int32_t C = p.capacity;
  const int32_t lo_t = hi > lo ? lo : hi;  // an empty range has no tiles

  if (warp == 0) {
    // ---------------------------------------------------- Q and KV loads
    grid_dependency_wait();  // Q and the chunk's own cache rows come from the preceding kernels
    const uint64_t pol = l2_evict_first_policy();
    if (elect_one()) {
      mbar_arrive_expect_tx(qfull, Cfg::QB);
#pragma unroll
      for (int j = 0; j < D / 64; ++j)
        tma_load_3d(qs + j * Cfg::QBOXB, &qmap, 64 * j, b * p.n_q_heads + x * GU, qb * QT,
                    qfull);
    }
    __syncwarp();
    bool ok = true;
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (ok && it.next(pos0, slot, ntok)) {
      const int st = i % NST;
      if (i >= NST) ok = mbar_wait(&empty[st], ((i / NST) - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (!(p.test_withhold && i == 0) && elect_one()) {
        mbar_arrive_expect_tx(&full[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(kv + st * Cfg::KB + j * Cfg::BOXB, &kmap, 64 * j, x, slot, b, &full[st],
                      pol);
      }
      __syncwarp();
      ++i;
    }
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      if (!(p.test_withhold && f == 0))
        mbar_wait(&full[f % NST], (f / NST) & 1, &no_abort, p.status);
    mbar_wait(qfull, 0, &no_abort, p.status);
  } else if (warp == 1) {
    // --------------------------------------------------------- QK MMA
    const uint32_t idesc = idesc_bf16_f32(Cfg::M, TILE, false, false);
    const uint64_t qdesc = smem_desc_sw128(smem_u32(qs), 16, 1024);  // Q, K-major
    const uint64_t kdesc = smem_desc_sw128(smem_u32(kv), 16, 1024);  // KV tile, K-major
    bool ok = mbar_wait(qfull, 0, abort_flag, p.status);
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (__all_sync(0xffffffffu, ok) && it.next(pos0, slot, ntok)) {
      const int st = i % NST, sb = i & 1;
      ok = mbar_wait(&full[st], (i / NST) & 1, abort_flag, p.status);
      if (ok && i >= 2) ok = mbar_wait(&sempty[sb], ((i >> 1) - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16(tmem + Cfg::S_COL + sb * TILE,
                        qdesc + ((j * Cfg::QBOXB + kk * 32) >> 4),
                        kdesc + ((st * Cfg::KB + j * Cfg::BOXB + kk * 32) >> 4), idesc,
                        (j | kk) != 0);
        tc_commit(&sfull[sb]);
      }
      __syncwarp();
      ++i;
    }
    if (elect_one()) tc_commit(&drain[0]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[0], 0, &no_abort, p.status);
  } else if (warp == 2) {
    // -------------------------------------------------------- P.V MMA
    const uint32_t idesc = idesc_bf16_f32(Cfg::M, DH, false, true);
    const uint64_t pdesc = smem_desc_sw128(smem_u32(ps), 16, 1024);  // P, K-major
    // This CTA's half of the tile as the MN-major B operand: 64-d chunks
    // Cfg::BOXB apart, 8 KV rows per 1 KiB.
    const uint64_t vdesc =
        smem_desc_sw128(smem_u32(kv + dh * (DH / 64) * Cfg::BOXB), Cfg::BOXB, 1024);
    bool ok = true;
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (ok && it.next(pos0, slot, ntok)) {
      const int st = i % NST, pb = i & 1;
      // The tile is in shared memory: the softmax saw S, so its QK read it.
      const bool w = mbar_wait(&pfull[pb], (i >> 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk)
            tc_mma_bf16(tmem + Cfg::O_COL, pdesc + ((pb * Cfg::PB + part * Cfg::PHB + kk * 32) >> 4),
                        vdesc + ((st * Cfg::KB + kk * 2048) >> 4), idesc,
                        !(i == 0 && part == 0 && kk == 0));
        tc_commit(&odone[pb]);
        tc_commit(&empty[st]);  // after this tile's QK and P.V
      }
      __syncwarp();
      ++i;
    }
    if (elect_one()) tc_commit(&drain[1]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[1], 0, &no_abort, p.status);
  } else if (warp >= 4) {
    // -------------------------------------------------------- softmax
    grid_dependency_wait();  // outputs are written below
    const int qd = warp & 3;
    const int t128 = threadIdx.x - 128;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int r = 16 * qd + (lane & 15);  // the row of lanes 0-15
    const int tq = r / GU, h = r % GU;
    const bool row_ok = lane < 16 && tq < nq;
    const int32_t prow = P0 + tq;
    if (bad && t128 == 0) atomicOr(p.status, kStatusSeqlen);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t done0 = 0, done1 = 0;  // phases consumed on odone[0], odone[1]
    // The P.V of tile tt (and so every earlier one) has completed; a barrier
    // never runs two phases ahead of its waiter, so parity waits cannot alias.
    auto ensure_pv = [&](uint32_t tt) {
      const uint32_t ph = tt >> 1;
      if (tt & 1) {
        for (; done1 <= ph; ++done1)
          if (ok && !mbar_wait(&odone[1], done1 & 1, abort_flag, p.status)) ok = false;
      } else {
        for (; done0 <= ph; ++done0)
          if (ok && !mbar_wait(&odone[0], done0 & 1, abort_flag, p.status)) ok = false;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (it.next(pos0, slot, ntok)) {
      const int sb = i & 1, pb = i & 1;
      float s[TILE];
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        tmem_ld64(tmem + lane_base + Cfg::S_COL + sb * TILE, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      } else {
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] = 0.f;
      }
      if (p.post != 0.f) {
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] = p.post * tanhf(s[c] * p.qscale);
      } else {
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] *= p.qscale;
      }
      // Column c (position pos0 + c) is in the row's range for c in [c_lo, c_hi).
      const bool inside = ntok == TILE && nq == QT && pos0 + TILE - 1 <= P0 &&
                          (p.window == 0 || pos0 >= P0 + QT - p.window);
      if (!(inside && ok && lane < 16)) {
        const int32_t c_lo = p.window > 0 ? prow + 1 - p.window - pos0 : 0;
        int32_t c_hi = prow - pos0 + 1 < ntok ? prow - pos0 + 1 : ntok;
        if (!(ok && row_ok)) c_hi = 0;
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] = (c >= c_lo && c < c_hi) ? s[c] : -INFINITY;
      }
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < TILE; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
      // --- move a row's reference when a score outgrew it; the TMEM loads and
      // stores are warp-wide, so the whole warp rescales (by 1 where it stays).
      const bool mine = mx > m_ref + kTau;
      if (__any_sync(0xffffffffu, mine)) {
        float alpha = 1.f;
        if (mine) {
          alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
          l *= alpha;
          m_ref = mx;
        }
        if (i > 0) {
          ensure_pv(i - 1);
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < DH / 32; ++cb) {
              float o[32];
              tmem_ld32(tmem + lane_base + Cfg::O_COL + cb * 32, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= alpha;
              tmem_st32_wait(tmem + lane_base + Cfg::O_COL + cb * 32, o);
            }
          }
        }
      }
      // --- weights and remainders (truncated bf16 parts), P buffer pb in
      // shared memory: row r, K-major with 128-byte swizzle.
      const float mr = m_ref == -INFINITY ? 0.f : m_ref;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      if (i >= 2) ensure_pv(i - 2);  // the P.V of tile i - 2 read this P buffer
      uint8_t *phi = ps + pb * Cfg::PB + r * 128, *plo = phi + Cfg::PHB;
#pragma unroll
      for (int ch = 0; ch < TILE / 8; ++ch) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pa = ex2_approx(s[8 * ch + 2 * e] - mr);
          const float pb2 = ex2_approx(s[8 * ch + 2 * e + 1] - mr);
          l4[e] += pa + pb2;
          const uint32_t ua = __float_as_uint(pa), ub = __float_as_uint(pb2);
          const float ra = pa - __uint_as_float(ua & 0xFFFF0000u);
          const float rb = pb2 - __uint_as_float(ub & 0xFFFF0000u);
          wh[e] = __byte_perm(ua, ub, 0x7632);
          wl[e] = __byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632);
        }
        if (lane < 16) {
          const uint32_t off = static_cast<uint32_t>((ch ^ (r & 7)) << 4);
          *reinterpret_cast<uint4 *>(phi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4 *>(plo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
        }
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      if (ok && ntok < TILE) {
        // Rows past the tile's end hold other slots (possibly NaN): clear this
        // CTA's half of them for P.V (the tile's QK is done: S was read).
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&full[i % NST], (i / NST) & 1, abort_flag, p.status));
        if (ok) {
          uint8_t *vt = kv + (i % NST) * Cfg::KB + dh * (DH / 64) * Cfg::BOXB;
          const int per_box = (TILE - ntok) * 8;
#pragma unroll 1
          for (int box = 0; box < DH / 64; ++box)
            for (int e = t128; e < per_box; e += 128)
              *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                         (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);
      ++i;
    }
    // --- the row's output (this CTA's 256 dims) and, from the first half, its LSE
    if (i > 0) ensure_pv(i - 1);
    const bool have_o = ok && i > 0;
    const float inv = (have_o && l > 0.f) ? __fdividef(1.f, l) : 0.f;
    const int64_t orow =
        (static_cast<int64_t>(qb * QT + tq) * p.batch + b) * p.n_q_heads + x * GU + h;
    uint16_t *dst = p.out + orow * D + dh * DH;
    if (have_o) tc_fence_after();
#pragma unroll 1
    for (int cb = 0; cb < DH / 32; ++cb) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_base + Cfg::O_COL + cb * 32, o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0.f;
      }
      if (row_ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
          pk.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
          pk.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
          pk.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
          *reinterpret_cast<uint4 *>(dst + cb * 32 + e) = pk;
        }
      }
    }
    if (row_ok && dh == 0 && p.lse != nullptr)
      p.lse[orow] = l > 0.f ? (m_ref + log2f(l)) * 0.69314718055994530942f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace gdattn
