// Flash prefill on the tcgen05 pair geometry (two query heads per KV head,
// separate K and V, head_dim 256): a multi-token step of more than 8 tokens,
// for example a prompt chunk.  Token t of sequence b sits at position
// p = L_b - T + t and attends [max(0, p + 1 - w), p + 1) (w = 0: [0, p + 1)),
// the same step gdattn_decode_multi defines for any T ("Gemma support"
// pull request, Performance: flash prefill for head_dim 256).
//
// One CTA takes one block: 64 query tokens of one (sequence, KV head), i.e.
// 128 query rows (row 2 tq + h: token tq of the block, head h), which is one
// M = 128 MMA.  Per 64-token KV tile:
//
//   S[128 x 64]   = Q[128 x 256] . K_tile^T[256 x 64]        (M=128, N=64,  K=256)
//   O[128 x 256] += P_hi[128 x 64] . V_tile[64 x 256]
//                 + P_lo[128 x 64] . V_tile[64 x 256]         (M=128, N=256, K=64 x 2)
//
// Every TMEM lane is a query row, so each softmax thread owns a row: its 64
// scores, mask, running maximum, row sum and the rescale of its O row need no
// exchange with other threads.  P is stored as the bf16 weights plus their bf16
// remainders (two K = 64 halves of the P.V product), the decode kernels' weight
// split, so the weights keep about 16 significant bits on a bf16 MMA.  The
// reference maximum of a row moves lazily: only when a score exceeds it by
// more than 2^8, and then the thread rescales its O row in TMEM after the
// previous P.V completed.
//
// The block's KV range is [max(0, P0 + 1 - w), P0 + nq) for its first position
// P0 and nq valid tokens, cut into 64-token tiles at the ring's wrap (slot =
// position mod C); a tile's scores are masked per row to the row's own window
// and causal bound, and V rows past a partial tile's end are cleared, since
// they may hold anything.
//
// Shared memory (1 CTA per SM): two K/V stages (32 KiB each of K and V), the
// block's Q (64 KiB, loaded once), and the two P halves (16 KiB each): 224 KiB.
// TMEM: S double buffered (2 x 64 columns) and O (256 columns).
//
// Warp roles (256 threads): warp 0 loads Q and K, warp 3 loads V, warp 1 issues
// QK and owns TMEM, warp 2 issues P.V, warps 4-7 run the softmax (warp 4 + s
// reads TMEM sub-partition s: rows 32 s .. 32 s + 31).  Every wait is bounded
// like the decode kernels' (the status word reports an expiry).
#pragma once

#include <cstdint>
#include <cuda.h>

#include "partition.cuh"
#include "ptx.cuh"
#include "tc_pair_decode.cuh"
#include "tc_pair_multi_decode.cuh"

namespace gdattn {

struct TcPrefillConfig {
  static constexpr int D = 256;
  static constexpr int G = 2;
  static constexpr int QT = 64;                   // query tokens per block
  static constexpr int M = QT * G;                // 128 query rows
  static constexpr int TILE = 64;                 // KV tokens per tile
  static constexpr int NST = 2;                   // K/V stages
  static constexpr int BOXB = TILE * 128;         // 64 KV rows x 64 d: 8 KiB
  static constexpr int KB = BOXB * (D / 64);      // 32 KiB
  static constexpr int STAGEB = 2 * KB;           // K then V
  static constexpr int QBOXB = M * 128;           // 128 rows x 64 d: 16 KiB
  static constexpr int QB = QBOXB * (D / 64);     // 64 KiB
  static constexpr int PHB = M * 128;             // one P half: 128 rows x 64 KV bf16
  static constexpr int OFF_Q = NST * STAGEB;
  static constexpr int OFF_P = OFF_Q + QB;
  static constexpr int OFF_BAR = OFF_P + 2 * PHB;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int kThreads = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;            // 2 buffers x 64 columns
  static constexpr uint32_t O_COL = 256;          // 256 columns
};
static_assert(TcPrefillConfig::SMEM <= 227 * 1024, "shared memory budget");

struct PrefillParams {
  const int32_t *seqlens;
  uint16_t *out;       // bf16 [T][B][Hq][D]
  float *lse;          // [T][B][Hq] or null
  uint32_t *status;
  int32_t batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t tokens;      // T
  int32_t nblocks;     // ceil(T / 64)
  int32_t window;      // w (0: global)
  int32_t capacity;    // C
  float qscale;        // scale * log2(e), or scale / cap with a soft-cap
  float post;          // cap * log2(e), or 0
  int32_t test_withhold;
};

// KV tiles of one block: [lo, hi) in positions, cut at multiples of the tile
// size from lo and at the ring's wrap.
struct PrefillTiles {
  int32_t lo, hi, C;
  int32_t pos;  // next tile's first position
  __device__ __forceinline__ void init(int32_t lo_, int32_t hi_, int32_t C_) {
    lo = lo_;
    hi = hi_;
    C = C_;
    pos = lo_;
  }
  // Next tile: first position, its slot and the number of tokens.
  __device__ __forceinline__ bool next(int32_t &p0, int32_t &slot, int32_t &ntok) {
    if (pos >= hi) return false;
    p0 = pos;
    slot = pos % C;
    int32_t n = hi - pos < TcPrefillConfig::TILE ? hi - pos : TcPrefillConfig::TILE;
    if (slot + n > C) n = C - slot;  // stop at the ring's end; the next tile starts at slot 0
    ntok = n;
    pos += n;
    return true;
  }
};

// Block c -> (sequence b, KV head x, query block qb), heaviest causal blocks first.
__device__ __forceinline__ void prefill_block(const PrefillParams &p, int32_t c, int32_t &b,
                                              int32_t &x, int32_t &qb) {
  const int32_t nb = p.nblocks;
  const int32_t u = c / nb;
  qb = nb - 1 - (c - u * nb);
  b = u / p.n_kv_heads;
  x = u - b * p.n_kv_heads;
}

__global__ void __launch_bounds__(TcPrefillConfig::kThreads, 1)
    tc_pair_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                           const __grid_constant__ CUtensorMap vmap,
                           const __grid_constant__ CUtensorMap qmap, const PrefillParams p) {
  using Cfg = TcPrefillConfig;
  constexpr int D = Cfg::D, NST = Cfg::NST, TILE = Cfg::TILE;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint8_t *ps = smem + Cfg::OFF_P;  // P_hi, then P_lo
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *kfull = bars;          // [NST] K TMA -> QK
  uint64_t *kempty = bars + 2;     // [NST] QK -> K TMA
  uint64_t *vfull = bars + 4;      // [NST] V TMA -> P.V (and the softmax, for partial tiles)
  uint64_t *vempty = bars + 6;     // [NST] P.V -> V TMA
  uint64_t *sfull = bars + 8;      // [2] QK -> softmax
  uint64_t *sempty = bars + 10;    // [2] softmax -> QK
  uint64_t *qfull = bars + 12;     // Q TMA -> QK
  uint64_t *pfull = bars + 13;     // softmax -> P.V
  uint64_t *odone = bars + 14;     // P.V -> softmax: a tile's P.V completed (P free, O final)
  uint64_t *drain = bars + 15;     // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 17);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 18);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int32_t b, x, qb;
  prefill_block(p, static_cast<int32_t>(blockIdx.x), b, x, qb);
  const int32_t T = p.tokens;
  const int32_t L = __ldg(p.seqlens + b);
  const int32_t P0 = L - T + qb * Cfg::QT;  // position of the block's first token
  const int32_t nq = min(Cfg::QT, T - qb * Cfg::QT);
  int32_t lo = p.window > 0 ? P0 + 1 - p.window : 0;
  if (lo < 0) lo = 0;
  const int32_t hi = P0 + nq;  // positions up to the block's last token
  // The range must be in the ring (positions [L - C, L)) and the sequence long
  // enough for its T tokens.
  const bool bad = L < T || (hi > lo && lo < L - p.capacity);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
    }
    mbar_init(qfull, 1);
    mbar_init(pfull, 4);
    mbar_init(odone, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
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

  if (warp == 0 || warp == 3) {
    // ------------------------------------------------ K (+Q) or V loads
    // Q and the chunk's own cache rows come from the preceding kernels.
    grid_dependency_wait();
    const bool is_k = warp == 0;
    const uint64_t pol = l2_evict_first_policy();
    if (is_k && elect_one()) {
      mbar_arrive_expect_tx(qfull, Cfg::QB);
#pragma unroll
      for (int j = 0; j < D / 64; ++j)
        tma_load_3d(qs + j * Cfg::QBOXB, &qmap, 64 * j, b * p.n_q_heads + x * Cfg::G,
                    qb * Cfg::QT, qfull);
    }
    __syncwarp();
    bool ok = true;
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (ok && it.next(pos0, slot, ntok)) {
      const int st = i % NST;
      if (i >= NST)
        ok = mbar_wait(is_k ? &kempty[st] : &vempty[st], ((i / NST) - 1) & 1, abort_flag,
                       p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (!(p.test_withhold && is_k && i == 0) && elect_one()) {
        uint8_t *dst = stages + st * Cfg::STAGEB + (is_k ? 0 : Cfg::KB);
        uint64_t *bar = is_k ? &kfull[st] : &vfull[st];
        mbar_arrive_expect_tx(bar, Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(dst + j * Cfg::BOXB, is_k ? &kmap : &vmap, 64 * j, x, slot, b, bar, pol);
      }
      __syncwarp();
      ++i;
    }
    // Never leave with copies in flight into shared memory.
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      if (!(p.test_withhold && is_k && f == 0))
        mbar_wait(is_k ? &kfull[f % NST] : &vfull[f % NST], (f / NST) & 1, &no_abort, p.status);
    if (is_k) mbar_wait(qfull, 0, &no_abort, p.status);
  } else if (warp == 1) {
    // --------------------------------------------------------- QK MMA
    const uint32_t idesc = idesc_bf16_f32(128, TILE, false, false);
    const uint64_t qdesc = smem_desc_sw128(smem_u32(qs), 16, 1024);      // Q, K-major
    const uint64_t kdesc = smem_desc_sw128(smem_u32(stages), 16, 1024);  // K tile, K-major
    bool ok = mbar_wait(qfull, 0, abort_flag, p.status);
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (__all_sync(0xffffffffu, ok) && it.next(pos0, slot, ntok)) {
      const int st = i % NST, sb = i & 1;
      ok = mbar_wait(&kfull[st], (i / NST) & 1, abort_flag, p.status);
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
                        kdesc + ((st * Cfg::STAGEB + j * Cfg::BOXB + kk * 32) >> 4), idesc,
                        (j | kk) != 0);
        tc_commit(&sfull[sb]);
        tc_commit(&kempty[st]);
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
    const uint32_t idesc = idesc_bf16_f32(128, D, false, true);
    const uint64_t pdesc = smem_desc_sw128(smem_u32(ps), 16, 1024);  // P, K-major
    // V tile as the MN-major B operand: 64-d chunks Cfg::BOXB apart, 8 KV rows per 1 KiB
    const uint64_t vdesc = smem_desc_sw128(smem_u32(stages + Cfg::KB), Cfg::BOXB, 1024);
    bool ok = true;
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (ok && it.next(pos0, slot, ntok)) {
      const int st = i % NST;
      bool w = mbar_wait(pfull, i & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[st], (i / NST) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk)
            tc_mma_bf16(tmem + Cfg::O_COL, pdesc + ((half * Cfg::PHB + kk * 32) >> 4),
                        vdesc + ((st * Cfg::STAGEB + kk * 2048) >> 4), idesc,
                        !(i == 0 && half == 0 && kk == 0));
        tc_commit(odone);
        tc_commit(&vempty[st]);
      }
      __syncwarp();
      ++i;
    }
    if (elect_one()) tc_commit(&drain[1]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[1], 0, &no_abort, p.status);
  } else {
    // -------------------------------------------------------- softmax
    grid_dependency_wait();  // outputs are written below
    const int qd = warp & 3;
    const int t128 = threadIdx.x - 128;  // thread within the softmax warps
    const int r = 32 * qd + lane;        // this thread's query row (TMEM lane)
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tq = r >> 1, h = r & 1;
    const bool row_ok = tq < nq;
    const int32_t prow = P0 + tq;  // the row's position
    const int32_t rlo = p.window > 0 ? prow + 1 - p.window : INT32_MIN;
    if (bad && t128 == 0) atomicOr(p.status, kStatusSeqlen);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t done = 0;  // odone phases consumed
    auto ensure_pv = [&](uint32_t tt) {  // the P.V of tile tt has completed
      if (done <= tt) {
        if (ok && !mbar_wait(odone, done & 1, abort_flag, p.status)) ok = false;
        ++done;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    uint8_t *phi = ps + r * 128, *plo = ps + Cfg::PHB + r * 128;
    while (it.next(pos0, slot, ntok)) {
      const int sb = i & 1;
      float s[TILE];
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        tmem_ld64(tmem + lane_base + Cfg::S_COL + sb * TILE, s);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      // Column c is position pos0 + c: in the row's range when it is at most
      // the row's own position and (with a window) at least prow + 1 - w.
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < TILE; ++c) {
        const int32_t pos = pos0 + c;
        const bool valid = ok && row_ok && c < ntok && pos <= prow && pos >= rlo;
        float v = s[c] * p.qscale;
        if (p.post != 0.f) v = p.post * tanhf(v);
        s[c] = valid ? v : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      // --- move the reference of a row when a score outgrew it.  The TMEM
      // loads and stores are warp-wide, so a warp with any such row rescales
      // all its rows, by 1 where the reference stays.
      const bool mine = mx > m_ref + kTau;
      if (__any_sync(0xffffffffu, mine)) {
        float alpha = 1.f;
        if (mine) {
          alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
          l *= alpha;
          m_ref = mx;
        }
        if (i > 0) {
          // O holds tiles < i: wait for the last of them, then rescale.
          ensure_pv(i - 1);
          if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int cb = 0; cb < D / 32; ++cb) {
              float o[32];
              tmem_ld32(tmem + lane_base + Cfg::O_COL + cb * 32, o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] *= alpha;
              tmem_st32_wait(tmem + lane_base + Cfg::O_COL + cb * 32, o);
            }
          }
        }
      }
      // --- weights, as bf16 hi + lo rows of P (K-major, 128-byte swizzle)
      if (i > 0) ensure_pv(i - 1);  // P is single-buffered: tile i - 1's P.V read it
#pragma unroll
      for (int ch = 0; ch < TILE / 8; ++ch) {
        uint32_t wh[4], wl[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = s[8 * ch + 2 * e], bb = s[8 * ch + 2 * e + 1];
          const float pa = (a == -INFINITY) ? 0.f : exp2f(a - m_ref);
          const float pb = (bb == -INFINITY) ? 0.f : exp2f(bb - m_ref);
          l += pa + pb;
          wh[e] = pack_bf16x2(pa, pb);
          wl[e] = pack_bf16x2(pa - bf16lo(wh[e]), pb - bf16hi(wh[e]));
        }
        const uint32_t off = static_cast<uint32_t>((ch ^ (r & 7)) << 4);
        *reinterpret_cast<uint4 *>(phi + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
        *reinterpret_cast<uint4 *>(plo + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      }
      if (ok && ntok < TILE) {
        // V rows past the tile's end hold other slots (possibly NaN): clear them.
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&vfull[i % NST], (i / NST) & 1, abort_flag, p.status));
        if (ok) {
          uint8_t *vt = stages + (i % NST) * Cfg::STAGEB + Cfg::KB;
          const int per_box = (TILE - ntok) * 8;
#pragma unroll 1
          for (int box = 0; box < D / 64; ++box)
            for (int e = t128; e < per_box; e += 128)
              *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                         (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(pfull);
      ++i;
    }
    // --- the row's output: O / l, and its LSE.  The whole warp loads (the
    // TMEM loads are warp-wide); rows past the block's tokens store nothing.
    if (i > 0) ensure_pv(i - 1);
    const bool have_o = ok && i > 0;  // warp-uniform
    const float inv = (have_o && l > 0.f) ? __fdividef(1.f, l) : 0.f;
    const int64_t orow =
        (static_cast<int64_t>(qb * Cfg::QT + tq) * p.batch + b) * p.n_q_heads + x * Cfg::G + h;
    uint16_t *dst = p.out + orow * D;
    if (have_o) tc_fence_after();
#pragma unroll 1
    for (int cb = 0; cb < D / 32; ++cb) {
      float o[32];
      if (have_o) {
        tmem_ld32(tmem + lane_base + Cfg::O_COL + cb * 32, o);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = 0.f;  // nothing attended, or a wait failed
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
    if (row_ok && p.lse != nullptr)
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
