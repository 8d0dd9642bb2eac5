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
// exchange with other threads.  P is stored as bf16 weights plus their bf16
// remainders (two K = 64 halves of the P.V product), like the decode kernels'
// weight split, so a weight keeps 2^-14 relative precision on a bf16 MMA.  The
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
// Shared memory (1 CTA per SM): a ring of three 32 KiB K tiles (a K tile is
// released as soon as its QK is done, so the K loads run further ahead), a ring
// of two V tiles, and the block's Q (64 KiB, loaded once): 224 KiB.  TMEM holds
// the rest: S double buffered (2 x 64 columns), P double buffered (each 32
// columns of bf16 pairs for the weights and 32 for their remainders, the A
// operand of P.V read from tensor memory), and O (256 columns).  With two P
// buffers the softmax of tile i waits only for the P.V of tile i - 2, so the
// tensor pipe is not left idle while P is written.
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
  static constexpr int NSTK = 3;                  // K ring
  static constexpr int NSTV = 2;                  // V ring
  static constexpr int BOXB = TILE * 128;         // 64 KV rows x 64 d: 8 KiB
  static constexpr int KB = BOXB * (D / 64);      // 32 KiB
  static constexpr int QBOXB = M * 128;           // 128 rows x 64 d: 16 KiB
  static constexpr int QB = QBOXB * (D / 64);     // 64 KiB
  static constexpr int OFF_V = NSTK * KB;
  static constexpr int OFF_Q = OFF_V + NSTV * KB;
  static constexpr int OFF_BAR = OFF_Q + QB;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr int kThreads = 256;
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr uint32_t S_COL = 0;            // 2 buffers x 64 columns
  static constexpr uint32_t P_COL = 128;          // 2 buffers x (32 hi + 32 lo) columns
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
  constexpr int D = Cfg::D, NSTK = Cfg::NSTK, NSTV = Cfg::NSTV, TILE = Cfg::TILE;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *ks = smem;                // K ring
  uint8_t *vs = smem + Cfg::OFF_V;   // V ring
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *kfull = bars;          // [NSTK] K TMA -> QK
  uint64_t *kempty = bars + 3;     // [NSTK] QK -> K TMA
  uint64_t *vfull = bars + 6;      // [NSTV] V TMA -> P.V (and the softmax, for partial tiles)
  uint64_t *vempty = bars + 8;     // [NSTV] P.V -> V TMA
  uint64_t *sfull = bars + 10;     // [2] QK -> softmax
  uint64_t *sempty = bars + 12;    // [2] softmax -> QK
  uint64_t *qfull = bars + 14;     // Q TMA -> QK
  uint64_t *pfull = bars + 15;     // [2] softmax -> P.V, per P buffer
  uint64_t *odone = bars + 17;     // [2] P.V -> softmax: the P.V of a tile using P buffer
                                   // i & 1 completed (that buffer free, O up to date)
  uint64_t *drain = bars + 19;     // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 21);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 22);

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
    for (int s = 0; s < NSTK; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < NSTV; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
    }
    mbar_init(qfull, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&pfull[s], 4);
      mbar_init(&odone[s], 1);
    }
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
      const int nst = is_k ? NSTK : NSTV;
      const int st = i % nst;
      if (i >= static_cast<uint32_t>(nst))
        ok = mbar_wait(is_k ? &kempty[st] : &vempty[st], ((i / nst) - 1) & 1, abort_flag,
                       p.status);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (!(p.test_withhold && is_k && i == 0) && elect_one()) {
        uint8_t *dst = (is_k ? ks : vs) + st * Cfg::KB;
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
    const uint32_t nst = is_k ? NSTK : NSTV;
    for (uint32_t f = i > nst ? i - nst : 0; f < i; ++f)
      if (!(p.test_withhold && is_k && f == 0))
        mbar_wait(is_k ? &kfull[f % nst] : &vfull[f % nst], (f / nst) & 1, &no_abort, p.status);
    if (is_k) mbar_wait(qfull, 0, &no_abort, p.status);
  } else if (warp == 1) {
    // --------------------------------------------------------- QK MMA
    const uint32_t idesc = idesc_bf16_f32(128, TILE, false, false);
    const uint64_t qdesc = smem_desc_sw128(smem_u32(qs), 16, 1024);      // Q, K-major
    const uint64_t kdesc = smem_desc_sw128(smem_u32(ks), 16, 1024);  // K tile, K-major
    bool ok = mbar_wait(qfull, 0, abort_flag, p.status);
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (__all_sync(0xffffffffu, ok) && it.next(pos0, slot, ntok)) {
      const int st = i % NSTK, sb = i & 1;
      ok = mbar_wait(&kfull[st], (i / NSTK) & 1, abort_flag, p.status);
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
    // V tile as the MN-major B operand: 64-d chunks Cfg::BOXB apart, 8 KV rows per 1 KiB
    const uint64_t vdesc = smem_desc_sw128(smem_u32(vs), Cfg::BOXB, 1024);
    bool ok = true;
    uint32_t i = 0;
    PrefillTiles it;
    it.init(lo_t, hi, C);
    int32_t pos0, slot, ntok;
    while (ok && it.next(pos0, slot, ntok)) {
      const int st = i % NSTV;
      const int pb = i & 1;
      bool w = mbar_wait(&pfull[pb], (i >> 1) & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[st], (i / NSTV) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        // A = P from tensor memory: 16 KV tokens are 8 columns of bf16 pairs.
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int kk = 0; kk < TILE / 16; ++kk)
            tc_mma_bf16_ta(tmem + Cfg::O_COL, tmem + Cfg::P_COL + pb * 64 + half * 32 + kk * 8,
                           vdesc + ((st * Cfg::KB + kk * 2048) >> 4), idesc,
                           !(i == 0 && half == 0 && kk == 0));
        tc_commit(&odone[pb]);
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
    if (bad && t128 == 0) atomicOr(p.status, kStatusSeqlen);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    // The P.V of tile tt (and so every earlier one: they complete in order) has
    // completed.  Each odone barrier's phases are consumed in order, and a
    // barrier never runs two phases ahead of its waiter (the P.V two tiles on
    // needs this warp's next P), so the parity waits cannot alias.
    uint32_t done0 = 0, done1 = 0;  // phases consumed on odone[0], odone[1]
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
      // Scores in log2 units (scale, then the soft-cap if there is one).
      if (p.post != 0.f) {
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] = p.post * tanhf(s[c] * p.qscale);
      } else {
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] *= p.qscale;
      }
      // Column c is position pos0 + c: in the row's range when it is at most
      // the row's own position and (with a window) at least prow + 1 - w, i.e.
      // c in [c_lo, c_hi).  A tile inside every row's range (all but the
      // window's first and the diagonal's tiles) needs no mask.
      const bool inside = ntok == TILE && nq == Cfg::QT && pos0 + TILE - 1 <= P0 &&
                          (p.window == 0 || pos0 >= P0 + Cfg::QT - p.window);
      if (!(inside && ok)) {
        int32_t c_lo = p.window > 0 ? prow + 1 - p.window - pos0 : 0;
        int32_t c_hi = prow - pos0 + 1 < ntok ? prow - pos0 + 1 : ntok;
        if (!(ok && row_ok)) c_hi = 0;
#pragma unroll
        for (int c = 0; c < TILE; ++c) s[c] = (c >= c_lo && c < c_hi) ? s[c] : -INFINITY;
      }
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < TILE; ++c) mx4[c & 3] = fmaxf(mx4[c & 3], s[c]);
      const float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
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
      // --- weights: the row's bf16 pairs (column j holds KV tokens 2j, 2j + 1)
      // and their remainders, into P buffer i & 1 in TMEM.  Both parts are
      // truncated to bf16 (upper halves of the fp32 bits; the remainder is
      // exact in fp32 before its own truncation), so the pair keeps a weight to
      // 2^-14 relative with integer operations only.  A row with no score yet
      // (reference -inf) has only masked columns here: 2^(-inf) = 0.
      const float mr = m_ref == -INFINITY ? 0.f : m_ref;
      float l4[4] = {0.f, 0.f, 0.f, 0.f};
      float wh[TILE / 2], wl[TILE / 2];
#pragma unroll
      for (int j = 0; j < TILE / 2; ++j) {
        const float pa = ex2_approx(s[2 * j] - mr);
        const float pb = ex2_approx(s[2 * j + 1] - mr);
        l4[j & 3] += pa + pb;
        const uint32_t ua = __float_as_uint(pa), ub = __float_as_uint(pb);
        const float ra = pa - __uint_as_float(ua & 0xFFFF0000u);
        const float rb = pb - __uint_as_float(ub & 0xFFFF0000u);
        wh[j] = __uint_as_float(__byte_perm(ua, ub, 0x7632));  // hi halves: a low, b high
        wl[j] = __uint_as_float(__byte_perm(__float_as_uint(ra), __float_as_uint(rb), 0x7632));
      }
      l += (l4[0] + l4[1]) + (l4[2] + l4[3]);
      if (i >= 2) ensure_pv(i - 2);  // the P.V of tile i - 2 read this P buffer
      if (ok) {
        tmem_st32_wait(tmem + lane_base + Cfg::P_COL + (i & 1) * 64, wh);
        tmem_st32_wait(tmem + lane_base + Cfg::P_COL + (i & 1) * 64 + 32, wl);
      }
      if (ok && ntok < TILE) {
        // V rows past the tile's end hold other slots (possibly NaN): clear them.
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&vfull[i % NSTV], (i / NSTV) & 1, abort_flag, p.status));
        if (ok) {
          uint8_t *vt = vs + (i % NSTV) * Cfg::KB;
          const int per_box = (TILE - ntok) * 8;
#pragma unroll 1
          for (int box = 0; box < D / 64; ++box)
            for (int e = t128; e < per_box; e += 128)
              *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                         (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();  // the cleared V rows, for the tensor core
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[i & 1]);
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
