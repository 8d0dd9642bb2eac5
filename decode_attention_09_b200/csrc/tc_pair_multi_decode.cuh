// Multi-token decode (a speculative-decoding verify step) on the tcgen05 pair
// geometry: two query heads per KV head, separate K and V, head_dim 256, with T
// query tokens per sequence (T <= 8) that attend causally within the window.
//
// Token t of sequence b sits at position p_t = L_b - T + t and attends
// [max(0, p_t + 1 - w), p_t + 1) (w = 0: [0, p_t + 1)).  The union of the T
// ranges is the last min(L_b, w + T - 1) positions, so the split planner and
// the tile iterator run over that union (the geometry's window is w + T - 1)
// and every cache byte of it is read once for all T tokens, instead of once
// per token.  Each score is then masked to its token's own range.
//
// The 2T query rows (row 2t + h: token t, head h) fill the QK MMA's 16 columns:
//
//   S^T[64 tok x 16]  = K_tile[64 x 256] . Q^T[256 x 16]   (M=64, N=16, K=256)
//   O^T[256 d x 32]  += V_tile^T[256 x 64] . P[64 x 32]     (M=128 x2, N=32, K=64)
//
// P row r holds query row r's bf16 weights (p_hi) and row 16 + r their
// remainders (p_lo), a two-piece weight split like the single-token pair
// kernel's (here both pieces truncated: 2^-14 relative), so O^T column r plus
// column 16 + r is row r's output (rows 2T..15 of both halves stay zero).  One 3-D TMA box {64 d, 2 heads, T tokens} per 64-d chunk brings
// a unit's 2T query rows from q [T][B][Hq][D] into the 16-row operand (rows 2T
// and up are never read back).
//
// S^T accumulates in one 16-column TMEM accumulator (two buffers), so a thread
// reads its token's 2T scores in one 16-column load.  Each softmax thread owns
// one cache token and one head and holds that head's T scores (lanes 0-15: head
// 0 of their token; lanes 16-31: head 1 of the token of lane - 16).  The
// reference max is kept per query row and moved lazily as in the single-token
// kernels.  P is triple buffered: the softmax of tile i needs only the P.V of
// tile i - 3 done.
//
// A part that covers its whole unit writes out and lse directly (token-major:
// [T][B][Hq][D] and [T][B][Hq]).  Split units are merged in the kernel by the
// softmax threads, each for the output elements it computed (2T rows x 2 dims):
// every part stores its partial (normalised O and LSE per row) and counts
// itself with one acq_rel atomic, and the part that completes the count folds
// all parts in slot order (its own from registers).  Nobody waits for another
// CTA, and the merge costs the last part one atomic and one round of loads of
// data already written.  No combine kernel runs.
//
// Warp roles (256 threads): warp 0 loads K (and Q), warp 7 loads V, warp 1
// issues QK and owns TMEM, warp 6 issues P.V, warps 2-5 run the softmax.  The
// stage ring, the dependency rule and the bounded waits are those of the
// single-token pair kernel.  The kernel is instantiated for each T.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "partition.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"
#include "tc_pair_decode.cuh"

namespace gdattn {

// The layer's own window (the geometry holds the union window w + T - 1).
struct MultiTokens {
  int32_t window;  // w (0: global)
};

struct TcPairMultiConfig {
  static constexpr int D = 256;
  static constexpr int G = 2;
  static constexpr int TMAX = 8;
  static constexpr int N = 16;                        // QK MMA width: 2T query rows
  static constexpr int NP = 32;                       // P.V MMA width: 2T hi + 2T lo rows
  static constexpr int TILE = 64;
  static constexpr int NST = 3;
  static constexpr int BOXB = TILE * 128;             // 8 KiB
  static constexpr int KB = BOXB * (D / 64);          // 32 KiB
  static constexpr int STAGEB = 2 * KB;               // K tile then V tile
  static constexpr int QBOXB = N * 128;               // 16 Q rows x 64 d
  static constexpr int QB = QBOXB * (D / 64);         // 8 KiB per Q buffer
  static constexpr int PB = NP * 128;                 // P: 32 rows x 64 tokens bf16, 4 KiB
  static constexpr int NPB = 3;                       // P buffers
  static constexpr int OFF_Q = NST * STAGEB;
  static constexpr int OFF_P = OFF_Q + 2 * QB;
  static constexpr int OFF_BAR = OFF_P + NPB * PB;
  static constexpr int OFF_RED = OFF_BAR + 512;
  static constexpr int SMEM = OFF_RED + 2 * 4 * N * 4 + 1024;
  static constexpr int kThreads = 256;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;                // 2 buffers x 16 columns
  static constexpr uint32_t O_COL = 128;              // 2 d-blocks x 32 columns
};
static_assert(TcPairMultiConfig::SMEM <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ void tma_load_3d(void *dst_smem, const CUtensorMap *map, int32_t c0,
                                            int32_t c1, int32_t c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst_smem)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// 32 consecutive columns; load and wait in one statement.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32_wait(uint32_t taddr, const float (&v)[32]) {
  uint32_t r[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(v[i]);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int T>
__global__ void __launch_bounds__(TcPairMultiConfig::kThreads, 1)
    tc_pair_multi_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                const __grid_constant__ CUtensorMap vmap,
                                const __grid_constant__ CUtensorMap qmap, const TcParams p,
                                const MultiTokens mt) {
  using Cfg = TcPairMultiConfig;
  constexpr int D = Cfg::D, NST = Cfg::NST, N = Cfg::N;
  constexpr int R = 2 * T;  // query rows of a unit
  static_assert(T >= 1 && T <= Cfg::TMAX, "1 to 8 tokens");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint8_t *ps = smem + Cfg::OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *kfull = bars;           // [NST]  K TMA -> QK
  uint64_t *kempty = bars + 3;      // [NST]  QK -> K TMA
  uint64_t *qfull = bars + 6;       // [2] TMA -> QK (Q of segment k in buffer k & 1)
  uint64_t *qempty = bars + 8;      // [2] QK -> TMA
  uint64_t *sfull = bars + 10;      // [2] QK -> softmax
  uint64_t *sempty = bars + 12;     // [2] softmax -> QK
  uint64_t *pfull = bars + 14;      // [NPB] softmax -> P.V
  uint64_t *ofull = bars + 17;      // [NPB] P.V -> softmax
  uint64_t *oempty = bars + 20;     // softmax -> P.V: O of a finished segment read out
  uint64_t *drain = bars + 21;      // [2] QK warp, P.V warp: all their MMAs done
  uint64_t *vfull = bars + 23;      // [NST]  V TMA -> P.V (and the softmax, for partial tiles)
  uint64_t *vempty = bars + 26;     // [NST]  P.V -> V TMA
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 29);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 30);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(bars + 31);  // 48 bytes
  uint32_t *sh_done = reinterpret_cast<uint32_t *>(bars + 37);  // a counted part's count
  float *redmax = reinterpret_cast<float *>(smem + Cfg::OFF_RED);  // [4 warps][16 rows]
  float *redsum = redmax + 4 * N;                                  // [4 warps][16 rows]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
    }
    for (int s = 0; s < Cfg::NPB; ++s) {
      mbar_init(&pfull[s], 4);
      mbar_init(&ofull[s], 1);
    }
    mbar_init(oempty, 4);
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
  const int32_t split_k = p.split_k > 1 ? p.split_k : 1;
  const bool usplit = split_k > 1;
  const int32_t crank = c % split_k;
  if (warp == 2) {
    if (usplit)
      plan_unit_split(p.geo, c / split_k, crank, split_k, Cfg::TILE, plan);
    else
      plan_chunk(p.geo, c, plan);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  if (c == 0 && warp == 2) {
    // An impossible length (L < T, or a range longer than the cache): flag it;
    // sequences that attend nothing get zero outputs and LSE -inf for every
    // token (the tokens of a shorter one before its start get them below).
    bool short_seq = false;
    for (int32_t b = lane; b < p.geo.batch; b += 32) short_seq |= __ldg(p.geo.seqlens + b) < T;
    if (__any_sync(0xffffffffu, short_seq) || plan->bad) {
      grid_dependency_wait();
      if (lane == 0) atomicOr(p.status, kStatusSeqlen);
      for (int32_t b = 0; b < p.geo.batch; ++b) {
        bool dummy = false;
        if (attended_count(__ldg(p.geo.seqlens + b), p.geo.window, p.geo.capacity, dummy) != 0)
          continue;
        for (int t = 0; t < T; ++t) {
          const int64_t base = (static_cast<int64_t>(t) * p.geo.batch + b) * p.n_q_heads;
          for (int e = lane; e < p.n_q_heads * D; e += 32) p.out[base * D + e] = 0;
          if (p.lse != nullptr)
            for (int e = lane; e < p.n_q_heads; e += 32) p.lse[base + e] = -INFINITY;
        }
      }
    }
  }

  const int32_t C = p.geo.capacity;

  if (warp == 0 || warp == 7) {
    // --------------------------------------------------- K (+Q) or V loads
    const bool is_k = warp == 0;
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    uint32_t i = 0, seg_count = 0, q_issued = 0;
    int32_t qrows[8] = {};       // (sequence, head-pair) row of segments whose Q is not issued
    uint32_t stage_seg[NST];
    auto issue_q = [&](bool block) -> bool {  // warp-uniform result
      const uint32_t qb = q_issued & 1;
      if (q_issued >= 2) {
        const uint32_t ph = ((q_issued >> 1) - 1) & 1;
        bool got = block ? mbar_wait(&qempty[qb], ph, abort_flag, p.status)
                         : mbar_try_wait(&qempty[qb], ph);
        if (!__all_sync(0xffffffffu, got)) {
          if (block) ok = false;
          return false;
        }
      }
      const int32_t qrow = qrows[q_issued & 7];
      if (elect_one()) {
        mbar_arrive_expect_tx(&qfull[qb], static_cast<uint32_t>(R) * 128 * (D / 64));
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_3d(qs + qb * Cfg::QB + j * Cfg::QBOXB, &qmap, 64 * j, qrow, 0, &qfull[qb]);
      }
      __syncwarp();
      ++q_issued;
      return true;
    };
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    bool waited = false;
    auto ensure_waited = [&]() {
      if (!waited) {
        grid_dependency_wait();
        waited = true;
      }
    };
    while (ok && it.next(C, row, ntok, first, last)) {
      // The newest T rows were written by this step's producers: read after the wait.
      const bool fresh = it.off + ntok > it.seg.n - T;
      if (is_k && first) {
        qrows[seg_count & 7] = it.seg.b * p.n_q_heads + it.seg.x * Cfg::G;
        ++seg_count;
      }
      if (i >= NST || fresh) ensure_waited();
      if (is_k) {
        while (ok && waited && q_issued < seg_count && issue_q(false)) {
        }
      }
      const int st = i % NST;
      if (i >= NST) {
        if (is_k) {
          while (ok && q_issued <= stage_seg[st]) issue_q(true);
          if (ok && !mbar_wait(&kempty[st], ((i / NST) - 1) & 1, abort_flag, p.status)) ok = false;
        } else {
          if (!mbar_wait(&vempty[st], ((i / NST) - 1) & 1, abort_flag, p.status)) ok = false;
        }
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      if (is_k) stage_seg[st] = seg_count - 1;
      if (!(p.test_withhold && is_k && i == 0) && elect_one()) {
        uint8_t *dst = stages + st * Cfg::STAGEB + (is_k ? 0 : Cfg::KB);
        uint64_t *bar = is_k ? &kfull[st] : &vfull[st];
        mbar_arrive_expect_tx(bar, Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(dst + j * Cfg::BOXB, is_k ? &kmap : &vmap, 64 * j, it.seg.x, row, it.seg.b,
                      bar, pol);
      }
      __syncwarp();
      ++i;
    }
    ensure_waited();
    if (is_k)
      while (ok && q_issued < seg_count) issue_q(true);
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      if (!(p.test_withhold && is_k && f == 0))
        mbar_wait(is_k ? &kfull[f % NST] : &vfull[f % NST], (f / NST) & 1, &no_abort, p.status);
    if (is_k)
      for (uint32_t k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
        mbar_wait(&qfull[k & 1], (k >> 1) & 1, &no_abort, p.status);
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK MMA
    const uint32_t idesc_qk = idesc_bf16_f32(64, N, false, false);
    const uint64_t kdesc = smem_desc_sw128(smem_u32(stages), 16, 1024);  // K tile, K-major
    const uint64_t qdesc = smem_desc_sw128(smem_u32(qs), 16, 1024);      // Q, K-major
    bool ok = true;
    uint32_t i = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (ok && it.next(C, row, ntok, first, last)) {
      if (first) {
        if (!mbar_wait(&qfull[nseg & 1], (nseg >> 1) & 1, abort_flag, p.status)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) break;
        ++nseg;
      }
      const uint32_t qb = (nseg - 1) & 1;
      const int st = i % NST, sb = i & 1;
      if (!mbar_wait(&kfull[st], (i / NST) & 1, abort_flag, p.status)) ok = false;
      if (ok && i >= 2 && !mbar_wait(&sempty[sb], ((i >> 1) - 1) & 1, abort_flag, p.status))
        ok = false;
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint64_t a0 = kdesc + ((st * Cfg::STAGEB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < D / 64; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = a0 + ((j * Cfg::BOXB + kk * 32) >> 4);
            const uint64_t bd = qdesc + ((qb * Cfg::QB + j * Cfg::QBOXB + kk * 32) >> 4);
            tc_mma_bf16(tmem + Cfg::S_COL + sb * 16, ad, bd, idesc_qk, j != 0 || kk != 0);
          }
        }
        tc_commit(&sfull[sb]);
        tc_commit(&kempty[st]);
        if (last) tc_commit(&qempty[qb]);
      }
      __syncwarp();
      ++i;
    }
    if (elect_one()) tc_commit(&drain[0]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[0], 0, &no_abort, p.status);
  } else if (warp == 6) {
    // ---------------------------------------------------------- P.V MMA
    const uint32_t idesc_pv = idesc_bf16_f32(128, Cfg::NP, true, false);
    const uint64_t vdesc =
        smem_desc_sw128(smem_u32(stages + Cfg::KB), Cfg::BOXB, 1024);  // V^T, MN-major
    const uint64_t pdesc = smem_desc_sw128(smem_u32(ps), 16, 1024);    // P, K-major
    bool ok = true;
    uint32_t t = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (ok && it.next(C, row, ntok, first, last)) {
      bool w = mbar_wait(&pfull[t % Cfg::NPB], (t / Cfg::NPB) & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[t % NST], (t / NST) & 1, abort_flag, p.status);
      if (w && first && nseg > 0) w = mbar_wait(oempty, (nseg - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      if (first) ++nseg;
      tc_fence_after();
      const uint64_t a0 = vdesc + (((t % NST) * Cfg::STAGEB) >> 4);
      const uint64_t b0 = pdesc + (((t % Cfg::NPB) * Cfg::PB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = b0 + ((kk * 32) >> 4);  // 16 tokens = 32 bytes of each P row
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            const uint64_t ad = a0 + ((2 * jb * Cfg::BOXB + kk * 2048) >> 4);
            tc_mma_bf16(tmem + Cfg::O_COL + jb * Cfg::NP, ad, bd, idesc_pv, !(first && kk == 0));
          }
        }
        tc_commit(&ofull[t % Cfg::NPB]);
        tc_commit(&vempty[t % NST]);
      }
      __syncwarp();
      ++t;
    }
    if (elect_one()) tc_commit(&drain[1]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[1], 0, &no_abort, p.status);
  } else {
    // ---------------------------------------------------------- softmax
    grid_dependency_wait();  // outputs and workspace are written below
    const int qd = warp & 3;
    const int t128 = threadIdx.x - 64;       // thread within the softmax warps
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 16 * qd + (lane & 15);  // tile token of this lane
    const int hd = lane >> 4;               // head of this lane: rows 2t + hd
    const int32_t unit_k = c / split_k;  // the unit of a part when units are cut into parts
    const bool has_part = plan->cs < plan->ce;
    // This thread's output elements: row r, dims 32 qd + lane and 128 + 32 qd + lane.
    int ed[2];
#pragma unroll
    for (int jb = 0; jb < 2; ++jb) ed[jb] = 128 * jb + 32 * qd + lane;
    // Output row of query row r of unit (b, x) in the token-major out / lse.
    auto out_row = [&](int32_t b, int32_t x, int r) -> int64_t {
      return (static_cast<int64_t>(r >> 1) * p.geo.batch + b) * p.n_q_heads + x * Cfg::G +
             (r & 1);
    };
    // One part of unit (b, x), whose parts sit in slots slot0 .. slot0 + np - 1,
    // this one in slot `own`: store it (unless a wait failed: has_own false;
    // an empty part stores LSE -inf), count it, and if it completes the count
    // fold every part in slot order and write the unit's outputs.  Counted
    // after a failed wait too, so the counters always return to zero.
    auto count_and_merge = [&](int32_t unit, int32_t b, int32_t x, int64_t slot0, int32_t np,
                               int64_t own, bool has_own, bool empty,
                               const float (&own_v)[2][R], const float (&own_l)[R]) {
      if (has_own) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) p.ws_o[(own * R + r) * D + ed[jb]] = own_v[jb][r];
          if (t128 == r) p.ws_lse[own * R + r] = own_l[r];
        }
      } else if (empty && t128 < R) {
        p.ws_lse[own * R + t128] = -INFINITY;
      }
      named_bar_sync(1, 128);  // every partial store before the count
      if (t128 == 0) *sh_done = atomic_add_acq_rel_gpu(p.counters + unit, 1u);
      named_bar_sync(1, 128);  // the acquire before every thread's reads
      if (*sh_done == static_cast<uint32_t>(np - 1)) {
        if (t128 == 0) p.counters[unit] = 0u;
        PartMerge mg[2][R];
        for (int32_t q = 0; q < np; ++q) {
          const int64_t sq = slot0 + q;
          float l[R], o0[R], o1[R];
          if (sq == own) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
              l[r] = has_own ? own_l[r] : -INFINITY;
              o0[r] = own_v[0][r];
              o1[r] = own_v[1][r];
            }
          } else {
#pragma unroll
            for (int r = 0; r < R; ++r) {
              l[r] = __ldcg(p.ws_lse + sq * R + r);
              o0[r] = __ldcg(p.ws_o + (sq * R + r) * D + ed[0]);
              o1[r] = __ldcg(p.ws_o + (sq * R + r) * D + ed[1]);
            }
          }
#pragma unroll
          for (int r = 0; r < R; ++r) {
            mg[0][r].add(l[r], o0[r]);
            mg[1][r].add(l[r], o1[r]);
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int64_t orow = out_row(b, x, r);
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) p.out[orow * D + ed[jb]] = f32_to_bf16_rn(mg[jb][r].out());
          if (t128 == 0 && p.lse != nullptr) p.lse[orow] = mg[0][r].lse();
        }
      }
      named_bar_sync(1, 128);  // sh_done read before the next count
    };
    // P row r holds query row r's bf16 weights and row N + r their remainders;
    // the rows of r >= R multiply O columns nobody reads: keep them zero.
    for (int e = t128; e < Cfg::NPB * Cfg::NP * 8; e += 128) {
      const int buf = e / (Cfg::NP * 8), r = (e % (Cfg::NP * 8)) >> 3;
      if ((r & (N - 1)) >= R)
        *reinterpret_cast<uint4 *>(ps + buf * Cfg::PB + r * 128 + (e & 7) * 16) =
            make_uint4(0u, 0u, 0u, 0u);
    }
    float m_ref[R];  // reference max of every query row (the same in all lanes)
    float lpart[T];  // this lane's share of the weight sum of row 2t + hd
#pragma unroll
    for (int r = 0; r < R; ++r) m_ref[r] = -INFINITY;
#pragma unroll
    for (int t = 0; t < T; ++t) lpart[t] = 0.f;
    bool ok = true;
    // ofull phases consumed on barriers 0, 1, 2.  Wait until the P.V of tile
    // tt has completed; phases are consumed in order and never lag by two, so
    // the parity waits cannot alias.
    uint32_t cons0 = 0, cons1 = 0, cons2 = 0;
    auto ensure_pv = [&](uint32_t tt) {
      const uint32_t b = tt % Cfg::NPB, ph = tt / Cfg::NPB;
      uint32_t &cons = b == 0 ? cons0 : (b == 1 ? cons1 : cons2);
      if (cons <= ph) {
        if (ok && !mbar_wait(&ofull[b], cons & 1, abort_flag, p.status)) ok = false;
        ++cons;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    uint32_t i = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (it.next(C, row, ntok, first, last)) {
      const int sb = i & 1, pb = i % Cfg::NPB;
      if (i >= Cfg::NPB) ensure_pv(i - Cfg::NPB);  // P buffer pb is free again
      if (first) {
#pragma unroll
        for (int r = 0; r < R; ++r) m_ref[r] = -INFINITY;
#pragma unroll
        for (int t = 0; t < T; ++t) lpart[t] = 0.f;
      }
      const Segment &sg = it.seg;
      const int32_t j = it.off + tok;  // offset of this lane's cache token in the unit's range
      // --- scores of tile i
      float s[T];
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      {
        // column r of S^T is query row r's score
        float acc[16];
        if (ok) {
          tc_fence_after();
          tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 16, acc);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sempty[sb]);
        } else {
#pragma unroll
          for (int r = 0; r < 16; ++r) acc[r] = 0.f;
        }
        // lanes 0-15 keep head 0 (even rows) of their token; lanes 16-31 take
        // head 1 (odd rows) of the token of lane - 16
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const float got = __shfl_xor_sync(0xffffffffu, acc[2 * t + 1], 16);
          s[t] = (lane < 16) ? acc[2 * t] : got;
        }
      }
      // Token t sits at offset n - T + t of the unit's range (positions
      // [L - n, L) are offsets [0, n)) and attends offsets up to its own, from
      // n - T + t + 1 - w on with a window w: this lane's cache token j is in
      // the range of the tokens t with j - (n - T) <= t <= j - (n - T + 1 - w)
      // (no upper bound without a window).
      const int32_t tmin = j - (sg.n - T);
      const int32_t tmax = mt.window > 0 ? j - (sg.n - T + 1 - mt.window) : T;
      const bool tok_ok = ok && tok < ntok;
      bool need = false;
#pragma unroll
      for (int t = 0; t < T; ++t) {
        const bool valid = tok_ok && t >= tmin && t <= tmax;
        float x = s[t] * p.qscale;
        if (p.post != 0.f) x = p.post * tanhf(x);
        s[t] = valid ? x : -INFINITY;
        const float mr = hd ? m_ref[2 * t + 1] : m_ref[2 * t];
        need |= s[t] > mr + kTau;
      }
      // --- move the references only when some score outgrew its own
      if (named_bar_or(1, 128, need)) {
#pragma unroll
        for (int t = 0; t < T; ++t) {
          float mx = s[t];
#pragma unroll
          for (int off = 1; off < 16; off <<= 1)
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
          if ((lane & 15) == 0) redmax[qd * N + 2 * t + hd] = mx;
        }
        named_bar_sync(1, 128);
        float alpha[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float tm = fmaxf(fmaxf(redmax[r], redmax[N + r]),
                                 fmaxf(redmax[2 * N + r], redmax[3 * N + r]));
          const float mn = fmaxf(m_ref[r], tm);
          alpha[r] = (m_ref[r] == -INFINITY) ? 0.f : exp2f(m_ref[r] - mn);
          m_ref[r] = mn;
        }
#pragma unroll
        for (int t = 0; t < T; ++t) lpart[t] *= hd ? alpha[2 * t + 1] : alpha[2 * t];
        if (!first) {
          // O holds tiles < i: wait for the last of them, then rescale it in TMEM.
          ensure_pv(i - 1);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
              float o[Cfg::NP];  // columns r (hi) and N + r (lo) of query row r
              tmem_ld32(tmem + lane_base + Cfg::O_COL + jb * Cfg::NP, o);
#pragma unroll
              for (int r = 0; r < R; ++r) {
                o[r] *= alpha[r];
                o[N + r] *= alpha[r];
              }
              tmem_st32_wait(tmem + lane_base + Cfg::O_COL + jb * Cfg::NP, o);
            }
          }
        }
      }
      // --- weights of this lane's (token, head): P rows 2t + hd and N + 2t + hd.
      // Both bf16 parts are truncations (the upper halves of the fp32 bits; the
      // remainder is exact in fp32 before its own), 2^-14 relative per weight.
      // A row with no score yet (reference -inf) has only masked scores: 2^-inf = 0.
      {
        uint8_t *pbuf = ps + pb * Cfg::PB;
#pragma unroll
        for (int t = 0; t < T; ++t) {
          const float mr0 = hd ? m_ref[2 * t + 1] : m_ref[2 * t];
          const float pe = ex2_approx(s[t] - (mr0 == -INFINITY ? 0.f : mr0));
          lpart[t] += pe;
          const uint32_t u = __float_as_uint(pe);
          const uint16_t hi = static_cast<uint16_t>(u >> 16);
          const uint16_t lo =
              static_cast<uint16_t>(__float_as_uint(pe - __uint_as_float(u & 0xFFFF0000u)) >> 16);
          *reinterpret_cast<uint16_t *>(pbuf + sw128_offset(2 * t + hd, tok)) = hi;
          *reinterpret_cast<uint16_t *>(pbuf + sw128_offset(N + 2 * t + hd, tok)) = lo;
        }
      }
      if (ok && ntok < Cfg::TILE) {
        // The V tile may still be in flight (it is loaded after K): wait for it.
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&vfull[i % NST], (i / NST) & 1, abort_flag, p.status));
      }
      if (ok && ntok < Cfg::TILE) {
        // V rows past the attended range may hold NaN: clear them (0 * NaN).
        uint8_t *vt = stages + (i % NST) * Cfg::STAGEB + Cfg::KB;
        const int per_box = (Cfg::TILE - ntok) * 8;
#pragma unroll 1
        for (int box = 0; box < D / 64; ++box)
          for (int e = t128; e < per_box; e += 128)
            *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                       (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);

      if (last) {
        // --- segment end: row sums, then O of the segment's last P.V
#pragma unroll
        for (int t = 0; t < T; ++t) {
          float ls = lpart[t];
#pragma unroll
          for (int off = 1; off < 16; off <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
          if ((lane & 15) == 0) redsum[qd * N + 2 * t + hd] = ls;
        }
        named_bar_sync(1, 128);
        if (i >= 1) ensure_pv(i - 1);
        ensure_pv(i);
        const bool single = sg.whole() && !usplit;
        const int64_t slot = static_cast<int64_t>(c) + sg.unit;
        // Normalised O and LSE of every row of this part.  A row that attends
        // nothing here (another token's positions only, or a token before the
        // sequence's start) has LSE -inf and weight 0 in any merge.
        float val[2][R], lse_v[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const float L = (redsum[r] + redsum[N + r]) + (redsum[2 * N + r] + redsum[3 * N + r]);
          const float inv = L > 0.f ? __fdividef(1.f, L) : 0.f;
          lse_v[r] = L > 0.f ? (m_ref[r] + log2f(L)) * 0.69314718055994530942f : -INFINITY;
          val[0][r] = inv;  // scaled below
          val[1][r] = inv;
        }
        if (ok) tc_fence_after();
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          float o[Cfg::NP];
#pragma unroll
          for (int e = 0; e < Cfg::NP; ++e) o[e] = 0.f;
          if (ok) tmem_ld32(tmem + lane_base + Cfg::O_COL + jb * Cfg::NP, o);
#pragma unroll
          for (int r = 0; r < R; ++r) val[jb][r] *= o[r] + o[N + r];
        }
        if (ok) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(oempty);
        }
        if (single) {
          if (ok) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const int64_t orow = out_row(sg.b, sg.x, r);
#pragma unroll
              for (int jb = 0; jb < 2; ++jb) p.out[orow * D + ed[jb]] = f32_to_bf16_rn(val[jb][r]);
              if (t128 == 0 && p.lse != nullptr) p.lse[orow] = lse_v[r];
            }
          }
        } else {
          int64_t slot0;
          int32_t np;
          if (usplit) {  // part crank of unit c / k sits in slot (c / k) * k + unit + crank
            slot0 = static_cast<int64_t>(unit_k) * split_k + unit_k;
            np = split_k;
          } else {
            int32_t cf, cl;
            unit_chunks(sg.unit_start, sg.n, plan->chunk, cf, cl);
            slot0 = static_cast<int64_t>(cf) + sg.unit;
            np = cl - cf + 1;
          }
          count_and_merge(sg.unit, sg.b, sg.x, slot0, np, slot, ok, false, val, lse_v);
        }
      }
      ++i;
    }
    if (usplit && !has_part) {
      // An empty part (the unit is shorter than its parts) still counts.
      float none_v[2][R], none_l[R];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        none_v[0][r] = none_v[1][r] = 0.f;
        none_l[r] = -INFINITY;
      }
      const int32_t b = unit_k / p.geo.units_per_seq, x = unit_k - b * p.geo.units_per_seq;
      const int64_t slot0 = static_cast<int64_t>(unit_k) * split_k + unit_k;
      count_and_merge(unit_k, b, x, slot0, split_k, slot0 + crank, false, true, none_v, none_l);
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
