// Split-KV decode attention over an fp8 e4m3 KV cache with per-row scales, on
// the 5th-generation tensor cores (tcgen05), for GQA pairs: two query heads per
// KV head, separate K and V, head_dim 256 (the Gemma-4 sliding-window
// geometry of tc_pair_decode.cuh, with half the cache bytes per token).
//
// A cache row (one token of one KV head) holds 256 e4m3 codes c_d and one float
// scale s; its values are c_d * s.  Scales are stored apart from the codes, per
// (sequence, KV head) and contiguous over the ring slots: scale[b][kv][slot].
//
// The codes go from TMA straight into kind::f8f6f4 MMAs; nothing is widened in
// shared memory, so shared-memory traffic per tile is the TMA write plus one
// MMA read.  The other operand of each product must then be e4m3 too:
//   * Q (bf16) is scaled per head by a power of two 2^a, so that its largest
//     element lies in [64, 128), and split into three e4m3 pieces, each one
//     holding 16 times the rounding error of the one before:
//         q 2^a = q1 + q2 / 16 + q3 / 256.
//     A bf16 value has 8 significant bits and a piece 4, so the split is exact
//     except for elements below 2^-6 of the head's largest, whose error stays
//     below 2^-18 of that largest element.
//   * The P.V weights w_t = p_t * s_v(t) (softmax weight times the V row's
//     scale) are split the same way after a power-of-two scaling 2^-e (below).
// The pieces are separate columns of the MMAs (rows of Q and of W), so each
// product gives three partial scores or outputs per head, combined in fp32 as
// X = X1 + X2 / 16 + X3 / 256.
//
// Per 64-token tile of a unit:
//
//   S^T[64 tok x 16]  = Kc[64 x 256] . Qp^T[256 x 16]     (M=64,  N=16, K=256: 8 MMAs)
//   O^T[256 d x 16]  += Vc^T[256 x 64] . Wp[64 x 16]       (M=128 x2, N=16, K=64: 4 MMAs)
//
// Column 2j + h of S^T and O^T is piece j of head h; rows 6-15 of Qp and Wp are
// zero.  The score of token t for head h is S_h(t) * s_k(t) * 2^-a_h * scale.
// K and V tiles arrive as 64-token x 128-code boxes with 128-byte swizzle: the
// K-major A operand of the first product and the MN-major A operand of the
// second (one box is exactly one 128-row block of M).
//
// Weight range: the softmax keeps the lazily moved reference of the bf16
// kernels (p_t <= 2^kTau) and, in the same way, a power-of-two exponent e with
// |s_v(t)| <= 2^(e-2) for every token seen so far.  A tile with a larger V
// scale raises e and rescales O in TMEM, as a reference move does, so
// |w_t 2^-e| <= 2^6, inside e4m3's range (448).  The output is O 2^e / L.
//
// Per-row scales of a tile (64 K scales, 64 V scales) are copied by the V
// producer with cp.async and counted on the V stage's barrier: the softmax
// reads them after the same wait a partial tile needs anyway, and the V stage
// is released only after its P.V, later than those reads.
//
// Q: TMA brings the pair's two bf16 rows; at the start of each segment the
// softmax warps convert them into the pieces buffer and release the bf16
// buffer; the QK warp waits for the pieces and releases the pieces buffer after
// the segment's last QK.
//
// Warp roles, the K/V rings, split planning and the in-kernel merge of split
// units are those of tc_pair_decode.cuh (no fused append here).  Every wait is
// bounded.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "combine.cuh"
#include "partition.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"
#include "tc_pair_decode.cuh"

namespace gdattn {

// Per-row scales of an fp8 cache: [B][Hkv][C] floats each (v_scale unused when
// K serves as V).
struct Fp8Scales {
  const float *k_scale;
  const float *v_scale;
};

struct TcPairFp8Config {
  static constexpr int D = 256;
  static constexpr int G = 2;
  static constexpr int N = 16;                        // MMA width (QK and P.V)
  static constexpr int TILE = 64;                     // tokens per tile
  static constexpr int NST = 6;                       // KV stages
  static constexpr int BOXB = TILE * 128;             // 64 tokens x 128 codes, 8 KiB
  static constexpr int KB = BOXB * (D / 128);         // K tile, 16 KiB
  static constexpr int STAGEB = 2 * KB;               // K tile then V tile, 32 KiB
  static constexpr int QPBOXB = N * 128;              // 16 piece rows x 128 codes, 2 KiB
  static constexpr int QPB = QPBOXB * (D / 128);      // Q pieces buffer, 4 KiB
  static constexpr int PB = N * 128;                  // weight pieces: 16 rows x 64 tokens (+64 unused)
  static constexpr int QB = G * D * 2;                // the pair's bf16 Q rows, 1 KiB
  static constexpr int SCB = 2 * TILE * 4;            // K then V scales of one tile
  static constexpr int OFF_QP = NST * STAGEB;         // 2 Q pieces buffers
  static constexpr int OFF_P = OFF_QP + 2 * QPB;      // 2 weight buffers
  static constexpr int OFF_Q = OFF_P + 2 * PB;        // 2 bf16 Q buffers
  static constexpr int OFF_SC = OFF_Q + 2 * QB;       // [NST] tile scales
  static constexpr int OFF_BAR = OFF_SC + NST * SCB;
  static constexpr int OFF_RED = OFF_BAR + 512;
  static constexpr int OFF_PART = OFF_RED + 256;      // the merger's own part
  static constexpr int PARTB = G * D * 4 + 64;        // O [G][D], then LSE [G]
  static constexpr int SMEM = OFF_PART + PARTB + 1024;
  static constexpr int kThreads = 288;
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr uint32_t S_COL = 0;                // 2 buffers x 2 partial sums x 16 columns
  static constexpr uint32_t O_COL = 64;               // 2 d-blocks x 16 columns
};
static_assert(TcPairFp8Config::TILE == TcConfig::TILE, "TileIter walks 64-token tiles");
static_assert(TcPairFp8Config::SMEM <= 227 * 1024, "shared memory budget");
static_assert(TcPairFp8Config::OFF_QP % 1024 == 0 && TcPairFp8Config::OFF_P % 1024 == 0,
              "swizzled operands need 1 KiB alignment");

// Byte offset of code (row n, token t < 64) in a K-major 128-byte-swizzled
// e4m3 tile: 16-byte chunk t / 16 of row n sits at chunk (t / 16) ^ (n % 8).
__device__ __forceinline__ uint32_t sw128_byte(int n, int t) {
  return static_cast<uint32_t>(n * 128 + ((((t >> 4) ^ (n & 7)) << 4) | (t & 15)));
}

// The V-scale exponent for a tile whose largest |s_v| is f: the smallest e
// with f <= 2^(e-2), kept within [-120, 120] so 2^e and 2^-e stay normal.
__device__ __forceinline__ int fp8_weight_exponent(float f) {
  if (!(f > 0.f)) return -120;
  const int e = ilogbf(f) + 3;
  return e < -120 ? -120 : (e > 120 ? 120 : e);
}

__global__ void __launch_bounds__(TcPairFp8Config::kThreads, 1)
    tc_pair_fp8_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                              const __grid_constant__ CUtensorMap vmap,
                              const __grid_constant__ CUtensorMap qmap, const TcParams p,
                              const Fp8Scales sc) {
  using Cfg = TcPairFp8Config;
  constexpr int G = Cfg::G, D = Cfg::D, NST = Cfg::NST, TILE = Cfg::TILE;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qp = smem + Cfg::OFF_QP;                                  // [2][QPB] Q pieces
  uint8_t *ps = smem + Cfg::OFF_P;                                   // [2][PB] weight pieces
  const uint16_t *qs = reinterpret_cast<const uint16_t *>(smem + Cfg::OFF_Q);  // [2][G][D]
  float *scl = reinterpret_cast<float *>(smem + Cfg::OFF_SC);       // [NST][2][TILE]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *kfull = bars;                 // [NST]  K TMA -> QK
  uint64_t *kempty = bars + NST;          // [NST]  QK -> K TMA
  uint64_t *vfull = bars + 2 * NST;       // [NST]  V TMA + scales -> P.V, softmax
  uint64_t *vempty = bars + 3 * NST;      // [NST]  P.V -> V TMA
  uint64_t *qfull = bars + 4 * NST;       // [2] Q TMA -> softmax (segment k in buffer k & 1)
  uint64_t *qempty = qfull + 2;           // [2] softmax (bf16 Q converted) -> Q TMA
  uint64_t *qready = qfull + 4;           // [2] softmax (pieces written) -> QK
  uint64_t *qpfree = qfull + 6;           // [2] QK (segment's last QK done) -> softmax
  uint64_t *sfull = qfull + 8;            // [2] QK -> softmax (S of tile i in buffer i & 1)
  uint64_t *sempty = qfull + 10;          // [2] softmax -> QK
  uint64_t *pfull = qfull + 12;           // [2] softmax -> P.V (weights of tile i)
  uint64_t *ofull = qfull + 14;           // [2] P.V -> softmax: P.V of tile i done
  uint64_t *oempty = qfull + 16;          // softmax -> P.V: O of a finished segment read out
  uint64_t *drain = qfull + 17;           // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(qfull + 19);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(qfull + 20);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(qfull + 21);      // 48 bytes
  uint32_t *sh_tag = reinterpret_cast<uint32_t *>(qfull + 27);
  static_assert((4 * NST + 28) * 8 <= 512, "barrier area");
  float *part_o = reinterpret_cast<float *>(smem + Cfg::OFF_PART);  // merger's own part [G][D]
  float *part_lse = part_o + G * D;                                  // [G]
  float *redmax = reinterpret_cast<float *>(smem + Cfg::OFF_RED);   // [4 warps][G]
  float *redsum = redmax + 4 * G;                                    // [4 warps][G]
  float *redsv = redsum + 4 * G;                                     // [4 warps]
  float *redq = redsv + 4;                                           // [4 warps]

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
      mbar_init(&qempty[s], 4);
      mbar_init(&qready[s], 4);
      mbar_init(&qpfree[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);
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
  const bool tagged = usplit && p.merge_in_kernel;
  const bool merger = tagged && crank == split_k - 1;
  uint64_t *tg_o = reinterpret_cast<uint64_t *>(p.ws_o);
  uint64_t *tg_lse = reinterpret_cast<uint64_t *>(p.ws_lse);
  if (warp == 2) {
    if (usplit)
      plan_unit_split(p.geo, c / split_k, crank, split_k, TILE, plan);
    else
      plan_chunk(p.geo, c, plan);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  if (c == 0 && warp == 2 && plan->bad) report_bad_seqlens<D>(p, lane);

  const int32_t C = p.geo.capacity;
  const int32_t Hkv = p.geo.units_per_seq;

  if (warp == 0) {
    // -------------------------------------------------------------- K, Q TMA
    // The schedule of the bf16 pair kernel: K tiles run ahead under the
    // dependency rule (rows before each sequence's newest one may be read
    // before the preceding kernel completes), and a segment's Q is loaded once
    // its buffer has been converted for segment k - 2.
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    uint32_t i = 0, seg_count = 0, q_issued = 0;
    int32_t qrows[8] = {};
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
        mbar_arrive_expect_tx(&qfull[qb], Cfg::QB);
        tma_load_2d(smem + Cfg::OFF_Q + qb * Cfg::QB, &qmap, 0, qrow, &qfull[qb]);
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
      if (first) {
        qrows[seg_count & 7] = it.seg.b * p.n_q_heads + it.seg.x * G;
        ++seg_count;
      }
      if (i >= NST || it.newest) ensure_waited();
      while (ok && waited && q_issued < seg_count && issue_q(false)) {
      }
      const int st = i % NST;
      if (i >= NST) {
        while (ok && q_issued <= stage_seg[st]) issue_q(true);
        if (ok && !mbar_wait(&kempty[st], ((i / NST) - 1) & 1, abort_flag, p.status)) ok = false;
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      stage_seg[st] = seg_count - 1;
      if (elect_one()) {
        uint8_t *kdst = stages + st * Cfg::STAGEB;
        mbar_arrive_expect_tx(&kfull[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 128; ++j)
          tma_load_4d(kdst + j * Cfg::BOXB, &kmap, 128 * j, it.seg.x, row, it.seg.b, &kfull[st],
                      pol);
      }
      __syncwarp();
      ++i;
    }
    ensure_waited();
    while (ok && q_issued < seg_count) issue_q(true);
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      mbar_wait(&kfull[f % NST], (f / NST) & 1, &no_abort, p.status);
    for (uint32_t k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
      mbar_wait(&qfull[k & 1], (k >> 1) & 1, &no_abort, p.status);
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK MMA
    const uint32_t idesc_qk = idesc_e4m3_f32(64, Cfg::N, false, false);
    const uint64_t kdesc = smem_desc_sw128(smem_u32(stages), 16, 1024);  // codes, K-major
    const uint64_t qdesc = smem_desc_sw128(smem_u32(qp), 16, 1024);      // Q pieces, K-major
    bool ok = true;
    uint32_t i = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (ok && it.next(C, row, ntok, first, last)) {
      if (first) {
        if (!mbar_wait(&qready[nseg & 1], (nseg >> 1) & 1, abort_flag, p.status)) ok = false;
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
      const uint64_t b0 = qdesc + ((qb * Cfg::QPB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int j = 0; j < D / 128; ++j) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 32 codes = 32 bytes of each row per MMA
            const uint64_t ad = a0 + ((j * Cfg::BOXB + kk * 32) >> 4);
            const uint64_t bd = b0 + ((j * Cfg::QPBOXB + kk * 32) >> 4);
            tc_mma_e4m3(tmem + Cfg::S_COL + sb * 32 + (kk & 1) * 16, ad, bd, idesc_qk,
                        (j != 0 || kk >= 2) ? 1u : 0u);
          }
        }
        tc_commit(&sfull[sb]);
        tc_commit(&kempty[st]);
        if (last) tc_commit(&qpfree[qb]);
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
    const uint32_t idesc_pv = idesc_e4m3_f32(128, Cfg::N, true, false);
    const uint64_t vdesc =
        smem_desc_sw128(smem_u32(stages + Cfg::KB), Cfg::BOXB, 1024);  // V^T codes, MN-major
    const uint64_t pdesc = smem_desc_sw128(smem_u32(ps), 16, 1024);    // weight pieces, K-major
    bool ok = true;
    uint32_t t = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (ok && it.next(C, row, ntok, first, last)) {
      bool w = mbar_wait(&pfull[t & 1], (t >> 1) & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[t % NST], (t / NST) & 1, abort_flag, p.status);
      if (w && first && nseg > 0) w = mbar_wait(oempty, (nseg - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      if (first) ++nseg;
      tc_fence_after();
      const uint64_t a0 = vdesc + (((t % NST) * Cfg::STAGEB) >> 4);
      const uint64_t b0 = pdesc + (((t & 1) * Cfg::PB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const uint64_t bd = b0 + ((k2 * 32) >> 4);  // 32 tokens = 32 bytes of each weight row
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            const uint64_t ad = a0 + ((jb * Cfg::BOXB + k2 * 32 * 128) >> 4);
            tc_mma_e4m3(tmem + Cfg::O_COL + jb * 16, ad, bd, idesc_pv,
                        (first && k2 == 0) ? 0u : 1u);
          }
        }
        tc_commit(&ofull[t & 1]);
        tc_commit(&vempty[t % NST]);
      }
      __syncwarp();
      ++t;
    }
    if (elect_one()) tc_commit(&drain[1]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[1], 0, &no_abort, p.status);
  } else if (warp == 7) {
    pair_merge_warp<G, D>(p, plan, c, lane, split_k, usplit, merger, tg_o, tg_lse, part_o,
                          part_lse);
  } else if (warp == 8) {
    // ------------------------------------------------ V loads and row scales
    // The K loads' schedule and dependency rule; a stage's V tile and the
    // tile's K and V scales complete its vfull barrier together.
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    uint32_t i = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    bool waited = false;
    while (ok && it.next(C, row, ntok, first, last)) {
      if (!waited && (i >= NST || it.newest)) {
        grid_dependency_wait();
        waited = true;
      }
      const int st = i % NST;
      if (i >= NST && !mbar_wait(&vempty[st], ((i / NST) - 1) & 1, abort_flag, p.status))
        ok = false;
      if (!__all_sync(0xffffffffu, ok)) break;
      const int64_t srow = (static_cast<int64_t>(it.seg.b) * Hkv + it.seg.x) * C + row;
      float *dst = scl + st * 2 * TILE;
#pragma unroll
      for (int j = lane; j < TILE; j += 32)
        if (j < ntok) {
          cp_async_4(dst + j, sc.k_scale + srow + j);
          cp_async_4(dst + TILE + j, sc.v_scale + srow + j);
        }
      cp_async_mbar_arrive(&vfull[st]);  // before the phase's last ordinary arrive below
      __syncwarp();
      if (elect_one()) {
        uint8_t *vdst = stages + st * Cfg::STAGEB + Cfg::KB;
        mbar_arrive_expect_tx(&vfull[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 128; ++j)
          tma_load_4d(vdst + j * Cfg::BOXB, &vmap, 128 * j, it.seg.x, row, it.seg.b, &vfull[st],
                      pol);
      }
      __syncwarp();
      ++i;
    }
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      mbar_wait(&vfull[f % NST], (f / NST) & 1, &no_abort, p.status);
  } else {
    // ---------------------------------------------------------- softmax
    grid_dependency_wait();  // outputs and workspace are written below
    uint32_t my_tag = 0;
    if (tagged && threadIdx.x == 64) my_tag = next_tag(__ldcg(p.epochs + c / split_k));
    const int t128 = threadIdx.x - 64;
    // M=64 puts tile token r in TMEM lane (r % 16) + 32 * (r / 16): lanes 0-15 of
    // each warp receive one token's scores.  Lanes 0-15 take head 0 of their
    // token, lanes 16-31 head 1 of the token of lane - 16.
    const int qd = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 16 * qd + (lane & 15);
    const int hd = lane >> 4;
    // Rows 6-15 of both pieces buffers and both weight buffers multiply columns
    // nobody reads; keep them zero (finite).
    for (int e = t128; e < 2 * 2 * 10 * 8; e += 128) {  // Q pieces: 2 buffers x 2 boxes x 10 rows
      const int bx = e / 80, r = e % 80;
      *reinterpret_cast<uint4 *>(qp + bx * Cfg::QPBOXB + (6 + (r >> 3)) * 128 + (r & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    for (int e = t128; e < 2 * 10 * 8; e += 128) {  // weights: 2 buffers x 10 rows
      const int bx = e / 80, r = e % 80;
      *reinterpret_cast<uint4 *>(ps + bx * Cfg::PB + (6 + (r >> 3)) * 128 + (r & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    float m_ref[G], lpart = 0.f;
    float cq[G];                   // scale * log2(e) (or / softcap) * 2^-a_h
    int ev = -127;                 // V-scale exponent e of the segment
    float sv_lim = 0.f, inv_e = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_ref[h] = -INFINITY;
      cq[h] = 0.f;
    }
    bool ok = true;
    uint32_t cons0 = 0, cons1 = 0;
    auto ensure_pv = [&](uint32_t t) {
      const uint32_t b = t & 1, ph = t >> 1;
      uint32_t &cons = b ? cons1 : cons0;
      if (cons <= ph) {
        if (ok && !mbar_wait(&ofull[b], cons & 1, abort_flag, p.status)) ok = false;
        ++cons;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    // Split segment k's bf16 Q rows into e4m3 pieces (thread: head t128 / 64,
    // elements 4 (t128 % 64) .. + 3).  Every softmax thread takes part, after
    // a failed wait too, so the named barrier stays matched.
    auto convert_q = [&](uint32_t k) {
      const uint32_t qb = k & 1;
      if (ok) ok = mbar_wait(&qfull[qb], (k >> 1) & 1, abort_flag, p.status);
      if (ok && k >= 2) ok = mbar_wait(&qpfree[qb], ((k >> 1) - 1) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      const int h = t128 >> 6, d0 = (t128 & 63) * 4;
      float q[4] = {0.f, 0.f, 0.f, 0.f};
      if (ok) {
        const uint2 raw = *reinterpret_cast<const uint2 *>(qs + qb * G * D + h * D + d0);
        q[0] = bf16lo(raw.x);
        q[1] = bf16hi(raw.x);
        q[2] = bf16lo(raw.y);
        q[3] = bf16hi(raw.y);
      }
      float am = fmaxf(fmaxf(fabsf(q[0]), fabsf(q[1])), fmaxf(fabsf(q[2]), fabsf(q[3])));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      if (lane == 0) redq[t128 >> 5] = am;
      named_bar_sync(1, 128);
      int a[G];
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float amax = fmaxf(redq[2 * hh], redq[2 * hh + 1]);
        int e = amax > 0.f ? 6 - ilogbf(amax) : 0;  // largest |q| 2^a in [64, 128)
        e = e < -120 ? -120 : (e > 120 ? 120 : e);
        a[hh] = e;
        cq[hh] = p.qscale * pow2f(-e);
      }
      if (ok) {
        const float s = pow2f(a[h]);
        float r[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) r[e] = q[e] * s;
        uint32_t word[3];
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const uint16_t lo = e4m3x2_rn(r[0], r[1]);
          const uint16_t hi = e4m3x2_rn(r[2], r[3]);
          word[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
          const float2 vlo = e4m3x2_to_float2(lo), vhi = e4m3x2_to_float2(hi);
          r[0] = (r[0] - vlo.x) * 16.f;
          r[1] = (r[1] - vlo.y) * 16.f;
          r[2] = (r[2] - vhi.x) * 16.f;
          r[3] = (r[3] - vhi.y) * 16.f;
        }
        uint8_t *dst = qp + qb * Cfg::QPB + (d0 >> 7) * Cfg::QPBOXB;
        const int t = d0 & 127;  // byte within the 128-byte row
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const int n = 2 * j + h;
          *reinterpret_cast<uint32_t *>(dst + n * 128 + ((((t >> 4) ^ (n & 7)) << 4) | (t & 15))) =
              word[j];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (ok && lane == 0) {
        mbar_arrive(&qempty[qb]);
        mbar_arrive(&qready[qb]);
      }
    };
    uint32_t i = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;

    while (it.next(C, row, ntok, first, last)) {
      const int sb = i & 1, pb = i & 1, st = i % NST;
      if (i >= 2) ensure_pv(i - 2);  // weight buffer pb is free again
      if (first) {
#pragma unroll
        for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY;
        lpart = 0.f;
        ev = -127;
        sv_lim = 0.f;
        convert_q(nseg++);
      }
      // --- scores of tile i: pieces of both partial accumulators
      float s0 = 0.f, s1 = 0.f;
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float v[16];
        tmem_ld8x2(tmem + lane_base + Cfg::S_COL + sb * 32, v);
        s0 = ((v[4] + v[12]) * 0.00390625f + (v[2] + v[10]) * 0.0625f) + (v[0] + v[8]);
        s1 = ((v[5] + v[13]) * 0.00390625f + (v[3] + v[11]) * 0.0625f) + (v[1] + v[9]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      const float other = __shfl_xor_sync(0xffffffffu, s1, 16);
      // The tile's row scales (and its V rows, cleared below when partial).
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&vfull[st], (i / NST) & 1, abort_flag, p.status));
      const bool valid = ok && tok < ntok;
      float sk = 0.f, sv = 0.f;
      if (valid) {
        sk = scl[st * 2 * TILE + tok];
        sv = scl[st * 2 * TILE + TILE + tok];
      }
      float x = ((lane < 16) ? s0 : other) * sk * (hd ? cq[1] : cq[0]);
      if (p.post != 0.f) x = p.post * tanhf(x);
      x = valid ? x : -INFINITY;
      const float asv = valid ? fabsf(sv) : 0.f;
      const float mine_ref = hd ? m_ref[1] : m_ref[0];
      // --- move the reference, or the V-scale exponent, only when outgrown
      if (named_bar_or(1, 128, x > mine_ref + kTau || asv > sv_lim)) {
        float tm = x, tv = asv;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) {
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
          tv = fmaxf(tv, __shfl_xor_sync(0xffffffffu, tv, off));
        }
        if ((lane & 15) == 0) redmax[qd * G + hd] = tm;
        if (lane == 0) redsv[qd] = tv;
        named_bar_sync(1, 128);
        float alpha[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float t = fmaxf(fmaxf(redmax[h], redmax[G + h]),
                                fmaxf(redmax[2 * G + h], redmax[3 * G + h]));
          const float mn = fmaxf(m_ref[h], t);
          alpha[h] = (m_ref[h] == -INFINITY) ? 0.f : exp2f(m_ref[h] - mn);
          m_ref[h] = mn;
        }
        const float tvm = fmaxf(fmaxf(redsv[0], redsv[1]), fmaxf(redsv[2], redsv[3]));
        int ev_new = fp8_weight_exponent(tvm);
        if (ev_new < ev) ev_new = ev;
        lpart *= hd ? alpha[1] : alpha[0];
        if (!first) {
          // O holds tiles < i in units of 2^ev: wait for the last of them, then
          // rescale it in TMEM to the new reference and exponent.
          ensure_pv(i - 1);
          if (ok) {
            const float beta = exp2f(static_cast<float>(ev - ev_new));
            const float f0 = alpha[0] * beta, f1 = alpha[1] * beta;
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
              float o[8];  // columns 2j + h: piece j of head h
              tmem_ld8(tmem + lane_base + Cfg::O_COL + jb * 16, o);
              o[0] *= f0;
              o[1] *= f1;
              o[2] *= f0;
              o[3] *= f1;
              o[4] *= f0;
              o[5] *= f1;
              tmem_st8_wait(tmem + lane_base + Cfg::O_COL + jb * 16, o);
            }
          }
        }
        ev = ev_new;
        sv_lim = pow2f(ev - 2);
        inv_e = pow2f(-ev);
      }
      // --- weight of this (token, head), as three e4m3 pieces in rows hd, 2 + hd, 4 + hd
      {
        const float mr = hd ? m_ref[1] : m_ref[0];
        const float pe = (x == -INFINITY) ? 0.f : exp2f(x - mr);
        lpart += pe;
        float w = valid ? pe * sv * inv_e : 0.f;  // |w| <= 2^6
        uint8_t *pbuf = ps + pb * Cfg::PB;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const uint16_t code = e4m3x2_rn(w, 0.f);
          pbuf[sw128_byte(2 * j + hd, tok)] = static_cast<uint8_t>(code & 0xFFu);
          w = (w - e4m3x2_to_float2(code).x) * 16.f;
        }
      }
      if (ok && ntok < TILE) {
        // V rows past the attended range hold other cache contents (possibly
        // NaN codes); they get weight 0, but 0 * NaN would still reach O.
        uint8_t *vt = stages + st * Cfg::STAGEB + Cfg::KB;
        const int per_box = (TILE - ntok) * 8;  // 16-byte chunks past row ntok
#pragma unroll 1
        for (int box = 0; box < D / 128; ++box)
          for (int e = t128; e < per_box; e += 128)
            *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                       (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);

      if (last) {
        // --- segment end: row sums, then the segment's last P.V, then O
        float ls = lpart;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if ((lane & 15) == 0) redsum[qd * G + hd] = ls;
        if (threadIdx.x == 64) *sh_tag = my_tag;
        named_bar_sync(1, 128);
        if (i >= 1) ensure_pv(i - 1);
        ensure_pv(i);
        const uint32_t tag = *sh_tag;
        const Segment &sg = it.seg;
        const bool single = sg.whole() && !usplit;
        const int64_t slot = static_cast<int64_t>(c) + sg.unit;
        const int h0 = sg.x * G;
        const float two_e = pow2f(ev < -120 ? -120 : ev);
        float L[G], f[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          L[h] = (redsum[h] + redsum[G + h]) + (redsum[2 * G + h] + redsum[3 * G + h]);
          f[h] = two_e * __fdividef(1.f, L[h]);
        }
        if (ok || (tagged && !merger)) {
          if (ok) tc_fence_after();
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (ok) tmem_ld8(tmem + lane_base + Cfg::O_COL + jb * 16, o);
            const int d = 128 * jb + 32 * qd + lane;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float val =
                  ((o[4 + h] * 0.00390625f + o[2 + h] * 0.0625f) + o[h]) * f[h];
              if (single)
                p.out[(static_cast<int64_t>(sg.b) * p.n_q_heads + h0 + h) * D + d] =
                    f32_to_bf16_rn(val);
              else if (merger)
                part_o[h * D + d] = val;
              else if (tagged)
                st_tagged(tg_o + (slot * G + h) * D + d, val, tag);
              else
                p.ws_o[(slot * G + h) * D + d] = val;
            }
          }
          if (ok) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(oempty);
          }
          if (qd == 0 && lane < G) {
            const float mr = lane ? m_ref[1] : m_ref[0];
            const float Lh = lane ? L[1] : L[0];
            const float lse_v = (mr + log2f(Lh)) * 0.69314718055994530942f;
            if (single) {
              if (p.lse != nullptr)
                p.lse[static_cast<int64_t>(sg.b) * p.n_q_heads + h0 + lane] = lse_v;
            } else if (merger) {
              part_lse[lane] = lse_v;
            } else if (tagged) {
              st_tagged(tg_lse + slot * G + lane, lse_v, tag);
            } else {
              p.ws_lse[slot * G + lane] = lse_v;
            }
          }
        }
        if (!single && p.merge_in_kernel && (!tagged || merger)) named_bar_sync(2, 160);
      }
      ++i;
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
