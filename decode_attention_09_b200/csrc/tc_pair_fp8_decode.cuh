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
// The pieces are separate columns of the MMAs (rows of Q and of W): piece j of
// head h is column 8 h + j, so each product gives three partial scores or
// outputs per head, combined in fp32 as X = X1 + X2 / 16 + X3 / 256.
//
// Per 128-token tile of a unit:
//
//   S^T[128 tok x 16]  = Kc[128 x 256] . Qp^T[256 x 16]    (M=128, N=16, K=256: 8 MMAs)
//   O^T[256 d x 16]   += Vc^T[256 x 128] . Wp[128 x 16]     (M=128 x2, N=16, K=128: 8 MMAs)
//
// Rows 8h+3 .. 8h+7 of Qp and Wp are zero.  The score of token t for head h is
// S_h(t) * s_k(t) * 2^-a_h * scale.
// K and V tiles arrive as 128-token x 128-code boxes with 128-byte swizzle: the
// K-major A operand of the first product and the MN-major A operand of the
// second (one box is exactly one 128-row block of M).
//
// The tile is twice the bf16 kernels' 64 tokens: with M = 128 every TMEM lane
// holds a token, so each softmax thread takes one token and both heads, and
// the softmax's fixed cost per tile (its waits, barrier and proxy fence) is
// spread over 128 tokens, which an fp8 tile streams in about the time a 64-token
// bf16 tile does.
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
// Warp roles (416 threads): warps 0, 1, 6 and 8 load K and Q, issue QK, issue
// P.V and load V as in tc_pair_decode.cuh; two softmax warpgroups, one per
// query head (warps 2-5: head 0, warps 9-12: head 1), share nothing but the
// tiles, so two softmax warps share each SM sub-partition; warp 7 has no role.
// Four weight buffers let the softmax run up to four tiles ahead of the P.V.
// Split planning and the tagged or counted merge of split units are those of
// the bf16 pair kernel, except that the softmax threads merge, each for the
// elements it computed, after their last tile (no fused append here).  Every
// wait is bounded.
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
  static constexpr int TILE = 128;                    // tokens per tile
  static constexpr int NST = 3;                       // KV stages
  static constexpr int BOXB = TILE * 128;             // 128 tokens x 128 codes, 16 KiB
  static constexpr int KB = BOXB * (D / 128);         // K tile, 32 KiB
  static constexpr int STAGEB = 2 * KB;               // K tile then V tile, 64 KiB
  static constexpr int QPBOXB = N * 128;              // 16 piece rows x 128 codes, 2 KiB
  static constexpr int QPB = QPBOXB * (D / 128);      // Q pieces buffer, 4 KiB
  static constexpr int PB = N * TILE;                 // weight pieces: 16 rows x 128 tokens
  static constexpr int NPB = 4;                       // weight buffers
  static constexpr int QB = G * D * 2;                // the pair's bf16 Q rows, 1 KiB
  static constexpr int SCB = 2 * TILE * 4;            // K then V scales of one tile
  static constexpr int OFF_QP = NST * STAGEB;         // 2 Q pieces buffers
  static constexpr int OFF_P = OFF_QP + 2 * QPB;      // NPB weight buffers
  static constexpr int OFF_Q = OFF_P + NPB * PB;      // 2 bf16 Q buffers
  static constexpr int OFF_SC = OFF_Q + 2 * QB;       // [NST] tile scales
  static constexpr int OFF_BAR = OFF_SC + NST * SCB;
  static constexpr int OFF_RED = OFF_BAR + 512;
  static constexpr int SMEM = OFF_RED + 256 + 1024;
  static constexpr int kSoftmaxThreads = 256;         // two warpgroups, one per head
  static constexpr int kThreads = 288 + 128;          // warps 0-8 as the bf16 pair kernel, 9-12
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr uint32_t S_COL = 0;                // 2 buffers x 2 partial sums x 16 columns
  static constexpr uint32_t O_COL = 64;               // 2 d-blocks x 16 columns
};
static_assert(TcPairFp8Config::SMEM <= 227 * 1024, "shared memory budget");
static_assert(TcPairFp8Config::OFF_QP % 1024 == 0 && TcPairFp8Config::OFF_P % 1024 == 0,
              "swizzled operands need 1 KiB alignment");

// Byte offset of code (row n, token t < 128) in a K-major 128-byte-swizzled
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
  using TileIter = TileIterT<TILE>;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qp = smem + Cfg::OFF_QP;                                  // [2][QPB] Q pieces
  uint8_t *ps = smem + Cfg::OFF_P;                                   // [NPB][PB] weight pieces
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
  constexpr int NPB = Cfg::NPB;
  uint64_t *pfull = qfull + 12;           // [NPB] softmax -> P.V (weights of tile i in buffer i % NPB)
  uint64_t *ofull = pfull + NPB;          // [NPB] P.V -> softmax: P.V of tile i done (barrier i % NPB)
  uint64_t *oempty = ofull + NPB;         // softmax -> P.V: O of a finished segment read out
  uint64_t *drain = oempty + 1;           // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(drain + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(drain + 3);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(drain + 4);       // 48 bytes
  uint32_t *sh_done = reinterpret_cast<uint32_t *>(drain + 10);    // a counted part's count
  static_assert((4 * NST + 12 + 2 * NPB + 3 + 11) * 8 <= 512, "barrier area");
  float *redmax = reinterpret_cast<float *>(smem + Cfg::OFF_RED);   // [G][4 warps]
  float *redsum = redmax + 4 * G;                                    // [G][4 warps]
  float *redsv = redsum + 4 * G;                                     // [G][4 warps]
  float *redq = redsv + 4 * G;                                       // [G][4 warps]

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
      mbar_init(&qempty[s], 8);  // arrivals: one per softmax warp
      mbar_init(&qready[s], 8);
      mbar_init(&qpfree[s], 1);
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 8);
    }
    for (int s = 0; s < NPB; ++s) {
      mbar_init(&pfull[s], 8);
      mbar_init(&ofull[s], 1);
    }
    mbar_init(oempty, 8);
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
      if (!(p.test_withhold && i == 0) && elect_one()) {
        uint8_t *kdst = stages + st * Cfg::STAGEB;
        mbar_arrive_expect_tx(&kfull[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 128; ++j)
          tma_load_4d(kdst + j * Cfg::BOXB, &kmap, 128 * j, it.seg.x, row,
                      cache_seq(p.geo, it.seg.b), &kfull[st],
                      pol);
      }
      __syncwarp();
      ++i;
    }
    ensure_waited();
    while (ok && q_issued < seg_count) issue_q(true);
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      if (!(p.test_withhold && f == 0)) mbar_wait(&kfull[f % NST], (f / NST) & 1, &no_abort, p.status);
    for (uint32_t k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
      mbar_wait(&qfull[k & 1], (k >> 1) & 1, &no_abort, p.status);
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK MMA
    const uint32_t idesc_qk = idesc_e4m3_f32(128, Cfg::N, false, false);
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
      bool w = mbar_wait(&pfull[t % NPB], (t / NPB) & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[t % NST], (t / NST) & 1, abort_flag, p.status);
      if (w && first && nseg > 0) w = mbar_wait(oempty, (nseg - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      if (first) ++nseg;
      tc_fence_after();
      const uint64_t a0 = vdesc + (((t % NST) * Cfg::STAGEB) >> 4);
      const uint64_t b0 = pdesc + (((t % NPB) * Cfg::PB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int k4 = 0; k4 < TILE / 32; ++k4) {
          const uint64_t bd = b0 + ((k4 * 32) >> 4);  // 32 tokens = 32 bytes of each weight row
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            const uint64_t ad = a0 + ((jb * Cfg::BOXB + k4 * 32 * 128) >> 4);
            tc_mma_e4m3(tmem + Cfg::O_COL + jb * 16, ad, bd, idesc_pv,
                        (first && k4 == 0) ? 0u : 1u);
          }
        }
        tc_commit(&ofull[t % NPB]);
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
    // no role: the softmax threads count and merge split parts
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
      const int32_t cb = cache_seq(p.geo, it.seg.b);
      const int64_t srow = (static_cast<int64_t>(cb) * Hkv + it.seg.x) * C + row;
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
          tma_load_4d(vdst + j * Cfg::BOXB, &vmap, 128 * j, it.seg.x, row, cb, &vfull[st],
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
    // Two warpgroups, one per query head of the pair (warps 2-5: head 0, warps
    // 9-12: head 1).  The heads share nothing but the tiles: each group has its
    // own reference max, V-scale exponent, row sums, MMA columns (8 h + j for
    // piece j) and named barrier, so the groups run independently and two
    // softmax warps share each SM sub-partition, hiding each other's latency.
    const int hw = warp >= 9 ? 1 : 0;                 // this group's head
    const uint32_t wg_bar = hw ? 3 : 1;               // its named barrier
    const int t128 = threadIdx.x - (hw ? 288 : 64);   // thread within the group
    const uint32_t hcol = 8 * hw;                     // its S / O columns and Q / W rows
    grid_dependency_wait();  // outputs and workspace are written below
    // This call's tag for the unit (the load completes while the tiles run).
    const int32_t unit = c / split_k;
    const int64_t slot0 = static_cast<int64_t>(unit) * split_k + unit;  // its part slots
    const uint32_t tag = tagged ? next_tag(__ldcg(p.epochs + unit)) : 0u;
    const bool has_part = plan->cs < plan->ce;
    if (tagged && !merger && !has_part) {  // an empty part: LSE -inf (each group its head)
      uint64_t *dst = tg_o + ((slot0 + crank) * G + hw) * D;
      for (int e = t128; e < D; e += 128) st_tagged(dst + e, 0.f, tag);
      if (t128 == 0) st_tagged(tg_lse + (slot0 + crank) * G + hw, -INFINITY, tag);
    }
    // M=128 puts tile token r in TMEM lane r: thread (warp, lane) takes token
    // 32 * (warp % 4) + lane (its TMEM sub-partition).
    const int qd = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 32 * qd + lane;
    // This thread's output elements: head hw, dims 32 qd + lane and 128 + 32 qd + lane.
    constexpr int NE = 2;
    int eh[NE], ed[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      eh[e] = hw;
      ed[e] = 128 * e + 32 * qd + lane;
    }
    float own_v[NE], own_l[NE];  // the merger's own part, merged after the loop
    bool has_own = false;
    // Rows 8h+3 .. 8h+7 of the pieces and weight buffers multiply columns
    // nobody reads; keep them zero (finite).
    for (int e = t128; e < 4 * 40; e += 128) {  // Q pieces: 2 buffers x 2 boxes x 5 rows
      const int bx = e / 40, r = e % 40;
      *reinterpret_cast<uint4 *>(qp + bx * Cfg::QPBOXB + (hcol + 3 + (r >> 3)) * 128 +
                                 (r & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int e = t128; e < NPB * 40; e += 128) {  // weights: NPB buffers x 5 rows
      const int bx = e / 40, r = e % 40;
      *reinterpret_cast<uint4 *>(ps + bx * Cfg::PB + (hcol + 3 + (r >> 3)) * 128 +
                                 (r & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    float *rmax = redmax + 4 * hw, *rsum = redsum + 4 * hw, *rsv = redsv + 4 * hw,
          *rq = redq + 4 * hw;  // [4 warps] each, per group
    float m_ref = -INFINITY, lpart = 0.f;
    float cq = 0.f;                // scale * log2(e) (or / softcap) * 2^-a
    int ev = -127;                 // V-scale exponent e of the segment
    float sv_lim = 0.f, inv_e = 0.f;
    bool ok = true;
    // Wait until the P.V of tile t has completed.  Completions are consumed in
    // tile order, and the P.V warp runs at most NPB tiles ahead of the
    // consumption, so a barrier never holds two unconsumed phases.
    uint32_t pv_done = 0;
    auto ensure_pv = [&](uint32_t t) {
      while (pv_done <= t) {
        if (ok && !mbar_wait(&ofull[pv_done % NPB], (pv_done / NPB) & 1, abort_flag, p.status))
          ok = false;
        ++pv_done;
      }
      ok = __all_sync(0xffffffffu, ok);
    };
    // Split this head's bf16 Q row of segment k into e4m3 pieces (thread:
    // elements 2 t128, 2 t128 + 1).  Every thread of the group takes part, after
    // a failed wait too, so the named barrier stays matched.
    auto convert_q = [&](uint32_t k) {
      const uint32_t qb = k & 1;
      if (ok) ok = mbar_wait(&qfull[qb], (k >> 1) & 1, abort_flag, p.status);
      if (ok && k >= 2) ok = mbar_wait(&qpfree[qb], ((k >> 1) - 1) & 1, abort_flag, p.status);
      ok = __all_sync(0xffffffffu, ok);
      const int d0 = 2 * t128;
      float q0 = 0.f, q1 = 0.f;
      if (ok) {
        const uint32_t raw = *reinterpret_cast<const uint32_t *>(qs + qb * G * D + hw * D + d0);
        q0 = bf16lo(raw);
        q1 = bf16hi(raw);
      }
      float am = fmaxf(fabsf(q0), fabsf(q1));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
      if (lane == 0) rq[t128 >> 5] = am;
      named_bar_sync(wg_bar, 128);
      const float amax = fmaxf(fmaxf(rq[0], rq[1]), fmaxf(rq[2], rq[3]));
      int a = amax > 0.f ? 6 - ilogbf(amax) : 0;  // largest |q| 2^a in [64, 128)
      a = a < -120 ? -120 : (a > 120 ? 120 : a);
      cq = p.qscale * pow2f(-a);
      if (ok) {
        const float s = pow2f(a);
        float r0 = q0 * s, r1 = q1 * s;
        uint8_t *dst = qp + qb * Cfg::QPB + (d0 >> 7) * Cfg::QPBOXB;
        const int t = d0 & 127;  // byte within the 128-byte row
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const uint16_t code = e4m3x2_rn(r0, r1);
          const int n = hcol + j;
          *reinterpret_cast<uint16_t *>(dst + n * 128 + ((((t >> 4) ^ (n & 7)) << 4) | (t & 15))) =
              code;
          const float2 back = e4m3x2_to_float2(code);
          r0 = (r0 - back.x) * 16.f;
          r1 = (r1 - back.y) * 16.f;
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
      const int sb = i & 1, pb = i % NPB, st = i % NST;
      if (i >= NPB) ensure_pv(i - NPB);  // weight buffer pb is free again
      if (first) {
        m_ref = -INFINITY;
        lpart = 0.f;
        ev = -127;
        sv_lim = 0.f;
        convert_q(nseg++);
      }
      // --- score of tile i: this head's pieces in both partial accumulators
      float sc = 0.f;
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float v0[4], v1[4];
        tmem_ld4(tmem + lane_base + Cfg::S_COL + sb * 32 + hcol, v0);
        tmem_ld4(tmem + lane_base + Cfg::S_COL + sb * 32 + 16 + hcol, v1);
        sc = ((v0[2] + v1[2]) * 0.00390625f + (v0[1] + v1[1]) * 0.0625f) + (v0[0] + v1[0]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      // The tile's row scales (and its V rows, cleared below when partial).
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&vfull[st], (i / NST) & 1, abort_flag, p.status));
      const bool valid = ok && tok < ntok;
      float sk = 0.f, sv = 0.f;
      if (valid) {
        sk = scl[st * 2 * TILE + tok];
        sv = scl[st * 2 * TILE + TILE + tok];
      }
      float x = sc * sk * cq;
      if (p.post != 0.f) x = p.post * tanhf(x);
      x = valid ? x : -INFINITY;
      const float asv = valid ? fabsf(sv) : 0.f;
      // --- move the reference, or the V-scale exponent, only when outgrown
      if (named_bar_or(wg_bar, 128, x > m_ref + kTau || asv > sv_lim)) {
        float tm = x, tv = asv;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
          tv = fmaxf(tv, __shfl_xor_sync(0xffffffffu, tv, off));
        }
        if (lane == 0) {
          rmax[qd] = tm;
          rsv[qd] = tv;
        }
        named_bar_sync(wg_bar, 128);
        const float t = fmaxf(fmaxf(rmax[0], rmax[1]), fmaxf(rmax[2], rmax[3]));
        const float mn = fmaxf(m_ref, t);
        const float alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mn);
        m_ref = mn;
        lpart *= alpha;
        const float tvm = fmaxf(fmaxf(rsv[0], rsv[1]), fmaxf(rsv[2], rsv[3]));
        int ev_new = fp8_weight_exponent(tvm);
        if (ev_new < ev) ev_new = ev;
        if (!first) {
          // O holds tiles < i in units of 2^ev: wait for the last of them, then
          // rescale this head's columns in TMEM to the new reference and exponent.
          ensure_pv(i - 1);
          if (ok) {
            const float f = alpha * exp2f(static_cast<float>(ev - ev_new));
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
              float o[4];  // columns hcol + j: piece j
              tmem_ld4(tmem + lane_base + Cfg::O_COL + jb * 16 + hcol, o);
              o[0] *= f;
              o[1] *= f;
              o[2] *= f;
              tmem_st4_wait(tmem + lane_base + Cfg::O_COL + jb * 16 + hcol, o);
            }
          }
        }
        ev = ev_new;
        sv_lim = pow2f(ev - 2);
        inv_e = pow2f(-ev);
      }
      // --- this token's weight as three e4m3 pieces, in weight rows hcol + j
      {
        const float pe = (x == -INFINITY) ? 0.f : exp2f(x - m_ref);
        lpart += pe;
        float w = valid ? pe * sv * inv_e : 0.f;  // |w| <= 2^6
        uint8_t *pbuf = ps + pb * Cfg::PB;
#pragma unroll
        for (int j = 0; j < 3; ++j) {
          const uint16_t code = e4m3x2_rn(w, 0.f);
          pbuf[sw128_byte(hcol + j, tok)] = static_cast<uint8_t>(code & 0xFFu);
          w = (w - e4m3x2_to_float2(code).x) * 16.f;
        }
      }
      if (ok && ntok < TILE) {
        // V rows past the attended range hold other cache contents (possibly
        // NaN codes); they get weight 0, but 0 * NaN would still reach O.  Group
        // h clears box h (d 128 h .. 128 h + 127).
        uint8_t *vt = stages + st * Cfg::STAGEB + Cfg::KB + hw * Cfg::BOXB;
        const int chunks = (TILE - ntok) * 8;  // 16-byte chunks past row ntok
        for (int e = t128; e < chunks; e += 128)
          *reinterpret_cast<uint4 *>(vt + (ntok + (e >> 3)) * 128 + (e & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);

      if (last) {
        // --- segment end: row sums, then the segment's last P.V, then O
        float ls = lpart;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if (lane == 0) rsum[qd] = ls;
        named_bar_sync(wg_bar, 128);
        if (i >= 1) ensure_pv(i - 1);
        ensure_pv(i);
        const Segment &sg = it.seg;
        const bool single = sg.whole() && !usplit;
        const int64_t slot = static_cast<int64_t>(c) + sg.unit;
        const int hq = sg.x * G + hw;  // this group's query head within the sequence
        const float L = (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
        const float f = pow2f(ev < -120 ? -120 : ev) * __fdividef(1.f, L);
        const float lse_v = (m_ref + log2f(L)) * 0.69314718055994530942f;
        float val[NE];
        if (ok) tc_fence_after();
#pragma unroll
        for (int jb = 0; jb < 2; ++jb) {
          float o[4] = {0.f, 0.f, 0.f, 0.f};
          if (ok) tmem_ld4(tmem + lane_base + Cfg::O_COL + jb * 16 + hcol, o);
          val[jb] = ((o[2] * 0.00390625f + o[1] * 0.0625f) + o[0]) * f;
        }
        if (ok) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(oempty);
        }
        const int64_t orow = static_cast<int64_t>(sg.b) * p.n_q_heads + hq;
        if (single) {
          if (ok) {
#pragma unroll
            for (int e = 0; e < NE; ++e) p.out[orow * D + ed[e]] = f32_to_bf16_rn(val[e]);
            if (p.lse != nullptr && t128 == 0) p.lse[orow] = lse_v;
          }
        } else if (merger) {  // merged with the other parts after the loop
          has_own = ok;
#pragma unroll
          for (int e = 0; e < NE; ++e) {
            own_v[e] = val[e];
            own_l[e] = lse_v;
          }
        } else if (tagged) {
          // Stored even after a failed wait, so the merger never waits for it in
          // vain (the status word reports the failure).
#pragma unroll
          for (int e = 0; e < NE; ++e) st_tagged(tg_o + (slot * G + hw) * D + ed[e], val[e], tag);
          if (t128 == 0) st_tagged(tg_lse + slot * G + hw, lse_v, tag);
        } else {
          // Counted parts: store the partial, count it with one acq_rel atomic
          // after a barrier of both groups, and the part that completes the
          // count merges the unit and resets its counter.  Counted after a
          // failed wait too, so the counters always return to zero.
          if (ok) {
#pragma unroll
            for (int e = 0; e < NE; ++e) p.ws_o[(slot * G + hw) * D + ed[e]] = val[e];
            if (t128 == 0) p.ws_lse[slot * G + hw] = lse_v;
          }
          named_bar_sync(2, Cfg::kSoftmaxThreads);  // every partial store before the count
          if (threadIdx.x == 64) *sh_done = atomic_add_acq_rel_gpu(p.counters + sg.unit, 1u);
          named_bar_sync(2, Cfg::kSoftmaxThreads);  // the acquire before every thread's reads
          int32_t cf, cl;
          unit_chunks(sg.unit_start, sg.n, plan->chunk, cf, cl);
          if (*sh_done == static_cast<uint32_t>(cl - cf)) {
            if (threadIdx.x == 64) p.counters[sg.unit] = 0u;
            PartMerge mg[NE];
            merge_counted_parts<G, D, NE>(p.ws_o, p.ws_lse, static_cast<int64_t>(cf) + sg.unit,
                                          cl - cf + 1, eh, ed, mg);
#pragma unroll
            for (int e = 0; e < NE; ++e) p.out[orow * D + ed[e]] = f32_to_bf16_rn(mg[e].out());
            if (p.lse != nullptr && t128 == 0) p.lse[orow] = mg[0].lse();
          }
          named_bar_sync(2, Cfg::kSoftmaxThreads);  // sh_done read before the next count
        }
      }
      ++i;
    }
    if (merger) {
      // --- the last part merges the unit: the other parts in part order, then
      // its own; clears what it consumed and advances the unit's epoch.
      PartMerge mg[NE];
      merge_tagged_parts<G, D, NE>(tg_o, tg_lse, slot0, split_k, tag, eh, ed, mg, p.status);
      if (has_own)
#pragma unroll
        for (int e = 0; e < NE; ++e) mg[e].add(own_l[e], own_v[e]);
      const int32_t b = unit / p.geo.units_per_seq, x = unit - b * p.geo.units_per_seq;
      const int64_t orow = static_cast<int64_t>(b) * p.n_q_heads + x * G + hw;
#pragma unroll
      for (int e = 0; e < NE; ++e) p.out[orow * D + ed[e]] = f32_to_bf16_rn(mg[e].out());
      if (p.lse != nullptr && t128 == 0) p.lse[orow] = mg[0].lse();
      named_bar_sync(wg_bar, 128);  // every thread of the group has read its head's LSE words
      if (t128 == 0) {
        for (int32_t r = 0; r + 1 < split_k; ++r)
          st_u64_volatile(tg_lse + (slot0 + r) * G + hw, 0ull);
        if (hw == 0) p.epochs[unit] = tag;  // no reader of the epoch is left in this call
      }
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
