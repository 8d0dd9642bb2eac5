// Split-KV decode attention on the 5th-generation tensor cores (tcgen05), for a
// GQA group of 16 (or 8) query heads over one KV head, head_dim 512: Gemma-4
// full-attention layers, where key == value (attention_k_eq_v), or, for models
// whose cached K and V differ, with a separate V cache.
//
// With 16 query rows per KV row the products are a dense contraction (32 flop
// per KV byte), far beyond what CUDA-core FMAs sustain at HBM speed, so both
// products run on tcgen05 with the accumulators in tensor memory (TMEM):
//
//   S^T[64 tok x 16 h]  = K_tile[64 x 512] . Q^T[512 x 16]   (M=64, N=16, K=512)
//   O^T[512 d x 32]    += V_tile^T[512 x 64] . P^T[64 x 32]  (M=128 x4, N=32, K=64)
//
// Consecutive MMAs never feed the same accumulator: S^T is split over four TMEM
// accumulators (one per 16-wide k-step within each 64-wide d-chunk, summed when
// S is read) and P.V is issued k-step by k-step across the four d-blocks, so the
// tensor pipe overlaps them instead of waiting on each accumulation.
//
// The weights are bf16 operands (A and B of one MMA share a type, and V is
// bf16), so each weight p is split into p_hi = bf16(p) and p_lo = bf16(p - p_hi):
// the 32 columns of P^T are the 16 heads' p_hi then their p_lo, and O^T for a head
// is the sum of its two column blocks.  That keeps the weights to ~2^-17
// relative error instead of 2^-8, which matters when a few large key rows
// dominate the weighted sum of values.
//
// K = V: the one 64-token tile in shared memory is the K-major A operand of the
// first product and the MN-major A operand of the second, so each cache byte
// crosses HBM once.  The tile arrives by TMA as eight 64x64 boxes with 128-byte
// swizzle, the canonical operand layout for both majors.  With a separate V the
// same ring of 64 KiB stages carries a tile's K and then its V in two
// consecutive ring slots: the K slot is released by its QK, the V slot by its
// P.V.
//
// A group of 8 query heads per KV head runs the same MMAs: Q rows 8-15 of a
// unit are the next unit's heads (or TMA zero fill), and their score columns,
// weights and outputs are computed but never stored.
//
// Softmax with a lazily moved reference: P = exp2(s - m_ref) with m_ref a
// running per-head reference that only moves when some score exceeds it by more
// than 2^kTau.  Until then O^T keeps accumulating in TMEM across tiles and the
// row sums stay in per-thread registers, so a tile costs one TMEM load of S, one
// barrier-with-vote and the P^T stores.  When the reference must move, the tile's
// exact per-head max is reduced, O^T in TMEM and the partial sums are rescaled
// by exp2(m_old - m_new), and the tile proceeds.  The result is exact: out is
// O/L and LSE is m_ref + log2 L for the final reference.
//
// Warp roles (224 threads): warp 0 issues TMA loads; warp 1 owns TMEM and issues
// the QK MMAs; warp 6 issues the P.V MMAs and releases KV stages (one elected
// lane each, so a P.V never waits behind the next tile's data); warps 2-5 run
// the softmax (TMEM sub-partition warp % 4).  S is double buffered in TMEM so
// the tensor core computes tile i+1 while tile i's softmax runs.  Every wait is
// bounded; on a timeout all roles fast-forward, drain their copies / MMAs and
// free TMEM.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "partition.cuh"
#include "ptx.cuh"

namespace gdattn {

struct TcParams {
  uint16_t *out;          // [B, Hq, D]
  float *lse;             // [B, Hq] or null
  float *ws_o;            // partial outputs [slots][G][D]
  float *ws_lse;          // partial lse [slots][G]
  uint32_t *status;
  uint32_t *counters;     // per unit: parts finished in this call (zero between calls)
  uint32_t *epochs;       // per unit: tag of the last call's tagged parts (see tc_pair_decode)
  int32_t merge_in_kernel;  // 1: the CTA finishing a unit's last part merges it
  int32_t split_k;        // > 1: unit u is cut into split_k whole-tile parts, part r on
                          // CTA u * split_k + r (units of even length); else flattened chunks
  Geometry geo;           // units_per_seq == n_kv_heads
  int32_t n_q_heads;
  float qscale;           // multiplies raw scores: scale*log2(e), or scale/softcap
  float post;             // softcap*log2(e), or 0 when soft-cap is off
  // Test hook (GDATTN_FLAG_TEST_WITHHOLD_KV): every CTA leaves its first KV tile
  // unloaded, so the wait for it runs out and the timeout path runs.
  int32_t test_withhold;
};
static_assert(sizeof(TcParams) == 112, "the test hook fits the parameter block's padding");

// Current-token append (k_new non-null): before the tile holding a unit's
// newest position is loaded, its row is copied from k_new / v_new
// ([B][Hkv][D]) into slot (L - 1) mod C of k_cache / v_cache.  A parameter of
// its own: the 16-head kernel without append keeps its smaller parameter block
// (a larger one measurably slowed that kernel's launches).
struct TcAppend {
  const uint16_t *k_new;
  const uint16_t *v_new;  // null when K serves as V
  uint16_t *k_cache;
  uint16_t *v_cache;
  int64_t batch_stride;   // cache elements from one sequence to the next
  int32_t n_kv_heads;
};

struct TcConfig {
  static constexpr int D = 512;
  static constexpr int G = 16;                        // QK MMA width: query rows per unit, padded
  static constexpr int TILE = 64;                     // tokens per tile
  static constexpr int NST = 3;                       // KV stages
  static constexpr int BOXB = TILE * 128;             // one 64-token x 64-d box
  static constexpr int STAGEB = BOXB * (D / 64);      // 64 KiB
  static constexpr int QB = G * D * 2;                // 16 KiB
  static constexpr int PB = TILE * 2 * G * 2;         // 4 KiB per P buffer: 64 tokens x 32 bf16
  static constexpr int OFF_Q = NST * STAGEB;
  static constexpr int OFF_P = OFF_Q + QB;
  static constexpr int OFF_BAR = OFF_P + 2 * PB;
  static constexpr int OFF_RED = OFF_BAR + 256;
  static constexpr int SMEM = OFF_RED + 2 * 4 * G * 4 + 1024;
  static constexpr int kThreads = 224;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;                // 2 buffers x 4 partial sums x 16 columns
  static constexpr uint32_t O_COL = 128;              // 4 d-blocks x (16 hi + 16 lo) columns
};

// The reference max moves when a score exceeds it by more than 2^kTau, so the
// weights stay below 256: no overflow in bf16 P, fp32 sums or O.
constexpr float kTau = 8.f;

using TileIter = TileIterT<TcConfig::TILE>;

// Reduce 16 per-lane values over the warp (op = max or sum): after it, lane l
// holds the reduction for value index (l >> 1) & 15.
template <bool MAX>
__device__ __forceinline__ float warp_reduce_scatter16(float (&r)[16], int lane) {
#pragma unroll
  for (int lev = 0; lev < 4; ++lev) {
    const int off = 16 >> lev, half = 8 >> lev;
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < half) {
        const float send = upper ? r[k] : r[k + half];
        const float keep = upper ? r[k + half] : r[k];
        const float got = __shfl_xor_sync(0xffffffffu, send, off);
        r[k] = MAX ? fmaxf(keep, got) : keep + got;
      }
  }
  const float got = __shfl_xor_sync(0xffffffffu, r[0], 1);
  return MAX ? fmaxf(r[0], got) : r[0] + got;
}

// Ring slots of tile t: K = V in one slot (t), or K in slot 2t and V in 2t + 1.
template <bool SHARED>
__device__ __forceinline__ uint32_t k_slot(uint32_t t) {
  return SHARED ? t : 2 * t;
}
template <bool SHARED>
__device__ __forceinline__ uint32_t v_slot(uint32_t t) {
  return SHARED ? t : 2 * t + 1;
}

// SHARED: K serves as V (vmap is not read).  GU: query heads per unit (16 or
// 8; the MMAs always take 16 rows).  APPEND: the current token's rows are
// written into the cache first (TcAppend).
template <bool APPEND, bool SHARED, int GU>
__device__ __forceinline__ void tc_decode_body(const CUtensorMap &kmap, const CUtensorMap &vmap,
                                               const CUtensorMap &qmap, const TcParams &p,
                                               const TcAppend &ap) {
  using Cfg = TcConfig;
  constexpr int G = Cfg::G, D = Cfg::D, NST = Cfg::NST;
  static_assert(GU == 16 || GU == 8, "query heads per unit");

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
  uint64_t *sfull = bars + 8;       // [2] MMA -> softmax (S of tile i in buffer i & 1)
  uint64_t *sempty = bars + 10;     // [2] softmax -> MMA
  uint64_t *pfull = bars + 12;      // [2] softmax -> MMA (P of tile i in buffer i & 1)
  uint64_t *ofull = bars + 14;      // [2] MMA -> softmax: P.V of tile i done (barrier i & 1)
  uint64_t *oempty = bars + 16;     // softmax -> MMA: O of a finished segment read out
  uint64_t *drain = bars + 17;      // [2] QK warp, P.V warp: all their MMAs done
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 19);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 20);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(bars + 21);  // 48 bytes, ends before +256
  float *redmax = reinterpret_cast<float *>(smem + Cfg::OFF_RED);  // [4 warps][16]
  float *redsum = redmax + 4 * G;                                  // [4 warps][16]

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
    }
    mbar_init(oempty, 4);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&kmap);
    if (!SHARED) prefetch_tensormap(&vmap);
    prefetch_tensormap(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  grid_launch_dependents();
  // The split plan reads only seqlens, so it (and the producer's first KV
  // loads below) may run before the preceding kernel has completed; every other
  // global access waits for it (griddepcontrol.wait) in the role that makes it.
  const int32_t split_k = p.split_k > 1 ? p.split_k : 1;
  const bool usplit = split_k > 1;  // unit c / split_k, part c % split_k (see TcParams)
  if (warp == 2) {
    if (usplit)
      plan_unit_split(p.geo, c / split_k, c % split_k, split_k, Cfg::TILE, plan);
    else
      plan_chunk(p.geo, c, plan);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_smem;

  if (c == 0 && warp == 2 && plan->bad) {
    grid_dependency_wait();
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
    // The whole warp walks the schedule and waits (values stay warp-uniform);
    // one elected lane issues the copies.  A new segment's Q may only replace
    // the previous one once that segment's last QK is done; instead of stalling
    // the KV stream on it, the Q load is issued as soon as that has happened,
    // and at the latest before waiting on a stage whose release needs it.
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    uint32_t n = 0, seg_count = 0, q_issued = 0;  // n: ring slots filled
    int32_t qrows[8] = {};       // Q rows of segments whose Q is not issued yet
    uint32_t stage_seg[NST];     // segment of the tile whose K or V went into each stage
    auto issue_q = [&](bool block) -> bool {  // warp-uniform result
      if (q_issued > 0) {
        bool got = block ? mbar_wait(qempty, (q_issued - 1) & 1, abort_flag, p.status)
                         : mbar_try_wait(qempty, (q_issued - 1) & 1);
        if (!__all_sync(0xffffffffu, got)) {
          if (block) ok = false;
          return false;
        }
      }
      const int32_t qrow = qrows[q_issued & 7];
      if (elect_one()) {
        mbar_arrive_expect_tx(qfull, Cfg::QB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_2d(qs + j * (G * 128), &qmap, 64 * j, qrow, qfull);
      }
      __syncwarp();
      ++q_issued;
      return true;
    };
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    // Until the preceding kernel completes, only cache rows of positions before
    // each sequence's newest one are read (earlier decode steps wrote them);
    // q and the newest row are loaded after griddepcontrol.wait.
    bool waited = false;
    auto ensure_waited = [&]() {
      if (!waited) {
        grid_dependency_wait();
        waited = true;
      }
    };
    while (ok && it.next(C, row, ntok, first, last)) {
      if (first) {
        // At most NST + 1 segments can be pending (see the wait below), so 8 slots do.
        qrows[seg_count & 7] = it.seg.b * p.n_q_heads + it.seg.x * GU;
        ++seg_count;
      }
#pragma unroll
      for (int part = 0; part < (SHARED ? 1 : 2); ++part) {  // K (= V), then a separate V
        if (n >= NST || it.newest) ensure_waited();
        while (ok && waited && q_issued < seg_count && issue_q(false)) {
        }
        const int st = n % NST;
        if (n >= NST) {
          // The slot in this stage is released by a QK or a P.V, which needs its Q.
          while (ok && q_issued <= stage_seg[st]) issue_q(true);
          if (ok && !mbar_wait(&empty[st], ((n / NST) - 1) & 1, abort_flag, p.status)) ok = false;
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        stage_seg[st] = seg_count - 1;
        if (APPEND && it.newest) {  // append the current token's row first
          const int32_t slot = (it.seg.first_pos + it.seg.n - 1) % C;
          const int64_t row_off = it.seg.b * ap.batch_stride +
                                  (static_cast<int64_t>(slot) * ap.n_kv_heads + it.seg.x) * D;
          const int64_t new_off =
              (static_cast<int64_t>(it.seg.b) * ap.n_kv_heads + it.seg.x) * D;
          if (part == 0)
            append_row(ap.k_cache + row_off, ap.k_new + new_off, D, lane);
          else
            append_row(ap.v_cache + row_off, ap.v_new + new_off, D, lane);
        }
        const CUtensorMap *map = part == 0 ? &kmap : &vmap;
        if (!(p.test_withhold && n == 0) && elect_one()) {
          mbar_arrive_expect_tx(&full[st], Cfg::STAGEB);
#pragma unroll
          for (int j = 0; j < D / 64; ++j)
            tma_load_4d(stages + st * Cfg::STAGEB + j * Cfg::BOXB, map, 64 * j, it.seg.x, row,
                        cache_seq(p.geo, it.seg.b), &full[st], pol);
        }
        __syncwarp();
        ++n;
      }
    }
    ensure_waited();
    while (ok && q_issued < seg_count) issue_q(true);
    // Drain: never leave with copies in flight into shared memory.
    volatile int no_abort = 0;
    for (uint32_t f = n > NST ? n - NST : 0; f < n; ++f)
      if (!(p.test_withhold && f == 0)) mbar_wait(&full[f % NST], (f / NST) & 1, &no_abort, p.status);
    if (q_issued > 0) mbar_wait(qfull, (q_issued - 1) & 1, &no_abort, p.status);
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK MMA
    // Converged warp: descriptors are warp-uniform, one elected lane issues
    // every MMA and commit (commits track that lane's MMAs).
    const uint32_t idesc_qk = idesc_bf16_f32(64, 16, false, false);
    // Base descriptors; an operand at byte offset o from a base is base + (o >> 4)
    // (the 14-bit start field holds address >> 4 and never carries: smem < 256 KiB).
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
        if (!mbar_wait(qfull, nseg & 1, abort_flag, p.status)) ok = false;
        if (!__all_sync(0xffffffffu, ok)) break;
        ++nseg;
      }
      const uint32_t ks = k_slot<SHARED>(i);
      const int st = ks % NST, sb = i & 1;
      if (!mbar_wait(&full[st], (ks / NST) & 1, abort_flag, p.status)) ok = false;
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
            const uint64_t bd = qdesc + ((j * (G * 128) + kk * 32) >> 4);
            tc_mma_bf16(tmem + Cfg::S_COL + sb * 64 + kk * 16, ad, bd, idesc_qk, j != 0);
          }
        }
        tc_commit(&sfull[sb]);
        if (!SHARED) tc_commit(&empty[st]);  // a separate K slot: its only reader is done
        if (last) tc_commit(qempty);
      }
      __syncwarp();
      ++i;
    }
    // Drain: wait until every issued MMA has completed before TMEM is freed.
    if (elect_one()) tc_commit(&drain[0]);
    __syncwarp();
    volatile int no_abort = 0;
    mbar_wait(&drain[0], 0, &no_abort, p.status);
  } else if (warp == 6) {
    // ---------------------------------------------------------- P.V MMA
    const uint32_t idesc_pv = idesc_bf16_f32(128, 32, true, true);
    const uint64_t vdesc = smem_desc_sw128(smem_u32(stages), Cfg::BOXB, 1024);  // V^T, MN-major
    const uint64_t pdesc = smem_desc(smem_u32(ps), 4096, 512, 4);               // P^T, MN-major SW64
    bool ok = true;
    uint32_t t = 0, nseg = 0;
    TileIter it;
    it.init(p.geo, *plan);
    int32_t row, ntok;
    bool first, last;
    while (ok && it.next(C, row, ntok, first, last)) {
      const uint32_t vs = v_slot<SHARED>(t);
      bool w = mbar_wait(&pfull[t & 1], (t >> 1) & 1, abort_flag, p.status);
      if (!SHARED && w) w = mbar_wait(&full[vs % NST], (vs / NST) & 1, abort_flag, p.status);
      // A segment's first P.V overwrites O: the previous segment must be read out.
      if (w && first && nseg > 0) w = mbar_wait(oempty, (nseg - 1) & 1, abort_flag, p.status);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      if (first) ++nseg;
      tc_fence_after();
      const uint64_t a0 = vdesc + (((vs % NST) * Cfg::STAGEB) >> 4);
      const uint64_t b0 = pdesc + (((t & 1) * Cfg::PB) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // P^T: MN-major, 64-byte swizzle, a token row of 32 bf16 = 64 B; 16 tokens
          // per k-step = two 512-byte atoms.
          const uint64_t bd = b0 + ((kk * 1024) >> 4);
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const uint64_t ad = a0 + ((2 * jb * Cfg::BOXB + kk * 2048) >> 4);
            tc_mma_bf16(tmem + Cfg::O_COL + jb * 32, ad, bd, idesc_pv, !(first && kk == 0));
          }
        }
        tc_commit(&ofull[t & 1]);
        tc_commit(&empty[vs % NST]);
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
    // M=64 puts tile token r in TMEM lane (r % 16) + 32 * (r / 16): lanes 0-15 of
    // each warp receive one token's 16 scores.  Lanes 16-31 take heads 8-15 of
    // the token of lane - 16, so every lane handles one token and 8 heads.
    const int qd = warp & 3;                 // TMEM sub-partition: lanes 32*qd ..
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 16 * qd + (lane & 15);   // tile token of this lane
    const int hb = (lane < 16) ? 0 : 8;      // first head of this lane (heads hb .. hb+7)
    float m_ref[G], lpart[8];
#pragma unroll
    for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY;
#pragma unroll
    for (int h = 0; h < 8; ++h) lpart[h] = 0.f;
    bool ok = true;
    uint32_t cons0 = 0, cons1 = 0;  // ofull phases consumed on barrier 0 / 1
    // Wait until the P.V of tile t has completed.  Phases are consumed in order
    // and never lag by two, so the parity waits cannot alias.
    auto ensure_pv = [&](uint32_t t) {
      const uint32_t b = t & 1, ph = t >> 1;
      uint32_t &cons = b ? cons1 : cons0;
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
      const int sb = i & 1, pb = i & 1;
      if (i >= 2) ensure_pv(i - 2);  // P buffer pb is free again
      if (first) {
#pragma unroll
        for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY;
#pragma unroll
        for (int h = 0; h < 8; ++h) lpart[h] = 0.f;
      }
      // --- scores of tile i: sum of the four partial accumulators
      float s16[16];
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float a[16], b[16], c2[16], d2[16];
        tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 64, a);
        tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 64 + 16, b);
        tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 64 + 32, c2);
        tmem_ld16(tmem + lane_base + Cfg::S_COL + sb * 64 + 48, d2);
#pragma unroll
        for (int h = 0; h < 16; ++h) s16[h] = (a[h] + b[h]) + (c2[h] + d2[h]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      float s[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        const float mine = s16[h], theirs = s16[8 + h];
        const float got = __shfl_xor_sync(0xffffffffu, (lane < 16) ? theirs : mine, 16);
        s[h] = (lane < 16) ? mine : got;
      }
      const bool valid = ok && tok < ntok;
      bool need = false;
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float x = s[h] * p.qscale;
        if (p.post != 0.f) x = p.post * tanhf(x);
        s[h] = valid ? x : -INFINITY;
        need |= s[h] > ((lane < 16) ? m_ref[h] : m_ref[8 + h]) + kTau;
      }
      // --- move the reference only when some score outgrew it
      if (named_bar_or(1, 128, need)) {
        float r[16];  // this lane's 8 heads in their slots, -inf elsewhere
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          r[h] = (lane < 16) ? s[h] : -INFINITY;
          r[8 + h] = (lane < 16) ? -INFINITY : s[h];
        }
        const float tm = warp_reduce_scatter16<true>(r, lane);
        if ((lane & 1) == 0) redmax[qd * G + (lane >> 1)] = tm;
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
#pragma unroll
        for (int h = 0; h < 8; ++h) lpart[h] *= (lane < 16) ? alpha[h] : alpha[8 + h];
        if (!first) {
          // O holds tiles < i: wait for the last of them, then rescale it in TMEM.
          ensure_pv(i - 1);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int cb = 0; cb < 8; ++cb) {  // 4 d-blocks x (hi, lo)
              float v[16];
              tmem_ld16(tmem + lane_base + Cfg::O_COL + cb * 16, v);
#pragma unroll
              for (int h = 0; h < G; ++h) v[h] *= alpha[h];
              tmem_st16_wait(tmem + lane_base + Cfg::O_COL + cb * 16, v);
            }
          }
        }
      }
      // --- weights: P^T row of this token, MN-major with 64-byte swizzle:
      // 16-byte chunks (hi 0-7, hi 8-15, lo 0-7, lo 8-15), chunk c of row r at
      // r * 64 + ((c ^ ((r >> 1) & 3)) * 16).
      {
        float pe[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float mr = (lane < 16) ? m_ref[h] : m_ref[8 + h];
          pe[h] = (s[h] == -INFINITY) ? 0.f : exp2f(s[h] - mr);
          lpart[h] += pe[h];
        }
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          hw[k] = pack_bf16x2(pe[2 * k], pe[2 * k + 1]);
          lw[k] = pack_bf16x2(pe[2 * k] - bf16lo(hw[k]), pe[2 * k + 1] - bf16hi(hw[k]));
        }
        uint8_t *prow = ps + pb * Cfg::PB + tok * 64;
        const int ch = hb >> 3;  // 0 or 1
        const int sw = (tok >> 1) & 3;
        *reinterpret_cast<uint4 *>(prow + ((ch ^ sw) << 4)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4 *>(prow + (((ch + 2) ^ sw) << 4)) =
            make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      if (ok && ntok < Cfg::TILE) {
        const uint32_t vs = v_slot<SHARED>(i);
        // A separate V tile may still be in flight (it is loaded after K): wait for it.
        if (!SHARED)
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&full[vs % NST], (vs / NST) & 1, abort_flag, p.status));
        // V rows past the attended range hold other cache contents (possibly
        // NaN); they get weight 0, but 0 * NaN would still reach O, so clear them.
        uint8_t *tile = stages + (vs % NST) * Cfg::STAGEB;
        const int per_box = (Cfg::TILE - ntok) * 8;  // 16-byte chunks past row ntok
        if (ok) {
#pragma unroll 1
          for (int box = 0; box < D / 64; ++box)
            for (int e = threadIdx.x - 64; e < per_box; e += 128)
              *reinterpret_cast<uint4 *>(tile + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                         (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);

      if (last) {
        // --- segment end: the row sums first (they do not need O), then wait
        // for the segment's last P.V and read O out
        float r[16];  // this lane's 8 partial sums in their slots, 0 elsewhere
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          r[h] = (lane < 16) ? lpart[h] : 0.f;
          r[8 + h] = (lane < 16) ? 0.f : lpart[h];
        }
        const float ls = warp_reduce_scatter16<false>(r, lane);
        if ((lane & 1) == 0) redsum[qd * G + (lane >> 1)] = ls;
        named_bar_sync(1, 128);
        if (i >= 1) ensure_pv(i - 1);
        ensure_pv(i);
        const Segment &sg = it.seg;
        const bool single = sg.whole() && !usplit;  // a split unit always has parts
        const int64_t slot = static_cast<int64_t>(c) + sg.unit;
        const int h0 = sg.x * GU;
        float inv[G];
#pragma unroll
        for (int h = 0; h < G; ++h)
          inv[h] = __fdividef(1.f, (redsum[h] + redsum[G + h]) + (redsum[2 * G + h] + redsum[3 * G + h]));
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            float v[16], w[16];
            tmem_ld16(tmem + lane_base + Cfg::O_COL + jb * 32, v);
            tmem_ld16(tmem + lane_base + Cfg::O_COL + jb * 32 + 16, w);
            const int d = 128 * jb + 32 * qd + lane;
#pragma unroll
            for (int h = 0; h < GU; ++h) {  // columns GU .. 15 are padding
              const float val = (v[h] + w[h]) * inv[h];
              if (single)
                p.out[(static_cast<int64_t>(sg.b) * p.n_q_heads + h0 + h) * D + d] =
                    f32_to_bf16_rn(val);
              else
                p.ws_o[(slot * GU + h) * D + d] = val;
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(oempty);
          if (qd == 0 && lane < GU) {  // LSE of head `lane`: one store per lane
            float mr = m_ref[0];
#pragma unroll
            for (int h = 1; h < G; ++h) mr = (lane == h) ? m_ref[h] : mr;
            const float L = (redsum[lane] + redsum[G + lane]) +
                            (redsum[2 * G + lane] + redsum[3 * G + lane]);
            const float lse_v = (mr + log2f(L)) * 0.69314718055994530942f;
            if (single) {
              if (p.lse != nullptr) p.lse[static_cast<int64_t>(sg.b) * p.n_q_heads + h0 + lane] = lse_v;
            } else {
              p.ws_lse[slot * GU + lane] = lse_v;
            }
          }
        }
      }
      ++i;
    }
    if (usplit && i == 0 && qd == 0 && lane < GU) {
      // An empty part (the unit is shorter than split_k tiles): LSE -inf.
      const int64_t slot = static_cast<int64_t>(c) + c / split_k;
      p.ws_lse[slot * GU + lane] = -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

// K = V (attention_k_eq_v): no V map in the parameter block.
template <int GU>
__global__ void __launch_bounds__(TcConfig::kThreads, 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  tc_decode_body<false, true, GU>(kmap, kmap, qmap, p, TcAppend{});
}

template <int GU>
__global__ void __launch_bounds__(TcConfig::kThreads, 1)
    tc_decode_append_kernel(const __grid_constant__ CUtensorMap kmap,
                            const __grid_constant__ CUtensorMap qmap, const TcParams p,
                            const TcAppend ap) {
  tc_decode_body<true, true, GU>(kmap, kmap, qmap, p, ap);
}

// Separate K and V caches.
template <int GU>
__global__ void __launch_bounds__(TcConfig::kThreads, 1)
    tc_decode_kv_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap,
                        const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  tc_decode_body<false, false, GU>(kmap, vmap, qmap, p, TcAppend{});
}

template <int GU>
__global__ void __launch_bounds__(TcConfig::kThreads, 1)
    tc_decode_kv_append_kernel(const __grid_constant__ CUtensorMap kmap,
                               const __grid_constant__ CUtensorMap vmap,
                               const __grid_constant__ CUtensorMap qmap, const TcParams p,
                               const TcAppend ap) {
  tc_decode_body<true, false, GU>(kmap, vmap, qmap, p, ap);
}

}  // namespace gdattn
