// Split-KV decode attention on the 5th-generation tensor cores (tcgen05) for
// GQA pairs: two query heads per KV head, separate K and V caches, head_dim
// 256 (Gemma-4 sliding-window layers).
//
// A pair of query rows is a thin contraction (2 flop per KV byte), yet on CUDA
// cores the dot products, their cross-lane reductions and the bf16 unpacking
// cost about three instructions per KV element, which caps an SM near 50 GB/s,
// below its share of HBM bandwidth.  The tensor core does the same work in 24
// MMA instructions per 64-token tile, so the SM only streams.  The MMAs are
// padded to N = 16 (the smallest width valid for both shapes below); the unused
// columns cost no extra instructions.
//
// One work unit is one (sequence, KV head); per 64-token tile of it:
//
//   S^T[64 tok x 16]  = K_tile[64 x 256] . Q^T[256 x 16]    (M=64,  N=16, K=256)
//   O^T[256 d x 16]  += V_tile^T[256 x 64] . P[64 x 16]      (M=128 x2, N=16, K=64)
//
// Q rows 0-1 are the pair's query heads (rows 2-15 are whatever follows them, or
// TMA zero fill; their score columns are never read).  P's columns are p_hi of
// heads 0, 1, then p_lo of heads 0, 1 (rows 4-15 stay zero), so O^T column h
// plus column 2 + h is head h's output: the same bf16 hi/lo split of the
// weights as the 16-head kernel, for fp32-grade weights on a bf16 MMA.
//
// K and V tiles arrive by TMA as 64-token x 64-d boxes with 128-byte swizzle:
// the K-major A operand of the first product and the MN-major A operand of the
// second.  P is stored K-major (a row of 64 token weights per column), the same
// canonical layout as Q.  S^T is split over four TMEM accumulators (one per
// 16-wide k-step within each 64-wide d-chunk) so consecutive MMAs never feed
// the same accumulator.  Softmax keeps a lazily moved reference max per head
// (see tc_decode.cuh), so a tile normally costs one TMEM load, one vote and two
// P stores per thread.
//
// A unit split over several CTAs is merged where its last part finishes: each
// CTA stores its part (normalised O and LSE) to the workspace and counts it in
// the unit's counter; the CTA that brings the count to the number of parts
// merges them (the LSE combine) and resets the counter for the next call.
// Nobody waits for another CTA and no combine kernel is launched.  Counting and
// merging run in a warp of their own, so the softmax warps hand a part over at
// a barrier and go straight on with the next segment.
//
// Unit split (p.split_k = k > 1, for units of even length): instead of the
// flattened chunks, unit u is cut into k whole-tile parts, part r on CTA
// u * k + r, so no CTA straddles two units.  The CTA of the last part merges,
// without counting: the other parts are stored as tagged words (each 64-bit
// word carries a float and the call's tag for the unit, so a load sees data
// and readiness at once), and its merge warp polls them while its own last
// tiles are still running, merging them in part order (the result does not
// depend on timing).  Its own part arrives through shared memory, so after
// its last tile no global round trip is left.  Consumed words are cleared;
// the tag is the unit's epoch + 1, read after the dependency wait and advanced
// by the merger once it has seen every part.  An empty part has LSE -inf.
//
// Warp roles (288 threads): warp 0 loads K (and Q), warp 8 loads V, warp 1
// issues QK and owns TMEM, warp 6 issues P.V, warps 2-5 run the softmax (TMEM
// sub-partition warp % 4), warp 7 counts and merges parts.  K and V have rings
// of their own over the same stages: a K tile is released as soon as its QK
// is done, a V tile after its P.V, so K loads run ahead and the ring turns
// over faster than with one release per stage.  Q is double buffered, so the
// next segment's Q is loaded while the current one is still in use.  Every
// wait is bounded.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "combine.cuh"
#include "partition.cuh"
#include "ptx.cuh"
#include "tc_decode.cuh"

namespace gdattn {

struct TcPairConfig {
  static constexpr int D = 256;
  static constexpr int G = 2;
  static constexpr int N = 16;                        // MMA width (QK and P.V)
  static constexpr int TILE = 64;                     // tokens per tile
  static constexpr int NST = 3;                       // KV stages
  static constexpr int BOXB = TILE * 128;             // one 64-token x 64-d box, 8 KiB
  static constexpr int KB = BOXB * (D / 64);          // K tile, 32 KiB
  static constexpr int STAGEB = 2 * KB;               // K tile then V tile, 64 KiB
  static constexpr int QBOXB = N * 128;               // 16 Q rows x 64 d, 2 KiB
  static constexpr int QB = QBOXB * (D / 64);         // 8 KiB per Q buffer
  static constexpr int PB = N * 128;                  // P: 16 rows x 64 tokens bf16, 2 KiB
  static constexpr int OFF_Q = NST * STAGEB;          // 2 Q buffers
  static constexpr int OFF_P = OFF_Q + 2 * QB;
  static constexpr int OFF_BAR = OFF_P + 2 * PB;
  static constexpr int OFF_RED = OFF_BAR + 512;
  static constexpr int OFF_PART = OFF_RED + 2 * 4 * G * 4;  // the merger's own part
  static constexpr int PARTB = G * D * 4 + 64;               // O [G][D], then LSE [G]
  static constexpr int SMEM = OFF_PART + PARTB + 1024;
  static constexpr int kThreads = 288;
  static constexpr uint32_t TMEM_COLS = 256;
  static constexpr uint32_t S_COL = 0;                // 2 buffers x 4 partial sums x 16 columns
  static constexpr uint32_t O_COL = 128;              // 2 d-blocks x 16 columns
};
static_assert(TcPairConfig::TILE == TcConfig::TILE, "TileIter walks 64-token tiles");
static_assert(TcPairConfig::SMEM <= 227 * 1024, "shared memory budget");

// Byte offset of element (row n, token t) in a K-major 128-byte-swizzled
// 64-column bf16 tile: 16-byte chunk t / 8 of row n sits at chunk (t / 8) ^ (n % 8).
__device__ __forceinline__ uint32_t sw128_offset(int n, int t) {
  return static_cast<uint32_t>(n * 128 + ((((t >> 3) ^ (n & 7)) << 4) | ((t & 7) << 1)));
}

// One warp, when the planner saw an impossible sequence length (L < 1, or a
// range longer than the cache): flag it in the status word and give every
// sequence that attends nothing a zero output and LSE -inf.
template <int D>
__device__ __forceinline__ void report_bad_seqlens(const TcParams &p, int lane) {
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

// Warp 7 of the bf16 pair kernel: counts split parts and merges them (see the
// file comment).  Partials are normalised O [G][D] and LSE [G] per part.  (The
// fp8 pair kernel merges in its softmax threads instead, with the helpers
// below.)
template <int G, int D>
__device__ __forceinline__ void pair_merge_warp(const TcParams &p, const ChunkPlan *plan, int c,
                                                int lane, int32_t split_k, bool usplit,
                                                bool merger, uint64_t *tg_o, uint64_t *tg_lse,
                                                const float *part_o, const float *part_lse) {
  // -------------------------------------------------- part count, merge
  // Segment by segment in the softmax warps' order: after a partial is
  // stored (barrier 2), count it with one acq_rel atomic; the CTA whose count
  // completes the unit merges all of its parts (lane c takes float4 columns
  // c, c + 32, c + 64, c + 96) and resets the counter.  Parts are counted
  // after a failed wait too, so the counters always return to zero.
  if (p.merge_in_kernel) {
    grid_dependency_wait();  // counters, workspace and outputs
    // Count one part of unit `unit` (parts in slots slot0 .. slot0 + np - 1);
    // the last one merges.
    auto count_and_merge = [&](int32_t unit, int32_t b, int32_t x, int64_t slot0, int32_t np) {
      uint32_t done = 0;
      if (lane == 0) done = atomic_add_acq_rel_gpu(p.counters + unit, 1u);
      done = __shfl_sync(0xffffffffu, done, 0);
      __syncwarp();  // lane 0's acquire before every lane's reads
      if (done != static_cast<uint32_t>(np - 1)) return;
      if (lane == 0) p.counters[unit] = 0u;
      constexpr int NC = G * D / 4 / 32;  // float4 columns per lane
      const float *o_col[NC];
      const float *l_col[NC];
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        const int e = lane + 32 * k, h = e / (D / 4), d = (e % (D / 4)) * 4;
        o_col[k] = p.ws_o + (slot0 * G + h) * D + d;
        l_col[k] = p.ws_lse + slot0 * G + h;
      }
      float4 res[NC];
      float m[NC], z[NC];
      merge_columns<NC, 4>(o_col, l_col, G * D, G, np, true, res, m, z);
#pragma unroll
      for (int k = 0; k < NC; ++k) {
        const int e = lane + 32 * k, h = e / (D / 4), d = (e % (D / 4)) * 4;
        const int64_t orow = static_cast<int64_t>(b) * p.n_q_heads + x * G + h;
        store_bf16x4(p.out + orow * D + d, res[k]);
        if (d == 0 && p.lse != nullptr)
          p.lse[orow] = (m[k] == -INFINITY) ? -INFINITY : m[k] + logf(z[k]);
      }
    };
    if (usplit) {
      // Part r of unit c / k sits in slot (c / k) * k + unit + r.
      const int32_t unit = c / split_k, crank = c % split_k;
      const int32_t b = unit / p.geo.units_per_seq, x = unit - b * p.geo.units_per_seq;
      const int64_t slot0 = static_cast<int64_t>(unit) * split_k + unit;
      const bool has_part = plan->cs < plan->ce;
      uint32_t tag = 0;
      if (lane == 0) tag = next_tag(__ldcg(p.epochs + unit));
      tag = __shfl_sync(0xffffffffu, tag, 0);
      if (!merger) {
        if (!has_part) {  // an empty part: LSE -inf
          uint64_t *dst = tg_o + (slot0 + crank) * G * D;
          for (int e = lane; e < G * D; e += 32) st_tagged(dst + e, 0.f, tag);
          if (lane < G) st_tagged(tg_lse + (slot0 + crank) * G + lane, -INFINITY, tag);
        }
      } else {
        // Lane l merges elements [16 l, 16 l + 16) of the unit's G x D outputs.
        constexpr int PER = G * D / 32;
        static_assert(PER == 16 && D % PER == 0, "lane mapping");
        const int h = (PER * lane) / D, d0 = (PER * lane) % D;
        float m = -INFINITY, z = 0.f, acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
        auto fold = [&](float lse_r, const float (&o)[PER]) {
          if (lse_r == -INFINITY) return;  // an empty part: weight 0
          const float mn = fmaxf(m, lse_r);
          const float r_old = (m == -INFINITY) ? 0.f : __expf(m - mn);
          const float w = __expf(lse_r - mn);
          z = z * r_old + w;
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] = fmaf(w, o[e], acc[e] * r_old);
          m = mn;
        };
        for (int32_t r = 0; r + 1 < split_k; ++r) {
          uint64_t *src = tg_o + ((slot0 + r) * G + h) * D + d0;
          uint64_t *lsrc = tg_lse + (slot0 + r) * G + h;
          uint64_t wv[PER], wl = 0;
          const long long t0 = clock64();
          while (true) {
#pragma unroll
            for (int e = 0; e < PER; e += 2) ld_tagged2(src + e, wv[e], wv[e + 1]);
            wl = ld_u64_volatile(lsrc);
            bool ready = tag_of(wl) == tag;
#pragma unroll
            for (int e = 0; e < PER; ++e) ready &= tag_of(wv[e]) == tag;
            if (__all_sync(0xffffffffu, ready)) break;
            if (clock64() - t0 > kWaitLimitCycles) {
              if (lane == 0) atomicOr(p.status, kStatusTimeout);
              break;
            }
          }
          float o[PER];
#pragma unroll
          for (int e = 0; e < PER; ++e) o[e] = payload_of(wv[e]);
          fold(payload_of(wl), o);
          // Clear what was consumed, so no later call can mistake it for fresh.
#pragma unroll
          for (int e = 0; e < PER; ++e) st_u64_volatile(src + e, 0ull);
          if ((lane & (D / PER - 1)) == 0) st_u64_volatile(lsrc, 0ull);
        }
        if (has_part) {
          named_bar_sync(2, 160);  // the softmax warps left the own part in shared memory
          float o[PER];
#pragma unroll
          for (int e = 0; e < PER; ++e) o[e] = part_o[h * D + d0 + e];
          fold(part_lse[h], o);
        }
        const float inv_z = (m == -INFINITY) ? 0.f : __fdividef(1.f, z);
        const int64_t orow = static_cast<int64_t>(b) * p.n_q_heads + x * G + h;
        uint16_t *dst = p.out + orow * D + d0;
#pragma unroll
        for (int e = 0; e < PER; e += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(acc[e] * inv_z, acc[e + 1] * inv_z);
          pk.y = pack_bf16x2(acc[e + 2] * inv_z, acc[e + 3] * inv_z);
          pk.z = pack_bf16x2(acc[e + 4] * inv_z, acc[e + 5] * inv_z);
          pk.w = pack_bf16x2(acc[e + 6] * inv_z, acc[e + 7] * inv_z);
          *reinterpret_cast<uint4 *>(dst + e) = pk;
        }
        if (d0 == 0 && p.lse != nullptr) p.lse[orow] = (m == -INFINITY) ? -INFINITY : m + logf(z);
        if (lane == 0) p.epochs[unit] = tag;  // every part of this call has been read
      }
    } else {
      SegmentIter sit;
      sit.init(p.geo, *plan);
      Segment sg;
      while (sit.next(sg)) {
        if (sg.whole()) continue;
        named_bar_sync(2, 160);
        int32_t cf, cl;
        unit_chunks(sg.unit_start, sg.n, plan->chunk, cf, cl);
        count_and_merge(sg.unit, sg.b, sg.x, static_cast<int64_t>(cf) + sg.unit, cl - cf + 1);
      }
    }
  }
}

// ------------------------------------------------- merging in the softmax
// Helpers for a kernel whose softmax threads merge split parts themselves,
// each for the output elements it computed, after its own last tile (the fp8
// pair kernel: a merge warp kept alive through its main loop slowed the
// merging CTA's whole pipeline there).

// Running LSE merge of normalised parts for one output element (natural log).
struct PartMerge {
  float m = -INFINITY, z = 0.f, acc = 0.f;
  __device__ __forceinline__ void add(float lse, float o) {
    if (lse == -INFINITY) return;  // an empty part: weight 0
    const float mn = fmaxf(m, lse);
    const float r_old = (m == -INFINITY) ? 0.f : __expf(m - mn);
    const float w = __expf(lse - mn);
    z = z * r_old + w;
    acc = fmaf(w, o, acc * r_old);
    m = mn;
  }
  __device__ __forceinline__ float out() const {
    return m == -INFINITY ? 0.f : __fdividef(acc, z);
  }
  __device__ __forceinline__ float lse() const { return m == -INFINITY ? -INFINITY : m + logf(z); }
};

// Payloads of N tagged words once each carries `tag`: all loads are issued
// together, then the stragglers re-polled.  After kWaitLimitCycles (SM clock)
// it latches kStatusTimeout in *status and returns what it has.
template <int N>
__device__ __forceinline__ void await_tagged(const uint64_t *const (&addr)[N], uint32_t tag,
                                             float (&val)[N], uint32_t *status) {
  uint64_t w[N];
#pragma unroll
  for (int e = 0; e < N; ++e) w[e] = ld_u64_volatile(addr[e]);
  const long long t0 = clock64();
  while (true) {
    bool ready = true;
#pragma unroll
    for (int e = 0; e < N; ++e) ready &= tag_of(w[e]) == tag;
    if (ready) break;
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicOr(status, kStatusTimeout);
      break;
    }
#pragma unroll
    for (int e = 0; e < N; ++e)
      if (tag_of(w[e]) != tag) w[e] = ld_u64_volatile(addr[e]);
  }
#pragma unroll
  for (int e = 0; e < N; ++e) val[e] = payload_of(w[e]);
}

// The other parts of a tagged unit (all but the last, which merges): the
// elements (head h[e], dim d[e]) of part r are tagged words at
// tg_o[((slot0 + r) * G + h) * D + d], its LSEs at tg_lse[(slot0 + r) * G + h].
// Folds parts 0 .. k-2 in part order into mg[], clearing the O words it read.
template <int G, int D, int NE>
__device__ __forceinline__ void merge_tagged_parts(uint64_t *tg_o, uint64_t *tg_lse,
                                                   int64_t slot0, int32_t k, uint32_t tag,
                                                   const int (&h)[NE], const int (&d)[NE],
                                                   PartMerge (&mg)[NE], uint32_t *status) {
  for (int32_t r = 0; r + 1 < k; ++r) {
    const uint64_t *addr[2 * NE];
    float v[2 * NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      addr[e] = tg_o + ((slot0 + r) * G + h[e]) * D + d[e];
      addr[NE + e] = tg_lse + (slot0 + r) * G + h[e];
    }
    await_tagged<2 * NE>(addr, tag, v, status);
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      mg[e].add(v[NE + e], v[e]);
      st_u64_volatile(const_cast<uint64_t *>(addr[e]), 0ull);  // consumed: never mistaken later
    }
  }
}

// Counted merge of a unit whose parts are plain partials in slots slot0 ..
// slot0 + np - 1 (normalised O [slot][G][D], LSE [slot][G]): the element
// (h[e], d[e]) of every part, in part order.
template <int G, int D, int NE>
__device__ __forceinline__ void merge_counted_parts(const float *ws_o, const float *ws_lse,
                                                    int64_t slot0, int32_t np,
                                                    const int (&h)[NE], const int (&d)[NE],
                                                    PartMerge (&mg)[NE]) {
  for (int32_t r = 0; r < np; ++r)
#pragma unroll
    for (int e = 0; e < NE; ++e)
      mg[e].add(__ldcg(ws_lse + (slot0 + r) * G + h[e]),
                __ldcg(ws_o + ((slot0 + r) * G + h[e]) * D + d[e]));
}

// MULTI: a multi-token step, whose query sequence b reads cache sequence
// cache_seq(b); the single-token entry points read cache sequence b directly.
template <bool APPEND, bool MULTI>
__device__ __forceinline__ void tc_pair_decode_body(const CUtensorMap &kmap,
                                                    const CUtensorMap &vmap,
                                                    const CUtensorMap &qmap, const TcParams &p,
                                                    const TcAppend &ap) {
  using Cfg = TcPairConfig;
  constexpr int G = Cfg::G, D = Cfg::D, NST = Cfg::NST;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = smem;
  uint8_t *qs = smem + Cfg::OFF_Q;
  uint8_t *ps = smem + Cfg::OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
  uint64_t *kfull = bars;           // [NST]  K TMA -> QK
  uint64_t *kempty = bars + 3;      // [NST]  QK -> K TMA
  uint64_t *qfull = bars + 6;       // [2] TMA -> MMA (Q of segment k in buffer k & 1)
  uint64_t *qempty = bars + 8;      // [2] MMA -> TMA
  uint64_t *sfull = bars + 10;      // [2] MMA -> softmax (S of tile i in buffer i & 1)
  uint64_t *sempty = bars + 12;     // [2] softmax -> MMA
  uint64_t *pfull = bars + 14;      // [2] softmax -> MMA (P of tile i in buffer i & 1)
  uint64_t *ofull = bars + 16;      // [2] MMA -> softmax: P.V of tile i done (barrier i & 1)
  uint64_t *oempty = bars + 18;     // softmax -> MMA: O of a finished segment read out
  uint64_t *drain = bars + 19;      // [2] QK warp, P.V warp: all their MMAs done
  uint64_t *vfull = bars + 21;      // [NST]  V TMA -> P.V (and the softmax, for partial tiles)
  uint64_t *vempty = bars + 24;     // [NST]  P.V -> V TMA
  uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(bars + 27);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 28);
  ChunkPlan *plan = reinterpret_cast<ChunkPlan *>(bars + 29);  // 48 bytes, ends before +35
  uint32_t *sh_tag = reinterpret_cast<uint32_t *>(bars + 35);    // this call's tag for the unit
  float *part_o = reinterpret_cast<float *>(smem + Cfg::OFF_PART);  // merger's own part [G][D]
  float *part_lse = part_o + G * D;                                  // [G]
  float *redmax = reinterpret_cast<float *>(smem + Cfg::OFF_RED);  // [4 warps][G]
  float *redsum = redmax + 4 * G;                                  // [4 warps][G]

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
  // The split plan reads only seqlens, so it (and the producer's first KV
  // loads below) may run before the preceding kernel has completed; every other
  // global access waits for it (griddepcontrol.wait) in the role that makes it.
  const int32_t split_k = p.split_k > 1 ? p.split_k : 1;
  const bool usplit = split_k > 1;
  const int32_t crank = c % split_k;
  // Unit split with the merge in this kernel: tagged parts, merged by the last part.
  const bool tagged = usplit && p.merge_in_kernel;
  const bool merger = tagged && crank == split_k - 1;
  uint64_t *tg_o = reinterpret_cast<uint64_t *>(p.ws_o);      // [slots][G][D] tagged words
  uint64_t *tg_lse = reinterpret_cast<uint64_t *>(p.ws_lse);  // [slots][G] tagged words
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

  if (c == 0 && warp == 2 && plan->bad) report_bad_seqlens<D>(p, lane);

  const int32_t C = p.geo.capacity;

  if (warp == 0) {
    // -------------------------------------------------------------- TMA
    // As in the 16-head kernel: the warp walks the schedule, one elected lane
    // copies, and a segment's Q is loaded as soon as the previous segment's
    // last QK has released the buffer.
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    uint32_t i = 0, seg_count = 0, q_issued = 0;
    int32_t qrows[8] = {};       // Q rows of segments whose Q is not issued yet
    uint32_t stage_seg[NST];     // segment of the tile last loaded into each stage
    auto issue_q = [&](bool block) -> bool {  // warp-uniform result
      const uint32_t qb = q_issued & 1;
      if (q_issued >= 2) {  // buffer qb is free once segment q_issued - 2's last QK is done
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
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_2d(qs + qb * Cfg::QB + j * Cfg::QBOXB, &qmap, 64 * j, qrow, &qfull[qb]);
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
    // each sequence's newest one are read; q and the newest row come after.
    // (Sending the rest of the chunk to L2 before the wait was measured to
    // lose: the flood delays the latency-bound loads after the wait.)
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
        qrows[seg_count & 7] = it.seg.b * p.n_q_heads + it.seg.x * G;
        ++seg_count;
      }
      if (i >= NST || it.newest) ensure_waited();
      while (ok && waited && q_issued < seg_count && issue_q(false)) {
      }
      const int st = i % NST;
      if (i >= NST) {
        // The K tile in this stage is released after its QK, which needs its Q.
        while (ok && q_issued <= stage_seg[st]) issue_q(true);
        if (ok && !mbar_wait(&kempty[st], ((i / NST) - 1) & 1, abort_flag, p.status)) ok = false;
      }
      if (!__all_sync(0xffffffffu, ok)) break;
      stage_seg[st] = seg_count - 1;
      if (APPEND && it.newest) {  // append the current token's K row first
        const int32_t slot = (it.seg.first_pos + it.seg.n - 1) % C;
        append_row(ap.k_cache + it.seg.b * ap.batch_stride +
                       (static_cast<int64_t>(slot) * ap.n_kv_heads + it.seg.x) * D,
                   ap.k_new + (static_cast<int64_t>(it.seg.b) * ap.n_kv_heads + it.seg.x) * D, D,
                   lane);
      }
      const int32_t cb = MULTI ? cache_seq(p.geo, it.seg.b) : it.seg.b;
      if (!(p.test_withhold && i == 0) && elect_one()) {
        uint8_t *kdst = stages + st * Cfg::STAGEB;
        mbar_arrive_expect_tx(&kfull[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(kdst + j * Cfg::BOXB, &kmap, 64 * j, it.seg.x, row, cb, &kfull[st], pol);
      }
      __syncwarp();
      ++i;
    }
    ensure_waited();
    while (ok && q_issued < seg_count) issue_q(true);
    // Drain: never leave with copies in flight into shared memory.
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      if (!(p.test_withhold && f == 0)) mbar_wait(&kfull[f % NST], (f / NST) & 1, &no_abort, p.status);
    for (uint32_t k = q_issued > 2 ? q_issued - 2 : 0; k < q_issued; ++k)
      mbar_wait(&qfull[k & 1], (k >> 1) & 1, &no_abort, p.status);
  } else if (warp == 1) {
    // ----------------------------------------------------------- QK MMA
    const uint32_t idesc_qk = idesc_bf16_f32(64, Cfg::N, false, false);
    // An operand at byte offset o from a base descriptor is base + (o >> 4).
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
            tc_mma_bf16(tmem + Cfg::S_COL + sb * 64 + kk * 16, ad, bd, idesc_qk, j != 0);
          }
        }
        tc_commit(&sfull[sb]);
        tc_commit(&kempty[st]);
        if (last) tc_commit(&qempty[qb]);
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
    const uint32_t idesc_pv = idesc_bf16_f32(128, Cfg::N, true, false);
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
      bool w = mbar_wait(&pfull[t & 1], (t >> 1) & 1, abort_flag, p.status);
      if (w) w = mbar_wait(&vfull[t % NST], (t / NST) & 1, abort_flag, p.status);
      // A segment's first P.V overwrites O: the previous segment must be read out.
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
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t bd = b0 + ((kk * 32) >> 4);  // 16 tokens = 32 bytes of each P row
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            const uint64_t ad = a0 + ((2 * jb * Cfg::BOXB + kk * 2048) >> 4);
            tc_mma_bf16(tmem + Cfg::O_COL + jb * 16, ad, bd, idesc_pv, !(first && kk == 0));
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
    // ---------------------------------------------------------- V loads
    // Same schedule and dependency rule as the K loads (warp 0); a V tile is
    // released by its P.V.
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
      if (APPEND && it.newest) {  // append the current token's V row first
        const int32_t slot = (it.seg.first_pos + it.seg.n - 1) % C;
        append_row(ap.v_cache + it.seg.b * ap.batch_stride +
                       (static_cast<int64_t>(slot) * ap.n_kv_heads + it.seg.x) * D,
                   ap.v_new + (static_cast<int64_t>(it.seg.b) * ap.n_kv_heads + it.seg.x) * D, D,
                   lane);
      }
      const int32_t cb = MULTI ? cache_seq(p.geo, it.seg.b) : it.seg.b;
      if (elect_one()) {
        uint8_t *vdst = stages + st * Cfg::STAGEB + Cfg::KB;
        mbar_arrive_expect_tx(&vfull[st], Cfg::KB);
#pragma unroll
        for (int j = 0; j < D / 64; ++j)
          tma_load_4d(vdst + j * Cfg::BOXB, &vmap, 64 * j, it.seg.x, row, cb, &vfull[st], pol);
      }
      __syncwarp();
      ++i;
    }
    // Drain: never leave with copies in flight into shared memory.
    volatile int no_abort = 0;
    for (uint32_t f = i > NST ? i - NST : 0; f < i; ++f)
      mbar_wait(&vfull[f % NST], (f / NST) & 1, &no_abort, p.status);
  } else {
    // ---------------------------------------------------------- softmax
    grid_dependency_wait();  // outputs and workspace are written below
    // This call's tag for the unit (the load completes while the tiles run).
    uint32_t my_tag = 0;
    if (tagged && threadIdx.x == 64) my_tag = next_tag(__ldcg(p.epochs + c / split_k));
    // M=64 puts tile token r in TMEM lane (r % 16) + 32 * (r / 16): lanes 0-15 of
    // each warp receive one token's scores.  Lanes 0-15 take head 0 of their
    // token, lanes 16-31 head 1 of the token of lane - 16.
    const int qd = warp & 3;                 // TMEM sub-partition: lanes 32*qd ..
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const int tok = 16 * qd + (lane & 15);   // tile token of this lane
    const int hd = lane >> 4;                // head of this lane's score
    // P rows 2G .. N-1 multiply O columns nobody reads; keep them finite (zero).
    for (int e = threadIdx.x - 64; e < 2 * (Cfg::N - 2 * G) * 8; e += 128) {
      const int buf = e / ((Cfg::N - 2 * G) * 8), r = e % ((Cfg::N - 2 * G) * 8);
      *reinterpret_cast<uint4 *>(ps + buf * Cfg::PB + (2 * G + (r >> 3)) * 128 + (r & 7) * 16) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    float m_ref[G], lpart = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) m_ref[h] = -INFINITY;
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
        lpart = 0.f;
      }
      // --- scores of tile i: sum of the four partial accumulators
      float s0 = 0.f, s1 = 0.f;
      if (ok && !mbar_wait(&sfull[sb], (i >> 1) & 1, abort_flag, p.status)) ok = false;
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        tc_fence_after();
        float v[8];
        tmem_ld2x4(tmem + lane_base + Cfg::S_COL + sb * 64, v);
        s0 = (v[0] + v[2]) + (v[4] + v[6]);
        s1 = (v[1] + v[3]) + (v[5] + v[7]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
      }
      const float other = __shfl_xor_sync(0xffffffffu, s1, 16);
      const bool valid = ok && tok < ntok;
      float x = ((lane < 16) ? s0 : other) * p.qscale;
      if (p.post != 0.f) x = p.post * tanhf(x);
      x = valid ? x : -INFINITY;
      const float mine_ref = hd ? m_ref[1] : m_ref[0];
      // --- move the reference only when some score outgrew it
      if (named_bar_or(1, 128, x > mine_ref + kTau)) {
        float tm = x;
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) tm = fmaxf(tm, __shfl_xor_sync(0xffffffffu, tm, off));
        if ((lane & 15) == 0) redmax[qd * G + hd] = tm;
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
        lpart *= hd ? alpha[1] : alpha[0];
        if (!first) {
          // O holds tiles < i: wait for the last of them, then rescale it in TMEM.
          ensure_pv(i - 1);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int jb = 0; jb < 2; ++jb) {
              float o[4];  // columns: hi of heads 0, 1, lo of heads 0, 1
              tmem_ld4(tmem + lane_base + Cfg::O_COL + jb * 16, o);
              o[0] *= alpha[0];
              o[1] *= alpha[1];
              o[2] *= alpha[0];
              o[3] *= alpha[1];
              tmem_st4_wait(tmem + lane_base + Cfg::O_COL + jb * 16, o);
            }
          }
        }
      }
      // --- weight of this (token, head): hi part in P row hd, lo part in row G + hd
      {
        const float mr = hd ? m_ref[1] : m_ref[0];
        const float pe = (x == -INFINITY) ? 0.f : exp2f(x - mr);
        lpart += pe;
        const uint16_t hi = f32_to_bf16_rn(pe);
        const uint16_t lo = f32_to_bf16_rn(pe - __uint_as_float(static_cast<uint32_t>(hi) << 16));
        uint8_t *pbuf = ps + pb * Cfg::PB;
        *reinterpret_cast<uint16_t *>(pbuf + sw128_offset(hd, tok)) = hi;
        *reinterpret_cast<uint16_t *>(pbuf + sw128_offset(G + hd, tok)) = lo;
      }
      if (ok && ntok < Cfg::TILE) {
        // The V tile may still be in flight (it is loaded after K): wait for it.
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&vfull[i % NST], (i / NST) & 1, abort_flag, p.status));
      }
      if (ok && ntok < Cfg::TILE) {
        // V rows past the attended range hold other cache contents (possibly
        // NaN); they get weight 0, but 0 * NaN would still reach O, so clear them.
        uint8_t *vt = stages + (i % NST) * Cfg::STAGEB + Cfg::KB;
        const int per_box = (Cfg::TILE - ntok) * 8;  // 16-byte chunks past row ntok
#pragma unroll 1
        for (int box = 0; box < D / 64; ++box)
          for (int e = threadIdx.x - 64; e < per_box; e += 128)
            *reinterpret_cast<uint4 *>(vt + box * Cfg::BOXB + (ntok + (e >> 3)) * 128 +
                                       (e & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&pfull[pb]);

      if (last) {
        // --- segment end: the row sums first (they do not need O), then wait
        // for the segment's last P.V and read O out
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
        const bool single = sg.whole() && !usplit;  // a split unit always has parts
        const int64_t slot = static_cast<int64_t>(c) + sg.unit;
        const int h0 = sg.x * G;
        float L[G], inv[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          L[h] = (redsum[h] + redsum[G + h]) + (redsum[2 * G + h] + redsum[3 * G + h]);
          inv[h] = __fdividef(1.f, L[h]);
        }
        // A tagged part is stored even after a failed wait, so its merger never
        // waits for it in vain (the status word reports the failure).
        if (ok || (tagged && !merger)) {
          if (ok) tc_fence_after();
#pragma unroll
          for (int jb = 0; jb < 2; ++jb) {
            float o[4] = {0.f, 0.f, 0.f, 0.f};
            if (ok) tmem_ld4(tmem + lane_base + Cfg::O_COL + jb * 16, o);
            const int d = 128 * jb + 32 * qd + lane;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              const float val = (o[h] + o[G + h]) * inv[h];
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
          if (qd == 0 && lane < G) {  // LSE of head `lane`
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
        // Hand a partial over to the merge warp: counted parts, or the merger's own.
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

__global__ void __launch_bounds__(TcPairConfig::kThreads, 1)
    tc_pair_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                          const __grid_constant__ CUtensorMap vmap,
                          const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  tc_pair_decode_body<false, false>(kmap, vmap, qmap, p, TcAppend{});
}

__global__ void __launch_bounds__(TcPairConfig::kThreads, 1)
    tc_pair_decode_multi_kernel(const __grid_constant__ CUtensorMap kmap,
                                const __grid_constant__ CUtensorMap vmap,
                                const __grid_constant__ CUtensorMap qmap, const TcParams p) {
  tc_pair_decode_body<false, true>(kmap, vmap, qmap, p, TcAppend{});
}

__global__ void __launch_bounds__(TcPairConfig::kThreads, 1)
    tc_pair_decode_append_kernel(const __grid_constant__ CUtensorMap kmap,
                                 const __grid_constant__ CUtensorMap vmap,
                                 const __grid_constant__ CUtensorMap qmap, const TcParams p,
                                 const TcAppend ap) {
  tc_pair_decode_body<true, false>(kmap, vmap, qmap, p, ap);
}

}  // namespace gdattn
