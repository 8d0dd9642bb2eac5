// Device-side split of a decode step's KV work across CTAs.
//
// A "unit" is what one query-head group attends: (sequence b, KV-head group x),
// x in [0, units_per_seq).  Unit u = b * units_per_seq + x attends n_b positions
// (min(L_b, window) for a sliding layer, L_b otherwise).  All units' positions
// are laid end to end ("flattened") and cut into P equal chunks, one per CTA,
// so every CTA streams the same number of KV rows whatever the mix of context
// lengths in the batch.  A chunk may cover the tail of one unit, whole units and
// the head of another; each (chunk c, unit u) piece is a "segment".
//
// Segment results that do not cover their whole unit are written as partials
// to slot c + u of the workspace.  The slot is unique: if chunk c touches unit
// u and chunk c' > c touches unit u', then u' >= u, so c + u = c' + u' is
// impossible.  Slots used are < P + number of units.  A unit's partials sit in
// consecutive slots c_first + u .. c_last + u, which the combine kernel reads.
//
// The split depends only on the device-resident seqlens and on P, so it needs
// no host synchronisation and is captured in CUDA graphs as is.
//
// A CTA then walks its segments tile by tile (TileIterT): a segment's
// positions map to one or two runs of ring slots (the ring may wrap), and each
// run is cut into tiles of TILE tokens, so no tile crosses the ring's end.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace gdattn {

struct Geometry {
  const int32_t *seqlens;
  int32_t batch;
  int32_t units_per_seq;
  int32_t window;
  int32_t capacity;
  // Low 16 bits: P = gridDim.x of the decode kernel (< 2^16); high 16 bits: the
  // chunk alignment in tokens (chunk sizes are rounded up to a multiple of it).
  // Packed so the kernels' parameter block keeps its size.
  int32_t nchunks_align;
  int32_t cache_batch;  // sequences in the cache: query sequence b reads cache b % cache_batch
};

__device__ __forceinline__ int32_t geo_nchunks(const Geometry &g) {
  return g.nchunks_align & 0xFFFF;
}
__device__ __forceinline__ int32_t geo_align(const Geometry &g) { return g.nchunks_align >> 16; }

// The cache sequence query sequence b reads (several query sequences share one
// cache sequence in a multi-token step, laid out token-major).
__device__ __forceinline__ int32_t cache_seq(const Geometry &g, int32_t b) {
  return b < g.cache_batch ? b : b % g.cache_batch;  // no division in a single-token step
}

// Positions one decode step attends for context length L (clamped to the cache;
// an impossible L yields 0 and `bad`).
__device__ __forceinline__ int32_t attended_count(int32_t L, int32_t window, int32_t C,
                                                  bool &bad) {
  int32_t n = (window > 0 && L > window) ? window : L;
  if (L < 1) {
    bad = true;
    return 0;
  }
  if (n > C) {
    bad = true;
    n = C;
  }
  return n;
}

__device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__device__ __forceinline__ int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// Per-CTA plan, computed by one warp and shared through shared memory.
struct ChunkPlan {
  int64_t total;  // flattened positions over all units
  int64_t chunk;  // positions per CTA
  int64_t cs, ce; // this CTA's [start, end)
  int64_t pre0;   // flattened offset of sequence b0's first unit
  int32_t b0;     // first sequence whose units reach past cs
  int32_t bad;    // some seqlens entry was impossible
};

__device__ __forceinline__ int64_t warp_sum_i64(int64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int64_t warp_incl_scan_i64(int64_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Executed by all 32 lanes of one warp; lane 0 writes *plan.
__device__ void plan_chunk(const Geometry &g, int32_t c, ChunkPlan *plan) {
  const int lane = threadIdx.x & 31;
  bool bad = false;
  int64_t acc = 0;
  for (int32_t b = lane; b < g.batch; b += 32)
    acc += attended_count(__ldg(g.seqlens + b), g.window, g.capacity, bad);
  const int64_t total = warp_sum_i64(acc) * g.units_per_seq;
  const int anybad = __any_sync(0xffffffffu, bad);
  const int64_t chunk =
      total > 0 ? ceil_div64(ceil_div64(total, geo_nchunks(g)), geo_align(g)) * geo_align(g) : 1;
  const int64_t cs = imin64(static_cast<int64_t>(c) * chunk, total);
  const int64_t ce = imin64(cs + chunk, total);
  // First sequence whose flattened range ends after cs.
  int64_t base = 0;
  int32_t b0 = g.batch;
  int64_t pre0 = total;
  for (int32_t start = 0; start < g.batch; start += 32) {
    const int32_t b = start + lane;
    bool dummy = false;
    const int64_t span =
        b < g.batch ? static_cast<int64_t>(attended_count(__ldg(g.seqlens + b), g.window,
                                                          g.capacity, dummy)) *
                          g.units_per_seq
                    : 0;
    const int64_t incl = warp_incl_scan_i64(span, lane) + base;
    const unsigned hit = __ballot_sync(0xffffffffu, b < g.batch && incl > cs);
    if (hit) {
      const int first = __ffs(hit) - 1;
      const int64_t incl_first = __shfl_sync(0xffffffffu, incl, first);
      const int64_t span_first = __shfl_sync(0xffffffffu, span, first);
      b0 = start + first;
      pre0 = incl_first - span_first;
      break;
    }
    base = __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) {
    plan->total = total;
    plan->chunk = chunk;
    plan->cs = cs;
    plan->ce = ce;
    plan->pre0 = pre0;
    plan->b0 = b0;
    plan->bad = anybad;
  }
}

// One (chunk, unit) piece of work.
struct Segment {
  int32_t b, x, unit;
  int32_t n;          // positions the unit attends
  int32_t lo, hi;     // local offsets [lo, hi) within the unit's attended range
  int32_t first_pos;  // logical position of local offset 0 (= L_b - n)
  int64_t unit_start; // flattened offset of the unit
  // The segment covers its whole unit: the result is final, no partial.
  __device__ __forceinline__ bool whole() const { return lo == 0 && hi == n; }
};

// Walks the segments of one chunk in order.  Every thread of a CTA may run its
// own copy; all copies yield the same sequence.
struct SegmentIter {
  const Geometry *g;
  int64_t pos, ce, pre;
  int32_t b;

  __device__ __forceinline__ void init(const Geometry &geo, const ChunkPlan &p) {
    g = &geo;
    pos = p.cs;
    ce = p.ce;
    pre = p.pre0;
    b = p.b0;
  }

  __device__ __forceinline__ bool next(Segment &s) {
    while (pos < ce && b < g->batch) {
      bool dummy = false;
      const int32_t L = __ldg(g->seqlens + b);
      const int32_t n = attended_count(L, g->window, g->capacity, dummy);
      const int64_t span = static_cast<int64_t>(n) * g->units_per_seq;
      if (pre + span <= pos) {
        pre += span;
        ++b;
        continue;
      }
      const int32_t x = static_cast<int32_t>((pos - pre) / n);
      const int64_t ustart = pre + static_cast<int64_t>(x) * n;
      s.b = b;
      s.x = x;
      s.unit = b * g->units_per_seq + x;
      s.n = n;
      s.lo = static_cast<int32_t>(pos - ustart);
      s.hi = static_cast<int32_t>(imin64(static_cast<int64_t>(n), ce - ustart));
      s.first_pos = L - n;
      s.unit_start = ustart;
      pos = ustart + s.hi;
      return true;
    }
    return false;
  }
};

// Unit split: unit u (sequence u / units_per_seq, group u % units_per_seq) is
// cut into k parts; part r takes whole tiles [r * T / k, (r + 1) * T / k) of
// the unit's T = ceil(n / tile) tiles.
// The range is expressed as a chunk so the segment and tile iterators apply
// unchanged (it holds one segment, or none when the unit is too short).  Run
// by one whole warp.
__device__ void plan_unit_split(const Geometry &g, int32_t u, int32_t r, int32_t k, int32_t tile,
                                ChunkPlan *plan) {
  const int lane = threadIdx.x & 31;
  const int32_t b = u / g.units_per_seq;
  const int32_t x = u - b * g.units_per_seq;
  bool bad = false;
  int64_t all = 0, before = 0;
  for (int32_t bb = lane; bb < g.batch; bb += 32) {
    const int64_t n_bb = attended_count(__ldg(g.seqlens + bb), g.window, g.capacity, bad);
    all += n_bb;
    if (bb < b) before += n_bb;
  }
  const int64_t total = warp_sum_i64(all) * g.units_per_seq;
  const int64_t pre = warp_sum_i64(before) * g.units_per_seq;
  const int anybad = __any_sync(0xffffffffu, bad);
  bool dummy = false;
  const int32_t n = attended_count(__ldg(g.seqlens + b), g.window, g.capacity, dummy);
  const int64_t tiles = ceil_div64(n, tile);
  const int64_t lo = imin64(r * tiles / k * tile, n);
  const int64_t hi = imin64((r + 1) * tiles / k * tile, n);
  const int64_t ustart = pre + static_cast<int64_t>(x) * n;
  if (lane == 0) {
    plan->total = total;
    plan->chunk = hi - lo;
    plan->cs = ustart + lo;
    plan->ce = ustart + hi;
    plan->pre0 = pre;
    plan->b0 = b;
    plan->bad = anybad;
  }
}

// Chunks covering [unit_start, unit_start + n).
__device__ __forceinline__ void unit_chunks(int64_t unit_start, int32_t n, int64_t chunk,
                                            int32_t &c_first, int32_t &c_last) {
  c_first = static_cast<int32_t>(unit_start / chunk);
  c_last = static_cast<int32_t>((unit_start + n - 1) / chunk);
}

// Contiguous slot runs (at most two, the ring may wrap) of a segment.
struct SlotRuns {
  int32_t start0, len0, len1;  // second run starts at slot 0
  int32_t count;
  __device__ __forceinline__ int32_t start(int r) const { return r == 0 ? start0 : 0; }
  __device__ __forceinline__ int32_t len(int r) const { return r == 0 ? len0 : len1; }
};

__device__ __forceinline__ SlotRuns segment_runs(const Segment &s, int32_t C) {
  SlotRuns r;
  const int32_t len = s.hi - s.lo;
  const int32_t s0 = (s.first_pos + s.lo) % C;
  const int32_t first = min(len, C - s0);
  r.start0 = s0;
  r.len0 = first;
  r.len1 = len - first;
  r.count = r.len1 > 0 ? 2 : 1;
  return r;
}

// Tiles of one CTA, in order, across its segments.
template <int TILE>
struct TileIterT {
  SegmentIter seg_it;
  Segment seg;
  SlotRuns runs;
  int32_t run, t0;
  bool have_seg;
  bool newest;  // the last tile yielded holds the unit's newest position (L - 1)
  int32_t off;  // offset of the last tile's first token in its unit's attended range

  __device__ __forceinline__ void init(const Geometry &g, const ChunkPlan &p) {
    seg_it.init(g, p);
    have_seg = false;
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
    }
    row = runs.start(run) + t0;
    ntok = min(TILE, runs.len(run) - t0);
    off = seg.lo + (run == 1 ? runs.len0 : 0) + t0;
    newest = off + ntok == seg.n;
    t0 += TILE;
    if (t0 >= runs.len(run)) {
      ++run;
      t0 = 0;
    }
    last = (run >= runs.count);
    if (last) have_seg = false;
    return true;
  }
};

}  // namespace gdattn
