// Host check of the split planner in the library's csrc/partition.cuh, compiled
// for the CPU with the warp intrinsics it uses emulated by 32 cooperative
// lanes (ucontext fibers on one thread, switched round-robin at every warp
// exchange; tests/test_planner_host.py copies partition.cuh beside an empty
// ptx.cuh and builds this file against it).
//
// For random batches (ragged lengths, windows, ring capacities, query-head
// groups, chunk counts and alignments, impossible lengths) it checks:
// - plan_chunk: equal, aligned chunks that cover the flattened positions;
// - SegmentIter: every (unit, offset) of every unit is covered exactly once,
//   segments carry the right unit, length and first position, slots c + u are
//   unique, and unit_chunks names exactly the chunks that touched the unit;
// - segment_runs: the one or two slot runs are the positions modulo C;
// - TileIterT: each segment cut into tiles that follow one another, start at
//   the right slot, never cross the ring's end, and carry the right flags;
// - plan_unit_split: k parts on tile boundaries that cover a unit once (on up
//   to 14 units of each batch, evenly spaced, the last one included).
// Prints "ok <cases>" or the first failure, and exits non-zero on failure.
#include <ucontext.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <random>
#include <vector>

#define __device__
#define __forceinline__ inline
using std::min;

struct LaneIndex {
  unsigned x;
};
LaneIndex threadIdx;  // the running lane (set on every switch)

// 32 lanes as fibers.  A lane that reaches a barrier passes control to the
// next lane; the 32nd to arrive goes on, and the others resume in turn at their
// next switch, so every lane runs the code between two barriers once.
ucontext_t g_main, g_lane_ctx[32];
int g_arrived = 0;
bool g_finished[32];

void switch_to(int from, int to) {
  threadIdx.x = static_cast<unsigned>(to);
  swapcontext(&g_lane_ctx[from], &g_lane_ctx[to]);
  threadIdx.x = static_cast<unsigned>(from);
}

struct LaneBarrier {
  void wait() {
    const int lane = threadIdx.x & 31;
    if (++g_arrived == 32) {
      g_arrived = 0;
      return;
    }
    switch_to(lane, (lane + 1) & 31);
  }
};
LaneBarrier g_bar;
uint64_t g_slot[32];

// Every lane publishes v; each receives lane src's value.
template <class T>
T lane_exchange(T v, int src) {
  const int lane = threadIdx.x & 31;
  uint64_t bits = 0;
  std::memcpy(&bits, &v, sizeof(T));
  g_slot[lane] = bits;
  g_bar.wait();
  T r;
  std::memcpy(&r, &g_slot[src], sizeof(T));
  g_bar.wait();
  return r;
}
template <class T>
T __shfl_xor_sync(unsigned, T v, int o) {
  return lane_exchange(v, (threadIdx.x & 31) ^ o);
}
template <class T>
T __shfl_up_sync(unsigned, T v, int o) {
  const int lane = threadIdx.x & 31;
  return lane_exchange(v, lane >= o ? lane - o : lane);
}
template <class T>
T __shfl_sync(unsigned, T v, int src) {
  return lane_exchange(v, src);
}
unsigned __ballot_sync(unsigned, int pred) {
  const int lane = threadIdx.x & 31;
  g_slot[lane] = pred ? 1u : 0u;
  g_bar.wait();
  unsigned m = 0;
  for (int i = 0; i < 32; ++i)
    if (g_slot[i]) m |= 1u << i;
  g_bar.wait();
  return m;
}
int __any_sync(unsigned mask, int pred) { return __ballot_sync(mask, pred) != 0; }
int __ffs(unsigned x) { return __builtin_ffs(static_cast<int>(x)); }
template <class T>
T __ldg(const T *p) {
  return *p;
}

#include "partition.cuh"

using namespace gdattn;

namespace {

struct Case {
  std::vector<int32_t> seqlens;
  int32_t units_per_seq, window, capacity, nchunks, align;
};

Case draw_case(std::mt19937_64 &rng) {
  auto pick = [&](std::initializer_list<int32_t> xs) {
    return *(xs.begin() + std::uniform_int_distribution<size_t>(0, xs.size() - 1)(rng));
  };
  Case c;
  const int32_t batch = std::uniform_int_distribution<int32_t>(1, 70)(rng);
  c.units_per_seq = pick({1, 2, 8});
  c.window = pick({0, 1, 7, 64, 100, 1024});
  c.capacity = c.window > 0 ? c.window + pick({0, 0, 7, 500}) : pick({64, 1000, 3000});
  c.nchunks = std::uniform_int_distribution<int32_t>(1, 300)(rng);
  c.align = pick({1, 64, 128});
  const int32_t maxlen = pick({3, 70, 3000});
  for (int32_t b = 0; b < batch; ++b) {
    int32_t L = std::uniform_int_distribution<int32_t>(1, maxlen)(rng);
    if (std::uniform_int_distribution<int>(0, 40)(rng) == 0) L = 0;  // impossible length
    c.seqlens.push_back(L);
  }
  return c;
}

int32_t expected_count(int32_t L, int32_t w, int32_t C, bool &bad) {
  if (L < 1) {
    bad = true;
    return 0;
  }
  int32_t n = (w > 0 && L > w) ? w : L;
  if (n > C) {
    bad = true;
    n = C;
  }
  return n;
}

char g_err[512];
#define CHECK(cond, ...)                                  \
  do {                                                    \
    if (!(cond)) {                                        \
      if (g_err[0] == 0) snprintf(g_err, sizeof g_err, __VA_ARGS__); \
      return false;                                       \
    }                                                     \
  } while (0)

// Walks chunk c's tiles with TileIterT<TILE> against its segments: each
// segment's tiles follow one another from lo to hi, start at the slot of
// their first position, never cross the ring's end, are short only at the end
// of a slot run, and carry the first / last / newest flags of their place.
template <int TILE>
bool check_tiles(const Case &cs, const Geometry &g, const ChunkPlan &p, int32_t c,
                 const std::vector<Segment> &segs) {
  TileIterT<TILE> it;
  it.init(g, p);
  int32_t row, ntok;
  bool first, last;
  size_t si = 0;
  int32_t next_off = 0;
  bool in_seg = false;
  while (it.next(cs.capacity, row, ntok, first, last)) {
    CHECK(si < segs.size(), "chunk %d: tiles past its %zu segments", c, segs.size());
    const Segment &s = segs[si];
    CHECK(first == !in_seg, "chunk %d segment %zu: first flag", c, si);
    if (first) {
      next_off = s.lo;
      in_seg = true;
    }
    CHECK(it.seg.unit == s.unit && it.seg.lo == s.lo && it.seg.hi == s.hi,
          "chunk %d: tile of another segment", c);
    CHECK(it.off == next_off, "chunk %d unit %d: tile at offset %d, expected %d", c, s.unit,
          it.off, next_off);
    CHECK(ntok >= 1 && ntok <= TILE, "chunk %d unit %d: %d tokens", c, s.unit, ntok);
    CHECK(row == (s.first_pos + it.off) % cs.capacity, "chunk %d unit %d: row %d", c, s.unit,
          row);
    CHECK(row + ntok <= cs.capacity, "chunk %d unit %d: tile crosses the ring's end", c, s.unit);
    CHECK(ntok == TILE || last || row + ntok == cs.capacity,
          "chunk %d unit %d: short tile inside a run", c, s.unit);
    CHECK(it.newest == (it.off + ntok == s.n), "chunk %d unit %d: newest flag", c, s.unit);
    next_off += ntok;
    CHECK(next_off <= s.hi, "chunk %d unit %d: tiles past the segment", c, s.unit);
    if (last) {
      CHECK(next_off == s.hi, "chunk %d unit %d: segment ends at %d, not %d", c, s.unit,
            next_off, s.hi);
      ++si;
      in_seg = false;
    }
  }
  CHECK(si == segs.size() && !in_seg, "chunk %d: %zu of %zu segments tiled", c, si, segs.size());
  return true;
}

// Checks one chunk count's whole plan (lane 0 only; plans come from all lanes).
bool check_chunks(const Case &cs, const Geometry &g, const std::vector<ChunkPlan> &plans) {
  const int32_t B = static_cast<int32_t>(cs.seqlens.size());
  bool bad = false;
  std::vector<int32_t> n(B);
  int64_t total = 0;
  for (int32_t b = 0; b < B; ++b) {
    n[b] = expected_count(cs.seqlens[b], cs.window, cs.capacity, bad);
    total += static_cast<int64_t>(n[b]) * cs.units_per_seq;
  }
  const int32_t units = B * cs.units_per_seq;
  std::vector<std::vector<uint8_t>> cover(units);
  for (int32_t u = 0; u < units; ++u) cover[u].assign(n[u / cs.units_per_seq], 0);
  std::vector<int32_t> cmin(units, INT32_MAX), cmax(units, -1);
  std::vector<uint8_t> slot_used(cs.nchunks + units, 0);
  const int64_t chunk = plans[0].chunk;
  CHECK(total == 0 || (chunk % cs.align == 0 && chunk * cs.nchunks >= total &&
                       (chunk - cs.align) * cs.nchunks < total),
        "chunk %lld for total %lld, P %d, align %d", (long long)chunk, (long long)total,
        cs.nchunks, cs.align);
  for (int32_t c = 0; c < cs.nchunks; ++c) {
    const ChunkPlan &p = plans[c];
    CHECK(p.total == total && p.chunk == chunk && p.bad == (bad ? 1 : 0),
          "chunk %d: total %lld/%lld bad %d/%d", c, (long long)p.total, (long long)total, p.bad,
          bad);
    const int64_t cs0 = std::min<int64_t>(c * chunk, total);
    CHECK(p.cs == cs0 && p.ce == std::min<int64_t>(cs0 + chunk, total), "chunk %d bounds", c);
    SegmentIter it;
    it.init(g, p);
    Segment s;
    int64_t pos = p.cs;
    std::vector<Segment> segs;
    while (it.next(s)) {
      segs.push_back(s);
      const int32_t b = s.unit / cs.units_per_seq;
      CHECK(b == s.b && s.x == s.unit - b * cs.units_per_seq && s.unit < units,
            "chunk %d: unit %d of (%d, %d)", c, s.unit, s.b, s.x);
      CHECK(s.n == n[b] && s.first_pos == cs.seqlens[b] - n[b], "chunk %d unit %d: n/first",
            c, s.unit);
      CHECK(0 <= s.lo && s.lo < s.hi && s.hi <= s.n, "chunk %d unit %d: [%d, %d) of %d", c,
            s.unit, s.lo, s.hi, s.n);
      CHECK(s.unit_start + s.lo == pos, "chunk %d unit %d: not contiguous", c, s.unit);
      pos = s.unit_start + s.hi;
      for (int32_t o = s.lo; o < s.hi; ++o) ++cover[s.unit][o];
      CHECK(!slot_used[c + s.unit], "slot %d used twice", c + s.unit);
      slot_used[c + s.unit] = 1;
      cmin[s.unit] = std::min(cmin[s.unit], c);
      cmax[s.unit] = std::max(cmax[s.unit], c);
      int32_t cf, cl;
      unit_chunks(s.unit_start, s.n, chunk, cf, cl);
      CHECK(cf <= c && c <= cl, "unit %d: chunk %d outside [%d, %d]", s.unit, c, cf, cl);
      if (s.n <= cs.capacity) {
        const SlotRuns r = segment_runs(s, cs.capacity);
        CHECK(r.len0 + r.len1 == s.hi - s.lo && r.count == (r.len1 > 0 ? 2 : 1),
              "runs of unit %d", s.unit);
        int32_t k = 0;
        for (int run = 0; run < r.count; ++run)
          for (int32_t j = 0; j < r.len(run); ++j, ++k)
            CHECK(r.start(run) + j == (s.first_pos + s.lo + k) % cs.capacity,
                  "unit %d: slot of offset %d", s.unit, s.lo + k);
      }
    }
    CHECK(pos == p.ce || p.cs == p.ce, "chunk %d ends at %lld, not %lld", c, (long long)pos,
          (long long)p.ce);
    if (!check_tiles<64>(cs, g, p, c, segs) || !check_tiles<128>(cs, g, p, c, segs))
      return false;
  }
  for (int32_t u = 0; u < units; ++u) {
    for (size_t o = 0; o < cover[u].size(); ++o)
      CHECK(cover[u][o] == 1, "unit %d offset %zu covered %d times", u, o, cover[u][o]);
    if (!cover[u].empty()) {
      int32_t cf, cl;
      const int64_t ustart = [&] {
        int64_t s = 0;
        for (int32_t b = 0; b < u / cs.units_per_seq; ++b)
          s += static_cast<int64_t>(n[b]) * cs.units_per_seq;
        return s + static_cast<int64_t>(u % cs.units_per_seq) * n[u / cs.units_per_seq];
      }();
      unit_chunks(ustart, n[u / cs.units_per_seq], chunk, cf, cl);
      CHECK(cf == cmin[u] && cl == cmax[u], "unit %d: chunks [%d, %d] vs touched [%d, %d]", u,
            cf, cl, cmin[u], cmax[u]);
    }
  }
  return true;
}

// Checks the k parts of the listed units (part r of units[j] in plans[j * k + r]).
bool check_unit_split(const Case &cs, const Geometry &g, int32_t k, int32_t tile,
                      const std::vector<int32_t> &units, const std::vector<ChunkPlan> &plans) {
  for (size_t j = 0; j < units.size(); ++j) {
    const int32_t u = units[j];
    const int32_t b = u / cs.units_per_seq;
    bool bad = false;
    const int32_t n = expected_count(cs.seqlens[b], cs.window, cs.capacity, bad);
    std::vector<uint8_t> cover(n, 0);
    for (int32_t r = 0; r < k; ++r) {
      const ChunkPlan &p = plans[j * k + r];
      SegmentIter it;
      it.init(g, p);
      Segment s;
      int segs = 0;
      while (it.next(s)) {
        ++segs;
        CHECK(s.unit == u, "split part %d of unit %d yields unit %d", r, u, s.unit);
        CHECK(s.lo % tile == 0 && (s.hi % tile == 0 || s.hi == n), "part %d of unit %d: [%d, %d)",
              r, u, s.lo, s.hi);
        for (int32_t o = s.lo; o < s.hi; ++o) ++cover[o];
      }
      CHECK(segs <= 1, "part %d of unit %d: %d segments", r, u, segs);
    }
    for (int32_t o = 0; o < n; ++o)
      CHECK(cover[o] == 1, "unit %d offset %d covered %d times by %d parts", u, o, cover[o], k);
  }
  return true;
}

}  // namespace

void lane_body(int lane);
int g_n_cases = 0;
bool g_ok = true;
int g_done = 0;

void lane_entry(int lane) {
  threadIdx.x = static_cast<unsigned>(lane);
  lane_body(lane);
  g_finished[lane] = true;
  threadIdx.x = 0;
}

void lane_body(int lane) {
  std::mt19937_64 rng(12345);  // every lane draws the same cases
  bool lane_ok = true;
  for (int i = 0; i < g_n_cases; ++i) {
    const Case cs = draw_case(rng);
    Geometry g;
    g.seqlens = cs.seqlens.data();
    g.batch = static_cast<int32_t>(cs.seqlens.size());
    g.units_per_seq = cs.units_per_seq;
    g.window = cs.window;
    g.capacity = cs.capacity;
    g.nchunks_align = cs.nchunks | (cs.align << 16);
    g.cache_batch = g.batch;
    std::vector<ChunkPlan> plans(cs.nchunks);
    for (int32_t c = 0; c < cs.nchunks; ++c) plan_chunk(g, c, &plans[c]);
    // the unit split for k parts of `tile` tokens, on a sample of the units
    const int32_t k = 1 + static_cast<int32_t>(i % 5) * (i % 3 == 0 ? 4 : 1);
    const int32_t tile = (i & 1) ? 64 : 128;
    const int32_t units = g.batch * g.units_per_seq;
    const int32_t ustep = units > 12 ? units / 12 : 1;
    std::vector<int32_t> picked;
    for (int32_t u = 0; u < units; u += ustep) picked.push_back(u);
    if (picked.back() != units - 1) picked.push_back(units - 1);
    std::vector<ChunkPlan> parts(picked.size() * k);
    for (size_t j = 0; j < picked.size(); ++j)
      for (int32_t r = 0; r < k; ++r) plan_unit_split(g, picked[j], r, k, tile, &parts[j * k + r]);
    if (lane == 0 && lane_ok) {
      lane_ok = check_chunks(cs, g, plans) && check_unit_split(cs, g, k, tile, picked, parts);
      if (!lane_ok) {
        g_ok = false;
        fprintf(stderr, "case %d (batch %zu, groups %d, w %d, C %d, P %d, align %d, k %d): %s\n",
                i, cs.seqlens.size(), cs.units_per_seq, cs.window, cs.capacity, cs.nchunks,
                cs.align, k, g_err);
      } else {
        ++g_done;
      }
    }
  }
}

int main(int argc, char **argv) {
  g_n_cases = argc > 1 ? atoi(argv[1]) : 100;
  const size_t stack_bytes = 1 << 20;
  std::vector<std::vector<char>> stacks(32, std::vector<char>(stack_bytes));
  for (int lane = 0; lane < 32; ++lane) {
    getcontext(&g_lane_ctx[lane]);
    g_lane_ctx[lane].uc_stack.ss_sp = stacks[lane].data();
    g_lane_ctx[lane].uc_stack.ss_size = stack_bytes;
    g_lane_ctx[lane].uc_link = &g_main;
    makecontext(&g_lane_ctx[lane], reinterpret_cast<void (*)()>(lane_entry), 1, lane);
  }
  // Lane 0 starts; control comes back here whenever a lane returns, and the
  // lanes still parked after their last barrier are then run to their end.
  for (int round = 0; round < 33; ++round) {
    int lane = 0;
    while (lane < 32 && g_finished[lane]) ++lane;
    if (lane == 32) break;
    threadIdx.x = static_cast<unsigned>(lane);
    swapcontext(&g_main, &g_lane_ctx[lane]);
  }
  for (int lane = 0; lane < 32; ++lane)
    if (!g_finished[lane]) {
      fprintf(stderr, "lane %d did not finish\n", lane);
      return 1;
    }
  if (!g_ok) return 1;
  printf("ok %d\n", g_done);
  return 0;
}
