// C ABI of libgdattn (declared in include/gdattn.h): argument checks, the split
// planner, tensor-map encoding and kernel launches.  All compute is in the
// kernels included below.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gdattn.h"

#include "combine.cuh"
#include "core_decode.cuh"
#include "read_probe.cuh"
#include "tc_decode.cuh"
#include "tc_pair_decode.cuh"
#include "tc_pair_fp8_decode.cuh"
#include "tc_pair_multi_decode.cuh"
#include "tc_pair_prefill.cuh"
#include "tc_global_prefill.cuh"

using namespace gdattn;

// Split-KV scratch of gdattn_decode_noalloc: one array per device context,
// laid out like a caller workspace (the fixed header of status word, part
// counters and epochs, then partial LSE and partial O).
// A __device__ array without initialiser occupies no space in the binary.
constexpr size_t kNoallocScratchBytes = GDATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

namespace {

enum class PathKind { kNone, kCore, kTc, kTcPair };

struct LayerPlan {
  PathKind kind = PathKind::kNone;
  int32_t grid = 0;            // CTAs sharing the KV range (P)
  int32_t units_per_seq = 1;   // query-head groups per sequence
  int32_t heads_per_unit = 0;
  int64_t slots = 0;           // partial slots: P + units
  int32_t align = 1;           // chunk granularity in tokens (one tile / stage)
  bool merge_in_kernel = false;  // the decode kernel merges split units itself
  int32_t split_k = 1;           // > 1: each unit cut into split_k whole-tile parts
  bool tagged = false;           // parts stored as 64-bit (value, tag) words
  // A separate LSE-combine launch follows the decode kernel.
  bool needs_combine() const { return grid > 1 && !merge_in_kernel; }
  // Workspace: status word | per-unit part counters | per-unit epochs |
  // partial LSE | partial O.
  size_t off_cnt = 0, off_epoch = 0, off_lse = 0, off_o = 0, bytes = 0;
};

constexpr size_t kStatusBytes = 256;
// Every workspace starts with the same header, whatever the plan: the status
// word, then one part counter and one epoch per unit index below kMaxUnits.
// Counters must read zero and epochs must hold the last call's tag when a call
// starts; with fixed offsets no plan's partials ever land on them, so calls
// with different plans (geometry, batch, split) can take turns on one
// workspace.  A plan with more units is refused.
constexpr int64_t kMaxUnits = 16384;
constexpr size_t kOffCounters = kStatusBytes;
constexpr size_t kOffEpochs = kOffCounters + 4 * kMaxUnits;
constexpr size_t kHeaderBytes = kOffEpochs + 4 * kMaxUnits;
static_assert(kHeaderBytes % 256 == 0, "partials start 256-byte aligned");

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// ----------------------------------------------------------------- kernels
// Resolve the CUDA-core kernel instantiation for (D, G, Hkv, shared).
struct CoreKernel {
  void (*fn)(const CoreParams);
  int threads;
  int smem;
  int tokens_per_stage;
  int min_blocks;
};

template <int D, int G, int HKV, bool SH>
CoreKernel core_kernel_entry() {
  using Cfg = CoreConfig<D, G, HKV, SH>;
  return CoreKernel{core_decode_kernel<D, G, HKV, SH>, Cfg::kThreads, Cfg::SMEM, Cfg::T, 1};
}

template <int D, int G, int HKV>
CoreKernel core_pick_shared(bool shared) {
  return shared ? core_kernel_entry<D, G, HKV, true>() : core_kernel_entry<D, G, HKV, false>();
}

template <int D, int G>
CoreKernel core_pick_hkv(int hkv, bool shared) {
  switch (hkv) {
    case 1: return core_pick_shared<D, G, 1>(shared);
    case 2: return core_pick_shared<D, G, 2>(shared);
    case 4: return core_pick_shared<D, G, 4>(shared);
    case 8: return core_pick_shared<D, G, 8>(shared);
    default: return CoreKernel{nullptr, 0, 0, 0, 0};
  }
}

template <int D>
CoreKernel core_pick_g(int g, int hkv, bool shared) {
  switch (g) {
    case 1: return core_pick_hkv<D, 1>(hkv, shared);
    case 2: return core_pick_hkv<D, 2>(hkv, shared);
    case 4: return core_pick_hkv<D, 4>(hkv, shared);
    default: return CoreKernel{nullptr, 0, 0, 0, 0};
  }
}

CoreKernel core_pick(int d, int g, int hkv, bool shared) {
  switch (d) {
    case 256: return core_pick_g<256>(g, hkv, shared);
    case 512: return core_pick_g<512>(g, hkv, shared);
    default: return CoreKernel{nullptr, 0, 0, 0, 0};
  }
}

// Blocks of `fn` resident per SM with `smem` dynamic bytes (after opting in to
// the shared-memory size).  Cached per kernel.
template <class F>
int blocks_per_sm(F fn, int threads, int smem) {
  if (cudaFuncSetAttribute(reinterpret_cast<const void *>(fn),
                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 0;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem) != cudaSuccess) return 0;
  return nb;
}

struct KernelInfo {
  const void *key;
  int blocks;
};

// Resident blocks per SM for each kernel instantiation, measured once.
int cached_blocks_per_sm(const void *key, int threads, int smem,
                         int (*query)(const void *, int, int)) {
  static std::mutex mu;
  static KernelInfo cache[64];
  static int used = 0;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < used; ++i)
    if (cache[i].key == key) return cache[i].blocks;
  const int nb = query(key, threads, smem);
  if (nb > 0 && used < 64) cache[used++] = KernelInfo{key, nb};
  return nb;
}

int query_core(const void *fn, int threads, int smem) {
  return blocks_per_sm(reinterpret_cast<void (*)(const CoreParams)>(const_cast<void *>(fn)),
                       threads, smem);
}
int query_tc(const void *fn, int threads, int smem) {
  using TcFn = void (*)(const CUtensorMap, const CUtensorMap, const TcParams);
  return blocks_per_sm(reinterpret_cast<TcFn>(const_cast<void *>(fn)), threads, smem);
}
int query_tc_append(const void *fn, int threads, int smem) {
  using TcFn = void (*)(const CUtensorMap, const CUtensorMap, const TcParams, const TcAppend);
  return blocks_per_sm(reinterpret_cast<TcFn>(const_cast<void *>(fn)), threads, smem);
}
int query_tc_pair(const void *fn, int threads, int smem) {
  using TcFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const TcParams);
  return blocks_per_sm(reinterpret_cast<TcFn>(const_cast<void *>(fn)), threads, smem);
}
int query_tc_pair_fp8(const void *fn, int threads, int smem) {
  using TcFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const TcParams,
                        const Fp8Scales);
  return blocks_per_sm(reinterpret_cast<TcFn>(const_cast<void *>(fn)), threads, smem);
}
using MultiPassFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                             const TcParams, const MultiTokens);
int query_tc_pair_multi(const void *fn, int threads, int smem) {
  return blocks_per_sm(reinterpret_cast<MultiPassFn>(const_cast<void *>(fn)), threads, smem);
}
int query_prefill(const void *fn, int threads, int smem) {
  using Fn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const PrefillParams);
  return blocks_per_sm(reinterpret_cast<Fn>(const_cast<void *>(fn)), threads, smem);
}
// The single-pass multi-token kernel for T tokens (1..8), else null.
MultiPassFn multi_pass_kernel(int32_t T) {
  switch (T) {
    case 1: return tc_pair_multi_decode_kernel<1>;
    case 2: return tc_pair_multi_decode_kernel<2>;
    case 3: return tc_pair_multi_decode_kernel<3>;
    case 4: return tc_pair_multi_decode_kernel<4>;
    case 5: return tc_pair_multi_decode_kernel<5>;
    case 6: return tc_pair_multi_decode_kernel<6>;
    case 7: return tc_pair_multi_decode_kernel<7>;
    case 8: return tc_pair_multi_decode_kernel<8>;
    default: return nullptr;
  }
}
int query_tc_pair_append(const void *fn, int threads, int smem) {
  using TcFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const TcParams,
                        const TcAppend);
  return blocks_per_sm(reinterpret_cast<TcFn>(const_cast<void *>(fn)), threads, smem);
}

int query_probe(const void *fn, int threads, int smem) {
  return blocks_per_sm(reinterpret_cast<void (*)(const ReadProbeParams)>(const_cast<void *>(fn)),
                       threads, smem);
}

// ---------------------------------------------------------------- planning
gdattn_status check_desc(const gdattn_layer_desc *d) {
  if (d == nullptr) return GDATTN_ERR_INVALID_ARG;
  if (d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->head_dim <= 0 || d->cache_capacity <= 0)
    return GDATTN_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads != 0) return GDATTN_ERR_INVALID_ARG;
  if (d->window < 0 || d->split_ctas < 0 ||
      (d->flags & ~(GDATTN_FLAG_EVEN_UNITS | GDATTN_FLAG_TEST_WITHHOLD_KV)) != 0)
    return GDATTN_ERR_INVALID_ARG;
  if (!(d->softcap >= 0.f) || !std::isfinite(d->softcap) || !std::isfinite(d->scale))
    return GDATTN_ERR_INVALID_ARG;
  if (d->kv_shared != 0 && d->kv_shared != 1) return GDATTN_ERR_INVALID_ARG;
  const int64_t dense = static_cast<int64_t>(d->cache_capacity) * d->n_kv_heads * d->head_dim;
  if (d->cache_batch_stride != 0 && (d->cache_batch_stride < dense || d->cache_batch_stride % 8 != 0))
    return GDATTN_ERR_INVALID_ARG;
  return GDATTN_OK;
}

PathKind choose_path(const gdattn_layer_desc *d) {
  const int g = d->n_q_heads / d->n_kv_heads;
  if ((g == 16 || g == 8) && d->head_dim == 512) return PathKind::kTc;
  if (g == 2 && d->head_dim == 256 && d->kv_shared == 0) return PathKind::kTcPair;
  if ((d->head_dim == 256 || d->head_dim == 512) && (g == 1 || g == 2 || g == 4) &&
      (d->n_kv_heads == 1 || d->n_kv_heads == 2 || d->n_kv_heads == 4 || d->n_kv_heads == 8))
    return PathKind::kCore;
  return PathKind::kNone;
}

// fp8: plan for the fp8 cache kernel of the same path (only the pair path has one).
// tokens > 0: plan for the single-pass multi-token pair kernel (d's window is
// already the union window of the step); a unit then has 2 * tokens rows.
gdattn_status make_plan(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *d,
                        LayerPlan &pl, bool fp8 = false, int32_t tokens = 0) {
  gdattn_status st = check_desc(d);
  if (st != GDATTN_OK) return st;
  if (batch <= 0 || max_seqlen <= 0) return GDATTN_ERR_INVALID_ARG;
  pl.kind = choose_path(d);
  if (pl.kind == PathKind::kNone || ((fp8 || tokens > 0) && pl.kind != PathKind::kTcPair))
    return GDATTN_ERR_UNSUPPORTED;
  // Units (query-head groups) of the call: one per sequence on the CUDA-core
  // path, one per (sequence, KV head) on the tcgen05 paths.
  const int64_t units =
      static_cast<int64_t>(batch) * (pl.kind == PathKind::kCore ? 1 : d->n_kv_heads);
  if (units > kMaxUnits) return GDATTN_ERR_UNSUPPORTED;
  const int nsm = sm_count();
  if (nsm <= 0) return GDATTN_ERR_CUDA;
  int per_sm = 1, min_tokens = 64;
  if (pl.kind == PathKind::kCore) {
    const CoreKernel ck = core_pick(d->head_dim, d->n_q_heads / d->n_kv_heads, d->n_kv_heads,
                                    d->kv_shared != 0);
    if (ck.fn == nullptr) return GDATTN_ERR_UNSUPPORTED;
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(ck.fn), ck.threads, ck.smem,
                                  query_core);
    min_tokens = 2 * ck.tokens_per_stage;
    pl.align = ck.tokens_per_stage;
    pl.units_per_seq = 1;
    pl.heads_per_unit = d->n_q_heads;
  } else if (pl.kind == PathKind::kTc) {
    // Every instantiation of the 16-head kernel shares one configuration; the
    // queries also set each one's shared-memory attribute before its launch.
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kernel<16>),
                                  TcConfig::kThreads, TcConfig::SMEM, query_tc);
    const int others[] = {
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kernel<8>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_append_kernel<16>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_append),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_append_kernel<8>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_append),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kv_kernel<16>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_pair),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kv_kernel<8>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_pair),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kv_append_kernel<16>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_pair_append),
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_decode_kv_append_kernel<8>),
                             TcConfig::kThreads, TcConfig::SMEM, query_tc_pair_append)};
    for (int nb : others)
      if (nb != per_sm) return GDATTN_ERR_CUDA;
    min_tokens = 2 * TcConfig::TILE;
    pl.align = TcConfig::TILE;
    pl.units_per_seq = d->n_kv_heads;
    pl.heads_per_unit = d->n_q_heads / d->n_kv_heads;  // 8 or 16 (the kernel pads to 16)
  } else if (tokens > 0) {
    if (multi_pass_kernel(tokens) == nullptr) return GDATTN_ERR_UNSUPPORTED;
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(multi_pass_kernel(tokens)),
                                  TcPairMultiConfig::kThreads, TcPairMultiConfig::SMEM,
                                  query_tc_pair_multi);
    min_tokens = 2 * TcPairMultiConfig::TILE;
    pl.align = TcPairMultiConfig::TILE;
    pl.units_per_seq = d->n_kv_heads;
    pl.heads_per_unit = 2 * tokens;  // query rows of a unit: (token, head)
  } else if (fp8) {
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(tc_pair_fp8_decode_kernel),
                                  TcPairFp8Config::kThreads, TcPairFp8Config::SMEM,
                                  query_tc_pair_fp8);
    min_tokens = 2 * TcPairFp8Config::TILE;
    pl.align = TcPairFp8Config::TILE;
    pl.units_per_seq = d->n_kv_heads;
    pl.heads_per_unit = TcPairFp8Config::G;
  } else {
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(tc_pair_decode_kernel),
                                  TcPairConfig::kThreads, TcPairConfig::SMEM, query_tc_pair);
    if (cached_blocks_per_sm(reinterpret_cast<const void *>(tc_pair_decode_append_kernel),
                             TcPairConfig::kThreads, TcPairConfig::SMEM,
                             query_tc_pair_append) != per_sm ||
        cached_blocks_per_sm(reinterpret_cast<const void *>(tc_pair_decode_multi_kernel),
                             TcPairConfig::kThreads, TcPairConfig::SMEM, query_tc_pair) != per_sm)
      return GDATTN_ERR_CUDA;
    min_tokens = 2 * TcPairConfig::TILE;
    pl.align = TcPairConfig::TILE;
    pl.units_per_seq = d->n_kv_heads;
    pl.heads_per_unit = TcPairConfig::G;
  }
  if (per_sm <= 0) return GDATTN_ERR_CUDA;
  int64_t per_unit = max_seqlen;
  if (d->window > 0 && d->window < per_unit) per_unit = d->window;
  if (d->cache_capacity < per_unit) per_unit = d->cache_capacity;
  const int64_t total = units * per_unit;
  int64_t grid = (total + min_tokens - 1) / min_tokens;
  const int64_t cap = static_cast<int64_t>(nsm) * per_sm;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  if (d->split_ctas > 0) grid = d->split_ctas;
  // Even units on the tcgen05 kernels: cut every unit into k whole-tile parts,
  // k minimising the largest part (the smallest such k, for cheaper merges)
  // with all units * k CTAs resident at once.  No CTA then straddles two units.
  pl.split_k = 1;
  if ((d->flags & GDATTN_FLAG_EVEN_UNITS) && d->split_ctas == 0 && pl.kind != PathKind::kCore) {
    const int64_t tiles = (per_unit + pl.align - 1) / pl.align;
    int64_t best = tiles;
    // At most 64 parts per unit: the LSE merge of more parts costs more than the
    // shorter parts save (one 32 KiB unit of 16 heads merged from 128 parts took
    // longer than from 64).
    for (int64_t k = 2; k <= tiles && units * k <= cap && k <= 64; ++k) {
      const int64_t most = (tiles + k - 1) / k;
      if (most < best) {
        best = most;
        pl.split_k = static_cast<int32_t>(k);
      }
    }
    if (pl.split_k > 1) grid = units * pl.split_k;
  }
  if (grid > 65535) return GDATTN_ERR_INVALID_ARG;
  pl.grid = static_cast<int32_t>(grid);
  pl.slots = grid + units;
  // The pair kernels (single- and multi-token) merge split units themselves;
  // the 16-head kernel leaves them to the combine kernel.
  pl.merge_in_kernel = pl.kind == PathKind::kTcPair;
  // Parts of split units as tagged (value, tag) words: the single-token pair
  // kernels; the multi-token kernel stores plain partials and counts them.
  pl.tagged = pl.merge_in_kernel && pl.split_k > 1 && tokens == 0;
  const size_t elem = pl.tagged ? 8 : 4;
  pl.off_cnt = kOffCounters;
  pl.off_epoch = kOffEpochs;
  pl.off_lse = kHeaderBytes;
  pl.off_o = align256(pl.off_lse + static_cast<size_t>(pl.slots) * pl.heads_per_unit * elem);
  pl.bytes =
      align256(pl.off_o + static_cast<size_t>(pl.slots) * pl.heads_per_unit * d->head_dim * elem);
  return GDATTN_OK;
}

// --------------------------------------------------------------- launching
cudaLaunchConfig_t launch_config(dim3 grid, int threads, int smem, cudaStream_t stream,
                                 cudaLaunchAttribute *attr, bool pdl = true) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  // Programmatic dependent launch: the kernel may start while its predecessor
  // drains; every kernel here waits (griddepcontrol.wait) before touching memory.
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cfg;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// K or V cache [B][C][Hkv][D] as a 4-D tensor map {D, Hkv, C, B} read in
// 128-byte x 1-head x 64-token boxes with 128-byte swizzle: 64 bf16 elements,
// or 128 e4m3 codes (fp8), per box row.
bool encode_cache_map(EncodeTiledFn enc, CUtensorMap *map, const void *base, int32_t D,
                      int32_t Hkv, int32_t C, int32_t batch, int64_t bstride, uint32_t tile,
                      bool fp8 = false) {
  const cuuint64_t esz = fp8 ? 1 : 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(batch)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * esz,
                                 static_cast<cuuint64_t>(Hkv) * D * esz,
                                 static_cast<cuuint64_t>(bstride) * esz};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / esz), 1, tile, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [B * Hq][D] bf16 as a 2-D tensor map read in whole-row boxes of `rows`
// rows, unswizzled (row-major in shared memory).
bool encode_q_rows_map(EncodeTiledFn enc, CUtensorMap *map, const void *q, int32_t D,
                       int64_t total_rows, uint32_t rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(total_rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(D), rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [T][rows][D] bf16 (rows = B * Hq) as a 3-D tensor map read in
// {64 d, box_heads rows, box_tokens tokens} boxes with 128-byte swizzle: the
// query rows of a unit (box_heads heads x box_tokens tokens) land as consecutive
// 128-byte rows, token-major; tokens past T read as zeros.
bool encode_q_tokens_map(EncodeTiledFn enc, CUtensorMap *map, const void *q, int32_t D,
                         int64_t rows, int32_t T, int32_t box_tokens, int32_t box_heads = 2) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(rows) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_heads),
                             static_cast<cuuint32_t>(box_tokens)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// q [B * Hq][D] bf16 as a 2-D tensor map read in 64-d x 16-row boxes.
bool encode_q_map(EncodeTiledFn enc, CUtensorMap *map, const void *q, int32_t D, int64_t rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, 16};
  const cuuint32_t estr[2] = {1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(q), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// tokens > 0: the parts of a single-pass multi-token step (token-major out / lse).
gdattn_status launch_combine_internal(const LayerPlan &pl, const Geometry &geo, const float *ws_lse,
                                      const float *ws_o, const gdattn_layer_desc *d, void *out,
                                      float *lse, cudaStream_t stream, int32_t tokens = 0) {
  CombineParams cp = {};
  cp.tokens = tokens;
  cp.parts_o = ws_o;
  cp.parts_lse = ws_lse;
  cp.out = static_cast<uint16_t *>(out);
  cp.lse = lse;
  cp.n_q_heads = d->n_q_heads;
  cp.head_dim = d->head_dim;
  cp.geo = geo;
  cp.heads_per_unit = pl.heads_per_unit;
  cp.n_splits = 0;
  cp.split_k = pl.split_k;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg =
      launch_config(dim3(static_cast<unsigned>(geo.batch * pl.units_per_seq),
                         static_cast<unsigned>(pl.heads_per_unit)),
                    combine_threads(d->head_dim), 0, stream, attr);
  return cudaLaunchKernelEx(&cfg, combine_kernel<true>, cp) == cudaSuccess ? GDATTN_OK
                                                                            : GDATTN_ERR_CUDA;
}

// Host checks shared by both decode entry points (the workspace aside).
gdattn_status check_decode_args(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                const gdattn_layer_desc *desc, const void *out, const float *lse) {
  if (q == nullptr || k_cache == nullptr || seqlens == nullptr || out == nullptr || desc == nullptr)
    return GDATTN_ERR_INVALID_ARG;
  gdattn_status st = check_desc(desc);
  if (st != GDATTN_OK) return st;
  if ((desc->kv_shared == 1) != (v_cache == nullptr)) return GDATTN_ERR_INVALID_ARG;
  if (batch <= 0 || max_seqlen <= 0) return GDATTN_ERR_INVALID_ARG;
  if (choose_path(desc) == PathKind::kNone) return GDATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || (v_cache && !aligned16(v_cache)) ||
      !aligned16(out) || (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GDATTN_ERR_MISALIGNED;
  return GDATTN_OK;
}

// Enqueues the decode kernel (and the combine when the plan splits) with the
// split-KV scratch at `ws`: status word, then partial LSE, then partial O.
// k_new / v_new (optional): the current token's rows, appended by the kernel.
// pdl = false: a plain launch, for a decode that reads lengths the kernel just
// before it on the stream wrote (the kernels read seqlens before their
// dependency wait).
// cache_batch (> 0): sequences in the caches when it differs from batch (a
// multi-token step: query sequence b reads cache sequence b % cache_batch).
gdattn_status enqueue_decode(const LayerPlan &pl, const void *q, const void *k_cache,
                             const void *v_cache, const int32_t *seqlens, int32_t batch,
                             const gdattn_layer_desc *desc, void *out, float *lse, uint8_t *ws,
                             cudaStream_t stream, const void *k_new = nullptr,
                             const void *v_new = nullptr, bool pdl = true,
                             int32_t cache_batch = 0) {
  if (cache_batch <= 0) cache_batch = batch;
  uint32_t *status = reinterpret_cast<uint32_t *>(ws);
  uint32_t *counters = reinterpret_cast<uint32_t *>(ws + pl.off_cnt);
  uint32_t *epochs = reinterpret_cast<uint32_t *>(ws + pl.off_epoch);
  float *ws_lse = reinterpret_cast<float *>(ws + pl.off_lse);
  float *ws_o = reinterpret_cast<float *>(ws + pl.off_o);
  const int32_t D = desc->head_dim;
  const int32_t Hkv = desc->n_kv_heads;
  const int64_t bstride = desc->cache_batch_stride != 0
                              ? desc->cache_batch_stride
                              : static_cast<int64_t>(desc->cache_capacity) * Hkv * D;
  const float log2e = 1.4426950408889634f;
  const float qscale = desc->softcap > 0.f ? desc->scale / desc->softcap : desc->scale * log2e;
  const float post = desc->softcap > 0.f ? desc->softcap * log2e : 0.f;

  Geometry geo;
  geo.seqlens = seqlens;
  geo.batch = batch;
  geo.units_per_seq = pl.units_per_seq;
  geo.window = desc->window;
  geo.capacity = desc->cache_capacity;
  geo.nchunks_align = pl.grid | (pl.align << 16);  // grid < 2^16, align <= 128
  geo.cache_batch = cache_batch;

  cudaLaunchAttribute attr[1];
  if (pl.kind == PathKind::kCore) {
    const CoreKernel ck = core_pick(D, desc->n_q_heads / Hkv, Hkv, desc->kv_shared != 0);
    CoreParams cp;
    cp.q = static_cast<const uint16_t *>(q);
    cp.k = static_cast<const uint16_t *>(k_cache);
    cp.v = static_cast<const uint16_t *>(v_cache ? v_cache : k_cache);
    cp.batch_stride = bstride;
    cp.out = static_cast<uint16_t *>(out);
    cp.lse = lse;
    cp.ws_o = ws_o;
    cp.ws_lse = ws_lse;
    cp.status = status;
    cp.k_new = static_cast<const uint16_t *>(k_new);
    cp.v_new = static_cast<const uint16_t *>(v_new);
    cp.geo = geo;
    cp.n_q_heads = desc->n_q_heads;
    cp.qscale = qscale;
    cp.post = post;
    cp.test_withhold = (desc->flags & GDATTN_FLAG_TEST_WITHHOLD_KV) ? 1 : 0;
    cudaLaunchConfig_t cfg =
        launch_config(dim3(pl.grid), ck.threads, ck.smem, stream, attr, pdl);
    if (cudaLaunchKernelEx(&cfg, ck.fn, cp) != cudaSuccess) return GDATTN_ERR_CUDA;
  } else {
    EncodeTiledFn enc = encode_tiled();
    if (enc == nullptr) return GDATTN_ERR_CUDA;
    CUtensorMap kmap, vmap, qmap;
    if (!encode_cache_map(enc, &kmap, k_cache, D, Hkv, desc->cache_capacity, cache_batch,
                          bstride, TcConfig::TILE) ||
        !encode_q_map(enc, &qmap, q, D, static_cast<int64_t>(batch) * desc->n_q_heads))
      return GDATTN_ERR_CUDA;
    TcParams tp;
    tp.out = static_cast<uint16_t *>(out);
    tp.lse = lse;
    tp.ws_o = ws_o;
    tp.ws_lse = ws_lse;
    tp.status = status;
    TcAppend ap;
    ap.k_new = static_cast<const uint16_t *>(k_new);
    ap.v_new = static_cast<const uint16_t *>(v_new);
    ap.k_cache = static_cast<uint16_t *>(const_cast<void *>(k_cache));
    ap.v_cache = static_cast<uint16_t *>(const_cast<void *>(v_cache));
    ap.batch_stride = bstride;
    ap.n_kv_heads = Hkv;
    tp.counters = counters;
    tp.epochs = epochs;
    tp.test_withhold = (desc->flags & GDATTN_FLAG_TEST_WITHHOLD_KV) ? 1 : 0;
    tp.merge_in_kernel = pl.merge_in_kernel ? 1 : 0;
    tp.split_k = pl.split_k;
    tp.geo = geo;
    tp.n_q_heads = desc->n_q_heads;
    tp.qscale = qscale;
    tp.post = post;
    if (pl.kind == PathKind::kTc) {
      cudaLaunchConfig_t cfg =
          launch_config(dim3(pl.grid), TcConfig::kThreads, TcConfig::SMEM, stream, attr, pdl);
      const bool g8 = pl.heads_per_unit == 8;
      cudaError_t e;
      if (v_cache == nullptr) {
        if (k_new != nullptr)
          e = g8 ? cudaLaunchKernelEx(&cfg, tc_decode_append_kernel<8>, kmap, qmap, tp, ap)
                 : cudaLaunchKernelEx(&cfg, tc_decode_append_kernel<16>, kmap, qmap, tp, ap);
        else
          e = g8 ? cudaLaunchKernelEx(&cfg, tc_decode_kernel<8>, kmap, qmap, tp)
                 : cudaLaunchKernelEx(&cfg, tc_decode_kernel<16>, kmap, qmap, tp);
      } else {
        if (!encode_cache_map(enc, &vmap, v_cache, D, Hkv, desc->cache_capacity, cache_batch,
                              bstride, TcConfig::TILE))
          return GDATTN_ERR_CUDA;
        if (k_new != nullptr)
          e = g8 ? cudaLaunchKernelEx(&cfg, tc_decode_kv_append_kernel<8>, kmap, vmap, qmap, tp, ap)
                 : cudaLaunchKernelEx(&cfg, tc_decode_kv_append_kernel<16>, kmap, vmap, qmap, tp,
                                      ap);
        else
          e = g8 ? cudaLaunchKernelEx(&cfg, tc_decode_kv_kernel<8>, kmap, vmap, qmap, tp)
                 : cudaLaunchKernelEx(&cfg, tc_decode_kv_kernel<16>, kmap, vmap, qmap, tp);
      }
      if (e != cudaSuccess) return GDATTN_ERR_CUDA;
    } else {
      if (!encode_cache_map(enc, &vmap, v_cache, D, Hkv, desc->cache_capacity, cache_batch,
                            bstride, TcPairConfig::TILE))
        return GDATTN_ERR_CUDA;
      cudaLaunchConfig_t cfg = launch_config(dim3(pl.grid), TcPairConfig::kThreads,
                                             TcPairConfig::SMEM, stream, attr, pdl);
      const cudaError_t e =
          k_new != nullptr
              ? cudaLaunchKernelEx(&cfg, tc_pair_decode_append_kernel, kmap, vmap, qmap, tp, ap)
          : cache_batch != batch
              ? cudaLaunchKernelEx(&cfg, tc_pair_decode_multi_kernel, kmap, vmap, qmap, tp)
              : cudaLaunchKernelEx(&cfg, tc_pair_decode_kernel, kmap, vmap, qmap, tp);
      if (e != cudaSuccess) return GDATTN_ERR_CUDA;
    }
  }
  if (pl.needs_combine())
    return launch_combine_internal(pl, geo, ws_lse, ws_o, desc, out, lse, stream);
  return GDATTN_OK;
}

// Enqueues the fp8-cache pair kernel (it merges split units itself).
gdattn_status enqueue_decode_fp8(const LayerPlan &pl, const void *q, const void *k_codes,
                                 const void *v_codes, const float *k_scale, const float *v_scale,
                                 const int32_t *seqlens, int32_t batch,
                                 const gdattn_layer_desc *desc, void *out, float *lse,
                                 uint8_t *ws, cudaStream_t stream) {
  const int32_t D = desc->head_dim;
  const int32_t Hkv = desc->n_kv_heads;
  const int64_t bstride = desc->cache_batch_stride != 0
                              ? desc->cache_batch_stride
                              : static_cast<int64_t>(desc->cache_capacity) * Hkv * D;
  const float log2e = 1.4426950408889634f;
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return GDATTN_ERR_CUDA;
  CUtensorMap kmap, vmap, qmap;
  if (!encode_cache_map(enc, &kmap, k_codes, D, Hkv, desc->cache_capacity, batch, bstride,
                        TcPairFp8Config::TILE, true) ||
      !encode_cache_map(enc, &vmap, v_codes, D, Hkv, desc->cache_capacity, batch, bstride,
                        TcPairFp8Config::TILE, true) ||
      !encode_q_rows_map(enc, &qmap, q, D, static_cast<int64_t>(batch) * desc->n_q_heads,
                         TcPairFp8Config::G))
    return GDATTN_ERR_CUDA;
  TcParams tp;
  tp.out = static_cast<uint16_t *>(out);
  tp.lse = lse;
  tp.ws_o = reinterpret_cast<float *>(ws + pl.off_o);
  tp.ws_lse = reinterpret_cast<float *>(ws + pl.off_lse);
  tp.status = reinterpret_cast<uint32_t *>(ws);
  tp.counters = reinterpret_cast<uint32_t *>(ws + pl.off_cnt);
  tp.epochs = reinterpret_cast<uint32_t *>(ws + pl.off_epoch);
  tp.merge_in_kernel = 1;
  tp.test_withhold = (desc->flags & GDATTN_FLAG_TEST_WITHHOLD_KV) ? 1 : 0;
  tp.split_k = pl.split_k;
  tp.geo.seqlens = seqlens;
  tp.geo.batch = batch;
  tp.geo.units_per_seq = pl.units_per_seq;
  tp.geo.window = desc->window;
  tp.geo.capacity = desc->cache_capacity;
  tp.geo.nchunks_align = pl.grid | (pl.align << 16);
  tp.geo.cache_batch = batch;
  tp.n_q_heads = desc->n_q_heads;
  tp.qscale = desc->softcap > 0.f ? desc->scale / desc->softcap : desc->scale * log2e;
  tp.post = desc->softcap > 0.f ? desc->softcap * log2e : 0.f;
  Fp8Scales sc;
  sc.k_scale = k_scale;
  sc.v_scale = v_scale;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(dim3(pl.grid), TcPairFp8Config::kThreads,
                                         TcPairFp8Config::SMEM, stream, attr);
  return cudaLaunchKernelEx(&cfg, tc_pair_fp8_decode_kernel, kmap, vmap, qmap, tp, sc) ==
                 cudaSuccess
             ? GDATTN_OK
             : GDATTN_ERR_CUDA;
}

// ------------------------------------------------------ multi-query decode
// Per-token context lengths of a T-token step: lens[t][b] = seqlens[b] - (T - 1 - t).
__global__ void multi_lengths_kernel(const int32_t *seqlens, int32_t batch, int32_t T,
                                     int32_t *lens) {
  for (int32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < T * batch;
       i += gridDim.x * blockDim.x) {
    const int32_t t = i / batch, b = i - t * batch;
    lens[i] = seqlens[b] - (T - 1 - t);
  }
}

constexpr int32_t kMaxMultiTokens = 64;

// Multi-token steps of the pair geometry with at most 8 tokens run in one pass
// over the cache (tc_pair_multi_decode.cuh); the others as T x B sequences.
bool multi_single_pass(const gdattn_layer_desc *d, int32_t T) {
  return choose_path(d) == PathKind::kTcPair && T <= TcPairMultiConfig::TMAX;
}

// The layer as the single-pass kernel plans it: the union of the T tokens'
// windows, w + T - 1 positions (still 0 for a global layer).
gdattn_layer_desc union_window_desc(const gdattn_layer_desc *d, int32_t T) {
  gdattn_layer_desc u = *d;
  if (u.window > 0) u.window = u.window > INT32_MAX - (T - 1) ? INT32_MAX : u.window + (T - 1);
  return u;
}

// Multi-token steps of more than 8 tokens (prompt chunks) run as flash prefill
// on the pair geometry (tc_pair_prefill.cuh) and on the global geometry with
// K = V (tc_global_prefill.cuh), up to this many tokens.
constexpr int32_t kMaxPrefillTokens = 1 << 20;
bool prefill_geometry(const gdattn_layer_desc *d) {
  const PathKind k = choose_path(d);
  return k == PathKind::kTcPair || (k == PathKind::kTc && d->kv_shared == 1);
}
bool multi_prefill(const gdattn_layer_desc *d, int32_t T) {
  return prefill_geometry(d) && T > TcPairMultiConfig::TMAX;
}

using GlobalPrefillFn = void (*)(const CUtensorMap, const CUtensorMap, const PrefillParams);
int query_global_prefill(const void *fn, int threads, int smem) {
  return blocks_per_sm(reinterpret_cast<GlobalPrefillFn>(const_cast<void *>(fn)), threads, smem);
}

// Query tokens per prefill block, and CTAs per block (the global kernel splits
// the head dimension over two).
int32_t prefill_block_tokens(const gdattn_layer_desc *d) {
  return choose_path(d) == PathKind::kTcPair
             ? TcPrefillConfig::QT
             : TcGlobalPrefillConfig::M / (d->n_q_heads / d->n_kv_heads);
}
int32_t prefill_ctas_per_block(const gdattn_layer_desc *d) {
  return choose_path(d) == PathKind::kTcPair ? 1 : 2;
}

// Checks the prefill launch for this geometry (and sets the kernel's shared
// memory limit); the workspace is the fixed header alone (the status word).
gdattn_status plan_prefill(int32_t batch, int32_t T, const gdattn_layer_desc *d,
                           size_t *ws_bytes) {
  gdattn_status st = check_desc(d);
  if (st != GDATTN_OK) return st;
  if (batch <= 0 || T < 1 || T > kMaxPrefillTokens) return GDATTN_ERR_INVALID_ARG;
  if (!prefill_geometry(d)) return GDATTN_ERR_UNSUPPORTED;
  const int32_t qt = prefill_block_tokens(d);
  const int64_t nblocks = (T + qt - 1) / qt;
  if (static_cast<int64_t>(batch) * d->n_kv_heads * nblocks * prefill_ctas_per_block(d) >
      INT32_MAX)
    return GDATTN_ERR_UNSUPPORTED;
  int per_sm = 0;
  if (choose_path(d) == PathKind::kTcPair) {
    per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(tc_pair_prefill_kernel),
                                  TcPrefillConfig::kThreads, TcPrefillConfig::SMEM, query_prefill);
  } else {
    const void *fn = d->n_q_heads / d->n_kv_heads == 8
                         ? reinterpret_cast<const void *>(tc_global_prefill_kernel<8>)
                         : reinterpret_cast<const void *>(tc_global_prefill_kernel<16>);
    per_sm = cached_blocks_per_sm(fn, TcGlobalPrefillConfig::kThreads, TcGlobalPrefillConfig::SMEM,
                                  query_global_prefill);
  }
  if (per_sm <= 0) return GDATTN_ERR_CUDA;
  *ws_bytes = kHeaderBytes;
  return GDATTN_OK;
}

gdattn_status enqueue_prefill(const void *q, const void *k_cache, const void *v_cache,
                              const int32_t *seqlens, int32_t batch, int32_t T,
                              const gdattn_layer_desc *desc, void *out, float *lse, uint8_t *ws,
                              cudaStream_t stream) {
  const int32_t D = desc->head_dim;
  const int32_t Hkv = desc->n_kv_heads;
  const int64_t bstride = desc->cache_batch_stride != 0
                              ? desc->cache_batch_stride
                              : static_cast<int64_t>(desc->cache_capacity) * Hkv * D;
  const float log2e = 1.4426950408889634f;
  const bool pair = choose_path(desc) == PathKind::kTcPair;
  const int32_t GU = desc->n_q_heads / Hkv;
  const int32_t qt = prefill_block_tokens(desc);
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return GDATTN_ERR_CUDA;
  CUtensorMap kmap, vmap, qmap;
  if (!encode_cache_map(enc, &kmap, k_cache, D, Hkv, desc->cache_capacity, batch, bstride,
                        TcPrefillConfig::TILE) ||
      (pair && !encode_cache_map(enc, &vmap, v_cache, D, Hkv, desc->cache_capacity, batch,
                                 bstride, TcPrefillConfig::TILE)) ||
      !encode_q_tokens_map(enc, &qmap, q, D, static_cast<int64_t>(batch) * desc->n_q_heads, T,
                           qt, pair ? 2 : GU))
    return GDATTN_ERR_CUDA;
  PrefillParams pp;
  pp.seqlens = seqlens;
  pp.out = static_cast<uint16_t *>(out);
  pp.lse = lse;
  pp.status = reinterpret_cast<uint32_t *>(ws);
  pp.batch = batch;
  pp.n_q_heads = desc->n_q_heads;
  pp.n_kv_heads = Hkv;
  pp.tokens = T;
  pp.nblocks = (T + qt - 1) / qt;
  pp.window = desc->window;
  pp.capacity = desc->cache_capacity;
  pp.qscale = desc->softcap > 0.f ? desc->scale / desc->softcap : desc->scale * log2e;
  pp.post = desc->softcap > 0.f ? desc->softcap * log2e : 0.f;
  pp.test_withhold = (desc->flags & GDATTN_FLAG_TEST_WITHHOLD_KV) ? 1 : 0;
  const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(batch) * Hkv * pp.nblocks *
                                              prefill_ctas_per_block(desc));
  cudaLaunchAttribute attr[1];
  cudaError_t e;
  if (pair) {
    cudaLaunchConfig_t cfg = launch_config(dim3(grid), TcPrefillConfig::kThreads,
                                           TcPrefillConfig::SMEM, stream, attr);
    e = cudaLaunchKernelEx(&cfg, tc_pair_prefill_kernel, kmap, vmap, qmap, pp);
  } else {
    cudaLaunchConfig_t cfg = launch_config(dim3(grid), TcGlobalPrefillConfig::kThreads,
                                           TcGlobalPrefillConfig::SMEM, stream, attr);
    e = GU == 8 ? cudaLaunchKernelEx(&cfg, tc_global_prefill_kernel<8>, kmap, qmap, pp)
                : cudaLaunchKernelEx(&cfg, tc_global_prefill_kernel<16>, kmap, qmap, pp);
  }
  return e == cudaSuccess ? GDATTN_OK : GDATTN_ERR_CUDA;
}

// Enqueues the single-pass multi-token kernel (it merges split units itself);
// pl comes from make_plan over union_window_desc(desc, T).
gdattn_status enqueue_decode_multi_pass(const LayerPlan &pl, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *seqlens,
                                        int32_t batch, int32_t T, const gdattn_layer_desc *desc,
                                        void *out, float *lse, uint8_t *ws,
                                        cudaStream_t stream) {
  const gdattn_layer_desc ud = union_window_desc(desc, T);
  const int32_t D = desc->head_dim;
  const int32_t Hkv = desc->n_kv_heads;
  const int64_t bstride = desc->cache_batch_stride != 0
                              ? desc->cache_batch_stride
                              : static_cast<int64_t>(desc->cache_capacity) * Hkv * D;
  const float log2e = 1.4426950408889634f;
  EncodeTiledFn enc = encode_tiled();
  if (enc == nullptr) return GDATTN_ERR_CUDA;
  CUtensorMap kmap, vmap, qmap;
  if (!encode_cache_map(enc, &kmap, k_cache, D, Hkv, desc->cache_capacity, batch, bstride,
                        TcPairMultiConfig::TILE) ||
      !encode_cache_map(enc, &vmap, v_cache, D, Hkv, desc->cache_capacity, batch, bstride,
                        TcPairMultiConfig::TILE) ||
      !encode_q_tokens_map(enc, &qmap, q, D, static_cast<int64_t>(batch) * desc->n_q_heads, T,
                           T))
    return GDATTN_ERR_CUDA;
  Geometry geo;
  geo.seqlens = seqlens;
  geo.batch = batch;
  geo.units_per_seq = pl.units_per_seq;
  geo.window = ud.window;
  geo.capacity = desc->cache_capacity;
  geo.nchunks_align = pl.grid | (pl.align << 16);
  geo.cache_batch = batch;
  TcParams tp;
  tp.out = static_cast<uint16_t *>(out);
  tp.lse = lse;
  tp.ws_o = reinterpret_cast<float *>(ws + pl.off_o);
  tp.ws_lse = reinterpret_cast<float *>(ws + pl.off_lse);
  tp.status = reinterpret_cast<uint32_t *>(ws);
  tp.counters = reinterpret_cast<uint32_t *>(ws + pl.off_cnt);
  tp.epochs = reinterpret_cast<uint32_t *>(ws + pl.off_epoch);
  tp.merge_in_kernel = pl.merge_in_kernel ? 1 : 0;
  tp.test_withhold = (desc->flags & GDATTN_FLAG_TEST_WITHHOLD_KV) ? 1 : 0;
  tp.split_k = pl.split_k;
  tp.geo = geo;
  tp.n_q_heads = desc->n_q_heads;
  tp.qscale = desc->softcap > 0.f ? desc->scale / desc->softcap : desc->scale * log2e;
  tp.post = desc->softcap > 0.f ? desc->softcap * log2e : 0.f;
  const MultiTokens mt = {desc->window};
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(dim3(pl.grid), TcPairMultiConfig::kThreads,
                                         TcPairMultiConfig::SMEM, stream, attr);
  if (cudaLaunchKernelEx(&cfg, multi_pass_kernel(T), kmap, vmap, qmap, tp, mt) != cudaSuccess)
    return GDATTN_ERR_CUDA;
  if (pl.needs_combine())  // not with the in-kernel merge; kept for a plan without it
    return launch_combine_internal(pl, geo, tp.ws_lse, tp.ws_o, desc, out, lse, stream, T);
  return GDATTN_OK;
}

// Workspace of a multi-query step: the decode plan's, then the lengths [T][B].
size_t multi_lens_offset(const LayerPlan &pl) { return align256(pl.bytes); }
size_t multi_bytes(const LayerPlan &pl, int32_t batch, int32_t T) {
  return align256(multi_lens_offset(pl) + static_cast<size_t>(T) * batch * 4);
}

// -------------------------------------------------- fixed scratch (no alloc)
constexpr int kMaxDevices = 64;

// Process-unique id of the current CUDA context (cuCtxGetId), so that a
// context created after a reset is never mistaken for its predecessor even if
// it reuses the handle.  0 when the driver cannot say.
unsigned long long current_context_id() {
  using CtxGetCurrentFn = CUresult (*)(CUcontext *);
  using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
  static CtxGetCurrentFn get_current = []() -> CtxGetCurrentFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  static CtxGetIdFn get_id = []() -> CtxGetIdFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS ||
      ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Address of g_noalloc_scratch in the current device's context.  The first
// call in a context looks it up and enqueues a clear of the whole array on
// `stream`: the status word and the part counters must start at zero (every
// call leaves the counters at zero again); partial slots are written before
// they are read.  That first call must not be captured (the clear would only
// run at replay while later eager calls assumed it done): it returns
// GDATTN_ERR_INVALID_ARG while `stream` is capturing and records nothing.
gdattn_status noalloc_scratch(cudaStream_t stream, uint8_t **addr) {
  struct Entry {
    unsigned long long ctx_id;
    void *ptr;
  };
  static std::mutex mu;
  static Entry by_device[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDATTN_ERR_CUDA;
  unsigned long long ctx_id = current_context_id();
  if (ctx_id == 0) {
    // No current context yet: the runtime creates the device's primary
    // context (and makes it current) on its first call that needs one.
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return GDATTN_ERR_CUDA;
    ctx_id = current_context_id();
    if (ctx_id == 0) return GDATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  Entry &e = by_device[dev];
  if (e.ptr == nullptr || e.ctx_id != ctx_id) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return GDATTN_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return GDATTN_ERR_INVALID_ARG;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return GDATTN_ERR_CUDA;
    if (cudaMemsetAsync(p, 0, kNoallocScratchBytes, stream) != cudaSuccess) return GDATTN_ERR_CUDA;
    e.ptr = p;
    e.ctx_id = ctx_id;
  }
  *addr = static_cast<uint8_t *>(e.ptr);
  return GDATTN_OK;
}

}  // namespace

// ===================================================================== ABI
extern "C" {

int32_t gdattn_version(void) { return GDATTN_VERSION; }

const char *gdattn_status_string(gdattn_status s) {
  switch (s) {
    case GDATTN_OK: return "GDATTN_OK";
    case GDATTN_ERR_INVALID_ARG: return "GDATTN_ERR_INVALID_ARG";
    case GDATTN_ERR_UNSUPPORTED: return "GDATTN_ERR_UNSUPPORTED";
    case GDATTN_ERR_MISALIGNED: return "GDATTN_ERR_MISALIGNED";
    case GDATTN_ERR_WORKSPACE: return "GDATTN_ERR_WORKSPACE";
    case GDATTN_ERR_CUDA: return "GDATTN_ERR_CUDA";
    case GDATTN_ERR_DEVICE_TIMEOUT: return "GDATTN_ERR_DEVICE_TIMEOUT";
    case GDATTN_ERR_DEVICE_SEQLEN: return "GDATTN_ERR_DEVICE_SEQLEN";
  }
  return "GDATTN_UNKNOWN_STATUS";
}

size_t gdattn_workspace_size(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc) {
  LayerPlan pl;
  if (make_plan(batch, max_seqlen, desc, pl) != GDATTN_OK) return 0;
  return pl.bytes;
}

int32_t gdattn_plan_splits(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc) {
  LayerPlan pl;
  if (make_plan(batch, max_seqlen, desc, pl) != GDATTN_OK) return 0;
  return pl.grid;
}

int32_t gdattn_plan_launches(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc) {
  LayerPlan pl;
  if (make_plan(batch, max_seqlen, desc, pl) != GDATTN_OK) return 0;
  return pl.needs_combine() ? 2 : 1;
}

gdattn_status gdattn_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
  if (workspace == nullptr || workspace_bytes < kStatusBytes) return GDATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDATTN_ERR_MISALIGNED;
  return cudaMemsetAsync(workspace, 0, workspace_bytes, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? GDATTN_OK
             : GDATTN_ERR_CUDA;
}

gdattn_status gdattn_decode(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                            const gdattn_layer_desc *desc, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, void *stream) {
  // Host-only checks first: nothing below touches CUDA until they pass.
  gdattn_status st = check_decode_args(q, k_cache, v_cache, seqlens, batch, max_seqlen, desc,
                                       out, lse);
  if (st != GDATTN_OK) return st;
  if (workspace == nullptr) return GDATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDATTN_ERR_MISALIGNED;
  LayerPlan pl;
  st = make_plan(batch, max_seqlen, desc, pl);
  if (st != GDATTN_OK) return st;
  if (workspace_bytes < pl.bytes) return GDATTN_ERR_WORKSPACE;
  return enqueue_decode(pl, q, k_cache, v_cache, seqlens, batch, desc, out, lse,
                        static_cast<uint8_t *>(workspace), static_cast<cudaStream_t>(stream));
}

gdattn_status gdattn_decode_append(const void *q, const void *k_new, const void *v_new,
                                   void *k_cache, void *v_cache, const int32_t *seqlens,
                                   int32_t batch, int32_t max_seqlen,
                                   const gdattn_layer_desc *desc, void *out, float *lse,
                                   void *workspace, size_t workspace_bytes, void *stream) {
  gdattn_status st = check_decode_args(q, k_cache, v_cache, seqlens, batch, max_seqlen, desc,
                                       out, lse);
  if (st != GDATTN_OK) return st;
  if (k_new == nullptr || (desc->kv_shared == 1) != (v_new == nullptr))
    return GDATTN_ERR_INVALID_ARG;
  if (!aligned16(k_new) || (v_new && !aligned16(v_new))) return GDATTN_ERR_MISALIGNED;
  if (workspace == nullptr) return GDATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDATTN_ERR_MISALIGNED;
  LayerPlan pl;
  st = make_plan(batch, max_seqlen, desc, pl);
  if (st != GDATTN_OK) return st;
  if (workspace_bytes < pl.bytes) return GDATTN_ERR_WORKSPACE;
  return enqueue_decode(pl, q, k_cache, v_cache, seqlens, batch, desc, out, lse,
                        static_cast<uint8_t *>(workspace), static_cast<cudaStream_t>(stream),
                        k_new, v_new);
}

gdattn_status gdattn_decode_fp8(const void *q, const void *k_codes, const void *v_codes,
                                const float *k_scale, const float *v_scale,
                                const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                const gdattn_layer_desc *desc, void *out, float *lse,
                                void *workspace, size_t workspace_bytes, void *stream) {
  if (q == nullptr || k_codes == nullptr || v_codes == nullptr || k_scale == nullptr ||
      v_scale == nullptr || seqlens == nullptr || out == nullptr || desc == nullptr)
    return GDATTN_ERR_INVALID_ARG;
  gdattn_status st = check_desc(desc);
  if (st != GDATTN_OK) return st;
  if (batch <= 0 || max_seqlen <= 0) return GDATTN_ERR_INVALID_ARG;
  if (choose_path(desc) != PathKind::kTcPair) return GDATTN_ERR_UNSUPPORTED;
  if (desc->cache_batch_stride % 16 != 0) return GDATTN_ERR_MISALIGNED;  // TMA strides, bytes
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(k_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_scale) & 3u) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GDATTN_ERR_MISALIGNED;
  if (workspace == nullptr) return GDATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDATTN_ERR_MISALIGNED;
  LayerPlan pl;
  st = make_plan(batch, max_seqlen, desc, pl, true);
  if (st != GDATTN_OK) return st;
  if (workspace_bytes < pl.bytes) return GDATTN_ERR_WORKSPACE;
  return enqueue_decode_fp8(pl, q, k_codes, v_codes, k_scale, v_scale, seqlens, batch, desc, out,
                            lse, static_cast<uint8_t *>(workspace),
                            static_cast<cudaStream_t>(stream));
}

size_t gdattn_multi_workspace_size(int32_t batch, int32_t n_tokens, int32_t max_seqlen,
                                   const gdattn_layer_desc *desc) {
  if (batch <= 0 || desc == nullptr) return 0;
  if (multi_prefill(desc, n_tokens)) {
    size_t bytes = 0;
    return plan_prefill(batch, n_tokens, desc, &bytes) == GDATTN_OK ? bytes : 0;
  }
  if (n_tokens < 1 || n_tokens > kMaxMultiTokens) return 0;
  LayerPlan pl;
  if (multi_single_pass(desc, n_tokens)) {
    const gdattn_layer_desc ud = union_window_desc(desc, n_tokens);
    if (make_plan(batch, max_seqlen, &ud, pl, false, n_tokens) != GDATTN_OK) return 0;
    return pl.bytes;
  }
  if (make_plan(batch * n_tokens, max_seqlen, desc, pl) != GDATTN_OK) return 0;
  return multi_bytes(pl, batch, n_tokens);
}

gdattn_status gdattn_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *seqlens, int32_t batch, int32_t n_tokens,
                                  int32_t max_seqlen, const gdattn_layer_desc *desc, void *out,
                                  float *lse, void *workspace, size_t workspace_bytes,
                                  void *stream_) {
  gdattn_status st = check_decode_args(q, k_cache, v_cache, seqlens, batch, max_seqlen, desc,
                                       out, lse);
  if (st != GDATTN_OK) return st;
  const int32_t max_tokens = prefill_geometry(desc) ? kMaxPrefillTokens : kMaxMultiTokens;
  if (n_tokens < 1 || n_tokens > max_tokens || n_tokens > max_seqlen)
    return GDATTN_ERR_INVALID_ARG;
  // A ring holds positions [L - C, L): the first token's window must still be in it.
  if (desc->window > 0 && desc->cache_capacity < max_seqlen &&
      static_cast<int64_t>(desc->cache_capacity) <
          static_cast<int64_t>(desc->window) + n_tokens - 1)
    return GDATTN_ERR_INVALID_ARG;
  if (workspace == nullptr) return GDATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return GDATTN_ERR_MISALIGNED;
  if (multi_prefill(desc, n_tokens)) {
    size_t bytes = 0;
    st = plan_prefill(batch, n_tokens, desc, &bytes);
    if (st != GDATTN_OK) return st;
    if (workspace_bytes < bytes) return GDATTN_ERR_WORKSPACE;
    return enqueue_prefill(q, k_cache, v_cache, seqlens, batch, n_tokens, desc, out, lse,
                           static_cast<uint8_t *>(workspace), static_cast<cudaStream_t>(stream_));
  }
  if (multi_single_pass(desc, n_tokens)) {
    const gdattn_layer_desc ud = union_window_desc(desc, n_tokens);
    LayerPlan pl;
    st = make_plan(batch, max_seqlen, &ud, pl, false, n_tokens);
    if (st != GDATTN_OK) return st;
    if (workspace_bytes < pl.bytes) return GDATTN_ERR_WORKSPACE;
    return enqueue_decode_multi_pass(pl, q, k_cache, v_cache, seqlens, batch, n_tokens, desc, out,
                                     lse, static_cast<uint8_t *>(workspace),
                                     static_cast<cudaStream_t>(stream_));
  }
  // One decode over T x B query sequences, token-major (q, out, lse and the
  // lengths are [T][B] ...): query sequence t * B + b reads cache sequence b.
  const int32_t total = n_tokens * batch;
  LayerPlan pl;
  st = make_plan(total, max_seqlen, desc, pl);
  if (st != GDATTN_OK) return st;
  if (workspace_bytes < multi_bytes(pl, batch, n_tokens)) return GDATTN_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int32_t *lens = reinterpret_cast<int32_t *>(ws + multi_lens_offset(pl));
  multi_lengths_kernel<<<(total + 255) / 256, 256, 0, stream>>>(seqlens, batch, n_tokens, lens);
  if (cudaGetLastError() != cudaSuccess) return GDATTN_ERR_CUDA;
  return enqueue_decode(pl, q, k_cache, v_cache, lens, total, desc, out, lse, ws, stream, nullptr,
                        nullptr, false, batch);
}

gdattn_status gdattn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                    const gdattn_layer_desc *desc, void *out, float *lse,
                                    void *stream_) {
  gdattn_status st = check_decode_args(q, k_cache, v_cache, seqlens, batch, max_seqlen, desc,
                                       out, lse);
  if (st != GDATTN_OK) return st;
  LayerPlan pl;
  st = make_plan(batch, max_seqlen, desc, pl);
  if (st != GDATTN_OK) return st;
  if (pl.bytes > kNoallocScratchBytes) return GDATTN_ERR_WORKSPACE;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  uint8_t *scratch = nullptr;
  st = noalloc_scratch(stream, &scratch);
  if (st != GDATTN_OK) return st;
  return enqueue_decode(pl, q, k_cache, v_cache, seqlens, batch, desc, out, lse, scratch, stream);
}

gdattn_status gdattn_combine(const float *o_partial, const float *lse_partial, int32_t batch,
                             int32_t n_q_heads, int32_t n_splits, int32_t head_dim, void *out,
                             float *lse, void *stream) {
  if (o_partial == nullptr || lse_partial == nullptr || out == nullptr)
    return GDATTN_ERR_INVALID_ARG;
  if (batch <= 0 || n_q_heads <= 0 || n_splits <= 0 || head_dim <= 0 || head_dim % 4 != 0 ||
      head_dim > 1024 || n_splits > 8192 || batch > 65535 || n_q_heads > 65535)
    return GDATTN_ERR_INVALID_ARG;
  if (!aligned16(o_partial) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(lse_partial) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return GDATTN_ERR_MISALIGNED;
  if ((head_dim % 8) != 0 && (reinterpret_cast<uintptr_t>(out) & 7u)) return GDATTN_ERR_MISALIGNED;
  CombineParams cp = {};
  cp.parts_o = o_partial;
  cp.parts_lse = lse_partial;
  cp.out = static_cast<uint16_t *>(out);
  cp.lse = lse;
  cp.n_q_heads = n_q_heads;
  cp.head_dim = head_dim;
  cp.heads_per_unit = 0;
  cp.n_splits = n_splits;
  cp.split_k = 0;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = launch_config(dim3(batch, n_q_heads), combine_threads(head_dim), 0,
                                         static_cast<cudaStream_t>(stream), attr);
  return cudaLaunchKernelEx(&cfg, combine_kernel<false>, cp) == cudaSuccess ? GDATTN_OK
                                                                             : GDATTN_ERR_CUDA;
}

gdattn_status gdattn_read_probe(const void *src, size_t bytes, int32_t mode, uint32_t *sink,
                                void *stream_) {
  if (src == nullptr || sink == nullptr || bytes == 0 || (bytes & 15u) != 0 ||
      (mode != 0 && mode != 1))
    return GDATTN_ERR_INVALID_ARG;
  if (!aligned16(src) || (reinterpret_cast<uintptr_t>(sink) & 3u)) return GDATTN_ERR_MISALIGNED;
  const int nsm = sm_count();
  if (nsm <= 0) return GDATTN_ERR_CUDA;
  ReadProbeParams rp;
  rp.src = static_cast<const uint8_t *>(src);
  rp.bytes = static_cast<int64_t>(bytes);
  rp.sink = sink;
  rp.status = sink + 1;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (mode == 0) {
    const int per_sm = cached_blocks_per_sm(reinterpret_cast<const void *>(read_probe_ldg_kernel),
                                            kReadProbeThreads, 0, query_probe);
    if (per_sm <= 0) return GDATTN_ERR_CUDA;
    read_probe_ldg_kernel<<<nsm * per_sm, kReadProbeThreads, 0, stream>>>(rp);
  } else {
    using Cfg = ReadProbeBulkConfig;
    if (cached_blocks_per_sm(reinterpret_cast<const void *>(read_probe_bulk_kernel), Cfg::kThreads,
                             Cfg::SMEM, query_probe) <= 0)
      return GDATTN_ERR_CUDA;
    read_probe_bulk_kernel<<<nsm, Cfg::kThreads, Cfg::SMEM, stream>>>(rp);
  }
  return cudaGetLastError() == cudaSuccess ? GDATTN_OK : GDATTN_ERR_CUDA;
}

gdattn_status gdattn_check_device_status(void *workspace, void *stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (workspace == nullptr) {  // the fixed scratch of gdattn_decode_noalloc
    uint8_t *scratch = nullptr;
    const gdattn_status st = noalloc_scratch(stream, &scratch);
    if (st != GDATTN_OK) return st;
    workspace = scratch;
  }
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, stream) !=
          cudaSuccess ||
      cudaMemsetAsync(workspace, 0, sizeof(word), stream) != cudaSuccess ||
      cudaStreamSynchronize(stream) != cudaSuccess)
    return GDATTN_ERR_CUDA;
  if (word & kStatusTimeout) return GDATTN_ERR_DEVICE_TIMEOUT;
  if (word & kStatusSeqlen) return GDATTN_ERR_DEVICE_SEQLEN;
  return GDATTN_OK;
}

}  // extern "C"
