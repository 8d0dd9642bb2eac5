// Read-only HBM streaming probes: the practical ceiling a decode kernel's KV
// stream can reach on this GPU, measured with the same kinds of loads.
//
//  - read_probe_ldg_kernel: every thread streams 16-byte vectors with
//    non-coherent loads that do not allocate in L1 and are marked evict-first in
//    L2, eight loads in flight per thread, grid-stride over the buffer.
//  - read_probe_bulk_kernel: one CTA per SM; one lane issues 32 KiB bulk copies
//    (cp.async.bulk, no multicast) into a six-stage shared-memory ring, the way
//    the decode kernels feed their tensor cores; one warp releases the stages.
//
// Both XOR what they read into one word per CTA and fold it into *sink, so the
// loads cannot be dropped.  Waits are bounded like every other wait here.
#pragma once

#include <cstdint>

#include "partition.cuh"
#include "ptx.cuh"

namespace gdattn {

struct ReadProbeParams {
  const uint8_t *src;  // 16-byte aligned
  int64_t bytes;       // multiple of 16
  uint32_t *sink;
  uint32_t *status;    // bounded-wait expiry (bulk mode), may be null
};

__device__ __forceinline__ uint4 ldg_stream16(const void *p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

constexpr int kReadProbeThreads = 512;

__global__ void __launch_bounds__(kReadProbeThreads) read_probe_ldg_kernel(const ReadProbeParams p) {
  const uint64_t pol = l2_evict_first_policy();
  const int64_t n16 = p.bytes >> 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const uint4 *src = reinterpret_cast<const uint4 *>(p.src);
  uint32_t acc = 0;
  int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  constexpr int U = 8;
  for (; i + (U - 1) * stride < n16; i += U * stride) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) v[u] = ldg_stream16(src + i + u * stride, pol);
#pragma unroll
    for (int u = 0; u < U; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  for (; i < n16; i += stride) {
    const uint4 v = ldg_stream16(src + i, pol);
    acc ^= v.x ^ v.y ^ v.z ^ v.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(p.sink, acc);
}

struct ReadProbeBulkConfig {
  static constexpr int CHUNK = 32 * 1024;  // bytes per bulk copy and per stage
  static constexpr int NST = 6;
  static constexpr int SMEM = NST * CHUNK + 256 + 1024;
  static constexpr int kThreads = 64;      // warp 0 copies, warp 1 releases stages
};

__global__ void __launch_bounds__(ReadProbeBulkConfig::kThreads, 1)
    read_probe_bulk_kernel(const ReadProbeParams p) {
  using Cfg = ReadProbeBulkConfig;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + Cfg::NST * Cfg::CHUNK);
  uint64_t *empty = full + Cfg::NST;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + Cfg::NST);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // This CTA's contiguous share of the buffer, in whole chunks (the last CTA
  // also takes the remainder, copied as one shorter chunk).
  const int64_t nchunks = (p.bytes + Cfg::CHUNK - 1) / Cfg::CHUNK;
  const int64_t per = (nchunks + gridDim.x - 1) / gridDim.x;
  const int64_t c0 = imin64(nchunks, static_cast<int64_t>(blockIdx.x) * per);
  const int64_t c1 = imin64(nchunks, c0 + per);
  const int n = static_cast<int>(c1 - c0);
  uint32_t dummy = 0;
  uint32_t *status = p.status != nullptr ? p.status : &dummy;
  if (warp == 0) {
    const uint64_t pol = l2_evict_first_policy();
    bool ok = true;
    int issued = 0;
    for (int f = 0; f < n && ok; ++f) {
      const int st = f % Cfg::NST;
      if (f >= Cfg::NST)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&empty[st], ((f / Cfg::NST) - 1) & 1, abort_flag, status));
      if (!ok) break;
      const int64_t off = (c0 + f) * Cfg::CHUNK;
      const int64_t rest = p.bytes - off;
      const uint32_t len = static_cast<uint32_t>(rest < Cfg::CHUNK ? rest : Cfg::CHUNK);
      if (elect_one()) {
        mbar_arrive_expect_tx(&full[st], len);
        bulk_g2s(sm + st * Cfg::CHUNK, p.src + off, len, &full[st], pol);
      }
      __syncwarp();
      ++issued;
    }
    // Drain: never leave with copies in flight into shared memory.
    volatile int no_abort = 0;
    for (int f = issued > Cfg::NST ? issued - Cfg::NST : 0; f < issued; ++f)
      mbar_wait(&full[f % Cfg::NST], (f / Cfg::NST) & 1, &no_abort, status);
  } else {
    uint32_t acc = 0;
    for (int f = 0; f < n; ++f) {
      const int st = f % Cfg::NST;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&full[st], (f / Cfg::NST) & 1, abort_flag, status)))
        break;
      acc ^= reinterpret_cast<const uint32_t *>(sm + st * Cfg::CHUNK)[lane];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) atomicXor(p.sink, acc);
  }
  __syncthreads();
}

}  // namespace gdattn
