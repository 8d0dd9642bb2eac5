/*
 * libgdattn -- single-token (decode) attention over a per-layer KV cache for
 * Gemma-4-style hybrid stacks, split along the KV sequence, on NVIDIA B200
 * (sm_100a).
 *
 * What one call computes (one layer, one decode step, every sequence b of the
 * batch and every query head h):
 *
 *   G    = n_q_heads / n_kv_heads; query head h reads KV head kv = h / G
 *   L    = seqlens[b], the context length with the current token's K/V already
 *          in the cache
 *   positions attended: [max(0, L - window), L) when window > 0, else [0, L)
 *   slot(j) = j mod cache_capacity          (ring buffer for sliding layers)
 *   x_j  = scale * <q[b,h,:], K[b, slot(j), kv, :]>
 *   s_j  = softcap * tanh(x_j / softcap)    when softcap > 0, else x_j
 *   lse[b,h] = log sum_j exp(s_j)           (natural log)
 *   out[b,h,:] = sum_j exp(s_j - lse[b,h]) * V'[b, slot(j), kv, :],
 *                V' = K when kv_shared, else V
 *
 * Sources: sliding layers read exactly the last w positions from a rotating
 * cache and full layers read the whole context ("Gemma 4 12B" record, KV
 * GEOMETRY and serviceability join, item 6); sliding layers use head_dim 256
 * with 8 KV heads, full layers a larger head_dim (512) with one KV head and key
 * == value ("Gemma4-26B-A4B ... NO-GO", section 3 Break 4; "Gemma 4 12B" KV
 * GEOMETRY, attention_k_eq_v); attention soft-capping and K = V global attention
 * ("Gemma support" PR, summary); split decode attention for head sizes 256/512
 * ("Gemma support" PR, Performance); the split count must match the GPU so
 * that single-query global layers keep every SM busy ("Gemma 4 12B", item 4).
 *
 * Conventions for every entry point:
 *  - All tensors are caller-owned.  The library allocates no device or host
 *    memory and keeps no state between calls, and calls are thread-safe, with
 *    one exception: gdattn_decode_noalloc keeps its scratch in one array per
 *    device context inside the library, shared by all its calls (see there).
 *  - Device pointers must be 16-byte aligned and rows are contiguous along the
 *    head dimension.  bf16 means IEEE bfloat16, stored as 16-bit words.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously; no call synchronises except
 *    gdattn_check_device_status.  Decode and combine only enqueue kernels, so they
 *    can be captured into a CUDA graph.
 *  - Kernels are launched with programmatic dependent launch: gdattn_decode may
 *    start while the preceding kernel on the stream is still draining (once that
 *    kernel has signalled griddepcontrol.launch_dependents, or exited).  In that
 *    window it reads only seqlens and the cache rows of positions below each
 *    sequence's newest one (L_b - 1), i.e. rows written by earlier decode steps.
 *    q, the newest cache row, out, lse and the workspace are accessed only after
 *    the preceding kernel has completed.  A preceding kernel that triggers its
 *    dependents early must therefore not write seqlens or older cache rows after
 *    its trigger; kernels that never trigger early (the default) are unaffected.
 *  - Arguments are checked on the host before anything is enqueued; a failed
 *    check returns its status and launches nothing.  A launch failure returns
 *    GDATTN_ERR_CUDA.  Problems only the device can see (a context length that
 *    needs more slots than the cache has, a pipeline wait that ran out) are
 *    latched in the workspace status word and read by
 *    gdattn_check_device_status.
 */
#ifndef GDATTN_H_
#define GDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDATTN_VERSION 100

typedef enum gdattn_status {
  GDATTN_OK = 0,
  GDATTN_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, Hq % Hkv != 0, ... */
  GDATTN_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim or GQA group size */
  GDATTN_ERR_MISALIGNED = 3,    /* a device pointer or stride is not 16-byte aligned */
  GDATTN_ERR_WORKSPACE = 4,     /* workspace missing or smaller than gdattn_workspace_size */
  GDATTN_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
  GDATTN_ERR_DEVICE_TIMEOUT = 6,/* device: a bounded pipeline wait expired (result invalid) */
  GDATTN_ERR_DEVICE_SEQLEN = 7  /* device: seqlens[b] < 1, or the attended range needs more
                                   slots than cache_capacity (range clamped, result invalid) */
} gdattn_status;

/* Geometry and numerics of one attention layer. */
typedef struct gdattn_layer_desc {
  int32_t n_q_heads;      /* Hq > 0 */
  int32_t n_kv_heads;     /* Hkv > 0, Hq % Hkv == 0 */
  int32_t head_dim;       /* D: 256 or 512 */
  int32_t window;         /* 0: attend [0, L); w > 0: attend the last w positions [L-w, L) */
  float softcap;          /* 0: off; > 0: s = softcap * tanh(s / softcap), after the scale */
  float scale;            /* multiplies q.k (1/sqrt(D) for Gemma-4 geometries) */
  int32_t kv_shared;      /* 1: K serves as V (attention_k_eq_v); v_cache must be NULL */
  int32_t cache_capacity; /* C: slots per sequence; position j lives in slot j mod C */
  int64_t cache_batch_stride; /* elements from sequence b to b+1 in K (and V); 0 = C*Hkv*D;
                                 otherwise >= C*Hkv*D and a multiple of 8 */
  int32_t split_ctas;     /* 0: the planner picks how many CTAs share the KV range; > 0
                             forces that many (tests and tuning) */
  int32_t flags;          /* GDATTN_FLAG_* bits; other bits must be 0 */
} gdattn_layer_desc;

/*
 * The caller expects every sequence of a call to attend about the same number
 * of positions (uniform context lengths, or all of them past the window).  The
 * tcgen05 kernels then cut each (sequence, KV head) unit into the same number k
 * of whole-tile parts, one CTA each (k chosen so all parts run at once), so no
 * CTA straddles two units; the parts are merged as split-KV partials.  With
 * uneven lengths that split stays correct but loses balance.  Without the flag
 * (or with split_ctas > 0) the KV ranges of all units are laid end to end and
 * cut into equal chunks.
 */
#define GDATTN_FLAG_EVEN_UNITS 1

/*
 * Test hook for the device-side failure path, not for production calls: every
 * CTA of the decode kernel leaves its first KV tile unloaded, so the pipeline
 * wait for it runs out after the bounded wait limit (about 2 s at the maximum
 * SM clock).  The kernel then drains its copies and tensor-core work, frees
 * tensor memory and returns; the call latches GDATTN_ERR_DEVICE_TIMEOUT in the
 * workspace status word and its out and lse are invalid.  After any device
 * timeout, re-initialise the workspace (gdattn_workspace_init) before reusing
 * it: split merges may have left part counters set.
 */
#define GDATTN_FLAG_TEST_WITHHOLD_KV 2

/*
 * Bytes of device workspace gdattn_decode needs for this layer geometry and
 * batch on the current CUDA device.  max_seqlen is the host's upper bound on
 * seqlens[]; it only steers the split count.  Returns 0 on invalid arguments.
 *
 * Every workspace starts with the same 128 KiB + 256 B header: the status
 * word, then a part counter and a merge epoch for each (sequence, KV head)
 * unit index below 16384; the partial results of split ranges follow.  Since
 * the header never moves, calls with different geometries, batches or splits
 * may take turns on one workspace (ordered on one stream) if it holds the
 * largest of their sizes.  A call with batch * n_kv_heads > 16384 (times
 * n_tokens for gdattn_decode_multi) returns GDATTN_ERR_UNSUPPORTED.
 */
size_t gdattn_workspace_size(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc);

/*
 * Number of CTAs the planner splits this layer's KV range across (the value
 * gdattn_decode uses for the same arguments on the current device).  Returns 0
 * on invalid arguments.
 */
int32_t gdattn_plan_splits(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc);

/*
 * Kernel launches gdattn_decode makes for these arguments: the decode kernel,
 * plus the LSE-combine kernel when the KV range is split over more than one
 * CTA and the decode kernel does not merge split units itself (the tcgen05
 * pair kernel does).  Returns 0 on invalid arguments.
 */
int32_t gdattn_plan_launches(int32_t batch, int32_t max_seqlen, const gdattn_layer_desc *desc);

/*
 * Zero the workspace.  Its status word and per-unit part counters must start
 * at zero: call this once after allocating a workspace (or zero it yourself).
 * Every decode call leaves the counters at zero again; the status word latches
 * device-side errors until gdattn_check_device_status reads and clears it.
 */
gdattn_status gdattn_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode attention for one layer (the definition at the top of this file).
 *
 *  q        bf16 [batch, Hq, D], device, read only
 *  k_cache  bf16, device, read only; sequence b at k_cache + b*cache_batch_stride
 *           elements, laid out [C][Hkv][D] (token-major)
 *  v_cache  bf16, same layout as k_cache, or NULL when desc->kv_shared == 1
 *  seqlens  int32 [batch], device: L_b >= 1 and min(L_b, window or L_b) <= C
 *  batch    > 0;  max_seqlen: host upper bound of seqlens[] (> 0)
 *  out      bf16 [batch, Hq, D], device, written
 *  lse      fp32 [batch, Hq], device, written (natural log), or NULL
 *  workspace / workspace_bytes: device scratch of at least gdattn_workspace_size
 *           bytes, zeroed once by gdattn_workspace_init.  Calls that share a
 *           workspace must be ordered on one stream; they may differ in
 *           geometry and batch (see gdattn_workspace_size).
 *
 * Supported geometries (G = Hq / Hkv), by the kernel that runs them:
 *  - G == 2, D == 256, separate V, any Hkv: tcgen05 pair kernel;
 *  - G == 16, D == 512, kv_shared, any Hkv: tcgen05 16-head kernel;
 *  - otherwise D in {256, 512}, G in {1, 2, 4}, Hkv in {1, 2, 4, 8}: CUDA-core kernel.
 * Other geometries return GDATTN_ERR_UNSUPPORTED.
 */
gdattn_status gdattn_decode(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                            const gdattn_layer_desc *desc, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * The log-sum-exp combine of split decode attention ("Gemma support" PR,
 * Performance: split decode attention for head sizes 256/512; "Gemma 4 12B",
 * item 4: single-query global layers split the KV range into num_splits parts
 * whose partial results are merged).
 *
 * Merge n_splits partial results per (sequence, head), each normalised over its
 * own part of the position range:
 *   lse = log sum_s exp(lse_s),  out = sum_s exp(lse_s - lse) * o_s.
 * A part with lse_s = -INFINITY (empty) contributes nothing; if every part is
 * empty the result is lse = -INFINITY and out = 0.
 *
 *  o_partial    fp32 [batch, Hq, n_splits, D], device
 *  lse_partial  fp32 [batch, Hq, n_splits], device (natural log)
 *  out          bf16 [batch, Hq, D], device;  lse: fp32 [batch, Hq] or NULL
 *  head_dim     any multiple of 4 up to 1024; n_splits >= 1
 */
gdattn_status gdattn_combine(const float *o_partial, const float *lse_partial, int32_t batch,
                             int32_t n_q_heads, int32_t n_splits, int32_t head_dim, void *out,
                             float *lse, void *stream);

/*
 * gdattn_decode with the current token's append fused in: for every sequence b
 * the rows k_new[b] (and v_new[b]) are written into cache slot
 * (seqlens[b] - 1) mod C, then attention runs over the updated cache.  The
 * result equals writing those rows first and calling gdattn_decode; the
 * write is done by the CTA that loads that slot, just before it loads it, so
 * it costs no launch and no extra pass.
 *
 *  k_new     bf16 [batch, Hkv, D], device, read only (read after the preceding
 *            kernel on the stream has completed)
 *  v_new     bf16 [batch, Hkv, D], or NULL when desc->kv_shared == 1
 *  k_cache, v_cache: as in gdattn_decode, but written at those slots; nothing
 *            else in them is written, and the slot of a sequence whose length is
 *            rejected on the device is left untouched
 *  other arguments, checks and errors as gdattn_decode
 */
gdattn_status gdattn_decode_append(const void *q, const void *k_new, const void *v_new,
                                   void *k_cache, void *v_cache, const int32_t *seqlens,
                                   int32_t batch, int32_t max_seqlen,
                                   const gdattn_layer_desc *desc, void *out, float *lse,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * gdattn_decode over an fp8 cache: every cache row (one token of one KV head)
 * holds D codes in OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; no infinities, S.1111.111 is NaN) and one fp32 scale, and its
 * values are code_d * scale.  The quantized rotating cache is mlx-lm's
 * RotatingQuantizedKVCache idea ("Gemma 4 12B", serviceability join, item 6);
 * BF16 queries over an FP8 KV cache at a sliding-window boundary are what
 * FlashInfer's trtllm kernel got wrong on B200 (same record, item 2).  The
 * computation is the definition at the top of this file with those values for
 * K and V; q, out and lse stay bf16 / fp32.
 *
 *  k_codes  e4m3 bytes, device, read only; sequence b at k_codes +
 *           b*cache_batch_stride bytes, laid out [C][Hkv][D] (token-major)
 *  v_codes  e4m3 bytes, same layout
 *  k_scale  fp32 [batch][Hkv][C], device, read only: the scale of K row
 *           (b, kv, slot), contiguous over the slots (4-byte aligned)
 *  v_scale  fp32 [batch][Hkv][C], the V rows' scales
 *  other arguments as gdattn_decode.  cache_batch_stride counts bytes here and
 *  must be a multiple of 16 (0 = C*Hkv*D).  The workspace is sized by
 *  gdattn_workspace_size for the same desc.
 *
 * Supported geometry: G == 2, D == 256, separate V (the sliding layers), any
 * Hkv; others return GDATTN_ERR_UNSUPPORTED.  Scales must be finite; a zero
 * scale makes its row zero.  The kernel multiplies fp8 codes on the tensor
 * cores against q and the softmax weights each split into three e4m3 pieces;
 * the q split is exact for bf16 elements down to 2^-6 of the head's largest,
 * and the weight split's error is below 2^-13 relative (2^-17 absolute for the
 * smallest scaled weights); against the float64 definition of the dequantised
 * attention the output meets the bf16 entry points' gates (|dout| <= 8e-3, with a
 * one-bf16-ulp floor for outputs above 1, and |dlse| <= 1e-3).
 */
gdattn_status gdattn_decode_fp8(const void *q, const void *k_codes, const void *v_codes,
                                const float *k_scale, const float *v_scale,
                                const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                const gdattn_layer_desc *desc, void *out, float *lse,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Multi-query decode: T query tokens per sequence, the last T positions of its
 * context, each attending causally: the verify step of speculative decoding,
 * which "Gemma 4 12B" (serviceability join, item 2) runs with 7 draft tokens on
 * the sliding-window stack.  Query token t of sequence b sits at position
 * p = L_b - T + t and attends
 * [max(0, p + 1 - window), p + 1) (window 0: [0, p + 1)); the cache already
 * holds the rows of all T tokens.  Each token's result is exactly what
 * gdattn_decode gives for context length L_b - (T - 1 - t).
 *
 *  q         bf16 [T, batch, Hq, D] (token-major), device, read only
 *  out       bf16 [T, batch, Hq, D];  lse: fp32 [T, batch, Hq] or NULL
 *  n_tokens  T: 1 <= T <= 64, or up to 2^20 on the pair geometry and on the
 *            global geometry with K = V (a prompt chunk);  seqlens: L_b >= T,
 *            the length with all T tokens
 *  workspace at least gdattn_multi_workspace_size bytes (zeroed once by
 *            gdattn_workspace_init)
 *  other arguments, geometries and device-side errors as gdattn_decode.
 *
 * A ring cache holds positions [L_b - C, L_b), so with a window the first token
 * needs C >= window + T - 1 unless the cache never wraps (C >= max_seqlen);
 * otherwise GDATTN_ERR_INVALID_ARG.
 *
 * On the pair geometry (two query heads per KV head, head_dim 256, separate V)
 * with T <= 8 the step is one pass over the cache: a unit's 2T query rows (token,
 * head) share every K and V tile of the union of their windows, the last
 * min(L_b, window + T - 1) positions, and each score is masked to its own
 * token's range; split units are merged inside the kernel.  With T > 8 on the
 * same geometry the step is flash prefill ("Gemma support" pull request,
 * Performance: flash prefill for head_dim 256): one CTA per 64 query tokens of a
 * (sequence, KV head), 128 query rows per tensor-core tile, streaming that
 * block's KV range once; its workspace is the fixed header alone.  The global
 * geometry with K = V (8 or 16 query heads per KV head, head_dim 512) runs T > 8
 * as flash prefill too, in blocks of 64 query rows (64 / G tokens), each on two
 * CTAs that split the output's head dimension.  Otherwise
 * one small kernel writes the T per-token lengths into the workspace, then one
 * decode launch runs over T x batch query sequences (token-major) in which query
 * sequence t * batch + b reads cache sequence b; the T tokens of a sequence then
 * read the same cache rows from different CTAs at about the same time, so much
 * of the repetition is served from L2 rather than HBM.  A sequence with
 * L_b < T is a device-side error (GDATTN_ERR_DEVICE_SEQLEN); its tokens below
 * position 0 get a zero output and LSE -inf.
 */
size_t gdattn_multi_workspace_size(int32_t batch, int32_t n_tokens, int32_t max_seqlen,
                                   const gdattn_layer_desc *desc);

gdattn_status gdattn_decode_multi(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *seqlens, int32_t batch, int32_t n_tokens,
                                  int32_t max_seqlen, const gdattn_layer_desc *desc, void *out,
                                  float *lse, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * gdattn_decode without a caller workspace.  A library addition with no
 * counterpart in the pages; it computes exactly what gdattn_decode computes.
 *
 * Same arguments (workspace and workspace_bytes dropped), host checks, kernels
 * and results as gdattn_decode: for the same inputs on the same device both
 * produce bit-identical out and lse.  The split-KV scratch (status word,
 * part counters, partial LSE, partial O) is one fixed array inside the library,
 * GDATTN_NOALLOC_SCRATCH_BYTES per device context, reserved when the library's
 * device code is loaded, so no call allocates device or host memory.
 *  - The first call in each device context looks the array up
 *    (cudaGetSymbolAddress) and enqueues a clear of the whole array on
 *    `stream`; later calls only enqueue kernels.  That first call must not be
 *    captured into a CUDA graph: made while `stream` is capturing it returns
 *    GDATTN_ERR_INVALID_ARG and enqueues nothing.  A context created after a
 *    reset (cudaDeviceReset) counts as new: its first call looks up and clears
 *    the array again.
 *  - The array has the workspace layout of gdattn_workspace_size (fixed
 *    header, then partials), so calls with different geometries and batches
 *    may follow one another.
 *  - A layer whose gdattn_workspace_size exceeds GDATTN_NOALLOC_SCRATCH_BYTES
 *    returns GDATTN_ERR_WORKSPACE and enqueues nothing; use gdattn_decode.
 *  - One array per device: calls that can overlap in time on one device (on
 *    streams with no ordering between them, from host threads racing on one
 *    stream, or in graph replays that can run concurrently) race on it, and
 *    their results are undefined.  Calls ordered on one stream are safe,
 *    including the early start of programmatic dependent launch.
 *  - Device-side errors latch in the array's status word; read and clear them
 *    with gdattn_check_device_status(NULL, stream).
 */
#define GDATTN_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

gdattn_status gdattn_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                    const int32_t *seqlens, int32_t batch, int32_t max_seqlen,
                                    const gdattn_layer_desc *desc, void *out, float *lse,
                                    void *stream);

/*
 * Synchronise `stream`, read and clear the status word of `workspace` (NULL:
 * the fixed scratch of gdattn_decode_noalloc on the current device), and
 * return the first device-side error latched since the last check (GDATTN_OK
 * if none).
 */
gdattn_status gdattn_check_device_status(void *workspace, void *stream);

/*
 * Read-only streaming probe: the practical ceiling of HBM read bandwidth for
 * the loads the decode kernels use, to set their roofline fractions against.
 * A measurement utility with no counterpart in the pages.
 *
 *  src    device buffer of `bytes` bytes (16-byte aligned, bytes a multiple of
 *         16 and > 0), read once
 *  mode   0: every thread streams 16-byte vector loads (non-coherent, no L1
 *         allocation, evict-first in L2), grid of resident CTAs on all SMs;
 *         1: one CTA per SM copies 32 KiB chunks of its contiguous share into a
 *         six-stage shared-memory ring with bulk copies (cp.async.bulk)
 *  sink   uint32_t[2], device: the XOR of the data read is folded into sink[0]
 *         (so the loads cannot be removed); sink[1] latches the device status
 *         bits (a bounded wait that expired in mode 1)
 * One kernel launch on `stream`; time it with events around the call.
 */
gdattn_status gdattn_read_probe(const void *src, size_t bytes, int32_t mode, uint32_t *sink,
                                void *stream);

/* Static, human-readable name of a status code. */
const char *gdattn_status_string(gdattn_status status);

/* GDATTN_VERSION of the built library. */
int32_t gdattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDATTN_H_ */
