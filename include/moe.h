/*
 * moe.h -- C ABI of libmoe: one 4-bit-weight mixture-of-experts layer on an NVIDIA B200 (sm_100a).
 *
 * What one forward call computes (for every token t of x[T, H]):
 *   logits[e] = x_t . router[e] (+ router_bias[e])                        e = 0..E-1, fp32
 *   S_t       = the top_k experts by logit, descending (equal logits: lower index first)
 *   g_j       = softmax over all E logits, restricted to S_t and renormalised (sums to 1)
 *   s_t       = sigmoid(x_t . shared_gate)                   (only when has_shared != 0)
 *   FFN_e(x)  = W_down,e ( silu(W_gate,e x) * (W_up,e x) ),   silu(z) = z / (1 + exp(-z))
 *   out_t     = sum_j g_j FFN_{S_t[j]}(x_t) + s_t FFN_shared(x_t),   rounded to bf16
 * Each weight is  W[r][c] = q[r][c] * s[r][c/64] + b[r][c/64]  with a 4-bit code q and a per-
 * (row, 64-column group) bf16 scale s and bias b ("asymmetric int4, group 64").
 *
 * Where this comes from.  "Perplexity Open-Sources Lily, a Qwen-Specific Mac Engine That Beats
 * MLX-LM in Its Test", section "A runtime shaped around one model": each token is routed to eight
 * of 256 experts plus a shared expert, and expert loads are uneven.  Same page, section "The
 * optimizations follow the workload": during prefill the 4-bit weights are rebuilt inside the
 * grouped matrix multiplication instead of being expanded into a full weight array, and expert
 * routing stays on the GPU with no CPU synchronisation.  "A Rust + Metal Inference Engine for
 * Qwen3.6-35B-A3B on Apple Silicon" (body) and the "perplexity-lily-engine" note (body, limits
 * paragraph): decode is bound by weight bytes (the sparse GEMVs run near the memory wall).  The
 * gating formula, the sigmoid shared gate, SwiGLU and the int4/g64/bf16 format are this
 * library's layer definition; the pages do not spell them out.
 *
 * Conventions for every entry point below.
 *  - All tensor pointers are DEVICE pointers owned by the caller (except moe_forward_host and
 *    moe_forward_host_async, which take host pointers).  The library never frees or retains
 *    caller memory beyond the call, except that moe_create copies (repacks) the weights into
 *    memory the handle owns, so the caller may free its weight buffers as soon as moe_create has
 *    returned and its stream has been synchronised.
 *  - "stream" is a cudaStream_t passed as void* (NULL = the legacy default stream).  Calls are
 *    stream-ordered and asynchronous: they return after enqueueing work, with no host
 *    synchronisation, no device-to-host copy and no allocation (moe_create and moe_forward_host
 *    excepted; moe_forward_host_async enqueues its device-to-host copy without waiting for it).
 *    Outputs are overwritten, never accumulated into.
 *  - Return value: MOE_OK or one of the MOE_ERR_* codes.  No exception crosses the ABI.  An error
 *    found before launch returns its code and launches nothing; a text message is then available
 *    from moe_last_error() on the calling thread.  Errors found on the device (a timed-out wait,
 *    an out-of-range index, a value outside the fp16 operand range) are recorded in a status word
 *    and reported by the next moe_status() call.
 *  - One stream at a time per handle: calls on one handle must not overlap on the device (they
 *    share the handle's workspace).  Different handles are independent.
 *  - Layouts are row-major and densely packed.  bf16 and fp16 values are passed as uint16 bit
 *    patterns.  Pointers must be 16-byte aligned.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ----------------------------------------------------------------------------- */
#define MOE_OK                      0
#define MOE_ERR_INVALID_ARG         1  /* null/misaligned pointer, unsupported shape, bad flag */
#define MOE_ERR_UNSUPPORTED_DEVICE  2  /* device is not sm_100 (B200 class) */
#define MOE_ERR_TOO_LARGE           3  /* T > max_tokens */
#define MOE_ERR_CUDA                4  /* a CUDA runtime call failed (message in moe_last_error) */
#define MOE_ERR_DEVICE_TIMEOUT      5  /* a bounded device-side wait ran out (kernel returned early) */
#define MOE_ERR_DEVICE_BOUNDS       6  /* a device-side index check failed (access skipped) */
#define MOE_ERR_RANGE               7  /* a value did not fit the fp16 tensor-core operand range */

/* ---- configuration flags ---------------------------------------------------------------------- */
#define MOE_FLAG_ROUTER_SIMT     0x1u  /* compute the router on CUDA cores for every T */
#define MOE_FLAG_DECODE_UNFUSED  0x2u  /* decode calls: use the multi-kernel GEMV chain instead
                                          of the fused decode kernel (one launch per 8 tokens) */
#define MOE_FLAG_POISON_WORKSPACE 0x4u /* test aid: the handle's workspace starts filled with 0xFF
                                          bytes (NaN floats, -1 indices) instead of zeros, except
                                          the words the kernels count on starting at zero, so a
                                          read of workspace no kernel wrote shows up as a wrong or
                                          non-finite result (results are otherwise unchanged) */
#define MOE_FLAG_HOST_SYNC_ROUTING 0x8u /* ablation of GPU-resident routing: on the prefill path
                                          the host waits for the routing kernels and reads the tile
                                          count back before it launches the grouped GEMMs (grids
                                          sized from it); same results, one host round trip per
                                          call, so moe_forward synchronises its stream and cannot
                                          be captured in a CUDA graph */
#define MOE_FLAG_DEQUANT_TO_HBM  0x10u /* ablation of the in-GEMM 4-bit reconstruction: moe_create
                                          also writes the layer's weights dequantised to fp16 in
                                          the handle's memory (4x the bytes of the packed codes),
                                          and the prefill grouped GEMMs load those instead of
                                          rebuilding each tile from the 4-bit blocks (same results) */
#define MOE_FLAG_NO_ROUTER       0x20u /* a handle without a router: router, router_bias and
                                          shared_gate may be NULL and are not read; the handle
                                          serves moe_forward_routed (and moe_combine_rows) only,
                                          e.g. one rank's shard of experts in expert parallelism */
#define MOE_FLAG_NO_EXPERTS      0x40u /* a handle without expert weights: the q_*, s_*, b_* and
                                          shared-expert pointers may be NULL and are not read, no
                                          memory is allocated for them, and the handle serves
                                          moe_route (and moe_combine_rows) only: the router of an
                                          expert-parallel layer whose experts live on other GPUs */
#define MOE_FLAG_TEST_STALL      0x100u /* test only: the prefill producer withholds its loads on
                                          every call, and the fused decode kernel withholds
                                          one router result on the handle's first call, so bounded
                                          waits run out and the call reports
                                          MOE_ERR_DEVICE_TIMEOUT; nothing traps or hangs */

typedef struct moe_handle moe_handle;

/* Shapes of one layer.  Supported: hidden % 128 == 0, inter % 64 == 0, group == 64,
 * 1 <= top_k <= num_experts <= 256, top_k <= 32, 1 <= max_tokens <= 65536. */
typedef struct {
    int32_t hidden;            /* H */
    int32_t inter;             /* I: intermediate size of every expert, shared one included */
    int32_t num_experts;       /* E: routed experts */
    int32_t top_k;             /* k */
    int32_t group;             /* quantisation group along the input dimension (must be 64) */
    int32_t has_shared;        /* 1: one always-on shared expert with a sigmoid gate */
    int32_t max_tokens;        /* largest T that moe_forward / moe_route accept */
    int32_t decode_max_tokens; /* T <= this runs the sparse-GEMV decode path; larger T runs the
                                  bucketed grouped-GEMM prefill path.  0 = always prefill path;
                                  at most 65535.
                                  With decode_max_tokens >= 2 (or MOE_FLAG_DECODE_UNFUSED) the
                                  multi-kernel GEMV path needs top_k + has_shared <= 16. */
    uint32_t flags;            /* MOE_FLAG_* */
} moe_config;

/* Weights of one layer in the public ("natural") layout, all DEVICE pointers.
 *  q_gate, q_up : uint32 [E, I, H/8]   packed codes; nibble j (bits 4j..4j+3) of word w is
 *  q_down       : uint32 [E, H, I/8]   element 8w+j of the row (low nibble first)
 *  s_*, b_*     : bf16   [E, rows, cols/64]  scale and bias of each 64-column group
 *  qs_*, ss_*, bs_* : the shared expert, same layout without the leading E (NULL if no shared)
 *  router       : fp32 [E, H];  router_bias: fp32 [E] or NULL;  shared_gate: fp32 [H] or NULL */
typedef struct {
    const uint32_t *q_gate, *q_up, *q_down;
    const uint16_t *s_gate, *b_gate, *s_up, *b_up, *s_down, *b_down;
    const uint32_t *qs_gate, *qs_up, *qs_down;
    const uint16_t *ss_gate, *bs_gate, *ss_up, *bs_up, *ss_down, *bs_down;
    const float *router;
    const float *router_bias;
    const float *shared_gate;
} moe_weights;

/* Source: the layer interface this library exposes (create a layer, then run it on [T, H] bf16
 * activations on a stream); the pages describe the engine, not a layer-level call.
 * Create a layer on `device`: validate cfg, check the device is sm_100, allocate the handle's
 * workspace (sized for cfg->max_tokens) and repack the weights into the handle's own kernel
 * layout with kernels enqueued on `stream`.  moe_create synchronises `stream` before returning,
 * so the caller may free its weight buffers as soon as it returns.  On success *out receives the
 * handle.  Allocates device memory (the only entry point that does).  Scales/biases that are not
 * exactly representable in fp16 are rounded to nearest (the layer still works; the tensor-core
 * path computes in fp16), and nonzero scales below 2^-13 in magnitude are not reproduced exactly
 * by the tensor-core dequantisation (it also uses s / 16).  Errors: INVALID_ARG,
 * UNSUPPORTED_DEVICE, CUDA. */
MOE_API int moe_create(const moe_config *cfg, const moe_weights *w, int device, void *stream,
               moe_handle **out);

/* Source: the forward pass of the layer as defined at the top of this file; prefill runs the
 * bucketed grouped GEMM with in-GEMM 4-bit reconstruction and decode the sparse GEMV over the
 * selected experts ("Perplexity Open-Sources Lily...", section "The optimizations follow the
 * workload"; "A Rust + Metal Inference Engine..." body).
 * out[T, H] (bf16) = the layer applied to x[T, H] (bf16), both device pointers.  T == 0 is a
 * no-op returning MOE_OK.  Errors: INVALID_ARG (null/misaligned pointer, T < 0), TOO_LARGE
 * (T > max_tokens), CUDA (launch failure).  Device-side errors surface via moe_status(). */
MOE_API int moe_forward(moe_handle *h, const uint16_t *x, int32_t T, uint16_t *out, void *stream);

/* Source: library convenience (no passage): the forward pass with host buffers.
 * The same with HOST buffers: copies x to the device, runs moe_forward, copies out back and
 * synchronises `stream` before returning (so the host buffer is ready).  Pinned host memory is
 * fastest; pageable memory works.  Uses handle-owned device staging buffers (no allocation). */
MOE_API int moe_forward_host(moe_handle *h, const uint16_t *x_host, int32_t T, uint16_t *out_host,
                     void *stream);

/* Source: library convenience (no passage).
 * moe_forward_host without the final synchronisation: the copy in, the layer and the copy out are
 * enqueued on `stream` and the call returns.  x_host must stay unchanged and out_host unread until
 * the stream has passed the copy out (synchronise the stream or an event recorded after the call).
 * With pinned host memory the copies are asynchronous, so calls on different handles issued to
 * different streams overlap one layer's copies with another's kernels; pageable memory works but
 * its copies are staged through the driver and overlap little.  The handle's staging buffers are
 * reused by its next call, which is safe because calls on one handle are ordered on its stream.
 * Errors: as moe_forward_host (before launch), device errors via moe_status. */
MOE_API int moe_forward_host_async(moe_handle *h, const uint16_t *x_host, int32_t T, uint16_t *out_host,
                           void *stream);

/* Source: "Perplexity Open-Sources Lily...", section "The optimizations follow the workload":
 * expert routing is kept on the GPU with no CPU synchronisation; this call exposes its results.
 * Routing and bucketing only (the first steps of the prefill path), with their results copied
 * to caller device buffers (any output pointer may be NULL to skip it):
 *   idx[T, k] int32      experts per token, descending logit
 *   gates[T, k] fp32     renormalised softmax gates, same order
 *   shared_gate[T] fp32  sigmoid shared-expert gate (zeros when has_shared == 0)
 *   offsets[E+1] int32   bucket starts: offsets[e] = number of (token, slot) entries routed to
 *                        experts < e; offsets[E] = T*k
 *   perm[T*k] int32      perm[p] = t*k + j for the entry at bucket position p; buckets are in
 *                        expert order and each bucket lists its tokens in ascending order.
 * Errors as for moe_forward. */
MOE_API int moe_route(moe_handle *h, const uint16_t *x, int32_t T, int32_t *idx, float *gates,
              float *shared_gate, int32_t *offsets, int32_t *perm, void *stream);

/* Source: the forward pass defined at the top of this file with its routing step supplied by the
 * caller; the expert-parallel form of the layer (experts sharded over GPUs, rows dispatched to
 * the GPU that holds their expert) calls it on each shard (library design; the pages run one GPU).
 * out[T, H] (bf16) = for each row t of x[T, H] (bf16):
 *     sum_j gates[t, j] FFN_{idx[t, j]}(x_t)  +  shared_gate[t] FFN_shared(x_t)   (bf16 rounding)
 * with idx[T, k] int32 in [0, E) and gates[T, k] fp32 given by the caller (any values: no top-k,
 * no renormalisation, an expert may repeat within a row) and shared_gate[T] fp32 (NULL when
 * has_shared == 0; required otherwise).  The same kernels as moe_forward run after the routing
 * step (grouped GEMMs for T > decode_max_tokens, the GEMV chain otherwise).  An idx entry outside
 * [0, E) contributes nothing and is reported as MOE_ERR_DEVICE_BOUNDS by moe_status.
 * Errors: INVALID_ARG (null/misaligned pointer, handle created with MOE_FLAG_NO_EXPERTS),
 * TOO_LARGE, CUDA. */
MOE_API int moe_forward_routed(moe_handle *h, const uint16_t *x, int32_t T, const int32_t *idx,
                               const float *gates, const float *shared_gate, uint16_t *out, void *stream);

/* Source: the combine step of the forward pass (out_t = sum of the gated expert outputs) for rows
 * that come back from other GPUs in expert parallelism (library design).
 * out[T, H] (bf16) = bf16( base[t] + sum over j < k with pos[t, j] >= 0 of rows[pos[t, j]] ),
 * summed in fp32 in j order, for rows[n_rows, H] bf16, pos[T, k] int32 and base[T, H] bf16 (or
 * NULL for zeros), all device pointers; out may not alias rows or base.  Uses the handle's device
 * and status word only (any handle with matching H).  A pos entry >= n_rows is skipped and
 * reported as MOE_ERR_DEVICE_BOUNDS by moe_status.
 * Errors: INVALID_ARG (null/misaligned pointer, k outside [1, 32], n_rows < 0), CUDA. */
MOE_API int moe_combine_rows(moe_handle *h, const uint16_t *rows, int32_t n_rows, const int32_t *pos,
                             int32_t T, int32_t k, const uint16_t *base, uint16_t *out, void *stream);

/* Source: library convenience (no passage).
 * Synchronise the stream of the handle's last call, read and clear the device status word.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS, MOE_ERR_RANGE (the most severe
 * recorded, in that order of precedence reversed: timeout > bounds > range) or MOE_ERR_CUDA. */
MOE_API int moe_status(moe_handle *h);

/* Source: library convenience (no passage).
 * Debug: copy `bytes` of an internal workspace buffer to a caller device buffer (stream-ordered).
 * which: 0 = expert activations act[rows, I] (fp16, bucket order, prefill path),
 *        1 = fp16 copy of the activations x16[T, H] (prefill path),
 *        2 = router logits [T, E] (fp32, tensor-core router only),
 *        3 = fp32 combine accumulator [T, H].
 * Errors: INVALID_ARG when `which` is unknown or `bytes` exceeds the buffer. */
MOE_API int moe_debug_copy(moe_handle *h, int which, void *dst, size_t bytes, void *stream);

/* Source: library convenience (no passage).
 * Per-kernel timing.  While enabled, moe_forward records a CUDA event on the call's stream before
 * its first kernel and after each kernel it launches (events are created by moe_profile_enable;
 * up to 1024 calls are recorded, later calls run unrecorded).  Do not enable it while capturing a
 * CUDA graph.  moe_profile_read synchronises those events, writes per kernel slot the summed
 * device time in milliseconds (ms[MOE_PROF_SLOTS]) and the number of launches
 * (launches[MOE_PROF_SLOTS]), and clears the record.  Slots: 0 router logits, 1 top-k and gates,
 * 2 bucket scan, 3 scatter/gather, 4 gate/up grouped GEMM, 5 down grouped GEMM + combine,
 * 6 finalize, 7 decode gate/up GEMV, 8 decode down GEMV + combine, 9 fused decode of up to 8 tokens
 * (the whole layer in one kernel), 10 gather of token rows into bucket order.
 * Errors: INVALID_ARG, CUDA. */
#define MOE_PROF_SLOTS 11
MOE_API int moe_profile_enable(moe_handle *h, int enable);
MOE_API int moe_profile_read(moe_handle *h, float *ms, int32_t *launches);

/* Source: library convenience (no passage).
 * Bytes of device memory a handle with this configuration owns (repacked weights + workspace). */
MOE_API size_t moe_device_bytes(const moe_config *cfg);

/* Source: library convenience (no passage).
 * Message describing the last error returned on the calling thread ("" if none). */
MOE_API const char *moe_last_error(void);

/* Source: library convenience (no passage).
 * Free the handle and all device memory it owns.  Synchronises the device first.  NULL is a no-op. */
MOE_API void moe_destroy(moe_handle *h);

/* Routing for callers that cannot allocate device memory.  No counterpart on the pages: this is a
 * library convenience.  Some callers may not call cudaMalloc at all -- a thread recording a CUDA
 * graph (allocation is not a stream operation), a latency-critical serving loop kept out of the
 * allocator, a plug-in inside a framework that owns every device allocation -- and so cannot
 * create a moe_handle.  This entry point computes, for x[T, H] (bf16, device), the router's top-k
 * experts idx[T, k] (int32, device) and their renormalised gates gates[T, k] (fp32, device) from
 * the caller's router[E, H] (fp32, device, public layout) and optional router_bias[E] (fp32 or
 * NULL), with the same selection rule as moe_route (descending logit, ties to the lower index,
 * softmax renormalised over the selection), on the current device and `stream`.  The logits are
 * fp32 sums taken in 32-column slices on CUDA cores, a different summation order from
 * moe_route's tensor-core router at prefill sizes, so idx agrees with moe_route (and with the
 * exact result) whenever adjacent top-(k+1) logits are further apart than fp32 rounding, and the
 * gates agree to about 1e-6.  It allocates nothing:
 * its only scratch (split-K partial logits, T * (H/32) * E floats) lives in a fixed array of
 * MOE_ROUTE_STATIC_SCRATCH_FLOATS floats (1 MiB) compiled into the library, which every GPU that
 * loads the library holds until the process exits.  Larger requests return MOE_ERR_TOO_LARGE.
 * The array is shared by all calls and keeps the last call's contents (each call overwrites what
 * it reads, so nothing needs clearing); calls that overlap on the GPU race on it -- serialise
 * them.  The first call in a CUDA context looks up the array's device address
 * (cudaGetSymbolAddress) with that context current and caches it per context; make that first
 * call before any stream capture begins.  After cudaDeviceReset (or once the primary context has
 * been released and created again) the next call looks the address up again, so it too must be
 * made outside a capture.
 * Errors: INVALID_ARG (H % 32 != 0, k or E out of range, NULL pointer), TOO_LARGE, CUDA. */
#define MOE_ROUTE_STATIC_SCRATCH_FLOATS 262144
MOE_API int moe_route_static(const uint16_t *x, int32_t T, int32_t H, const float *router,
                             const float *router_bias, int32_t E, int32_t k, int32_t *idx,
                             float *gates, void *stream);

/* Source: library convenience (no passage).
 * Library version as major*10000 + minor*100 + patch. */
MOE_API int moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
