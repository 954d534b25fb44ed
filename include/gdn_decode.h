/*
 * gdn_decode.h -- C ABI of the B200 (sm_100a) fused sigmoid-gating Gated
 * DeltaNet decode / speculative-decode state update.
 *
 * The operation (the pages' fused_sigmoid_gating_delta_rule_update):
 *   "[Qwen3Next] Optimize fused_sigmoid_gating_delta_rule_update_kernel"
 *   (sglang PR 18271, Motivation, Highlights) and the vLLM PR 35777 summary
 *   (sections 执行摘要 and 实现拆解) describe one kernel that replaces
 *   fused_gdn_gating + fused_recurrent_gated_delta_rule, takes A_log, a, b
 *   and dt_bias, normalises q/k with rsqrt and serves both the single-token
 *   and the speculative (several tokens per sequence) decode paths.  For
 *   every sequence i, value head hv and token t of that sequence:
 *
 *     g     = -exp(A_log[hv]) * softplus(a[t,hv] + dt_bias[hv])
 *     beta  = sigmoid(b[t,hv])
 *     k^    = k[t,h] * rsqrt(|k[t,h]|^2 + 1e-6)               (GDN_L2NORM_QK)
 *     q^    = scale * q[t,h] * rsqrt(|q[t,h]|^2 + 1e-6)
 *     S     <- exp(g) * S                                    (S: fp32 [K, V])
 *     S     <- S + k^ (beta * (v[t,hv] - S^T k^))^T
 *     out[t,hv] = S^T q^                                     (rounded to bf16)
 *
 *   with h = hv / (HV / H): value heads are grouped contiguously under key
 *   heads (the `ba` reshape to (num_k_heads, 2*num_v_heads/num_k_heads) in
 *   the vLLM PR 37975 report, 实现拆解).  S is read once per sequence from
 *   state_pool[state_indices[i], hv], carried on chip across the sequence's
 *   tokens and written back in place.  A state index of -1 marks a padded
 *   sequence: its output rows are written as zeros and no state is touched.
 *   softplus(x) returns x for x > 20.
 *
 * Tensor descriptors.  Every tensor is passed as a gdn_tensor: a DEVICE
 * pointer, a dtype code, a rank (1..4), a shape and strides in ELEMENTS.
 * The caller owns all memory; the library allocates no device memory and
 * keeps no pointer after the call returns.  Strides must be >= 0.
 *
 *   argument        dtype      shape                              layout rules
 *   q, k            bf16|fp32  [T_tot, H, K] | [1, T_tot, H, K]   K contiguous; token and
 *                              (varlen) or [N, T, H, K] (fixed T) head strides x element
 *                                                                 size % 16 == 0; data
 *                                                                 16-byte aligned
 *   v, out          as q       same leading dims, [.., HV, V]     V contiguous; strides % 4
 *                                                                 == 0; data aligned to 4
 *                                                                 elements
 *   a, b            bf16|fp32  [T_tot, HV] | [1, T_tot, HV] |     any strides (packed `ba`
 *                              [N, T, HV]                         projections are fine)
 *   A_log, dt_bias  fp32   [HV]                                   any stride
 *   state_pool      fp32   [num_slots, HV, K, V]                  K, V contiguous (strides
 *                                                                 V, 1); slot/head strides
 *                                                                 % 4 == 0; 16-byte aligned
 *   state_indices   int32  [N]                                    contiguous
 *   cu_seqlens      int32  [N + 1] or NULL                        contiguous; NULL = every
 *                                                                 sequence has T tokens
 *   intermediate_   fp32   [T_tot, HV, K, V]                      as state_pool
 *     states (extra)
 *
 * With fixed T (cu_seqlens NULL) the leading [N, T] dims of q, k, v, a, b
 * and out must flatten to a single token dimension (stride[0] ==
 * T * stride[1] when N > 1 and T > 1).  Supported head sizes: K = V = 128.
 *
 * Ownership and aliasing.  state_pool is read and written in place (only
 * the slots named by state_indices); out and intermediate_states are
 * written; every other tensor is read only.  No written tensor may overlap
 * any other tensor.  The non-negative entries of state_indices must be
 * distinct (GDN_CHECK_INDICES verifies it on the host).
 *
 * Errors.  The call returns GDN_OK or a negative gdn_status.  Every argument
 * check happens on the host before anything is enqueued; on any error
 * nothing is launched and no memory is touched.  The call is asynchronous
 * on extra->stream (NULL: the legacy default stream) and can be captured in
 * a CUDA graph (unless GDN_CHECK_INDICES is set).  N = 0 or T_tot = 0 is
 * GDN_OK with no launch.  Problems only the device can see (a slot index
 * < -1 or >= num_slots, cu_seqlens not monotone or past T_tot) are reported
 * by OR-ing GDN_DEV_* bits into *extra->device_status (when given); the
 * offending sequence is skipped whole and nothing traps.
 */
#ifndef GDN_DECODE_H
#define GDN_DECODE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_DECODE_ABI_VERSION 2

#if defined(__GNUC__)
#define GDN_API __attribute__((visibility("default")))
#else
#define GDN_API
#endif

/* dtype codes */
#define GDN_DTYPE_BF16 1
#define GDN_DTYPE_F32  2
#define GDN_DTYPE_I32  3

/* flags */
#define GDN_L2NORM_QK          (1u << 0) /* L2-normalise q and k (default on) */
#define GDN_WRITE_INTERMEDIATE (1u << 1) /* store S after every token */
#define GDN_NO_FINAL_WRITEBACK (1u << 2) /* leave state_pool untouched */
#define GDN_CHECK_INDICES      (1u << 3) /* host check of indices / cu_seqlens
                                            (copies them to the host and
                                            synchronises extra->stream) */
#define GDN_LAUNCH_PDL         (1u << 4) /* programmatic dependent launch: the
                                            kernel may be scheduled while the
                                            previous kernel on the stream is
                                            still running; it waits for that
                                            kernel to complete before reading
                                            any input, so results are unchanged */

/* status codes returned by the host call */
#define GDN_OK               0
#define GDN_ERR_NULL_ARG    (-1) /* a required pointer or descriptor is NULL */
#define GDN_ERR_DTYPE       (-2) /* wrong dtype code */
#define GDN_ERR_SHAPE       (-3) /* wrong rank, shape or inconsistent sizes */
#define GDN_ERR_ALIGN       (-4) /* pointer or stride breaks an alignment rule */
#define GDN_ERR_ALIAS       (-5) /* a written tensor overlaps another tensor */
#define GDN_ERR_UNSUPPORTED (-6) /* head size, tile or schedule not built */
#define GDN_ERR_ARG         (-7) /* bad scalar: scale <= 0 or not finite, unknown flag */
#define GDN_ERR_INDICES     (-8) /* GDN_CHECK_INDICES found a bad or repeated slot,
                                    or bad cu_seqlens */
#define GDN_ERR_CUDA        (-9) /* the CUDA runtime refused the launch or copy */
#define GDN_ERR_SCRATCH     (-10) /* gdn_decode_update_static_scratch: the call needs
                                     more scratch than GDN_STATIC_SCRATCH_BYTES */

/* work schedules (gdn_extra.schedule); all compute the same update */
#define GDN_SCHEDULE_AUTO      0 /* library choice, by the mean tokens per sequence
                                    L = T_tot / N and the pair count P = N * HV.
                                    When the call qualifies for the chunked
                                    kernels (bf16 activations, fused gates, no
                                    per-token states, v rows 16-byte aligned):
                                    GDN_SCHEDULE_CHUNKED_SPLIT if the caller gives
                                    a large enough workspace and L >= 80
                                    (2 P <= the device's SM count), >= 144
                                    (P < 128), >= 192 (P < 256) or >= 512
                                    (P < 512); else GDN_SCHEDULE_CHUNKED if
                                    L >= 20 (P < 64), >= 14 (P < 512) or >= 13.
                                    Otherwise GDN_SCHEDULE_PER_TILE */
#define GDN_SCHEDULE_PER_TILE  1 /* one CTA per (sequence, value head, V-tile); the
                                    state tile moves through registers.  Tiles
                                    (tile_v x tile_rows): 8x8, 16x16, 32x16,
                                    32x32, 64x16, 64x32.  Library choice: 64x32
                                    when every sequence has one token, else
                                    32x32 with >= 2048 (sequence, value head)
                                    pairs, 8x8 with <= 64, else 16x16; with
                                    fp32 activations 32x16 for one token, else
                                    16x16 */
#define GDN_SCHEDULE_PIPELINED 2 /* one persistent CTA per SM; whole-head state
                                    tiles stream through a shared-memory ring of
                                    bulk async copies (cp.async.bulk) */
#define GDN_SCHEDULE_CHUNKED   3 /* one CTA per (sequence, value head), two per SM;
                                    tokens in chunks of 64 through the closed
                                    form of the delta rule over a chunk, every
                                    matrix product on the tcgen05 tensor cores and
                                    every intermediate on chip (no workspace);
                                    bf16 activations, gates from A_log/a/b/dt_bias,
                                    no GDN_WRITE_INTERMEDIATE; v aligned like q */
#define GDN_SCHEDULE_CHUNKED_SPLIT 4 /* the same chunked algorithm as two kernels:
                                    the products that do not depend on the state
                                    (decay scan, A, T = (I + A)^-1, W, U, the
                                    masked q.k matrix) for every 64-token block
                                    of the packed token range at once, written to
                                    the caller's workspace; then the recurrence
                                    through the state: two CTAs per (sequence,
                                    value head), each on half of the state's
                                    columns, while 2 P <= the SM count; else
                                    one per pair.  Same restrictions as
                                    GDN_SCHEDULE_CHUNKED, plus a workspace of
                                    gdn_chunked_workspace_bytes(T_tot, HV) bytes
                                    in gdn_extra */

/* bits OR-ed into *device_status by the kernel */
#define GDN_DEV_BAD_SLOT    1u
#define GDN_DEV_BAD_SEQLENS 2u
#define GDN_DEV_TIMEOUT     4u  /* a bounded wait inside the kernel gave up (the
                                   call's results are then incomplete) */

typedef struct gdn_tensor {
    void *data;          /* device pointer */
    int32_t dtype;       /* GDN_DTYPE_* */
    int32_t ndim;        /* 1..4 */
    int64_t shape[4];
    int64_t stride[4];   /* in elements */
} gdn_tensor;

typedef struct gdn_extra {
    void *stream;                          /* cudaStream_t; NULL = legacy default */
    const gdn_tensor *intermediate_states; /* required with GDN_WRITE_INTERMEDIATE */
    uint32_t *device_status;               /* device word for GDN_DEV_* bits, or NULL */
    int32_t tile_v;                        /* per-tile schedule: V-tile width (16, 32
                                              or 64; 0 = library choice) */
    int32_t tile_rows;                     /* per-tile schedule: state rows per thread
                                              (16 or 32; 0 = library choice) */
    int32_t schedule;                      /* GDN_SCHEDULE_* (0 = library choice) */
    int32_t reserved;                      /* must be 0 */
    void *workspace;                       /* device scratch for GDN_SCHEDULE_CHUNKED_SPLIT
                                              (256-byte aligned, owned by the caller,
                                              overlapping no tensor of the call; its
                                              contents need no initialisation and are
                                              garbage afterwards), or NULL */
    uint64_t workspace_bytes;              /* its size in bytes */
} gdn_extra;

/*
 * One fused decode / speculative-decode update (see the top of this file).
 * The first eleven arguments follow the pages' parameter order; `scale` is
 * normally 1/sqrt(K); `extra` may be NULL (default stream, no intermediate
 * states, no status word, library tile choice).
 */
GDN_API int gdn_decode_update(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                      const gdn_tensor *a, const gdn_tensor *b,
                      const gdn_tensor *A_log, const gdn_tensor *dt_bias,
                      const gdn_tensor *state_pool, const gdn_tensor *state_indices,
                      const gdn_tensor *cu_seqlens, const gdn_tensor *out,
                      float scale, uint32_t flags, const gdn_extra *extra);

/*
 * The recurrence of the unfused pair: the pages name the two kernels the
 * fused op replaces, fused_gdn_gating then fused_recurrent_gated_delta_rule
 * (vLLM PR 35777 summary, 执行摘要 / 实现拆解), and the sglang variant
 * with precomputed gates, fused_recurrent_gated_delta_rule_update_fwd
 * ("[Qwen3Next] Optimize ...", Code Review).  Same as gdn_decode_update,
 * except that each token's decay and beta come from arrays:
 *     S <- exp(g[t,hv]) * S;   S <- S + k^ (beta[t,hv] * (v - S^T k^))^T
 *   g     fp32       [tokens..., HV] (same leading dims as a would have)
 *   beta  bf16|fp32  [tokens..., HV]
 * Every other argument, flag, error and the extra struct are as for
 * gdn_decode_update.  GDN_SCHEDULE_PIPELINED is not built for this entry
 * point (GDN_ERR_UNSUPPORTED).
 */
GDN_API int gdn_recurrent_update(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                                 const gdn_tensor *g, const gdn_tensor *beta,
                                 const gdn_tensor *state_pool, const gdn_tensor *state_indices,
                                 const gdn_tensor *cu_seqlens, const gdn_tensor *out,
                                 float scale, uint32_t flags, const gdn_extra *extra);

/*
 * The gating step alone (the pages' fused_gdn_gating, the first kernel of
 * the unfused pair): for every (token, value head)
 *     g[t,hv]    = -exp(A_log[hv]) * softplus(a[t,hv] + dt_bias[hv])
 *     beta[t,hv] = sigmoid(b[t,hv])
 *   A_log, dt_bias  fp32       [HV]
 *   a, b            bf16|fp32  [T_tot, HV]   (rank 2, any strides)
 *   g               fp32       [T_tot, HV]
 *   beta            bf16|fp32  [T_tot, HV]
 * g and beta must not overlap each other or any input.  extra: only the
 * stream is used (NULL: default stream; schedule and reserved must be 0).
 * Asynchronous; T_tot = 0 is GDN_OK with no launch.
 */
GDN_API int gdn_gating(const gdn_tensor *A_log, const gdn_tensor *a, const gdn_tensor *dt_bias,
                       const gdn_tensor *b, const gdn_tensor *g, const gdn_tensor *beta,
                       const gdn_extra *extra);

/* Static text for a gdn_status value (never NULL; "unknown gdn status" for
   a value that is not one). */
GDN_API const char *gdn_status_string(int status);

/* GDN_DECODE_ABI_VERSION of the loaded library. */
GDN_API int gdn_version(void);

/*
 * Bytes of workspace GDN_SCHEDULE_CHUNKED_SPLIT needs for a call with T_tot
 * tokens and HV value heads (K = V = 128): one 131,584-byte record per
 * (64-token block of the packed token range, value head).  0 for T_tot <= 0
 * or HV <= 0; UINT64_MAX when the size does not fit in 64 bits.  Host-only
 * arithmetic, no CUDA call.
 */
GDN_API uint64_t gdn_chunked_workspace_bytes(int64_t T_tot, int64_t HV);

/* Size of the library's built-in scratch array (64 MiB; see below). */
#define GDN_STATIC_SCRATCH_BYTES (64ull << 20)

/* GDN_STATIC_SCRATCH_BYTES of the loaded library (host-only, no CUDA call). */
GDN_API uint64_t gdn_static_scratch_bytes(void);

/*
 * gdn_decode_update on the split chunked schedule, with NO device allocation
 * by anyone: for callers that cannot allocate device memory -- code handed
 * device buffers by a host program that owns every allocation (an inference
 * server's memory planner, a plugin inside another framework), or code that
 * must not call cudaMalloc because it may synchronise the device or fail
 * under a fixed memory budget.  The pages have no counterpart of this entry
 * point; it is an interface convenience of this library.
 *
 * Arguments and results are those of gdn_decode_update; the caller still
 * passes every input and output.  The workspace is a fixed 64 MiB array
 * inside the library (GDN_STATIC_SCRATCH_BYTES), created on every GPU that
 * loads the library and kept until the process exits.  So:
 *   - a call may need at most GDN_STATIC_SCRATCH_BYTES of workspace, i.e.
 *     gdn_chunked_workspace_bytes(T_tot, HV) <= 64 MiB (510 records: about
 *     4,000 tokens at HV = 8); larger calls return GDN_ERR_SCRATCH before
 *     anything is launched;
 *   - extra->workspace must be NULL (and workspace_bytes 0), extra->schedule
 *     0 or GDN_SCHEDULE_CHUNKED_SPLIT; the call runs the split chunked
 *     kernels, with their restrictions (bf16 activations, fused gates, no
 *     GDN_WRITE_INTERMEDIATE);
 *   - every call on a device shares the one array, which keeps the previous
 *     call's contents.  Nothing in it needs to start at zero (each call writes
 *     every workspace byte it reads before reading it), but two calls that
 *     can overlap on the GPU (different streams, or different host threads,
 *     on the same device) race on it: order such calls, e.g. on one stream;
 *   - the array's device address is looked up (cudaGetSymbolAddress, with
 *     the call's device current) on every call whose stream is not
 *     capturing, so it follows the module if the device's context is torn
 *     down and created again; a call inside a stream capture reuses the
 *     address found by the last call on that device outside capture.  The
 *     first call on a device may load the library's module there: make it
 *     before any stream capture on the device.
 *   - sizes are checked before anything else: a shape whose dims exceed
 *     INT32_MAX returns GDN_ERR_SHAPE, a call too large for the array
 *     GDN_ERR_SCRATCH, and a non-NULL extra->workspace, a nonzero
 *     extra->workspace_bytes or a schedule other than 0 /
 *     GDN_SCHEDULE_CHUNKED_SPLIT GDN_ERR_ARG, all before any CUDA call.
 * The library allocates no device memory for this call.
 */
GDN_API int gdn_decode_update_static_scratch(const gdn_tensor *q, const gdn_tensor *k, const gdn_tensor *v,
                                             const gdn_tensor *a, const gdn_tensor *b,
                                             const gdn_tensor *A_log, const gdn_tensor *dt_bias,
                                             const gdn_tensor *state_pool, const gdn_tensor *state_indices,
                                             const gdn_tensor *cu_seqlens, const gdn_tensor *out,
                                             float scale, uint32_t flags, const gdn_extra *extra);

/*
 * One step of a host-fed update loop, issued in a single call: the pinned
 * host -> device copy of the step's packed inputs, the update, and the
 * device -> host copy of its output, each on its own stream and ordered by
 * events, so that a loop keeping several such steps in flight overlaps the
 * transfers of neighbouring steps with the update (the step's cost on the
 * host is one call instead of a dozen runtime calls).  Host plumbing: the
 * pages have no counterpart of it.
 *
 * Per slot (a set of buffers reused every `depth` steps) the caller keeps one
 * gdn_host_step; per call the library enqueues, in order:
 *   copy_in:  [wait ev_ran, if `reused`] copy in_bytes host_in -> dev_in;
 *             record ev_h2d
 *   compute:  wait ev_h2d; [wait ev_d2h, if `reused`]; gdn_decode_update with
 *             the descriptors below (they describe views of dev_in and
 *             dev_out; extra->stream is the compute stream); record ev_ran
 *   copy_out: wait ev_ran; copy out_bytes dev_out -> host_out; record ev_d2h
 * `reused` (nonzero when the slot served an earlier step) makes the copy in
 * wait until that step's update has read dev_in, and the update wait until
 * that step's output has left dev_out.  Nothing waits on the host: the
 * caller synchronises on ev_h2d before rewriting host_in and on ev_d2h
 * before reading host_out.  host_in / host_out should be pinned (page-locked)
 * for the copies to be asynchronous.  Streams and events are the caller's
 * (cudaStream_t / cudaEvent_t, events preferably without timing).
 *
 * Returns the update's status (nothing after a failed update is enqueued),
 * GDN_ERR_NULL_ARG for a missing pointer, or GDN_ERR_CUDA when the runtime
 * refuses a copy or an event operation (steps enqueued before it stay
 * enqueued).
 */
typedef struct {
    const gdn_tensor *q, *k, *v, *a, *b, *A_log, *dt_bias, *state_pool, *state_indices, *cu_seqlens, *out;
    float scale;
    uint32_t flags;
    const gdn_extra *extra;       /* required: its stream is the compute stream */
    const void *host_in;
    void *dev_in;
    uint64_t in_bytes;
    const void *dev_out;
    void *host_out;
    uint64_t out_bytes;
    void *copy_in_stream;         /* cudaStream_t */
    void *copy_out_stream;        /* cudaStream_t */
    void *ev_h2d, *ev_ran, *ev_d2h; /* cudaEvent_t */
    int32_t reused;
} gdn_host_step;

GDN_API int gdn_host_step_issue(const gdn_host_step *step);

#ifdef __cplusplus
}
#endif

#endif /* GDN_DECODE_H */
