/*
 * libtc -- the Tensor Cache layer on NVIDIA B200 (sm_100a).
 *
 * The layer is the one of "Tensor Cache: Eviction-conditioned Associative
 * Memory for Transformers" (arXiv 2605.22884).  Per batch b and head h it
 * combines two read paths over the keys/values seen so far:
 *
 *   L1 (§3.1, eq. (1))  y_local_t = softmax_j(<q_t,k_j>/sqrt(d_k)) v_j over
 *                       the window j = t-W+1 .. t (exact causal attention);
 *   L2 (§3.2)           A in R^{d_k x d_v}, A = 0 at the start, written only
 *                       when a pair leaves the window (Fig. 2 step (3)):
 *                       A <- lambda_h A + eta_h k_{t-W} v_{t-W}^T,
 *                       read as the row vector m_t = q_t A (abstract, read
 *                       identity q (k (x) v) = <q,k> v);
 *   fusion (Fig. 2 (5)) y_t = y_local_t + sigmoid(g_h) m_t.
 *
 * Read-after-write order: inside step t the eviction of token t-W is written
 * into A BEFORE q_t reads A, and k_t is inserted into the window before the
 * softmax.  The query at step t therefore sees token t-W through A and tokens
 * t-W+1..t through the window: every earlier token reaches it through exactly
 * one path (§3.2).
 *
 * Conventions shared by every call:
 *  - Layouts are row-major and contiguous.  q, k: [B,H,T,d_k]; v, y:
 *    [B,H,T,d_v]; A: [B,H,d_k,d_v] (so m = q A is a row-vector product);
 *    lambda, eta, g: [H] float32.  A is always float32.
 *  - Every pointer is a device pointer unless the function name ends in
 *    _host.  Every device pointer must be 16-byte aligned.
 *  - The caller owns every buffer; libtc never allocates device or pinned
 *    memory.  Scratch space ("workspace") is caller-provided, sized by the
 *    matching *_workspace_size query.
 *  - Work is enqueued asynchronously on the caller's stream (NULL = legacy
 *    default stream).  A call returns once its kernels are enqueued.
 *  - Host-side validation failures return an error code and enqueue nothing.
 *    A kernel launch failure returns TC_ERR_CUDA.
 *  - The library is stateless apart from one per-device status word that
 *    kernels set when they detect a device-side error (read and cleared by
 *    tc_get_device_status).
 */
#ifndef TC_H
#define TC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TC_API __attribute__((visibility("default")))
#else
#define TC_API
#endif

/* Same type as cudaStream_t; declared here so this header needs no CUDA
 * headers. */
typedef struct CUstream_st *tc_stream_t;

typedef enum tc_status {
    TC_OK = 0,
    TC_ERR_INVALID_ARG = 1,    /* null / misaligned / host pointer, bad size */
    TC_ERR_UNSUPPORTED = 2,    /* valid request outside the supported set    */
    TC_ERR_NO_DEVICE = 3,      /* no CUDA device, or not an sm_100 device    */
    TC_ERR_CUDA = 4,           /* a CUDA runtime call or launch failed       */
    TC_ERR_DEVICE_BOUNDS = 5,  /* a kernel caught an out-of-range index      */
    TC_ERR_DEVICE_TIMEOUT = 6, /* a bounded device wait ran out              */
    TC_ERR_WORKSPACE = 7       /* workspace missing or smaller than queried  */
} tc_status;

typedef enum tc_dtype {
    TC_F32 = 0, /* float32 q/k/v/y, float32 arithmetic                     */
    TC_BF16 = 1 /* bfloat16 q/k/v/y (RNE output), float32 accumulation/state */
} tc_dtype;

/* tc_prefill_desc.flags */
#define TC_PREFILL_L1_ONLY 1u    /* skip L2 entirely: y = y_local (sigmoid(g) = 0
                                    taken literally, no A work); A_final unused */
#define TC_PREFILL_STATE_ONLY 2u /* L2 write path alone: only A_final is
                                    computed (the chunk scan over the call's
                                    evictions); q and y are not used and may be
                                    NULL.  Not combinable with L1_ONLY. */
#define TC_PREFILL_DELTA_RULE 4u /* write evictions with the delta rule
                                    (TC_WRITE_DELTA below) instead of the outer
                                    product.  Each write then reads A, so the
                                    chunk scan does not apply: the portable path
                                    runs the writes of a head in token order. */
#define TC_PREFILL_CHUNK_MEAN 8u /* ablation, with TC_PREFILL_STATE_ONLY only:
                                    the chunk-mean shortcut the paper warns
                                    against (abstract; §1), A <- lambda A +
                                    eta kbar vbar^T once per chunk of C
                                    evictions (kbar, vbar the chunk's means),
                                    instead of the exact weighted sum.  It adds
                                    C^2 - C spurious cross terms per chunk; it
                                    exists to measure that error. */

/* Shapes of one prefill call.  Supported: B, H >= 1; T >= 0; 1 <= d_k, d_v
 * <= 128; W >= 1; C >= 1. */
typedef struct tc_prefill_desc {
    int64_t B, H, T; /* batch, heads, tokens                                 */
    int64_t dk, dv;  /* key and value head dimensions                        */
    int64_t W;       /* window length (ring capacity) of L1                  */
    int64_t C;       /* eviction chunk length of the state scan; the result
                        does not depend on C beyond rounding                  */
    tc_dtype dtype;  /* dtype of q, k, v and y                               */
    uint32_t flags;  /* TC_PREFILL_* bits                                    */
} tc_prefill_desc;

/* Bytes of device workspace tc_prefill needs for desc (0 if none).  Returns
 * (size_t)-1 when desc is NULL or invalid. */
TC_API size_t tc_prefill_workspace_size(const tc_prefill_desc *desc);

/* Training / prefill form of the layer over T tokens from an empty state
 * (ring empty, A = 0).
 *
 * Computes y [B,H,T,d_v] (dtype of desc) and, unless TC_PREFILL_L1_ONLY is
 * set, A_final [B,H,d_k,d_v] float32 = A after the last eviction (all zero
 * when T <= W).  A is obtained by the parallel weighted-sum chunk scan of
 * the paper (abstract; §1 contributions; §2 training considerations):
 *   A_{c+1} = lambda^{C_c} A_c + eta sum_{i<C_c} lambda^{C_c-1-i} k_i v_i^T
 * over chunks of evictions, which equals the per-token writes exactly in
 * real arithmetic; the chunk-mean shortcut is never used.
 *
 * q, k, v: device inputs.  lambda, eta, g: [H] float32 device.
 * y: device output.  With T = 0, q, k, v and y may be NULL.  A_final: device output, may be NULL only with
 * TC_PREFILL_L1_ONLY.  workspace: device scratch of at least
 * tc_prefill_workspace_size(desc) bytes (NULL allowed when that is 0); its
 * contents on entry are ignored and on exit are undefined.
 * Inputs must not overlap outputs.
 *
 * Paths: bf16 with d_k = d_v in {64, 128} runs on the tensor cores, by
 * default on the general path (per-chunk sums, a chunk scan, and a window
 * kernel that also computes the memory's reads); d = 64 with W a multiple of
 * 128 can run on the fused kernel instead (tc_set_prefill_path).  Other
 * calls run on the portable float32 kernels.  Both tensor-core paths keep A
 * in float32 and meet the same tolerances; they are not bit-identical.
 *
 * Errors: TC_ERR_INVALID_ARG, TC_ERR_UNSUPPORTED, TC_ERR_WORKSPACE,
 * TC_ERR_NO_DEVICE, TC_ERR_CUDA.  On error nothing is enqueued except for
 * TC_ERR_CUDA, after which the outputs are undefined. */
TC_API tc_status tc_prefill(const tc_prefill_desc *desc, const void *q, const void *k, const void *v,
                     const float *lambda, const float *eta, const float *g, void *y,
                     float *A_final, void *workspace, size_t workspace_bytes, tc_stream_t stream);

/* Continuation of a sequence: the same layer over desc->T new tokens that
 * start at global position t0 >= 0, given what the tokens before t0 left
 * behind.  It serves chunked prefill, a prefill that resumes after decode
 * steps, and sequence sharding across GPUs (each rank continues from the
 * previous ranks' tokens).  The paper defines the layer token by token (Fig. 2:
 * evict, write A, insert, read); this entry point computes exactly what that
 * loop computes for tokens t0 .. t0+T-1 when started from:
 *
 *   halo_k, halo_v  [B,H,n,d_k] / [B,H,n,d_v], dtype of desc, device: the keys
 *                   and values of tokens t0-n .. t0-1, oldest first, where
 *                   n = min(t0, W) (the window content at t0).  NULL allowed
 *                   when n = 0.
 *   A_init          [B,H,d_k,d_v] float32 device: A after every eviction before
 *                   t0 (evictions e < t0 - W).  NULL means A = 0.
 *
 * q, k, v, y are the new tokens' rows [B,H,T,d].  A_final is A after the
 * last eviction of the call.  With TC_PREFILL_STATE_ONLY only A_final is
 * computed.  bf16 with d_k = d_v in {64, 128} runs on the general
 * tensor-core path (any W, any t0; the fused kernel when selected, for d =
 * 64, W a multiple of 128 and t0 = 0 or t0 >= W); other calls run on the
 * portable float32 path.
 * Workspace: tc_prefill_from_state_workspace_size(desc, t0) bytes.  Errors
 * as tc_prefill, plus TC_ERR_INVALID_ARG for t0 < 0 or a missing halo. */
TC_API size_t tc_prefill_from_state_workspace_size(const tc_prefill_desc *desc, int64_t t0);
TC_API tc_status tc_prefill_from_state(const tc_prefill_desc *desc, int64_t t0,
                                       const void *halo_k, const void *halo_v,
                                       const float *A_init, const void *q, const void *k,
                                       const void *v, const float *lambda, const float *eta,
                                       const float *g, void *y, float *A_final, void *workspace,
                                       size_t workspace_bytes, tc_stream_t stream);

/* Variable-length prefill: desc->B sequences of different lengths in one
 * call, each the layer over its own tokens from an empty state (ring empty,
 * A = 0), exactly as tc_prefill would run it alone.  Each sequence runs its
 * own streaming step (§3.2, Fig. 2); nothing passes between sequences.
 *
 *   cu_seqlens  int64 device [desc->B + 1], 8-byte aligned: sequence b holds
 *               the packed token rows cu_seqlens[b] .. cu_seqlens[b+1]-1.
 *               cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = total,
 *               every length <= desc->T.  Empty sequences are allowed.
 *   total       packed token rows, 0 <= total <= 2^30.
 *   desc->T     the longest length (it sizes the schedule and workspace).
 *   q, k, v, y  packed token-major [total, H, d] (head rows of one token
 *               adjacent); may be NULL when total = 0.
 *   A_final     [B, H, d_k, d_v] float32, A after each sequence's last
 *               eviction (0 for a sequence of at most W tokens); may be NULL
 *               only with TC_PREFILL_L1_ONLY.
 *   workspace   tc_prefill_varlen_workspace_size(desc) bytes.
 *
 * Supported: the tensor-core paths only (bf16, d_k = d_v in {64, 128}, any
 * W, flags 0 or TC_PREFILL_L1_ONLY; d = 64 with W a multiple of 128 runs the
 * fused kernel unless tc_set_prefill_path selects the general path, the rest
 * the general tensor-core path); other descriptions
 * return TC_ERR_UNSUPPORTED (and (size_t)-1 from the size query).  The offsets are
 * device data, so the host cannot check them: the kernels do.  A sequence
 * whose offsets are negative, decreasing, past total or longer than desc->T
 * is skipped (its rows of y are not written, its A_final is zero) and the
 * call sets TC_ERR_DEVICE_BOUNDS in the device status word
 * (tc_get_device_status); nothing outside the buffers is read or written.
 * Other errors as tc_prefill. */
TC_API size_t tc_prefill_varlen_workspace_size(const tc_prefill_desc *desc);
TC_API tc_status tc_prefill_varlen(const tc_prefill_desc *desc, const int64_t *cu_seqlens,
                                   int64_t total, const void *q, const void *k, const void *v,
                                   const float *lambda, const float *eta, const float *g, void *y,
                                   float *A_final, void *workspace, size_t workspace_bytes,
                                   tc_stream_t stream);

/* Exclusive prefix of L2 states over consecutive pieces of one sequence
 * (sequence sharding: piece s is the part of the sequence held by rank s).
 * Piece s alone, started from A = 0, leaves dA_s after its E_s evictions
 * (tc_prefill_from_state with TC_PREFILL_STATE_ONLY and A_init = NULL).
 * Every eviction does A <- lambda A + eta k v^T (§3.2, Fig. 2 step (3)), so
 * the state before piece n_parts is
 *   A_out = sum_s lambda^(E_{s+1} + ... + E_{n_parts-1}) dA_s,
 * computed as A <- lambda^{E_s} A + dA_s for s = 0 .. n_parts-1.
 *   dA     [n_parts][B,H,d_k,d_v] float32 device
 *   E      [n_parts] int64 device (eviction counts)
 *   lambda [H] float32 device;  A_out [B,H,d_k,d_v] float32 device.
 * n_parts = 0 gives A_out = 0.  Errors: TC_ERR_INVALID_ARG, TC_ERR_NO_DEVICE,
 * TC_ERR_CUDA.  Asynchronous on stream. */
TC_API tc_status tc_state_fold(int64_t B, int64_t H, int64_t dk, int64_t dv, int64_t n_parts,
                               const float *dA, const int64_t *E, const float *lambda,
                               float *A_out, tc_stream_t stream);

/* Backward of the layer (outer-product write) over T tokens from an empty
 * state, for training: with L = sum_t <dy_t, y_t> it computes
 *   dq, dk, dv  [B,H,T,d] float32 (gradients of q, k, v; input layout),
 *   dlambda, deta, dg  [H] float32 (summed over the batch).
 * The pages train lambda, eta and g end to end (§2 training
 * considerations); the formulas are reverse mode through the token loop of
 * Fig. 2.  The window part is the usual softmax backward over the W keys:
 * for bf16 with d_k = d_v in {64, 128} two tcgen05 kernels (scores and their
 * gradients in TMEM, P and dS fed back to the tensor cores as bf16 hi + lo
 * pairs, float32 accumulation), otherwise two float32 SIMT kernels.  The
 * memory part is the reverse scan of dL/dA_t taken in chunks (per-chunk
 * sums, a scan over the chunks, per-chunk gradients): tcgen05 kernels with
 * chunks of 128 for bf16 with d = 64, float32 SIMT with chunks of 32
 * otherwise.  Every sum has a fixed order: two calls give the same bits.
 * q, k, v, dy: device, dtype of desc (dy has y's layout); desc->flags must
 * be 0 (C is not used).  Up to six launches.  Workspace:
 * tc_backward_workspace_size(desc) bytes (about
 * B*H*(2 T' + 2 d_k d_v ceil((T-W)/32)) floats, T' = T rounded up to a
 * multiple of 64).  A bounded wait inside the tensor-core kernels that runs
 * out leaves TC_ERR_DEVICE_TIMEOUT in the device status word.  Errors as
 * tc_prefill. */
TC_API size_t tc_backward_workspace_size(const tc_prefill_desc *desc);
TC_API tc_status tc_backward(const tc_prefill_desc *desc, const void *q, const void *k,
                             const void *v, const float *lambda, const float *eta, const float *g,
                             const void *dy, float *dq, float *dk, float *dv, float *dlambda,
                             float *deta, float *dg, void *workspace, size_t workspace_bytes,
                             tc_stream_t stream);

/* Number of kernel launches one tc_backward call enqueues for desc, or -1
 * when desc is NULL, invalid or has flags set.  When tensor_cores is not
 * NULL it receives 1 if the call runs the tcgen05 kernels (bf16,
 * d_k = d_v = 64, on a device that has them) and 0 for the float32 SIMT
 * kernels. */
TC_API int tc_backward_launch_count(const tc_prefill_desc *desc, int *tensor_cores);

/* Number of kernel launches one tc_prefill call enqueues for desc on the
 * current device (the path depends on shapes and dtype), or -1 when desc is
 * NULL or invalid.  tc_decode_step always enqueues exactly one. */
TC_API int tc_prefill_launch_count(const tc_prefill_desc *desc);

/* Device staging bytes tc_prefill_host needs: tc_prefill_workspace_size
 * plus room for q, k, v, y, A_final and the [H] parameters on the device.
 * Returns (size_t)-1 when desc is NULL or invalid. */
TC_API size_t tc_prefill_host_workspace_size(const tc_prefill_desc *desc);

/* tc_prefill with HOST inputs and outputs (use pinned memory for overlap).
 * Enqueues on stream: host-to-device copies of q, k, v, lambda, eta, g into
 * the caller's device workspace, the prefill, and device-to-host copies of y
 * and A_final.  The host buffers must stay valid until the stream reaches
 * that point; synchronize the stream before reading y or A_final.
 * A_final may be NULL (it is then not copied back). */
TC_API tc_status tc_prefill_host(const tc_prefill_desc *desc, const void *q, const void *k,
                          const void *v, const float *lambda, const float *eta, const float *g,
                          void *y, float *A_final, void *workspace, size_t workspace_bytes,
                          tc_stream_t stream);

/* Size of the scratch array compiled into the library for
 * tc_prefill_no_alloc: 16 MiB per GPU that loads the library. */
#define TC_NO_ALLOC_SCRATCH_BYTES (16u << 20)

/* tc_prefill without a workspace, for callers that cannot allocate device
 * memory (a host framework that owns every allocation, a real-time path that
 * must not block in an allocator, a plugin with no allocator to call).  The
 * paper has no counterpart: this is a deployment convenience of this library.
 *
 * Same arguments, results and errors as tc_prefill, except that the scratch
 * space is a fixed array inside the library (TC_NO_ALLOC_SCRATCH_BYTES,
 * resident on every GPU that loads the library until the process exits).
 * Returns TC_ERR_WORKSPACE, enqueuing nothing, when desc would need more
 * scratch than that (tc_prefill_workspace_size(desc) tells how much).  Under
 * TC_PATH_AUTO a call that both tensor-core paths take runs on the fused
 * kernel when only its scratch fits (the general path keeps per-chunk
 * states: 100 MiB at B = 8, H = 12, T = 4096, d = 64).
 * The first call on each device looks up the array's device address with
 * that device current; make that first call before any stream capture.  The
 * address is cached until a call fails with TC_ERR_CUDA; after a
 * cudaDeviceReset the array may sit elsewhere, so treat the next call as a
 * first call again (outside any capture).
 * All calls share the array and leave their data in it; no call depends on
 * what an earlier one left, but calls whose kernels may overlap on the GPU
 * (unordered streams) race on it and must not be issued that way.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
TC_API tc_status tc_prefill_no_alloc(const tc_prefill_desc *desc, const void *q, const void *k,
                                     const void *v, const float *lambda, const float *eta,
                                     const float *g, void *y, float *A_final, tc_stream_t stream);

/* Streaming state of one layer: the L1 ring buffer, the L2 matrix and the
 * clock.  All arrays are caller-owned device memory, updated in place.
 *   ring_k [B,H,W,d_k], ring_v [B,H,W,d_v] in kv_dtype: slot s holds the
 *     token t' < t with t' mod W = s among the last min(t,W) tokens;
 *   A [B,H,d_k,d_v] float32: the L2 state after the evictions so far;
 *   t: number of tokens consumed so far (the next step's clock).
 * A prefill over T tokens continues as a stream with t = T, A = A_final and
 * token j (for the last min(T,W) tokens) copied to slot j mod W. */
/* Write rule of Fig. 2 step (3), A <- lambda A + eta update(k_old, v_old):
 *   TC_WRITE_OUTER  update = k_old v_old^T (the paper's layer);
 *   TC_WRITE_DELTA  update = k_old (v_old - k_old^T A)^T, the optional delta
 *                   (Widrow-Hoff error-correcting) rule the figure mentions.
 *                   The pages give no formula; k_old^T A is read from A
 *                   before the write, i.e. the memory's current prediction
 *                   of v_old from k_old. */
typedef enum tc_write_rule { TC_WRITE_OUTER = 0, TC_WRITE_DELTA = 1 } tc_write_rule;

typedef struct tc_decode_state {
    int64_t B, H, dk, dv, W;
    int64_t t;
    tc_dtype kv_dtype; /* dtype of ring_k/ring_v and of q_t, k_t, v_t, y_t */
    void *ring_k;
    void *ring_v;
    float *A;
    const float *lambda; /* [H] */
    const float *eta;    /* [H] */
    const float *g;      /* [H] */
    tc_write_rule write_rule; /* TC_WRITE_OUTER (0, the paper's layer) or TC_WRITE_DELTA */
} tc_decode_state;

/* One streaming step (§3.2, Fig. 2) for every (b,h), in the paper's order:
 * (2) if t >= W the pair in slot pos = t mod W is evicted, (3) written
 * A <- lambda A + eta k_old v_old^T (or the delta update of write_rule),
 * (4) (k_t, v_t) is stored in slot pos,
 * (5) y_t = softmax-attention(q_t, filled slots) + sigmoid(g) q_t A.
 * Before the ring fills (t < W) slots t+1..W-1 are masked out.
 *
 * q_t, k_t: [B,H,d_k]; v_t, y_t: [B,H,d_v]; device, kv_dtype.
 * On TC_OK the kernels are enqueued and state->t is incremented on the host.
 * Supported: d_k = d_v in {16, 32, 64, 128}, 1 <= W.
 * Errors: as tc_prefill (state->t is unchanged on error). */
TC_API tc_status tc_decode_step(tc_decode_state *state, const void *q_t, const void *k_t,
                         const void *v_t, void *y_t, tc_stream_t stream);

/* tc_decode_step for a ragged batch: every batch row b has its own clock
 * t_rows[b] (device int64 [B]) instead of the shared state->t (which is
 * ignored and not advanced).  Row b takes one step of Fig. 2 at t_rows[b]:
 * its ring slot is t_rows[b] mod W, it evicts only when t_rows[b] >= W, and
 * its window covers min(t_rows[b] + 1, W) filled slots.  A row with a
 * negative clock is empty: its ring, A and y are left untouched.  After the
 * step the library advances every non-negative clock by one on the device
 * (a second, small kernel on the same stream), so the caller can start rows
 * (write their clock) and retire them (write -1) between steps without host
 * synchronisation.  Errors as tc_decode_step; t_rows must be 8-byte aligned
 * device memory. */
TC_API tc_status tc_decode_step_ragged(tc_decode_state *state, int64_t *t_rows, const void *q_t,
                                       const void *k_t, const void *v_t, void *y_t,
                                       tc_stream_t stream);

/* Device staging bytes tc_decode_step_host needs (q_t, k_t, v_t, y_t).
 * Returns (size_t)-1 when state is NULL or invalid. */
TC_API size_t tc_decode_step_host_workspace_size(const tc_decode_state *state);

/* tc_decode_step with HOST q_t, k_t, v_t and y_t (the state stays on the
 * device): copies the inputs into the device workspace, runs the step and
 * copies y_t back, all enqueued on stream. */
TC_API tc_status tc_decode_step_host(tc_decode_state *state, const void *q_t, const void *k_t,
                              const void *v_t, void *y_t, void *workspace,
                              size_t workspace_bytes, tc_stream_t stream);

/* Limit, in nanoseconds, of every bounded wait inside the tensor-core prefill
 * kernels (an mbarrier wait for a copy, a tensor-core product or another warp).
 * A wait that runs out makes the kernel drain its copies and products, record
 * TC_ERR_DEVICE_TIMEOUT in the device status word and return, so a stalled
 * pipeline ends with an error instead of a hung GPU.  0 restores the default
 * of 2 s, far beyond any legitimate wait.  Process-wide; it applies to calls
 * made after it and is meant for tests of that failure path (a limit of a
 * microsecond makes the first wait of a real call run out).  Not thread-safe
 * against concurrent calls. */
TC_API void tc_set_wait_limit_ns(uint64_t ns);

/* Which tensor-core prefill runs a call that both can take: bf16, d_k = d_v
 * = 64, W a multiple of 128 and t0 = 0 or t0 >= W (plain, L1-only and
 * variable-length calls, and the window part of a delta-rule call).
 *   TC_PATH_AUTO     the faster of the two on B200 (the default): the
 *                    general path for fixed-length calls, the fused kernel
 *                    for variable-length calls
 *   TC_PATH_FUSED    the fused kernel: span summaries, their prefix, and one
 *                    kernel that carries the memory's state on chip
 *   TC_PATH_GENERAL  the general path: per-chunk sums, a chunk scan, and the
 *                    window kernel that also computes the memory's reads
 * Calls that only one path takes run there whatever the setting.  Both give
 * results within the same tolerances of the definition (float32 state, bf16
 * P); they are not bit-identical to each other.  Process-wide; applies to
 * calls, workspace-size and launch-count queries made after it, so query the
 * workspace after choosing.  Not thread-safe against concurrent calls.
 * Returns TC_ERR_INVALID_ARG (and keeps the setting) for any other value. */
#define TC_PATH_AUTO 0
#define TC_PATH_FUSED 1
#define TC_PATH_GENERAL 2
TC_API tc_status tc_set_prefill_path(int path);

/* The current setting of tc_set_prefill_path. */
TC_API int tc_get_prefill_path(void);

/* The path (TC_PATH_FUSED or TC_PATH_GENERAL) a fixed-length call described
 * by desc would take now, continuing at t0 (0 for tc_prefill; the delta
 * rule's window part counts); -1 when desc is NULL
 * or invalid or neither tensor-core path takes it (the float32 SIMT path
 * then runs).  Needs no device. */
TC_API int tc_prefill_path_for(const tc_prefill_desc *desc, int64_t t0);

/* Synchronizes stream, then returns and clears the device status word of the
 * current device: TC_OK, TC_ERR_DEVICE_BOUNDS or TC_ERR_DEVICE_TIMEOUT. */
TC_API tc_status tc_get_device_status(tc_stream_t stream);

/* Static description of a status code (never NULL). */
TC_API const char *tc_status_string(tc_status status);

/* Library version, "major.minor.patch". */
TC_API const char *tc_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TC_H */
