/*
 * zcmoe — forward pass of a mixture-of-experts layer with zero-computation
 * experts, for NVIDIA B200 (sm_100a).  C ABI of libzcmoe.so.
 *
 * The layer (LongCat-Flash technical summary, zhangjingwei.cn, section 二 架構,
 * part 1 "零計算專家", and 模型配置):
 *   - N FFN experts (ids 0..N-1) and Z zero-computation experts (ids N..N+Z-1);
 *     a zero expert returns its input and costs nothing;
 *   - router logits over all E = N+Z experts are softmaxed (LongCat-Flash-Lite
 *     N-gram article, onthewifi.com, part 02: fused "softmax + top-k + scaling");
 *   - top-k is taken on score + per-expert bias; the bias only selects
 *     (LongCat-Flash tech-report thread, web3.cnouyi.fund: DeepSeek-V3-style
 *     auxiliary-loss-free bias, with a decay schedule on its update);
 *   - the gate of a chosen expert is routed_scale * its unbiased score;
 *   - chosen FFN experts apply a SwiGLU FFN, W_d (silu(W_g x) * (W_u x));
 *   - the output is the gate-weighted sum;
 *   - a PID controller moves the bias so the FFN/zero selection ratio tracks a
 *     target (zhangjingwei.cn, 二.1, "計算預算控制").
 *
 * Conventions for every entry point:
 *   - Return 0 (ZCMOE_OK) or a negative ZCMOE_E* code; zcmoe_last_error() then
 *     holds a message (thread-local).  Nothing aborts, traps or exits.
 *   - "device" pointers are CUDA device memory of the current device; "host"
 *     pointers are ordinary CPU memory.  All tensors are dense row-major.
 *   - zcmoe_forward and zcmoe_update_bias only enqueue work on `stream` and do
 *     not synchronise the host; the caller orders calls on one handle (one
 *     stream at a time; concurrent calls on one handle are undefined).
 */
#ifndef ZCMOE_H
#define ZCMOE_H

#include <stdint.h>
#include <cuda_runtime.h>

#if defined(__GNUC__)
#define ZCMOE_API __attribute__((visibility("default")))
#else
#define ZCMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define ZCMOE_OK 0
#define ZCMOE_EINVAL (-1)       /* null pointer, bad shape, misaligned pointer or size    */
#define ZCMOE_ERANGE (-2)       /* T < 0 or T > max_tokens                                 */
#define ZCMOE_ENOMEM (-3)       /* device or host allocation failed                        */
#define ZCMOE_ECUDA (-4)        /* a CUDA runtime/driver call or launch failed             */
#define ZCMOE_EUNSUPPORTED (-5) /* device is not sm_100, or dtype/shape has no kernel      */
#define ZCMOE_ETIMEOUT (-6)     /* a device-side wait gave up (reported by zcmoe_check)    */

typedef struct zcmoe_s *zcmoe_t;

typedef enum { ZCMOE_F32 = 0, ZCMOE_BF16 = 1, ZCMOE_FP8 = 2, ZCMOE_FP4 = 3, ZCMOE_NVFP4 = 4 } zcmoe_dtype;

/* Layer shape and routing constants.  Sizes are element counts.
 * Limits: 1 <= n_ffn, 0 <= n_zero, E = n_ffn + n_zero <= 1024, 1 <= top_k <= min(E, 32),
 * d and inter multiples of 64, 1 <= max_tokens <= 2^20.
 * dtype: ZCMOE_BF16 -> x, y, all weights bf16, fp32 accumulation (tensor cores);
 *        ZCMOE_F32  -> everything fp32 with fp32 CUDA-core arithmetic (no TF32);
 *        ZCMOE_FP8  -> x, y and all weights bf16 at the interface, FFN experts on
 *                      block-scaled FP8 (technical summary, 六 定制內核 "量化": DeepSeek-V3's
 *                      blocks, one scale per [1,128] of activations and per [128,128]
 *                      of weights): E4M3 codes, power-of-two E8M0 scales (the
 *                      smallest 2^E with block max <= 448 * 2^E), fp32 accumulation.
 *                      zcmoe_create quantizes the expert weights into memory of its
 *                      own and reads w_gate / w_up / w_down only then; x rows are
 *                      quantized per [1,128] on the way into the gate/up GEMM and
 *                      silu(g)*u per [1,128] before the down GEMM; the router, the
 *                      combine and y stay bf16.  Needs d a multiple of 512 and inter
 *                      a multiple of 128;
 *        ZCMOE_FP4  -> as ZCMOE_FP8 with W4A4 experts (a LongCat-Flash news page,
 *                      gate.com post: expert weights and activations in 4 bits; the
 *                      format is not named): MXFP4, E2M1 codes with one E8M0 scale
 *                      (the smallest 2^E with block max <= 6 * 2^E) per 32 elements
 *                      along the reduction dimension of x, silu(g)*u and every weight
 *                      row.  Needs d a multiple of 512 and inter a multiple of 256;
 *        ZCMOE_NVFP4 -> the same W4A4 experts in NVFP4: E2M1 codes with one UE4M3
 *                      scale (an unsigned E4M3 value) per 16 elements along the
 *                      reduction dimension and one fp32 scale g per tensor
 *                      (zcmoe_quantize_nv4 gives the rule): g = amax / 2688 for
 *                      each expert's W_g, W_u and W_d (computed at create), g = 1
 *                      for x rows and silu(g)*u rows.  Same shape limits as ZCMOE_FP4. */
typedef struct {
  int32_t d;            /* hidden size                                   */
  int32_t n_ffn;        /* N, FFN experts                                */
  int32_t n_zero;       /* Z, zero-computation experts                   */
  int32_t inter;        /* FFN expert intermediate size                  */
  int32_t top_k;        /* experts chosen per token                      */
  int32_t max_tokens;   /* largest T accepted by zcmoe_forward           */
  int32_t dtype;        /* zcmoe_dtype                                   */
  float routed_scale;   /* gate = routed_scale * score (the "scaling" of the fused router); finite; 1.0 if unsure */
  const float *init_bias;    /* host [E] or NULL (zeros); copied at create; also the controller's b0 */
  const float *logit_offset; /* host [E] or NULL; copied; added to every token's logits before softmax */
} zcmoe_config;

/* Device weight pointers, BORROWED: the caller keeps them alive and unchanged
 * until zcmoe_destroy.  Element type = config dtype.  16-byte aligned.
 *   w_router [E, d]; w_gate [N, inter, d]; w_up [N, inter, d]; w_down [N, d, inter]. */
typedef struct {
  const void *w_router;
  const void *w_gate;
  const void *w_up;
  const void *w_down;
} zcmoe_weights;

/* Controller gains (the pages give none; see zcmoe_update_bias). */
typedef struct {
  float kp, ki, kd;
  float decay;                /* eta <- eta * decay before every step (eta starts at 1) */
  float target_ffn_per_token; /* K: target mean number of FFN experts per token, 0 <= K <= top_k */
} zcmoe_gains;

/* Optional device outputs of one forward, for tests and inspection; any field
 * may be NULL.  Shapes: logits/scores [T, E] fp32, idx [T, k] int32 (expert id,
 * slot order = biased score descending then id ascending), gate [T, k] fp32,
 * counts [E] int32, offsets [N+1] int32 (exclusive scan of FFN counts; offsets[N] = P),
 * perm [T*k] int32 (first P entries valid: FFN pairs t*k+j ordered by expert then
 * token), pos [T, k] int32 (row of pair (t,j) in the permuted order, -1 for zero experts),
 * expert_out [T*k, d] config dtype, bf16 for ZCMOE_FP8 / ZCMOE_FP4 (first P rows valid: the FFN expert outputs F_e(x_t),
 * one row per pair in the permuted order, before gating). */
typedef struct {
  float *logits;
  float *scores;
  int32_t *idx;
  float *gate;
  int32_t *counts;
  int32_t *offsets;
  int32_t *perm;
  int32_t *pos;
  void *expert_out;
} zcmoe_debug;

/* Creates a layer handle: validates shapes and alignment, allocates the handle's
 * device state (bias, controller state and accumulators, workspace for
 * max_tokens), and builds the TMA descriptors of the weights.  Requires the
 * current device to be sm_100.  On error *out is left NULL. */
ZCMOE_API int zcmoe_create(const zcmoe_config *cfg, const zcmoe_weights *w, zcmoe_t *out);

/* One forward pass over T tokens (zhangjingwei.cn 二.1; onthewifi.com part 02):
 * x [T, d] device (config dtype) -> y [T, d] device (config dtype), y must not
 * overlap x.  Also adds this batch's per-expert selection counts and T to the
 * controller accumulators.  T == 0 is a no-op.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_forward(zcmoe_t h, const void *x, int64_t T, void *y, cudaStream_t stream, const zcmoe_debug *dbg);

/* The same forward pass from and to HOST memory.  x [T, d] (host) is copied into
 * one of two handle-owned device staging buffers on an internal copy stream (so
 * the upload for the next call overlaps this call's compute), `stream` waits for
 * it, runs zcmoe_forward, and copies y [T, d] back to host memory on `stream`.
 * The staging buffers (3 x max_tokens x d elements) and the copy stream are
 * created on the first call.  Use page-locked host buffers so the copies are
 * asynchronous; x_host may be reused once `stream` has passed this call's
 * forward, and y_host is complete once `stream` has been synchronised. */
ZCMOE_API int zcmoe_forward_host(zcmoe_t h, const void *x_host, int64_t T, void *y_host, cudaStream_t stream);

/* The same, pipelined over calls: the download of this call's y runs on an internal stream
 * beside the NEXT call's forward (and its upload beside the previous call's), so a loop of
 * calls overlaps both copies with the compute.  y_host is complete once `stream` has passed
 * the next zcmoe_forward_host_async / zcmoe_forward_host on this handle, or a
 * zcmoe_forward_host_flush; keep it untouched until then.  x_host may be reused once
 * `stream` has passed this call's forward. */
ZCMOE_API int zcmoe_forward_host_async(zcmoe_t h, const void *x_host, int64_t T, void *y_host, cudaStream_t stream);
/* Makes `stream` wait for the download of the last zcmoe_forward_host_async. */
ZCMOE_API int zcmoe_forward_host_flush(zcmoe_t h, cudaStream_t stream);

/* One bias-controller step (zhangjingwei.cn 二.1 "PID controller"; web3.cnouyi.fund
 * "decay schedule"), fp32 with every operation rounded once:
 *   load l_i = c_i / T_acc from the accumulated counts; target tau_i = K/N for FFN
 *   experts, (k-K)/Z for zero experts; e_i = tau_i - l_i; eta <- eta*decay;
 *   I_i <- I_i + eta*e_i; b_i <- ((kp*eta*e_i + ki*I_i) + kd*eta*(e_i - e_prev_i)) + b0_i;
 *   e_prev_i <- e_i; the accumulators are reset.  No-op while T_acc == 0.
 * kp, ki, kd and decay must be finite and 0 <= K <= top_k (K = top_k without zero
 * experts), else ZCMOE_EINVAL with nothing enqueued.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_update_bias(zcmoe_t h, const zcmoe_gains *g, cudaStream_t stream);

/* Data-parallel exchange of the accumulators.  read: copies the handle's
 * accumulators into dst [E+1] int64 device (counts, then T_acc); write: replaces
 * them with src [E+1].  A replica group sums the read buffers (all-reduce) and
 * writes the sum back before zcmoe_update_bias, so every replica takes the same
 * bit-exact controller step.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_read_counts(zcmoe_t h, int64_t *dst, cudaStream_t stream);
ZCMOE_API int zcmoe_write_counts(zcmoe_t h, const int64_t *src, cudaStream_t stream);

/* Host copies of the controller state (any pointer may be NULL): bias [E] fp32,
 * accumulated counts [E] int64, accumulated tokens [1] int64, eta [1] fp32.
 * Synchronises the device. */
ZCMOE_API int zcmoe_get_state(zcmoe_t h, float *bias, int64_t *counts, int64_t *tokens, float *eta);

/* Replaces the bias (host [E] fp32).  Does not change b0 or the controller state.  Synchronous. */
ZCMOE_API int zcmoe_set_bias(zcmoe_t h, const float *bias);

/* The whole mutable state of the bias controller, for checkpoint and resume (the
 * PID of zcmoe_update_bias; LongCat-Flash technical summary, 二.1 "計算預算控制").
 * All host pointers:
 *   bias [E] fp32    the current bias;
 *   integ [E] fp32   the PID's integral I;
 *   eprev [E] fp32   the previous step's error;
 *   eta [1] fp32     the decayed step factor;
 *   counts [E] int64, tokens [1] int64   the selections accumulated since the last step.
 * zcmoe_get_controller fills every non-NULL pointer; it synchronises the device.
 * zcmoe_set_controller replaces all six (none may be NULL; counts and tokens must be
 * >= 0 and eta finite, else ZCMOE_EINVAL with nothing changed); synchronous.
 * b0, the initial bias the PID adds, is fixed at create from init_bias.  A handle
 * created with the same init_bias and given another handle's controller state takes
 * bit-identical controller steps from there on. */
ZCMOE_API int zcmoe_get_controller(zcmoe_t h, float *bias, float *integ, float *eprev, float *eta, int64_t *counts,
                                   int64_t *tokens);
ZCMOE_API int zcmoe_set_controller(zcmoe_t h, const float *bias, const float *integ, const float *eprev,
                                   const float *eta, const int64_t *counts, const int64_t *tokens);

/* Synchronises the device and reports a device-side timeout (ZCMOE_ETIMEOUT) if a
 * kernel's bounded wait gave up since the last check; clears the flag. */
ZCMOE_API int zcmoe_check(zcmoe_t h);

/* Failure-detection self-test: launches one kernel that waits, through the same
 * bounded-wait routine the pipelined kernels use, on a barrier that nothing
 * releases, so the wait gives up after limit_ns (1e3 .. 1e9) and records a
 * timeout.  A later zcmoe_check then returns ZCMOE_ETIMEOUT (site 99) and the
 * context stays usable.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_selftest_wait(zcmoe_t h, int64_t limit_ns, cudaStream_t stream);

/* Stage timing for measurement.  zcmoe_profile_begin starts recording CUDA
 * events between the stages of every later zcmoe_forward on this handle;
 * zcmoe_profile_end synchronises, writes per-stage device time summed over the
 * recorded forwards into ms[ZCMOE_NUM_STAGES] (host) and the number of forwards
 * into *n_forwards, and stops recording.  Stages, in order: router GEMM,
 * softmax/top-k, integer stage, the copy of the FFN pairs' rows into expert order
 * (quantized for FP8 / FP4 layers), gate/up GEMM, down GEMM, combine. */
#define ZCMOE_NUM_STAGES 7
ZCMOE_API int zcmoe_profile_begin(zcmoe_t h);
ZCMOE_API int zcmoe_profile_end(zcmoe_t h, float *ms, int32_t *n_forwards);

/* Routing stage without any device allocation (the pages have no counterpart:
 * this is an interface for callers, not a step of the method).
 *
 * For callers that cannot call cudaMalloc: code running inside a framework's
 * memory pool or under a fixed device-memory budget, where a raw allocation
 * would bypass the pool or exceed the budget, and latency-critical loops where
 * cudaMalloc/cudaFree could synchronise the device.  No handle is needed.
 *
 * Computes, from caller-owned device buffers, exactly what zcmoe_forward's
 * routing stage computes: scores = softmax(logits) over E = n_ffn + n_zero
 * experts, top-k on score + bias (ties to the lower id), gate = routed_scale *
 * score, then counts [E], offsets [n_ffn+1], perm [T*k] (first offsets[n_ffn]
 * entries valid) and pos [T, k], with the layouts of zcmoe_debug.
 *   logits [T, E] fp32, bias [E] fp32 (inputs); idx, gate [T, k]; counts,
 *   offsets, perm, pos (outputs).  All device pointers, all caller-owned.
 *
 * Its only scratch is one fixed 1 MiB device array inside the library
 * (reserved on every GPU that loads it, until the process exits).  A call needs
 * align8(ceil(T/256) * E * 4) + (E+1) * 8 + (n_ffn+5) * 4 bytes of it; larger
 * requests return ZCMOE_ERANGE with the largest allowed T in zcmoe_last_error()
 * (E = 768 with 512 FFN experts allows T <= 86,528; E = 96 with 64 FFN experts
 * allows T <= 698,112).  routed_scale must be finite (ZCMOE_EINVAL otherwise).
 * Every argument check happens before anything is enqueued.  The first call on
 * each device looks up the array's device address (with that device current)
 * and caches it with the device's current context; a call in a new context (for
 * example after cudaDeviceReset) looks it up again.  Make a device's first call
 * before any stream capture.  All calls share the array and it keeps
 * the previous call's contents (whatever must start at zero is cleared on each
 * call), so calls whose executions can overlap on the GPU (for example on two
 * streams) race with each other: order them on one stream or synchronise
 * between them.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_route_noalloc(const float *logits, const float *bias, int64_t T, int32_t n_ffn, int32_t n_zero,
                                  int32_t top_k, float routed_scale, int32_t *idx, float *gate, int32_t *counts,
                                  int32_t *offsets, int32_t *perm, int32_t *pos, cudaStream_t stream);

/* Frees the handle's own memory; never touches the borrowed weights.  NULL is a no-op. */
ZCMOE_API int zcmoe_destroy(zcmoe_t h);

/* Backward pass of the last zcmoe_forward on this handle (training), bf16 layers.
 * LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the weight
 * gradients use a fused GemmAdd (each GEMM adds its fp32 product into the
 * gradient accumulator in its epilogue) and the input gradient a deterministic
 * ScatterAdd (a per-token sum in slot order: the same bits on every run).
 * The chain rule runs through the forward with its routing held fixed (the
 * selection is not differentiable); the bias only selects and gets no
 * gradient, nor does the logit offset.
 *   x  [T, d] device bf16: the tensor the last forward read, unchanged;
 *   dy [T, d] device bf16: the gradient of the loss with respect to y;
 *   dx [T, d] device bf16: written;
 *   g_router [E, d], g_gate [N, inter, d], g_up [N, inter, d], g_down [N, d, inter]:
 *      device fp32 accumulators, caller-owned; the gradients are ADDED into them;
 *      NULL skips that weight gradient.
 * T must equal the last forward's T.  The first call allocates the backward's
 * workspace (about (6 d + 4 inter) * 2 bytes per padded row plus [T, E] and
 * [T, d] buffers).  Returns ZCMOE_EUNSUPPORTED for FP32 / FP8 / FP4 layers.
 * Asynchronous on `stream`. */
ZCMOE_API int zcmoe_backward(zcmoe_t h, const void *x, const void *dy, int64_t T, void *dx, float *g_router,
                             float *g_gate, float *g_up, float *g_down, cudaStream_t stream);

/* zcmoe_backward with flags.  ZCMOE_GRAD_OVERWRITE: the weight gradients are WRITTEN into
 * g_router / g_gate / g_up / g_down instead of added (the epilogue stores its product; an expert
 * that no token picked gets zeros), so the accumulators are not read: half the HBM traffic of the
 * weight gradients, for the first micro-batch of an accumulation.  Other bits: ZCMOE_EINVAL. */
#define ZCMOE_GRAD_OVERWRITE 1u
ZCMOE_API int zcmoe_backward_ex(zcmoe_t h, const void *x, const void *dy, int64_t T, void *dx, float *g_router,
                                float *g_gate, float *g_up, float *g_down, uint32_t flags, cudaStream_t stream);

/* Training mode for zcmoe_backward, bf16 layers.  on = 1: every later forward also
 * stores the gate/up GEMM's outputs G = X W_g^T and U = X W_u^T of its FFN pairs
 * (rounded to bf16; 4 * inter bytes per padded pair row, allocated here, about
 * 2.1 GB at T 16384, k 12, 512 experts, inter 2048), and a backward after such a
 * forward reads them instead of recomputing them (one GEMM fewer: the SwiGLU
 * backward runs in the dH GEMM's epilogue).  on = 0: forwards store nothing and
 * the backward recomputes G and U; the buffer is freed.  Call it outside stream
 * capture, with no forward or backward of this handle in flight.  Returns
 * ZCMOE_EUNSUPPORTED for FP32 / FP8 / FP4 layers, ZCMOE_ENOMEM if the buffer
 * cannot be allocated (training mode then stays off). */
ZCMOE_API int zcmoe_save_for_backward(zcmoe_t h, int32_t on);

/* ---------------------------------------------------------------- expert parallelism
 * LongCat-Flash technical summary (zhangjingwei.cn), 五 訓練基礎設施: the FFN layers are
 * partitioned by expert across an EP group (no tensor parallelism).  Rank r of an EP group of
 * ep_size ranks holds FFN experts [r * n_local, (r + 1) * n_local), n_local = n_ffn / ep_size;
 * every rank routes its own tokens over all n_ffn + n_zero experts.  A forward is three calls
 * with two exchanges between them, which the caller runs (NCCL all-to-all, for example):
 *   1. zcmoe_ep_dispatch: routing and the copy of the FFN pairs' rows into expert order,
 *      so the rows for rank r are the contiguous block of its experts;
 *   exchange the per-expert counts and the rows (rank r gets its experts' rows);
 *   2. zcmoe_ep_experts: the local experts on the received rows;
 *   exchange the outputs back (the reverse of the row exchange);
 *   3. zcmoe_ep_combine: the gate-weighted sum on the token's rank.
 * Zero-computation experts need no weights: their picks never leave the token's rank
 * (the combine adds them from x).  The bias controller counts every rank's own picks
 * (zcmoe_read_counts / zcmoe_write_counts sum them over the group, as with data
 * parallelism).  bf16 layers; zcmoe_forward, zcmoe_backward and zcmoe_save_for_backward
 * return ZCMOE_EUNSUPPORTED on a handle with ep_size > 1. */

/* Like zcmoe_create, for rank ep_rank of an EP group of ep_size ranks: `local` holds the
 * router's full [E, d] weights and this rank's experts only (w_gate, w_up [n_local, inter, d],
 * w_down [n_local, d, inter], borrowed).  max_recv_rows bounds the rows one zcmoe_ep_experts
 * call takes (its workspace is max(max_tokens * top_k, max_recv_rows) rows of d + inter + d
 * bf16 values).  n_ffn must be a multiple of ep_size; ep_size > 1 needs ZCMOE_BF16. */
ZCMOE_API int zcmoe_create_ep(const zcmoe_config *cfg, const zcmoe_weights *local, int32_t ep_rank, int32_t ep_size,
                              int64_t max_recv_rows, zcmoe_t *out);

/* Stage 1.  x [T, d] device bf16.  Writes xsend [T * top_k, d] device bf16 (caller-owned; the
 * first P rows are the FFN pairs' rows, sorted by expert, then token, then slot) and offsets
 * [n_ffn + 1] device int32 (expert e's rows are [offsets[e], offsets[e+1]); P = offsets[n_ffn]).
 * Keeps the routing for zcmoe_ep_combine and adds the counts to the controller's accumulators.
 * dbg (nullable) receives this chunk's routing as zcmoe_forward's does (expert_out is not
 * written).  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_ep_dispatch(zcmoe_t h, const void *x, int64_t T, void *xsend, int32_t *offsets,
                                cudaStream_t stream, const zcmoe_debug *dbg);

/* Stage 2.  xrecv [P_recv, d] device bf16: the rows received from the ep_size source ranks in rank
 * order, each source's rows grouped by this rank's local experts in expert order; counts
 * [ep_size * n_local] HOST int32: counts[s * n_local + e] = the rows source s sent for local
 * expert e (they must sum to P_recv <= max(max_tokens * top_k, max_recv_rows)).  Writes yrecv
 * [P_recv, d] device bf16: row q = the expert's output for row q of xrecv.  Reads `counts` before
 * returning; the computation is asynchronous on `stream` (the call waits for the previous call's
 * upload of the row layout). */
ZCMOE_API int zcmoe_ep_experts(zcmoe_t h, const void *xrecv, const int32_t *counts, int64_t P_recv, void *yrecv,
                               cudaStream_t stream);

/* Stage 3.  x [T, d] device bf16: the tokens of the last dispatch; yback [P, d] device bf16: the
 * expert outputs in xsend's row order.  Writes y [T, d] device bf16.  T must equal the last
 * dispatch's.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_ep_combine(zcmoe_t h, const void *x, const void *yback, int64_t T, void *y, cudaStream_t stream);

/* Block quantization to FP8 E4M3 with E8M0 scales, the rule ZCMOE_FP8 layers use
 * (round to nearest even; scale 2^E the smallest power of two with the block's
 * largest magnitude <= 448 * 2^E, E + 127 clamped to [0, 254]; an all-zero block
 * takes 2^0).  No handle needed.
 *   src [rows, cols] device, ZCMOE_BF16 or ZCMOE_F32 (src_dtype), 16-byte aligned;
 *   cols a positive multiple of 128; block_rows 1 ([1,128] blocks) or 128
 *   ([128,128] blocks; the last row block may be partial);
 *   codes [rows, cols] uint8 device; scales [ceil(rows / block_rows), cols / 128]
 *   uint8 device (E8M0 bytes).  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_quantize_e4m3(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, int32_t block_rows,
                                  uint8_t *codes, uint8_t *scales, cudaStream_t stream);

/* MXFP4 quantization, the rule ZCMOE_FP4 layers use: E2M1 codes (0, 0.5, 1, 1.5, 2,
 * 3, 4, 6), round to nearest even, saturating at 6; one E8M0 scale per 32
 * consecutive elements of a row, the smallest power of two 2^E with the block's
 * largest magnitude <= 6 * 2^E (E + 127 clamped to [0, 254]; 2^0 for an all-zero
 * block).  No handle needed.
 *   src [rows, cols] device, ZCMOE_BF16 or ZCMOE_F32, 16-byte aligned; cols a
 *   positive multiple of 256; codes [rows, cols / 2] uint8 device, two codes per
 *   byte with the even element in the low nibble; scales [rows, cols / 32] uint8
 *   device.  Asynchronous on `stream`. */
ZCMOE_API int zcmoe_quantize_mx4(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, uint8_t *codes,
                                 uint8_t *scales, cudaStream_t stream);

/* NVFP4 quantization, the rule ZCMOE_NVFP4 layers use: value = e2m1 * s * g, with E2M1
 * codes as in zcmoe_quantize_mx4, one UE4M3 block scale s per 16 consecutive elements
 * of a row and one fp32 tensor scale g.  s is the smallest positive E4M3 value with
 * the block's largest magnitude amax <= 6 s g, decided in fp32 on
 * t = fl32(amax / fl32(6 g)) (448 at most; 1.0 for an all-zero block); the codes are
 * e2m1(fl32(x * fl32(1 / fl32(s g)))), round to nearest even, saturating at 6.
 * The pages report W4A4 without naming a format; this two-level scale is the
 * NVFP4 reading, kept beside MXFP4.  No handle needed.
 *   src [rows, cols] device, ZCMOE_BF16 or ZCMOE_F32, 16-byte aligned; cols a
 *   positive multiple of 256;
 *   global_scale: g > 0 (finite) to quantize under that scale (activations use 1);
 *   0 to derive it as the layer does for a weight matrix, g = fl32(amax(src) / 2688)
 *   (so the largest block scale is 448; 1 for an all-zero tensor), written to
 *   global_out (one float, device, required then; ignored otherwise);
 *   codes [rows, cols / 2] uint8 device, two codes per byte with the even element in
 *   the low nibble; scales [rows, cols / 16] uint8 device (E4M3 bytes).
 *   Asynchronous on `stream`. */
ZCMOE_API int zcmoe_quantize_nv4(const void *src, int32_t src_dtype, int64_t rows, int64_t cols, float global_scale,
                                 uint8_t *codes, uint8_t *scales, float *global_out, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Dense FFN path and the shortcut-connected overlap (ScMoE).
 *
 * LongCat-Flash technical summary (zhangjingwei.cn), 二 架構 part 2 "快捷連接 MoE":
 * the first MLA block's output goes straight to the MoE block, so the dense FFN
 * of the preceding block does not wait for the MoE layer and the two can run at
 * the same time; 五 訓練基礎設施 "ScMoE結構和分塊" and 六 推理與部署 (single-batch
 * overlap) use that window to hide the MoE's dispatch/combine traffic.  模型配置:
 * the dense path is 12288 wide on the 6144 hidden size.
 *
 * The dense FFN is y = W_down (silu(W_gate x) * (W_up x)), the form of an FFN
 * expert (the pages do not name the dense path's activation): bf16 operands,
 * fp32 accumulation on the tensor cores, the SwiGLU product rounded once to
 * bf16 before the down projection, y rounded once to bf16. */
typedef struct zcmoe_dense_s *zcmoe_dense_t;

/* d and inter positive multiples of 64; 1 <= max_tokens <= 2^20.  bf16 only. */
typedef struct {
  int32_t d;
  int32_t inter;
  int32_t max_tokens;
} zcmoe_dense_config;

/* Device pointers, bf16, 16-byte aligned, borrowed (not copied) until
 * zcmoe_dense_destroy: w_gate [inter, d], w_up [inter, d], w_down [d, inter]. */
typedef struct {
  const void *w_gate;
  const void *w_up;
  const void *w_down;
} zcmoe_dense_weights;

/* Checks the shapes, allocates the intermediate [max_tokens, inter] bf16 and
 * the internal stream and events that zcmoe_forward_overlap uses, and builds
 * the weights' TMA descriptors.  Requires sm_100.  On error *out is left NULL. */
ZCMOE_API int zcmoe_dense_create(const zcmoe_dense_config *cfg, const zcmoe_dense_weights *w, zcmoe_dense_t *out);

/* x [T, d] device bf16 -> y [T, d] device bf16; y must not overlap x.  T == 0 is
 * a no-op.  Asynchronous on `stream`; one stream at a time per handle. */
ZCMOE_API int zcmoe_dense_forward(zcmoe_dense_t h, const void *x, int64_t T, void *y, cudaStream_t stream);

/* The MoE layer and the dense FFN over the same T tokens, run concurrently:
 *   y_moe = zcmoe_forward(moe, x_moe, T),  y_dense = zcmoe_dense_forward(dense, x_dense, T),
 * with results identical, bit for bit, to the two calls made one after the
 * other (the MoE's controller accumulators advance exactly as in zcmoe_forward).
 * The dense FFN runs on the dense handle's internal stream, forked from and
 * joined back into `stream`: its gate/up GEMM starts when the MoE router GEMM
 * has finished and runs beside the MoE's memory-bound stages (softmax/top-k,
 * integer stage, row copy); its down GEMM starts when the MoE down GEMM has
 * finished and runs beside the combine.  When the call returns, all the work of
 * both is ordered before anything later enqueued on `stream`, so the call can
 * be captured into a CUDA graph on `stream`.
 * Requires: both handles live, the MoE handle bf16, equal d, 0 <= T <= both
 * max_tokens, 16-byte aligned buffers; y_moe and y_dense overlap neither each
 * other nor x_moe / x_dense (x_moe == x_dense is allowed). */
ZCMOE_API int zcmoe_forward_overlap(zcmoe_t moe, zcmoe_dense_t dense, const void *x_moe, const void *x_dense,
                                    int64_t T, void *y_moe, void *y_dense, cudaStream_t stream);

/* ZCMOE_OK, or ZCMOE_ETIMEOUT if one of the dense handle's kernels gave up a
 * bounded wait since the last check (the flag is then cleared).  Synchronises
 * the device. */
ZCMOE_API int zcmoe_dense_check(zcmoe_dense_t h);

/* Frees the dense handle's own memory and stream; never touches the borrowed
 * weights.  NULL is a no-op. */
ZCMOE_API int zcmoe_dense_destroy(zcmoe_dense_t h);

/* Message for the last failing call on this thread ("" if none). */
ZCMOE_API const char *zcmoe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ZCMOE_H */
