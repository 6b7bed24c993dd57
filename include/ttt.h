/*
 * ttt.h - C ABI of the B200 (sm_100a) library for the chunked TTT-KVB fast-weight layer
 * and its rewrite as chunked linear attention.
 *
 * The layer (per batch element and head, row vectors; "Test-Time Training with KV Binding
 * Is Secretly Linear Attention", section 前置知识 / LaCT, and "Test-Time Training Done
 * Right" notes, section 2.1):
 *     phi(x) = silu(x W0) * (x W2),   f(x) = phi(x) W1,
 *     W0, W2 in R^{h x m}, W1 in R^{m x h}, m = r h,
 *     chunk loss  L_c = - sum_{i in chunk c} eta_i <f(k_i), v_i>.
 * Each chunk takes one gradient step (step size 1, eta inside the loss) from the
 * chunk-start weights; the chunk's queries then read f(q) with the updated weights
 * (TTT_ORDER_UPDATE_APPLY) or with the chunk-start weights (TTT_ORDER_APPLY_UPDATE,
 * "Test-Time Training Done Right" notes, section 2.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers are DEVICE pointers unless stated otherwise. Tensors are dense, row-major,
 * contiguous:
 *     q, k, v, out : [B, H, N, h]  element type ttt_desc.dtype (fp32 or bf16)
 *     eta          : [B, H, N]     fp32 per-token learning rate
 *     alpha        : [B, H, C]     fp32 per-chunk momentum factor, C = ceil(N / chunk)
 *     W0, W2       : [H, h, m]     fp32 (or [H, m, h] when w_in_layout = 1)
 *     W1           : [H, m, h]     fp32 (or [H, h, m] when w1_layout = 1)
 * Initial weights are per head and broadcast over the batch; every (batch, head) starts
 * from them (fast weights are reset per sequence). The last chunk may be shorter than
 * `chunk`. q == k (same pointer) is allowed: the query and key features are then
 * computed once.
 *
 * Ownership: the caller owns every buffer. The library allocates no device memory; the
 * scratch it needs lives in the caller's workspace (size from ttt_workspace_bytes). Work
 * is enqueued on the caller's stream and returns before it completes.
 *
 * Errors: arguments are checked on the host before anything is enqueued; a failed check
 * returns a status and enqueues nothing (no exceptions cross the ABI). A bounded wait
 * that runs out inside a kernel, or a failed debug check (ttt_set_debug_checks), is
 * recorded in a per-device error word; ttt_last_device_status() synchronises the stream,
 * reads and clears it. ttt_last_error_message() gives a human-readable detail of the
 * calling thread's last failure. In bf16 mode every contraction runs on the tensor cores;
 * a problem the tensor-core engine cannot take is refused with TTT_ERR_UNSUPPORTED (it is
 * never rerouted to another engine).
 *
 * Precision: in TTT_DTYPE_BF16 mode the dense contractions take bf16 operands (q, k, v,
 * the fp32 weights rounded to bf16, the features rounded to bf16) and accumulate in
 * fp32 on the tensor cores; states, weights, momentum and all elementwise math stay
 * fp32. Newton-Schulz, which bf16 operands would not keep within the parity tolerance,
 * runs its products on the tensor cores at more than bf16 operand precision: as three
 * bf16 terms hi*hi + hi*lo + lo*hi of split operands for matrices up to 128 x 256, as tf32
 * products of the fp32 matrices (10-bit mantissa) for larger ones. In TTT_DTYPE_FP32 mode
 * every step is fp32 on the CUDA cores.
 */
#ifndef TTT_B200_TTT_H_
#define TTT_B200_TTT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t. NULL selects the legacy default stream. */
typedef struct CUstream_st* ttt_stream_t;

typedef enum ttt_status {
  TTT_OK = 0,
  TTT_ERR_INVALID_ARG = 1,  /* a size, flag or pointer is invalid (see the message) */
  TTT_ERR_UNSUPPORTED = 2,  /* valid request the library does not implement */
  TTT_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or smaller than required */
  TTT_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  TTT_ERR_TIMEOUT = 5,      /* a bounded device-side wait ran out */
  TTT_ERR_DEVICE = 6        /* a debug check failed: a workspace guard was overwritten, or
                               an output holds NaN/Inf (see ttt_set_debug_checks) */
} ttt_status;

enum { TTT_DTYPE_FP32 = 0, TTT_DTYPE_BF16 = 1 };
enum { TTT_ORDER_UPDATE_APPLY = 0, TTT_ORDER_APPLY_UPDATE = 1 };
enum { TTT_UPDATE_W0 = 1, TTT_UPDATE_W1 = 2, TTT_UPDATE_W2 = 4, TTT_UPDATE_ALL = 7 };
enum {
  TTT_PATH_PARALLEL = 0,
  TTT_PATH_RECURRENT = 1,
  TTT_PATH_LINEAR = 2,
  TTT_PATH_PARALLEL_MOMENTUM = 3,
  TTT_PATH_PARALLEL_BWD = 4
};

/* Problem description. All fields are read; unused ones must be 0 unless noted. */
typedef struct ttt_desc {
  int32_t B;            /* batch size, >= 0 */
  int32_t H;            /* heads, >= 0 */
  int32_t N;            /* tokens per sequence, >= 0 */
  int32_t h;            /* head (input/output) width, >= 1 */
  int32_t m;            /* hidden width of the SwiGLU map, >= 1 */
  int32_t chunk;        /* tokens per update chunk, >= 1 */
  int32_t dtype;        /* TTT_DTYPE_FP32 or TTT_DTYPE_BF16 (q, k, v and out) */
  int32_t order;        /* TTT_ORDER_UPDATE_APPLY or TTT_ORDER_APPLY_UPDATE */
  int32_t sign;         /* +1 gradient descent, -1 gradient ascent */
  int32_t update_mask;  /* recurrent: which of W0/W1/W2 are fast (TTT_UPDATE_*) */
  int32_t renorm;       /* recurrent: 1 = per-column weight renormalisation */
  int32_t momentum;     /* recurrent: 1 = momentum M <- alpha_c M + g (needs alpha) */
  int32_t ns_steps;     /* recurrent: Newton-Schulz steps on each update, 0..8 */
  int32_t w_in_layout;  /* 0: W0, W2 are [H,h,m]; 1: they are [H,m,h] (e.g. gate/up) */
  int32_t w1_layout;    /* 0: W1 and S_final are [.,m,h]; 1: [.,h,m] (e.g. down proj) */
} ttt_desc;

/*
 * Workspace size in bytes for `path` (one of TTT_PATH_*), or 0 when the description is
 * invalid for that path. Host-only; touches no device.
 */
size_t ttt_workspace_bytes(const ttt_desc* desc, int32_t path);

/*
 * Parallel last-layer-only form ("Test-Time Training with KV Binding Is Secretly Linear
 * Attention", sections 方法步骤详情 (Theorem 5.2 and simplification steps 1-2) and
 * 前置知识 / 前缀扫描; "NVIDIA团队揭秘", section 四): W0, W2 frozen, no renormalisation,
 * so the features are static and the W1 updates are associative:
 *     Delta S_c = sign * phi(K_c)^T diag(eta_c) V_c,
 *     S_c = W1 + sum_{c' <= c} Delta S_c'   (update_apply; c' < c for apply_update),
 *     O_c = phi(Q_c) S_c.
 * With q == k, W0 = Wg^T, W2 = Wu^T, W1 = W_down^T, v = the target values and
 * apply_update this is the In-Place TTT chunk update ("In-Place Test-Time Training",
 * sections 3.1 and 3.4).
 *
 *   desc       problem; update_mask, renorm, momentum, ns_steps must be 0
 *   q, k, v    [B,H,N,h] dtype
 *   eta        [B,H,N] fp32
 *   W0, W2     per-head input-side weights (layout per w_in_layout), fp32
 *   W1         per-head initial state (layout per w1_layout), fp32
 *   out        [B,H,N,h] dtype, written
 *   S_final    nullable; [B,H,m,h] (or [B,H,h,m]) fp32 state after the last chunk
 *   workspace  >= ttt_workspace_bytes(desc, TTT_PATH_PARALLEL) bytes, 256-byte aligned
 */
ttt_status ttt_la_parallel_fwd(const ttt_desc* desc, const void* q, const void* k,
                               const void* v, const float* eta, const float* W0,
                               const float* W2, const float* W1, void* out,
                               float* S_final, void* workspace, size_t workspace_bytes,
                               ttt_stream_t stream);

/*
 * One contiguous shard of a sequence in the parallel form, for a sequence split over
 * devices (context parallelism: "In-Place Test-Time Training", section 3.4, the chunk
 * deltas of earlier shards enter a shard only through their sum; "Test-Time Training with
 * KV Binding Is Secretly Linear Attention", 前置知识 / 前缀扫描). The same computation as
 * ttt_la_parallel_fwd on the shard's tokens, except that the state the shard starts from
 * is, for every (batch, head),
 *     W1[head] (zero when W1 is NULL) + sum_{i < n_prior} prior[i, batch, head],
 * and that `out` may be NULL, in which case only S_final is formed (no query-side work).
 * A sequence over R shards: shard r calls this with W1 = NULL, out = NULL to get its total
 * delta T_r; the totals are gathered in rank order; shard r calls it again with W1,
 * prior = T_0 .. T_{r-1} (n_prior = r) and out: its outputs are those of the unsharded
 * call, and the last shard's S_final is the sequence's final state.
 *
 *   desc       as for ttt_la_parallel_fwd; every shard but the last must hold whole chunks
 *   W1         nullable; per-head initial state (layout per w1_layout)
 *   prior      [n_prior, B, H, m, h] fp32 (W1's layout per entry; 16-byte aligned), or
 *              NULL with n_prior = 0; n_prior <= 4096
 *   out        nullable [B,H,N,h] dtype; S_final nullable, but not both NULL
 *   workspace  >= ttt_workspace_bytes(desc, TTT_PATH_PARALLEL) bytes
 * Errors and streams as for ttt_la_parallel_fwd.
 */
ttt_status ttt_la_parallel_fwd_shard(const ttt_desc* desc, const void* q, const void* k,
                                     const void* v, const float* eta, const float* W0,
                                     const float* W2, const float* W1, const float* prior,
                                     int32_t n_prior, void* out, float* S_final, void* workspace,
                                     size_t workspace_bytes, ttt_stream_t stream);

/*
 * The outputs pass of a shard that reuses the key side of the state-only pass before it.
 * A state-only call of ttt_la_parallel_fwd_shard (out = NULL) leaves in its workspace the
 * blocked input weights and every chunk's delta; this call then forms the chunk states from
 * W1 + sum_{i < n_prior} prior[i] and those deltas, and the outputs, without recomputing
 * phi(K) (same section as above: the deltas do not depend on the initial state). So a
 * shard's two passes cost one key side, one scan each and one query side.
 *
 *   desc       identical to the state-only call's
 *   q          [B,H,N,h] dtype (the same tokens as the state-only call's k when q == k)
 *   W1, prior, n_prior, S_final   as for ttt_la_parallel_fwd_shard
 *   out        [B,H,N,h] dtype, not NULL
 *   workspace  the state-only call's workspace and size, untouched since
 * TTT_ERR_UNSUPPORTED when the problem takes the sequential schedule (its state-only pass
 * keeps no chunk deltas: call ttt_la_parallel_fwd_shard again with out instead);
 * TTT_ERR_INVALID_ARG unless the last ttt_la_parallel_fwd_shard call on this host thread
 * was a successful state-only call with the same descriptor, workspace and size (each
 * outputs pass consumes it). Streams as for ttt_la_parallel_fwd.
 */
ttt_status ttt_la_parallel_fwd_shard_outputs(const ttt_desc* desc, const void* q,
                                             const float* W1, const float* prior,
                                             int32_t n_prior, void* out, float* S_final,
                                             void* workspace, size_t workspace_bytes,
                                             ttt_stream_t stream);

/*
 * Parallel last-layer-only form with momentum and orthogonalisation of the W1 update
 * ("Test-Time Training with KV Binding Is Secretly Linear Attention", section 方法步骤详情:
 * simplification variant 2 keeps momentum and Newton-Schulz; the pages' recurrent -> parallel
 * throughput comparison is made on it). W0, W2 frozen and no renormalisation make each
 * chunk's W1 gradient independent of W1, so for all chunks at once
 *     D_c = sign * phi(K_c)^T diag(eta_c) V_c,
 *     M_c = alpha_c M_{c-1} + D_c            (momentum = 1; M_{-1} = 0; else M_c = D_c),
 *     U_c = NS_{ns_steps}(M_c)               (ns_steps > 0; else U_c = M_c),
 *     S_c = W1 + sum_{c' <= c} U_c'          (update_apply; c' < c for apply_update),
 *     O_c = phi(Q_c) S_c.
 * NS is the pages' iteration (coefficients 3.4445, -4.7750, 2.0315 on X = M / (||M||_F +
 * 1e-7), rows <= cols orientation). This equals the recurrent form with update_mask = W1,
 * the same momentum and ns_steps and no renormalisation.
 *
 *   desc       problem; update_mask and renorm must be 0; momentum 0 or 1; ns_steps 0..8;
 *              w1_layout 0
 *   alpha      [B,H,ceil(N/chunk)] fp32 momentum factors (needed when momentum = 1)
 *   other arguments as for ttt_la_parallel_fwd; workspace >=
 *   ttt_workspace_bytes(desc, TTT_PATH_PARALLEL_MOMENTUM)
 */
ttt_status ttt_la_parallel_momentum_fwd(const ttt_desc* desc, const void* q, const void* k,
                                        const void* v, const float* eta, const float* alpha,
                                        const float* W0, const float* W2, const float* W1,
                                        void* out, float* S_final, void* workspace,
                                        size_t workspace_bytes, ttt_stream_t stream);

/*
 * Backward pass of ttt_la_parallel_fwd (training; "Test-Time Training with KV Binding Is
 * Secretly Linear Attention", section 方法步骤详情: the parallel form is what makes the
 * layer trainable at scale). Given the gradient dout of the outputs (and optionally
 * dS_final of the final state), computes the gradients of every input by the chain rule
 * through O_c = phi(Q_c) S_c, S_c = W1 + sum Delta S_c' and Delta S_c = sign phi(K_c)^T
 * diag(eta_c) V_c. With R_c = dS_final + sum_{c' >= c} phi(Q_c')^T dO_c', the gradient of
 * Delta S_c is R_c (update_apply) or R_{c+1} (apply_update) and dW1 = R_0. The forward
 * quantities are recomputed, nothing is saved between the calls.
 *
 *   desc        as for ttt_la_parallel_fwd; default weight layouts only
 *   q, k, v, eta, W0, W2, W1   the forward inputs (q and k distinct)
 *   dout        [B,H,N,h] dtype
 *   dS_final    nullable; [B,H,m,h] fp32
 *   dq, dk, dv  [B,H,N,h] dtype, written (distinct buffers)
 *   deta        [B,H,N] fp32, written
 *   dW0, dW2    [H,h,m] fp32, dW1 [H,m,h] fp32, written (summed over the batch)
 *   workspace   >= ttt_workspace_bytes(desc, TTT_PATH_PARALLEL_BWD) bytes, 256-byte aligned
 * Errors and streams as for ttt_la_parallel_fwd.
 */
ttt_status ttt_la_parallel_bwd(const ttt_desc* desc, const void* q, const void* k,
                               const void* v, const float* eta, const float* W0,
                               const float* W2, const float* W1, const void* dout,
                               const float* dS_final, void* dq, void* dk, void* dv,
                               float* deta, float* dW0, float* dW2, float* dW1,
                               void* workspace, size_t workspace_bytes, ttt_stream_t stream);

/*
 * Parallel form with identity features: the end of the simplification ladder ("Test-Time
 * Training with KV Binding Is Secretly Linear Attention", section 方法步骤详情,
 * variants 3-6: the inner MLP reduced to one linear map, phi(x) = x), i.e. chunked linear
 * attention with a per-token step size:
 *     Delta S_c = sign * K_c^T diag(eta_c) V_c,
 *     S_c = S0 + sum_{c' <= c} Delta S_c'   (update_apply; c' < c for apply_update),
 *     O_c = Q_c S_c.
 *
 *   desc       problem; m must equal h; w_in_layout 0; update_mask, renorm, momentum,
 *              ns_steps must be 0
 *   q, k, v    [B,H,N,h] dtype
 *   eta        [B,H,N] fp32
 *   S0         per-head initial state [H,h,h] fp32 (transposed when w1_layout = 1)
 *   out        [B,H,N,h] dtype, written
 *   S_final    nullable; [B,H,h,h] fp32 state after the last chunk (S0's layout)
 *   workspace  >= ttt_workspace_bytes(desc, TTT_PATH_LINEAR) bytes, 256-byte aligned
 * Errors, streams and aliasing as for ttt_la_parallel_fwd.
 */
ttt_status ttt_linear_attn_fwd(const ttt_desc* desc, const void* q, const void* k,
                               const void* v, const float* eta, const float* S0, void* out,
                               float* S_final, void* workspace, size_t workspace_bytes,
                               ttt_stream_t stream);

/*
 * Parallel form for callers that cannot allocate device memory. No paper counterpart:
 * same arguments and results as ttt_la_parallel_fwd, minus the workspace. Some callers
 * have no way to obtain device memory of their own: a plug-in hosted by a runtime that
 * owns every device allocation and hands out none, or a real-time loop that must not call
 * cudaMalloc after start-up because an allocation can synchronise the device and stall
 * other streams. For them the scratch lives in one array built into the library,
 * TTT_STATIC_SCRATCH_BYTES (64 MiB) per device, reserved on every GPU that loads the
 * library until the process exits.
 *
 * - Problems whose workspace (ttt_workspace_bytes(desc, TTT_PATH_PARALLEL)) exceeds
 *   TTT_STATIC_SCRATCH_BYTES are rejected with TTT_ERR_WORKSPACE; nothing is enqueued.
 * - The first call on a device looks up that device's copy of the array (with that device
 *   current); make that first call before any stream capture begins.
 * - Every call on a device uses the same array. Calls whose work overlaps on the GPU
 *   (different streams, or different host threads, without ordering between them) race on
 *   it and give wrong results: order them. No state is carried from one call to the next;
 *   every scratch byte a call reads it has written earlier in the same call.
 * - Nothing is allocated: no cudaMalloc, no cudaFree, no allocating library routine.
 */
#define TTT_STATIC_SCRATCH_BYTES (64ull << 20)
ttt_status ttt_la_parallel_fwd_noalloc(const ttt_desc* desc, const void* q, const void* k,
                                       const void* v, const float* eta, const float* W0,
                                       const float* W2, const float* W1, void* out,
                                       float* S_final, ttt_stream_t stream);

/*
 * Recurrent LaCT form ("Test-Time Training Done Right" notes, sections 2.1-2.3; "Test-Time
 * Training with KV Binding Is Secretly Linear Attention", 前置知识 / LaCT): per chunk, at
 * the chunk-start weights, the gradients
 *     G = -diag(eta) V,  dW1 = phi^T G,  D = G W1^T,
 *     dW2 = K^T (D * silu(K W0)),  dW0 = K^T (D * (K W2) * silu'(K W0));
 * then for every fast matrix X (update_mask): optional momentum M_X <- alpha_c M_X + g_X
 * (M = 0 at the start), optional Newton-Schulz orthogonalisation of the update
 * (X = U / (||U||_F + 1e-7) in the orientation with rows <= cols, then ns_steps times
 * X <- 3.4445 X + (-4.7750 A + 2.0315 A^2) X with A = X X^T), the step
 * X <- X - sign * u, and optional renormalisation of each column (output unit) over the
 * input dimension to the column norm the matrix had at the start of the call.
 *
 *   desc       problem; w_in_layout and w1_layout must be 0; h, m <= 1536
 *   alpha      [B,H,C] fp32, required when desc->momentum, else ignored (may be NULL)
 *   W0, W2, W1 per-head initial weights [H,h,m], [H,h,m], [H,m,h] fp32
 *   out        [B,H,N,h] dtype, written
 *   W0_out, W2_out  nullable; [B,H,h,m] fp32 weights after the last chunk
 *   W1_out     nullable; [B,H,m,h] fp32
 *   M_io       nullable; [B,H,(h*m + m*h + h*m)] fp32 momentum (W0 part [h,m], then W1
 *              part [m,h], then W2 part [h,m]); read as the initial momentum and
 *              overwritten with the final one. NULL means "start from 0, discard".
 *   workspace  >= ttt_workspace_bytes(desc, TTT_PATH_RECURRENT) bytes, 256-byte aligned
 *
 * Streams: with more than one chunk, part of the work (each chunk's outputs and the W1
 * gradient) runs on a second stream that the library creates once per host thread and
 * device; it forks from `stream` with events and is joined back into `stream` before the
 * call returns, on error paths too. Everything the call enqueues is therefore ordered
 * before later work on `stream`, and the call can be captured into a CUDA graph from
 * `stream` (the fork and join become graph dependencies). If the second stream cannot be
 * created, all work stays on `stream`.
 */
ttt_status ttt_lact_recurrent_fwd(const ttt_desc* desc, const void* q, const void* k,
                                  const void* v, const float* eta, const float* alpha,
                                  const float* W0, const float* W2, const float* W1,
                                  void* out, float* W0_out, float* W2_out, float* W1_out,
                                  float* M_io, void* workspace, size_t workspace_bytes,
                                  ttt_stream_t stream);

/*
 * LM-aligned value target ("In-Place Test-Time Training", section 3.2, eq. 3):
 *     Vbar = Conv1D(X0) W_target,  (Conv1D(X0))_t = sum_{j=0..3} conv_w[j] * X0[t-j]
 * (causal, depthwise, zero before the first token).
 *
 *   X0        [N,d] bf16 token embeddings
 *   conv_w    [4,d] fp32 taps (tap j multiplies X0[t-j])
 *   W_target  [d,d] bf16
 *   vbar      [N,d] bf16, written
 *   workspace >= ttt_lm_target_workspace_bytes(N, d) bytes, 256-byte aligned
 */
size_t ttt_lm_target_workspace_bytes(int32_t N, int32_t d);
ttt_status ttt_lm_target(int32_t N, int32_t d, const void* X0, const float* conv_w,
                         const void* W_target, void* vbar, void* workspace,
                         size_t workspace_bytes, ttt_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the device error word of the current
 * device: TTT_OK, TTT_ERR_TIMEOUT (a bounded wait ran out) or TTT_ERR_DEVICE (a debug
 * check failed, see ttt_set_debug_checks); or TTT_ERR_CUDA when the synchronisation itself
 * failed.
 */
ttt_status ttt_last_device_status(ttt_stream_t stream);

/*
 * Debug checks (no paper counterpart: the library's own stand-in for a device memory
 * checker). `flags` is a combination of
 *   TTT_CHECK_GUARDS  every region a call carves from its workspace gets a 256-byte guard
 *                     in front of the first region and right after each region's end;
 *                     ttt_workspace_bytes / ttt_lm_target_workspace_bytes grow to hold
 *                     them. Each call fills its guards with a fixed pattern before its
 *                     first kernel and compares them after its last one; a changed guard
 *                     (a write outside its region) sets the device error word.
 *   TTT_CHECK_FINITE  after its last kernel each call scans its outputs (out, final
 *                     states / weights, momentum, gradients) for NaN or Inf.
 * A failed check is reported by ttt_last_device_status as TTT_ERR_DEVICE, with the check
 * named in ttt_last_error_message. The checks never stop or fault a kernel; they cost
 * extra launches. The setting is process-wide; change it only while no call is in flight
 * and size workspaces after changing it (a workspace sized with guards off is too small
 * with guards on: TTT_ERR_WORKSPACE). Unknown flags: TTT_ERR_INVALID_ARG.
 */
enum { TTT_CHECK_GUARDS = 1, TTT_CHECK_FINITE = 2 };
ttt_status ttt_set_debug_checks(int32_t flags);
int32_t ttt_get_debug_checks(void);

/*
 * Compares, now (enqueued on `stream`), the guards of a workspace that a call with the
 * same `desc` and `path` planned with TTT_CHECK_GUARDS on; a changed guard is reported by
 * the next ttt_last_device_status. TTT_ERR_INVALID_ARG when guards are off.
 */
ttt_status ttt_debug_check_workspace(const ttt_desc* desc, int32_t path, void* workspace,
                                     size_t workspace_bytes, ttt_stream_t stream);

/*
 * Diagnostic for the failure path: launches one block that waits on a barrier nobody
 * arrives at, giving up after `timeout_ns` nanoseconds (1e5 .. 1e10). The wait records
 * TTT_ERR_TIMEOUT in the device error word and the kernel returns normally, so the
 * context stays usable. No paper counterpart: it exercises the library's own bounded
 * waits.
 */
ttt_status ttt_debug_wait_timeout(int64_t timeout_ns, ttt_stream_t stream);

/*
 * Kernel tracing (no paper counterpart; the library's own profiling hook). After
 * ttt_trace_enable(capacity), every kernel the library enqueues, on the current device, is
 * bracketed by two CUDA events recorded on the stream it is launched on, until
 * `capacity` kernels have been recorded. The events are created here (host-side CUDA
 * objects, no device memory). ttt_trace_count() gives the number recorded;
 * ttt_trace_get(i, ...) waits for record i to complete and returns a static kernel name
 * and its duration in milliseconds. ttt_trace_disable() stops recording and releases the
 * events. Tracing is process-wide and not meant for concurrent callers.
 */
ttt_status ttt_trace_enable(int32_t capacity);
ttt_status ttt_trace_disable(void);
int32_t ttt_trace_count(void);
ttt_status ttt_trace_get(int32_t index, const char** kernel_name, float* milliseconds);

/* Static, never NULL. */
const char* ttt_status_str(ttt_status status);

/* Detail of the calling thread's last non-OK status ("" if none). Static storage. */
const char* ttt_last_error_message(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int32_t ttt_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTT_B200_TTT_H_ */
