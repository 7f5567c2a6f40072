/*
 * wkv.h -- C ABI of libwkv, the RWKV-4 WKV time-mixing operator on NVIDIA
 * B200 (sm_100a).
 *
 * The operator (RWKV paper review, "[논문 리뷰] Reinvention RNNs for the
 * Transformer Era: RWKV", section "WKV 연산자", eq. wkv_t; 0-based t, decay
 * written as the signed per-step log-decay w, normally w = -exp(time_decay)):
 *
 *   y_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *       / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     )
 *
 * independently for every batch row b and channel c (w, u are per channel).
 * Its RNN form (same review, section "RNN-유사추론", eq. WKV_t) keeps per
 * channel the hidden sums A_t = sum_{i<t} e^{(t-1-i) w + k_i} v_i and
 * B_t = sum_{i<t} e^{(t-1-i) w + k_i}, so y_t = (A_t + e^{u+k_t} v_t) /
 * (B_t + e^{u+k_t}) and A_{t+1} = e^w A_t + e^{k_t} v_t (same for B).
 *
 * Three calls follow the review's two execution modes:
 *   wkv_forward   time-parallel mode ("Transformer-유사학습": the whole
 *                 sequence at once, WKV evaluated as a scan over time);
 *   wkv_backward  gradients of a scalar loss for the same mode;
 *   wkv_step      RNN mode ("RNN-유사추론" / "자기 회귀 디코딩" steps 4 and 7):
 *                 one token per sequence against a stored state.
 * wkv_token_shift forms the operator's inputs' time interpolation (the
 * "토큰 변환" token shift), and its backward.
 * wkv_backward_state adds the gradients through the recurrent state for
 * sequences split across calls; wkv_forward_gated / wkv_backward_gated add
 * the receptance gate o = sigma(r) * y of the time-mixing block's output.
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *   allocates and frees nothing; scratch lives in a caller-provided
 *   workspace.  One exception: wkv_backward_static keeps its scratch in a
 *   file-scope device array of the library (see there).  Between calls the
 *   library caches, per device, the occupancy of its kernels, the TMA
 *   tensor maps it encoded for recently used buffers (keyed by address,
 *   shape and element type, so a buffer reused with another shape gets a
 *   new map) and that array's set-up; nothing else is kept.
 * - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *   NULL = legacy default stream).  The return value covers host-side
 *   argument checks and the launch itself; conditions detected on the device
 *   (a bounded wait that gave up) are read later with wkv_get_status().
 *   A call that returns an error has launched nothing, except WKV_ERR_CUDA,
 *   which reports a failed launch.
 * - Layout: k, v, y, grad_y, grad_k, grad_v (and r, o, grad_o, grad_r of
 *   the gated calls) are [B, T, C] row-major with C
 *   fastest (the (B, T, d) layout of the sequence model); w, u, grad_w,
 *   grad_u are [C] float32.
 * - Element type of k, v, y, grad_y, grad_k, grad_v: WKV_F32 or WKV_BF16
 *   (bfloat16 storage, float32 arithmetic, round-to-nearest-even stores).
 *   w, u, states, checkpoints and parameter gradients are always float32.
 * - State: three float32 planes [3][B][C] holding (a, b, p) per (b, c), with
 *   A = a * e^p and B = b * e^p.  The form is not unique; any (a, b, p) with
 *   b >= 0 is accepted.  The empty state is (0, 0, -inf); p = -inf is
 *   accepted as input.  State outputs are normalised so that p is the
 *   largest exponent seen (b >= 1 after at least one token).
 * - w and u must be finite.  NaN or Inf in k, v, grad_y propagate to the
 *   outputs; they are not checked.
 * - Alignment: every tensor pointer must be aligned to its element size;
 *   misaligned pointers give WKV_ERR_UNSUPPORTED.  Any C >= 1 is accepted.
 * - Sizes: B, C >= 1 and T >= 0 (N >= 1 for wkv_step); B*T*C < 2^62;
 *   T < 2^31.  T = 0 copies state_in to state_out (if given).
 * - Not thread-safe per workspace: calls that share a workspace must be
 *   ordered on one stream.
 */
#ifndef LIBWKV_WKV_H
#define LIBWKV_WKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define WKV_VERSION 140 /* 1.4.0: chain kernels; a checkpoint every 16 tokens */

/* Element type of the [B, T, C] tensors. */
typedef enum { WKV_F32 = 0, WKV_BF16 = 1 } wkv_dtype;

/* Return codes. */
typedef enum {
  WKV_OK = 0,
  WKV_ERR_INVALID_ARG = -1, /* required pointer NULL, size out of range, bad dtype/op */
  WKV_ERR_UNSUPPORTED = -2, /* misaligned pointer or unsupported aliasing */
  WKV_ERR_WORKSPACE = -3,   /* workspace NULL, misaligned or smaller than required */
  WKV_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  WKV_ERR_TIMEOUT = -5      /* device side: a bounded cross-block wait gave up */
} wkv_status;

/* Operation selector for wkv_workspace_size. */
enum { WKV_OP_FORWARD = 0, WKV_OP_BACKWARD = 1, WKV_OP_STEP = 2 };

/* Kernel selector (wkv_options.kernel). */
enum { WKV_KERNEL_AUTO = 0, WKV_KERNEL_SEQUENTIAL = 1, WKV_KERNEL_CHUNKED = 2,
       WKV_KERNEL_CHUNKED_REGS = 3, /* 4 and 5 are retired */
       WKV_KERNEL_SEGMENT = 6, WKV_KERNEL_CLUSTER = 7, WKV_KERNEL_TILE = 8,
       WKV_KERNEL_CHAIN = 9 };

/*
 * Optional knobs for the *_ex calls.  A NULL options pointer, or all fields
 * zero, means the defaults.  None of them changes the result beyond
 * floating-point rounding order.
 *   kernel      WKV_KERNEL_AUTO picks by problem shape; SEQUENTIAL runs one
 *               thread per (b, c) chain over all of T; CHUNKED splits T into
 *               64-token chunks joined by a single-pass scan over published
 *               chunk summaries (TMA-fed when rows are 16-byte aligned);
 *               CHUNKED_REGS forces its register-tile variant (no TMA).
 *               SEGMENT (the default when rows are 16-byte aligned) gives
 *               each warp one segment of one chain at a time, its length
 *               chosen per launch: a first pass (summary; in the backward the
 *               forward recompute and the adjoint aggregate), a fixed-order
 *               join with the chain's other segments (through per-record
 *               flags, or after one grid barrier when every warp holds a
 *               single segment), and a second pass from L2 (replay; in the
 *               backward the reverse sweep), the backward reducing dL/dw and
 *               dL/du in the same launch.  CLUSTER (forward only) gives each
 *               chain a thread-block cluster whose warps take its segments
 *               round by round and join them through distributed shared
 *               memory.  TILE (forward and backward) gives each warp units
 *               of 32 (fp32) or 64 (bf16) tokens of one chain whose tiles
 *               stay in shared memory between the unit's two passes, joins
 *               units by a decoupled look-back over records that carry their
 *               own validity tags (no fences), and, in the forward, runs the
 *               next unit's first pass before the current unit's join.
 *               CHAIN (16-byte aligned rows) gives each warp whole chains,
 *               run in
 *               time order from a ring of TMA tiles with the state (or the
 *               adjoint) carried in registers: no joins and a single pass
 *               over every token, for problems whose chains alone fill the
 *               GPU's warp schedulers; where it does not apply, the call
 *               runs TILE.  AUTO runs CHAIN on 16-byte aligned rows when the
 *               chains (batch rows x 32-channel tiles) number 60 % or more
 *               of the warp schedulers (4 per SM), else TILE when a chain
 *               has at most about four resident warps' units in flight, else
 *               SEGMENT, and the chunked kernels on unaligned rows.  Values 4 and 5 are retired and rejected with
 *               WKV_ERR_INVALID_ARG.
 *   spin_limit  bound on any one device-side wait (a predecessor's record,
 *               a shared-memory load, the grid barrier) in microseconds (the
 *               chunked kernels count polls of at most about 1 us each);
 *               past it the wait gives up with WKV_ERR_TIMEOUT (0 = default,
 *               about one second).
 *   test_hold_first_chunk
 *               test hook: blocks of the first chunk in scan order never
 *               publish their results, so the blocks that depend on them must
 *               run out their wait limit.  Results are then invalid and
 *               wkv_get_status() returns WKV_ERR_TIMEOUT.
 */
typedef struct {
  int kernel;
  int test_hold_first_chunk;
  int64_t spin_limit;
} wkv_options;

/*
 * Bytes of workspace the given operation needs (0 for WKV_OP_STEP, which
 * needs none).  The workspace is any device buffer of at least that size,
 * aligned to 256 bytes, ZERO-FILLED ONCE before its first use (cudaMemset or
 * wkv_workspace_init); the library keeps it consistent from then on.  One
 * workspace sized for the largest call may serve forward and backward calls
 * of any shape, as long as those calls are ordered on one stream.
 * Returns 0 for invalid arguments.
 */
size_t wkv_workspace_size(int op, int64_t B, int64_t T, int64_t C, int dtype);

/* Zero-fills a workspace on `stream` (asynchronous). */
int wkv_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Bytes of the forward checkpoint buffer: the state at every 16th token,
 * float32 [ceil(T/16)][3][B][C].  Its contents are private to the library
 * (the exponent is stored in base 2); it only carries the forward's
 * per-chunk states to wkv_backward so the backward does not rescan.
 */
size_t wkv_ckpt_size(int64_t B, int64_t T, int64_t C);

/*
 * wkv_forward -- time-parallel forward.
 *   B, T, C    batch, sequence length, channels.
 *   dtype      element type of k, v, y.
 *   w, u       [C] float32 decay (per-step log-decay, normally < 0) and bonus.
 *   k, v       [B, T, C] inputs.
 *   state_in   [3][B][C] state before token 0, or NULL for the empty state.
 *   y          [B, T, C] output; must not overlap k or v.
 *   state_out  [3][B][C] state after token T-1, or NULL.  May equal state_in.
 *   ckpt       wkv_ckpt_size() bytes to receive the checkpoints for
 *              wkv_backward, or NULL.
 *   ws         workspace of wkv_workspace_size(WKV_OP_FORWARD, ...) bytes.
 * Errors: INVALID_ARG (NULL w/u/k/v/y, bad sizes or dtype), UNSUPPORTED
 * (misaligned, y overlapping k/v), WORKSPACE, CUDA.
 */
int wkv_forward(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                const float *u, const void *k, const void *v, const float *state_in,
                void *y, float *state_out, float *ckpt, void *ws, size_t ws_bytes,
                void *stream);

int wkv_forward_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                   const float *u, const void *k, const void *v,
                   const float *state_in, void *y, float *state_out, float *ckpt,
                   void *ws, size_t ws_bytes, void *stream, const wkv_options *opt);

/*
 * wkv_backward -- gradients of a scalar loss L given grad_y = dL/dy.
 *   state_in   the state the forward started from, or NULL (empty).
 *   ckpt       the checkpoints the forward wrote for the same inputs, or NULL
 *              to have them recomputed here (one extra read of k and v).
 *   grad_w     [C] float32, receives dL/dw summed over the batch (overwritten).
 *              A caller holding time_decay (w = -exp(time_decay)) gets
 *              dL/dtime_decay = grad_w * w.
 *   grad_u     [C] float32, receives dL/du summed over the batch (overwritten).
 *   grad_k, grad_v  [B, T, C] outputs (element type dtype); must not overlap
 *              the inputs.
 *   ws         workspace of wkv_workspace_size(WKV_OP_BACKWARD, ...) bytes.
 * The state after the last token receives no gradient, and state_in gets
 * none.  gw and gu are reduced in a fixed order, so repeated calls give
 * bit-identical results.
 * Errors: as wkv_forward (NULL grad_y/grad_w/grad_u/grad_k/grad_v is
 * INVALID_ARG).
 */
int wkv_backward(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                 const float *u, const void *k, const void *v, const void *grad_y,
                 const float *state_in, const float *ckpt, float *grad_w,
                 float *grad_u, void *grad_k, void *grad_v, void *ws,
                 size_t ws_bytes, void *stream);

int wkv_backward_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                    const float *u, const void *k, const void *v,
                    const void *grad_y, const float *state_in, const float *ckpt,
                    float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                    void *ws, size_t ws_bytes, void *stream, const wkv_options *opt);

/*
 * wkv_backward_state -- wkv_backward with the state terms of a sequence
 * split across calls (truncated back-propagation through time: the RNN form
 * of the RWKV review, section "RNN-유사추론", carried from one call to the
 * next through state_in / state_out).
 *   state_out       [3][B][C] the state after the last token in the
 *                   representation grad_state_out refers to: the forward's
 *                   state_out, or any (a, b, p) of that state.  Only its p
 *                   plane is read.  Required when grad_state_out is given.
 *   grad_state_out  [3][B][C] float32 dL/d(a, b, p) of that state, or NULL
 *                   (no loss term on the final state).  The loss is taken to
 *                   depend on a state only through the sums it represents,
 *                   A = a e^p and B = b e^p (true of every call of this
 *                   library), so dL/dA = ga e^{-p}, dL/dB = gb e^{-p}; the p
 *                   component carries nothing more (it equals a ga + b gb)
 *                   and is not read.  An empty state (p = -inf) passes no
 *                   gradient.
 *   grad_state_in   [3][B][C] float32 output dL/d(a, b, p) of state_in as
 *                   given: (dL/dA_0 e^p, dL/dB_0 e^p, a dL/da + b dL/db), or
 *                   NULL.  Zeros when state_in is NULL (the empty state).
 *                   Must not overlap any other argument.
 * Everything else is as in wkv_backward; grad_w also receives the final-state
 * term's share.  Chaining: a call's grad_state_in, passed with its state_in
 * as the previous call's grad_state_out and state_out, gives that call the
 * gradients a single call over both ranges would give.
 * Errors: as wkv_backward; grad_state_out without state_out is INVALID_ARG.
 */
int wkv_backward_state(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                       const float *u, const void *k, const void *v, const void *grad_y,
                       const float *state_in, const float *ckpt, const float *state_out,
                       const float *grad_state_out, float *grad_w, float *grad_u,
                       void *grad_k, void *grad_v, float *grad_state_in, void *ws,
                       size_t ws_bytes, void *stream);

int wkv_backward_state_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                          const float *u, const void *k, const void *v, const void *grad_y,
                          const float *state_in, const float *ckpt, const float *state_out,
                          const float *grad_state_out, float *grad_w, float *grad_u,
                          void *grad_k, void *grad_v, float *grad_state_in, void *ws,
                          size_t ws_bytes, void *stream, const wkv_options *opt);

/*
 * wkv_forward_gated -- the time-mixing output with its receptance gate:
 *   o_t = sigma(r_t) * y_t,   sigma(x) = 1 / (1 + e^{-x}),
 * y the WKV output above (RWKV paper review, section "출력 게이팅(Output
 * Gating)": o_t = W_o (sigma(r_t) * WKV_t); the W_o projection is a plain
 * GEMM and stays with the caller).  The gate is applied as y is stored, so o
 * costs one extra read of r and no pass over y.
 *   r          [B, T, C] gate input (element type dtype).
 *   o          [B, T, C] output; must not overlap k, v or r.
 * Every other argument is as in wkv_forward: state_out and ckpt describe the
 * WKV recurrence (the gate does not enter it), so the checkpoints serve
 * wkv_backward_gated and wkv_backward alike.
 * Errors: as wkv_forward (NULL r is INVALID_ARG when T > 0).
 */
int wkv_forward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                      const float *u, const void *k, const void *v, const void *r,
                      const float *state_in, void *o, float *state_out, float *ckpt,
                      void *ws, size_t ws_bytes, void *stream);

int wkv_forward_gated_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                         const float *u, const void *k, const void *v, const void *r,
                         const float *state_in, void *o, float *state_out, float *ckpt,
                         void *ws, size_t ws_bytes, void *stream, const wkv_options *opt);

/*
 * wkv_backward_gated -- gradients of a scalar loss L given grad_o = dL/do
 * for o = sigma(r) * y:
 *   dL/dy = grad_o sigma(r)  (fed to the WKV backward),
 *   dL/dr = grad_o y sigma(r) (1 - sigma(r)).
 *   r, grad_o  [B, T, C] (element type dtype).
 *   grad_r     [B, T, C] output; must not overlap any input or grad_k/grad_v.
 * Everything else is as in wkv_backward (ckpt from wkv_forward_gated or
 * wkv_forward of the same k, v, state_in; grad_w, grad_u overwritten and
 * reduced in a fixed order).  The segment backward (k, v, r, grad_o and
 * grad_k 16-byte aligned, C * element size a multiple of 16) forms both
 * gradients in its own passes and holds dL/dy in grad_k's rows until it
 * overwrites them with dL/dk; with the other kernels grad_r is first used
 * as scratch for dL/dy.  Either way the outputs' contents are only defined
 * once the call has completed without error.
 * Errors: as wkv_backward (NULL r/grad_r is INVALID_ARG when T > 0).
 */
int wkv_backward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                       const float *u, const void *k, const void *v, const void *r,
                       const void *grad_o, const float *state_in, const float *ckpt,
                       float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                       void *grad_r, void *ws, size_t ws_bytes, void *stream);

int wkv_backward_gated_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                          const float *u, const void *k, const void *v, const void *r,
                          const void *grad_o, const float *state_in, const float *ckpt,
                          float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                          void *grad_r, void *ws, size_t ws_bytes, void *stream,
                          const wkv_options *opt);

/*
 * wkv_token_shift -- the token shift that forms the time-mixing inputs
 * (RWKV review, section "토큰 변환": each of R, K, V is a linear
 * interpolation of the current and the previous token), n interpolations
 * from one read of x:
 *   out_m[t] = mu_m * x[t] + (1 - mu_m) * x[t-1],   m < n, per channel,
 * x[-1] = x_prev (the previous call's last token) or 0 when x_prev is NULL.
 *   n          1..4 interpolated inputs.
 *   mu         [n][C] float32 mixing coefficients.
 *   x          [B, T, C] (element type dtype).
 *   x_prev     [B, C] (dtype) or NULL.
 *   out        [n][B, T, C] (dtype): n consecutive tensors; must not overlap
 *              x, x_prev or mu.
 * Needs no workspace.  Errors: INVALID_ARG (n outside 1..4, NULL mu, NULL
 * x/out with T > 0, bad sizes or dtype), UNSUPPORTED (misaligned,
 * overlapping), CUDA.
 */
int wkv_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int n,
                    const float *mu, const void *x, const void *x_prev, void *out,
                    void *stream);

/* Bytes of the workspace wkv_token_shift_backward needs (0 for bad sizes). */
size_t wkv_token_shift_workspace_size(int64_t B, int64_t T, int64_t C, int n);

/*
 * wkv_token_shift_backward -- gradients of a scalar loss L given
 * grad_out = dL/dout [n][B, T, C]:
 *   grad_x[t]   = sum_m mu_m grad_out_m[t] + (1 - mu_m) grad_out_m[t+1]
 *                 (grad_out_m[T] = 0), [B, T, C] (dtype);
 *   grad_mu     [n][C] float32, sum over b, t of grad_out_m[t] (x[t] - x[t-1]),
 *               added in a fixed order (bit-reproducible; overwritten);
 *   grad_x_prev [B, C] (dtype) sum_m (1 - mu_m) grad_out_m[0], or NULL.
 * x, x_prev, mu as in the forward.  Outputs must not overlap the inputs or
 * one another.  ws: wkv_token_shift_workspace_size() bytes, 256-byte
 * aligned (contents need not be initialised).
 * Errors: as wkv_token_shift; NULL grad_mu is INVALID_ARG; WORKSPACE.
 */
int wkv_token_shift_backward(int64_t B, int64_t T, int64_t C, int dtype, int n,
                             const float *mu, const void *x, const void *x_prev,
                             const void *grad_out, void *grad_x, float *grad_mu,
                             void *grad_x_prev, void *ws, size_t ws_bytes, void *stream);

/*
 * wkv_step -- one RNN-mode token for N independent sequences (float32).
 *   k_t, v_t   [N, C] inputs of this token.
 *   state_in   [3][N][C] state before the token (required).
 *   y_t        [N, C] output.
 *   state_out  [3][N][C] state after the token; may equal state_in (update in
 *              place); must not partly overlap it.
 * Equivalent to wkv_forward with T = 1.  Needs no workspace.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA.
 */
int wkv_step(int64_t N, int64_t C, const float *w, const float *u,
             const float *k_t, const float *v_t, const float *state_in, float *y_t,
             float *state_out, void *stream);

/*
 * wkv_backward_static -- wkv_backward for callers that cannot allocate.
 *
 * The paper has no counterpart; this is a deployment convenience.  Callers
 * running where cudaMalloc is not allowed (inside an allocator or memory-pool
 * callback, in plugin hosts that only hand out fixed buffers, on threads of
 * runtimes that forbid device allocation) cannot provide the workspace
 * wkv_backward needs.  This entry point takes the same arguments minus the
 * workspace and uses a file-scope static device array of
 * WKV_STATIC_SCRATCH_BYTES instead; it calls no cudaMalloc/cudaFree and no
 * allocating library routine.  Inputs and outputs are still the caller's.
 *   - Limit: problems with wkv_workspace_size(WKV_OP_BACKWARD, B, T, C, dtype)
 *     above WKV_STATIC_SCRATCH_BYTES are rejected with WKV_ERR_WORKSPACE.
 *   - Set-up: every call looks up the array's device address in the current
 *     context with cudaGetSymbolAddress (which allocates nothing), so a
 *     device reset or another context on the same device never leaves a
 *     stale address.  The first call that meets an address (the first call
 *     on each device, with that device current) zero-fills the array
 *     synchronously (cudaMemset, cudaDeviceSynchronize); make that first
 *     call before any stream capture.
 *   - Every call in a context shares the one array, which keeps the previous
 *     call's contents.  Calls whose executions overlap on the GPU (other
 *     streams, other host threads) race on it and give wrong results; order
 *     them on one stream.
 *   - Each GPU that loads the library holds the array until the process
 *     exits.  A device-side wait that gave up is read, like wkv_get_status,
 *     with wkv_backward_static_status.
 * Returns the codes of wkv_backward, plus WKV_ERR_CUDA if the set-up fails.
 * Argument errors are found before anything is launched.
 */
#define WKV_STATIC_SCRATCH_BYTES (16u << 20) /* 16 MiB */
int wkv_backward_static(int64_t B, int64_t T, int64_t C, int dtype, const float *w,
                        const float *u, const void *k, const void *v, const void *grad_y,
                        const float *state_in, const float *ckpt, float *grad_w,
                        float *grad_u, void *grad_k, void *grad_v, void *stream);

/*
 * wkv_get_status for wkv_backward_static's array in the current context:
 * waits for `stream`, then returns and clears the device-side status word
 * (WKV_OK, or WKV_ERR_TIMEOUT if a bounded wait of an earlier call gave up
 * and its gradients are invalid).  WKV_ERR_CUDA if the look-up, the
 * synchronisation or the copy failed.
 */
int wkv_backward_static_status(void *stream);

/*
 * Waits for `stream`, then returns and clears the device-side status word of
 * the workspace: WKV_OK, or WKV_ERR_TIMEOUT if a bounded wait of an earlier
 * call on it gave up (its results are then invalid).  WKV_ERR_CUDA if the
 * synchronisation or the copy failed, WKV_ERR_WORKSPACE for a NULL ws.
 */
int wkv_get_status(void *ws, void *stream);

/* Static string for a return code ("unknown status" otherwise). */
const char *wkv_strerror(int status);

/*
 * The cudaError_t value (as an int) behind the calling thread's most recent
 * WKV_ERR_CUDA return, 0 if there was none; wkv_cuda_error_name gives its
 * name ("cudaErrorInvalidValue", ...).  Diagnostics only: the value is not
 * cleared by later successful calls.
 */
int wkv_last_cuda_error(void);
const char *wkv_cuda_error_name(int err);

/* WKV_VERSION of the built library. */
int wkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LIBWKV_WKV_H */
