/*
 * linattn.h -- C ABI of libwkv's causal linear attention on NVIDIA B200
 * (sm_100a tensor cores).  Same shared library as wkv.h.
 *
 * The operator (linear attention post, "Transformers are RNNs: 선형 어텐션으로
 * 만드는 빠른 자기회귀 트랜스포머", section "인과 마스킹과 누적합"; 0-based
 * positions), for every head h independently:
 *
 *   S_i = sum_{j<=i} phi(K_j) V_j^T        (D x M)
 *   Z_i = sum_{j<=i} phi(K_j)              (D)
 *   V'_i = phi(Q_i)^T S_i / (phi(Q_i)^T Z_i)
 *
 * with the feature map of section "특징 맵 선택과 계산 비용",
 * phi(x) = elu(x) + 1 (x + 1 for x > 0, e^x otherwise; always positive, so
 * the denominator is positive and no epsilon is added).  The backward gives
 * the gradients of a scalar loss L with respect to Q, K and V from
 * dL/dV' (section "상수 메모리 기울기 계산": a forward cumulative sum for
 * phi(Q), reverse cumulative sums for phi(K) and V, then the chain rule
 * through the normalisation and phi).
 *
 * How it is computed: positions are cut into chunks of 128.  Per chunk the
 * causal part is the masked product tril(phi(Q) phi(K)^T) V and the earlier
 * chunks enter through phi(Q) S_prev, every product a dense tcgen05 MMA with
 * bfloat16 operands and float32 accumulation in tensor memory; the chunk
 * states are summed in a fixed order, so results are bit-reproducible.
 *
 * Conventions (those of wkv.h where not stated here)
 * ----------------------------------------------------
 * - Device pointers owned by the caller; every call is asynchronous on
 *   `stream` (a cudaStream_t as void*).  The library allocates nothing.
 * - Layout: q, k, grad_q, grad_k are [BH, N, D]; v, out, grad_out, grad_v
 *   are [BH, N, M]; all row-major (the feature index fastest), bfloat16.
 *   BH counts independent problems (batch x heads).  Results are rounded to
 *   nearest even into bfloat16.
 * - Supported head sizes: D = M = 32 (the pages' experiments: 8 heads of 32
 *   dimensions).  Other sizes return WKV_ERR_UNSUPPORTED.
 * - Sizes: BH >= 1, N >= 0, BH * N < 2^31.  N = 0 writes nothing but the
 *   (zero) state; the tensor pointers may then be null.
 * - Alignment: every tensor pointer 16-byte aligned (WKV_ERR_UNSUPPORTED
 *   otherwise); the workspace 256-byte aligned.
 * - Workspace: linattn_workspace_size() bytes, zero-filled once before its
 *   first use (the first 256 bytes are a header like the one of wkv.h's
 *   workspaces; wkv_get_status() reads it).  Calls that share a workspace
 *   must be ordered on one stream.
 * - Return codes are those of wkv.h (WKV_OK, WKV_ERR_*).  A call that
 *   returns an error other than WKV_ERR_CUDA has launched nothing.
 *   Conditions detected on the device (a bounded wait that gave up) are
 *   read with wkv_get_status(ws, stream).
 * - NaN or Inf in the inputs propagate; they are not checked.
 */
#ifndef LIBWKV_LINATTN_H
#define LIBWKV_LINATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LINATTN_OP_FORWARD 0
#define LINATTN_OP_BACKWARD 1

/* Bytes of workspace for `op` at these sizes (0 if the sizes are invalid or
 * unsupported). */
size_t linattn_workspace_size(int op, int64_t BH, int64_t N, int D, int M);

/*
 * Causal linear attention forward (section "인과 마스킹과 누적합").
 *   q, k      [BH, N, D] bf16, read
 *   v         [BH, N, M] bf16, read
 *   out       [BH, N, M] bf16, written: V'
 *   state_out nullable; float32, written: S_{N-1} as [BH][D][M] followed by
 *             Z_{N-1} as [BH][D] (BH*(D*M + D) floats; zeros when N = 0)
 *   ws        workspace of linattn_workspace_size(LINATTN_OP_FORWARD, ...)
 * Returns WKV_OK, WKV_ERR_INVALID_ARG (null or overlapping-by-identity
 * pointers, negative sizes), WKV_ERR_UNSUPPORTED (head size, alignment),
 * WKV_ERR_WORKSPACE (too small) or WKV_ERR_CUDA (launch failed).
 */
int linattn_forward(int64_t BH, int64_t N, int D, int M, const void *q, const void *k, const void *v, void *out,
                    float *state_out, void *ws, size_t ws_bytes, void *stream);

/*
 * Gradients of L given grad_out = dL/dV' (section "상수 메모리 기울기 계산").
 *   q, k, v   as in linattn_forward, read
 *   grad_out  [BH, N, M] bf16, read
 *   grad_q, grad_k [BH, N, D] bf16, written; grad_v [BH, N, M] bf16, written
 *   ws        workspace of linattn_workspace_size(LINATTN_OP_BACKWARD, ...)
 * The forward is recomputed from q, k, v (nothing from linattn_forward is
 * needed).  Return codes as linattn_forward.
 */
int linattn_backward(int64_t BH, int64_t N, int D, int M, const void *q, const void *k, const void *v,
                     const void *grad_out, void *grad_q, void *grad_k, void *grad_v, void *ws, size_t ws_bytes,
                     void *stream);

/*
 * The same gradients from the forward's saved state (the saved-statistics
 * form of the backward): `ws` must be the workspace that the linattn_forward
 * call computing `out` from these q, k, v used, sized
 * linattn_workspace_size(LINATTN_OP_BACKWARD, ...) (a backward-sized
 * workspace serves the forward too), with no other call on it since.  That
 * call left in it each chunk's prefix state and its denominators; this call
 * reads them instead of recomputing the forward, and needs the forward's
 * output:
 *   out       [BH, N, M] bf16, read: linattn_forward's output
 * Other arguments and return codes as linattn_backward.  Results differ from
 * linattn_backward's by rounding only (dL/d den uses the bf16 output).
 */
int linattn_backward_saved(int64_t BH, int64_t N, int D, int M, const void *q, const void *k, const void *v,
                           const void *out, const void *grad_out, void *grad_q, void *grad_k, void *grad_v, void *ws,
                           size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* LIBWKV_LINATTN_H */
