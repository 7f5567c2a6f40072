// wkv_gate.cu -- elementwise steps of the output gate o = sigma(r) * wkv
// (RWKV paper review, "[논문 리뷰] Reinvention RNNs for the Transformer Era:
// RWKV", section "출력 게이팅(Output Gating)", without the W_o projection).
//
// The segment kernels apply the gate inside their own store loops; these
// kernels serve the other kernels (rows that are not 16-byte aligned, a
// caller-chosen non-segment kernel):
//   gate_apply   o <- sigma(r) * o             (after the ungated forward)
//   gate_pre     t <- grad_o * sigma(r)         (the WKV output's gradient)
//   gate_post    t <- grad_o * t * sigma'(r)    (t holds wkv on entry)
// Streaming grid-stride loops over the B*T*C elements, 4 per thread per
// step when every pointer is 16-byte aligned.
#include <algorithm>

#include "wkv_internal.cuh"

namespace wkv {

namespace {

constexpr int kOpApply = 0, kOpPre = 1, kOpPost = 2;

// Four consecutive elements (16-byte aligned for float, 8-byte for bf16).
__device__ __forceinline__ void ld4(const float *p, float (&x)[4]) {
  const float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
  x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
}
__device__ __forceinline__ void st4(float *p, const float (&x)[4]) {
  __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
}
__device__ __forceinline__ void ld4(const uint16_t *p, float (&x)[4]) {
  const uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p));
  x[0] = __uint_as_float(q.x << 16), x[1] = __uint_as_float(q.x & 0xffff0000u);
  x[2] = __uint_as_float(q.y << 16), x[3] = __uint_as_float(q.y & 0xffff0000u);
}
__device__ __forceinline__ unsigned pack_bf16x2(float lo, float hi) {
  unsigned r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void st4(uint16_t *p, const float (&x)[4]) {
  __stcs(reinterpret_cast<uint2 *>(p), make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3])));
}

template <int OP>
__device__ __forceinline__ float gate_op(float x, float go, float r) {
  if constexpr (OP == kOpApply) {
    return gate_sigmoid(r) * x;
  } else if constexpr (OP == kOpPre) {
    return go * gate_sigmoid(r);
  } else {
    float s, ds;
    gate_sigmoid_slope(r, s, ds);
    return go * x * ds;
  }
}

// x: in/out (o for apply, t for pre/post); go unused by apply.
template <typename E, int OP>
__global__ void __launch_bounds__(256) gate_kernel(E *x, const E *go, const E *r, int64_t n, bool vec) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (vec) {
    const int64_t n4 = n / 4;
    for (int64_t q = i; q < n4; q += stride) {
      float xs[4] = {0.f, 0.f, 0.f, 0.f}, gs[4] = {0.f, 0.f, 0.f, 0.f}, rs[4];
      if (OP != kOpPre) ld4(x + 4 * q, xs);  // pre only writes x
      ld4(r + 4 * q, rs);
      if (OP != kOpApply) ld4(go + 4 * q, gs);
#pragma unroll
      for (int j = 0; j < 4; ++j) xs[j] = gate_op<OP>(xs[j], gs[j], rs[j]);
      st4(x + 4 * q, xs);
    }
    i += n4 * 4;  // the scalar loop below takes the tail
  }
  for (; i < n; i += stride) {
    const float g = OP != kOpApply ? IO<E>::ld(go + i) : 0.f;
    const float xi = OP != kOpPre ? IO<E>::ld(x + i) : 0.f;
    IO<E>::st(x + i, gate_op<OP>(xi, g, IO<E>::ld(r + i)));
  }
}

template <typename E>
cudaError_t launch_gate_t(int op, void *x, const void *go, const void *r, int64_t n, int num_sms,
                          cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const bool vec = ((uintptr_t)x % 16) == 0 && ((uintptr_t)r % 16) == 0 && ((uintptr_t)go % 16) == 0;
  const int64_t per = vec ? 4 : 1;
  const int64_t want = (n / per + 255) / 256;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)num_sms * 8));
  E *xe = static_cast<E *>(x);
  const E *ge = static_cast<const E *>(go), *re = static_cast<const E *>(r);
  auto kern = op == kOpApply ? gate_kernel<E, kOpApply> : op == kOpPre ? gate_kernel<E, kOpPre> : gate_kernel<E, kOpPost>;
  return launch_kernel(kern, dim3((unsigned)grid), dim3(256), 0, st, xe, ge, re, n, vec);
}

}  // namespace

// op: 0 apply, 1 pre, 2 post (see the file comment).
cudaError_t launch_gate(int op, int dtype, void *x, const void *go, const void *r, int64_t n, int num_sms,
                        cudaStream_t st) {
  return dtype == 0 ? launch_gate_t<float>(op, x, go, r, n, num_sms, st)
                    : launch_gate_t<uint16_t>(op, x, go, r, n, num_sms, st);
}

}  // namespace wkv
