// wkv_step.cu -- RNN-mode decode step of libwkv.
//
// One token for N independent sequences: the output and the state update of
// the RWKV paper review's RNN form ("[논문 리뷰] Reinvention RNNs for the
// Transformer Era: RWKV", section "RNN-유사추론", eq. WKV_t; the decoding
// loop of section "자기 회귀 디코딩", step 4 "update the WKV state" and step
// 7 "store A_t, B_t").  Per (n, c):
//
//   y   = (A + e^{u+k} v) / (B + e^{u+k})
//   A' = e^w A + e^k v,   B' = e^w B + e^k
//
// over the stored max-rescaled state (a, b, p), A = a e^p, B = b e^p, in
// natural-log exponents (the C ABI's state format).  The kernel is a pure
// stream: 36 bytes per (n, c) (state 12 in + 12 out, k, v, y), read and
// written once, 128-bit vectorised when the layout allows.
//
// Exponent drift: when the stored maximum simply decays (p' = p + w), the
// float sum p + w is rounded.  The exact rounding error err = (p + w) - p'
// (two-sum) is folded back into the scale of the old sums, a' = a (1 + err),
// so repeated steps do not accumulate a drift in the exponent.
#include "wkv_internal.cuh"

namespace wkv {

__device__ __forceinline__ void two_sum(float x, float y, float &s, float &e) {
  s = __fadd_rn(x, y);
  const float yv = __fsub_rn(s, x);
  const float xv = __fsub_rn(s, yv);
  e = __fadd_rn(__fsub_rn(x, xv), __fsub_rn(y, yv));
}

__device__ __forceinline__ void step_one(float w, float u, float k, float v, float &a, float &b,
                                         float &p, float &y) {
  p = fmaxf(p, -1.0e38f);  // the empty state may arrive as p = -inf
  const float uk = u + k;
  const float q = fmaxf(p, uk);
  const float e1 = expf(p - q), e2 = expf(uk - q);
  y = (a * e1 + v * e2) / (b * e1 + e2);
  float pw, err;
  two_sum(p, w, pw, err);  // p + w = pw + err exactly
  if (k > pw) {
    const float so = expf((pw - k) + err);
    a = fmaf(a, so, v);
    b = fmaf(b, so, 1.f);
    p = k;
  } else {
    const float sn = expf(k - pw);
    a = fmaf(a, err, a) + v * sn;  // a e^{err} ~ a (1 + err): |err| <= ulp(pw)/2
    b = fmaf(b, err, b) + sn;
    p = pw;
  }
}

template <bool VEC>
__global__ void __launch_bounds__(256) step_kernel(StepArgs s) {
  const int64_t NC = s.N * s.C;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (VEC) {
    const int64_t n4 = NC / 4;
    const float4 *ai = reinterpret_cast<const float4 *>(s.state_in);
    const float4 *bi = reinterpret_cast<const float4 *>(s.state_in + NC);
    const float4 *pi = reinterpret_cast<const float4 *>(s.state_in + 2 * NC);
    float4 *ao = reinterpret_cast<float4 *>(s.state_out);
    float4 *bo = reinterpret_cast<float4 *>(s.state_out + NC);
    float4 *po = reinterpret_cast<float4 *>(s.state_out + 2 * NC);
    const float4 *k4 = reinterpret_cast<const float4 *>(s.k);
    const float4 *v4 = reinterpret_cast<const float4 *>(s.v);
    float4 *y4 = reinterpret_cast<float4 *>(s.y);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += stride) {
      const int64_t c0 = (i * 4) % s.C;  // C % 4 == 0: the 4 lanes share a row
      const float4 w4 = *reinterpret_cast<const float4 *>(s.w + c0);
      const float4 u4 = *reinterpret_cast<const float4 *>(s.u + c0);
      float4 a = __ldcs(ai + i), b = __ldcs(bi + i), p = __ldcs(pi + i);
      const float4 k = __ldcs(k4 + i), v = __ldcs(v4 + i);
      float4 y;
      step_one(w4.x, u4.x, k.x, v.x, a.x, b.x, p.x, y.x);
      step_one(w4.y, u4.y, k.y, v.y, a.y, b.y, p.y, y.y);
      step_one(w4.z, u4.z, k.z, v.z, a.z, b.z, p.z, y.z);
      step_one(w4.w, u4.w, k.w, v.w, a.w, b.w, p.w, y.w);
      __stcs(y4 + i, y);
      __stcs(ao + i, a);
      __stcs(bo + i, b);
      __stcs(po + i, p);
    }
  } else {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < NC; i += stride) {
      const int64_t c = i % s.C;
      float a = s.state_in[i], b = s.state_in[NC + i], p = s.state_in[2 * NC + i], y;
      step_one(s.w[c], s.u[c], s.k[i], s.v[i], a, b, p, y);
      s.y[i] = y;
      s.state_out[i] = a;
      s.state_out[NC + i] = b;
      s.state_out[2 * NC + i] = p;
    }
  }
}

cudaError_t launch_step(const StepArgs &a, bool vec, int num_sms, cudaStream_t st) {
  const int64_t NC = a.N * a.C;
  const int64_t items = vec ? NC / 4 : NC;
  int64_t blocks = (items + 255) / 256;
  const int64_t cap = (int64_t)num_sms * 8;  // 8 blocks of 256 per SM, grid-stride beyond
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return vec ? launch_kernel(step_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, st, a)
             : launch_kernel(step_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, st, a);
}

}  // namespace wkv
