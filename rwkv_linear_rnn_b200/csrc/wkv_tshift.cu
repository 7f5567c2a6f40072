// wkv_tshift.cu -- token shift of libwkv: the interpolation of the current
// and the previous token that forms the time-mixing inputs (RWKV paper
// review, "[논문 리뷰] Reinvention RNNs for the Transformer Era: RWKV",
// section "토큰 변환"):
//
//   out_m[t] = mu_m x[t] + (1 - mu_m) x[t-1]   (m < n, per channel),
//
// x[-1] being the previous call's last token (x_prev) or zero.  One read of
// x serves all n interpolations.  HBM-bound and elementwise along channels;
// the time shift is carried in registers: a thread owns V consecutive
// channels of one batch row over a strip of kStrip tokens and keeps x[t-1]
// from the previous step, so x is read once (plus one row per strip).
//
// Backward, per strip in reverse time: gx[t] = sum_m mu_m g_m[t] +
// (1 - mu_m) g_m[t+1]; per-strip partial sums of dL/dmu_m = sum g_m[t]
// (x[t] - x[t-1]) go to the workspace and a second kernel adds them per
// channel in a fixed order (float64), so the result is reproducible;
// dL/dx_prev = sum_m (1 - mu_m) g_m[0].
#include <algorithm>

#include "wkv_internal.cuh"

namespace wkv {

constexpr int kStrip = 32;          // tokens per thread strip
constexpr int kStripsPerBlock = 8;  // strips per backward block (one per warp)

int64_t token_shift_strips(int64_t T) { return (T + kStrip - 1) / kStrip; }
// rows of dL/dmu partials the backward writes: one per (b, block of strips)
int64_t token_shift_rows(int64_t B, int64_t T) {
  return B * ((token_shift_strips(T) + kStripsPerBlock - 1) / kStripsPerBlock);
}

namespace {

template <typename E, int V>
struct Vec;
template <>
struct Vec<float, 4> {
  static __device__ __forceinline__ void ld(const float *p, float (&x)[4]) {
    const float4 q = __ldcs(reinterpret_cast<const float4 *>(p));
    x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
  }
  static __device__ __forceinline__ void st(float *p, const float (&x)[4]) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <>
struct Vec<uint16_t, 4> {
  static __device__ __forceinline__ void ld(const uint16_t *p, float (&x)[4]) {
    const uint2 q = __ldcs(reinterpret_cast<const uint2 *>(p));
    x[0] = __uint_as_float(q.x << 16), x[1] = __uint_as_float(q.x & 0xffff0000u);
    x[2] = __uint_as_float(q.y << 16), x[3] = __uint_as_float(q.y & 0xffff0000u);
  }
  static __device__ __forceinline__ unsigned pack(float lo, float hi) {
    unsigned r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
  }
  static __device__ __forceinline__ void st(uint16_t *p, const float (&x)[4]) {
    __stcs(reinterpret_cast<uint2 *>(p), make_uint2(pack(x[0], x[1]), pack(x[2], x[3])));
  }
};
template <typename E>
struct Vec<E, 1> {
  static __device__ __forceinline__ void ld(const E *p, float (&x)[1]) { x[0] = IO<E>::ld(p); }
  static __device__ __forceinline__ void st(E *p, const float (&x)[1]) { IO<E>::st(p, x[0]); }
};

struct TsArgs {
  int64_t B, T, C;
  int n;
  const float *mu;  // [n][C]
  const void *x, *x_prev;
  void *out;        // [n][B][T][C]
  const void *g;    // [n][B][T][C] (backward)
  void *gx, *gx_prev;
  float *part;      // [B][nstrip][n][C] partial dL/dmu (backward)
  float *gmu;       // [n][C] dL/dmu (backward)
  int64_t nstrip;
};

// Thread -> (b, strip, channel group); consecutive threads take consecutive
// channel groups of the same rows, so every row access is coalesced.
template <typename E, int V, int N>
__global__ void __launch_bounds__(256) tshift_fwd_kernel(TsArgs a) {
  const int64_t ncg = a.C / V;
  const int64_t units = a.B * a.nstrip * ncg;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < units;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t cg = u % ncg, rs = u / ncg;
    const int64_t s = rs % a.nstrip, b = rs / a.nstrip;
    const int64_t c = cg * V, t0 = s * kStrip;
    const int nt = (int)min((int64_t)kStrip, a.T - t0);
    const E *x = static_cast<const E *>(a.x) + (b * a.T) * a.C + c;
    E *out = static_cast<E *>(a.out) + (b * a.T) * a.C + c;
    const int64_t plane = a.B * a.T * a.C;
    float mu[N][V];
#pragma unroll
    for (int m = 0; m < N; ++m)
#pragma unroll
      for (int j = 0; j < V; ++j) mu[m][j] = __ldg(a.mu + m * a.C + c + j);
    float prev[V];
    if (t0 > 0) {
      Vec<E, V>::ld(x + (t0 - 1) * a.C, prev);
    } else if (a.x_prev) {
      Vec<E, V>::ld(static_cast<const E *>(a.x_prev) + b * a.C + c, prev);
    } else {
#pragma unroll
      for (int j = 0; j < V; ++j) prev[j] = 0.f;
    }
    // groups of 4 rows: the loads of a group are issued before its math
    for (int t = 0; t < nt; t += 4) {
      float xs[4][V];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (t + i < nt) Vec<E, V>::ld(x + (t0 + t + i) * a.C, xs[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (t + i < nt) {
#pragma unroll
          for (int m = 0; m < N; ++m) {
            float o[V];
#pragma unroll
            for (int j = 0; j < V; ++j) o[j] = fmaf(mu[m][j], xs[i][j] - prev[j], prev[j]);
            Vec<E, V>::st(out + m * plane + (t0 + t + i) * a.C, o);
          }
#pragma unroll
          for (int j = 0; j < V; ++j) prev[j] = xs[i][j];
        }
      }
    }
  }
}

// The backward of one strip (b, s) of channel group cg: writes gx (and
// gx_prev for the first strip) and adds the strip's dL/dmu terms to acc.
template <typename E, int V, int N>
__device__ __forceinline__ void strip_bwd(const TsArgs &a, int64_t b, int64_t s, int64_t cg, float (&acc)[N][V]) {
  {
    const int64_t c = cg * V, t0 = s * kStrip;
    const int nt = (int)min((int64_t)kStrip, a.T - t0);
    const int64_t plane = a.B * a.T * a.C;
    const E *x = static_cast<const E *>(a.x) + (b * a.T) * a.C + c;
    const E *g = static_cast<const E *>(a.g) + (b * a.T) * a.C + c;
    E *gx = static_cast<E *>(a.gx) + (b * a.T) * a.C + c;
    float mu[N][V], gn[N][V];
#pragma unroll
    for (int m = 0; m < N; ++m)
#pragma unroll
      for (int j = 0; j < V; ++j) {
        mu[m][j] = __ldg(a.mu + m * a.C + c + j);
        gn[m][j] = 0.f;
      }
    // g_m[t+1] after the strip (zero after the last token)
    if (t0 + nt < a.T) {
#pragma unroll
      for (int m = 0; m < N; ++m) Vec<E, V>::ld(g + m * plane + (t0 + nt) * a.C, gn[m]);
    }
    float xc[V];  // x[t] of the current step
    Vec<E, V>::ld(x + (t0 + nt - 1) * a.C, xc);
#pragma unroll 4
    for (int t = nt - 1; t >= 0; --t) {
      float xp[V], gs[N][V];
      if (t0 + t > 0) {
        Vec<E, V>::ld(x + (t0 + t - 1) * a.C, xp);
      } else if (a.x_prev) {
        Vec<E, V>::ld(static_cast<const E *>(a.x_prev) + b * a.C + c, xp);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) xp[j] = 0.f;
      }
#pragma unroll
      for (int m = 0; m < N; ++m) Vec<E, V>::ld(g + m * plane + (t0 + t) * a.C, gs[m]);
      float o[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        float sum = 0.f;
#pragma unroll
        for (int m = 0; m < N; ++m) {
          sum = fmaf(mu[m][j], gs[m][j], sum);
          sum = fmaf(1.f - mu[m][j], gn[m][j], sum);
          acc[m][j] = fmaf(gs[m][j], xc[j] - xp[j], acc[m][j]);
          gn[m][j] = gs[m][j];
        }
        o[j] = sum;
        xc[j] = xp[j];
      }
      Vec<E, V>::st(gx + (t0 + t) * a.C, o);
    }
    if (t0 == 0 && a.gx_prev) {  // gn holds g_m[0] now
      float o[V];
#pragma unroll
      for (int j = 0; j < V; ++j) {
        float sum = 0.f;
#pragma unroll
        for (int m = 0; m < N; ++m) sum = fmaf(1.f - mu[m][j], gn[m][j], sum);
        o[j] = sum;
      }
      Vec<E, V>::st(static_cast<E *>(a.gx_prev) + b * a.C + c, o);
    }
  }
}

// A block covers 8 strips (one per warp) x 32 channel groups (one per lane)
// of one batch row, and adds its 8 strips' dL/dmu partials in shared memory
// in a fixed order before writing one partial row; the final reduction then
// has 8x fewer rows to add.
template <typename E, int V, int N>
__global__ void __launch_bounds__(256) tshift_bwd_kernel(TsArgs a) {
  __shared__ float red[kStripsPerBlock][N][32 * V];
  const int64_t ncg = a.C / V;
  const int64_t ncgb = (ncg + 31) / 32, nsb = (a.nstrip + kStripsPerBlock - 1) / kStripsPerBlock;
  const int64_t blocks = a.B * nsb * ncgb;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int64_t ub = blockIdx.x; ub < blocks; ub += gridDim.x) {  // block-uniform loop
    const int64_t cgb = ub % ncgb, rsb = ub / ncgb;
    const int64_t sb = rsb % nsb, b = rsb / nsb;
    const int64_t s = sb * kStripsPerBlock + w, cg = cgb * 32 + lane;
    float acc[N][V];
#pragma unroll
    for (int m = 0; m < N; ++m)
#pragma unroll
      for (int j = 0; j < V; ++j) acc[m][j] = 0.f;
    if (s < a.nstrip && cg < ncg) strip_bwd<E, V, N>(a, b, s, cg, acc);
#pragma unroll
    for (int m = 0; m < N; ++m)
#pragma unroll
      for (int j = 0; j < V; ++j) red[w][m][lane * V + j] = acc[m][j];
    __syncthreads();
    for (int k = threadIdx.x; k < N * 32 * V; k += blockDim.x) {
      const int m = k / (32 * V), col = k - m * 32 * V;
      const int64_t ch = cgb * 32 * V + col;
      if (ch < a.C) {
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < kStripsPerBlock; ++i) sum += red[i][m][col];
        __stcg(a.part + ((b * nsb + sb) * N + m) * a.C + ch, sum);
      }
    }
    __syncthreads();  // red is reused by the next block unit
  }
}

// dL/dmu[m][c]: the per-block partials added in a fixed order (float64).
// Block = 32 columns x 8 row groups: group k adds rows k, k+8, ... in
// order, eight loads in flight per step, and the eight group sums are then
// added in order.
__global__ void __launch_bounds__(256) tshift_reduce_kernel(const float *part, int64_t rows, int64_t cols,
                                                             float *gmu) {
  __shared__ double s[8][32];
  const int cl = threadIdx.x & 31, grp = threadIdx.x >> 5;
  const int64_t i = (int64_t)blockIdx.x * 32 + cl;  // m * C + c
  double sum = 0.0;
  if (i < cols) {
    for (int64_t r0 = grp; r0 < rows; r0 += 64) {
      float xs[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t r = r0 + 8 * j;
        xs[j] = r < rows ? __ldcg(part + r * cols + i) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) sum += (double)xs[j];
    }
  }
  s[grp][cl] = sum;
  __syncthreads();
  if (grp == 0 && i < cols) {
    double t = 0.0;
#pragma unroll
    for (int k = 0; k < 8; ++k) t += s[k][cl];
    gmu[i] = (float)t;
  }
}

template <typename E, int V, int N>
cudaError_t launch_ts(const TsArgs &a, bool bwd, int num_sms, cudaStream_t st) {
  const int64_t units = a.B * a.nstrip * (a.C / V);
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>((units + 255) / 256, (int64_t)num_sms * 16));
  if (!bwd) return launch_kernel(tshift_fwd_kernel<E, V, N>, dim3((unsigned)grid), dim3(256), 0, st, a);
  const int64_t ncgb = (a.C / V + 31) / 32;
  const int64_t bunits = a.B * token_shift_rows(1, a.T) * ncgb;
  const int64_t bgrid = std::max<int64_t>(1, std::min<int64_t>(bunits, (int64_t)num_sms * 8));
  cudaError_t e = launch_kernel(tshift_bwd_kernel<E, V, N>, dim3((unsigned)bgrid), dim3(256), 0, st, a);
  if (e != cudaSuccess) return e;
  const int64_t cols = (int64_t)a.n * a.C;
  return launch_kernel(tshift_reduce_kernel, dim3((unsigned)((cols + 31) / 32)), dim3(256), 0, st,
                       (const float *)a.part, token_shift_rows(a.B, a.T), cols, a.gmu);
}

template <typename E, int V>
cudaError_t launch_ts_n(const TsArgs &a, bool bwd, int num_sms, cudaStream_t st) {
  switch (a.n) {
    case 1: return launch_ts<E, V, 1>(a, bwd, num_sms, st);
    case 2: return launch_ts<E, V, 2>(a, bwd, num_sms, st);
    case 3: return launch_ts<E, V, 3>(a, bwd, num_sms, st);
    default: return launch_ts<E, V, 4>(a, bwd, num_sms, st);
  }
}

}  // namespace



// vec: every row pointer allows 4-channel vector accesses (C % 4 == 0 and
// the pointers aligned to 4 elements).  Forward: out.  Backward: g, gx,
// gx_prev (nullable), part (workspace), gmu.
cudaError_t launch_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int n, const float *mu, const void *x,
                               const void *x_prev, void *out, const void *g, void *gx, void *gx_prev, float *part,
                               float *gmu, bool bwd, bool vec, int num_sms, cudaStream_t st) {
  TsArgs a{};
  a.B = B; a.T = T; a.C = C; a.n = n; a.mu = mu; a.x = x; a.x_prev = x_prev; a.out = out;
  a.g = g; a.gx = gx; a.gx_prev = gx_prev; a.part = part; a.gmu = gmu; a.nstrip = token_shift_strips(T);
  if (dtype == 0)
    return vec ? launch_ts_n<float, 4>(a, bwd, num_sms, st) : launch_ts_n<float, 1>(a, bwd, num_sms, st);
  return vec ? launch_ts_n<uint16_t, 4>(a, bwd, num_sms, st) : launch_ts_n<uint16_t, 1>(a, bwd, num_sms, st);
}

}  // namespace wkv
