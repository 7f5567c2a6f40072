// wkv_scan3.cu -- reduce / scan / replay forward of libwkv.
//
// The review's time-parallel mode ("[논문 리뷰] Reinvention RNNs for the
// Transformer Era: RWKV", section "Transformer-유사학습": every step except
// WKV is parallel over batch and time, WKV itself is a scan) evaluated with
// the associative combine of two sequence summaries, in three launches:
//
//   fwd_sum_kernel     one warp per (chain, 64-token chunk): the summary of
//                      the chunk from the empty state (one ex2 per token).
//                      A chain is one batch row and 32 channels; lanes are
//                      channels, so every load is a 128-byte row segment.
//   fwd_prefix_kernel  one block per chain: the state at the start of every
//                      chunk, joined in a fixed bracketing (two-level: 32
//                      groups folded in parallel, then the group totals),
//                      so the result is bit-reproducible.  These states are
//                      also the backward's checkpoints.
//   fwd_replay_kernel  one warp per (chain, chunk): the recurrence of eq.
//                      WKV_t ("RNN-유사추론") over the chunk from its start
//                      state, writing y (and the final state).
//
// Everything is independent across warps except the tiny prefix step.  k and
// v are read twice (summary, replay); when they fit in L2 the second read
// does not reach HBM.
#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_split.cuh"

namespace wkv {

bool fwd_tma_eligible(const FwdArgs &a, int dtype);
cudaError_t launch_scan3_tma(const Scan3Args &a, int dtype, int num_sms, cudaStream_t st);


// Rows [t, t + n) of column c (clamped to valid rows) into registers.
template <typename E>
__device__ __forceinline__ void load_batch(const E *kp, const E *vp, int64_t C, int n,
                                           float (&K)[kS3Batch], float (&V)[kS3Batch]) {
  if (n > 0) {
    load_rows<E, kS3Batch>(kp, C, n, K);
    load_rows<E, kS3Batch>(vp, C, n, V);
  }
}

// ------------------------------------------------------------ summaries ---
template <typename E>
__global__ void __launch_bounds__(256) fwd_sum_kernel(Scan3Args a) {
  const FwdArgs &p = a.f;
  const int lane = threadIdx.x & 31;
  const int64_t unit = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int64_t nsum = (a.npos - 1) * p.nchains;  // the last chunk needs no summary
  if (unit >= nsum) return;
  const int64_t chunk = unit / p.nchains, chain = unit - chunk * p.nchains;
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C;
  const int64_t t0 = chunk * kS3Chunk;
  const int n = (int)min((int64_t)kS3Chunk, T - t0);
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const int64_t off = (b * T + t0) * C + (cok ? c : C - 1);
  const E *kp = static_cast<const E *>(p.k) + off;
  const E *vp = static_cast<const E *>(p.v) + off;

  constexpr int NB = kS3Chunk / kS3Batch;
  float K0[kS3Batch], V0[kS3Batch], K1[kS3Batch], V1[kS3Batch];
  load_batch<E>(kp, vp, C, min(n, kS3Batch), K0, V0);
  St acc = st_empty();
#pragma unroll
  for (int bt = 0; bt < NB; ++bt) {
    float(&Kc)[kS3Batch] = (bt & 1) ? K1 : K0;
    float(&Vc)[kS3Batch] = (bt & 1) ? V1 : V0;
    float(&Kn)[kS3Batch] = (bt & 1) ? K0 : K1;
    float(&Vn)[kS3Batch] = (bt & 1) ? V0 : V1;
    const int nb = max(0, min(kS3Batch, n - bt * kS3Batch));
    if (bt + 1 < NB) {
      const int nn = max(0, min(kS3Batch, n - (bt + 1) * kS3Batch));
      load_batch<E>(kp + (int64_t)(bt + 1) * kS3Batch * C, vp + (int64_t)(bt + 1) * kS3Batch * C, C,
                    nn, Kn, Vn);
    }
    float Ks[kS3Batch];
#pragma unroll
    for (int j = 0; j < kS3Batch; ++j) Ks[j] = Kc[j] * kLog2e;
    const St s = summarize<kS3Batch>(Ks, Vc, w2, nb);
    acc = combine(acc, s, (float)nb, w2);
  }
  float *d = a.sums + (chunk * 4) * p.nchains * 32 + chain * 32 + lane;
  const int64_t plane = p.nchains * 32;
  d[0] = acc.a;
  d[plane] = acc.b;
  d[2 * plane] = acc.P;
  d[3 * plane] = acc.n;
}

// --------------------------------------------------------------- prefix ---
// Block = 32 warps = 32 groups of consecutive chunks of one chain.
__global__ void __launch_bounds__(1024) fwd_prefix_kernel(Scan3Args a) {
  const FwdArgs &p = a.f;
  __shared__ float s_tot[32][128];
  __shared__ float s_exc[32][128];
  const int g = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t chain = blockIdx.x;
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const int64_t nsum = a.npos - 1;  // summaries exist for chunks [0, npos-1)
  const int64_t m = (nsum + 31) / 32;
  const int64_t j0 = min((int64_t)g * m, nsum), j1 = min(j0 + m, nsum);
  const int64_t plane = p.nchains * 32;
  auto sum_at = [&](int64_t j) {
    const float *d = a.sums + (j * 4) * plane + chain * 32 + lane;
    return St{d[0], d[plane], d[2 * plane], d[3 * plane]};
  };
  auto len_at = [&](int64_t j) { return (float)min((int64_t)kS3Chunk, T - j * kS3Chunk); };
  // level 1: fold each group
  St acc = st_empty();
  for (int64_t j = j0; j < j1; ++j) acc = combine(acc, sum_at(j), len_at(j), w2);
  put_st(s_tot[g], lane, acc);
  __syncthreads();
  // level 2: exclusive prefix over the groups
  if (g == 0) {
    St run = cok ? load_state_in(p.state_in, b * C + c, BC) : st_empty();
    for (int q = 0; q < 32; ++q) {
      put_st(s_exc[q], lane, run);
      const int64_t q0 = min((int64_t)q * m, nsum), q1 = min(q0 + m, nsum);
      run = combine(run, get_st(s_tot[q], lane), (float)((q1 - q0) * kS3Chunk), w2);
    }
  }
  __syncthreads();
  // level 3: chunk start states of this group; the group after the last
  // summary also writes the start of the final chunk
  St run = get_st(s_exc[g], lane);
  if (cok) {
    for (int64_t j = j0; j < j1; ++j) {
      store_ckpt(a.carry, j, b * C + c, BC, run, w2);
      run = combine(run, sum_at(j), len_at(j), w2);
    }
    // The start of the final chunk (which has no summary) comes from the
    // group holding the last summary, or from group 0 when there is none.
    const bool writer = (nsum == 0) ? (g == 0) : (j0 < j1 && j1 == nsum);
    if (writer) store_ckpt(a.carry, nsum, b * C + c, BC, run, w2);
  }
}

// --------------------------------------------------------------- replay ---
template <typename E>
__global__ void __launch_bounds__(256) fwd_replay_kernel(Scan3Args a) {
  const FwdArgs &p = a.f;
  const int lane = threadIdx.x & 31;
  const int64_t unit = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (unit >= a.npos * p.nchains) return;
  const int64_t chunk = unit / p.nchains, chain = unit - chunk * p.nchains;
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t t0 = chunk * kS3Chunk;
  const int n = (int)min((int64_t)kS3Chunk, T - t0);
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
  const int64_t off = (b * T + t0) * C + (cok ? c : C - 1);
  const E *kp = static_cast<const E *>(p.k) + off;
  const E *vp = static_cast<const E *>(p.v) + off;
  E *yp = p.y ? static_cast<E *>(p.y) + (b * T + t0) * C + c : nullptr;
  Run st{0.f, 0.f, kEmptyP, 0.f};
  if (cok) {
    const float *ck = a.carry + chunk * 3 * BC + b * C + c;
    st = Run{ck[0], ck[BC], ck[2 * BC], 0.f};
  }

  constexpr int NB = kS3Chunk / kS3Batch;
  float K0[kS3Batch], V0[kS3Batch], K1[kS3Batch], V1[kS3Batch];
  load_batch<E>(kp, vp, C, min(n, kS3Batch), K0, V0);
#pragma unroll
  for (int bt = 0; bt < NB; ++bt) {
    float(&Kc)[kS3Batch] = (bt & 1) ? K1 : K0;
    float(&Vc)[kS3Batch] = (bt & 1) ? V1 : V0;
    float(&Kn)[kS3Batch] = (bt & 1) ? K0 : K1;
    float(&Vn)[kS3Batch] = (bt & 1) ? V0 : V1;
    const int nb = max(0, min(kS3Batch, n - bt * kS3Batch));
    if (bt + 1 < NB) {
      const int nn = max(0, min(kS3Batch, n - (bt + 1) * kS3Batch));
      load_batch<E>(kp + (int64_t)(bt + 1) * kS3Batch * C, vp + (int64_t)(bt + 1) * kS3Batch * C, C,
                    nn, Kn, Vn);
    }
    if (nb == kS3Batch) {
#pragma unroll
      for (int j = 0; j < kS3Batch; ++j) {
        const float yv = fwd_token(st, Kc[j] * kLog2e, Vc[j], u2, w2);
        if (yp && cok) IO<E>::st(yp + (int64_t)(bt * kS3Batch + j) * C, yv);
      }
    } else {
#pragma unroll
      for (int j = 0; j < kS3Batch; ++j) {
        if (j < nb) {
          const float yv = fwd_token(st, Kc[j] * kLog2e, Vc[j], u2, w2);
          if (yp && cok) IO<E>::st(yp + (int64_t)(bt * kS3Batch + j) * C, yv);
        }
      }
    }
  }
  if (p.state_out && cok && t0 + n == T) store_state(p.state_out, b * C + c, BC, run_state(st), w2);
}

// ---------------------------------------------------------------- launch ---
template <typename E>
static cudaError_t launch_scan3_t(const Scan3Args &a, cudaStream_t st) {
  const int64_t nsum = (a.npos - 1) * a.f.nchains;
  if (nsum > 0) {
    fwd_sum_kernel<E><<<(unsigned)((nsum + 7) / 8), 256, 0, st>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  fwd_prefix_kernel<<<(unsigned)a.f.nchains, 1024, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t units = a.npos * a.f.nchains;
  fwd_replay_kernel<E><<<(unsigned)((units + 7) / 8), 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_fwd_prefix(const Scan3Args &a, cudaStream_t st) {
  fwd_prefix_kernel<<<(unsigned)a.f.nchains, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

// sums / carry point into the workspace (carry may be the caller's ckpt).
cudaError_t launch_forward_scan3(const FwdArgs &f, int dtype, float *sums, float *carry,
                                 int num_sms, cudaStream_t st) {
  Scan3Args a{f, sums, carry, (f.T + kS3Chunk - 1) / kS3Chunk};
  if (fwd_tma_eligible(f, dtype)) return launch_scan3_tma(a, dtype, num_sms, st);
  return dtype == 0 ? launch_scan3_t<float>(a, st) : launch_scan3_t<uint16_t>(a, st);
}

int64_t scan3_chunk() { return kS3Chunk; }

}  // namespace wkv
