// wkv_forward.cu -- forward kernels of libwkv.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), evaluated in the
// RNN form of section "RNN-유사추론" (eq. WKV_t) over the max-rescaled state.
// The review's "Transformer-유사학습" section runs WKV as a scan over time;
// the two kernels here are the two ways of running that scan:
//
//   fwd_seq_kernel      one thread per (b, c) chain walks all of T.  Used when
//                       there are enough chains to fill the GPU.
//   fwd_chunked_kernel  one block per (b, 32-channel tile, 128-token chunk).
//                       Each warp summarises a 16-token segment, the block
//                       joins its segments, and chunks are joined along T by
//                       a single-pass scan over published per-chunk
//                       summaries (a Fenwick tree, so the result does not
//                       depend on block timing); then every warp replays its
//                       segment from the carried-in state.  k and v are read
//                       from HBM once and stay in registers between passes.
#include "wkv_internal.cuh"

namespace wkv {

// Running state of one channel with the anchored exponent P = fma(n, w, Panc).
struct Run {
  float a, b, Panc, n;
};

__device__ __forceinline__ Run run_from(const St &s) { return Run{s.a, s.b, s.P, 0.f}; }
__device__ __forceinline__ St run_state(const Run &r, float w2) {
  return St{r.a, r.b, fmaf(r.n, w2, r.Panc)};
}

// One token: output y_t = (A_t + e^{u+k} v) / (B_t + e^{u+k}) from the state
// before the token, then A_{t+1} = e^w A_t + e^k v, B_{t+1} = e^w B_t + e^k.
// Base-2 exponents (K = k log2 e, u2 = u log2 e, w2 = w log2 e).  In each pair
// of scale factors one is exactly 1, so a token costs two ex2 and one rcp.
__device__ __forceinline__ float fwd_token(Run &s, float K, float V, float u2, float w2) {
  const float P = fmaf(s.n, w2, s.Panc);
  const float UK = u2 + K;
  const float d = P - UK;
  const float x = ex2(-fabsf(d));
  const bool pw = d >= 0.f;
  const float e1 = pw ? 1.f : x, e2 = pw ? x : 1.f;
  const float y = fmaf(s.a, e1, V * e2) * rcp(fmaf(s.b, e1, e2));
  const float n1 = s.n + 1.f;
  const float Pc = fmaf(n1, w2, s.Panc);
  const float d2 = K - Pc;
  const float x2 = ex2(-fabsf(d2));
  const bool kw = d2 > 0.f;
  const float so = kw ? x2 : 1.f, sn = kw ? 1.f : x2;
  s.a = fmaf(s.a, so, V * sn);
  s.b = fmaf(s.b, so, sn);
  s.Panc = kw ? K : s.Panc;
  s.n = kw ? 0.f : n1;
  return y;
}

// Initial state of chain (b, c) from the caller's natural-log state.
__device__ __forceinline__ St load_state_in(const float *st, int64_t i, int64_t BC) {
  if (!st) return st_empty();
  St s;
  s.a = st[i];
  s.b = st[BC + i];
  s.P = fmaxf(st[2 * BC + i] * kLog2e, kEmptyP);
  return s;
}
__device__ __forceinline__ void store_state(float *st, int64_t i, int64_t BC, const St &s) {
  st[i] = s.a;
  st[BC + i] = s.b;
  st[2 * BC + i] = s.P * kLn2;
}
// Checkpoint (base-2 exponent) of the state before token ci * kCkpt.
__device__ __forceinline__ void store_ckpt(float *ck, int64_t ci, int64_t i, int64_t BC,
                                           const St &s) {
  float *d = ck + ci * 3 * BC;
  d[i] = s.a;
  d[BC + i] = s.b;
  d[2 * BC + i] = s.P;
}

// ------------------------------------------------------------------------
// Sequential scan: one thread per (b, c).  Consecutive threads take
// consecutive channels, so every load/store instruction of a warp touches
// one contiguous 128-byte (fp32) row segment.  k, v are prefetched U tokens
// ahead.
// ------------------------------------------------------------------------
template <typename E, int U>
__global__ void __launch_bounds__(256) fwd_seq_kernel(FwdArgs p) {
  static_assert(kCkpt % U == 0, "checkpoint interval must be a multiple of U");
  const int64_t BC = p.B * p.C;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BC) return;
  const int64_t b = idx / p.C, c = idx - b * p.C;
  const float w2 = p.w[c] * kLog2e, u2 = p.u[c] * kLog2e;
  const int64_t T = p.T, C = p.C;
  const E *kp = static_cast<const E *>(p.k) + b * T * C + c;
  const E *vp = static_cast<const E *>(p.v) + b * T * C + c;
  E *yp = p.y ? static_cast<E *>(p.y) + b * T * C + c : nullptr;
  Run s = run_from(load_state_in(p.state_in, idx, BC));

  float Kc[U], Vc[U], Kn[U], Vn[U];
  if (T > 0) {
    const int n0 = (int)min((int64_t)U, T);
    load_rows<E, U>(kp, C, n0, Kc);
    load_rows<E, U>(vp, C, n0, Vc);
  }
  for (int64_t t0 = 0; t0 < T; t0 += U) {
    // prefetch the next U rows (clamped to the last row; ignored past T)
    if (t0 + U < T) {
      const int n1 = (int)min((int64_t)U, T - t0 - U);
      load_rows<E, U>(kp + (t0 + U) * C, C, n1, Kn);
      load_rows<E, U>(vp + (t0 + U) * C, C, n1, Vn);
    }
    if (p.ckpt && (t0 % kCkpt) == 0) store_ckpt(p.ckpt, t0 / kCkpt, idx, BC, run_state(s, w2));
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (t0 + j < T) {
        const float y = fwd_token(s, Kc[j] * kLog2e, Vc[j], u2, w2);
        if (yp) IO<E>::st(yp + (t0 + j) * C, y);
      }
    }
    if (s.n > 1048576.f) {  // keep n exact as a float: re-anchor (one rounding)
      s.Panc = fmaf(s.n, w2, s.Panc);
      s.n = 0.f;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      Kc[j] = Kn[j];
      Vc[j] = Vn[j];
    }
  }
  if (p.state_out) store_state(p.state_out, idx, BC, run_state(s, w2));
}

// ------------------------------------------------------------------------
// Chunked scan.  Block = W warps; warp `wi` owns tokens [t0, t0 + L) of the
// block's chunk for the 32 channels of its tile (lane = channel).
// ------------------------------------------------------------------------

// Summary of a segment from the empty state: the state after its last valid
// token, A = sum_j e^{(n-1-j) w + k_j} v_j.  Exponents are formed directly
// (one fma each) against the segment maximum, so it costs one ex2 per token.
template <int L>
__device__ __forceinline__ St summarize(const float (&K)[L], const float (&V)[L], float w2,
                                        int nvalid) {
  float e[L];
  float m = kEmptyP;
  const float last = (float)(nvalid - 1);
#pragma unroll
  for (int j = 0; j < L; ++j) {
    e[j] = fmaf(last - (float)j, w2, K[j]);
    if (j < nvalid) m = fmaxf(m, e[j]);
  }
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int j = 0; j < L; ++j) {
    if (j < nvalid) {
      const float x = ex2(e[j] - m);
      a = fmaf(x, V[j], a);
      b += x;
    }
  }
  return St{a, b, m};
}

template <typename E, int W, int L>
__global__ void __launch_bounds__(W * 32) fwd_chunked_kernel(FwdArgs p) {
  constexpr int TC = W * L;
  static_assert(TC % kCkpt == 0 && kCkpt % L == 0, "chunk/ckpt geometry");
  __shared__ unsigned s_tile, s_epoch;
  __shared__ float s_agg[W][3][32];  // warp segment summaries
  __shared__ float s_pre[W][3][32];  // block-local exclusive prefix of each warp
  __shared__ float s_carry[3][32];   // state at the start of the block's chunk

  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  take_ticket(p.hdr, &s_tile, &s_epoch);
  __syncthreads();
  const int64_t tile = s_tile;
  const unsigned epoch = s_epoch;
  if (tile >= p.nchains * p.nchunks) {  // stale ticket counter: touch nothing
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, -4 /* WKV_ERR_CUDA */);
    finish_block(p.hdr, gridDim.x);
    return;
  }
  const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t tc0 = chunk * TC;                 // first token of the chunk
  const int64_t t0 = tc0 + (int64_t)wi * L;       // first token of this warp
  const int nvalid = (int)max((int64_t)0, min((int64_t)L, T - t0));
  const int chunk_len = (int)min((int64_t)TC, T - tc0);
  const float w2 = cok ? p.w[c] * kLog2e : 0.f;
  const float u2 = cok ? p.u[c] * kLog2e : 0.f;

  float K[L], V[L];
  if (nvalid > 0) {  // warp-uniform
    const int64_t off = (b * T + t0) * C + (cok ? c : C - 1);
    load_rows<E, L>(static_cast<const E *>(p.k) + off, C, nvalid, K);
    load_rows<E, L>(static_cast<const E *>(p.v) + off, C, nvalid, V);
#pragma unroll
    for (int j = 0; j < L; ++j) {
      const bool ok = cok && j < nvalid;
      K[j] = ok ? K[j] * kLog2e : 0.f;
      V[j] = ok ? V[j] : 0.f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < L; ++j) K[j] = V[j] = 0.f;
  }

  // Pass 1: segment summary.
  {
    const St s = summarize<L>(K, V, w2, nvalid);
    s_agg[wi][0][lane] = s.a;
    s_agg[wi][1][lane] = s.b;
    s_agg[wi][2][lane] = s.P;
  }
  __syncthreads();

  // Warp 0: block-local prefixes, then the chunk scan along T.
  if (wi == 0) {
    St acc = st_empty();
#pragma unroll
    for (int i = 0; i < W; ++i) {
      s_pre[i][0][lane] = acc.a;
      s_pre[i][1][lane] = acc.b;
      s_pre[i][2][lane] = acc.P;
      const St si{s_agg[i][0][lane], s_agg[i][1][lane], s_agg[i][2][lane]};
      const int li = (int)max((int64_t)0, min((int64_t)L, T - (tc0 + (int64_t)i * L)));
      acc = combine(acc, si, (float)li, w2);
    }
    const St initial = cok ? load_state_in(p.state_in, b * C + c, BC) : st_empty();
    const St excl = chunk_scan(p.flags, p.desc, chunk, chain, p.nchains, acc, (float)chunk_len,
                               (float)TC, initial, st_empty(), epoch, p.hdr, p.spin_limit,
                               chunk + 1 < p.nchunks, !(p.hold_first && chunk == 0), w2, lane);
    s_carry[0][lane] = excl.a;
    s_carry[1][lane] = excl.b;
    s_carry[2][lane] = excl.P;
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);

  // Pass 2: replay the segment from the carried-in state.
  if (nvalid > 0) {
    const St cin{s_carry[0][lane], s_carry[1][lane], s_carry[2][lane]};
    const St pre{s_pre[wi][0][lane], s_pre[wi][1][lane], s_pre[wi][2][lane]};
    const St start = combine(cin, pre, (float)min(wi * L, chunk_len), w2);
    if (p.ckpt && cok && (t0 % kCkpt) == 0) store_ckpt(p.ckpt, t0 / kCkpt, b * C + c, BC, start);
    Run s = run_from(start);
    E *yp = p.y ? static_cast<E *>(p.y) + (b * T + t0) * C + c : nullptr;
#pragma unroll
    for (int j = 0; j < L; ++j) {
      if (j < nvalid) {
        const float y = fwd_token(s, K[j], V[j], u2, w2);
        if (yp && cok) IO<E>::st(yp + (int64_t)j * C, y);
      }
    }
    if (p.state_out && cok && t0 + nvalid == T) store_state(p.state_out, b * C + c, BC, run_state(s, w2));
  }
}

// ---------------------------------------------------------------- launch ---
constexpr int kSeqU = 8;
constexpr int kFwdW = 8, kFwdL = 16;

int64_t fwd_chunk_tokens() { return kFwdW * kFwdL; }

template <typename E>
static cudaError_t launch_fwd_t(const FwdArgs &a, bool chunked, cudaStream_t st) {
  if (!chunked) {
    const int64_t BC = a.B * a.C;
    const unsigned grid = (unsigned)((BC + 255) / 256);
    fwd_seq_kernel<E, kSeqU><<<grid, 256, 0, st>>>(a);
  } else {
    const int64_t tiles = a.nchains * a.nchunks;
    fwd_chunked_kernel<E, kFwdW, kFwdL><<<(unsigned)tiles, kFwdW * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_forward(const FwdArgs &a, int dtype, bool chunked, cudaStream_t st) {
  return dtype == 0 ? launch_fwd_t<float>(a, chunked, st) : launch_fwd_t<uint16_t>(a, chunked, st);
}

}  // namespace wkv
