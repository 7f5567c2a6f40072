// wkv_backward.cu -- backward kernels of libwkv.
//
// Gradients of L with g_t = dL/dy_t, for the WKV operator of the RWKV paper
// review ("[논문 리뷰] Reinvention RNNs for the Transformer Era: RWKV", section
// "WKV 연산자", eq. wkv_t) in its RNN form (section "RNN-유사추론", eq. WKV_t).
// With D_t = B_t + e^{u+k_t} and the adjoints Ahat_t = dL/dA_t,
// Hhat_t = -dL/dB_t, which satisfy the reverse-time recurrence
//
//   Ahat_t = g_t / D_t + e^w Ahat_{t+1},   Hhat_t = g_t y_t / D_t + e^w Hhat_{t+1}
//
// (zero after the last token), the gradients are
//
//   dL/dv_t = e^{u+k_t} g_t / D_t + e^{k_t} Ahat_{t+1}
//   dL/dk_t = v_t dL/dv_t - e^{u+k_t} g_t y_t / D_t - e^{k_t} Hhat_{t+1}
//   dL/du   = sum e^{u+k_t} g_t (v_t - y_t) / D_t
//   dL/dw   = sum e^w (A_t Ahat_{t+1} - B_t Hhat_{t+1}).
//
// This is the back-propagation-through-time the review credits the RNN form
// with (its "BPTT friendly" property); like the key/value gradients of the
// linear-attention post ("Transformers are RNNs", gradient section) it is a
// reverse-time decayed cumulative sum, so it splits into chunks joined by the
// same deterministic chunk scan as the forward, run from the last chunk
// backwards.
//
// bwd_chunked_kernel: one block per (b, 32-channel tile, 64-token chunk), 8
// warps of 8 tokens.  Per block: (1) load k, v, g once into registers;
// (2) rebuild each warp's starting state from the forward checkpoint of the
// chunk plus the summaries of the earlier warps; (3) recompute the forward
// (y_t, D_t, state) of the segment into registers; (4) run the adjoint
// recurrence over the segment from zero to get its aggregate; (5) join the
// aggregates across warps and, by the chunk scan, across later chunks; (6) run the
// adjoint recurrence again from the true carry, emitting dL/dk, dL/dv and
// per-block partial sums of dL/dw, dL/du.  reduce_wu_kernel then adds the
// partials per channel in a fixed order (deterministic).
//
// The adjoints are held as Ahat = ah 2^-r, Hhat = hh 2^-r with r the running
// minimum of (log2 D_t - lag * w): with that choice every factor formed below
// is at most 1 (the terms e^{k_t} Ahat_{t+1} and e^w A_t Ahat_{t+1} are
// weighted sums of g_s / D_s with weights <= 1), so nothing overflows.
#include "wkv_internal.cuh"
#include "wkv_math.cuh"

namespace wkv {

template <typename E, int W, int L>
__global__ void __launch_bounds__(W * 32) bwd_chunked_kernel(BwdArgs p) {
  constexpr int TC = W * L;
  static_assert(TC % kCkpt == 0, "backward chunks start on checkpoints");
  __shared__ unsigned s_tile, s_epoch;
  __shared__ float s_f[W][128];      // forward summaries, then warp start states (St planes)
  __shared__ float s_adj[W][3][32];  // adjoint aggregates, then later-warp suffixes
  __shared__ float s_carry[3][32];   // adjoint at the end of the block's chunk
  __shared__ float s_g[2][W][32];    // per-warp partial dL/dw, dL/du

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
  const int64_t rpos = tile / p.nchains, chain = tile - rpos * p.nchains;
  const int64_t chunk = p.nchunks - 1 - rpos;  // last chunk first
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t tc0 = chunk * TC;
  const int64_t t0 = tc0 + (int64_t)wi * L;
  const int nvalid = (int)max((int64_t)0, min((int64_t)L, T - t0));
  const int chunk_len = (int)min((int64_t)TC, T - tc0);
  const float w2 = cok ? p.w[c] * kLog2e : 0.f;
  const float u2 = cok ? p.u[c] * kLog2e : 0.f;

  float K[L], V[L], G[L];
  const int64_t off = (b * T + t0) * C + c;
  if (nvalid > 0) {  // warp-uniform
    const int64_t loff = (b * T + t0) * C + (cok ? c : C - 1);
    load_rows<E, L>(static_cast<const E *>(p.k) + loff, C, nvalid, K);
    load_rows<E, L>(static_cast<const E *>(p.v) + loff, C, nvalid, V);
    load_rows<E, L>(static_cast<const E *>(p.gy) + loff, C, nvalid, G);
#pragma unroll
    for (int j = 0; j < L; ++j) {
      const bool ok = cok && j < nvalid;
      K[j] = ok ? K[j] * kLog2e : 0.f;
      V[j] = ok ? V[j] : 0.f;
      G[j] = ok ? G[j] : 0.f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < L; ++j) K[j] = V[j] = G[j] = 0.f;
  }

  // (2) warp start states: checkpoint, then the earlier warps' summaries.
  if (wi < W - 1) {
    const St s = summarize<L>(K, V, w2, nvalid);
    put_st(s_f[wi], lane, s);
  }
  __syncthreads();
  if (wi == 0) {
    St acc = st_empty();
    if (cok) {
      const float *ck = p.ckpt + chunk * (TC / kCkpt) * 3 * BC + b * C + c;
      acc = St{ck[0], ck[BC], ck[2 * BC]};
    }
#pragma unroll
    for (int i = 0; i < W; ++i) {
      St si{};
      if (i < W - 1) si = get_st(s_f[i], lane);
      put_st(s_f[i], lane, acc);
      if (i < W - 1) {
        const int li = (int)max((int64_t)0, min((int64_t)L, T - (tc0 + (int64_t)i * L)));
        acc = combine(acc, si, (float)li, w2);
      }
    }
  }
  __syncthreads();

  // (3) forward recompute of the segment.
  float q_[L], gam[L], eta[L], e2_[L], a_[L], b_[L], so_[L], sn_[L], P1_[L];
  {
    const St st0 = get_st(s_f[wi], lane);
    float sa = st0.a, sb = st0.b, Panc = st0.P, n = st0.n;
#pragma unroll
    for (int j = 0; j < L; ++j) {
      if (j < nvalid) {
        const float P = fmaf(n, w2, Panc);
        const float UK = u2 + K[j];
        const float d = P - UK;
        const float x = ex2(-fabsf(d));
        const bool pw = d >= 0.f;
        const float e1 = pw ? 1.f : x, e2 = pw ? x : 1.f;
        const float rden = rcp(fmaf(sb, e1, e2));
        const float y = fmaf(sa, e1, V[j] * e2) * rden;
        q_[j] = fmaxf(P, UK);
        gam[j] = G[j] * rden;
        eta[j] = gam[j] * y;
        e2_[j] = e2;
        a_[j] = sa;
        b_[j] = sb;
        const float n1 = n + 1.f;
        const float Pc = fmaf(n1, w2, Panc);
        const float d2 = K[j] - Pc;
        const float x2 = ex2(-fabsf(d2));
        const bool kw = d2 > 0.f;
        const float so = kw ? x2 : 1.f, sn = kw ? 1.f : x2;
        sa = fmaf(sa, so, V[j] * sn);
        sb = fmaf(sb, so, sn);
        P1_[j] = kw ? K[j] : Pc;
        Panc = kw ? K[j] : Panc;
        n = kw ? 0.f : n1;
        so_[j] = so;
        sn_[j] = sn;
      }
    }
  }

  // (4) adjoint aggregate of the segment (zero adjoint after it).
  {
    float ah = 0.f, hh = 0.f, Ranc = kEmptyR, m = 0.f;
#pragma unroll
    for (int j = L - 1; j >= 0; --j) {
      if (j < nvalid) {
        const float m1 = m + 1.f;
        const float Rc = fmaf(-m1, w2, Ranc);
        const float d = q_[j] - Rc;
        const float x = ex2(-fabsf(d));
        const bool reset = d < 0.f;
        const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
        ah = fmaf(ah, fo, gam[j] * fg);
        hh = fmaf(hh, fo, eta[j] * fg);
        Ranc = reset ? q_[j] : Ranc;
        m = reset ? 0.f : m1;
      }
    }
    s_adj[wi][0][lane] = ah;
    s_adj[wi][1][lane] = hh;
    s_adj[wi][2][lane] = fmaf(-m, w2, Ranc);
  }
  __syncthreads();

  // (5) warp 0: suffix folds within the block, then the chunk scan.
  if (wi == 0) {
    Adj acc = adj_empty();
#pragma unroll
    for (int i = W - 1; i >= 0; --i) {
      const Adj ai{s_adj[i][0][lane], s_adj[i][1][lane], s_adj[i][2][lane]};
      s_adj[i][0][lane] = acc.ah;
      s_adj[i][1][lane] = acc.hh;
      s_adj[i][2][lane] = acc.r;
      const int li = (int)max((int64_t)0, min((int64_t)L, T - (tc0 + (int64_t)i * L)));
      acc = rcombine(ai, acc, (float)li, w2);
    }
    Adj excl = chunk_scan(p.flags, p.desc, rpos, chain, p.nchains, acc, (float)chunk_len, (float)TC,
                          adj_empty(), adj_empty(), epoch, p.hdr, p.spin_limit, rpos + 1 < p.nchunks,
                          !(p.hold_first && rpos == 0), w2, lane);
    // the adjoint after the last token (a loss term on the final state, if
    // any) decays across the tokens after this chunk (the scan counts every
    // later chunk as full, so it is joined here with the exact count)
    if (p.gs_out && cok) {
      const int64_t bc = b * C + c;
      Adj fin;
      end_adjoint(p.gs_out[bc], p.gs_out[BC + bc], p.p_out[bc], fin.ah, fin.hh, fin.r);
      excl = rcombine(excl, fin, (float)(T - tc0 - chunk_len), w2);
    }
    s_carry[0][lane] = excl.ah;
    s_carry[1][lane] = excl.hh;
    s_carry[2][lane] = excl.r;
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);

  // (6) adjoint recurrence from the true carry; gradients.
  float gw = 0.f, gu = 0.f;
  if (nvalid > 0) {
    const Adj later{s_adj[wi][0][lane], s_adj[wi][1][lane], s_adj[wi][2][lane]};
    const Adj cin{s_carry[0][lane], s_carry[1][lane], s_carry[2][lane]};
    const int lsuf = max(0, chunk_len - (wi + 1) * L);
    const Adj start = rcombine(later, cin, (float)lsuf, w2);
    float ah = start.ah, hh = start.hh, Ranc = start.r, m = 0.f;
    E *gkp = static_cast<E *>(p.gk) + off;
    E *gvp = static_cast<E *>(p.gv) + off;
#pragma unroll
    for (int j = L - 1; j >= 0; --j) {
      if (j < nvalid) {
        const float rn = fmaf(-m, w2, Ranc);  // scale of Ahat_{t+1}
        const float E1 = ex2(P1_[j] - rn);
        const float tn = sn_[j] * E1, to = so_[j] * E1;
        const float gv = fmaf(gam[j], e2_[j], tn * ah);
        const float gk = fmaf(V[j], gv, -fmaf(eta[j], e2_[j], tn * hh));
        gu = fmaf(e2_[j], fmaf(gam[j], V[j], -eta[j]), gu);
        gw = fmaf(to, fmaf(a_[j], ah, -b_[j] * hh), gw);
        if (cok) {
          IO<E>::st(gkp + (int64_t)j * C, gk);
          IO<E>::st(gvp + (int64_t)j * C, gv);
        }
        const float m1 = m + 1.f;
        const float Rc = fmaf(-m1, w2, Ranc);
        const float d = q_[j] - Rc;
        const float x = ex2(-fabsf(d));
        const bool reset = d < 0.f;
        const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
        ah = fmaf(ah, fo, gam[j] * fg);
        hh = fmaf(hh, fo, eta[j] * fg);
        Ranc = reset ? q_[j] : Ranc;
        m = reset ? 0.f : m1;
      }
    }
    // warp 0 of the first chunk ends at token 0: the initial state's gradient
    if (p.gs_in && cok && t0 == 0) store_state_grad(p.gs_in, p.state_in, b * C + c, BC, ah, hh, fmaf(-m, w2, Ranc));
  }
  s_g[0][wi][lane] = gw;
  s_g[1][wi][lane] = gu;
  __syncthreads();
  if (wi == 0 && cok) {
    float sw = 0.f, su = 0.f;
#pragma unroll
    for (int i = 0; i < W; ++i) {
      sw += s_g[0][i][lane];
      su += s_g[1][i][lane];
    }
    p.part[(chunk * 2 + 0) * BC + b * C + c] = sw;
    p.part[(chunk * 2 + 1) * BC + b * C + c] = su;
  }
}

// Per-channel sum of the per-(chunk, b) partials in a fixed order (float64
// accumulation).  Block = 32 channels x 8 row groups.
__global__ void __launch_bounds__(256) reduce_wu_kernel(const float *part, int64_t nchunks,
                                                        int64_t B, int64_t C, float *gw,
                                                        float *gu) {
  __shared__ double s[2][8][32];
  const int cl = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t c = (int64_t)blockIdx.x * 32 + cl;
  const int64_t BC = B * C, R = nchunks * B;
  double sw = 0.0, su = 0.0;
  if (c < C) {
    for (int64_t r = g; r < R; r += 8) {
      const int64_t ch = r / B, b = r - ch * B;
      sw += (double)part[(ch * 2 + 0) * BC + b * C + c];
      su += (double)part[(ch * 2 + 1) * BC + b * C + c];
    }
  }
  s[0][g][cl] = sw;
  s[1][g][cl] = su;
  __syncthreads();
  if (g == 0 && c < C) {
    double tw = 0.0, tu = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      tw += s[0][i][cl];
      tu += s[1][i][cl];
    }
    gw[c] = (float)tw;
    gu[c] = (float)tu;
  }
}

// T = 0: the state passes through unchanged, so the initial state's
// gradient is the final state's, moved from the representation with
// exponent p_out to the caller's state_in: dL/d(a, b) scale by e^{p_in -
// p_out}, dL/dp = a dL/da + b dL/db.  gs_out null, an empty final state or
// a null state_in give zeros.
__global__ void __launch_bounds__(256) state_grad_t0_kernel(const float *gs_out, const float *p_out,
                                                            const float *s_in, float *gs_in, int64_t BC) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < BC; i += (int64_t)gridDim.x * blockDim.x) {
    float ga = 0.f, gb = 0.f, gp = 0.f;
    if (gs_out && s_in && p_out[i] != -INFINITY) {
      const float f = expf(s_in[2 * BC + i] - p_out[i]);
      ga = gs_out[i] * f;
      gb = gs_out[BC + i] * f;
      gp = fmaf(s_in[i], ga, s_in[BC + i] * gb);
    }
    gs_in[i] = ga;
    gs_in[BC + i] = gb;
    gs_in[2 * BC + i] = gp;
  }
}

cudaError_t launch_state_grad_t0(const float *gs_out, const float *p_out, const float *s_in, float *gs_in,
                                 int64_t BC, int num_sms, cudaStream_t st) {
  const int64_t want = (BC + 255) / 256;
  const int64_t grid = want < (int64_t)num_sms * 8 ? want : (int64_t)num_sms * 8;
  return launch_kernel(state_grad_t0_kernel, dim3((unsigned)(grid > 0 ? grid : 1)), dim3(256), 0, st, gs_out,
                       p_out, s_in, gs_in, BC);
}

// ---------------------------------------------------------------- launch ---
constexpr int kBwdW = 8, kBwdL = 8;

template <typename E>
static cudaError_t launch_bwd_t(const BwdArgs &a, float *gw, float *gu, cudaStream_t st) {
  const int64_t tiles = a.nchains * a.nchunks;
  cudaError_t e = launch_kernel(bwd_chunked_kernel<E, kBwdW, kBwdL>, dim3((unsigned)tiles), dim3(kBwdW * 32), 0,
                                st, a);
  if (e != cudaSuccess) return e;
  return launch_kernel(reduce_wu_kernel, dim3((unsigned)((a.C + 31) / 32)), dim3(256), 0, st,
                       (const float *)a.part, a.nchunks, a.B, a.C, gw, gu);
}

cudaError_t launch_reduce_wu(const float *part, int64_t nchunks, int64_t B, int64_t C, float *gw,
                             float *gu, cudaStream_t st) {
  return launch_kernel(reduce_wu_kernel, dim3((unsigned)((C + 31) / 32)), dim3(256), 0, st, part, nchunks, B, C,
                       gw, gu);
}

cudaError_t launch_backward(const BwdArgs &a0, int dtype, float *gw, float *gu, cudaStream_t st) {
  BwdArgs a = a0;
  a.nchunks = (a.T + kBwdW * kBwdL - 1) / (kBwdW * kBwdL);  // this kernel's chunks, not checkpoints
  return dtype == 0 ? launch_bwd_t<float>(a, gw, gu, st) : launch_bwd_t<uint16_t>(a, gw, gu, st);
}

}  // namespace wkv
