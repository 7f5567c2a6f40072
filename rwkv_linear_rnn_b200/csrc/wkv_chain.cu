// wkv_chain.cu -- chain-resident forward and backward kernels of libwkv
// (the default path on sm_100a when rows are 16-byte aligned).
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), run in the RNN
// form of section "RNN-유사추론" (eq. WKV_t) over the max-rescaled state.
//
// One block owns one chain -- a batch row b and a tile of 32 channels -- and
// walks its whole time axis in tiles of TC = W*L tokens, so the state carried
// from tile to tile never leaves shared memory: no cross-block traffic at
// all.  Inside a tile the W compute warps split the time axis (warp w owns
// rows [w*L, (w+1)*L)):
//
//   pass 1   each warp summarises its segment from the empty state;
//   join     after one named barrier each warp joins the tile's carried-in
//            state with the summaries of the earlier warps (the associative
//            combine that makes the review's "scan over time" possible);
//   pass 2   each warp replays its segment from that state and writes y.
//
// A producer warp streams the k and v tiles of the chain into an S-stage
// shared-memory ring with 2-D TMA loads (cp.async.bulk.tensor, no
// multicast) completing on mbarriers, so HBM reads run ahead of the
// arithmetic.  k and v are read from HBM exactly once.
//
// The backward kernel walks the chain from its last tile to its first,
// carrying the adjoint instead of the state; see bwd_chain_kernel.
#include <cuda.h>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Tokens of warp segment `w` of the tile starting at token tc0.
template <int L>
__device__ __forceinline__ int seg_len(int64_t T, int64_t tc0, int w) {
  return (int)max((int64_t)0, min((int64_t)L, T - (tc0 + (int64_t)w * L)));
}

// ---------------------------------------------------------------- forward ---
template <typename E, int W, int L, int S>
struct ChainFwdLayout {
  static constexpr int TC = W * L;
  static constexpr int TILEB = TC * 32 * (int)sizeof(E);       // one array, one tile
  static constexpr int STAGE_OFF = 0;                          // [S][2][TC][32] E
  static constexpr int SUMS_OFF = S * 2 * TILEB;                // [2][W][4][32] f32
  static constexpr int CARRY_OFF = SUMS_OFF + 2 * W * 128 * 4;  // [2][4][32] f32
  static constexpr int BAR_OFF = CARRY_OFF + 2 * 128 * 4;       // full[S], empty[S]
  static constexpr int FLAG_OFF = BAR_OFF + 2 * S * 8;
  static constexpr int BYTES = FLAG_OFF + 16;
};

template <typename E, int W, int L, int S>
__global__ void __launch_bounds__((W + 1) * 32) fwd_chain_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                 const __grid_constant__ CUtensorMap vmap,
                                                                 FwdArgs p) {
  using Lay = ChainFwdLayout<E, W, L, S>;
  constexpr int TC = Lay::TC;
  extern __shared__ __align__(1024) unsigned char smem[];
  volatile int *abort = reinterpret_cast<volatile int *>(smem + Lay::FLAG_OFF);
  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t chain = blockIdx.x;
  const int64_t b = chain / p.nct;
  const int64_t ct = chain - b * p.nct;
  const int64_t c = ct * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t npos = (T + TC - 1) / TC;
  const int64_t budget = p.spin_limit * 1000;  // ns
  const uint32_t bar0 = smem_addr(smem + Lay::BAR_OFF);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto stage = [&](int s, int arr) {
    return reinterpret_cast<E *>(smem + Lay::STAGE_OFF + (size_t)(s * 2 + arr) * Lay::TILEB);
  };
  float *sums = reinterpret_cast<float *>(smem + Lay::SUMS_OFF);
  float *carry = reinterpret_cast<float *>(smem + Lay::CARRY_OFF);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), W);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (wi == 0) {
    const St s0 = cok ? load_state_in(p.state_in, b * C + c, BC) : st_empty();
    put_st(carry, lane, s0);
  }
  __syncthreads();

  if (wi == W) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t i = 0; i < npos; ++i) {
        const int s = (int)(i % S);
        if (i >= S && !mbar_wait(empty(s), (uint32_t)((i / S) - 1) & 1u, budget, abort)) {
          *abort = 1;
          break;
        }
        if (*abort) break;
        const int x = (int)(ct * 32);
        const int y = (int)(b * T + i * TC);
        mbar_expect_tx(full(s), 2u * Lay::TILEB);
        tma_load_2d(smem_addr(stage(s, 0)), &kmap, x, y, full(s));
        tma_load_2d(smem_addr(stage(s, 1)), &vmap, x, y, full(s));
        issued = i + 1;
      }
      if (*abort)  // every issued load lands before the block may exit
        for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(full((int)(i % S)), (uint32_t)(i / S) & 1u, budget, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------- compute
  const int w = wi;
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
  for (int64_t i = 0; i < npos; ++i) {
    const int s = (int)(i % S);
    // On a failed wait the block keeps iterating on invalid data so that every
    // compute warp still reaches every named barrier (no partial exits).
    if (!mbar_wait(full(s), (uint32_t)(i / S) & 1u, budget, abort)) {
      if (!*abort && lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
      *abort = 1;
    }
    const int64_t tc0 = i * TC;
    const int64_t t0 = tc0 + (int64_t)w * L;
    const int nvalid = seg_len<L>(T, tc0, w);
    const E *kr = stage(s, 0) + w * L * 32 + lane;
    const E *vr = stage(s, 1) + w * L * 32 + lane;
    float K[L], V[L];
#pragma unroll
    for (int j = 0; j < L; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
    }
    // pass 1
    const St sm = summarize<L>(K, V, w2, nvalid);
    float *sb = sums + (i & 1) * W * 128;
    put_st(sb + w * 128, lane, sm);
    named_barrier(1, W * 32);
    // join: carried-in state, then the earlier warps' segments
    St start = get_st(carry + (i & 1) * 128, lane);
#pragma unroll
    for (int q = 0; q < W - 1; ++q) {
      if (q < w) {
        const St sq = get_st(sb + q * 128, lane);
        start = combine(start, sq, (float)seg_len<L>(T, tc0, q), w2);
      }
    }
    if (w == W - 1) {
      const St nxt = combine(start, sm, (float)nvalid, w2);
      put_st(carry + ((i + 1) & 1) * 128, lane, nxt);
    }
    if (w == 0 && p.ckpt && cok) store_ckpt(p.ckpt, i, b * C + c, BC, start, w2);  // TC == kCkpt
    // pass 2
    if (nvalid > 0) {
      Run st = run_from(start);
      E *yp = p.y ? static_cast<E *>(p.y) + (b * T + t0) * C + c : nullptr;
#pragma unroll
      for (int j = 0; j < L; ++j) {
        if (j < nvalid) {
          const float yv = fwd_token(st, K[j], V[j], u2, w2);
          if (yp && cok) IO<E>::st(yp + (int64_t)j * C, yv);
        }
      }
      if (p.state_out && cok && t0 + nvalid == T)
        store_state(p.state_out, b * C + c, BC, run_state(st), w2);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }
}

// --------------------------------------------------------------- backward ---
// Adjoint of one channel with the lag-weighted terms used for dL/dw:
//   Ahat_t = dL/dA_t = sum_{s>=t} e^{(s-t) w} G_s,           G_s = g_s / D_s
//   Hhat_t = -dL/dB_t = sum_{s>=t} e^{(s-t) w} H_s,          H_s = g_s y_s / D_s
//   Ahat'_t = d Ahat_t / dw = sum_{s>=t} (s-t) e^{(s-t) w} G_s   (Hhat' alike)
// held as (ah, hh, ahp, hhp) * 2^-r.  With them
//   dL/dw = sum_t e^{k_t} (v_t Ahat'_{t+1} - Hhat'_{t+1})  [+ A_0 Ahat'_0 - B_0 Hhat'_0]
// (the bracket is the initial state's share), which avoids storing the
// forward sums A_t, B_t for the reverse sweep.
struct Adj5 {
  float ah, hh, ahp, hhp, r;
};
__device__ __forceinline__ Adj5 adj5_empty() { return Adj5{0.f, 0.f, 0.f, 0.f, kEmptyR}; }

// X (earlier, lenX tokens) then Y (later): Y's adjoint decays across X by
// e^{lenX w}; its w-derivative adds lenX times Y's adjoint.
__device__ __forceinline__ Adj5 rcombine5(const Adj5 &X, const Adj5 &Y, float lenX, float w2) {
  const float rY = fmaf(-lenX, w2, Y.r);
  const float d = X.r - rY;
  const float x = ex2(-fabsf(d));
  const bool xs = d <= 0.f;
  const float fx = xs ? 1.f : x, fy = xs ? x : 1.f;
  Adj5 o;
  o.ah = fmaf(X.ah, fx, Y.ah * fy);
  o.hh = fmaf(X.hh, fx, Y.hh * fy);
  o.ahp = fmaf(X.ahp, fx, fmaf(lenX, Y.ah, Y.ahp) * fy);
  o.hhp = fmaf(X.hhp, fx, fmaf(lenX, Y.hh, Y.hhp) * fy);
  o.r = fminf(X.r, rY);
  return o;
}

template <typename E, int W, int L, int S>
struct ChainBwdLayout {
  static constexpr int TC = W * L;
  static constexpr int TILEB = TC * 32 * (int)sizeof(E);
  static constexpr int STAGE_OFF = 0;                            // [S][3][TC][32] E (k, v, g)
  static constexpr int FSUM_OFF = S * 3 * TILEB;                 // [2][W][4][32]
  static constexpr int ASUM_OFF = FSUM_OFF + 2 * W * 128 * 4;    // [2][W][5][32]
  static constexpr int ACARRY_OFF = ASUM_OFF + 2 * W * 160 * 4;  // [2][5][32]
  static constexpr int GRED_OFF = ACARRY_OFF + 2 * 160 * 4;      // [2][W][32]
  static constexpr int BAR_OFF = GRED_OFF + 2 * W * 32 * 4;      // full[S], empty[S]
  static constexpr int FLAG_OFF = BAR_OFF + 2 * S * 8;
  static constexpr int BYTES = FLAG_OFF + 16;
};

__device__ __forceinline__ void put5(float *d, int lane, const Adj5 &a) {
  d[lane] = a.ah;
  d[32 + lane] = a.hh;
  d[64 + lane] = a.ahp;
  d[96 + lane] = a.hhp;
  d[128 + lane] = a.r;
}
__device__ __forceinline__ Adj5 get5(const float *d, int lane) {
  return Adj5{d[lane], d[32 + lane], d[64 + lane], d[96 + lane], d[128 + lane]};
}

// Per-chain backward.  Tiles run from the last to the first.  Per tile:
// (1) forward summaries of the warp segments and (2) the segment start states
// from the tile's checkpoint; (3) forward recompute of each segment into
// registers (q_t = log2 D_t scale, g/D, g y/D, e^{u+k-q}); (4) the adjoint
// aggregate of each segment from zero; (5) the adjoint at each segment end
// from the tile's carried-in adjoint and the later segments; (6) the final
// reverse sweep: dL/dk, dL/dv, and per-lane sums of dL/dw, dL/du.
template <typename E, int W, int L, int S>
__global__ void __launch_bounds__((W + 1) * 32, 2) bwd_chain_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                 const __grid_constant__ CUtensorMap vmap,
                                                                 const __grid_constant__ CUtensorMap gmap,
                                                                 BwdArgs p) {
  using Lay = ChainBwdLayout<E, W, L, S>;
  constexpr int TC = Lay::TC;
  static_assert(TC == kCkpt, "backward tile must equal the checkpoint interval");
  extern __shared__ __align__(1024) unsigned char smem[];
  volatile int *abort = reinterpret_cast<volatile int *>(smem + Lay::FLAG_OFF);
  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t chain = blockIdx.x;
  const int64_t b = chain / p.nct;
  const int64_t ct = chain - b * p.nct;
  const int64_t c = ct * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t npos = (T + TC - 1) / TC;
  const int64_t budget = p.spin_limit * 1000;
  const uint32_t bar0 = smem_addr(smem + Lay::BAR_OFF);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto stage = [&](int s, int arr) {
    return reinterpret_cast<E *>(smem + Lay::STAGE_OFF + (size_t)(s * 3 + arr) * Lay::TILEB);
  };
  float *fsum = reinterpret_cast<float *>(smem + Lay::FSUM_OFF);
  float *asum = reinterpret_cast<float *>(smem + Lay::ASUM_OFF);
  float *acarry = reinterpret_cast<float *>(smem + Lay::ACARRY_OFF);
  float *gred = reinterpret_cast<float *>(smem + Lay::GRED_OFF);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), W);
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (wi == 0) put5(acarry, lane, adj5_empty());  // no gradient after the last token
  __syncthreads();

  if (wi == W) {
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t i = 0; i < npos; ++i) {
        const int s = (int)(i % S);
        if (i >= S && !mbar_wait(empty(s), (uint32_t)((i / S) - 1) & 1u, budget, abort)) {
          *abort = 1;
          break;
        }
        if (*abort) break;
        const int x = (int)(ct * 32);
        const int y = (int)(b * T + (npos - 1 - i) * TC);
        mbar_expect_tx(full(s), 3u * Lay::TILEB);
        tma_load_2d(smem_addr(stage(s, 0)), &kmap, x, y, full(s));
        tma_load_2d(smem_addr(stage(s, 1)), &vmap, x, y, full(s));
        tma_load_2d(smem_addr(stage(s, 2)), &gmap, x, y, full(s));
        issued = i + 1;
      }
      if (*abort)
        for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(full((int)(i % S)), (uint32_t)(i / S) & 1u, budget, nullptr);
    }
    return;
  }

  const int w = wi;
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
  float gw_acc = 0.f, gu_acc = 0.f;
  for (int64_t i = 0; i < npos; ++i) {
    const int s = (int)(i % S);
    if (!mbar_wait(full(s), (uint32_t)(i / S) & 1u, budget, abort)) {
      if (!*abort && lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
      *abort = 1;
    }
    const int64_t q = npos - 1 - i;  // tile index along time
    const int64_t tc0 = q * TC;
    const int64_t t0 = tc0 + (int64_t)w * L;
    const int nvalid = seg_len<L>(T, tc0, w);
    float K[L], V[L], G[L];
    {
      const E *kr = stage(s, 0) + w * L * 32 + lane;
      const E *vr = stage(s, 1) + w * L * 32 + lane;
      const E *gr = stage(s, 2) + w * L * 32 + lane;
#pragma unroll
      for (int j = 0; j < L; ++j) {
        K[j] = to_f32(kr[j * 32]) * kLog2e;
        V[j] = to_f32(vr[j * 32]);
        G[j] = to_f32(gr[j * 32]);
      }
    }
    // (1) forward summary of the segment
    {
      const St fs = summarize<L>(K, V, w2, nvalid);
      put_st(fsum + (i & 1) * W * 128 + w * 128, lane, fs);
    }
    named_barrier(1, W * 32);
    // (2) segment start state: checkpoint of the tile, then earlier segments
    St start = st_empty();
    if (cok) {
      const float *ck = p.ckpt + q * 3 * BC + b * C + c;
      start = St{ck[0], ck[BC], ck[2 * BC]};
    }
    {
      const float *fb = fsum + (i & 1) * W * 128;
#pragma unroll
      for (int r = 0; r < W - 1; ++r) {
        if (r < w) {
          const St sr = get_st(fb + r * 128, lane);
          start = combine(start, sr, (float)seg_len<L>(T, tc0, r), w2);
        }
      }
    }
    // (3) forward recompute: q_t (scale of D_t), g/D, g y/D and e^{u+k-q}
    float qv[L], gam[L], eta[L], e2v[L];
    {
      float sa = start.a, sb = start.b, Panc = start.P, n = start.n;
#pragma unroll
      for (int j = 0; j < L; ++j) {
        qv[j] = 0.f;
        gam[j] = eta[j] = e2v[j] = 0.f;
        if (j < nvalid) {
          const float P = fmaf(n, w2, Panc);
          const float UK = u2 + K[j];
          const float d = P - UK;
          const float x = ex2(-fabsf(d));
          const bool pw = d >= 0.f;
          const float e1 = pw ? 1.f : x, e2 = pw ? x : 1.f;
          const float rden = rcp(fmaf(sb, e1, e2));
          const float y = fmaf(sa, e1, V[j] * e2) * rden;
          qv[j] = fmaxf(P, UK);
          gam[j] = G[j] * rden;
          eta[j] = gam[j] * y;
          e2v[j] = e2;
          const float n1 = n + 1.f;
          const float Pc = fmaf(n1, w2, Panc);
          const float d2 = K[j] - Pc;
          const float x2 = ex2(-fabsf(d2));
          const bool kw = d2 > 0.f;
          const float so = kw ? x2 : 1.f, sn = kw ? 1.f : x2;
          sa = fmaf(sa, so, V[j] * sn);
          sb = fmaf(sb, so, sn);
          Panc = kw ? K[j] : Panc;
          n = kw ? 0.f : n1;
        }
      }
    }
    // (4) adjoint aggregate of the segment from zero at its end
    Adj5 agg;
    {
      float ah = 0.f, hh = 0.f, ahp = 0.f, hhp = 0.f, Ranc = kEmptyR, m = 0.f;
#pragma unroll
      for (int j = L - 1; j >= 0; --j) {
        if (j < nvalid) {
          const float m1 = m + 1.f;
          const float Rc = fmaf(-m1, w2, Ranc);
          const float d = qv[j] - Rc;
          const float x = ex2(-fabsf(d));
          const bool reset = d < 0.f;
          const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
          ahp = fo * (ah + ahp);
          hhp = fo * (hh + hhp);
          ah = fmaf(ah, fo, gam[j] * fg);
          hh = fmaf(hh, fo, eta[j] * fg);
          Ranc = reset ? qv[j] : Ranc;
          m = reset ? 0.f : m1;
        }
      }
      agg = Adj5{ah, hh, ahp, hhp, fmaf(-m, w2, Ranc)};
      put5(asum + (i & 1) * W * 160 + w * 160, lane, agg);
    }
    named_barrier(1, W * 32);
    // (5) adjoint at the end of this segment: tile carry, then later segments
    Adj5 acc = get5(acarry + (i & 1) * 160, lane);
    {
      const float *ab = asum + (i & 1) * W * 160;
#pragma unroll
      for (int r = W - 1; r >= 1; --r) {
        if (r > w) acc = rcombine5(get5(ab + r * 160, lane), acc, (float)seg_len<L>(T, tc0, r), w2);
      }
    }
    if (w == 0) put5(acarry + ((i + 1) & 1) * 160, lane, rcombine5(agg, acc, (float)nvalid, w2));
    // (6) final reverse sweep
    if (nvalid > 0) {
      float ah = acc.ah, hh = acc.hh, ahp = acc.ahp, hhp = acc.hhp, Ranc = acc.r, m = 0.f;
      E *gkp = static_cast<E *>(p.gk) + (b * T + t0) * C + c;
      E *gvp = static_cast<E *>(p.gv) + (b * T + t0) * C + c;
#pragma unroll
      for (int j = L - 1; j >= 0; --j) {
        if (j < nvalid) {
          const float rn = fmaf(-m, w2, Ranc);  // scale of the adjoint after token t
          const float tn = ex2(K[j] - rn);     // e^{k_t} 2^{-r_{t+1}} (<= 1)
          const float gv = fmaf(gam[j], e2v[j], tn * ah);
          const float gk = fmaf(V[j], gv, -fmaf(eta[j], e2v[j], tn * hh));
          gw_acc = fmaf(tn, fmaf(V[j], ahp, -hhp), gw_acc);
          gu_acc = fmaf(e2v[j], fmaf(gam[j], V[j], -eta[j]), gu_acc);
          if (cok) {
            IO<E>::st(gkp + (int64_t)j * C, gk);
            IO<E>::st(gvp + (int64_t)j * C, gv);
          }
          const float m1 = m + 1.f;
          const float Rc = fmaf(-m1, w2, Ranc);
          const float d = qv[j] - Rc;
          const float x = ex2(-fabsf(d));
          const bool reset = d < 0.f;
          const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
          ahp = fo * (ah + ahp);
          hhp = fo * (hh + hhp);
          ah = fmaf(ah, fo, gam[j] * fg);
          hh = fmaf(hh, fo, eta[j] * fg);
          Ranc = reset ? qv[j] : Ranc;
          m = reset ? 0.f : m1;
        }
      }
      if (t0 == 0 && cok) {
        // share of the initial state A_0, B_0 (zero for the empty state)
        const float *ck = p.ckpt + b * C + c;
        const float r0 = fmaf(-m, w2, Ranc);
        gw_acc = fmaf(ex2(ck[2 * BC] - r0), fmaf(ck[0], ahp, -ck[BC] * hhp), gw_acc);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }
  // per-chain partial sums of dL/dw, dL/du (warps in a fixed order)
  gred[w * 32 + lane] = gw_acc;
  gred[(W + w) * 32 + lane] = gu_acc;
  named_barrier(1, W * 32);
  if (w == 0 && cok) {
    float sw = 0.f, su = 0.f;
#pragma unroll
    for (int r = 0; r < W; ++r) {
      sw += gred[r * 32 + lane];
      su += gred[(W + r) * 32 + lane];
    }
    p.part[b * C + c] = sw;
    p.part[BC + b * C + c] = su;
  }
}

// ---------------------------------------------------------------- launch ---
constexpr int kChainFW = 8, kChainFL = 8, kChainFS = 4;
constexpr int kChainBW = 8, kChainBL = 8, kChainBS = 3;
static_assert(kChainFW * kChainFL == kCkpt && kChainBW * kChainBL == kCkpt, "tile = checkpoint interval");

template <typename K>
static cudaError_t prep(K kern, int bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

template <typename E>
static cudaError_t launch_fwd_chain_t(const FwdArgs &a, int dtype, cudaStream_t st) {
  using Lay = ChainFwdLayout<E, kChainFW, kChainFL, kChainFS>;
  CUtensorMap km, vm;
  if (!encode_rows(&km, a.k, dtype, a.B * a.T, a.C, Lay::TC) ||
      !encode_rows(&vm, a.v, dtype, a.B * a.T, a.C, Lay::TC))
    return cudaErrorInvalidValue;
  auto kern = fwd_chain_kernel<E, kChainFW, kChainFL, kChainFS>;
  cudaError_t e = prep(kern, Lay::BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)a.nchains, (kChainFW + 1) * 32, Lay::BYTES, st>>>(km, vm, a);
  return cudaGetLastError();
}

template <typename E>
static cudaError_t launch_bwd_chain_t(const BwdArgs &a, int dtype, cudaStream_t st) {
  using Lay = ChainBwdLayout<E, kChainBW, kChainBL, kChainBS>;
  CUtensorMap km, vm, gm;
  if (!encode_rows(&km, a.k, dtype, a.B * a.T, a.C, Lay::TC) ||
      !encode_rows(&vm, a.v, dtype, a.B * a.T, a.C, Lay::TC) ||
      !encode_rows(&gm, a.gy, dtype, a.B * a.T, a.C, Lay::TC))
    return cudaErrorInvalidValue;
  auto kern = bwd_chain_kernel<E, kChainBW, kChainBL, kChainBS>;
  cudaError_t e = prep(kern, Lay::BYTES);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)a.nchains, (kChainBW + 1) * 32, Lay::BYTES, st>>>(km, vm, gm, a);
  return cudaGetLastError();
}

cudaError_t launch_forward_chain(const FwdArgs &a, int dtype, cudaStream_t st) {
  return dtype == 0 ? launch_fwd_chain_t<float>(a, dtype, st) : launch_fwd_chain_t<uint16_t>(a, dtype, st);
}
cudaError_t launch_backward_chain(const BwdArgs &a, int dtype, cudaStream_t st) {
  return dtype == 0 ? launch_bwd_chain_t<float>(a, dtype, st) : launch_bwd_chain_t<uint16_t>(a, dtype, st);
}

}  // namespace wkv
