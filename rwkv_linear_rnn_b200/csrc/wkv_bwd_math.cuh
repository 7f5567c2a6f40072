// wkv_bwd_math.cuh -- per-batch arithmetic of the backward kernels
// (internal): the adjoint record, its reverse-time join and the forward
// recompute of one batch.  The gradient is back-propagation through the
// recurrence of the RWKV review's RNN form ("[논문 리뷰] Reinvention RNNs for
// the Transformer Era: RWKV", section "RNN-유사추론"), taken as a
// reverse-time scan (linear attention post, "상수 메모리 기울기 계산").
#pragma once

#include "wkv_internal.cuh"
#include "wkv_math.cuh"

namespace wkv {

// Adjoint aggregate with the lag-weighted terms used for dL/dw (the same
// record as the chain backward's): Ahat = ah 2^-r, Hhat = hh 2^-r,
// Ahat' = ahp 2^-r, Hhat' = hhp 2^-r.
struct Adj5s {
  float ah, hh, ahp, hhp, r;
};
__device__ __forceinline__ Adj5s adj5s_empty() { return Adj5s{0.f, 0.f, 0.f, 0.f, kEmptyR}; }

// Lane-major adjoint records: (ah, hh, ahp, hhp) as one float4 per lane,
// then r in a plane after them (two loads per lane instead of five).
__device__ __forceinline__ void rec_store_adj(float *desc, int64_t tile, const Adj5s &s, int lane) {
  float *d = desc + tile * kDescFloats;
  __stcg(reinterpret_cast<float4 *>(d) + lane, make_float4(s.ah, s.hh, s.ahp, s.hhp));
  __stcg(d + 128 + lane, s.r);
}
__device__ __forceinline__ Adj5s rec_load_adj(const float *desc, int64_t tile, int lane) {
  const float *d = desc + tile * kDescFloats;
  const float4 v = __ldcg(reinterpret_cast<const float4 *>(d) + lane);
  return Adj5s{v.x, v.y, v.z, v.w, __ldcg(d + 128 + lane)};
}
__device__ __forceinline__ void publish_adj(float *desc, unsigned *flags, int64_t tile, const Adj5s &s,
                                           unsigned epoch, int lane) {
  rec_store_adj(desc, tile, s, lane);
  __syncwarp();
  if (lane == 0) st_release(flags + tile, (epoch_tag(epoch) << 2) | kAgg);
  __syncwarp();
}

// X (earlier, lenX tokens) then Y (later): Y's adjoint decays across X by
// 2^{lenX w2}; its w-derivative gains lenX times Y's adjoint.
__device__ __forceinline__ Adj5s rjoin(const Adj5s &X, const Adj5s &Y, float lenX, float w2) {
  const float rY = fmaf(-lenX, w2, Y.r);
  const float d = X.r - rY;
  const float x = ex2(-fabsf(d));
  const bool xs = d <= 0.f;
  const float fx = xs ? 1.f : x, fy = xs ? x : 1.f;
  Adj5s o;
  o.ah = fmaf(X.ah, fx, Y.ah * fy);
  o.hh = fmaf(X.hh, fx, Y.hh * fy);
  o.ahp = fmaf(X.ahp, fx, fmaf(lenX, Y.ah, Y.ahp) * fy);
  o.hhp = fmaf(X.hhp, fx, fmaf(lenX, Y.hh, Y.hhp) * fy);
  o.r = fminf(X.r, rY);
  return o;
}

// Forward recompute of one batch of RB tokens from the anchored state
// (xa, xb) 2^{xP + xn w2}: per token the scale qv of the denominator
// (D_t = den_t 2^{qv_t}), gam = g / den, eta = gam y and e2 = e^{u+k} / 2^{qv};
// the state advances past the batch.  Batch fast path when every lane allows
// it (see fast_prep), else the per-token rescaled recurrence.
// Returns true (warp-uniform) when the batch ran on the fast path; then M is
// its reference exponent: qv_j = M + j w2e, and e2 2^{-u2 - w2e} is the
// factor 2^{K_j - M - (j+1) w2e} with which token j entered the state.
// WY: Yw[j] is multiplied by the recomputed output y_j (the gated
// backward's dL/dr = grad_o sigma'(r) y).
template <int RB, bool WY>
__device__ __forceinline__ bool recompute_batch(const float (&K)[RB], const float (&V)[RB],
                                                const float (&Gy)[RB], float w2, float u2,
                                                const FastC &fc, float &xa, float &xb, float &xP,
                                                float &xn, float (&qv)[RB], float (&gam)[RB],
                                                float (&eta)[RB], float (&e2v)[RB], float &M,
                                                float (&Yw)[RB]) {
  const float E0 = fmaf(xn, w2, xP);
  float kj[RB];
  const bool ok = fast_prep<RB>(K, E0, u2, fc.w2e, kj, M);
  if (__all_sync(0xffffffffu, ok)) {
    const float s0 = ex2(E0 - M);
    float al = xa * s0, be = xb * s0;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const float e0 = ex2(kj[j] - M);
      const float eu = e0 * fc.cu, ek = e0 * fc.cw;
      const float rden = rcp(be + eu);
      const float y = fmaf(eu, V[j], al) * rden;
      gam[j] = Gy[j] * rden;  // qv is formed by the caller if it needs it: M + j w2e
      eta[j] = gam[j] * y;
      if constexpr (WY) Yw[j] *= y;
      e2v[j] = eu;
      al = fmaf(al, fc.ewm, ek * V[j]);
      be = fmaf(be, fc.ewm, ek);
    }
    xa = al;
    xb = be;
    xP = M;
    xn = fc.nend;
    return true;
  }
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    const float P = fmaf(xn, w2, xP);
    const float UK = u2 + K[j];
    const float d = P - UK;
    const float x = ex2(-fabsf(d));
    const bool pw = d >= 0.f;
    const float e1 = pw ? 1.f : x, e2 = pw ? x : 1.f;
    const float rden = rcp(fmaf(xb, e1, e2));
    const float y = fmaf(xa, e1, V[j] * e2) * rden;
    qv[j] = fmaxf(P, UK);
    gam[j] = Gy[j] * rden;
    eta[j] = gam[j] * y;
    if constexpr (WY) Yw[j] *= y;
    e2v[j] = e2;
    const float n1 = xn + 1.f;
    const float Pc = fmaf(n1, w2, xP);
    const float d2 = K[j] - Pc;
    const float x2 = ex2(-fabsf(d2));
    const bool kw = d2 > 0.f;
    const float so = kw ? x2 : 1.f, snw = kw ? 1.f : x2;
    xa = fmaf(xa, so, V[j] * snw);
    xb = fmaf(xb, so, snw);
    xP = kw ? K[j] : xP;
    xn = kw ? 0.f : n1;
  }
  return false;
}

// dL/dw, dL/du from the per-(segment, batch row) partials [nseg][2][B][C]:
// called by every warp of the launch after a grid barrier.  A channel
// tile's rows are split into `ngroups` groups; each (tile, group) task sums
// its rows in a fixed order in float64, and the last task of a tile to
// finish adds the group sums in group order.  The order is fixed by the
// shapes alone, so the result is bit-reproducible.  The group sums use the
// descriptor region as scratch (the records are dead by then); the tile
// counters must read zero at the barrier.
__device__ __forceinline__ void reduce_wu_partials(const BwdArgs &p, float *gw, float *gu, unsigned *tile_cnt,
                                                   int64_t nseg, int64_t ngroups, int g, int G, int lane) {
  const int64_t C = p.C, BC = p.B * p.C;
  const int64_t R = nseg * p.B;  // partial rows (segment position, b) per channel
  const int64_t ng = ngroups;
  double *scratch = reinterpret_cast<double *>(p.desc);  // records are dead after the barrier
  for (int64_t task = g; task < p.nct * ng; task += G) {
    const int64_t ct = task / ng, grp = task - ct * ng;
    const int64_t c = ct * 32 + lane;
    const int64_t r0 = grp * R / ng, r1 = (grp + 1) * R / ng;
    double sw = 0.0, su = 0.0;
    if (c < C) {
      // rows in fixed order; eight loads in flight per step
      for (int64_t r = r0; r < r1; r += 8) {
        float xw[8], xu[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int64_t rr = min(r + j, r1 - 1);
          const int64_t ps = rr / p.B, bb = rr - ps * p.B;
          xw[j] = __ldcg(p.part + (ps * 2 + 0) * BC + bb * C + c);
          xu[j] = __ldcg(p.part + (ps * 2 + 1) * BC + bb * C + c);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (r + j < r1) {
            sw += (double)xw[j];
            su += (double)xu[j];
          }
        }
      }
    }
    double *dst = scratch + (ct * ng + grp) * 64;
    __stcg(dst + lane, sw);
    __stcg(dst + 32 + lane, su);
    __syncwarp();
    unsigned last = 0;
    if (lane == 0) {
      __threadfence();
      last = atomicAdd(tile_cnt + ct, 1u) == (unsigned)(ng - 1);
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (last) {
      __threadfence();
      double tw = 0.0, tu = 0.0;
      for (int64_t k = 0; k < ng; k += 8) {  // group sums in fixed order, eight loads in flight
        double xw[8], xu[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int64_t kk = min(k + j, ng - 1);
          xw[j] = __ldcg(scratch + (ct * ng + kk) * 64 + lane);
          xu[j] = __ldcg(scratch + (ct * ng + kk) * 64 + 32 + lane);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (k + j < ng) {
            tw += xw[j];
            tu += xu[j];
          }
        }
      }
      if (c < C) {
        gw[c] = (float)tw;
        gu[c] = (float)tu;
      }
    }
  }
}

}  // namespace wkv
