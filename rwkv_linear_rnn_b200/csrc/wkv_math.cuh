// wkv_math.cuh -- per-token arithmetic of the WKV operator shared by the
// forward kernels (internal).  See wkv_internal.cuh for the numerical scheme
// (max-rescaled sums, base-2 exponents, anchored exponent bookkeeping).
#pragma once

#include "wkv_internal.cuh"

namespace wkv {

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(uint16_t h) { return __uint_as_float(((unsigned)h) << 16); }

// Running state of one channel with the anchored exponent P = fma(n, w, Panc).
struct Run {
  float a, b, Panc, n;
};

__device__ __forceinline__ Run run_from(const St &s) { return Run{s.a, s.b, s.P, s.n}; }
__device__ __forceinline__ St run_state(const Run &r) { return St{r.a, r.b, r.Panc, r.n}; }

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

// summarize for a full batch: the maximum exponent by a plain max and the
// state anchored at it with no decay steps (the anchor is one rounding off
// exact, like any exponent formed from an anchored one).
template <int L>
__device__ __forceinline__ St summarize_full(const float (&K)[L], const float (&V)[L], float w2) {
  float e[L];
  float m = -3.0e38f;
#pragma unroll
  for (int j = 0; j < L; ++j) {
    e[j] = fmaf((float)(L - 1 - j), w2, K[j]);
    m = fmaxf(m, e[j]);
  }
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int j = 0; j < L; ++j) {
    const float x = ex2(e[j] - m);
    a = fmaf(x, V[j], a);
    b += x;
  }
  return St{a, b, m, 0.f};
}

// Batch fast path.  Within a batch of RB tokens the state can be held
// against one reference exponent M instead of the running maximum, which
// removes the per-token compare/select chain.  Two per-channel modes:
//   undecayed (RB |w2| < 40): A_t = alpha 2^{M + t w2}; alpha is a plain sum,
//     token j enters with the exactly formed weight 2^{K_j - (j+1) w2 - M},
//     so no rounding accumulates through repeated decay; after the batch the
//     state is (alpha, beta) at the anchored exponent (M, RB);
//   decaying (RB |w2| >= 40): A_t = alpha 2^M, alpha <- alpha 2^{w2} + ...;
//     every old term shrinks by at least 2^-2.5 per token, so the rounding of
//     the repeated factor stays negligible; the state ends at (M, 0).
// With kj_j = K_j - j w2e (w2e = w2 undecayed, 0 decaying) and
// M = max(E0, max_j kj_j), token j costs e0 = 2^{kj_j - M}, eu = e0 2^{u2}
// (the bonus term e^{u+k}), ek = e0 2^{-w2e} (the term that enters the
// state), y = (alpha + eu v) / (beta + eu).  Everything stays in the float
// range when M - min_j kj_j < 100 (every ek >= 2^-100 relative),
// M - min_j (kj_j + u2) < 64 (denominator >= 2^-64) and u2 < 64; the caller
// votes and otherwise runs the batch on the per-token rescaled path.
struct FastC {
  float w2e;   // decay folded into the exponents (undecayed mode) or 0
  float ewm;   // per-token multiplicative decay (decaying mode) or 1
  float cw;    // 2^{-w2e}
  float cu;    // 2^{u2}
  float nend;  // anchored decay count of the state after a batch
};
template <int RB>
__device__ __forceinline__ FastC fast_consts(float w2, float u2) {
  const bool decaying = fabsf(w2) * (float)RB >= 40.f;
  FastC f;
  f.w2e = decaying ? 0.f : w2;
  f.ewm = decaying ? ex2(w2) : 1.f;
  f.cw = ex2(-f.w2e);
  f.cu = ex2(u2);
  f.nend = decaying ? 0.f : (float)RB;
  return f;
}
// kj and the reference M of a batch; true if this lane may take the fast path.
template <int RB>
__device__ __forceinline__ bool fast_prep(const float (&K)[RB], float E0, float u2, float w2e,
                                          float (&kj)[RB], float &M) {
  float mx = E0, mn = 3.0e38f;
#pragma unroll
  for (int j = 0; j < RB; ++j) {
    kj[j] = fmaf(-(float)j, w2e, K[j]);
    mx = fmaxf(mx, kj[j]);
    mn = fminf(mn, kj[j]);
  }
  M = mx;
  return (mx - mn < 100.f) && (mx - mn - u2 < 64.f) && (u2 < 64.f);
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
__device__ __forceinline__ void store_state(float *st, int64_t i, int64_t BC, const St &s,
                                            float w2) {
  st[i] = s.a;
  st[BC + i] = s.b;
  st[2 * BC + i] = st_exp(s, w2) * kLn2;
}
// Checkpoint (base-2 exponent) of the state before token ci * kCkpt.
__device__ __forceinline__ void store_ckpt(float *ck, int64_t ci, int64_t i, int64_t BC,
                                           const St &s, float w2) {
  float *d = ck + ci * 3 * BC;
  d[i] = s.a;
  d[BC + i] = s.b;
  d[2 * BC + i] = st_exp(s, w2);
}

// Summary of a segment from the empty state: the state after its last valid
// token, A = sum_j e^{(n-1-j) w + k_j} v_j.  Exponents are formed directly
// (one fma each) against the segment maximum, so it costs one ex2 per token;
// the maximum is returned in anchored form (its key, decay steps after it).
template <int L>
__device__ __forceinline__ St summarize(const float (&K)[L], const float (&V)[L], float w2,
                                        int nvalid) {
  float e[L];
  float m = kEmptyP, anc = kEmptyP, nanc = 0.f;
  const float last = (float)(nvalid - 1);
#pragma unroll
  for (int j = 0; j < L; ++j) {
    e[j] = fmaf(last - (float)j, w2, K[j]);
    if (j < nvalid && e[j] > m) {
      m = e[j];
      anc = K[j];
      nanc = last - (float)j;
    }
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
  return St{a, b, anc, nanc};
}

}  // namespace wkv
