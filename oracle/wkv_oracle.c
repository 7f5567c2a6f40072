/*
 * wkv_oracle.c -- float64 CPU oracle for the RWKV-4 WKV operator.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the independent checker for the
 * CUDA library: only the test suite, the smoke check and the benchmark's CPU
 * baseline load it.  It shares no code, header or constant with the GPU path.
 * Everything is computed in IEEE double with plain libm `exp`/`log`, no
 * fast-math, no blocking and no reordering beyond what each definition
 * states.
 *
 * Sources (web pages, cited by title and section):
 *   [RWKV review]  "[논문 리뷰] Reinvention RNNs for the Transformer Era: RWKV"
 *                  (velog, BITLAB), sections "WKV 연산자" (eq. wkv_t),
 *                  "RNN-유사추론" (eq. WKV_t and its hidden state A_t, B_t),
 *                  "Transformer-유사학습" (time-parallel mode, WKV as a scan),
 *                  "Background / Transformer" (softmax attention eq.).
 *   [Linear attention post] "Transformers are RNNs: 선형 어텐션으로 만드는 빠른
 *                  자기회귀 트랜스포머" (juhoplayground), section on gradient
 *                  computation (forward cumulative sum, reverse-time
 *                  cumulative sum for the key/value gradients).
 *
 * Conventions (readings of the pages, listed in the design notes):
 *   - time is 0-based, t = 0..T-1; the page writes 1-based sums;
 *   - the decay is passed as w itself (normally w = -exp(time_decay) < 0) and
 *     enters as e^{(t-1-i) w}; the review writes e^{-(t-1-i) w} with w > 0,
 *     the same operator under w -> -w;
 *   - tensors are [B, T, C] row-major with C fastest; w, u are [C];
 *   - a recurrent state is the triple (a, b, p) per (batch, channel), stored
 *     as three planes [3][B][C], meaning A = a * e^p and B = b * e^p, where
 *     A_t, B_t are the review's per-channel hidden sums.  An empty state is
 *     A = B = 0.  State outputs are written in the canonical form
 *     (A/B, 1, ln B), or (0, 0, -inf) when B = 0;
 *   - gradients of w and u are summed over the batch (w, u are per channel).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX(b, t, c) (((b) * T + (t)) * C + (c))

int wkv_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void wkv_oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Initial hidden sums (A_0, B_0) for chain (b, c); zero when no state. */
static void initial_sums(const double *state_in, int64_t B, int64_t C, int64_t b,
                         int64_t c, double *A0, double *B0) {
  if (!state_in) {
    *A0 = 0.0;
    *B0 = 0.0;
    return;
  }
  const double a = state_in[(0 * B + b) * C + c];
  const double bb = state_in[(1 * B + b) * C + c];
  const double p = state_in[(2 * B + b) * C + c];
  const double s = exp(p); /* exp(-inf) = 0 for the empty state */
  *A0 = a * s;
  *B0 = bb * s;
}

static void write_state(double *state_out, int64_t B, int64_t C, int64_t b,
                        int64_t c, double A, double Bs) {
  if (!state_out) return;
  if (Bs > 0.0) {
    state_out[(0 * B + b) * C + c] = A / Bs;
    state_out[(1 * B + b) * C + c] = 1.0;
    state_out[(2 * B + b) * C + c] = log(Bs);
  } else {
    state_out[(0 * B + b) * C + c] = 0.0;
    state_out[(1 * B + b) * C + c] = 0.0;
    state_out[(2 * B + b) * C + c] = -INFINITY;
  }
}

/* ------------------------------------------------------------------------
 * Direct O(T^2) forward: the defining sum, eq. wkv_t of [RWKV review]
 * (section "WKV 연산자"), evaluated per output t as a normalised, shifted
 * exponential average (log-sum-exp shift by the largest exponent):
 *
 *   y_t = ( sum_{i<t} e^{(t-1-i) w + k_i} v_i + e^{u + k_t} v_t + e^{t w} A_0 )
 *       / ( sum_{i<t} e^{(t-1-i) w + k_i}     + e^{u + k_t}     + e^{t w} B_0 )
 *
 * The A_0/B_0 term is the initial hidden state decayed t times (it is absent
 * for the empty state the page assumes).
 * ------------------------------------------------------------------------ */
static double direct_one(int64_t T, int64_t C, const double *kc, const double *vc,
                         double w, double u, int has_state, double a0, double b0,
                         double p0, int64_t t, double *den_out,
                         double *mexp_out) {
  (void)T;
  /* largest exponent among the terms of y_t */
  double m = u + kc[t * C];
  for (int64_t i = 0; i < t; ++i) {
    const double s = (double)(t - 1 - i) * w + kc[i * C];
    if (s > m) m = s;
  }
  if (has_state && p0 + (double)t * w > m) m = p0 + (double)t * w;
  double num = 0.0, den = 0.0;
  for (int64_t i = 0; i < t; ++i) {
    const double e = exp((double)(t - 1 - i) * w + kc[i * C] - m);
    num += e * vc[i * C];
    den += e;
  }
  {
    const double e = exp(u + kc[t * C] - m);
    num += e * vc[t * C];
    den += e;
  }
  if (has_state) {
    const double e = exp(p0 + (double)t * w - m);
    num += a0 * e;
    den += b0 * e;
  }
  if (den_out) *den_out = den;
  if (mexp_out) *mexp_out = m;
  return num / den;
}

static void state_triplet(const double *state_in, int64_t B, int64_t C, int64_t b,
                          int64_t c, int *has, double *a0, double *b0, double *p0) {
  if (!state_in) {
    *has = 0;
    *a0 = *b0 = 0.0;
    *p0 = -INFINITY;
    return;
  }
  *a0 = state_in[(0 * B + b) * C + c];
  *b0 = state_in[(1 * B + b) * C + c];
  *p0 = state_in[(2 * B + b) * C + c];
  *has = isfinite(*p0) && (*a0 != 0.0 || *b0 != 0.0);
}

void wkv_oracle_fwd_direct(int64_t B, int64_t T, int64_t C, const double *w,
                           const double *u, const double *k, const double *v,
                           const double *state_in, double *y) {
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t c = 0; c < C; ++c) {
      int has;
      double a0, b0, p0;
      state_triplet(state_in, B, C, b, c, &has, &a0, &b0, &p0);
      const double *kc = k + IDX(b, 0, c);
      const double *vc = v + IDX(b, 0, c);
      for (int64_t t = 0; t < T; ++t)
        y[IDX(b, t, c)] =
            direct_one(T, C, kc, vc, w[c], u[c], has, a0, b0, p0, t, NULL, NULL);
    }
}

/* Direct evaluation at sampled points (b[j], t[j], c[j]), O(t) each; used to
 * check large problems without the O(T^2) cost of the full direct form. */
void wkv_oracle_fwd_points(int64_t B, int64_t T, int64_t C, const double *w,
                           const double *u, const double *k, const double *v,
                           const double *state_in, int64_t npts,
                           const int64_t *pb, const int64_t *pt,
                           const int64_t *pc, double *y) {
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t j = 0; j < npts; ++j) {
    const int64_t b = pb[j], t = pt[j], c = pc[j];
    int has;
    double a0, b0, p0;
    state_triplet(state_in, B, C, b, c, &has, &a0, &b0, &p0);
    y[j] = direct_one(T, C, k + IDX(b, 0, c), v + IDX(b, 0, c), w[c], u[c], has,
                      a0, b0, p0, t, NULL, NULL);
  }
}

/* ------------------------------------------------------------------------
 * Recurrent forward: eq. WKV_t of [RWKV review] (section "RNN-유사추론"),
 *
 *   y_t = (A_t + e^{u + k_t} v_t) / (B_t + e^{u + k_t}),
 *
 * with the hidden sums advanced one token at a time.  The page does not print
 * the update of A_t, B_t; the one consistent with eq. wkv_t (A_t is the sum
 * over i < t of e^{(t-1-i) w + k_i} v_i) is
 *
 *   A_{t+1} = e^w A_t + e^{k_t} v_t,   B_{t+1} = e^w B_t + e^{k_t}.
 *
 * Plain (unscaled) sums in double: exponents in the intended inputs stay far
 * below the double range.
 * ------------------------------------------------------------------------ */
void wkv_oracle_fwd_recur(int64_t B, int64_t T, int64_t C, const double *w,
                          const double *u, const double *k, const double *v,
                          const double *state_in, double *y, double *state_out) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t c = 0; c < C; ++c) {
      double A, Bs;
      initial_sums(state_in, B, C, b, c, &A, &Bs);
      const double ew = exp(w[c]);
      for (int64_t t = 0; t < T; ++t) {
        const double kt = k[IDX(b, t, c)], vt = v[IDX(b, t, c)];
        const double e_cur = exp(u[c] + kt);
        if (y) y[IDX(b, t, c)] = (A + e_cur * vt) / (Bs + e_cur);
        const double e_k = exp(kt);
        A = ew * A + e_k * vt;
        Bs = ew * Bs + e_k;
      }
      write_state(state_out, B, C, b, c, A, Bs);
    }
}

/* One RNN-mode step ([RWKV review] "자기 회귀 디코딩", steps 4 and 7):
 * output y from the stored state and the new (k, v), then the stored state
 * advanced by one token.  Shapes: k, v, y are [N, C]; states [3][N][C]. */
void wkv_oracle_step(int64_t N, int64_t C, const double *w, const double *u,
                     const double *k, const double *v, const double *state_in,
                     double *y, double *state_out) {
  const int64_t T = 1;
  wkv_oracle_fwd_recur(N, T, C, w, u, k, v, state_in, y, state_out);
}

/* ------------------------------------------------------------------------
 * Direct backward: derivatives of the defining sum.  With
 *   alpha_{t,i} = (weight of v_i in y_t) = e^{s_{t,i}} / D_t,
 *   s_{t,i} = (t-1-i) w + k_i (i < t),  s_{t,t} = u + k_t,
 * and g_t = dL/dy_t:
 *   dL/dv_i = sum_{t>=i} g_t alpha_{t,i}
 *   dL/dk_i = sum_{t>=i} g_t alpha_{t,i} (v_i - y_t)
 *   dL/du   = sum_{b,t} g_t alpha_{t,t} (v_t - y_t)
 *   dL/dw   = sum_{b,t} g_t [ sum_{i<t} (t-1-i) alpha_{t,i} (v_i - y_t)
 *                             + t e^{t w} (A_0 - B_0 y_t) / D_t ]
 * (the last term only with an initial state).  This is the softmax Jacobian
 * of the masked attention form ([RWKV review], "Background / Transformer").
 * ------------------------------------------------------------------------ */
void wkv_oracle_bwd_direct(int64_t B, int64_t T, int64_t C, const double *w,
                           const double *u, const double *k, const double *v,
                           const double *state_in, const double *gy, double *gw,
                           double *gu, double *gk, double *gv) {
  double *pw = (double *)calloc((size_t)(B * C), sizeof(double));
  double *pu = (double *)calloc((size_t)(B * C), sizeof(double));
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
  for (int64_t b = 0; b < B; ++b)
    for (int64_t c = 0; c < C; ++c) {
      int has;
      double a0, b0, p0;
      state_triplet(state_in, B, C, b, c, &has, &a0, &b0, &p0);
      const double *kc = k + IDX(b, 0, c);
      const double *vc = v + IDX(b, 0, c);
      const double wc = w[c], uc = u[c];
      for (int64_t i = 0; i < T; ++i) {
        gk[IDX(b, i, c)] = 0.0;
        gv[IDX(b, i, c)] = 0.0;
      }
      double sw = 0.0, su = 0.0;
      for (int64_t t = 0; t < T; ++t) {
        double den, m;
        const double yt = direct_one(T, C, kc, vc, wc, uc, has, a0, b0, p0, t, &den, &m);
        const double g = gy[IDX(b, t, c)];
        double dw = 0.0;
        for (int64_t i = 0; i < t; ++i) {
          const double alpha = exp((double)(t - 1 - i) * wc + kc[i * C] - m) / den;
          gv[IDX(b, i, c)] += g * alpha;
          gk[IDX(b, i, c)] += g * alpha * (vc[i * C] - yt);
          dw += (double)(t - 1 - i) * alpha * (vc[i * C] - yt);
        }
        {
          const double alpha = exp(uc + kc[t * C] - m) / den;
          gv[IDX(b, t, c)] += g * alpha;
          gk[IDX(b, t, c)] += g * alpha * (vc[t * C] - yt);
          su += g * alpha * (vc[t * C] - yt);
        }
        if (has) {
          const double e = exp(p0 + (double)t * wc - m) / den;
          dw += (double)t * e * (a0 - b0 * yt);
        }
        sw += g * dw;
      }
      pw[b * C + c] = sw;
      pu[b * C + c] = su;
    }
  for (int64_t c = 0; c < C; ++c) {
    double sw = 0.0, su = 0.0;
    for (int64_t b = 0; b < B; ++b) {
      sw += pw[b * C + c];
      su += pu[b * C + c];
    }
    gw[c] = sw;
    gu[c] = su;
  }
  free(pw);
  free(pu);
}

/* ------------------------------------------------------------------------
 * Recurrent backward (back-propagation through time of the RNN form).
 * Forward sums as in wkv_oracle_fwd_recur; then, walking t from T-1 down to
 * 0 with the adjoints Ah = dL/dA_{t+1}, Bh = dL/dB_{t+1} (zero after the last
 * token):
 *   dL/dv_t = g_t e^{u+k_t} / D_t              + e^{k_t} Ah
 *   dL/dk_t = g_t e^{u+k_t} (v_t - y_t) / D_t  + e^{k_t} (v_t Ah + Bh)
 *   dL/du  += g_t e^{u+k_t} (v_t - y_t) / D_t
 *   dL/dw  += e^w (A_t Ah + B_t Bh)
 *   Ah <- g_t / D_t + e^w Ah,   Bh <- -g_t y_t / D_t + e^w Bh
 * where D_t = B_t + e^{u+k_t}.  The reverse walk is the structure the
 * [Linear attention post] gives for its key/value gradients (a reverse-time
 * cumulative sum), here with the WKV decay e^w between steps.
 * ------------------------------------------------------------------------ */
void wkv_oracle_bwd_recur(int64_t B, int64_t T, int64_t C, const double *w,
                          const double *u, const double *k, const double *v,
                          const double *state_in, const double *gy, double *gw,
                          double *gu, double *gk, double *gv) {
  double *pw = (double *)calloc((size_t)(B * C), sizeof(double));
  double *pu = (double *)calloc((size_t)(B * C), sizeof(double));
#pragma omp parallel
  {
    double *As = (double *)malloc(sizeof(double) * (size_t)(T + 1));
    double *Bv = (double *)malloc(sizeof(double) * (size_t)(T + 1));
#pragma omp for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
      for (int64_t c = 0; c < C; ++c) {
        const double wc = w[c], uc = u[c], ew = exp(wc);
        initial_sums(state_in, B, C, b, c, &As[0], &Bv[0]);
        for (int64_t t = 0; t < T; ++t) {
          const double e_k = exp(k[IDX(b, t, c)]);
          As[t + 1] = ew * As[t] + e_k * v[IDX(b, t, c)];
          Bv[t + 1] = ew * Bv[t] + e_k;
        }
        double Ah = 0.0, Bh = 0.0, sw = 0.0, su = 0.0;
        for (int64_t t = T - 1; t >= 0; --t) {
          const double kt = k[IDX(b, t, c)], vt = v[IDX(b, t, c)];
          const double g = gy[IDX(b, t, c)];
          const double e_cur = exp(uc + kt), e_k = exp(kt);
          const double D = Bv[t] + e_cur;
          const double yt = (As[t] + e_cur * vt) / D;
          gv[IDX(b, t, c)] = g * e_cur / D + e_k * Ah;
          gk[IDX(b, t, c)] = g * e_cur * (vt - yt) / D + e_k * (vt * Ah + Bh);
          su += g * e_cur * (vt - yt) / D;
          sw += ew * (As[t] * Ah + Bv[t] * Bh);
          Ah = g / D + ew * Ah;
          Bh = -g * yt / D + ew * Bh;
        }
        pw[b * C + c] = sw;
        pu[b * C + c] = su;
      }
    free(As);
    free(Bv);
  }
  for (int64_t c = 0; c < C; ++c) {
    double sw = 0.0, su = 0.0;
    for (int64_t b = 0; b < B; ++b) {
      sw += pw[b * C + c];
      su += pu[b * C + c];
    }
    gw[c] = sw;
    gu[c] = su;
  }
  free(pw);
  free(pu);
}

/*
 * Back-propagation through the recurrence with the state terms, for
 * sequences split across calls (truncated BPTT, the RNN mode of [RWKV
 * review] "RNN-유사추론" carried between calls):
 *   gA_T, gB_T  [B][C] dL/dA_T, dL/dB_T for the hidden sums after the last
 *               token (NULL: no loss term on the final state);
 *   gA_0, gB_0  [B][C] receive dL/dA_0, dL/dB_0 for the sums before token 0
 *               (NULL: not wanted).
 * The same reverse walk as wkv_oracle_bwd_recur, started from the given
 * adjoints instead of zero; every other output is as there.
 */
void wkv_oracle_bwd_recur_state(int64_t B, int64_t T, int64_t C, const double *w,
                                const double *u, const double *k, const double *v,
                                const double *state_in, const double *gy, const double *gA_T,
                                const double *gB_T, double *gw, double *gu, double *gk,
                                double *gv, double *gA_0, double *gB_0) {
  double *pw = (double *)calloc((size_t)(B * C), sizeof(double));
  double *pu = (double *)calloc((size_t)(B * C), sizeof(double));
#pragma omp parallel
  {
    double *As = (double *)malloc(sizeof(double) * (size_t)(T + 1));
    double *Bv = (double *)malloc(sizeof(double) * (size_t)(T + 1));
#pragma omp for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b)
      for (int64_t c = 0; c < C; ++c) {
        const double wc = w[c], uc = u[c], ew = exp(wc);
        initial_sums(state_in, B, C, b, c, &As[0], &Bv[0]);
        for (int64_t t = 0; t < T; ++t) {
          const double e_k = exp(k[IDX(b, t, c)]);
          As[t + 1] = ew * As[t] + e_k * v[IDX(b, t, c)];
          Bv[t + 1] = ew * Bv[t] + e_k;
        }
        /* adjoints of A_T, B_T: the loss term on the final state */
        double Ah = gA_T ? gA_T[b * C + c] : 0.0;
        double Bh = gB_T ? gB_T[b * C + c] : 0.0;
        double sw = 0.0, su = 0.0;
        for (int64_t t = T - 1; t >= 0; --t) {
          const double kt = k[IDX(b, t, c)], vt = v[IDX(b, t, c)];
          const double g = gy[IDX(b, t, c)];
          const double e_cur = exp(uc + kt), e_k = exp(kt);
          const double D = Bv[t] + e_cur;
          const double yt = (As[t] + e_cur * vt) / D;
          gv[IDX(b, t, c)] = g * e_cur / D + e_k * Ah;
          gk[IDX(b, t, c)] = g * e_cur * (vt - yt) / D + e_k * (vt * Ah + Bh);
          su += g * e_cur * (vt - yt) / D;
          sw += ew * (As[t] * Ah + Bv[t] * Bh);
          Ah = g / D + ew * Ah;
          Bh = -g * yt / D + ew * Bh;
        }
        pw[b * C + c] = sw;
        pu[b * C + c] = su;
        if (gA_0) gA_0[b * C + c] = Ah;
        if (gB_0) gB_0[b * C + c] = Bh;
      }
    free(As);
    free(Bv);
  }
  for (int64_t c = 0; c < C; ++c) {
    double sw = 0.0, su = 0.0;
    for (int64_t b = 0; b < B; ++b) {
      sw += pw[b * C + c];
      su += pu[b * C + c];
    }
    gw[c] = sw;
    gu[c] = su;
  }
  free(pw);
  free(pu);
}
