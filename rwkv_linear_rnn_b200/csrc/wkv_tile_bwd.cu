// wkv_tile_bwd.cu -- tile backward of libwkv (the default backward on
// sm_100a when the [B, T, C] rows are 16-byte aligned): dL/dk, dL/dv,
// dL/dw, dL/du in one launch.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"); the gradient is
// back-propagation through the recurrence of section "RNN-유사추론", taken in
// the reverse-time scan form of the linear attention post ("Transformers are
// RNNs: 선형 어텐션으로 만드는 빠른 자기회귀 트랜스포머", section "상수 메모리
// 기울기 계산": the cumulative sums behind the key and value gradients run
// backwards in time).
//
// With D_t the denominator, G_t = g_t / D_t and H_t = g_t y_t / D_t, the
// adjoints of the past sums obey Ahat_t = G_t + e^w Ahat_{t+1} (and Hhat
// likewise), a linear recurrence with a constant factor, so the time axis
// splits into units whose adjoint aggregates join associatively (rjoin).  A
// unit is one chain (batch row b, 32 channels = lanes) and L tokens; warps
// are persistent and own units statically in reverse position order (every
// chain's last unit first).  Per unit:
//   load    TMA copies bring the unit's k, v and grad_y tiles into the warp's
//           shared memory; the next unit's copies go into the other buffer
//           before this unit is computed;
//   pass 1  forward recompute from the checkpoint at the unit start (the
//           state at every batch start kept in shared memory) and the unit's
//           adjoint aggregate;
//   join    the aggregate is published, then the adjoint at the unit end is
//           formed by a decoupled look-back over the chain's later units:
//           the nearest published inclusive suffix, then the aggregates
//           between, folded in scan order (bit-reproducible, as the forward);
//   pass 2  batches last to first: recompute from the saved state, reverse
//           sweep; dL/dk, dL/dv overwrite k, v in shared memory and leave by
//           TMA stores; per-unit partials of dL/dw, dL/du.
// dL/dw and dL/du are summed in a fixed order by the last unit of each chain
// and the last chain of each channel tile to finish, with no grid barrier.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "wkv_bwd_math.cuh"
#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_tile.cuh"

// Build-time knobs of the ungated kernels: the blocks per SM their
// registers are sized for, and the tokens per unit for bf16 tensors.
#ifndef WKV_TILEB_MINB
#define WKV_TILEB_MINB 2
#endif
#ifndef WKV_TILEB_LBF16
#define WKV_TILEB_LBF16 kTileLBF16
#endif
#ifndef WKV_TILEB_RB
#define WKV_TILEB_RB 8
#endif

namespace wkv {

bool encode_btc(CUtensorMap *m, const void *ptr, int dtype, int64_t B, int64_t T, int64_t C, int box_t);

struct TileBwdArgs {
  BwdArgs p;
  float *gw, *gu;
  float4 *chain_sum;        // [B][C] per-chain sums, then [ceil(nseg/16)][B][C] first-level sums
  float4 *rec;         // [units][2 slots][2 words][32 lanes] tagged adjoint records
  int64_t nseg;        // units per chain
};


// Adjoint records, 2 KB per unit, tagged as the forward's (see wkv_tile.cuh):
// slot 0 the unit's aggregate, slot 1 its inclusive suffix (the adjoint at
// the unit's start from everything after it), each in two 16-byte words per
// lane, (ah, hh, ahp, tag) and (hhp, r, tag, 0).
constexpr int kBwdRecWords = 128;
__device__ __forceinline__ void adj_put(float4 *rec, int64_t unit, int slot, const Adj5s &s, unsigned tag,
                                        int lane) {
  float4 *d = rec + unit * kBwdRecWords + slot * 64 + lane;
  st_relaxed_v4(d, make_float4(s.ah, s.hh, s.ahp, tagf(tag)));
  st_relaxed_v4(d + 32, make_float4(s.hhp, s.r, tagf(tag), 0.f));
}
// Loads a record; `ok` is cleared unless both of this lane's words carry `tag`.
__device__ __forceinline__ Adj5s adj_get(const float4 *rec, int64_t unit, int slot, unsigned tag, int lane,
                                         bool &ok) {
  const float4 *d = rec + unit * kBwdRecWords + slot * 64 + lane;
  const float4 x = ld_relaxed_v4(d), y = ld_relaxed_v4(d + 32);
  ok = ok && tag_is(x.w, tag) && tag_is(y.z, tag);
  return Adj5s{x.x, x.y, x.z, y.x, y.y};
}

// The adjoint at the end of the unit at scan position rpos (rpos 0 = the
// chain's last unit): the fold, in scan order from the adjoint after the
// chain's last token, of the aggregates of scan positions 0 .. rpos-1, found
// and checked as in the forward's look-back.  Scan position 0 holds `nlast`
// tokens, the others L.  Bounded like the forward's.
__device__ Adj5s tile_lookback_adj(const unsigned *status, const float4 *rec, int rpos, int chain, int nchains,
                                   unsigned epoch, const Adj5s &a_end, float len, float nlast, float w2,
                                   int64_t budget_ns, WsHeader *hdr, int lane, bool &failed) {
  const unsigned t_agg = tile_flag(epoch, kFlagAgg), t_inc = tile_flag(epoch, kFlagInc);
  const int q = rpos - 1 - lane;
  const unsigned *sw = status + (int64_t)(q < 0 ? 0 : q) * nchains + chain;
  const uint64_t t0 = global_ns();
  unsigned backoff = 32;
  Adj5s acc = a_end;
  for (;;) {
    unsigned st = 2u;
    if (q >= 0) {
      const unsigned f = ld_relaxed(sw);
      st = f == t_inc ? 2u : (f == t_agg ? 1u : 0u);
    }
    const unsigned inc = __ballot_sync(0xffffffffu, st == 2u);
    const unsigned none = __ballot_sync(0xffffffffu, st == 0u);
    const int first = inc ? __ffs(inc) - 1 : 32;
    if (first < 32 && (none & ((1u << first) - 1u)) == 0u) {
      const int q0 = rpos - 1 - first;
      bool ok = true;
      acc = q0 < 0 ? a_end : adj_get(rec, (int64_t)q0 * nchains + chain, 1, t_inc, lane, ok);
#pragma unroll 1
      for (int d0 = 0; d0 < first; d0 += 4) {
        Adj5s r[4];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          if (d0 + jj < first) r[jj] = adj_get(rec, (int64_t)(q0 + 1 + d0 + jj) * nchains + chain, 0, t_agg, lane, ok);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int m = q0 + 1 + d0 + jj;
          if (d0 + jj < first) acc = rjoin(r[jj], acc, m == 0 ? nlast : len, w2);
        }
      }
      if (__all_sync(0xffffffffu, ok)) return acc;
    }
    if (failed || (int64_t)(global_ns() - t0) > budget_ns || launch_aborted(hdr, epoch)) {
      if (lane == 0) raise_timeout(hdr, epoch);
      failed = true;
      return acc;
    }
    __nanosleep(backoff);
    backoff = backoff < 256u ? backoff * 2u : 256u;
  }
}

// Shared memory per block: every warp's two buffers of NARR tiles [L][32]
// (k, v, grad_y, and r when gated); then per warp the forward state at each
// batch start of the current unit, [L/RB][3][32] floats; then two mbarriers
// per warp.
template <typename E, int L, int RB, int NARR>
struct TileBwdLayout {
  static constexpr int ARR = L * 32 * (int)sizeof(E);
  static constexpr int BUF = NARR * ARR;
  static constexpr int WARP = 2 * BUF;
  static constexpr int STS = (L / RB) * 96 * 4;
  static_assert(ARR % 128 == 0 && STS % 16 == 0, "TMA destinations stay 128-byte aligned");
  static constexpr int bytes(int nw) { return nw * (WARP + STS + 16); }
};

// STATE: the state terms of a sequence split across calls: the folds start
// from the adjoint after the last token (the final state's gradient), the
// chain's last unit sweeps exactly to token T-1 (its zero-filled padding would
// decay that adjoint), and the first unit writes the initial state's gradient.
// GATE: the loss depends on o = sigma(r) * y; grad_y is dL/do.  Pass 1 reads
// grad_o and r with k, v, forms the WKV gradient grad_o sigma(r) for its
// aggregate and leaves it in grad_o's tile (in the tensor's element type) for
// pass 2, and forms dL/dr = grad_o sigma'(r) y from its recompute into r's
// tile, which leaves by TMA with dL/dk and dL/dv.  Nothing but the
// algorithmic bytes crosses HBM.
template <typename E, int L, int RB, int NW, bool STATE, bool GATE>
__global__ void __launch_bounds__(NW * 32, NW == 4 ? WKV_TILEB_MINB : 3) bwd_tile_kernel(const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap,
                                                           const __grid_constant__ CUtensorMap gmap,
                                                           const __grid_constant__ CUtensorMap rmap,
                                                           const __grid_constant__ CUtensorMap gkmap,
                                                           const __grid_constant__ CUtensorMap gvmap,
                                                           const __grid_constant__ CUtensorMap grmap,
                                                           TileBwdArgs a) {
  static_assert(L % kCkpt == 0 && kCkpt % RB == 0, "units start on checkpoints");
  static_assert(!(STATE && GATE), "no entry point combines the state terms and the gate");
  constexpr int NB = L / RB;
  constexpr int NARR = GATE ? 4 : 3;
  using Lay = TileBwdLayout<E, L, RB, NARR>;
  const BwdArgs &p = a.p;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = NW;
  unsigned char *wbuf = smem + (size_t)wl * Lay::WARP;
  float *sts = reinterpret_cast<float *>(smem + (size_t)nw * Lay::WARP + (size_t)wl * Lay::STS);
  const uint32_t bar0 = smem_addr(smem + (size_t)nw * (Lay::WARP + Lay::STS)) + 16u * wl;
  if (lane == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8u, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const int G = (int)gridDim.x * nw;
  const int g = (int)blockIdx.x * nw + wl;
  const int nseg = (int)a.nseg, nchains = (int)p.nchains, nct = (int)p.nct;
  const int total = nseg * nchains;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  const uint64_t pol = l2_policy_evict_first();
  const int nlast = (int)(T - (int64_t)(nseg - 1) * L);  // tokens of a chain's last unit

  auto issue = [&](int unit, int bf) {
    const int rpos = unit / nchains, chain = unit - rpos * nchains;
    const int b = chain / nct;
    const int x = (chain - b * nct) * 32;
    const int y = (nseg - 1 - rpos) * L;
    const uint32_t dst = smem_addr(wbuf + (size_t)bf * Lay::BUF), bar = bar0 + 8u * bf;
    mbar_expect_tx(bar, (uint32_t)Lay::BUF);
    tma_load_3d(dst, &kmap, x, y, b, bar, pol);
    tma_load_3d(dst + Lay::ARR, &vmap, x, y, b, bar, pol);
    tma_load_3d(dst + 2 * Lay::ARR, &gmap, x, y, b, bar, pol);
    if constexpr (GATE) tma_load_3d(dst + 3 * Lay::ARR, &rmap, x, y, b, bar, pol);
  };
  int iss_it = -1, wt_it = -1;
  if (lane == 0 && g < total) {
    issue(g, 0);
    iss_it = 0;
  }
  bool failed = false;
  int it = 0;
#pragma unroll 1
  for (int unit = g; unit < total; unit += G, ++it) {
    const int bf = it & 1;
    const int rpos = unit / nchains, chain = unit - rpos * nchains;
    const int b = chain / nct;
    const int x0 = (chain - b * nct) * 32;
    const int64_t c = (int64_t)x0 + lane;
    const bool cok = c < C;
    const int pos = nseg - 1 - rpos;
    const int64_t t0 = (int64_t)pos * L;
    const int n = (int)min((int64_t)L, T - t0);
    const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
    const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
    const int64_t bc = (int64_t)b * C + c;
    const FastC fc = fast_consts<RB>(w2, u2);
    E *kt = reinterpret_cast<E *>(wbuf + (size_t)bf * Lay::BUF) + lane;
    E *vt = kt + L * 32;
    E *gt = kt + 2 * L * 32;
    E *rt = kt + 3 * L * 32;  // gate input, then dL/dr (GATE only)
    if (!failed) {
      if (mbar_wait(bar0 + 8u * bf, (uint32_t)(it >> 1) & 1u, budget, nullptr)) {
        wt_it = it;
      } else {
        failed = true;
        if (lane == 0) raise_timeout(p.hdr, epoch);
      }
    }
    auto load_batch = [&](int bt, float(&K)[RB], float(&V)[RB], float(&Gy)[RB]) {
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        K[j] = to_f32(kt[(bt * RB + j) * 32]) * kLog2e;
        V[j] = to_f32(vt[(bt * RB + j) * 32]);
        Gy[j] = to_f32(gt[(bt * RB + j) * 32]);
      }
    };

    // ---- pass 1: forward recompute and the unit's adjoint aggregate
    float fa = 0.f, fb = 0.f, fP = kEmptyP, fn = 0.f;
    if (cok) {
      const float *ck = p.ckpt + (t0 / kCkpt) * 3 * BC + bc;
      fa = ck[0];
      fb = ck[BC];
      fP = ck[2 * BC];
    }
    float ah = 0.f, hh = 0.f, ahp = 0.f, hhp = 0.f, Em = -kEmptyR;
#pragma unroll 1
    for (int bt = 0; bt < NB; ++bt) {
      sts[bt * 96 + lane] = fa;
      sts[bt * 96 + 32 + lane] = fb;
      sts[bt * 96 + 64 + lane] = fmaf(fn, w2, fP);
      float K[RB], V[RB], Gy[RB], Gd[RB];
      load_batch(bt, K, V, Gy);
      if constexpr (GATE) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          float sg, ds;
          gate_sigmoid_slope(to_f32(rt[(bt * RB + j) * 32]), sg, ds);
          Gd[j] = Gy[j] * ds;
          Gy[j] *= sg;
        }
      }
      float qv[RB], gam[RB], eta[RB], e2v[RB], Mb;
      const bool fast =
          recompute_batch<RB, GATE>(K, V, Gy, w2, u2, fc, fa, fb, fP, fn, qv, gam, eta, e2v, Mb, Gd);
      if constexpr (GATE) {
        // the WKV gradient for pass 2 and dL/dr = grad_o sigma'(r) y, in place
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          gt[(bt * RB + j) * 32] = from_f32<E>(Gy[j]);
          rt[(bt * RB + j) * 32] = from_f32<E>(Gd[j]);
        }
      }
      const float lag0 = (float)(bt * RB);
      if (fast) {
        // token j's aggregate exponent is lag0 w2 - M + j (w2 - w2e): a batch
        // constant times (2^{w2 - w2e})^j, so the batch enters as four sums
        float f = 1.f, sg = 0.f, se = 0.f, sgl = 0.f, sel = 0.f;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const float gf = gam[j] * f, ef = eta[j] * f;
          sg += gf;
          se += ef;
          sgl = fmaf((float)j, gf, sgl);
          sel = fmaf((float)j, ef, sel);
          f *= fc.ewm;
        }
        const float es = fmaf(lag0, w2, -Mb);
        const float da = es - Em;
        const float xa = ex2(-fabsf(da));
        const bool up = da > 0.f;
        const float fo = up ? xa : 1.f, fg = up ? 1.f : xa;
        ah = fmaf(ah, fo, sg * fg);
        hh = fmaf(hh, fo, se * fg);
        ahp = fmaf(ahp, fo, fmaf(lag0, sg, sgl) * fg);
        hhp = fmaf(hhp, fo, fmaf(lag0, se, sel) * fg);
        Em = up ? es : Em;
        continue;
      }
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        // token s = t0 + lag enters the aggregate with 2^{lag w2 - q_s}
        const float lag = lag0 + (float)j;
        const float es = fmaf(lag, w2, -qv[j]);
        const float da = es - Em;
        const float xa = ex2(-fabsf(da));
        const bool up = da > 0.f;
        const float fo = up ? xa : 1.f, fg = up ? 1.f : xa;
        const float gg = gam[j] * fg, ee = eta[j] * fg;
        ah = fmaf(ah, fo, gg);
        hh = fmaf(hh, fo, ee);
        ahp = fmaf(ahp, fo, lag * gg);
        hhp = fmaf(hhp, fo, lag * ee);
        Em = up ? es : Em;
      }
    }
    const Adj5s agg{ah, hh, ahp, hhp, -Em};
    // the next unit's tiles go into the other buffer, once the stores that
    // last read it are done reading (issued after pass 1, by when they are)
    if (lane == 0 && unit + G < total && !failed) {
      bulk_wait_read_all();
      issue(unit + G, bf ^ 1);
      iss_it = it + 1;
    }

    // ---- join: the adjoint at the unit end
    const bool has_next = rpos + 1 < nseg;
    const bool held = p.hold_first && rpos == 0;  // test hook: never publish
    Adj5s acc = adj5s_empty();
    if constexpr (STATE) {
      if (p.gs_out && cok) end_adjoint(p.gs_out[bc], p.gs_out[BC + bc], p.p_out[bc], acc.ah, acc.hh, acc.r);
    }
    if (rpos > 0) {
      if (has_next && !held) {
        const unsigned t = tile_flag(epoch, kFlagAgg);
        adj_put(a.rec, unit, 0, agg, t, lane);
        if (lane == 0) st_relaxed_u32(p.flags + unit, t);
      }
      acc = tile_lookback_adj(p.flags, a.rec, rpos, chain, nchains, epoch, acc, (float)L, (float)nlast, w2, budget,
                              p.hdr, lane, failed);
    }
    if (has_next && !held) {
      const unsigned t = tile_flag(epoch, kFlagInc);
      adj_put(a.rec, unit, 1, rjoin(agg, acc, (float)n, w2), t, lane);
      if (lane == 0) st_relaxed_u32(p.flags + unit, t);
    }

    // ---- pass 2: batches last to first, recompute then reverse sweep
    float gw_acc = 0.f, gu_acc = 0.f;
    float rah = acc.ah, rhh = acc.hh, rahp = acc.ahp, rhhp = acc.hhp, Ranc = acc.r, m = 0.f;
#pragma unroll 1
    for (int bi = 0; bi < NB; ++bi) {
      const int bt = NB - 1 - bi;
      const int nb = n - bt * RB;  // valid tokens of the batch (may be <= 0 in a chain's last unit)
      if constexpr (STATE) {
        if (nb <= 0) continue;  // only padding past T: nothing to sweep
      }
      float K[RB], V[RB], Gy[RB], Gd[RB];
      load_batch(bt, K, V, Gy);
      float qv[RB], gam[RB], eta[RB], e2v[RB], Mb;
      bool fast;
      {
        float xa = sts[bt * 96 + lane], xb = sts[bt * 96 + 32 + lane], xP = sts[bt * 96 + 64 + lane];
        float xn = 0.f;
        fast = recompute_batch<RB, false>(K, V, Gy, w2, u2, fc, xa, xb, xP, xn, qv, gam, eta, e2v, Mb, Gd);
      }
      E *gkp = kt + bt * RB * 32;
      E *gvp = vt + bt * RB * 32;
      // Fast sweep: the adjoint in the batch's coordinates, a_t = A_t 2^{M + t w2e},
      // obeys a_t = gam_t + ewm a_{t+1} (and a'_t = ewm (a'_{t+1} + a_{t+1}) for
      // the lag-weighted one); e^{k_t} A_{t+1} = ek_t a_{t+1}.  The carried
      // adjoint enters scaled by 2^{M + RB w2e - r}, bounded for the float range.
      const float rn_end = fmaf(-m, w2, Ranc);
      const float xin = fmaf((float)RB, fc.w2e, Mb) - rn_end;
      if (__all_sync(0xffffffffu, fast && xin < 100.f && (!STATE || nb >= RB))) {
        const float F = ex2(xin);
        float ra = rah * F, rh = rhh * F, rap = rahp * F, rhp = rhhp * F;
        const float ck = fc.cw * ex2(-u2);  // ek = e2 * ck
#pragma unroll
        for (int j = RB - 1; j >= 0; --j) {
          const float ek = e2v[j] * ck;
          const float gv = fmaf(gam[j], e2v[j], ek * ra);
          const float gk = fmaf(V[j], gv, -fmaf(eta[j], e2v[j], ek * rh));
          gw_acc = fmaf(ek, fmaf(V[j], rap, -rhp), gw_acc);
          gu_acc = fmaf(e2v[j], fmaf(gam[j], V[j], -eta[j]), gu_acc);
          gkp[j * 32] = from_f32<E>(gk);
          gvp[j * 32] = from_f32<E>(gv);
          rap = fc.ewm * (rap + ra);
          rhp = fc.ewm * (rhp + rh);
          ra = fmaf(ra, fc.ewm, gam[j]);
          rh = fmaf(rh, fc.ewm, eta[j]);
        }
        rah = ra;
        rhh = rh;
        rahp = rap;
        rhhp = rhp;
        Ranc = Mb;
        m = 0.f;
        continue;
      }
      if (fast) {  // the fast recompute leaves the scales implicit: D_t = den 2^{M + j w2e}
#pragma unroll
        for (int j = 0; j < RB; ++j) qv[j] = fmaf((float)j, fc.w2e, Mb);
      }
#pragma unroll
      for (int j = RB - 1; j >= 0; --j) {
        if (STATE && j >= nb) continue;  // past T
        const float rn = fmaf(-m, w2, Ranc);  // scale of the adjoint after token t
        const float tn = ex2(K[j] - rn);      // e^{k_t} 2^{-r_{t+1}} (<= 1)
        const float gv = fmaf(gam[j], e2v[j], tn * rah);
        const float gk = fmaf(V[j], gv, -fmaf(eta[j], e2v[j], tn * rhh));
        gw_acc = fmaf(tn, fmaf(V[j], rahp, -rhhp), gw_acc);
        gu_acc = fmaf(e2v[j], fmaf(gam[j], V[j], -eta[j]), gu_acc);
        gkp[j * 32] = from_f32<E>(gk);
        gvp[j * 32] = from_f32<E>(gv);
        const float m1 = m + 1.f;
        const float Rc = fmaf(-m1, w2, Ranc);
        const float d = qv[j] - Rc;
        const float x = ex2(-fabsf(d));
        const bool reset = d < 0.f;
        const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
        rahp = fo * (rah + rahp);
        rhhp = fo * (rhh + rhhp);
        rah = fmaf(rah, fo, gam[j] * fg);
        rhh = fmaf(rhh, fo, eta[j] * fg);
        Ranc = reset ? qv[j] : Ranc;
        m = reset ? 0.f : m1;
      }
    }
    if (cok) {
      if (t0 == 0) {
        // share of the initial state A_0, B_0 (zero for the empty state)
        const float *ck = p.ckpt + bc;
        const float r0 = fmaf(-m, w2, Ranc);
        gw_acc = fmaf(ex2(ck[2 * BC] - r0), fmaf(ck[0], rahp, -ck[BC] * rhhp), gw_acc);
      }
      if constexpr (STATE) {
        if (t0 == 0 && p.gs_in) store_state_grad(p.gs_in, p.state_in, bc, BC, rah, rhh, fmaf(-m, w2, Ranc));
      }
    }
    // dL/dw, dL/du: the unit's partial as a tagged word, then the
    // fixed-order sums (reduce_partials)
    const unsigned t_part = tile_flag(epoch, 3u);
    float4 *part = reinterpret_cast<float4 *>(p.part);
    if (cok) {
      st_relaxed_v4(part + (int64_t)pos * BC + bc, make_float4(gw_acc, gu_acc, tagf(t_part), 0.f));
      reduce_partials(part, a.chain_sum + BC, a.chain_sum, a.gw, a.gu, pos, nseg, b, p.B, c, C, t_part, budget,
                      p.hdr, epoch);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const uint32_t src = smem_addr(wbuf + (size_t)bf * Lay::BUF);
      tma_store_3d(&gkmap, x0, (int)t0, b, src);
      tma_store_3d(&gvmap, x0, (int)t0, b, src + Lay::ARR);
      if constexpr (GATE) tma_store_3d(&grmap, x0, (int)t0, b, src + 3 * Lay::ARR);
      bulk_commit();
    }
    __syncwarp();
  }
  if (lane == 0) {
    bulk_wait_all();
    for (int j = wt_it + 1; j <= iss_it; ++j)
      mbar_wait(bar0 + 8u * (j & 1), (uint32_t)(j >> 1) & 1u, budget, nullptr);
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

template <typename E, int L, int RB, int NW, bool STATE, bool GATE>
static cudaError_t launch_bwd_tile_t(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *rec,
                                     float4 *chain_sum, int num_sms, cudaStream_t st) {
  CUtensorMap km, vm, gm, gkm, gvm, rm, grm;
  if (!encode_btc(&km, p.k, dtype, p.B, p.T, p.C, L) || !encode_btc(&vm, p.v, dtype, p.B, p.T, p.C, L) ||
      !encode_btc(&gm, p.gy, dtype, p.B, p.T, p.C, L) || !encode_btc(&gkm, p.gk, dtype, p.B, p.T, p.C, L) ||
      !encode_btc(&gvm, p.gv, dtype, p.B, p.T, p.C, L))
    return cudaErrorInvalidValue;
  rm = gm;  // placeholders without the gate
  grm = gkm;
  if (GATE && (!encode_btc(&rm, p.r, dtype, p.B, p.T, p.C, L) || !encode_btc(&grm, p.gr, dtype, p.B, p.T, p.C, L)))
    return cudaErrorInvalidValue;
  constexpr int smem = TileBwdLayout<E, L, RB, GATE ? 4 : 3>::bytes(NW);
  auto kern = bwd_tile_kernel<E, L, RB, NW, STATE, GATE>;
  int occ = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, NW * 32, smem, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  TileBwdArgs a{};
  a.p = p;
  a.gw = gw;
  a.gu = gu;
  a.chain_sum = chain_sum;
  a.rec = rec;
  a.nseg = (p.T + L - 1) / L;
  const int64_t units = a.nseg * p.nchains;
  if (units >= (int64_t)1 << 31) return cudaErrorInvalidValue;
  const int64_t max_warps = (int64_t)occ * num_sms * NW;
  const int64_t rounds = (units + max_warps - 1) / max_warps;
  const int64_t grid = ((units + rounds - 1) / rounds + NW - 1) / NW;
  void *args[] = {&km, &vm, &gm, &rm, &gkm, &gvm, &grm, &a};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3(NW * 32), args, (size_t)smem,
                                     st);
}

// Warps per block: four (two blocks of 4 per SM fit the ungated tiles), two
// for the gated kernel (its four tiles per buffer: three blocks of 2 fit).
cudaError_t launch_backward_tile(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *rec, float4 *chain_sum,
                                 int num_sms, cudaStream_t st) {
  if (p.r && (p.gs_out || p.gs_in)) return cudaErrorInvalidValue;  // no entry point asks for both
  if (p.r)
    return dtype == 0 ? launch_bwd_tile_t<float, kTileLF32, 8, 2, false, true>(p, dtype, gw, gu, rec, chain_sum,
                                                                                num_sms, st)
                      : launch_bwd_tile_t<uint16_t, kTileLBF16, 8, 2, false, true>(p, dtype, gw, gu, rec, chain_sum,
                                                                                    num_sms, st);
  if (p.gs_out || p.gs_in)
    return dtype == 0 ? launch_bwd_tile_t<float, kTileLF32, 8, kTileWarps, true, false>(
                            p, dtype, gw, gu, rec, chain_sum, num_sms, st)
                      : launch_bwd_tile_t<uint16_t, WKV_TILEB_LBF16, 8, kTileWarps, true, false>(
                            p, dtype, gw, gu, rec, chain_sum, num_sms, st);
  return dtype == 0 ? launch_bwd_tile_t<float, kTileLF32, WKV_TILEB_RB, kTileWarps, false, false>(
                          p, dtype, gw, gu, rec, chain_sum, num_sms, st)
                    : launch_bwd_tile_t<uint16_t, WKV_TILEB_LBF16, WKV_TILEB_RB, kTileWarps, false, false>(
                          p, dtype, gw, gu, rec, chain_sum, num_sms, st);
}

}  // namespace wkv
