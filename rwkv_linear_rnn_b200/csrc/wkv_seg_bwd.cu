// wkv_seg_bwd.cu -- segment backward of libwkv (the default backward on
// sm_100a when rows are 16-byte aligned): dL/dk, dL/dv, dL/dw, dL/du in one
// launch.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"); the gradient is
// back-propagation through the recurrence of section "RNN-유사추론" (the
// review's BPTT remark), taken in the reverse-time scan form of the linear
// attention post ("Transformers are RNNs: 선형 어텐션으로 만드는 빠른 자기회귀
// 트랜스포머", section "상수 메모리 기울기 계산": the cumulative sums for the
// key/value gradients run backwards in time).
//
// With D_t the denominator, G_t = g_t / D_t and H_t = g_t y_t / D_t, the
// adjoints of the past sums obey a reverse recurrence with the constant
// factor e^w:
//   Ahat_t = G_t + e^w Ahat_{t+1},   Hhat_t = H_t + e^w Hhat_{t+1},
// so a segment of tokens has an aggregate (its adjoint at the segment start
// from a zero adjoint at its end) that joins associatively with the adjoint
// carried in from later segments (rcombine5).  One warp owns one segment: a
// chain (batch row b, 32 channels = lanes) and TS consecutive tokens.  Warps
// are persistent and take segments in reverse position order (all chains'
// last segment first):
//   pass 1  stream k, v, g through the warp's TMA ring in forward order,
//           recompute the forward from the checkpoint at the segment start
//           and accumulate the segment's adjoint aggregate (in forward order:
//           token s enters with weight e^{(s - t0) w}), keeping the forward
//           state at every batch start (8 tokens) in shared memory;
//   join    publish the aggregate, then fold, in a fixed order, the records
//           of at most kBwdBlockSeg later segments of the chain (the suffix
//           that closes the previous block of segments, then the aggregates
//           of the later segments of this block) into the adjoint at the
//           segment end;
//   pass 2  stream the 8-token batches again, last first (still in L2:
//           pass 1 loads carry an evict-last hint), recompute each batch's
//           forward from its saved start state and sweep it in reverse,
//           writing dL/dk, dL/dv; per-unit partial sums of dL/dw, dL/du go
//           to the workspace.
// After a bounded grid barrier the warps reduce the partials per channel in
// a fixed two-level order (group sums, then the last group of a channel tile
// adds the group sums), so the result is bit-reproducible.
#include <cuda.h>

#include <algorithm>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_ring.cuh"
#include "wkv_bwd_math.cuh"

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

struct SegBwdArgs {
  BwdArgs p;
  float *gw, *gu;
  unsigned *tile_cnt;  // [nct] group counters of the final reduction
  int64_t nseg;        // segments per chain
  int64_t ngroups;     // row groups per channel tile in the final reduction
  int ts;              // tokens per segment (a multiple of the checkpoint interval)
  int nb;              // batches per segment (ts / rows per batch)
};

#ifndef WKV_SEGB_BLOCK
#define WKV_SEGB_BLOCK 4
#endif
constexpr int kBwdBlockSeg = WKV_SEGB_BLOCK;  // segments per suffix block (at most one per lane)
static_assert(kBwdBlockSeg >= 1 && kBwdBlockSeg <= 32, "one lane per record");
#ifndef WKV_SEGB_MINB
#define WKV_SEGB_MINB 4
#endif

// Shared memory of a block of NW warps: the warp rings (with their
// mbarriers), then per warp the forward state at each batch start of the
// current segment: [NB][3][32] floats (a, b, exponent).  NARR: tensors per
// ring item (k, v, grad, and the gate input when gated).
template <typename E, int S, int RB, int NARR>
struct SegBwdSmem {
  using RingL = WarpRing<E, S, NARR, RB>;
  static constexpr int ring_bytes(int nw) { return (RingL::block_bytes(nw) + 15) / 16 * 16; }
  static constexpr int bytes(int nw, int nb) { return ring_bytes(nw) + nw * nb * 96 * 4; }
};

// BAR: every warp owns at most one segment; all warps run pass 1, meet at a
// grid barrier and fold the later segments' aggregates without polling.
// Otherwise segments are joined through per-record flags.
// GATE: the loss depends on o = sigma(r) * y.  Pass 1's ring items carry
// grad_o and r as the third and fourth tensors; pass 1 forms the WKV
// gradient grad_o sigma(r), writes dL/dr = grad_o y sigma'(r) from its
// recompute, and leaves grad_o sigma(r) in grad_k's rows (which pass 2
// overwrites with dL/dk after reading them).  Pass 2's items carry k, v and
// those rows, as in the ungated kernel: grad_o and r are not re-read, and
// only k, v and the scratch rows need to stay in L2 between the passes.
// The scratch rows are written with generic stores and read by TMA: each
// writer fences them for the async proxy, and a unit's pass-2 items are
// issued only after its pass 1 is done.
// STATE: the state terms of a sequence split across calls: the folds start
// from the adjoint after the last token (the final state's gradient), the
// last segment's sweep stops exactly at token T-1 (its padding would decay
// that adjoint), and the first segment writes the initial state's gradient.
// A variant of its own so that the common path keeps its instruction
// schedule.
template <typename E, int S, int RB, bool BAR, bool GATE, bool STATE>
__global__ void __launch_bounds__(128, WKV_SEGB_MINB) bwd_seg_kernel(const __grid_constant__ CUtensorMap kmap,
                                                      const __grid_constant__ CUtensorMap vmap,
                                                      const __grid_constant__ CUtensorMap gmap,
                                                      const __grid_constant__ CUtensorMap rmap,
                                                      const __grid_constant__ CUtensorMap smap,
                                                      SegBwdArgs a) {
  constexpr int NARR = GATE ? 4 : 3;
  using Sm = SegBwdSmem<E, S, RB, NARR>;
  const int TS = a.ts;         // tokens per segment (segments start on checkpoints)
  const int NB = a.nb;         // ring items (batches of RB tokens) per pass
  const int IPU = 2 * NB;      // ring items per segment
  const BwdArgs &p = a.p;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = (int)(blockDim.x >> 5);
  Ring<E, S, NARR, RB> ring(smem, wl, nw);
  ring.init(lane);
  float *sts = reinterpret_cast<float *>(smem + Sm::ring_bytes(nw)) + wl * NB * 96;
  const CUtensorMap *maps[NARR];
  maps[0] = &kmap;
  maps[1] = &vmap;
  maps[2] = &gmap;
  if constexpr (GATE) maps[NARR - 1] = &rmap;
  // The reduction counters are cleared here; the grid barrier orders these
  // stores before every increment (a workspace reused for another shape may
  // hold anything at their offset).
  if (blockIdx.x == 0)
    for (int64_t i = threadIdx.x; i < p.nct; i += blockDim.x) a.tile_cnt[i] = 0u;
  // unit indices fit 31 bits (the launcher checks nseg * nchains)
  const int G = (int)gridDim.x * nw;
  const int g = (int)blockIdx.x * nw + wl;
  const int nseg = (int)a.nseg, nchains = (int)p.nchains, nct = (int)p.nct;
  const int total = nseg * nchains;
  const int nu = total > g ? (total - g + G - 1) / G : 0;
  const int nitems = nu * IPU;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  const unsigned want = (epoch_tag(epoch) << 2) | kAgg;

  // Lane 0 issues ring items ahead of the consumer, in consumption order.
  // Item r of a unit: pass 1 batch r (r < NB), pass 2 batch IPU-1-r (last
  // batch first).  Running counters (item, stage, unit) avoid divisions.
  int iss_k = 0, iss_unit = g, iss_r = 0, iss_s = 0, iss_x = 0, iss_row0 = 0;
  int iss_done = 0;  // copies actually issued (lane 0)
  // GATE: items at or past iss_lim wait (a unit's pass-2 items read rows its
  // pass 1 writes); `consumed` counts the items taken
  int iss_lim = GATE ? NB : 1 << 30, consumed = 0;
  if (lane == 0) {
    if (!ring.aligned()) {  // cannot happen with this layout; never issue a misaligned copy
      atomicCAS(&p.hdr->status, 0, -4);
      iss_k = nitems;
    }
  }
  auto issue_next = [&]() {
    if (iss_r == 0) {
      const int rpos = iss_unit / nchains, chain = iss_unit - rpos * nchains;
      const int b = chain / nct;
      iss_x = (chain - b * nct) * 32;
      iss_row0 = (int)((int64_t)b * T + (int64_t)(nseg - 1 - rpos) * TS);
    }
    const int bt = iss_r < NB ? iss_r : IPU - 1 - iss_r;
    if constexpr (GATE) {
      // pass 1: k, v (kept in L2 for pass 2), grad_o, r (read once);
      // pass 2: k, v and the WKV-gradient rows left in grad_k
      const int y = iss_row0 + bt * RB;
      const uint32_t bar = ring.bar(iss_s);
      const uint64_t first = l2_policy_evict_first();
      constexpr uint32_t AB = (uint32_t)WarpRing<E, S, NARR, RB>::ARR_BYTES;
      if (iss_r < NB) {
        const uint64_t keep = l2_policy_evict_last();
        mbar_expect_tx(bar, 4u * AB);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 0)), &kmap, iss_x, y, bar, keep);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 1)), &vmap, iss_x, y, bar, keep);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 2)), &gmap, iss_x, y, bar, first);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 3)), &rmap, iss_x, y, bar, first);
      } else {
        mbar_expect_tx(bar, 3u * AB);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 0)), &kmap, iss_x, y, bar, first);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 1)), &vmap, iss_x, y, bar, first);
        tma_load_2d_hint(smem_addr(ring.stage(iss_s, 2)), &smap, iss_x, y, bar, first);
      }
    } else {
      ring.issue_stage(maps, iss_s, iss_x, iss_row0 + bt * RB,
                       iss_r < NB ? l2_policy_evict_last() : l2_policy_evict_first());
    }
    ++iss_k;
    iss_done = iss_k;
    iss_s = iss_s + 1 == S ? 0 : iss_s + 1;
    if (++iss_r == IPU) {
      iss_r = 0;
      iss_unit += G;
    }
  };
  if (lane == 0)
    while (iss_k < min(min(S - 1, nitems), iss_lim)) issue_next();
  bool failed = false;
  int cs = 0;           // stage of the next item to consume
  uint32_t cph = 0;     // its mbarrier phase parity
  // Gy: the WKV output's gradient; with the gate, in pass 1 (first) Gy is
  // formed as grad_o sigma(r) and Gd receives grad_o sigma'(r).
  auto take = [&](float(&K)[RB], float(&V)[RB], float(&Gy)[RB], float(&Gd)[RB], bool first) {
    if (!failed && !mbar_wait(ring.bar(cs), cph, budget, nullptr)) {
      failed = true;
      if (lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    }
    const E *kr = ring.stage(cs, 0) + lane;
    const E *vr = ring.stage(cs, 1) + lane;
    const E *gr = ring.stage(cs, 2) + lane;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
      Gy[j] = to_f32(gr[j * 32]);
    }
    if constexpr (GATE) {
      if (first) {
        const E *rr = ring.stage(cs, NARR - 1) + lane;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          float sg, ds;
          gate_sigmoid_slope(to_f32(rr[j * 32]), sg, ds);
          Gd[j] = Gy[j] * ds;
          Gy[j] *= sg;
        }
      }
    }
    __syncwarp();  // the stage is read; it may be refilled
    if (++cs == S) {
      cs = 0;
      cph ^= 1u;
    }
    ++consumed;
    // after a failed wait nothing new is issued
    if (lane == 0 && iss_k < nitems && !failed && iss_k < iss_lim) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_next();
    }
  };
  // Tokens past T (only in a chain's last segment) are computed on whatever
  // the loads brought but enter with a zero gradient, so they add nothing.
  auto mask_tail = [&](float(&Gy)[RB], int nb) {
    if (nb < RB) {
#pragma unroll
      for (int j = 0; j < RB; ++j) Gy[j] = j < nb ? Gy[j] : 0.f;
    }
  };

  const int iters = BAR ? 1 : nu;  // with BAR every warp passes the barrier once
  for (int i = 0; i < iters; ++i) {
    const bool has = i < nu;
    const int unit = has ? g + i * G : 0;
    const int rpos = unit / nchains, chain = unit - rpos * nchains;
    const int b = chain / nct;
    const int64_t c = (int64_t)(chain - b * nct) * 32 + lane;
    const bool cok = c < C;
    const int pos = nseg - 1 - rpos;
    const int64_t t0 = (int64_t)pos * TS;
    const int n = (int)min((int64_t)TS, T - t0);
    const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
    const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
    const int64_t bc = (int64_t)b * C + c;
    const FastC fc = fast_consts<RB>(w2, u2);

    // ---- pass 1: forward recompute and the segment's adjoint aggregate
    // The forward state is (fa, fb) 2^E with E = fP + fn w2 (anchored).
    float fa = 0.f, fb = 0.f, fP = kEmptyP, fn = 0.f;
    if (cok) {
      const float *ck = p.ckpt + (t0 / kCkpt) * 3 * BC + bc;
      fa = ck[0];
      fb = ck[BC];
      fP = ck[2 * BC];
    }
    float ah = 0.f, hh = 0.f, ahp = 0.f, hhp = 0.f, Em = -kEmptyR;
#pragma unroll 1
    for (int bt = 0; bt < (has ? NB : 0); ++bt) {
      sts[bt * 96 + lane] = fa;
      sts[bt * 96 + 32 + lane] = fb;
      sts[bt * 96 + 64 + lane] = fmaf(fn, w2, fP);
      float K[RB], V[RB], Gy[RB], Gd[RB];
      take(K, V, Gy, Gd, true);
      mask_tail(Gy, n - bt * RB);
      float qv[RB], gam[RB], eta[RB], e2v[RB], Mb;
      const bool fast =
          recompute_batch<RB, GATE>(K, V, Gy, w2, u2, fc, fa, fb, fP, fn, qv, gam, eta, e2v, Mb, Gd);
      if constexpr (GATE) {
        // dL/dr = grad_o sigma'(r) y, and the WKV gradient for pass 2 in
        // grad_k's rows (a plain store: it should stay in L2 until read)
        if (cok) {
          const int64_t row = ((int64_t)b * T + t0 + bt * RB) * C + c;
          E *grp = static_cast<E *>(p.gr) + row;
          E *gsp = static_cast<E *>(p.gk) + row;
          const int jn = n - bt * RB;
#pragma unroll
          for (int j = 0; j < RB; ++j) {
            if (j < jn) {
              IO<E>::st(grp + (int64_t)j * C, Gd[j]);
              IO<E>::st_keep(gsp + (int64_t)j * C, Gy[j]);
            }
          }
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
    if constexpr (GATE) {
      // pass 1 of this unit is done: its scratch rows are written.  Make them
      // visible to the async proxy, then issue the held items (this unit's
      // pass 2 and the next unit's pass 1).
      asm volatile("fence.proxy.async.global;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        iss_lim = (i + 1) * IPU + NB;
        if (!failed)
          while (iss_k < nitems && iss_k < iss_lim && iss_k < consumed + S - 1) issue_next();
      }
      __syncwarp();
    }

    const int nlast = (int)(T - (nseg - 1) * TS);  // tokens of the chain's last segment
    // the adjoint after the chain's last token (a loss term on the final
    // state, if any): the start of every fold
    Adj5s acc = adj5s_empty();
    if constexpr (STATE) {
      if (p.gs_out && cok) end_adjoint(p.gs_out[bc], p.gs_out[BC + bc], p.p_out[bc], acc.ah, acc.hh, acc.r);
    }
    if constexpr (BAR) {
      // ---- join after the grid barrier: fold the later segments in order
      if (has && rpos + 1 < nseg) rec_store_adj(p.desc, unit, agg, lane);
      grid_barrier(p.hdr, gridDim.x, budget);
      if (!has) continue;
#pragma unroll 1
      for (int j0 = 0; j0 < rpos; j0 += 8) {
        Adj5s rec[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j0 + j < rpos) rec[j] = rec_load_adj(p.desc, (int64_t)(j0 + j) * nchains + chain, lane);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j0 + j < rpos) acc = rjoin(rec[j], acc, j0 + j == 0 ? (float)nlast : (float)TS, w2);
      }
    } else {
    // ---- join: adjoint at the segment end from the later segments' records
    const int q = rpos - rpos % kBwdBlockSeg;  // first (latest) segment of this block
    const int nrec = (rpos - q) + (q > 0 ? 1 : 0);
    const int rec0 = q > 0 ? q - 1 : q;
    const bool block_end = (rpos % kBwdBlockSeg) == kBwdBlockSeg - 1;
    const bool held = p.hold_first && rpos == 0;  // test hook: never publish
    if (!block_end && rpos + 1 < nseg && !held) publish_adj(p.desc, p.flags, unit, agg, epoch, lane);
    {
      const bool act = lane < nrec;
      const unsigned *fl = p.flags + (int64_t)(rec0 + lane) * nchains + chain;
      bool ready = !act;
      const uint64_t t_start = global_ns();
      unsigned backoff = 32;
      while (true) {
        if (!ready) ready = ld_acquire(fl) == want;
        if (__all_sync(0xffffffffu, ready)) break;
        if ((int64_t)(global_ns() - t_start) > budget) {
          if (lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
          break;
        }
        __nanosleep(backoff);
        backoff = backoff < 512u ? backoff * 2u : 512u;
      }
      __syncwarp();
    }
#pragma unroll 1
    for (int j0 = 0; j0 < nrec; j0 += 8) {
      Adj5s rec[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < nrec) rec[j] = rec_load_adj(p.desc, (int64_t)(rec0 + j0 + j) * nchains + chain, lane);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < nrec) {
          const int rp = rec0 + j0 + j;
          if (q > 0 && rp == q - 1)
            acc = rec[j];  // adjoint at the start of the previous block's last segment
          else
            acc = rjoin(rec[j], acc, rp == 0 ? (float)nlast : (float)TS, w2);
        }
      }
    }
    if (block_end && rpos + 1 < nseg && !held)
      publish_adj(p.desc, p.flags, unit, rjoin(agg, acc, (float)n, w2), epoch, lane);
    }

    // ---- pass 2: batches last to first, recompute then reverse sweep
    float gw_acc = 0.f, gu_acc = 0.f;
    float rah = acc.ah, rhh = acc.hh, rahp = acc.ahp, rhhp = acc.hhp, Ranc = acc.r, m = 0.f;
#pragma unroll 1
    for (int bi = 0; bi < NB; ++bi) {
      const int bt = NB - 1 - bi;
      float K[RB], V[RB], Gy[RB], Gd[RB];
      take(K, V, Gy, Gd, false);
      const int nb = n - bt * RB;  // valid tokens of the batch (may be <= 0 or > RB)
      mask_tail(Gy, nb);
      float qv[RB], gam[RB], eta[RB], e2v[RB], Mb;
      bool fast;
      {
        float xa = sts[bt * 96 + lane], xb = sts[bt * 96 + 32 + lane], xP = sts[bt * 96 + 64 + lane];
        float xn = 0.f;
        fast = recompute_batch<RB, false>(K, V, Gy, w2, u2, fc, xa, xb, xP, xn, qv, gam, eta, e2v, Mb, Gd);
      }
      E *gkp = static_cast<E *>(p.gk) + ((int64_t)b * T + t0 + bt * RB) * C + c;
      E *gvp = static_cast<E *>(p.gv) + ((int64_t)b * T + t0 + bt * RB) * C + c;
      // Fast sweep: the adjoint in the batch's coordinates, a_t = A_t 2^{M + t w2e},
      // obeys a_t = gam_t + ewm a_{t+1} (and a'_t = ewm (a'_{t+1} + a_{t+1}) for
      // the lag-weighted one); e^{k_t} A_{t+1} = ek_t a_{t+1}.  The carried
      // adjoint enters scaled by 2^{M + RB w2e - r}, bounded for the float range.
      if constexpr (STATE) {
        if (nb <= 0) continue;  // only tokens past T (a chain's last segment): nothing to sweep
      }
      const float rn_end = fmaf(-m, w2, Ranc);
      const float xin = fmaf((float)RB, fc.w2e, Mb) - rn_end;
      // (with STATE a partial batch takes the per-token sweep, which stops at
      // the last token: the carried adjoint starts after token T-1, not after
      // the batch's padding; without it the adjoint there is zero and the
      // padding, whose gradient is masked, adds nothing)
      if (__all_sync(0xffffffffu, fast && xin < 100.f && (!STATE || nb >= RB))) {
        const float F = ex2(xin);
        float ra = rah * F, rh = rhh * F, rap = rahp * F, rhp = rhhp * F;
        const float ck = fc.cw * ex2(-u2);  // ek = e2 * ck
        const int jmax = cok ? min(nb, RB) : 0;  // tokens to store (all of a full batch)
#pragma unroll
        for (int j = RB - 1; j >= 0; --j) {
          const float ek = e2v[j] * ck;
          const float gv = fmaf(gam[j], e2v[j], ek * ra);
          const float gk = fmaf(V[j], gv, -fmaf(eta[j], e2v[j], ek * rh));
          gw_acc = fmaf(ek, fmaf(V[j], rap, -rhp), gw_acc);
          gu_acc = fmaf(e2v[j], fmaf(gam[j], V[j], -eta[j]), gu_acc);
          if (j < jmax) {
            IO<E>::st(gkp + (int64_t)j * C, gk);
            IO<E>::st(gvp + (int64_t)j * C, gv);
          }
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
        if (cok && j < nb) {
          IO<E>::st(gkp + (int64_t)j * C, gk);
          IO<E>::st(gvp + (int64_t)j * C, gv);
        }
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
      p.part[(int64_t)(pos * 2 + 0) * BC + bc] = gw_acc;
      p.part[(int64_t)(pos * 2 + 1) * BC + bc] = gu_acc;
    }
  }
  if (failed && lane == 0)  // every issued load lands before the block exits
    for (int k = max(0, iss_done - S); k < iss_done; ++k)
      mbar_wait(ring.bar(k % S), (uint32_t)(k / S) & 1u, budget, nullptr);

  // ---- dL/dw, dL/du: fixed-order two-level reduction of the partials
  grid_barrier(p.hdr, (BAR ? 2u : 1u) * gridDim.x, budget);
  reduce_wu_partials(p, a.gw, a.gu, a.tile_cnt, (int64_t)nseg, a.ngroups, g, G, lane);
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

template <typename E, int S, int RB, bool GATE, bool STATE>
static cudaError_t launch_bwd_seg_t(const BwdArgs &p, int dtype, float *gw, float *gu, unsigned *tile_cnt,
                                    int64_t scratch_doubles, int num_sms, int ts_max, cudaStream_t st) {
  CUtensorMap km, vm, gm, rm;
  if (!encode_rows(&km, p.k, dtype, p.B * p.T, p.C, RB) || !encode_rows(&vm, p.v, dtype, p.B * p.T, p.C, RB) ||
      !encode_rows(&gm, p.gy, dtype, p.B * p.T, p.C, RB))
    return cudaErrorInvalidValue;
  rm = gm;  // unused without the gate
  CUtensorMap sm = gm;
  if (GATE && (!encode_rows(&rm, p.r, dtype, p.B * p.T, p.C, RB) ||
               !encode_rows(&sm, p.gk, dtype, p.B * p.T, p.C, RB)))
    return cudaErrorInvalidValue;
  constexpr int NARR = GATE ? 4 : 3;
  constexpr int kWarps = 4;
  static_assert(kCkpt % RB == 0, "checkpoints fall on batch starts");
  // Resident warps for a segment length (the per-warp batch states in shared
  // memory grow with it); the smaller occupancy of the two join variants.
  auto max_warps_for = [&](int ts, int &smem, int64_t &mw) -> cudaError_t {
    smem = SegBwdSmem<E, S, RB, NARR>::bytes(kWarps, ts / RB);
    int occ = 1 << 30;
    for (const void *kern : {(const void *)bwd_seg_kernel<E, S, RB, false, GATE, STATE>,
                             (const void *)bwd_seg_kernel<E, S, RB, true, GATE, STATE>}) {
      int o = 0;
      cudaError_t e = blocks_per_sm(kern, kWarps * 32, smem, &o);
      if (e != cudaSuccess) return e;
      occ = std::min(occ, o);
    }
    mw = (int64_t)occ * num_sms * kWarps;
    return occ < 1 ? cudaErrorInvalidConfiguration : cudaSuccess;
  };
  // Segment length: the shortest multiple of 32 tokens (>= 64, whole
  // checkpoint intervals) that lets every segment have its own resident
  // warp (barrier join, most warps); otherwise the longest (fewest joins
  // per token).
  static_assert(32 % kCkpt == 0, "segments start on checkpoints");
  int ts = ts_max, smem = 0;
  int64_t max_warps = 0;
  bool fits = false;
  for (int cand = 64; cand <= ts_max; cand += 32) {
    int sm = 0;
    int64_t mw = 0;
    cudaError_t e = max_warps_for(cand, sm, mw);
    if (e != cudaSuccess) return e;
    if ((p.T + cand - 1) / cand * p.nchains <= mw) {
      ts = cand, smem = sm, max_warps = mw, fits = true;
      break;
    }
  }
  if (!fits) {
    cudaError_t e = max_warps_for(ts, smem, max_warps);
    if (e != cudaSuccess) return e;
  }
  SegBwdArgs a{};
  a.p = p;
  a.gw = gw;
  a.gu = gu;
  a.tile_cnt = tile_cnt;
  a.ts = ts;
  a.nb = ts / RB;
  a.nseg = (p.T + ts - 1) / ts;
  const int64_t units = a.nseg * p.nchains;
  if (units >= (int64_t)1 << 31) return cudaErrorInvalidValue;  // unit indices are 31-bit
  // One resident wave (cooperative launch: every warp a segment may wait on,
  // and every block of the grid barrier, is running).  Warps take segments
  // round-robin; the grid is trimmed so that every warp gets the same number
  // of segments (no final round with most warps idle).
  const int64_t rounds = (units + max_warps - 1) / max_warps;
  const int64_t want = (units + rounds - 1) / rounds;
  const int64_t grid = (want + kWarps - 1) / kWarps;
  const int64_t G = grid * kWarps;
  // row groups per channel tile: enough to spread the partial rows over the
  // warps, at least 8 rows each, and the group sums must fit the scratch
  const int64_t R = a.nseg * p.B;
  int64_t ng = std::max<int64_t>(1, std::min<int64_t>(G / p.nct, R / 8));
  while (ng > 1 && p.nct * ng * 64 > scratch_doubles) --ng;
  a.ngroups = ng;
  // Barrier join when every warp has one segment (all first passes run
  // together anyway) and chains have few segments (each fold reads all the
  // later ones); the test hook needs the flag join.
  const bool bar = rounds == 1 && a.nseg <= 32 && !p.hold_first;
  const void *kern = bar ? (const void *)bwd_seg_kernel<E, S, RB, true, GATE, STATE>
                         : (const void *)bwd_seg_kernel<E, S, RB, false, GATE, STATE>;
  void *args[] = {&km, &vm, &gm, &rm, &sm, &a};
  return cudaLaunchCooperativeKernel(kern, dim3((unsigned)grid), dim3(kWarps * 32), args, (size_t)smem, st);
}

// Tile parameters (compile-time tunables): the longest segment (tokens),
// ring stages, rows per ring item.
#ifndef WKV_SEGB_TS
#define WKV_SEGB_TS 128
#endif
#ifndef WKV_SEGB_S_F32
#define WKV_SEGB_S_F32 3
#endif
#ifndef WKV_SEGB_S_BF16
#define WKV_SEGB_S_BF16 4
#endif
#ifndef WKV_SEGB_RB
#define WKV_SEGB_RB 8
#endif

// Ring stages of the gated variant (its first-pass items carry four arrays).
// fp32: two stages, measured faster than three (65.8 vs 68.7 us on B8 T1024
// C768: the smaller ring lets 4 blocks share an SM).  bf16: three stages,
// faster than four (525 vs 615 us on B8 T4096 C2048) and than two.
#ifndef WKV_SEGB_S_F32_GATE
#define WKV_SEGB_S_F32_GATE 2
#endif
#ifndef WKV_SEGB_S_BF16_GATE
#define WKV_SEGB_S_BF16_GATE 3
#endif

cudaError_t launch_backward_seg(const BwdArgs &p, int dtype, float *gw, float *gu, unsigned *tile_cnt,
                                int64_t scratch_doubles, int num_sms, cudaStream_t st) {
  const int64_t sc = scratch_doubles;
  const int ts = WKV_SEGB_TS;
  if (p.r && (p.gs_out || p.gs_in)) return cudaErrorInvalidValue;  // no entry point asks for both
  if (p.r)
    return dtype == 0
               ? launch_bwd_seg_t<float, WKV_SEGB_S_F32_GATE, WKV_SEGB_RB, true, false>(p, dtype, gw, gu, tile_cnt,
                                                                                         sc, num_sms, ts, st)
               : launch_bwd_seg_t<uint16_t, WKV_SEGB_S_BF16_GATE, WKV_SEGB_RB, true, false>(
                     p, dtype, gw, gu, tile_cnt, sc, num_sms, ts, st);
  if (p.gs_out || p.gs_in)
    return dtype == 0
               ? launch_bwd_seg_t<float, WKV_SEGB_S_F32, WKV_SEGB_RB, false, true>(p, dtype, gw, gu, tile_cnt, sc,
                                                                                    num_sms, ts, st)
               : launch_bwd_seg_t<uint16_t, WKV_SEGB_S_BF16, WKV_SEGB_RB, false, true>(p, dtype, gw, gu, tile_cnt,
                                                                                       sc, num_sms, ts, st);
  return dtype == 0
             ? launch_bwd_seg_t<float, WKV_SEGB_S_F32, WKV_SEGB_RB, false, false>(p, dtype, gw, gu, tile_cnt, sc,
                                                                                   num_sms, ts, st)
             : launch_bwd_seg_t<uint16_t, WKV_SEGB_S_BF16, WKV_SEGB_RB, false, false>(p, dtype, gw, gu, tile_cnt,
                                                                                      sc, num_sms, ts, st);
}

}  // namespace wkv
