// wkv_chain.cu -- chain kernels of libwkv: one warp runs one chain (batch
// row b, 32 channels = the 32 lanes) through all of its tokens in order.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), run in the RNN
// form of section "RNN-유사추론" over the max-rescaled state; the gradient
// is back-propagation through that recurrence, taken backwards in time as
// in the linear attention post ("Transformers are RNNs: 선형 어텐션으로
// 만드는 빠른 자기회귀 트랜스포머", section "상수 메모리 기울기 계산").
//
// When a problem has about as many chains as the GPU has warp schedulers,
// splitting the time axis buys nothing: every scheduler already has a chain
// to run, and the joins of a time-parallel scan (summaries, look-backs, a
// second pass over every token) more than double the instructions per token.
// Here a chain's state, or its adjoint, is carried from one unit of L tokens
// to the next in registers.  A block holds four such compute warps (one per
// scheduler of an SM) and a fifth warp that issues every TMA copy of the
// block: per compute warp, S stages of input stay in flight; the compute
// warp writes its outputs over the inputs it has consumed and signals the
// stage through an mbarrier; the TMA warp stores them and reloads the stage
// once the store has read it.  No compute warp ever waits on a copy
// instruction, and the copy engine, not the warps, moves every byte.
//
// Forward, per unit: the recurrence over the unit's tokens, in batches of
// RB tokens on the batch fast path of wkv_math.cuh where the warp allows it;
// y, the checkpoints every 16 tokens and the final state are written.
// Backward, per unit, units last to first: batches of one checkpoint
// interval, last to first, each from its checkpoint (loaded by TMA with the
// unit's tiles): recompute, reverse sweep of the adjoint, dL/dk and dL/dv.
// dL/dw and dL/du are summed per chain (per unit in float, across units in
// float64), and the chain of the last batch row of each channel tile adds
// the B chains in batch-row order: the result is bit-reproducible.
// GATE variants fuse the output gate o = sigma(r) * y into both.
#include <cuda.h>

#include "wkv_bwd_math.cuh"
#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_tile.cuh"

// Build-time knobs.  Tokens per batch of the forward's fast path (bf16,
// ungated; fp32 and gated calls use at most 32):
#ifndef WKV_CHAIN_FRB
#define WKV_CHAIN_FRB 64
#endif
// tokens per bf16 unit of the forward and the backward, TMA stages per warp
// of the backward (the forward takes as many stages as 48 KB of input per
// warp hold), and nanoseconds the TMA warp sleeps between polls that find
// nothing to do:
#ifndef WKV_CHAIN_LF
#define WKV_CHAIN_LF 128
#endif
#ifndef WKV_CHAIN_SLEEP
#define WKV_CHAIN_SLEEP 500
#endif
#ifndef WKV_CHAIN_LB
#define WKV_CHAIN_LB 128
#endif
#ifndef WKV_CHAIN_SB
#define WKV_CHAIN_SB 2
#endif

namespace wkv {

bool encode_btc(CUtensorMap *m, const void *ptr, int dtype, int64_t B, int64_t T, int64_t C, int box_t);
bool encode_ckpt(CUtensorMap *m, const float *ck, int64_t B, int64_t C, int64_t nck, int box_ck);

constexpr int kChainWarps = 4;  // compute warps per block, one per scheduler (and the TMA warp)
// tokens per forward batch of fp32 calls (a unit of 32 tokens) and of gated
// calls (their third input array in registers)
constexpr int kFrbF32 = WKV_CHAIN_FRB < kTileLF32 ? WKV_CHAIN_FRB : kTileLF32;
constexpr int kChainFwdBytes = 48 * 1024;  // input stages per warp of the forward

// Largest and smallest of n values as balanced trees: log2(n) dependent
// steps instead of n (with one warp per scheduler, dependent chains are
// what the arithmetic waits on).  Max and min are exact, so the order does
// not change the result.
template <int N>
__device__ __forceinline__ void tree_minmax(const float (&x)[N], float &mx, float &mn) {
  static_assert((N & (N - 1)) == 0, "power of two");
  float a[N / 2], b[N / 2];
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    a[i] = fmaxf(x[2 * i], x[2 * i + 1]);
    b[i] = fminf(x[2 * i], x[2 * i + 1]);
  }
#pragma unroll
  for (int s = N / 4; s >= 1; s /= 2) {
#pragma unroll
    for (int i = 0; i < s; ++i) {
      a[i] = fmaxf(a[i], a[i + s]);
      b[i] = fminf(b[i], b[i + s]);
    }
  }
  mx = a[0];
  mn = b[0];
}

// fast_prep of wkv_math.cuh with the reductions as trees (same results).
template <int RB>
__device__ __forceinline__ bool fast_prep_tree(const float (&K)[RB], float E0, float u2, float w2e, float (&kj)[RB],
                                               float &M) {
#pragma unroll
  for (int j = 0; j < RB; ++j) kj[j] = fmaf(-(float)j, w2e, K[j]);
  float mx, mn;
  tree_minmax<RB>(kj, mx, mn);
  mx = fmaxf(E0, mx);
  mn = fminf(3.0e38f, mn);
  M = mx;
  return (mx - mn < 100.f) && (mx - mn - u2 < 64.f) && (u2 < 64.f);
}

// Round two floats to the element type and store them (bf16: one packed
// conversion for both, to nearest even).
template <typename E>
__device__ __forceinline__ void store2(E *p0, E *p1, float x0, float x1);
template <>
__device__ __forceinline__ void store2<float>(float *p0, float *p1, float x0, float x1) {
  *p0 = x0;
  *p1 = x1;
}
template <>
__device__ __forceinline__ void store2<uint16_t>(uint16_t *p0, uint16_t *p1, float x0, float x1) {
  unsigned u;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(x1), "f"(x0));  // x1 to the upper half
  *p0 = (uint16_t)(u & 0xffffu);
  *p1 = (uint16_t)(u >> 16);
}

// mbar_wait for the TMA warp, which shares a scheduler with a compute warp:
// between polls it sleeps instead of spinning, leaving the issue slots to
// the compute warp (the copies it then issues have stages of slack).
__device__ __forceinline__ bool mbar_wait_sleepy(uint32_t bar, uint32_t parity, int64_t budget_ns) {
#if WKV_CHAIN_SLEEP
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if ((int64_t)(global_ns() - t0) > budget_ns) return false;
    __nanosleep(WKV_CHAIN_SLEEP);
  }
  return true;
#else
  return mbar_wait(bar, parity, budget_ns, nullptr);
#endif
}


// Per warp: S input stages of NARR tiles [L][32] (and XST bytes more),
// NOUT output tiles twice (double-buffered staging), STS bytes of scratch;
// after every warp's region, S mbarriers per warp.
template <typename E, int L, int NARR, int NOUT, int S, int STS, int XST = 0>
struct ChainLayout {
  static constexpr int ARR = L * 32 * (int)sizeof(E);
  static constexpr int STAGE = NARR * ARR + XST;  // + XST bytes more per stage (after the tiles)
  static constexpr int OUT = NOUT * ARR;
  static constexpr int WARP = S * STAGE + 2 * OUT + STS;
  static_assert(ARR % 128 == 0 && STS % 128 == 0 && XST % 128 == 0, "TMA buffers stay 128-byte aligned");
  static constexpr int bytes(int nw) { return nw * (WARP + 8 * S); }
};

// ------------------------------------------------------------- forward ---
template <typename E, int L, int RB, int S, bool GATE>
__global__ void __launch_bounds__((kChainWarps + 1) * 32, 1) fwd_chain_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                        const __grid_constant__ CUtensorMap vmap,
                                                                        const __grid_constant__ CUtensorMap rmap,
                                                                        const __grid_constant__ CUtensorMap ymap,
                                                                        FwdArgs p) {
  static_assert(L % RB == 0 && RB % kCkpt == 0, "batches hold whole checkpoint intervals");
  constexpr int NARR = GATE ? 3 : 2;
  using Lay = ChainLayout<E, L, NARR, 0, S, 0>;  // y overwrites k in the stage
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // per compute warp w: full[S] (its stages landed), done[S] (it is done
  // with a stage and y is in it)
  const uint32_t barb = smem_addr(smem + (size_t)kChainWarps * Lay::WARP);
  auto full = [&](int w, int s) { return barb + 8u * (2 * S * w + s); };
  auto done = [&](int w, int s) { return barb + 8u * (2 * S * w + S + s); };
  auto stage = [&](int w, int s) { return smem + (size_t)w * Lay::WARP + (size_t)s * Lay::STAGE; };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * S * kChainWarps; ++i) mbar_init(barb + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int nseg = (int)((T + L - 1) / L);
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);

  if (wl == kChainWarps) {
    // ------------------------------------------------------ the TMA warp
    // Every copy of the block's compute warps: their first S units, then
    // round by round (unit t of every warp) the y stores from the stages
    // they are done with and, once those have read them, the loads of unit
    // t + S into the same stages.
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();  // inputs are read once
      int nw = 0;
      int xw[kChainWarps], bw[kChainWarps];
      for (int w = 0; w < kChainWarps; ++w) {
        const int64_t ch = (int64_t)blockIdx.x * kChainWarps + w;
        if (ch < p.nchains) {
          bw[w] = (int)(ch / p.nct);
          xw[w] = (int)(ch - (int64_t)bw[w] * p.nct) * 32;
          nw = w + 1;
        }
      }
      auto load = [&](int w, int t) {
        const int s = t % S;
        const uint32_t dst = smem_addr(stage(w, s)), bar = full(w, s);
        mbar_expect_tx(bar, (uint32_t)Lay::STAGE);
        tma_load_3d(dst, &kmap, xw[w], t * L, bw[w], bar, pol);
        tma_load_3d(dst + Lay::ARR, &vmap, xw[w], t * L, bw[w], bar, pol);
        if constexpr (GATE) tma_load_3d(dst + 2 * Lay::ARR, &rmap, xw[w], t * L, bw[w], bar, pol);
      };
      for (int w = 0; w < nw; ++w)
        for (int t = 0; t < S && t < nseg; ++t) load(w, t);
      int issued = min(S, nseg) - 1;
      bool failed = false;
      for (int t = 0; t < nseg && !failed; ++t) {
        const int s = t % S;
        for (int w = 0; w < nw; ++w) {
          if (!mbar_wait_sleepy(done(w, s), (uint32_t)(t / S) & 1u, budget)) {
            raise_timeout(p.hdr, epoch);
            failed = true;
            break;
          }
          if (p.y) tma_store_3d(&ymap, xw[w], t * L, bw[w], smem_addr(stage(w, s)));
        }
        bulk_commit();
        bulk_wait_read_all();  // this round's stores are done with their stages
        if (failed || t + S >= nseg) continue;
        for (int w = 0; w < nw; ++w) load(w, t + S);
        issued = t + S;
      }
      bulk_wait_all();  // every y store complete before the block exits
      if (failed)       // and every issued load landed
        for (int w = 0; w < nw; ++w)
          for (int t = max(0, issued - S + 1); t <= issued; ++t)
            mbar_wait(full(w, t % S), (uint32_t)(t / S) & 1u, budget, nullptr);
    }
    return;
  }

  // -------------------------------------------------------- compute warps
  const int64_t chain = (int64_t)blockIdx.x * kChainWarps + wl;
  if (chain >= p.nchains) return;  // warp-uniform; no block-wide barrier follows
  const int b = (int)(chain / p.nct);
  const int x0 = (int)(chain - (int64_t)b * p.nct) * 32;
  const int64_t c = (int64_t)x0 + lane;
  const bool cok = c < C;
  const int64_t bc = (int64_t)b * C + c;
  const float w = cok ? __ldg(p.w + c) : 0.f, u = cok ? __ldg(p.u + c) : 0.f;
  const float w2 = w * kLog2e, u2 = u * kLog2e;
  unsigned char *const wbuf = stage(wl, 0);
  Run st = run_from(cok ? load_state_in(p.state_in, bc, BC) : st_empty());
  const TileFast fc = tile_fast<RB>(w, w2, u2);
  bool failed = false;
#pragma unroll 1
  for (int t = 0; t < nseg; ++t) {
    const int s = t % S;
    if (!__all_sync(0xffffffffu, mbar_wait(full(wl, s), (uint32_t)(t / S) & 1u, budget, nullptr))) {
      failed = true;
      if (lane == 0) raise_timeout(p.hdr, epoch);
      break;
    }
    const E *ks = reinterpret_cast<const E *>(wbuf + (size_t)s * Lay::STAGE) + lane;
    const E *vs = ks + L * 32;
    const E *rs = ks + 2 * L * 32;
    E *ys = const_cast<E *>(ks);  // y overwrites k (a batch's keys are in registers before its y is written)
    const int64_t t0 = (int64_t)t * L;
    const int n = (int)min((int64_t)L, T - t0);
#pragma unroll 1
    for (int bt = 0; bt < L / RB; ++bt) {
      const int nb = n - bt * RB;
      if (nb <= 0) break;
      const int64_t tb = t0 + bt * RB;
      if (p.ckpt && cok && (tb % kCkpt) == 0) store_ckpt(p.ckpt, tb / kCkpt, bc, BC, run_state(st), w2);
      const E *kb = ks + bt * RB * 32;
      const E *vb = vs + bt * RB * 32;
      const E *rb = rs + bt * RB * 32;
      E *yb = ys + bt * RB * 32;
      const float E0 = fmaf(st.n, w2, st.Panc);
      // the batch's inputs into registers first: the y stores below may
      // alias them as far as the compiler knows, and a load ordered behind
      // a store would expose its latency on every token
      float kj[RB], Vj[RB], Rj[RB];
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        kj[j] = fmaf(-(float)j, fc.we, to_f32(kb[j * 32]));
        Vj[j] = to_f32(vb[j * 32]);
        if constexpr (GATE) Rj[j] = to_f32(rb[j * 32]);
      }
      float mx, mn;
      tree_minmax<RB>(kj, mx, mn);
      const float M = fmaxf(E0, mx * kLog2e);
      const float span = M - mn * kLog2e;  // >= 0
      // the range conditions of the tile forward's fast path (wkv_tile.cu)
      const bool dens_ok = span < 100.f && span - u2 - fc.sh < 60.f;
      const bool state_ok = fc.ewm == 1.f && E0 - M > -90.f;
      const bool ok = fc.ok && (dens_ok || state_ok);
      if (__all_sync(0xffffffffu, ok && nb >= RB)) {
        const float s0 = ex2(E0 - M + fc.sh);
        float al = st.a * s0, be = st.b * s0;
        float yprev = 0.f;
        // the sums at the checkpoints inside the batch, stored after it
        float cka[RB / kCkpt], ckb[RB / kCkpt];
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j > 0 && j % kCkpt == 0) {
            cka[j / kCkpt] = al;
            ckb[j / kCkpt] = be;
          }
          const float e0 = ex2(fmaf(kj[j], kLog2e, -M));
          const float V = Vj[j];
          const float eu = e0 * fc.cu;
          float yv;
          if constexpr (GATE)  // sigma(r) y = num / (den (1 + 2^{-r log2 e})): one reciprocal for both
            yv = fmaf(eu, V, al) * rcp((be + eu) * (1.f + ex2(-Rj[j] * kLog2e)));
          else
            yv = fmaf(eu, V, al) * rcp(be + eu);
          al = fmaf(al, fc.ewm, e0 * V);
          be = fmaf(be, fc.ewm, e0);
          if (j & 1)
            store2<E>(yb + (j - 1) * 32, yb + j * 32, yprev, yv);
          else
            yprev = yv;
        }
        st = Run{al, be, M, fc.nend};
        // after j tokens the sums sit at the exponent M + (j - 1) w2
        // (undecayed mode) or M (decaying mode)
        if (p.ckpt && cok) {
#pragma unroll
          for (int q = 1; q < RB / kCkpt; ++q)
            store_ckpt(p.ckpt, tb / kCkpt + q, bc, BC,
                       St{cka[q], ckb[q], M, fc.nend == 0.f ? 0.f : (float)(q * kCkpt - 1)}, w2);
        }
      } else {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            if (j > 0 && j % kCkpt == 0 && p.ckpt && cok)
              store_ckpt(p.ckpt, (tb + j) / kCkpt, bc, BC, run_state(st), w2);
            float yv = fwd_token(st, to_f32(kb[j * 32]) * kLog2e, Vj[j], u2, w2);
            if constexpr (GATE) yv *= gate_sigmoid(Rj[j]);
            yb[j * 32] = from_f32<E>(yv);
          }
        }
      }
    }
    fence_proxy_async_smem();  // y before the async proxy reads it
    __syncwarp();
    if (lane == 0) mbar_arrive(done(wl, s));  // the TMA warp stores y and reloads the stage
  }
  if (!failed && p.state_out && cok) store_state(p.state_out, bc, BC, run_state(st), w2);
}

// ------------------------------------------------------------ backward ---
struct ChainBwdArgs {
  BwdArgs p;
  float *gw, *gu;
  float4 *chain_sum;  // [B][C] tagged per-chain sums of dL/dw, dL/du
};

// recompute_batch of wkv_bwd_math.cuh with the batch maximum taken as a
// tree.  WY: Yw[j] is multiplied by the recomputed output y_j (the gated
// backward's dL/dr = grad_o sigma'(r) y).
template <int RB, bool WY>
__device__ __forceinline__ bool chain_recompute(const float (&K)[RB], const float (&V)[RB], const float (&Gy)[RB],
                                                float w2, float u2, const FastC &fc, float xa, float xb, float xP,
                                                float (&qv)[RB], float (&gam)[RB], float (&eta)[RB],
                                                float (&e2v)[RB], float &M, float (&Yw)[RB]) {
  const float E0 = xP;
  float kj[RB];
  const bool ok = fast_prep_tree<RB>(K, E0, u2, fc.w2e, kj, M);
  if (__all_sync(0xffffffffu, ok)) {
    const float s0 = ex2(E0 - M);
    float al = xa * s0, be = xb * s0;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      const float e0 = ex2(kj[j] - M);
      const float eu = e0 * fc.cu, ek = e0 * fc.cw;
      const float rden = rcp(be + eu);
      const float y = fmaf(eu, V[j], al) * rden;
      gam[j] = Gy[j] * rden;
      eta[j] = gam[j] * y;
      if constexpr (WY) Yw[j] *= y;
      e2v[j] = eu;
      al = fmaf(al, fc.ewm, ek * V[j]);
      be = fmaf(be, fc.ewm, ek);
    }
    return true;
  }
  float xn = 0.f;
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

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void *map, int x, int y, int z, int w, uint32_t bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(bar), "l"(policy)
      : "memory");
}

// Batches are one checkpoint interval (RB = kCkpt tokens), so every batch
// starts on a checkpoint: the unit's checkpoints arrive by TMA with its k,
// v and grad_y tiles (a fourth region of the stage, [L/RB][3][32] floats)
// and are the batch-start states as they are; no forward pass over the
// unit precedes its sweep.
// GATE: the loss depends on o = sigma(r) * y and grad_y is dL/do (the tile
// backward's gate, wkv_tile_bwd.cu): r arrives with k, v and grad_o, the
// WKV gradient is grad_o sigma(r), and dL/dr = grad_o sigma'(r) y from the
// recomputed y overwrites r and leaves with dL/dk and dL/dv.
// STATE: the state terms of a sequence split across calls (as the tile
// backward's): a chain's adjoint starts from the final state's gradient,
// its last batch sweeps exactly to token T-1 (the zero-filled padding would
// decay that adjoint), and its first unit writes the initial state's
// gradient.
template <typename E, int L, int RB, int S, bool GATE, bool STATE>
__global__ void __launch_bounds__((kChainWarps + 1) * 32, 1) bwd_chain_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                        const __grid_constant__ CUtensorMap vmap,
                                                                        const __grid_constant__ CUtensorMap gmap,
                                                                        const __grid_constant__ CUtensorMap rmap,
                                                                        const __grid_constant__ CUtensorMap ckmap,
                                                                        const __grid_constant__ CUtensorMap gkmap,
                                                                        const __grid_constant__ CUtensorMap gvmap,
                                                                        const __grid_constant__ CUtensorMap grmap,
                                                                        ChainBwdArgs a) {
  static_assert(L % kCkpt == 0 && RB == kCkpt, "batches are checkpoint intervals");
  static_assert(!(STATE && GATE), "no entry point combines the state terms and the gate");
  constexpr int NB = L / RB;
  constexpr int NARR = GATE ? 4 : 3;  // k, v, grad_y (and r)
  constexpr int CKB = NB * 96 * 4;    // the unit's checkpoints
  using Lay = ChainLayout<E, L, NARR, 0, S, 0, CKB>;  // the gradients overwrite k, v (and r) in the stage
  const BwdArgs &p = a.p;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // per compute warp w: full[S] (its stages landed), done[S] (it is done
  // with a stage and its outputs are in it)
  const uint32_t barb = smem_addr(smem + (size_t)kChainWarps * Lay::WARP);
  auto full = [&](int w, int s) { return barb + 8u * (2 * S * w + s); };
  auto done = [&](int w, int s) { return barb + 8u * (2 * S * w + S + s); };
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * S * kChainWarps; ++i) mbar_init(barb + 8u * i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int G = (int)gridDim.x * kChainWarps;
  const int nchains = (int)p.nchains, nct = (int)p.nct;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int nseg = (int)((T + L - 1) / L);
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  const unsigned t_sum = tile_flag(epoch, 3u);
  // units of compute warp w: chain gw + (j / nseg) G, position
  // nseg - 1 - j % nseg, followed by cursors (no divisions in the unit loop)
  auto units_of = [&](int w) {
    const int gw = (int)blockIdx.x * kChainWarps + w;
    return (nchains > gw ? (nchains - gw + G - 1) / G : 0) * nseg;
  };
  struct Cursor {
    int chain, pos, b, x0;
  };
  auto first = [&](int w) {
    const int gw = (int)blockIdx.x * kChainWarps + w;
    Cursor u{gw, nseg - 1, gw / nct, 0};
    u.x0 = (gw - u.b * nct) * 32;
    return u;
  };
  auto next = [&](Cursor &u) {
    if (--u.pos < 0) {
      u.pos = nseg - 1;
      u.chain += G;
      u.b = u.chain / nct;
      u.x0 = (u.chain - u.b * nct) * 32;
    }
  };
  auto stage = [&](int w, int s) { return smem + (size_t)w * Lay::WARP + (size_t)s * Lay::STAGE; };

  if (wl == kChainWarps) {
    // ------------------------------------------------------ the TMA warp
    // Issues every copy of the block's compute warps, so that none of them
    // waits on a copy instruction: each warp's first S units, then round by
    // round (unit j of every warp): the stores of dL/dk and dL/dv from the
    // stages the warps are done with, and, once those stores have read
    // them, the loads of units j + S into the same stages.
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      Cursor ic[kChainWarps], sc[kChainWarps];  // the next unit to load, to store
      int tot[kChainWarps], maxtot = 0;
      for (int w = 0; w < kChainWarps; ++w) {
        ic[w] = sc[w] = first(w);
        tot[w] = units_of(w);
        maxtot = max(maxtot, tot[w]);
      }
      auto load = [&](int w, int j) {
        const int s = j % S;
        const uint32_t dst = smem_addr(stage(w, s)), bar = full(w, s);
        mbar_expect_tx(bar, (uint32_t)Lay::STAGE);
        const Cursor &u = ic[w];
        tma_load_3d(dst, &kmap, u.x0, u.pos * L, u.b, bar, pol);
        tma_load_3d(dst + Lay::ARR, &vmap, u.x0, u.pos * L, u.b, bar, pol);
        tma_load_3d(dst + 2 * Lay::ARR, &gmap, u.x0, u.pos * L, u.b, bar, pol);
        if constexpr (GATE) tma_load_3d(dst + 3 * Lay::ARR, &rmap, u.x0, u.pos * L, u.b, bar, pol);
        tma_load_4d(dst + NARR * Lay::ARR, &ckmap, u.x0, u.b, 0, u.pos * NB, bar, pol);
        next(ic[w]);
      };
      int issued[kChainWarps];
      for (int w = 0; w < kChainWarps; ++w) {
        issued[w] = -1;
        for (int j = 0; j < S && j < tot[w]; ++j) {
          load(w, j);
          issued[w] = j;
        }
      }
      bool failed = false;
      for (int j = 0; j < maxtot && !failed; ++j) {
        const int s = j % S;
        for (int w = 0; w < kChainWarps; ++w) {
          if (j >= tot[w]) continue;
          if (!mbar_wait_sleepy(done(w, s), (uint32_t)(j / S) & 1u, budget)) {
            raise_timeout(p.hdr, epoch);
            failed = true;
            break;
          }
          const uint32_t src = smem_addr(stage(w, s));
          tma_store_3d(&gkmap, sc[w].x0, sc[w].pos * L, sc[w].b, src);
          tma_store_3d(&gvmap, sc[w].x0, sc[w].pos * L, sc[w].b, src + Lay::ARR);
          if constexpr (GATE) tma_store_3d(&grmap, sc[w].x0, sc[w].pos * L, sc[w].b, src + 3 * Lay::ARR);
          next(sc[w]);
        }
        bulk_commit();
        bulk_wait_read_all();  // this round's stores are done with their stages
        if (failed) break;
        for (int w = 0; w < kChainWarps; ++w)
          if (j + S < tot[w]) {
            load(w, j + S);
            issued[w] = j + S;
          }
      }
      bulk_wait_all();  // every store complete before the block exits
      if (failed) {
        // every issued load lands before the block exits (each warp's
        // stages in order; those it consumed have completed already)
        for (int w = 0; w < kChainWarps; ++w)
          for (int j = max(0, issued[w] - S + 1); j <= issued[w]; ++j)
            mbar_wait(full(w, j % S), (uint32_t)(j / S) & 1u, budget, nullptr);
      }
    }
    __syncthreads();
    finish_block(p.hdr, gridDim.x);
    return;
  }

  // -------------------------------------------------------- compute warps
  const int total = units_of(wl);
  unsigned char *const wbuf = stage(wl, 0);
  bool failed = false;
  int b = 0, x0 = 0;
  int64_t c = 0, bc = 0;
  bool cok = false;
  float w2 = 0.f, u2 = 0.f;
  FastC fc{};
  float rah = 0.f, rhh = 0.f, rahp = 0.f, rhhp = 0.f, Ranc = kEmptyR, m = 0.f;
  double gw_d = 0.0, gu_d = 0.0;
  Cursor uc = first(wl);
#pragma unroll 1
  for (int j = 0; j < total; ++j, next(uc)) {
    const int s = j % S;
    const int pos = uc.pos;
    if (pos == nseg - 1) {
      // a new chain: its constants, and the adjoint after its last token (empty)
      b = uc.b;
      x0 = uc.x0;
      c = (int64_t)x0 + lane;
      cok = c < C;
      bc = (int64_t)b * C + c;
      w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
      u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
      fc = fast_consts<RB>(w2, u2);
      rah = rhh = rahp = rhhp = 0.f;
      Ranc = kEmptyR;
      m = 0.f;
      gw_d = gu_d = 0.0;
      if constexpr (STATE) {
        if (p.gs_out && cok) end_adjoint(p.gs_out[bc], p.gs_out[BC + bc], p.p_out[bc], rah, rhh, Ranc);
      }
    }
    if (!__all_sync(0xffffffffu, mbar_wait(full(wl, s), (uint32_t)(j / S) & 1u, budget, nullptr))) {
      failed = true;
      if (lane == 0) raise_timeout(p.hdr, epoch);
      break;
    }
    const int64_t t0 = (int64_t)pos * L;
    const int n = (int)min((int64_t)L, T - t0);
    const E *kt = reinterpret_cast<const E *>(wbuf + (size_t)s * Lay::STAGE) + lane;
    const E *vt = kt + L * 32;
    const E *gt = kt + 2 * L * 32;
    E *rt = const_cast<E *>(kt) + 3 * L * 32;  // gate input, then dL/dr (GATE only)
    // a batch's inputs; with the gate, Gy becomes grad_o sigma(r) and Gd
    // grad_o sigma'(r) (times y once the recompute has formed it)
    auto load_batch = [&](int bt, float(&K)[RB], float(&V)[RB], float(&Gy)[RB], float(&Gd)[RB]) {
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        K[q] = to_f32(kt[(bt * RB + q) * 32]) * kLog2e;
        V[q] = to_f32(vt[(bt * RB + q) * 32]);
        Gy[q] = to_f32(gt[(bt * RB + q) * 32]);
        if constexpr (GATE) {
          float sg, ds;
          gate_sigmoid_slope(to_f32(rt[(bt * RB + q) * 32]), sg, ds);
          Gd[q] = Gy[q] * ds;
          Gy[q] *= sg;
        }
      }
    };

    // the batch-start states: the unit's checkpoints ([NB][3][32] floats)
    const float *sts = reinterpret_cast<const float *>(wbuf + (size_t)s * Lay::STAGE + NARR * Lay::ARR);

    // ---- batches last to first, recompute then reverse sweep; dL/dk and
    // dL/dv overwrite k and v of the stage (a batch's k and v are in
    // registers before its sweep writes them)
    E *okp = const_cast<E *>(kt);
    E *ovp = const_cast<E *>(vt);
    float gw_acc = 0.f, gu_acc = 0.f;
#pragma unroll 1
    for (int bi = 0; bi < NB; ++bi) {
      const int bt = NB - 1 - bi;
      if (n - bt * RB <= 0) continue;  // only padding past T: nothing to sweep
      float K[RB], V[RB], Gy[RB], Gd[RB];
      load_batch(bt, K, V, Gy, Gd);
      float qv[RB], gam[RB], eta[RB], e2v[RB], Mb;
      const bool fast = chain_recompute<RB, GATE>(K, V, Gy, w2, u2, fc, sts[bt * 96 + lane],
                                                  sts[bt * 96 + 32 + lane], sts[bt * 96 + 64 + lane], qv, gam,
                                                  eta, e2v, Mb, Gd);
      if constexpr (GATE) {
        // dL/dr over r (this batch's r is in registers already)
#pragma unroll
        for (int q = 0; q < RB; q += 2)
          store2<E>(rt + (bt * RB + q) * 32, rt + (bt * RB + q + 1) * 32, Gd[q], Gd[q + 1]);
      }
      E *gkp = okp + bt * RB * 32;
      E *gvp = ovp + bt * RB * 32;
      // the reverse sweep of the tile backward (wkv_tile_bwd.cu): fast in the
      // batch's coordinates when the carried adjoint's scale allows, else per
      // token with the running anchor
      const float rn_end = fmaf(-m, w2, Ranc);
      const float xin = fmaf((float)RB, fc.w2e, Mb) - rn_end;
      const int nv = n - bt * RB;  // rows of the batch inside T
      if (__all_sync(0xffffffffu, fast && xin < 100.f && (!STATE || nv >= RB))) {
        const float F = ex2(xin);
        float ra = rah * F, rh = rhh * F, rap = rahp * F, rhp = rhhp * F;
        const float ckf = fc.cw * ex2(-u2);  // ek = e2 * ckf
#pragma unroll
        for (int q = RB - 1; q >= 0; --q) {
          const float ek = e2v[q] * ckf;
          const float gv = fmaf(gam[q], e2v[q], ek * ra);
          const float gk = fmaf(V[q], gv, -fmaf(eta[q], e2v[q], ek * rh));
          gw_acc = fmaf(ek, fmaf(V[q], rap, -rhp), gw_acc);
          gu_acc = fmaf(e2v[q], fmaf(gam[q], V[q], -eta[q]), gu_acc);
          store2<E>(gkp + q * 32, gvp + q * 32, gk, gv);
          rap = fc.ewm * (rap + ra);
          rhp = fc.ewm * (rhp + rh);
          ra = fmaf(ra, fc.ewm, gam[q]);
          rh = fmaf(rh, fc.ewm, eta[q]);
        }
        rah = ra;
        rhh = rh;
        rahp = rap;
        rhhp = rhp;
        Ranc = Mb;
        m = 0.f;
        continue;
      }
      if (fast) {  // the fast recompute leaves the scales implicit: D_t = den 2^{M + q w2e}
#pragma unroll
        for (int q = 0; q < RB; ++q) qv[q] = fmaf((float)q, fc.w2e, Mb);
      }
#pragma unroll
      for (int q = RB - 1; q >= 0; --q) {
        if (STATE && q >= nv) continue;  // past T
        const float rn = fmaf(-m, w2, Ranc);  // scale of the adjoint after token t
        const float tn = ex2(K[q] - rn);      // e^{k_t} 2^{-r_{t+1}} (<= 1)
        const float gv = fmaf(gam[q], e2v[q], tn * rah);
        const float gk = fmaf(V[q], gv, -fmaf(eta[q], e2v[q], tn * rhh));
        gw_acc = fmaf(tn, fmaf(V[q], rahp, -rhhp), gw_acc);
        gu_acc = fmaf(e2v[q], fmaf(gam[q], V[q], -eta[q]), gu_acc);
        store2<E>(gkp + q * 32, gvp + q * 32, gk, gv);
        const float m1 = m + 1.f;
        const float Rc = fmaf(-m1, w2, Ranc);
        const float d = qv[q] - Rc;
        const float x = ex2(-fabsf(d));
        const bool reset = d < 0.f;
        const float fg = reset ? 1.f : x, fo = reset ? x : 1.f;
        rahp = fo * (rah + rahp);
        rhhp = fo * (rhh + rhhp);
        rah = fmaf(rah, fo, gam[q] * fg);
        rhh = fmaf(rhh, fo, eta[q] * fg);
        Ranc = reset ? qv[q] : Ranc;
        m = reset ? 0.f : m1;
      }
    }
    if (pos == 0 && cok) {
      // share of the initial state A_0, B_0 (zero for the empty state): the
      // checkpoint before token 0
      const float r0 = fmaf(-m, w2, Ranc);
      gw_acc = fmaf(ex2(sts[64 + lane] - r0), fmaf(sts[lane], rahp, -sts[32 + lane] * rhhp), gw_acc);
      if constexpr (STATE) {
        if (p.gs_in) store_state_grad(p.gs_in, p.state_in, bc, BC, rah, rhh, r0);
      }
    }
    gw_d += (double)gw_acc;
    gu_d += (double)gu_acc;
    fence_proxy_async_smem();  // dL/dk, dL/dv before the async proxy reads them
    __syncwarp();
    if (lane == 0) mbar_arrive(done(wl, s));  // the TMA warp stores them and reloads the stage
    if (pos == 0 && cok) {
      // the chain's sums, then (last batch row) the B chains in batch-row order
      st_relaxed_v4(a.chain_sum + bc, make_float4((float)gw_d, (float)gu_d, tagf(t_sum), 0.f));
      if (b == (int)p.B - 1) {
        double sw, su;
        if (!sum_tagged(a.chain_sum + c, C, (int)p.B, t_sum, sw, su, budget)) raise_timeout(p.hdr, epoch);
        a.gw[c] = (float)sw;
        a.gu[c] = (float)su;
      }
    }
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

// ------------------------------------------------------------------ host ---
template <typename E, int L, int RB, bool GATE>
static cudaError_t launch_fwd_chain_t(const FwdArgs &f, int dtype, cudaStream_t st) {
  CUtensorMap km, vm, rm, ym;
  if (!encode_btc(&km, f.k, dtype, f.B, f.T, f.C, L) || !encode_btc(&vm, f.v, dtype, f.B, f.T, f.C, L))
    return cudaErrorInvalidValue;
  rm = vm;
  ym = km;  // unused placeholders when there is no gate / no y
  if (GATE && !encode_btc(&rm, f.r, dtype, f.B, f.T, f.C, L)) return cudaErrorInvalidValue;
  if (f.y && !encode_btc(&ym, f.y, dtype, f.B, f.T, f.C, L)) return cudaErrorInvalidValue;
  constexpr int STG = (GATE ? 3 : 2) * L * 32 * (int)sizeof(E);
  constexpr int S = kChainFwdBytes / STG > 2 ? kChainFwdBytes / STG : 2;
  // the compute warps' stages, then two barriers per stage and warp
  constexpr int smem = kChainWarps * (ChainLayout<E, L, GATE ? 3 : 2, 0, S, 0>::WARP + 16 * S);
  auto kern = fwd_chain_kernel<E, L, RB, S, GATE>;
  int occ = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, (kChainWarps + 1) * 32, smem, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  if ((f.T + L - 1) / L >= (int64_t)1 << 31 || f.T >= (int64_t)1 << 31) return cudaErrorInvalidValue;
  const int64_t grid = (f.nchains + kChainWarps - 1) / kChainWarps;
  if (grid >= (int64_t)1 << 31) return cudaErrorInvalidValue;
  return launch_kernel(kern, dim3((unsigned)grid), dim3((kChainWarps + 1) * 32), (size_t)smem, st, km, vm, rm, ym,
                       f);
}

cudaError_t launch_forward_chain(const FwdArgs &f, int dtype, cudaStream_t st) {
  if (f.r)
    return dtype == 0 ? launch_fwd_chain_t<float, kTileLF32, kFrbF32, true>(f, dtype, st)
                      : launch_fwd_chain_t<uint16_t, WKV_CHAIN_LF, kFrbF32, true>(f, dtype, st);
  return dtype == 0 ? launch_fwd_chain_t<float, kTileLF32, kFrbF32, false>(f, dtype, st)
                    : launch_fwd_chain_t<uint16_t, WKV_CHAIN_LF, WKV_CHAIN_FRB, false>(f, dtype, st);
}

template <typename E, int L, int RB, int S, bool GATE, bool STATE>
static cudaError_t launch_bwd_chain_t(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *chain_sum,
                                      int num_sms, cudaStream_t st) {
  CUtensorMap km, vm, gm, rm, ckm, gkm, gvm, grm;
  constexpr int NB = L / RB;
  if (!encode_btc(&km, p.k, dtype, p.B, p.T, p.C, L) || !encode_btc(&vm, p.v, dtype, p.B, p.T, p.C, L) ||
      !encode_btc(&gm, p.gy, dtype, p.B, p.T, p.C, L) || !encode_btc(&gkm, p.gk, dtype, p.B, p.T, p.C, L) ||
      !encode_btc(&gvm, p.gv, dtype, p.B, p.T, p.C, L) ||
      !encode_ckpt(&ckm, p.ckpt, p.B, p.C, (p.T + kCkpt - 1) / kCkpt, NB))
    return cudaErrorInvalidValue;
  rm = gm;  // placeholders without the gate
  grm = gkm;
  if (GATE && (!encode_btc(&rm, p.r, dtype, p.B, p.T, p.C, L) || !encode_btc(&grm, p.gr, dtype, p.B, p.T, p.C, L)))
    return cudaErrorInvalidValue;
  // the compute warps' stages, then two barriers per stage and warp
  constexpr int smem = kChainWarps * (ChainLayout<E, L, GATE ? 4 : 3, 0, S, 0, NB * 96 * 4>::WARP + 16 * S);
  auto kern = bwd_chain_kernel<E, L, RB, S, GATE, STATE>;
  int occ = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, (kChainWarps + 1) * 32, smem, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int64_t nseg = (p.T + L - 1) / L;
  if (nseg * p.nchains >= (int64_t)1 << 31) return cudaErrorInvalidValue;  // unit indices are 31-bit
  // one resident wave (cooperative launch: the last batch row's chains wait
  // on the other rows' sums), the chains dealt out evenly
  const int64_t max_warps = (int64_t)occ * num_sms * kChainWarps;
  const int64_t rounds = (p.nchains + max_warps - 1) / max_warps;
  const int64_t grid = ((p.nchains + rounds - 1) / rounds + kChainWarps - 1) / kChainWarps;
  ChainBwdArgs a{};
  a.p = p;
  a.gw = gw;
  a.gu = gu;
  a.chain_sum = chain_sum;
  void *args[] = {&km, &vm, &gm, &rm, &ckm, &gkm, &gvm, &grm, &a};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3((kChainWarps + 1) * 32), args,
                                     (size_t)smem, st);
}

cudaError_t launch_backward_chain(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *chain_sum, int num_sms,
                                  cudaStream_t st) {
  if (p.r && (p.gs_out || p.gs_in)) return cudaErrorInvalidValue;  // no entry point asks for both
  if (p.r)  // the gate's fourth tile per stage: 64-token units (32 fp32), three stages
    return dtype == 0 ? launch_bwd_chain_t<float, kTileLF32, kCkpt, 3, true, false>(p, dtype, gw, gu, chain_sum,
                                                                                      num_sms, st)
                      : launch_bwd_chain_t<uint16_t, kTileLBF16, kCkpt, 3, true, false>(p, dtype, gw, gu, chain_sum,
                                                                                         num_sms, st);
  if (p.gs_out || p.gs_in)
    return dtype == 0 ? launch_bwd_chain_t<float, kTileLF32, kCkpt, WKV_CHAIN_SB, false, true>(p, dtype, gw, gu,
                                                                                                 chain_sum, num_sms, st)
                      : launch_bwd_chain_t<uint16_t, WKV_CHAIN_LB, kCkpt, WKV_CHAIN_SB, false, true>(
                            p, dtype, gw, gu, chain_sum, num_sms, st);
  return dtype == 0 ? launch_bwd_chain_t<float, kTileLF32, kCkpt, WKV_CHAIN_SB, false, false>(p, dtype, gw, gu,
                                                                                                chain_sum, num_sms, st)
                    : launch_bwd_chain_t<uint16_t, WKV_CHAIN_LB, kCkpt, WKV_CHAIN_SB, false, false>(
                          p, dtype, gw, gu, chain_sum, num_sms, st);
}

}  // namespace wkv

