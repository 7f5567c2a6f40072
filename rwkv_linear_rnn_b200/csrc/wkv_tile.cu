// wkv_tile.cu -- tile forward of libwkv: the default forward on sm_100a when
// the [B, T, C] rows are 16-byte aligned.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), run in the RNN
// form of section "RNN-유사추론" (eq. WKV_t) over the max-rescaled state; the
// time axis is split into units joined by an associative scan, as in section
// "Transformer-유사학습" (WKV done as a scan).
//
// A unit is one chain (batch row b, 32 channels = the 32 lanes of a warp)
// and L consecutive tokens.  Warps are persistent and own units statically
// (warp g takes units g, g + G, g + 2G, ... in position-major order: every
// chain's unit 0, then every chain's unit 1, ...).  Per unit:
//   load    one TMA copy per tensor brings the unit's k, v (and r) tile into
//           the warp's shared memory; the next unit's copy is issued into
//           the other buffer before this unit is computed, so HBM traffic
//           overlaps the arithmetic;
//   pass 1  the unit's summary from the resident tile (one ex2 per token);
//   join    the summary is published, then the state entering the unit is
//           formed by a decoupled look-back over the chain's earlier units:
//           the nearest unit that has published its inclusive prefix, then
//           the summaries of the units after it, folded left to right.  Every
//           prefix is therefore the same left fold of unit summaries from the
//           chain start, whoever computes it: results are bit-reproducible;
//   pass 2  the recurrence replayed from the joined state over the resident
//           tile; y overwrites k in shared memory and leaves by one TMA store;
//           checkpoints every 16 tokens and the final state are written.
// HBM traffic is the algorithmic 12 B (fp32) / 6 B (bf16) per channel-token
// plus two 16-byte records per unit and lane.
#include <cuda.h>

#include <algorithm>
#include <atomic>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_tile.cuh"

namespace wkv {

bool encode_btc(CUtensorMap *m, const void *ptr, int dtype, int64_t B, int64_t T, int64_t C, int box_t);

// Summary of 32 full tokens from the empty state (pass 1): A = sum_j e^{(31-j) w + k_j} v_j
// and B, against their largest exponent.  ks, vs: this lane's column.
template <typename E>
__device__ __forceinline__ St tile_summary32(const E *ks, const E *vs, float w) {
  float e[32];
  float m = -3.0e38f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    e[j] = fmaf((float)(31 - j), w, to_f32(ks[j * 32]));
    m = fmaxf(m, e[j]);
  }
  const float m2 = m * kLog2e;
  float a = 0.f, b = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float x = ex2(fmaf(e[j], kLog2e, -m2));
    a = fmaf(x, to_f32(vs[j * 32]), a);
    b += x;
  }
  return St{a, b, m2, 0.f};
}

// The state entering unit `pos` of a chain: the left fold, from the chain's
// initial state, of the summaries of units 0 .. pos-1.  The status words say
// how far back the nearest published inclusive prefix is (lane l inspects
// unit pos-1-l; positions before the chain start count as a prefix: the
// initial state), provided every unit after it has its summary out.  The
// prefix and those summaries are then loaded together and every lane checks
// the tags of its words; the warp folds them, in position order, only when
// all of them check, and reads again otherwise.  Bounded: past `budget_ns`
// (or once the launch is aborted) the status word of the workspace gets
// WKV_ERR_TIMEOUT and the fold goes on with whatever the records hold.
__device__ St tile_lookback(const unsigned *status, const float4 *rec, int pos, int chain, int nchains,
                            unsigned epoch, const St &s_in, float len, float w2, int64_t budget_ns,
                            WsHeader *hdr, int lane, bool &failed) {
  const unsigned t_agg = tile_flag(epoch, kFlagAgg), t_inc = tile_flag(epoch, kFlagInc);
  const int q = pos - 1 - lane;
  const unsigned *sw = status + (int64_t)(q < 0 ? 0 : q) * nchains + chain;
  const uint64_t t0 = global_ns();
  unsigned backoff = 32;
  St acc = s_in;
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
      const int q0 = pos - 1 - first;
      bool ok = true;
      acc = s_in;
      if (q0 >= 0) {
        const float4 *d = rec + ((int64_t)q0 * nchains + chain) * kFwdRecWords + lane;
        const float4 x = ld_relaxed_v4(d + 32), y = ld_relaxed_v4(d + 64);
        ok = tag_is(x.w, t_inc) && tag_is(y.y, t_inc);
        acc = St{x.x, x.y, x.z, y.x};
      }
      // the summaries of units q0+1 .. pos-1, eight loads in flight per step
#pragma unroll 1
      for (int d0 = 0; d0 < first; d0 += 8) {
        float4 r[8];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (d0 + jj < first) r[jj] = ld_relaxed_v4(rec + ((int64_t)(q0 + 1 + d0 + jj) * nchains + chain) * kFwdRecWords + lane);
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          if (d0 + jj < first) {
            ok = ok && tag_is(r[jj].w, t_agg);
            acc = combine(acc, St{r[jj].x, r[jj].y, r[jj].z, 0.f}, len, w2);
          }
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

// NARR tensors per unit (k, v, and the gate input r with GATE).  Shared
// memory per warp: three buffers of NARR tiles [L][32], then (after all
// warps' buffers) three mbarriers per warp.
template <typename E, int L, int NARR>
struct TileLayout {
  static constexpr int NBUF = 3;
  static constexpr int ARR = L * 32 * (int)sizeof(E);
  static constexpr int BUF = NARR * ARR;
  static constexpr int WARP = NBUF * BUF;
  static_assert(ARR % 128 == 0, "TMA destinations stay 128-byte aligned");
  static constexpr int bytes(int nw) { return nw * WARP + nw * 8 * NBUF; }
};

constexpr int kSpecDepth = 8;  // records prefetched for a predicted look-back

// Coordinates of a unit and this lane's per-channel constants.
struct TileUnit {
  int pos, chain, b, x0, n;
  int64_t c, t0, bc;
  bool cok;
  float w, u, w2, u2;
};

// The warp's units are u_0, u_1, ... (u_t = g + t G).  Software pipelined
// over its units, one step per unit: step t runs pass 1 of u_{t+1} and
// publishes its summary, prefetches the tiles of u_{t+2}, then joins u_t and
// runs its pass 2.  By the time u_t looks back, the summaries of the units
// before it that other warps run in the same step were published one step
// earlier, and so were the prefixes of the step before: the look-back finds
// its records out instead of waiting for peers at the same stage.  Three
// tile buffers rotate: u_t's (pass 2), u_{t+1}'s (pass 1), u_{t+2}'s (in
// flight).
template <typename E, int L, int RB, bool GATE>
__global__ void __launch_bounds__(kTileFwdWarps * 32, 3) fwd_tile_kernel(const __grid_constant__ CUtensorMap kmap,
                                                                      const __grid_constant__ CUtensorMap vmap,
                                                                      const __grid_constant__ CUtensorMap rmap,
                                                                      const __grid_constant__ CUtensorMap ymap,
                                                                      TileFwdArgs a) {
  static_assert(L % 32 == 0 && L % RB == 0 && kCkpt % RB == 0, "units hold whole checkpoint intervals");
  constexpr int NARR = GATE ? 3 : 2;
  using Lay = TileLayout<E, L, NARR>;
  constexpr int NBUF = Lay::NBUF;
  const FwdArgs &p = a.f;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = (int)(blockDim.x >> 5);
  unsigned char *wbuf = smem + (size_t)wl * Lay::WARP;
  const uint32_t bar0 = smem_addr(smem + (size_t)nw * Lay::WARP) + 8u * NBUF * wl;
  if (lane == 0) {
    for (int k = 0; k < NBUF; ++k) mbar_init(bar0 + 8u * k, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const int G = (int)gridDim.x * nw;
  const int g = (int)blockIdx.x * nw + wl;
  const int nseg = (int)a.nseg, nchains = (int)p.nchains, nct = (int)p.nct;
  const int total = nseg * nchains;
  const int nu = total > g ? (total - g + G - 1) / G : 0;  // units of this warp
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  const uint64_t pol = l2_policy_evict_first();  // inputs are read once
  const unsigned t_agg = tile_flag(epoch, kFlagAgg), t_inc = tile_flag(epoch, kFlagInc);

  auto unit_of = [&](int t) -> TileUnit {
    TileUnit U;
    const int unit = g + t * G;
    U.pos = unit / nchains;
    U.chain = unit - U.pos * nchains;
    U.b = U.chain / nct;
    U.x0 = (U.chain - U.b * nct) * 32;
    U.c = (int64_t)U.x0 + lane;
    U.cok = U.c < C;
    U.t0 = (int64_t)U.pos * L;
    U.n = (int)min((int64_t)L, T - U.t0);
    U.bc = (int64_t)U.b * C + U.c;
    U.w = U.cok ? __ldg(p.w + U.c) : 0.f;
    U.u = U.cok ? __ldg(p.u + U.c) : 0.f;
    U.w2 = U.w * kLog2e;
    U.u2 = U.u * kLog2e;
    return U;
  };
  // lane 0: the TMA copies of step t's unit into buffer t % NBUF
  int iss_t = -1, wt_t = -1;
  auto issue = [&](int t) {
    const int unit = g + t * G;
    const int pos = unit / nchains, chain = unit - pos * nchains;
    const int b = chain / nct;
    const int x = (chain - b * nct) * 32;
    const int bf = t % NBUF;
    const uint32_t dst = smem_addr(wbuf + (size_t)bf * Lay::BUF), bar = bar0 + 8u * bf;
    mbar_expect_tx(bar, (uint32_t)Lay::BUF);
    tma_load_3d(dst, &kmap, x, pos * L, b, bar, pol);
    tma_load_3d(dst + Lay::ARR, &vmap, x, pos * L, b, bar, pol);
    if constexpr (GATE) tma_load_3d(dst + 2 * Lay::ARR, &rmap, x, pos * L, b, bar, pol);
    iss_t = t;
  };
  bool failed = false;
  auto wait_tiles = [&](int t) {
    if (failed) return;
    if (mbar_wait(bar0 + 8u * (t % NBUF), (uint32_t)(t / NBUF) & 1u, budget, nullptr)) {
      wt_t = t;
    } else {
      failed = true;
      if (lane == 0) raise_timeout(p.hdr, epoch);
    }
  };
  // pass 1 of step t's unit and its publication: the summary, or, for a
  // chain's first unit, its inclusive prefix right away
  auto pass1 = [&](int t, const TileUnit &U) -> St {
    const E *ks = reinterpret_cast<const E *>(wbuf + (size_t)(t % NBUF) * Lay::BUF) + lane;
    const E *vs = ks + L * 32;
    St agg = st_empty();
    if (U.pos + 1 >= nseg) return agg;  // a chain's last unit: nobody needs its summary
    agg = tile_summary32<E>(ks, vs, U.w);
#pragma unroll
    for (int h = 1; h < L / 32; ++h)
      agg = combine(agg, tile_summary32<E>(ks + h * 1024, vs + h * 1024, U.w), 32.f, U.w2);
    if (p.hold_first && U.pos == 0) return agg;  // test hook: never publish
    const int64_t unit = (int64_t)g + (int64_t)t * G;
    if (U.pos == 0) {
      const St s_in = U.cok ? load_state_in(p.state_in, U.bc, BC) : st_empty();
      tile_put_inc(a.rec, unit, combine(s_in, agg, (float)L, U.w2), t_inc, lane);
      if (lane == 0) st_relaxed_u32(p.flags + unit, t_inc);
    } else {
      tile_put_agg(a.rec, unit, agg, U.w2, t_agg, lane);
      if (lane == 0) st_relaxed_u32(p.flags + unit, t_agg);
    }
    return agg;
  };

  if (lane == 0) {
    if (nu > 0) issue(0);
    if (nu > 1) issue(1);
  }
  St agg_cur = st_empty();
  TileUnit cur = unit_of(0);
  if (nu > 0) {
    wait_tiles(0);
    agg_cur = pass1(0, cur);
  }
#pragma unroll 1
  for (int t = 0; t < nu; ++t) {
    // ---- u_t's look-back, predicted: the units of its chain that run in
    // step t (positions from p0) published their summaries in step t-1, and
    // the unit before them (position p0-1, run in step t-1) its prefix; a
    // chain's first unit publishes only its prefix, so the fold starts from
    // the prefix at position qi = max(p0 - 1, 0) and adds the summaries of
    // positions qi+1 .. pos-1.  Their loads are issued now and checked after
    // the next unit's pass 1.
    const int p0 = max(0, (int)(((int64_t)t * G - cur.chain + nchains - 1) / nchains));
    const int qi = max(p0 - 1, 0);
    const int dspec = cur.pos - 1 - qi;
    const bool spec = cur.pos > 0 && dspec <= kSpecDepth;
    float4 sx = make_float4(0.f, 0.f, 0.f, 0.f), sy = sx, sa[kSpecDepth];
    if (spec) {
      const float4 *d = a.rec + ((int64_t)qi * nchains + cur.chain) * kFwdRecWords + lane;
      sx = ld_relaxed_v4(d + 32);
      sy = ld_relaxed_v4(d + 64);
#pragma unroll
      for (int j = 0; j < kSpecDepth; ++j)
        if (j < dspec) sa[j] = ld_relaxed_v4(a.rec + ((int64_t)(qi + 1 + j) * nchains + cur.chain) * kFwdRecWords + lane);
    }
    // ---- pass 1 of the next unit
    TileUnit nxt = cur;
    St agg_nxt = st_empty();
    if (t + 1 < nu) {
      nxt = unit_of(t + 1);
      wait_tiles(t + 1);
      agg_nxt = pass1(t + 1, nxt);
    }
    // ---- the tiles of u_{t+2} go into the buffer u_{t-1} used, once its y
    // store is done reading it (issued a step ago, it is by now)
    if (lane == 0 && t + 2 < nu && !failed) {
      bulk_wait_read_all();
      issue(t + 2);
    }
    // ---- join u_t
    const TileUnit &U = cur;
    const bool has_next = U.pos + 1 < nseg;
    const St s_in = U.cok ? load_state_in(p.state_in, U.bc, BC) : st_empty();
    St carry = s_in;
    if (U.pos > 0) {
      bool got = false;
      if (spec) {
        // the predicted records; a word that does not check yet is read
        // again until it does (its unit runs in this step or the last, and
        // publishes without waiting on this warp), within the wait bound
        const float4 *dinc = a.rec + ((int64_t)qi * nchains + U.chain) * kFwdRecWords + lane;
        const uint64_t t_start = global_ns();
        for (;;) {
          bool ok = tag_is(sx.w, t_inc) && tag_is(sy.y, t_inc);
#pragma unroll
          for (int j = 0; j < kSpecDepth; ++j) ok = ok && (j >= dspec || tag_is(sa[j].w, t_agg));
          if (__all_sync(0xffffffffu, ok)) {
            got = true;
            break;
          }
          if ((int64_t)(global_ns() - t_start) > budget || launch_aborted(p.hdr, epoch)) break;
          __nanosleep(64);
          if (!(tag_is(sx.w, t_inc) && tag_is(sy.y, t_inc))) {
            sx = ld_relaxed_v4(dinc + 32);
            sy = ld_relaxed_v4(dinc + 64);
          }
#pragma unroll
          for (int j = 0; j < kSpecDepth; ++j)
            if (j < dspec && !tag_is(sa[j].w, t_agg))
              sa[j] = ld_relaxed_v4(a.rec + ((int64_t)(qi + 1 + j) * nchains + U.chain) * kFwdRecWords + lane);
        }
        if (got) {
          St acc = St{sx.x, sx.y, sx.z, sy.x};
#pragma unroll
          for (int j = 0; j < kSpecDepth; ++j)
            if (j < dspec) acc = combine(acc, St{sa[j].x, sa[j].y, sa[j].z, 0.f}, (float)L, U.w2);
          carry = acc;
        }
      }
      if (!got)
        carry = tile_lookback(p.flags, a.rec, U.pos, U.chain, nchains, epoch, s_in, (float)L, U.w2, budget, p.hdr,
                              lane, failed);
      if (has_next && !(p.hold_first && U.pos == 0)) {
        const int64_t unit = (int64_t)g + (int64_t)t * G;
        tile_put_inc(a.rec, unit, combine(carry, agg_cur, (float)L, U.w2), t_inc, lane);
        if (lane == 0) st_relaxed_u32(p.flags + unit, t_inc);
      }
    }

    // ---- pass 2 of u_t: replay from the joined state; y overwrites k in place
    E *ks = reinterpret_cast<E *>(wbuf + (size_t)(t % NBUF) * Lay::BUF) + lane;
    const E *vs = ks + L * 32;
    const E *rs = ks + 2 * L * 32;
    const float w2 = U.w2, u2 = U.u2;
    Run st = run_from(carry);
    const TileFast fc = tile_fast<RB>(U.w, w2, u2);
#pragma unroll 1
    for (int bt = 0; bt < L / RB; ++bt) {
      const int nb = U.n - bt * RB;
      if (nb <= 0) break;
      const int64_t tb = U.t0 + bt * RB;
      if (p.ckpt && U.cok && (tb % kCkpt) == 0) store_ckpt(p.ckpt, tb / kCkpt, U.bc, BC, run_state(st), w2);
      E *kb = ks + bt * RB * 32;
      const E *vb = vs + bt * RB * 32;
      const E *rb = rs + bt * RB * 32;
      const float E0 = fmaf(st.n, w2, st.Panc);
      float kj[RB];
      float mx = -3.0e38f, mn = 3.0e38f;
#pragma unroll
      for (int j = 0; j < RB; ++j) {
        kj[j] = fmaf(-(float)j, fc.we, to_f32(kb[j * 32]));
        mx = fmaxf(mx, kj[j]);
        mn = fminf(mn, kj[j]);
      }
      const float M = fmaxf(E0, mx * kLog2e);
      const float span = M - mn * kLog2e;  // >= 0
      // Every denominator stays in the float range if every token's own
      // bonus term does (span bound), or, in the undecayed mode, if the
      // carried state's term does: it does not decay inside the batch, and
      // terms it dwarfs by more than 2^-36 may underflow harmlessly.  (In the
      // decaying mode a dominant state can itself decay out of range within
      // the batch, so only the span bound applies.)
      const bool dens_ok = span < 100.f && span - u2 - fc.sh < 60.f;
      const bool state_ok = fc.ewm == 1.f && E0 - M > -90.f;
      const bool ok = fc.ok && (dens_ok || state_ok);
      if (__all_sync(0xffffffffu, ok && nb >= RB)) {
        const float s0 = ex2(E0 - M + fc.sh);
        float al = st.a * s0, be = st.b * s0;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const float e0 = ex2(fmaf(kj[j], kLog2e, -M));
          const float V = to_f32(vb[j * 32]);
          const float eu = e0 * fc.cu;
          float yv = fmaf(eu, V, al) * rcp(be + eu);
          if constexpr (GATE) yv *= gate_sigmoid(to_f32(rb[j * 32]));
          al = fmaf(al, fc.ewm, e0 * V);
          be = fmaf(be, fc.ewm, e0);
          kb[j * 32] = from_f32<E>(yv);
        }
        st = Run{al, be, M, fc.nend};
      } else {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            float yv = fwd_token(st, to_f32(kb[j * 32]) * kLog2e, to_f32(vb[j * 32]), u2, w2);
            if constexpr (GATE) yv *= gate_sigmoid(to_f32(rb[j * 32]));
            kb[j * 32] = from_f32<E>(yv);
          }
        }
      }
    }
    if (p.state_out && U.cok && !has_next) store_state(p.state_out, U.bc, BC, run_state(st), w2);
    fence_proxy_async_smem();  // y (and this step's reads) before the async proxy reuses the buffer
    __syncwarp();
    if (p.y && lane == 0) {
      tma_store_3d(&ymap, U.x0, (int)U.t0, U.b, smem_addr(wbuf + (size_t)(t % NBUF) * Lay::BUF));
      bulk_commit();
    }
    __syncwarp();
    cur = nxt;
    agg_cur = agg_nxt;
  }
  if (lane == 0) {
    bulk_wait_all();  // every y store complete before the block exits
    for (int t = wt_t + 1; t <= iss_t; ++t)  // and every issued load landed (after a failure)
      mbar_wait(bar0 + 8u * (t % NBUF), (uint32_t)(t / NBUF) & 1u, budget, nullptr);
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

// ------------------------------------------------------------------ host ---
template <typename E, int L, int RB, bool GATE>
static cudaError_t launch_fwd_tile_t(const FwdArgs &f, float4 *rec, int dtype, int num_sms, cudaStream_t st) {
  CUtensorMap km, vm, rm, ym;
  if (!encode_btc(&km, f.k, dtype, f.B, f.T, f.C, L) || !encode_btc(&vm, f.v, dtype, f.B, f.T, f.C, L))
    return cudaErrorInvalidValue;
  rm = vm;
  ym = km;  // unused placeholders when there is no gate / no y
  if (GATE && !encode_btc(&rm, f.r, dtype, f.B, f.T, f.C, L)) return cudaErrorInvalidValue;
  if (f.y && !encode_btc(&ym, f.y, dtype, f.B, f.T, f.C, L)) return cudaErrorInvalidValue;
  constexpr int NARR = GATE ? 3 : 2;
  constexpr int smem = TileLayout<E, L, NARR>::bytes(kTileFwdWarps);
  auto kern = fwd_tile_kernel<E, L, RB, GATE>;
  int occ = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, kTileFwdWarps * 32, smem, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  TileFwdArgs a{};
  a.f = f;
  a.rec = rec;
  a.nseg = (f.T + L - 1) / L;
  const int64_t units = a.nseg * f.nchains;
  if (units >= (int64_t)1 << 31) return cudaErrorInvalidValue;  // unit indices are 31-bit
  // one resident wave (cooperative launch: every unit a look-back waits on
  // belongs to a running warp); the grid is trimmed so that every warp owns
  // the same number of units
  const int64_t max_warps = (int64_t)occ * num_sms * kTileFwdWarps;
  const int64_t rounds = (units + max_warps - 1) / max_warps;
  const int64_t grid = ((units + rounds - 1) / rounds + kTileFwdWarps - 1) / kTileFwdWarps;
  void *args[] = {&km, &vm, &rm, &ym, &a};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3(kTileFwdWarps * 32), args,
                                     (size_t)smem, st);
}

int tile_fwd_tokens(int dtype) { return dtype == 0 ? kTileLF32 : kTileLBF16; }

cudaError_t launch_forward_tile(const FwdArgs &f, float4 *rec, int dtype, int num_sms, cudaStream_t st) {
  if (f.r)
    return dtype == 0 ? launch_fwd_tile_t<float, kTileLF32, kTileRB, true>(f, rec, dtype, num_sms, st)
                      : launch_fwd_tile_t<uint16_t, kTileLBF16, kTileRB, true>(f, rec, dtype, num_sms, st);
  return dtype == 0 ? launch_fwd_tile_t<float, kTileLF32, kTileRB, false>(f, rec, dtype, num_sms, st)
                    : launch_fwd_tile_t<uint16_t, kTileLBF16, kTileRB, false>(f, rec, dtype, num_sms, st);
}

}  // namespace wkv
