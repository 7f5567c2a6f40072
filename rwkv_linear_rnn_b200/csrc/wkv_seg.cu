// wkv_seg.cu -- segment forward of libwkv (the default forward on sm_100a
// when rows are 16-byte aligned).
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), run in the RNN
// form of section "RNN-유사추론" (eq. WKV_t) over the max-rescaled state; the
// time axis is split as in section "Transformer-유사학습" (WKV done as a scan).
//
// One warp owns one segment: a chain (batch row b, 32 channels = the 32
// lanes) and TS consecutive tokens.  Warps are persistent and take segments
// in position-major order (all chains' segment 0, then segment 1, ...).
//   pass 1  stream the segment's k, v rows through the warp's TMA ring and
//           form the segment summary (one ex2 per token);
//   join    publish it, then fold, in a fixed order, the records of at most
//           32 earlier segments of the same chain: the inclusive prefix that
//           the last segment of the previous 32-segment block published, then
//           the summaries of the earlier segments of this block.  The fold
//           order depends only on the segment position, so results are
//           bit-reproducible; there are no chains of waits beyond one record
//           per block of 32 segments;
//   pass 2  stream the same rows again (they are still in L2: pass 1 loads
//           with an evict-last hint, pass 2 with evict-first) and replay the
//           recurrence from the joined state, writing y, the checkpoints at
//           every 16-token boundary, and the final state.
// Per token: pass 1 is one ex2 and ~8 FMA-pipe ops, pass 2 two ex2 + one rcp
// and ~22 ops.  HBM traffic is the algorithmic 12 B (fp32) / 6 B (bf16) per
// channel-token plus a 16-byte record per segment and lane.
#include <cuda.h>

#include <algorithm>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_ring.cuh"

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

struct SegArgs {
  FwdArgs f;
  int64_t nseg;  // segments per chain
  int ts;        // tokens per segment (a multiple of the batch rows)
  int nbt;       // batches per segment (ts / rows per batch)
};

#ifndef WKV_SEGF_BLOCK
#define WKV_SEGF_BLOCK 16
#endif
constexpr int kBlockSeg = WKV_SEGF_BLOCK;  // segments per prefix block (at most one per lane)
static_assert(kBlockSeg >= 1 && kBlockSeg <= 32, "one lane per record");

// BAR: every warp owns at most one segment and the rows fit in L2; all
// warps run pass 1, meet at one grid barrier, and fold their predecessors'
// summaries without polling.  Otherwise segments are joined through
// per-record flags (decoupled, at most kBlockSeg records per fold).
// GATE: the output is sigma(r) * wkv (the gate input r arrives with the
// second pass's rows as a third ring array).
template <typename E, int S, int RB, bool BAR, bool GATE>
__global__ void __launch_bounds__(128, 4) fwd_seg_kernel(const __grid_constant__ CUtensorMap kmap,
                                                      const __grid_constant__ CUtensorMap vmap,
                                                      const __grid_constant__ CUtensorMap rmap,
                                                      SegArgs a) {
  static_assert(kCkpt % RB == 0, "checkpoints fall on batch starts");
  const int TS = a.ts;       // tokens per segment
  const int NBT = a.nbt;     // ring items per pass
  const int IPU = 2 * NBT;   // ring items per segment
  const FwdArgs &p = a.f;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = (int)(blockDim.x >> 5);
  constexpr int NARR = GATE ? 3 : 2;
  Ring<E, S, NARR, RB> ring(smem, wl, nw);
  ring.init(lane);
  const CUtensorMap *maps[NARR];
  maps[0] = &kmap;
  maps[1] = &vmap;
  if constexpr (GATE) maps[NARR - 1] = &rmap;
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

  // Lane 0 issues ring items ahead of the consumer, in consumption order
  // (pass 1 batches, then the same batches again for pass 2), tracking the
  // item's stage and unit with running counters.
  int iss_k = 0, iss_done = 0, iss_unit = g, iss_r = 0, iss_s = 0, iss_x = 0, iss_row0 = 0;
  if (lane == 0 && !ring.aligned()) {  // cannot happen with this layout; never issue a misaligned copy
    atomicCAS(&p.hdr->status, 0, -4);
    iss_k = nitems;
  }
  auto issue_next = [&]() {
    if (iss_r == 0) {
      const int pos = iss_unit / nchains, chain = iss_unit - pos * nchains;
      const int b = chain / nct;
      iss_x = (chain - b * nct) * 32;
      iss_row0 = (int)((int64_t)b * T + (int64_t)pos * TS);
    }
    const int bt = iss_r < NBT ? iss_r : iss_r - NBT;
    // pass 1 needs k, v only; pass 2 also the gate input
    ring.issue_stage_n(maps, iss_s, iss_x, iss_row0 + bt * RB,
                       iss_r < NBT ? l2_policy_evict_last() : l2_policy_evict_first(), iss_r < NBT ? 2 : NARR);
    iss_done = ++iss_k;
    iss_s = iss_s + 1 == S ? 0 : iss_s + 1;
    if (++iss_r == IPU) {
      iss_r = 0;
      iss_unit += G;
    }
  };
  if (lane == 0)
    while (iss_k < min(S - 1, nitems)) issue_next();
  bool failed = false;
  int cs = 0;
  uint32_t cph = 0;
  // Consume the next item: K (base-2 scaled) and V of its RB rows, and
  // (gated second pass) the gate sigma(r) of each row in R.
  auto take = [&](float(&K)[RB], float(&V)[RB], float(&R)[RB], bool want_r) {
    if (!failed && !mbar_wait(ring.bar(cs), cph, budget, nullptr)) {
      failed = true;
      if (lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    }
    const E *kr = ring.stage(cs, 0) + lane;
    const E *vr = ring.stage(cs, 1) + lane;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
    }
    if constexpr (GATE) {
      if (want_r) {
        const E *rr = ring.stage(cs, NARR - 1) + lane;
#pragma unroll
        for (int j = 0; j < RB; ++j) R[j] = gate_sigmoid(to_f32(rr[j * 32]));
      }
    }
    __syncwarp();  // the stage is read; it may be refilled
    if (++cs == S) {
      cs = 0;
      cph ^= 1u;
    }
    if (lane == 0 && iss_k < nitems && !failed) {  // after a failed wait nothing new is issued
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue_next();
    }
  };

  const int iters = BAR ? 1 : nu;  // with BAR every warp passes the barrier once
  for (int i = 0; i < iters; ++i) {
    const bool has = i < nu;
    const int unit = has ? g + i * G : 0;
    const int pos = unit / nchains, chain = unit - pos * nchains;
    const int b = chain / nct;
    const int64_t c = (int64_t)(chain - b * nct) * 32 + lane;
    const bool cok = c < C;
    const int64_t t0 = (int64_t)pos * TS;
    const int n = (int)min((int64_t)TS, T - t0);
    const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
    const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
    const int64_t bc = (int64_t)b * C + c;

    // ---- pass 1: segment summary
    St agg = st_empty();
#pragma unroll 1
    for (int bt = 0; bt < (has ? NBT : 0); ++bt) {
      float K[RB], V[RB], R[RB];
      take(K, V, R, false);
      const int nb = max(0, min(RB, n - bt * RB));
      const St sb = nb == RB ? summarize_full<RB>(K, V, w2) : summarize<RB>(K, V, w2, nb);
      agg = combine(agg, sb, (float)nb, w2);
    }

    St carry;
    if constexpr (BAR) {
      // ---- join after the grid barrier: every summary is out; fold the
      // chain's earlier segments in order
      if (has && pos + 1 < nseg) rec_store_st(p.desc, unit, agg, lane);
      grid_barrier(p.hdr, gridDim.x, budget);
      if (!has) continue;
      carry = cok ? load_state_in(p.state_in, bc, BC) : st_empty();
#pragma unroll 1
      for (int j0 = 0; j0 < pos; j0 += 12) {  // twelve records in flight per step
        St rec[12];
#pragma unroll
        for (int j = 0; j < 12; ++j)
          if (j0 + j < pos) rec[j] = rec_load_st(p.desc, (int64_t)(j0 + j) * nchains + chain, lane);
#pragma unroll
        for (int j = 0; j < 12; ++j)
          if (j0 + j < pos) carry = combine(carry, rec[j], (float)TS, w2);
      }
    } else {
    // ---- join: fold the earlier records of this chain (fixed order)
    const int q = pos - pos % kBlockSeg;  // first segment of this block
    const int nrec = (pos - q) + (q > 0 ? 1 : 0);
    const int rec0 = q > 0 ? q - 1 : q;  // position of record 0
    // publish own summary now (the block's last segment publishes its
    // inclusive prefix below instead; the chain's last segment nothing)
    const bool block_end = (pos % kBlockSeg) == kBlockSeg - 1;
    const bool held = p.hold_first && pos == 0;  // test hook: never publish
    if (!block_end && pos + 1 < nseg && !held) publish_st(p.desc, p.flags, unit, agg, epoch, lane);
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
    carry = (q == 0 && cok) ? load_state_in(p.state_in, bc, BC) : st_empty();
#pragma unroll 1
    for (int j0 = 0; j0 < nrec; j0 += 8) {
      St rec[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < nrec) rec[j] = rec_load_st(p.desc, (int64_t)(rec0 + j0 + j) * nchains + chain, lane);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < nrec) {
          const int rp = rec0 + j0 + j;
          if (q > 0 && rp == q - 1)
            carry = rec[j];  // inclusive prefix of everything before this block
          else
            carry = combine(carry, rec[j], (float)TS, w2);  // summaries of full segments
        }
      }
    }
    if (block_end && pos + 1 < nseg && !held)
      publish_st(p.desc, p.flags, unit, combine(carry, agg, (float)n, w2), epoch, lane);
    }

    // ---- pass 2: replay from the carried-in state
    Run st = run_from(carry);
    const FastC fc = fast_consts<RB>(w2, u2);
#pragma unroll 1
    for (int bt = 0; bt < NBT; ++bt) {
      float K[RB], V[RB], R[RB];
      take(K, V, R, true);
      if constexpr (!GATE) {
#pragma unroll
        for (int j = 0; j < RB; ++j) R[j] = 1.f;
      }
      const int nb = max(0, min(RB, n - bt * RB));
      const int64_t tb = t0 + bt * RB;
      if (p.ckpt && cok && nb > 0 && (tb % kCkpt) == 0)
        store_ckpt(p.ckpt, tb / kCkpt, bc, BC, run_state(st), w2);
      E *yp = (p.y && cok) ? static_cast<E *>(p.y) + ((int64_t)b * T + tb) * C + c : nullptr;
      const float E0 = fmaf(st.n, w2, st.Panc);
      float kj[RB], M;
      const bool ok = fast_prep<RB>(K, E0, u2, fc.w2e, kj, M);
      if (__all_sync(0xffffffffu, nb == RB && ok)) {
        const float s0 = ex2(E0 - M);
        float al = st.a * s0, be = st.b * s0;
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const float e0 = ex2(kj[j] - M);
          const float eu = e0 * fc.cu, ek = e0 * fc.cw;
          const float yv = fmaf(eu, V[j], al) * rcp(be + eu);
          al = fmaf(al, fc.ewm, ek * V[j]);
          be = fmaf(be, fc.ewm, ek);
          if (yp) IO<E>::st(yp + (int64_t)j * C, GATE ? yv * R[j] : yv);
        }
        st = Run{al, be, M, fc.nend};
      } else if (nb == RB) {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          const float yv = fwd_token(st, K[j], V[j], u2, w2);
          if (yp) IO<E>::st(yp + (int64_t)j * C, GATE ? yv * R[j] : yv);
        }
      } else {
#pragma unroll
        for (int j = 0; j < RB; ++j) {
          if (j < nb) {
            const float yv = fwd_token(st, K[j], V[j], u2, w2);
            if (yp) IO<E>::st(yp + (int64_t)j * C, GATE ? yv * R[j] : yv);
          }
        }
      }
    }
    if (p.state_out && cok && pos == nseg - 1) store_state(p.state_out, bc, BC, run_state(st), w2);
  }
  if (failed && lane == 0)  // every issued load lands before the block exits
    for (int k = max(0, iss_done - S); k < iss_done; ++k)
      mbar_wait(ring.bar(k % S), (uint32_t)(k / S) & 1u, budget, nullptr);
  // the last block to finish advances the launch epoch (no flag is read after this)
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

template <typename E, int S, int RB, bool BAR, bool GATE>
static cudaError_t launch_seg_k(const CUtensorMap &km, const CUtensorMap &vm, const CUtensorMap &rm, SegArgs a,
                                int64_t grid, int smem, cudaStream_t st) {
  auto kern = fwd_seg_kernel<E, S, RB, BAR, GATE>;
  CUtensorMap k2 = km, v2 = vm, r2 = rm;
  void *args[] = {&k2, &v2, &r2, &a};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3(128), args, (size_t)smem, st);
}

template <typename E, int S, int RB, bool GATE>
static cudaError_t launch_seg_t(const FwdArgs &f, int dtype, int num_sms, int ts_max, cudaStream_t st) {
  CUtensorMap km, vm, rm;
  if (!encode_rows(&km, f.k, dtype, f.B * f.T, f.C, RB) || !encode_rows(&vm, f.v, dtype, f.B * f.T, f.C, RB))
    return cudaErrorInvalidValue;
  rm = vm;  // unused without the gate
  if (GATE && !encode_rows(&rm, f.r, dtype, f.B * f.T, f.C, RB)) return cudaErrorInvalidValue;
  constexpr int kWarps = 4;
  constexpr int smem = WarpRing<E, S, GATE ? 3 : 2, RB>::block_bytes(kWarps);
  // the grid is sized for the smaller occupancy of the two join variants
  int occ = 1 << 30;
  for (const void *kern : {(const void *)fwd_seg_kernel<E, S, RB, false, GATE>,
                           (const void *)fwd_seg_kernel<E, S, RB, true, GATE>}) {
    int o = 0;
    cudaError_t e = blocks_per_sm(kern, kWarps * 32, smem, &o);
    if (e != cudaSuccess) return e;
    occ = std::min(occ, o);
  }
  if (occ < 1) return cudaErrorInvalidConfiguration;
  // Segment length: as short as it takes to give every resident warp a
  // segment (more warps hide more latency), but not longer than ts_max (the
  // rows between a segment's two passes must stay in L2) nor shorter than
  // four batches (the join costs a segment a fixed amount).
  const int64_t max_warps0 = (int64_t)occ * num_sms * kWarps;
  const int64_t segs_wanted = std::max<int64_t>(1, max_warps0 / f.nchains);
  int64_t ts = (f.T + segs_wanted - 1) / segs_wanted;
  ts = (ts + RB - 1) / RB * RB;
  ts = std::max<int64_t>(4 * RB, std::min<int64_t>(ts, ts_max));
  SegArgs a{f, (f.T + ts - 1) / ts, (int)ts, (int)(ts / RB)};
  const int64_t units = a.nseg * f.nchains;
  if (units >= (int64_t)1 << 31) return cudaErrorInvalidValue;  // unit indices are 31-bit
  // One resident wave (cooperative launch: every warp a segment may wait on
  // is running); warps take segments round-robin in position-major order and
  // the grid is trimmed so that every warp gets the same number of them.
  const int64_t max_warps = (int64_t)occ * num_sms * kWarps;
  const int64_t rounds = (units + max_warps - 1) / max_warps;
  const int64_t grid = ((units + rounds - 1) / rounds + kWarps - 1) / kWarps;
  // Barrier join when every warp has one segment (all first passes run
  // together anyway) and chains have few segments (each fold reads all of
  // its predecessors); the test hook needs the flag join.
  const bool bar = rounds == 1 && a.nseg <= 32 && !f.hold_first;
  return bar ? launch_seg_k<E, S, RB, true, GATE>(km, vm, rm, a, grid, smem, st)
             : launch_seg_k<E, S, RB, false, GATE>(km, vm, rm, a, grid, smem, st);
}

// Tile parameters per element type (compile-time tunables): the longest
// segment (tokens), ring stages, rows per ring item.
#ifndef WKV_SEGF_TS_F32
#define WKV_SEGF_TS_F32 128
#endif
#ifndef WKV_SEGF_S_F32
#define WKV_SEGF_S_F32 3
#endif
#ifndef WKV_SEGF_TS_BF16
#define WKV_SEGF_TS_BF16 256
#endif
#ifndef WKV_SEGF_S_BF16
#define WKV_SEGF_S_BF16 4
#endif
#ifndef WKV_SEGF_RB
#define WKV_SEGF_RB 16
#endif

// Ring stages of the gated variant (its stages hold a third array; for bf16
// three stages measured faster than four: 224 vs 256 us on B8 T4096 C2048).
#ifndef WKV_SEGF_S_F32_GATE
#define WKV_SEGF_S_F32_GATE WKV_SEGF_S_F32
#endif
#ifndef WKV_SEGF_S_BF16_GATE
#define WKV_SEGF_S_BF16_GATE 3
#endif

cudaError_t launch_forward_seg(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st) {
  if (f.r)
    return dtype == 0 ? launch_seg_t<float, WKV_SEGF_S_F32_GATE, WKV_SEGF_RB, true>(f, dtype, num_sms,
                                                                                      WKV_SEGF_TS_F32, st)
                      : launch_seg_t<uint16_t, WKV_SEGF_S_BF16_GATE, WKV_SEGF_RB, true>(f, dtype, num_sms,
                                                                                          WKV_SEGF_TS_BF16, st);
  return dtype == 0
             ? launch_seg_t<float, WKV_SEGF_S_F32, WKV_SEGF_RB, false>(f, dtype, num_sms, WKV_SEGF_TS_F32, st)
             : launch_seg_t<uint16_t, WKV_SEGF_S_BF16, WKV_SEGF_RB, false>(f, dtype, num_sms, WKV_SEGF_TS_BF16, st);
}

}  // namespace wkv
