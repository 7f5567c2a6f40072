// wkv_clu.cu -- cluster forward of libwkv: one thread-block cluster per
// chain, segments joined through distributed shared memory.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), run in the RNN
// form of section "RNN-유사추론" over the max-rescaled state, with the time
// axis cut into segments joined by the associative combine (section
// "Transformer-유사학습": WKV done as a scan).
//
// A chain (batch row b, 32 channels = the lanes of a warp) is owned by one
// cluster of CB blocks of W warps: P = CB * W warp slots.  The chain's time
// axis is walked in rounds of P segments of TS tokens; in every round slot s
// takes segment s:
//   pass 1  stream the segment's k, v rows through the warp's TMA ring
//           (evict-last) and write its summary to this block's shared
//           memory;
//   join    one cluster barrier; slot s folds the round's carry-in state and
//           the summaries of slots 0 .. s-1 (read from the owning blocks'
//           shared memory over the cluster's distributed shared memory), in
//           slot order, so results are bit-reproducible;
//   pass 2  replay the segment from L2 (evict-first): y, checkpoints and,
//           for the round's last segment, the state carried into the next
//           round (written into every block of the cluster) and the final
//           state.
// Clusters never wait on one another: no flags, no grid barrier, no
// cooperative launch, nothing in the workspace but the status word.
#include <cooperative_groups.h>
#include <cuda.h>

#include <algorithm>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_ring.cuh"

namespace cg = cooperative_groups;

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

struct CluArgs {
  FwdArgs f;
  int ts;      // tokens per segment (a multiple of the batch rows)
  int nbt;     // batches per segment
  int cb;      // blocks per cluster
  int rounds;  // rounds per chain
};

// Shared memory of a block: warp rings (with their mbarriers), then the
// round-parity double buffers of the warps' summaries [2][W][4][32] and of
// the round carry [2][4][32].
template <typename E, int S, int RB, int W>
struct CluSmem {
  using RingL = WarpRing<E, S, 2, RB>;
  static constexpr int RING = (RingL::block_bytes(W) + 15) / 16 * 16;
  static constexpr int SUMS = RING;                    // float [2][W][128]
  static constexpr int CARRY = SUMS + 2 * W * 128 * 4;  // float [2][128]
  static constexpr int BYTES = CARRY + 2 * 128 * 4;
};

template <typename E, int S, int RB, int W>
__global__ void __launch_bounds__(W * 32, 16 / W) fwd_clu_kernel(const __grid_constant__ CUtensorMap kmap,
                                                         const __grid_constant__ CUtensorMap vmap,
                                                         CluArgs a) {
  using Sm = CluSmem<E, S, RB, W>;
  static_assert(kCkpt % RB == 0, "checkpoints fall on batch starts");
  const FwdArgs &p = a.f;
  extern __shared__ __align__(1024) unsigned char smem[];
  cg::cluster_group cluster = cg::this_cluster();
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = (int)cluster.block_rank();
  const int CB = a.cb, P = CB * W;
  const int slot = rank * W + wl;
  const int TS = a.ts, NBT = a.nbt, R = a.rounds;
  const int chain = (int)(blockIdx.x / CB);
  const int nct = (int)p.nct;
  const int b = chain / nct;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t c = (int64_t)(chain - b * nct) * 32 + lane;
  const bool cok = c < C;
  const int64_t bc = (int64_t)b * C + c;
  const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
  const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
  const int64_t budget = p.spin_limit * 1000;
  float *sums = reinterpret_cast<float *>(smem + Sm::SUMS);
  float *carry_buf = reinterpret_cast<float *>(smem + Sm::CARRY);

  Ring<E, S, 2, RB> ring(smem, wl, W);
  ring.init(lane);
  const CUtensorMap *const maps[2] = {&kmap, &vmap};
  // tokens of this slot's segment in round r (<= 0: none)
  auto seg_n = [&](int r) { return (int)min((int64_t)TS, T - ((int64_t)r * P + slot) * TS); };

  // Lane 0 issues ring items in consumption order: for every round in which
  // this slot has tokens, the NBT batches of pass 1, then the same again.
  int nitems = 0;
  for (int r = 0; r < R; ++r) nitems += seg_n(r) > 0 ? 2 * NBT : 0;
  int iss_k = 0, iss_done = 0, iss_r = 0, iss_round = 0, iss_s = 0, iss_row0 = 0;
  const int x0 = (chain - b * nct) * 32;
  if (lane == 0 && !ring.aligned()) {  // cannot happen with this layout; never issue a misaligned copy
    if (p.hdr) atomicCAS(&p.hdr->status, 0, -4);
    iss_k = nitems;
  }
  auto issue_next = [&]() {
    if (iss_r == 0) {
      while (seg_n(iss_round) <= 0) ++iss_round;  // rounds without tokens issue nothing
      iss_row0 = (int)((int64_t)b * T + ((int64_t)iss_round * P + slot) * TS);
    }
    const bool p2 = iss_r >= NBT;
    const int bt = p2 ? iss_r - NBT : iss_r;
    ring.issue_stage(maps, iss_s, x0, iss_row0 + bt * RB, p2 ? l2_policy_evict_first() : l2_policy_evict_last());
    iss_done = ++iss_k;
    iss_s = iss_s + 1 == S ? 0 : iss_s + 1;
    if (++iss_r == 2 * NBT) {
      iss_r = 0;
      ++iss_round;
    }
  };
  if (lane == 0)
    while (iss_k < min(S - 1, nitems)) issue_next();
  bool failed = false;
  int cs = 0;
  uint32_t cph = 0;
  auto take = [&](float(&K)[RB], float(&V)[RB]) {
    if (!failed && !mbar_wait(ring.bar(cs), cph, budget, nullptr)) {
      failed = true;
      if (lane == 0 && p.hdr) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    }
    const E *kr = ring.stage(cs, 0) + lane;
    const E *vr = ring.stage(cs, 1) + lane;
#pragma unroll
    for (int j = 0; j < RB; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
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

  // slot of the last segment of round r (the one that carries into r+1)
  auto last_slot = [&](int r) {
    const int64_t left = T - (int64_t)r * P * TS;
    return (int)min((int64_t)P, (left + TS - 1) / TS) - 1;
  };
  const FastC fc = fast_consts<RB>(w2, u2);
  for (int r = 0; r < R; ++r) {
    const int n = seg_n(r);
    const int64_t t0 = ((int64_t)r * P + slot) * TS;
    // ---- pass 1: segment summary
    St agg = st_empty();
#pragma unroll 1
    for (int bt = 0; bt < (n > 0 ? NBT : 0); ++bt) {
      float K[RB], V[RB];
      take(K, V);
      const int nb = max(0, min(RB, n - bt * RB));
      const St sb = nb == RB ? summarize_full<RB>(K, V, w2) : summarize<RB>(K, V, w2, nb);
      agg = combine(agg, sb, (float)nb, w2);
    }
    put_st(sums + ((r & 1) * W + wl) * 128, lane, agg);

    // ---- join: carry of the round, then the earlier slots, in slot order
    cluster.sync();
    St carry;
    if (r == 0)
      carry = cok ? load_state_in(p.state_in, bc, BC) : st_empty();
    else
      carry = get_st(carry_buf + (r & 1) * 128, lane);
    if (n > 0) {
#pragma unroll 1
      for (int j0 = 0; j0 < slot; j0 += 8) {  // eight summaries in flight per step
        St rec[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j0 + j < slot) {
            const int q = j0 + j;
            rec[j] = get_st(cluster.map_shared_rank(sums + ((r & 1) * W + (q % W)) * 128, q / W), lane);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j0 + j < slot) carry = combine(carry, rec[j], (float)TS, w2);
      }
    }

    // ---- pass 2: replay from the carried-in state
    if (n > 0) {
      Run st = run_from(carry);
#pragma unroll 1
      for (int bt = 0; bt < NBT; ++bt) {
        float K[RB], V[RB];
        take(K, V);
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
            if (yp) IO<E>::st(yp + (int64_t)j * C, yv);
          }
          st = Run{al, be, M, fc.nend};
        } else if (nb == RB) {
#pragma unroll
          for (int j = 0; j < RB; ++j) {
            const float yv = fwd_token(st, K[j], V[j], u2, w2);
            if (yp) IO<E>::st(yp + (int64_t)j * C, yv);
          }
        } else {
#pragma unroll
          for (int j = 0; j < RB; ++j) {
            if (j < nb) {
              const float yv = fwd_token(st, K[j], V[j], u2, w2);
              if (yp) IO<E>::st(yp + (int64_t)j * C, yv);
            }
          }
        }
      }
      if (slot == last_slot(r)) {
        const St fin = run_state(st);
        if (r + 1 < R) {  // the next round's carry, into every block of the cluster
          for (int q = 0; q < CB; ++q)
            put_st(cluster.map_shared_rank(carry_buf + ((r + 1) & 1) * 128, q), lane, fin);
        } else if (p.state_out && cok) {
          store_state(p.state_out, bc, BC, fin, w2);
        }
      }
    }
  }
  if (failed && lane == 0)  // every issued load lands before the block exits
    for (int k = max(0, iss_done - S); k < iss_done; ++k)
      mbar_wait(ring.bar(k % S), (uint32_t)(k / S) & 1u, budget, nullptr);
  // no block may exit while another may still read its shared memory
  cluster.sync();
}

// Tile parameters (compile-time tunables): warps per block, ring stages,
// rows per batch; the longest segment per element type.
#ifndef WKV_CLU_W
#define WKV_CLU_W 4
#endif
#ifndef WKV_CLU_TS_F32
#define WKV_CLU_TS_F32 128
#endif
#ifndef WKV_CLU_TS_BF16
#define WKV_CLU_TS_BF16 256
#endif

template <typename E, int S, int RB, int W>
static cudaError_t launch_clu_t(const FwdArgs &f, int dtype, int num_sms, int ts_max, cudaStream_t st) {
  CUtensorMap km, vm;
  if (!encode_rows(&km, f.k, dtype, f.B * f.T, f.C, RB) || !encode_rows(&vm, f.v, dtype, f.B * f.T, f.C, RB))
    return cudaErrorInvalidValue;
  using Sm = CluSmem<E, S, RB, W>;
  auto kern = fwd_clu_kernel<E, S, RB, W>;
  int occ = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, W * 32, Sm::BYTES, &occ);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  // Slots per chain: enough warps to fill the GPU once (at least one block,
  // at most eight per cluster); then rounds so that segments stay within
  // ts_max (their rows must still be in L2 for the second pass).
  const int64_t warps = (int64_t)occ * num_sms * W;
  const int cb = (int)std::max<int64_t>(1, std::min<int64_t>(8, warps / (f.nchains * W)));
  const int64_t P = (int64_t)cb * W;
  const int64_t rounds = std::max<int64_t>(1, (f.T + P * ts_max - 1) / (P * ts_max));
  int64_t ts = (f.T + P * rounds - 1) / (P * rounds);
  ts = std::max<int64_t>(RB, (ts + RB - 1) / RB * RB);
  CluArgs a{f, (int)ts, (int)(ts / RB), cb, (int)((f.T + P * ts - 1) / (P * ts))};
  if (a.rounds < 1) a.rounds = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(f.nchains * cb));
  cfg.blockDim = dim3(W * 32);
  cfg.dynamicSmemBytes = Sm::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cb;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, km, vm, a);
}

cudaError_t launch_forward_clu(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st) {
  return dtype == 0 ? launch_clu_t<float, 3, 16, WKV_CLU_W>(f, dtype, num_sms, WKV_CLU_TS_F32, st)
                    : launch_clu_t<uint16_t, 4, 16, WKV_CLU_W>(f, dtype, num_sms, WKV_CLU_TS_BF16, st);
}

}  // namespace wkv
