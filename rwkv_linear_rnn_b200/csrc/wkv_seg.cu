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
//           every 64-token boundary, and the final state.
// Per token: pass 1 is one ex2 and ~8 FMA-pipe ops, pass 2 two ex2 + one rcp
// and ~22 ops.  HBM traffic is the algorithmic 12 B (fp32) / 6 B (bf16) per
// channel-token plus a 16-byte record per segment and lane.
#include <cuda.h>

#include <algorithm>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_ring.cuh"
#include "wkv_split.cuh"

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

struct SegArgs {
  FwdArgs f;
  int64_t nseg;  // segments per chain
};

constexpr int kBlockSeg = 32;  // segments per prefix block (one lane each)

// Geometry of a segment (computed once per segment).
struct Seg {
  int64_t pos, chain, b;
  int x;         // first channel of the chain (TMA column)
  int64_t row0;  // b*T + first token (TMA row)
};
__device__ __forceinline__ Seg seg_of(const FwdArgs &p, int64_t unit, int TS) {
  Seg s;
  s.pos = unit / p.nchains;
  s.chain = unit - s.pos * p.nchains;
  s.b = s.chain / p.nct;
  s.x = (int)((s.chain - s.b * p.nct) * 32);
  s.row0 = s.b * p.T + s.pos * TS;
  return s;
}

template <typename E, int TS, int S>
__global__ void __launch_bounds__(128) fwd_seg_kernel(const __grid_constant__ CUtensorMap kmap,
                                                      const __grid_constant__ CUtensorMap vmap,
                                                      SegArgs a) {
  constexpr int NBT = TS / kS3Batch;  // batches per pass
  constexpr int IPU = 2 * NBT;        // ring items per segment
  static_assert(TS % kCkpt == 0, "segments start on checkpoints");
  const FwdArgs &p = a.f;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ring<E, S> ring(smem, wl, (int)(blockDim.x >> 5));
  ring.init(lane);
  const CUtensorMap *const maps[2] = {&kmap, &vmap};
  const int64_t G = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + wl;
  const int64_t total = a.nseg * p.nchains;
  const int64_t nu = total > g ? (total - g + G - 1) / G : 0;
  const int64_t nitems = nu * IPU;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t budget = p.spin_limit * 1000;
  unsigned epoch = 0;
  if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
  epoch = __shfl_sync(0xffffffffu, epoch, 0);
  const unsigned want = (epoch_tag(epoch) << 2) | kAgg;

  // Lane 0 issues ring items ahead of the consumer; the geometry of the
  // segment being prefetched is cached so it is computed once per segment.
  int64_t pf_i = -1;
  Seg pf{};
  uint64_t pol_keep = 0, pol_drop = 0;
  if (lane == 0) {
    pol_keep = l2_policy_evict_last();
    pol_drop = l2_policy_evict_first();
  }
  auto issue = [&](int64_t k) {
    const int64_t i = k / IPU;
    const int r = (int)(k % IPU);
    if (i != pf_i) {
      pf_i = i;
      pf = seg_of(p, g + i * G, TS);
    }
    const int y = (int)(pf.row0 + (r % NBT) * kS3Batch);
    const bool ok = ring.issue_hint(maps, k, pf.x, y, r < NBT ? pol_keep : pol_drop);
    if (!ok) atomicCAS(&p.hdr->status, 0, -4 /* misaligned stage: nothing issued */);
  };
  if (lane == 0)
    for (int64_t k = 0; k < min((int64_t)S - 1, nitems); ++k) issue(k);
  bool failed = false;
  // Consume item k: K (base-2 scaled) and V of its 16 rows.
  auto take = [&](int64_t k, float(&K)[kS3Batch], float(&V)[kS3Batch]) {
    const int s = (int)(k % S);
    if (!failed && !mbar_wait(ring.bar(s), (uint32_t)(k / S) & 1u, budget, nullptr)) {
      failed = true;
      if (lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    }
    const E *kr = ring.stage(s, 0) + lane;
    const E *vr = ring.stage(s, 1) + lane;
#pragma unroll
    for (int j = 0; j < kS3Batch; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
    }
    __syncwarp();  // the stage is read; it may be refilled
    if (lane == 0 && k + S - 1 < nitems) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(k + S - 1);
    }
  };

  for (int64_t i = 0; i < nu; ++i) {
    const Seg sg = seg_of(p, g + i * G, TS);
    const int64_t c = sg.x + lane;
    const bool cok = c < C;
    const int64_t t0 = sg.pos * TS;
    const int n = (int)min((int64_t)TS, T - t0);
    const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
    const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
    const int64_t base_item = i * IPU;

    // ---- pass 1: segment summary
    St agg = st_empty();
    for (int bt = 0; bt < NBT; ++bt) {
      float K[kS3Batch], V[kS3Batch];
      take(base_item + bt, K, V);
      const int nb = max(0, min(kS3Batch, n - bt * kS3Batch));
      agg = combine(agg, summarize<kS3Batch>(K, V, w2, nb), (float)nb, w2);
    }

    // ---- join: fold the earlier records of this chain (fixed order)
    const int64_t q = sg.pos - sg.pos % kBlockSeg;  // first segment of this block
    const int nrec = (int)(sg.pos - q) + (q > 0 ? 1 : 0);
    const int64_t rec0 = q > 0 ? q - 1 : q;  // position of record 0
    // publish own summary now (the block's last segment publishes its
    // inclusive prefix below instead; the chain's last segment nothing)
    const bool block_end = (sg.pos % kBlockSeg) == kBlockSeg - 1;
    const int64_t unit = sg.pos * p.nchains + sg.chain;
    const bool held = p.hold_first && sg.pos == 0;  // test hook: never publish
    if (!block_end && sg.pos + 1 < a.nseg && !held) publish(p.desc, p.flags, unit, 0, agg, epoch, lane);
    {
      const bool act = lane < nrec;
      const unsigned *fl = p.flags + (rec0 + lane) * p.nchains + sg.chain;
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
    St carry = (q == 0 && cok) ? load_state_in(p.state_in, sg.b * C + c, BC) : st_empty();
    for (int j0 = 0; j0 < nrec; j0 += 8) {
      St rec[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j0 + j < nrec) rec[j] = desc_load<St>(p.desc, (rec0 + j0 + j) * p.nchains + sg.chain, 0, lane);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j0 + j < nrec) {
          const int64_t rp = rec0 + j0 + j;
          if (q > 0 && rp == q - 1)
            carry = rec[j];  // inclusive prefix of everything before this block
          else
            carry = combine(carry, rec[j], (float)TS, w2);  // summaries of full segments
        }
      }
    }
    if (block_end && sg.pos + 1 < a.nseg && !held)
      publish(p.desc, p.flags, unit, 0, combine(carry, agg, (float)n, w2), epoch, lane);

    // ---- pass 2: replay from the carried-in state
    Run st = run_from(carry);
    for (int bt = 0; bt < NBT; ++bt) {
      float K[kS3Batch], V[kS3Batch];
      take(base_item + NBT + bt, K, V);
      const int nb = max(0, min(kS3Batch, n - bt * kS3Batch));
      const int64_t tb = t0 + bt * kS3Batch;
      if (p.ckpt && cok && nb > 0 && (tb % kCkpt) == 0)
        store_ckpt(p.ckpt, tb / kCkpt, sg.b * C + c, BC, run_state(st), w2);
      E *yp = (p.y && cok) ? static_cast<E *>(p.y) + (sg.b * T + tb) * C + c : nullptr;
      if (nb == kS3Batch) {
#pragma unroll
        for (int j = 0; j < kS3Batch; ++j) {
          const float yv = fwd_token(st, K[j], V[j], u2, w2);
          if (yp) IO<E>::st(yp + (int64_t)j * C, yv);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kS3Batch; ++j) {
          if (j < nb) {
            const float yv = fwd_token(st, K[j], V[j], u2, w2);
            if (yp) IO<E>::st(yp + (int64_t)j * C, yv);
          }
        }
      }
    }
    if (p.state_out && cok && sg.pos == a.nseg - 1)
      store_state(p.state_out, sg.b * C + c, BC, run_state(st), w2);
  }
  if (failed && lane == 0)  // every issued load lands before the block exits
    for (int64_t k = max((int64_t)0, nitems - S); k < nitems; ++k)
      mbar_wait(ring.bar((int)(k % S)), (uint32_t)(k / S) & 1u, budget, nullptr);
  // the last block to finish advances the launch epoch (no flag is read after this)
  __syncthreads();
  finish_block(p.hdr, gridDim.x);
}

constexpr int kSegRing = 4;

template <typename E, int TS>
static cudaError_t launch_seg_t(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st) {
  CUtensorMap km, vm;
  if (!encode_rows(&km, f.k, dtype, f.B * f.T, f.C, kS3Batch) ||
      !encode_rows(&vm, f.v, dtype, f.B * f.T, f.C, kS3Batch))
    return cudaErrorInvalidValue;
  constexpr int kWarps = 4;
  constexpr int smem = WarpRing<E, kSegRing>::block_bytes(kWarps);
  auto kern = fwd_seg_kernel<E, TS, kSegRing>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kWarps * 32, smem)) != cudaSuccess)
    return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  SegArgs a{f, (f.T + TS - 1) / TS};
  const int64_t units = a.nseg * f.nchains;
  // one resident wave (cooperative launch: every warp a segment may wait on
  // is running), warps take segments round-robin in position-major order
  const int64_t grid = std::min<int64_t>((units + kWarps - 1) / kWarps, (int64_t)occ * num_sms);
  void *args[] = {&km, &vm, &a};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3(kWarps * 32),
                                     args, (size_t)smem, st);
}

int64_t seg_tokens(int dtype) { return dtype == 0 ? 128 : 256; }

cudaError_t launch_forward_seg(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st) {
  return dtype == 0 ? launch_seg_t<float, 128>(f, dtype, num_sms, st)
                    : launch_seg_t<uint16_t, 256>(f, dtype, num_sms, st);
}

}  // namespace wkv
