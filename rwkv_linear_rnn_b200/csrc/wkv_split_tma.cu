// wkv_split_tma.cu -- TMA-fed summary and replay kernels of the split
// forward (see wkv_scan3.cu for the scheme; these are the variants used when
// rows are 16-byte aligned, the TMA rule).
//
// Each warp streams its rows through a private ring of S shared-memory
// stages (16 rows x 32 columns x {k, v}) filled by 2-D TMA loads
// (cp.async.bulk.tensor, no multicast) that lane 0 issues S-1 batches ahead,
// so every warp keeps ~3 batches of loads in flight without holding them in
// registers.  Warps are persistent: warp g of G handles units g, g+G, ...
// where a unit is one chain (batch row, 32 channels) and one 64-token chunk.
#include <cuda.h>

#include <algorithm>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"
#include "wkv_split.cuh"
#include "wkv_ring.cuh"

namespace wkv {

bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C, int box_rows);

struct UnitPos {
  int64_t chunk, chain, b, c;
  int x, n;
  int64_t row0;  // b*T + first token of the chunk
};
__device__ __forceinline__ UnitPos unit_pos(const FwdArgs &p, int64_t unit, int lane) {
  UnitPos u;
  u.chunk = unit / p.nchains;
  u.chain = unit - u.chunk * p.nchains;
  u.b = u.chain / p.nct;
  const int64_t ct = u.chain - u.b * p.nct;
  u.c = ct * 32 + lane;
  u.x = (int)(ct * 32);
  const int64_t t0 = u.chunk * kS3Chunk;
  u.n = (int)min((int64_t)kS3Chunk, p.T - t0);
  u.row0 = u.b * p.T + t0;
  return u;
}

// Drives one warp over its batches: `body(item, K, V)` gets each batch of 16
// rows of k (base-2 scaled) and v as registers, in order.
template <typename E, int S, typename Body>
__device__ __forceinline__ void ring_loop(const CUtensorMap *km, const CUtensorMap *vm,
                                          const FwdArgs &p, int64_t g, int64_t G, int64_t nitems,
                                          Body body) {
  constexpr int NB = kS3Chunk / kS3Batch;
  extern __shared__ __align__(1024) unsigned char smem[];
  const int wl = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Ring<E, S> r(smem, wl, (int)(blockDim.x >> 5));
  r.init(lane);
  const CUtensorMap *const maps[2] = {km, vm};
  const int64_t budget = p.spin_limit * 1000;
  auto issue = [&](int64_t it) {
    const UnitPos u = unit_pos(p, g + (it / NB) * G, 0);
    if (!r.issue(maps, it, u.x, (int)(u.row0 + (it % NB) * kS3Batch)))
      atomicCAS(&p.hdr->status, 0, -4 /* WKV_ERR_CUDA: misaligned stage, nothing issued */);
  };
  if (lane == 0)
    for (int64_t it = 0; it < min((int64_t)S - 1, nitems); ++it) issue(it);
  bool failed = false;
  for (int64_t it = 0; it < nitems; ++it) {
    const int s = (int)(it % S);
    if (!failed && !mbar_wait(r.bar(s), (uint32_t)(it / S) & 1u, budget, nullptr)) {
      failed = true;
      if (lane == 0) atomicCAS(&p.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    }
    float K[kS3Batch], V[kS3Batch];
    const E *kr = r.stage(s, 0) + lane;
    const E *vr = r.stage(s, 1) + lane;
#pragma unroll
    for (int j = 0; j < kS3Batch; ++j) {
      K[j] = to_f32(kr[j * 32]) * kLog2e;
      V[j] = to_f32(vr[j * 32]);
    }
    __syncwarp();  // every lane has read the stage before it is refilled
    if (lane == 0 && it + S - 1 < nitems) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(it + S - 1);
    }
    body(it, K, V);
  }
  if (failed && lane == 0)  // every issued load lands before the block exits
    for (int64_t it = max((int64_t)0, nitems - S); it < nitems; ++it)
      mbar_wait(r.bar((int)(it % S)), (uint32_t)(it / S) & 1u, budget, nullptr);
}

template <typename E, int S>
__global__ void __launch_bounds__(128) fwd_sum_tma_kernel(const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap,
                                                          Scan3Args a) {
  const FwdArgs &p = a.f;
  constexpr int NB = kS3Chunk / kS3Batch;
  const int lane = threadIdx.x & 31;
  const int64_t G = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t nsum = (a.npos - 1) * p.nchains;  // the last chunk needs no summary
  const int64_t nunits = nsum > g ? (nsum - g + G - 1) / G : 0;
  St acc = st_empty();
  float w2 = 0.f;
  ring_loop<E, S>(&kmap, &vmap, p, g, G, nunits * NB,
                  [&](int64_t it, const float(&K)[kS3Batch], const float(&V)[kS3Batch]) {
                    const int bt = (int)(it % NB);
                    const UnitPos u = unit_pos(p, g + (it / NB) * G, lane);
                    if (bt == 0) {
                      acc = st_empty();
                      w2 = u.c < p.C ? __ldg(p.w + u.c) * kLog2e : 0.f;
                    }
                    const int nb = max(0, min(kS3Batch, u.n - bt * kS3Batch));
                    acc = combine(acc, summarize<kS3Batch>(K, V, w2, nb), (float)nb, w2);
                    if (bt == NB - 1) {
                      const int64_t plane = p.nchains * 32;
                      float *d = a.sums + (u.chunk * 4) * plane + u.chain * 32 + lane;
                      d[0] = acc.a;
                      d[plane] = acc.b;
                      d[2 * plane] = acc.P;
                      d[3 * plane] = acc.n;
                    }
                  });
}

// Replay.  The chunk start state comes from the prefix kernel (a.carry), or
// with `fold` set is folded here, in a fixed order, from the summaries of the
// earlier chunks of the same chain and written to a.carry (the checkpoint).
template <typename E, int S>
__global__ void __launch_bounds__(128) fwd_replay_tma_kernel(const __grid_constant__ CUtensorMap kmap,
                                                             const __grid_constant__ CUtensorMap vmap,
                                                             Scan3Args a, int fold) {
  const FwdArgs &p = a.f;
  constexpr int NB = kS3Chunk / kS3Batch;
  const int lane = threadIdx.x & 31;
  const int64_t G = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t g = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t total = a.npos * p.nchains;
  const int64_t nunits = total > g ? (total - g + G - 1) / G : 0;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  Run st{0.f, 0.f, kEmptyP, 0.f};
  float w2 = 0.f, u2 = 0.f;
  ring_loop<E, S>(&kmap, &vmap, p, g, G, nunits * NB,
                  [&](int64_t it, const float(&K)[kS3Batch], const float(&V)[kS3Batch]) {
                    const int bt = (int)(it % NB);
                    const UnitPos u = unit_pos(p, g + (it / NB) * G, lane);
                    const bool cok = u.c < C;
                    if (bt == 0) {
                      w2 = cok ? __ldg(p.w + u.c) * kLog2e : 0.f;
                      u2 = cok ? __ldg(p.u + u.c) * kLog2e : 0.f;
                      St start = st_empty();
                      if (fold) {
                        start = cok ? load_state_in(p.state_in, u.b * C + u.c, BC) : st_empty();
                        const int64_t plane = p.nchains * 32;
                        for (int64_t j = 0; j < u.chunk; ++j) {
                          const float *d = a.sums + (j * 4) * plane + u.chain * 32 + lane;
                          start = combine(start, St{d[0], d[plane], d[2 * plane], d[3 * plane]},
                                          (float)min((int64_t)kS3Chunk, T - j * kS3Chunk), w2);
                        }
                        if (cok) store_ckpt(a.carry, u.chunk, u.b * C + u.c, BC, start, w2);
                      } else if (cok) {
                        const float *ck = a.carry + u.chunk * 3 * BC + u.b * C + u.c;
                        start = St{ck[0], ck[BC], ck[2 * BC], 0.f};
                      }
                      st = run_from(start);
                    }
                    const int nb = max(0, min(kS3Batch, u.n - bt * kS3Batch));
                    const int64_t tb = u.chunk * kS3Chunk + bt * kS3Batch;
                    E *yp = (p.y && cok) ? static_cast<E *>(p.y) + (u.b * T + tb) * C + u.c : nullptr;
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
                    if (bt == NB - 1 && p.state_out && cok && u.chunk == a.npos - 1)
                      store_state(p.state_out, u.b * C + u.c, BC, run_state(st), w2);
                  });
}

constexpr int kRingS = 4;         // stages per warp
constexpr int64_t kFoldMax = 64;  // chains of up to this many chunks fold in the replay

template <typename E>
static cudaError_t launch_t(const Scan3Args &a, int dtype, int num_sms, cudaStream_t st) {
  CUtensorMap km, vm;
  if (!encode_rows(&km, a.f.k, dtype, a.f.B * a.f.T, a.f.C, kS3Batch) ||
      !encode_rows(&vm, a.f.v, dtype, a.f.B * a.f.T, a.f.C, kS3Batch))
    return cudaErrorInvalidValue;
  constexpr int kWarps = 4;
  constexpr int smem = WarpRing<E, kRingS>::block_bytes(kWarps);
  auto ksum = fwd_sum_tma_kernel<E, kRingS>;
  auto krep = fwd_replay_tma_kernel<E, kRingS>;
  cudaError_t e = cudaFuncSetAttribute(ksum, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(krep, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int occ_s = 0, occ_r = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_s, ksum, kWarps * 32, smem);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_r, krep, kWarps * 32, smem);
  occ_s = std::max(occ_s, 1);
  occ_r = std::max(occ_r, 1);
  const int64_t nsum = (a.npos - 1) * a.f.nchains;
  if (nsum > 0) {
    const int64_t grid = std::min<int64_t>((nsum + kWarps - 1) / kWarps, (int64_t)occ_s * num_sms);
    ksum<<<(unsigned)grid, kWarps * 32, smem, st>>>(km, vm, a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  const int fold = a.npos <= kFoldMax ? 1 : 0;
  if (!fold && (e = launch_fwd_prefix(a, st)) != cudaSuccess) return e;
  const int64_t units = a.npos * a.f.nchains;
  const int64_t grid = std::min<int64_t>((units + kWarps - 1) / kWarps, (int64_t)occ_r * num_sms);
  krep<<<(unsigned)grid, kWarps * 32, smem, st>>>(km, vm, a, fold);
  return cudaGetLastError();
}

cudaError_t launch_scan3_tma(const Scan3Args &a, int dtype, int num_sms, cudaStream_t st) {
  return dtype == 0 ? launch_t<float>(a, dtype, num_sms, st) : launch_t<uint16_t>(a, dtype, num_sms, st);
}

}  // namespace wkv
