// wkv_forward.cu -- forward kernels of libwkv.
//
// The operator is eq. wkv_t of the RWKV paper review ("[논문 리뷰] Reinvention
// RNNs for the Transformer Era: RWKV", section "WKV 연산자"), evaluated in the
// RNN form of section "RNN-유사추론" (eq. WKV_t) over the max-rescaled state.
// The review's "Transformer-유사학습" section runs WKV as a scan over time;
// the two kernels here are the two ways of running that scan:
//
//   fwd_seq_kernel      one thread per (b, c) chain walks all of T.  Used when
//                       there are enough chains to fill the GPU.
//   fwd_chunked_kernel  one block per (b, 32-channel tile, 128-token chunk).
//                       Each warp summarises a 16-token segment, the block
//                       joins its segments, and chunks are joined along T by
//                       a single-pass scan over published per-chunk
//                       summaries (a Fenwick tree, so the result does not
//                       depend on block timing); then every warp replays its
//                       segment from the carried-in state.  k and v are read
//                       from HBM once and stay in registers between passes.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include <mutex>

#include "wkv_internal.cuh"
#include "wkv_math.cuh"

namespace wkv {

// ------------------------------------------------------------------------
// Sequential scan: one thread per (b, c).  Consecutive threads take
// consecutive channels, so every load/store instruction of a warp touches
// one contiguous 128-byte (fp32) row segment.  k, v are prefetched U tokens
// ahead.
// ------------------------------------------------------------------------
template <typename E, int U>
__global__ void __launch_bounds__(256) fwd_seq_kernel(FwdArgs p) {
  static_assert(kCkpt % U == 0, "checkpoint interval must be a multiple of U");
  const int64_t BC = p.B * p.C;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BC) return;
  const int64_t b = idx / p.C, c = idx - b * p.C;
  const float w2 = p.w[c] * kLog2e, u2 = p.u[c] * kLog2e;
  const int64_t T = p.T, C = p.C;
  const E *kp = static_cast<const E *>(p.k) + b * T * C + c;
  const E *vp = static_cast<const E *>(p.v) + b * T * C + c;
  E *yp = p.y ? static_cast<E *>(p.y) + b * T * C + c : nullptr;
  Run s = run_from(load_state_in(p.state_in, idx, BC));

  float Kc[U], Vc[U], Kn[U], Vn[U];
  if (T > 0) {
    const int n0 = (int)min((int64_t)U, T);
    load_rows<E, U>(kp, C, n0, Kc);
    load_rows<E, U>(vp, C, n0, Vc);
  }
  for (int64_t t0 = 0; t0 < T; t0 += U) {
    // prefetch the next U rows (clamped to the last row; ignored past T)
    if (t0 + U < T) {
      const int n1 = (int)min((int64_t)U, T - t0 - U);
      load_rows<E, U>(kp + (t0 + U) * C, C, n1, Kn);
      load_rows<E, U>(vp + (t0 + U) * C, C, n1, Vn);
    }
    if (p.ckpt && (t0 % kCkpt) == 0) store_ckpt(p.ckpt, t0 / kCkpt, idx, BC, run_state(s), w2);
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (t0 + j < T) {
        const float y = fwd_token(s, Kc[j] * kLog2e, Vc[j], u2, w2);
        if (yp) IO<E>::st(yp + (t0 + j) * C, y);
      }
    }
    if (s.n > 1048576.f) {  // keep n exact as a float: re-anchor (one rounding)
      s.Panc = fmaf(s.n, w2, s.Panc);
      s.n = 0.f;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      Kc[j] = Kn[j];
      Vc[j] = Vn[j];
    }
  }
  if (p.state_out) store_state(p.state_out, idx, BC, run_state(s), w2);
}

// ------------------------------------------------------------------------
// Chunked scan.  Block = W warps; warp `wi` owns tokens [t0, t0 + L) of the
// block's chunk for the 32 channels of its tile (lane = channel).
// ------------------------------------------------------------------------

template <typename E, int W, int L>
__global__ void __launch_bounds__(W * 32) fwd_chunked_kernel(FwdArgs p) {
  constexpr int TC = W * L;
  static_assert(TC % kCkpt == 0 && kCkpt % L == 0, "chunk/ckpt geometry");
  __shared__ unsigned s_tile, s_epoch;
  __shared__ float s_agg[W][128];  // warp segment summaries (St planes)
  __shared__ float s_pre[W][128];  // block-local exclusive prefix of each warp
  __shared__ float s_carry[128];   // state at the start of the block's chunk

  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  take_ticket(p.hdr, &s_tile, &s_epoch);
  __syncthreads();
  const int64_t tile = s_tile;
  const unsigned epoch = s_epoch;
  if (tile >= p.nchains * p.nchunks) {  // stale ticket counter: touch nothing
    if (threadIdx.x == 0) atomicCAS(&p.hdr->status, 0, -4 /* WKV_ERR_CUDA */);
    finish_block(p.hdr, gridDim.x);
    return;
  }
  const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
  const int64_t b = chain / p.nct;
  const int64_t c = (chain - b * p.nct) * 32 + lane;
  const bool cok = c < p.C;
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  const int64_t tc0 = chunk * TC;                 // first token of the chunk
  const int64_t t0 = tc0 + (int64_t)wi * L;       // first token of this warp
  const int nvalid = (int)max((int64_t)0, min((int64_t)L, T - t0));
  const int chunk_len = (int)min((int64_t)TC, T - tc0);
  const float w2 = cok ? p.w[c] * kLog2e : 0.f;
  const float u2 = cok ? p.u[c] * kLog2e : 0.f;

  float K[L], V[L];
  if (nvalid > 0) {  // warp-uniform
    const int64_t off = (b * T + t0) * C + (cok ? c : C - 1);
    load_rows<E, L>(static_cast<const E *>(p.k) + off, C, nvalid, K);
    load_rows<E, L>(static_cast<const E *>(p.v) + off, C, nvalid, V);
#pragma unroll
    for (int j = 0; j < L; ++j) {
      const bool ok = cok && j < nvalid;
      K[j] = ok ? K[j] * kLog2e : 0.f;
      V[j] = ok ? V[j] : 0.f;
    }
  } else {
#pragma unroll
    for (int j = 0; j < L; ++j) K[j] = V[j] = 0.f;
  }

  // Pass 1: segment summary.
  {
    const St s = summarize<L>(K, V, w2, nvalid);
    put_st(s_agg[wi], lane, s);
  }
  __syncthreads();

  // Warp 0: block-local prefixes, then the chunk scan along T.
  if (wi == 0) {
    St acc = st_empty();
#pragma unroll
    for (int i = 0; i < W; ++i) {
      put_st(s_pre[i], lane, acc);
      const St si = get_st(s_agg[i], lane);
      const int li = (int)max((int64_t)0, min((int64_t)L, T - (tc0 + (int64_t)i * L)));
      acc = combine(acc, si, (float)li, w2);
    }
    const St initial = cok ? load_state_in(p.state_in, b * C + c, BC) : st_empty();
    const St excl = chunk_scan(p.flags, p.desc, chunk, chain, p.nchains, acc, (float)chunk_len,
                               (float)TC, initial, st_empty(), epoch, p.hdr, p.spin_limit,
                               chunk + 1 < p.nchunks, !(p.hold_first && chunk == 0), w2, lane);
    put_st(s_carry, lane, excl);
  }
  __syncthreads();
  finish_block(p.hdr, gridDim.x);

  // Pass 2: replay the segment from the carried-in state.
  if (nvalid > 0) {
    const St cin = get_st(s_carry, lane);
    const St pre = get_st(s_pre[wi], lane);
    const St start = combine(cin, pre, (float)min(wi * L, chunk_len), w2);
    if (p.ckpt && cok && (t0 % kCkpt) == 0) store_ckpt(p.ckpt, t0 / kCkpt, b * C + c, BC, start, w2);
    Run s = run_from(start);
    E *yp = p.y ? static_cast<E *>(p.y) + (b * T + t0) * C + c : nullptr;
#pragma unroll
    for (int j = 0; j < L; ++j) {
      if (j < nvalid) {
        const float y = fwd_token(s, K[j], V[j], u2, w2);
        if (yp && cok) IO<E>::st(yp + (int64_t)j * C, y);
      }
    }
    if (p.state_out && cok && t0 + nvalid == T) store_state(p.state_out, b * C + c, BC, run_state(s), w2);
  }
}

// ------------------------------------------------------------------------
// TMA-fed persistent chunked scan (the default forward on sm_100a).
//
// Block = W compute warps + 1 scan warp + 1 producer warp; grid = one
// resident wave (cooperative launch), block g owns tiles g, g+G, g+2G, ...
// of the (position-major) tile order.  A tile is 32 channels x TC = W*L
// tokens of one batch row.
//   producer  lane 0 streams the k and v tiles into an S-stage shared ring
//             with 2-D TMA loads that complete on mbarriers.
//   compute   warp w owns rows [w*L, (w+1)*L) of every tile.  Iteration i:
//             pass 1 (segment summary) of tile i, then pass 2 (replay, y) of
//             tile i-1 from the carried-in state the scan warp prepared.
//   scan      joins tile i's W summaries, runs the cross-block chunk scan
//             (Fenwick nodes, deterministic) and writes each warp's
//             starting state.  Running one tile behind the compute warps
//             keeps its global-memory round trips off their critical path.
// k and v are read from HBM once; pass 2 re-reads them from shared memory.
// ------------------------------------------------------------------------
template <typename E, int W, int L, int S>
struct TmaFwdLayout {
  static constexpr int TC = W * L;
  static constexpr int ROWB = 32 * (int)sizeof(E);
  static constexpr int TILEB = TC * ROWB;                 // one array, one tile
  static constexpr int STAGE_OFF = 0;                     // [S][2][TC][32] E
  static constexpr int SUMS_OFF = S * 2 * TILEB;          // [2][W][4][32] f32
  static constexpr int CARRY_OFF = SUMS_OFF + 2 * W * 128 * 4;
  static constexpr int BAR_OFF = CARRY_OFF + 2 * W * 128 * 4;  // full[S] empty[S] sfull[2] cfull[2]
  static constexpr int FLAG_OFF = BAR_OFF + (2 * S + 4) * 8;  // abort flag
  static constexpr int BYTES = FLAG_OFF + 16;
};

template <typename E, int W, int L, int S>
__global__ void __launch_bounds__((W + 2) * 32) fwd_tma_kernel(const __grid_constant__ CUtensorMap kmap,
                                                               const __grid_constant__ CUtensorMap vmap,
                                                               FwdArgs p) {
  using Lay = TmaFwdLayout<E, W, L, S>;
  constexpr int TC = Lay::TC;
  extern __shared__ __align__(1024) unsigned char smem[];
  int &s_abort = *reinterpret_cast<int *>(smem + Lay::FLAG_OFF);
  const int wi = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ntiles = p.nchains * p.nchunks;
  const int64_t G = gridDim.x;
  const int64_t n = (ntiles - (int64_t)blockIdx.x + G - 1) / G;  // this block's tiles
  const uint32_t bar0 = smem_addr(smem + Lay::BAR_OFF);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };
  auto sfull = [&](int b) { return bar0 + 8u * (2 * S + b); };
  auto cfull = [&](int b) { return bar0 + 8u * (2 * S + 2 + b); };
  const int64_t T = p.T, C = p.C, BC = p.B * p.C;
  auto stage_ptr = [&](int s, int arr) {
    return reinterpret_cast<const E *>(smem + Lay::STAGE_OFF + (size_t)(s * 2 + arr) * Lay::TILEB);
  };
  float *sums = reinterpret_cast<float *>(smem + Lay::SUMS_OFF);
  float *carry = reinterpret_cast<float *>(smem + Lay::CARRY_OFF);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), W);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull(b), W);
      mbar_init(cfull(b), 1);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  volatile int *abort = &s_abort;
  const int64_t lim = p.spin_limit * 1000;  // wait budget in ns (default ~1 s)

  if (wi == W + 1) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t i = 0; i < n; ++i) {
        const int s = (int)(i % S);
        if (i >= S && !mbar_wait(empty(s), (uint32_t)((i / S) - 1) & 1u, lim, abort)) break;
        if (*abort) break;
        const int64_t tile = (int64_t)blockIdx.x + i * G;
        const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
        const int64_t b = chain / p.nct;
        const int x = (int)((chain - b * p.nct) * 32);
        const int y = (int)(b * T + chunk * TC);
        mbar_expect_tx(full(s), 2u * Lay::TILEB);
        tma_load_2d(smem_addr(stage_ptr(s, 0)), &kmap, x, y, full(s));
        tma_load_2d(smem_addr(stage_ptr(s, 1)), &vmap, x, y, full(s));
        issued = i + 1;
      }
      if (*abort) {
        // Let every load this block issued land before the block can exit.
        for (int64_t i = (issued > S ? issued - S : 0); i < issued; ++i)
          mbar_wait(full((int)(i % S)), (uint32_t)(i / S) & 1u, lim, nullptr);
      }
    }
  } else if (wi == W) {
    // -------------------------------------------------------------- scan
    unsigned epoch = 0;
    if (lane == 0) epoch = ld_relaxed(&p.hdr->epoch);
    epoch = __shfl_sync(0xffffffffu, epoch, 0);
    for (int64_t i = 0; i < n; ++i) {
      const int buf = (int)(i & 1);
      if (!mbar_wait(sfull(buf), (uint32_t)(i >> 1) & 1u, lim, abort)) {
        if (lane == 0) {
          *abort = 1;
          raise_timeout(p.hdr, epoch);
        }
        break;
      }
      const int64_t tile = (int64_t)blockIdx.x + i * G;
      const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
      const int64_t b = chain / p.nct;
      const int64_t c = (chain - b * p.nct) * 32 + lane;
      const bool cok = c < C;
      const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
      const int chunk_len = (int)min((int64_t)TC, T - chunk * TC);
      // local prefixes of the W segments (block-local, from the empty state)
      St pre[W];
      St acc = st_empty();
      const float *sb = sums + buf * W * 128;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        pre[w] = acc;
        const St si = get_st(sb + w * 128, lane);
        const int lw = (int)max((int64_t)0, min((int64_t)L, T - (chunk * TC + (int64_t)w * L)));
        acc = combine(acc, si, (float)lw, w2);
      }
      const St initial = cok ? load_state_in(p.state_in, b * C + c, BC) : st_empty();
      const St excl = chunk_scan(p.flags, p.desc, chunk, chain, p.nchains, acc, (float)chunk_len,
                                 (float)TC, initial, st_empty(), epoch, p.hdr, p.spin_limit,
                                 chunk + 1 < p.nchunks, !(p.hold_first && chunk == 0), w2, lane);
      float *cb = carry + buf * W * 128;
#pragma unroll
      for (int w = 0; w < W; ++w) {
        const St st = combine(excl, pre[w], (float)min(w * L, chunk_len), w2);
        put_st(cb + w * 128, lane, st);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(cfull(buf));
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence();
      const unsigned prev = atomicAdd(&p.hdr->done, 1u);
      if (prev == gridDim.x - 1u) {
        p.hdr->ticket = 0u;
        p.hdr->done = 0u;
        __threadfence();
        atomicAdd(&p.hdr->epoch, 1u);
      }
    }
  } else {
    // ----------------------------------------------------------- compute
    const int w = wi;
    for (int64_t i = 0; i <= n; ++i) {
      if (i < n) {
        const int s = (int)(i % S);
        if (!mbar_wait(full(s), (uint32_t)(i / S) & 1u, lim, abort)) {
          *abort = 1;
          break;
        }
        const int64_t tile = (int64_t)blockIdx.x + i * G;
        const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
        const int64_t b = chain / p.nct;
        const int64_t c = (chain - b * p.nct) * 32 + lane;
        const bool cok = c < C;
        const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
        const int nvalid = (int)max((int64_t)0, min((int64_t)L, T - (chunk * TC + (int64_t)w * L)));
        const E *kr = stage_ptr(s, 0) + (size_t)w * L * 32 + lane;
        const E *vr = stage_ptr(s, 1) + (size_t)w * L * 32 + lane;
        float K[L], V[L];
#pragma unroll
        for (int j = 0; j < L; ++j) {
          K[j] = to_f32(kr[j * 32]) * kLog2e;
          V[j] = to_f32(vr[j * 32]);
        }
        const St sm = summarize<L>(K, V, w2, nvalid);
        put_st(sums + (i & 1) * W * 128 + w * 128, lane, sm);
        __syncwarp();
        if (lane == 0) mbar_arrive(sfull((int)(i & 1)));
      }
      if (i >= 1) {
        const int64_t j = i - 1;
        const int s = (int)(j % S);
        if (!mbar_wait(cfull((int)(j & 1)), (uint32_t)(j >> 1) & 1u, lim, abort)) {
          *abort = 1;
          break;
        }
        const int64_t tile = (int64_t)blockIdx.x + j * G;
        const int64_t chunk = tile / p.nchains, chain = tile - chunk * p.nchains;
        const int64_t b = chain / p.nct;
        const int64_t c = (chain - b * p.nct) * 32 + lane;
        const bool cok = c < C;
        const float w2 = cok ? __ldg(p.w + c) * kLog2e : 0.f;
        const float u2 = cok ? __ldg(p.u + c) * kLog2e : 0.f;
        const int64_t t0 = chunk * TC + (int64_t)w * L;
        const int nvalid = (int)max((int64_t)0, min((int64_t)L, T - t0));
        const St start = get_st(carry + (j & 1) * W * 128 + w * 128, lane);
        if (nvalid > 0) {
          if (p.ckpt && cok && (t0 % kCkpt) == 0) store_ckpt(p.ckpt, t0 / kCkpt, b * C + c, BC, start, w2);
          const E *kr = stage_ptr(s, 0) + (size_t)w * L * 32 + lane;
          const E *vr = stage_ptr(s, 1) + (size_t)w * L * 32 + lane;
          Run st = run_from(start);
          E *yp = p.y ? static_cast<E *>(p.y) + (b * T + t0) * C + c : nullptr;
#pragma unroll
          for (int q = 0; q < L; ++q) {
            if (q < nvalid) {
              const float yv = fwd_token(st, to_f32(kr[q * 32]) * kLog2e, to_f32(vr[q * 32]), u2, w2);
              if (yp && cok) IO<E>::st(yp + (int64_t)q * C, yv);
            }
          }
          if (p.state_out && cok && t0 + nvalid == T)
            store_state(p.state_out, b * C + c, BC, run_state(st), w2);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(s));
      }
    }
  }
}

// ---------------------------------------------------------------- launch ---
constexpr int kSeqU = 8;
constexpr int kFwdW = 4, kFwdL = 16;            // register-tile fallback kernel
constexpr int kTmaW = 4, kTmaL = 16, kTmaS = 4;  // TMA kernel
static_assert(kFwdW * kFwdL == kTmaW * kTmaL, "both chunked kernels use one chunk length");

int64_t fwd_chunk_tokens() { return kFwdW * kFwdL; }

// A driver entry point, looked up through the runtime (null if missing).
static void *driver_entry(const char *name) {
  void *f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return f;
}

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  // looked up once (thread-safe static initialisation)
  static const auto fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(driver_entry("cuTensorMapEncodeTiled"));
  return fn;
}

// The tensor-map encoder is a driver-API call and needs a context current in
// the calling thread.  A thread whose only CUDA use so far is this library
// (an autograd worker, say) may have none: the runtime binds the device's
// primary context on its first runtime call that needs one, and a thread
// that never made such a call has none.  Bind it then; a context the caller
// made current is left alone.
static bool ensure_context() {
  static const auto get = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(driver_entry("cuCtxGetCurrent"));
  CUcontext ctx = nullptr;
  if (get && get(&ctx) == CUDA_SUCCESS && ctx) return true;
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess;
}

// Encoded tensor maps, remembered by their arguments.  A map is a pure
// function of (rank, address, element type, extents, box): the same key
// always encodes to the same 128 bytes, whichever context or thread asks, so
// a hit is returned as is and a training loop that calls with the same
// buffers pays for each encoding once.  A small table with round-robin
// replacement; the lock is held only for the lookup or the insertion.
namespace {
struct MapKey {
  const void *ptr;
  int64_t d0, d1, d2;
  int dtype, rank, box;
  bool operator==(const MapKey &o) const {
    return ptr == o.ptr && d0 == o.d0 && d1 == o.d1 && d2 == o.d2 && dtype == o.dtype && rank == o.rank &&
           box == o.box;
  }
};
constexpr int kMapSlots = 64;
struct MapCache {
  std::mutex mu;
  MapKey key[kMapSlots];
  bool used[kMapSlots] = {};
  alignas(64) CUtensorMap map[kMapSlots];
  int next = 0;
};
MapCache &map_cache() {
  static MapCache c;
  return c;
}
bool map_lookup(const MapKey &k, CUtensorMap *out) {
  MapCache &c = map_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  for (int i = 0; i < kMapSlots; ++i)
    if (c.used[i] && c.key[i] == k) {
      memcpy(out, &c.map[i], sizeof(CUtensorMap));
      return true;
    }
  return false;
}
void map_insert(const MapKey &k, const CUtensorMap &m) {
  MapCache &c = map_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  const int i = c.next;
  c.next = (c.next + 1) % kMapSlots;
  c.key[i] = k;
  memcpy(&c.map[i], &m, sizeof(CUtensorMap));
  c.used[i] = true;
}

struct OccKey {
  int dev;
  const void *kern;
  int threads, smem;
};
constexpr int kOccSlots = 256;
struct OccCache {
  std::mutex mu;
  OccKey key[kOccSlots];
  int blocks[kOccSlots];
  int n = 0;
  // per (device, kernel): the dynamic shared memory limit set so far
  OccKey limit[kOccSlots];
  int nlimit = 0;
};
OccCache &occ_cache() {
  static OccCache c;
  return c;
}
}  // namespace

cudaError_t blocks_per_sm(const void *kern, int threads, int smem, int *blocks) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  OccCache &c = occ_cache();
  std::lock_guard<std::mutex> lock(c.mu);
  for (int i = 0; i < c.n; ++i)
    if (c.key[i].dev == dev && c.key[i].kern == kern && c.key[i].threads == threads && c.key[i].smem == smem) {
      *blocks = c.blocks[i];
      return cudaSuccess;
    }
  // The limit only ever grows, so a size remembered earlier stays launchable.
  int li = -1;
  for (int i = 0; i < c.nlimit; ++i)
    if (c.limit[i].dev == dev && c.limit[i].kern == kern) li = i;
  if (li < 0 || c.limit[li].smem < smem) {
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if (li < 0 && c.nlimit < kOccSlots) li = c.nlimit++;
    if (li >= 0) c.limit[li] = OccKey{dev, kern, 0, smem};
  }
  int o = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, threads, smem)) != cudaSuccess) return e;
  if (c.n < kOccSlots) {
    c.key[c.n] = OccKey{dev, kern, threads, smem};
    c.blocks[c.n++] = o;
  }
  *blocks = o;
  return cudaSuccess;
}

// [B*T, C] view of a [B, T, C] tensor, boxes of 32 columns x `rows` rows.
bool encode_rows(CUtensorMap *m, const void *ptr, int dtype, int64_t rows, int64_t C,
                 int box_rows) {
  const MapKey key{ptr, C, rows, 0, dtype, 2, box_rows};
  if (map_lookup(key, m)) return true;
  auto enc = tensor_map_encoder();
  if (!enc || !ensure_context()) return false;
  const size_t es = dtype == 0 ? 4 : 2;
  cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(C * es)};
  cuuint32_t box[2] = {32u, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1u, 1u};
  // L2 fills promoted to the box row (32 columns) and no further: a wider
  // fill fetches the neighbouring chain's bytes on this chain's behalf, and
  // they may leave L2 before that chain's warp reads them
  const auto promo = dtype == 0 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
  if (enc(m, dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
          const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, promo, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_insert(key, *m);
  return true;
}

// [B, T, C] tensor as a 3-D map (C fastest), boxes of 32 channels x `box_t`
// tokens x 1 batch row.  Loads past T or C read zeros and stores there are
// clipped, so a box never reaches into the next batch row.
bool encode_btc(CUtensorMap *m, const void *ptr, int dtype, int64_t B, int64_t T, int64_t C, int box_t) {
  const MapKey key{ptr, C, T, B, dtype, 3, box_t};
  if (map_lookup(key, m)) return true;
  auto enc = tensor_map_encoder();
  if (!enc || !ensure_context()) return false;
  const size_t es = dtype == 0 ? 4 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[2] = {(cuuint64_t)(C * es), (cuuint64_t)(T * C * es)};
  cuuint32_t box[3] = {32u, (cuuint32_t)box_t, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  // a box row is 32 channels (128 bytes fp32, 64 bytes bf16) of one token;
  // L2 fills are promoted to that size and no further, so the neighbouring
  // chain-tile's bytes are not fetched on this tile's behalf
  if (enc(m, dtype == 0 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
          const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_NONE, dtype == 0 ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_64B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_insert(key, *m);
  return true;
}

// Checkpoints [nck][3][B][C] float32 as a 4-D map (channels fastest),
// boxes of 32 channels x 1 batch row x 3 planes x box_ck checkpoints: one
// chain's consecutive checkpoints land as [box_ck][3][32] floats.  Indices
// past nck or C read zeros.
bool encode_ckpt(CUtensorMap *m, const float *ck, int64_t B, int64_t C, int64_t nck, int box_ck) {
  const MapKey key{ck, C, B, nck, 0, 104, box_ck};
  if (map_lookup(key, m)) return true;
  auto enc = tensor_map_encoder();
  if (!enc || !ensure_context()) return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)B, 3u, (cuuint64_t)nck};
  cuuint64_t strides[3] = {(cuuint64_t)(C * 4), (cuuint64_t)(B * C * 4), (cuuint64_t)(3 * B * C * 4)};
  cuuint32_t box[4] = {32u, 1u, 3u, (cuuint32_t)box_ck};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  if (enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(ck), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_insert(key, *m);
  return true;
}

// [BH, N, width] bfloat16 tensor as a 3-D map (width fastest), boxes of
// width x 128 rows x 1 head in the 64-byte swizzle, which is the layout the
// tensor cores read their operands in (width * 2 must be 64 bytes).  Rows
// past N read zeros and stores there are clipped.
bool encode_heads_sw64(CUtensorMap *m, const void *ptr, int64_t BH, int64_t N, int width) {
  const MapKey key{ptr, width, N, BH, 1, 103, 128};
  if (map_lookup(key, m)) return true;
  auto enc = tensor_map_encoder();
  if (!enc || !ensure_context() || width * 2 != 64) return false;
  cuuint64_t dims[3] = {(cuuint64_t)width, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)(width * 2), (cuuint64_t)(N * width * 2)};
  cuuint32_t box[3] = {(cuuint32_t)width, 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  if (enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_insert(key, *m);
  return true;
}

// TMA needs 16-byte aligned rows and base addresses, and row indices < 2^31.
bool fwd_tma_eligible(const FwdArgs &a, int dtype) {
  const int64_t es = dtype == 0 ? 4 : 2;
  return (a.C * es) % 16 == 0 && ((uintptr_t)a.k % 16) == 0 && ((uintptr_t)a.v % 16) == 0 &&
         a.B * a.T + 4096 < (int64_t(1) << 31) && tensor_map_encoder() != nullptr;  // rows past T stay int
}

template <typename E>
static cudaError_t launch_fwd_tma_t(const FwdArgs &a, int dtype, int num_sms, cudaStream_t st) {
  using Lay = TmaFwdLayout<E, kTmaW, kTmaL, kTmaS>;
  CUtensorMap km, vm;
  if (!encode_rows(&km, a.k, dtype, a.B * a.T, a.C, Lay::TC) ||
      !encode_rows(&vm, a.v, dtype, a.B * a.T, a.C, Lay::TC))
    return cudaErrorInvalidValue;
  auto kern = fwd_tma_kernel<E, kTmaW, kTmaL, kTmaS>;
  const int threads = (kTmaW + 2) * 32;
  int per_sm = 0;
  cudaError_t e = blocks_per_sm((const void *)kern, threads, Lay::BYTES, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const int64_t tiles = a.nchains * a.nchunks;
  const int64_t grid = tiles < (int64_t)per_sm * num_sms ? tiles : (int64_t)per_sm * num_sms;
  FwdArgs args = a;
  void *kargs[] = {&km, &vm, &args};
  return cudaLaunchCooperativeKernel((const void *)kern, dim3((unsigned)grid), dim3(threads), kargs,
                                     (size_t)Lay::BYTES, st);
}

template <typename E>
static cudaError_t launch_fwd_t(const FwdArgs &a, int kind, int dtype, int num_sms, cudaStream_t st) {
  if (kind == 0) {
    const int64_t BC = a.B * a.C;
    const unsigned grid = (unsigned)((BC + 255) / 256);
    return launch_kernel(fwd_seq_kernel<E, kSeqU>, dim3(grid), dim3(256), 0, st, a);
  }
  if (kind == 2) return launch_fwd_tma_t<E>(a, dtype, num_sms, st);
  const int64_t tiles = a.nchains * a.nchunks;
  return launch_kernel(fwd_chunked_kernel<E, kFwdW, kFwdL>, dim3((unsigned)tiles), dim3(kFwdW * 32), 0, st, a);
}

// kind: 0 sequential, 1 register-tile chunked, 2 TMA chunked.
cudaError_t launch_forward(const FwdArgs &a, int dtype, int kind, int num_sms, cudaStream_t st) {
  return dtype == 0 ? launch_fwd_t<float>(a, kind, dtype, num_sms, st)
                    : launch_fwd_t<uint16_t>(a, kind, dtype, num_sms, st);
}

}  // namespace wkv
