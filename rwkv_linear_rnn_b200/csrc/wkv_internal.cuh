// wkv_internal.cuh -- device helpers and launch descriptors shared by the
// libwkv kernels (internal; not part of the C ABI).
//
// Numerical scheme.  The WKV sums are carried in the max-rescaled form
// (a, b, P): A = a * 2^P, B = b * 2^P, where A_t, B_t are the hidden sums of
// the RNN form (RWKV paper review, "[논문 리뷰] Reinvention RNNs for the
// Transformer Era: RWKV", section "RNN-유사추론", eq. WKV_t).  Inside the
// kernels every exponent is in base 2 (k, u, w are multiplied by log2(e) on
// load) so that each exponential is one ex2.approx instruction; states that
// cross the C ABI use natural-log exponents.  P is the largest exponent of
// any term of the sum, so a, b stay in [0, #tokens] and nothing overflows.
//
// Exponent bookkeeping: while no new token takes over the maximum, the
// exponent after n decays is formed as fma(n, w, P_anchor) (one rounding)
// instead of by n repeated additions (n roundings), so long decays do not
// drift.  The same anchoring is used for the adjoint scale in the backward.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace wkv {

constexpr float kLog2e = 1.4426950408889634f;  // log2(e)
constexpr float kLn2 = 0.6931471805599453f;    // ln(2)
// Exponent of the empty state.  Finite so that differences never form
// inf - inf; 2^(anything - 1e38) flushes to exactly 0.
constexpr float kEmptyP = -1.0e38f;
// Scale of the empty adjoint (Ahat = ahat * 2^-r with r = +1e38).
constexpr float kEmptyR = 1.0e38f;
constexpr int kCkpt = 16;  // tokens between forward checkpoints

// -------------------------------------------------------------- launch ---
// Launch with the launch's own status.  (A <<<...>>> launch followed by
// cudaGetLastError would also return a stale error that an unrelated runtime
// call left in the calling thread.)
template <typename... P, typename... A>
inline cudaError_t launch_kernel(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                 A &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<A &&>(args)...);
}

// Resident blocks per SM of `kern` launched with `threads` threads and `smem`
// bytes of dynamic shared memory, on the current device.  The first query of
// each (device, kernel, threads, smem) raises the kernel's dynamic shared
// memory limit as far as needed and asks the occupancy calculator; the answer
// is remembered, so later launches make no runtime call for it.
cudaError_t blocks_per_sm(const void *kern, int threads, int smem, int *blocks);

// ---------------------------------------------------------------- math ---
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Forward state of one channel: A = a 2^E, B = b 2^E with the exponent in
// anchored form E = P + n w (P: the exponent of the term that set the
// maximum, n: decay steps since then, an exact integer in a float).  Carrying
// (P, n) instead of the rounded sum keeps E within one rounding of exact
// through any number of joins, however long the sequence.
struct St {
  float a, b, P, n;
};
__device__ __forceinline__ St st_empty() { return St{0.f, 0.f, kEmptyP, 0.f}; }
__device__ __forceinline__ float st_exp(const St &s, float w2) { return fmaf(s.n, w2, s.P); }

// Sequence X followed by a sequence Y of lenY tokens: X's sums decay lenY
// times (exponent + lenY * w), then the two are added at the larger scale.
// This is the associative combine that lets the time axis be split into
// chunks ("Transformer-유사학습": the serial WKV part is done as a scan).
__device__ __forceinline__ St combine(const St &X, const St &Y, float lenY, float w2) {
  const float nx = X.n + lenY;
  const float Ex = fmaf(nx, w2, X.P);
  const float Ey = fmaf(Y.n, w2, Y.P);
  const float d = Ex - Ey;
  const float x = ex2(-fabsf(d));
  const bool xw = d >= 0.f;
  const float fx = xw ? 1.f : x, fy = xw ? x : 1.f;
  St r;
  r.a = fmaf(X.a, fx, Y.a * fy);
  r.b = fmaf(X.b, fx, Y.b * fy);
  r.P = xw ? X.P : Y.P;
  r.n = xw ? nx : Y.n;
  return r;
}

// Adjoint of one channel for the backward: Ahat = ah 2^-r, Hhat = hh 2^-r,
// where Ahat_t = dL/dA_t and Hhat_t = -dL/dB_t.
struct Adj {
  float ah, hh, r;
};
__device__ __forceinline__ Adj adj_empty() { return Adj{0.f, 0.f, kEmptyR}; }

// Reverse-time combine: X (earlier, lenX tokens) then Y (later).  The adjoint
// at the start of X gains Y's adjoint decayed across X (factor 2^{lenX w}).
__device__ __forceinline__ Adj rcombine(const Adj &X, const Adj &Y, float lenX, float w2) {
  const float rY = fmaf(-lenX, w2, Y.r);
  const float d = X.r - rY;
  const float x = ex2(-fabsf(d));
  const bool xs = d <= 0.f;  // X has the larger magnitude scale 2^-r
  const float fx = xs ? 1.f : x, fy = xs ? x : 1.f;
  Adj o;
  o.ah = fmaf(X.ah, fx, Y.ah * fy);
  o.hh = fmaf(X.hh, fx, Y.hh * fy);
  o.r = fminf(X.r, rY);
  return o;
}

// ---------------------------------------------------------- element I/O ---
template <typename E>
struct IO;
template <>
struct IO<float> {
  static __device__ __forceinline__ float ld(const float *p) { return __ldcs(p); }
  static __device__ __forceinline__ void st(float *p, float x) { __stcs(p, x); }
  // a store whose line should stay in L2 (read back soon)
  static __device__ __forceinline__ void st_keep(float *p, float x) { *p = x; }
};
template <>
struct IO<uint16_t> {  // bfloat16 storage
  static __device__ __forceinline__ float ld(const uint16_t *p) {
    unsigned short h;
    asm("ld.global.cs.u16 %0, [%1];" : "=h"(h) : "l"(p));
    return __uint_as_float(((unsigned)h) << 16);
  }
  static __device__ __forceinline__ void st(uint16_t *p, float x) {
    unsigned short h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
    asm volatile("st.global.cs.u16 [%0], %1;" ::"l"(p), "h"(h));
  }
  static __device__ __forceinline__ void st_keep(uint16_t *p, float x) {
    unsigned short h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
    asm volatile("st.global.u16 [%0], %1;" ::"l"(p), "h"(h) : "memory");
  }
};

// Load L rows (stride elements apart) of one column.  All L loads are issued
// back to back from always-valid addresses -- rows at or past `nvalid` repeat
// the last valid row and the caller ignores them -- so that the warp has
// every load in flight before it first waits on one.  (Guarding each load
// with a condition lets the compiler pair each load with its first use and
// serialises the round trips.)  Requires nvalid >= 1.
template <typename E, int L>
__device__ __forceinline__ void load_rows(const E *base, int64_t stride, int nvalid,
                                          float (&out)[L]) {
#pragma unroll
  for (int j = 0; j < L; ++j) out[j] = IO<E>::ld(base + (int64_t)min(j, nvalid - 1) * stride);
}

// ------------------------------------------------------ workspace header ---
// The first 256 bytes of every workspace.  Zero-filled once by the caller.
struct WsHeader {
  unsigned epoch;      // launches completed on this workspace
  unsigned ticket;     // next tile ticket of the running launch
  unsigned done;       // blocks finished in the running launch
  unsigned abort_tag;  // epoch+1 of a launch in which a wait gave up
  int status;          // first device-side error (sticky until read)
  unsigned bar;        // blocks arrived at the grid barrier of the running launch
  unsigned pad[58];
};
static_assert(sizeof(WsHeader) == 256, "header size");

// Tile status flags: (epoch tag << 2) | 1 once the tile's record is
// published.  A flag from an earlier launch carries an older tag and reads
// as "not ready".
constexpr unsigned kAgg = 1u;
__device__ __forceinline__ unsigned epoch_tag(unsigned epoch) { return epoch & 0x3FFFFFFFu; }

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(unsigned *p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Per-tile descriptor: one record (the Fenwick node of the chunk) of up to
// four float planes of 32 lanes each.
constexpr int kDescFloats = 5 * 32;

template <typename S>
__device__ __forceinline__ void desc_store(float *desc, int64_t tile, int which, const S &s,
                                           int lane) {
  constexpr int NF = sizeof(S) / sizeof(float);
  static_assert(NF * 32 <= kDescFloats, "record too large");
  float *d = desc + tile * kDescFloats + which * NF * 32;
  const float *f = reinterpret_cast<const float *>(&s);
#pragma unroll
  for (int i = 0; i < NF; ++i) __stcg(d + i * 32 + lane, f[i]);
}
template <typename S>
__device__ __forceinline__ S desc_load(const float *desc, int64_t tile, int which, int lane) {
  constexpr int NF = sizeof(S) / sizeof(float);
  const float *d = desc + tile * kDescFloats + which * NF * 32;
  S s;
  float *f = reinterpret_cast<float *>(&s);
#pragma unroll
  for (int i = 0; i < NF; ++i) f[i] = __ldcg(d + i * 32 + lane);
  return s;
}

// Lane-major records of the segment kernels: a St record is one float4 per
// lane (a single 16-byte load per lane, 512 bytes per warp); an adjoint
// record of five floats adds a fifth plane after it.
__device__ __forceinline__ void rec_store_st(float *desc, int64_t tile, const St &s, int lane) {
  float4 *d = reinterpret_cast<float4 *>(desc + tile * kDescFloats) + lane;
  __stcg(d, make_float4(s.a, s.b, s.P, s.n));
}
__device__ __forceinline__ St rec_load_st(const float *desc, int64_t tile, int lane) {
  const float4 v = __ldcg(reinterpret_cast<const float4 *>(desc + tile * kDescFloats) + lane);
  return St{v.x, v.y, v.z, v.w};
}

// A state in four planes of 32 lanes (shared or global memory).
__device__ __forceinline__ void put_st(float *d, int lane, const St &s) {
  d[lane] = s.a;
  d[32 + lane] = s.b;
  d[64 + lane] = s.P;
  d[96 + lane] = s.n;
}
__device__ __forceinline__ St get_st(const float *d, int lane) {
  return St{d[lane], d[32 + lane], d[64 + lane], d[96 + lane]};
}

// Publish a lane-major St record and then its flag (as publish below).
__device__ __forceinline__ void publish_st(float *desc, unsigned *flags, int64_t tile, const St &s,
                                          unsigned epoch, int lane) {
  rec_store_st(desc, tile, s, lane);
  __syncwarp();
  if (lane == 0) st_release(flags + tile, (epoch_tag(epoch) << 2) | kAgg);
  __syncwarp();
}

// Publish a record and then its flag (all lanes of the warp call this
// together).  The warp barrier orders every lane's record stores before lane
// 0's flag store, and the flag store is a gpu-scope release, which is
// cumulative: a reader that acquires the flag sees the whole record.
template <typename S>
__device__ __forceinline__ void publish(float *desc, unsigned *flags, int64_t tile, int which,
                                       const S &s, unsigned epoch, int lane) {
  desc_store(desc, tile, which, s, lane);
  __syncwarp();
  if (lane == 0) st_release(flags + tile, (epoch_tag(epoch) << 2) | kAgg);
  __syncwarp();
}

// Record a device-side error for this launch (first one wins) and mark the
// launch aborted so that other waiting blocks give up at once.
__device__ __forceinline__ void raise_timeout(WsHeader *h, unsigned epoch) {
  atomicCAS(&h->status, 0, -5 /* WKV_ERR_TIMEOUT */);
  atomicExch(&h->abort_tag, epoch + 1u);
}

// Block start: take a ticket (tiles are processed in ticket order, so every
// tile a block waits on belongs to a block that has already started) and
// read the launch epoch.
__device__ __forceinline__ void take_ticket(WsHeader *h, unsigned *s_tile, unsigned *s_epoch) {
  if (threadIdx.x == 0) {
    *s_tile = atomicAdd(&h->ticket, 1u);
    *s_epoch = ld_relaxed(&h->epoch);
  }
}

// Block end (after its last flag access): the last block of the launch
// resets the ticket and the counter and advances the epoch.
__device__ __forceinline__ void finish_block(WsHeader *h, unsigned nblocks) {
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&h->done, 1u);
    if (prev == nblocks - 1u) {
      h->ticket = 0u;
      h->done = 0u;
      h->bar = 0u;
      __threadfence();
      atomicAdd(&h->epoch, 1u);
    }
  }
}

// ------------------------------------------ deterministic chunk scan ---
// The time axis of every (b, channel tile) chain is cut into chunks; chunk
// `pos` (in scan order) publishes one record, the Fenwick node F(pos): the
// summary of the lowbit(pos+1) chunks ending at pos, joined in a fixed
// binary bracketing.  A chunk's exclusive prefix is the join of the nodes of
// the binary decomposition of pos.  Every combine therefore happens in an
// order fixed by pos alone: results are bit-identical from run to run,
// whatever order the blocks run in.  A block waits only on nodes of smaller
// positions, and the dependency depth is log2(#chunks).
//
// Position-ordered join: L covers the positions before R; R holds lenR
// tokens.  Forward: earlier positions are earlier in time.  Backward: scan
// order runs from the end of the sequence, so R is earlier in time.
__device__ __forceinline__ St pjoin(const St &L, const St &R, float lenR, float w2) {
  return combine(L, R, lenR, w2);
}
__device__ __forceinline__ Adj pjoin(const Adj &L, const Adj &R, float lenR, float w2) {
  return rcombine(R, L, lenR, w2);
}

__device__ __forceinline__ bool launch_aborted(WsHeader *h, unsigned epoch) {
  return ld_relaxed(&h->abort_tag) == epoch + 1u;
}

// Wait until every active lane's node (position q) is published.  Bounded:
// after `spin_limit` polls (or once another block of the launch gave up) the
// launch is marked aborted, the status word gets WKV_ERR_TIMEOUT and false is
// returned; the caller then goes on with invalid data so nothing hangs.
__device__ __forceinline__ bool wait_nodes(const unsigned *flags, int64_t q, bool active,
                                           int64_t chain, int64_t nchains, unsigned epoch,
                                           WsHeader *h, int64_t spin_limit, int lane) {
  const unsigned want = (epoch_tag(epoch) << 2) | kAgg;
  bool ready = !active;
  int64_t waits = 0;
  unsigned backoff = 32;
  while (true) {
    if (!ready) ready = ld_acquire(flags + (q * nchains + chain)) == want;
    if (__all_sync(0xffffffffu, ready)) {
      __syncwarp();
      return true;
    }
    if (++waits > spin_limit || launch_aborted(h, epoch)) {
      if (lane == 0) raise_timeout(h, epoch);
      __syncwarp();
      return false;
    }
    __nanosleep(backoff);
    backoff = backoff < 1024u ? backoff * 2u : 1024u;
  }
}

// Called by one warp per block.  `agg` is the block's own summary (agg_len
// tokens), `full_len` the tokens of a full chunk, `base0` the value before
// position 0 (initial state forward, empty adjoint backward).  Publishes
// F(pos) when a later position needs it (`need_node`) unless `publish_ok` is
// false (test hook), and returns the exclusive prefix of pos.
template <typename S>
__device__ S chunk_scan(unsigned *flags, float *desc, int64_t pos, int64_t chain, int64_t nchains,
                        const S &agg, float agg_len, float full_len, const S &base0,
                        const S &empty, unsigned epoch, WsHeader *h, int64_t spin_limit,
                        bool need_node, bool publish_ok, float w2, int lane) {
  const int64_t tile = pos * nchains + chain;
  // (1) F(pos) = F(pos-2^(n-1)) + ... + F(pos-2) + F(pos-1) + agg, bracketed
  //     from the right, n = log2(lowbit(pos+1)).
  const int64_t lb = (pos + 1) & -(pos + 1);
  const int nup = need_node ? 63 - __clzll((unsigned long long)lb) : 0;
  wait_nodes(flags, lane < nup ? pos - ((int64_t)1 << lane) : 0, lane < nup, chain, nchains,
             epoch, h, spin_limit, lane);
  S F = agg;
  float flen = agg_len;
  for (int i = 0; i < nup; ++i) {
    const int64_t s = (int64_t)1 << i;
    const S left = desc_load<S>(desc, (pos - s) * nchains + chain, 0, lane);
    F = pjoin(left, F, flen, w2);
    flen += (float)s * full_len;
  }
  if (need_node && publish_ok) publish(desc, flags, tile, 0, F, epoch, lane);
  // (2) exclusive prefix: nodes x-1 for x = pos, pos minus its lowest set
  //     bit, ... (one per set bit of pos), joined from the right.
  const int nd = __popcll((unsigned long long)pos);
  int64_t xl = pos;
  for (int k = 0; k < lane && k < nd; ++k) xl &= xl - 1;
  wait_nodes(flags, lane < nd ? xl - 1 : 0, lane < nd, chain, nchains, epoch, h, spin_limit, lane);
  S acc = empty;
  float acc_len = 0.f;
  int64_t x = pos;
  for (int k = 0; k < nd; ++k) {
    const int64_t sz = x & -x;
    const S node = desc_load<S>(desc, (x - 1) * nchains + chain, 0, lane);
    acc = pjoin(node, acc, acc_len, w2);
    acc_len += (float)sz * full_len;
    x &= x - 1;
  }
  return pjoin(base0, acc, acc_len, w2);
}

// ------------------------------------------------- mbarrier / TMA (sm_100a) ---
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase of `bar` with the given parity to complete.
// Gives up (returns false) after `budget_ns` nanoseconds or once *abort is
// set (abort may be null).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int64_t budget_ns,
                                          volatile int *abort) {
  const uint64_t t0 = global_ns();
  for (unsigned i = 0;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 15u) {
      if (abort && *abort) return false;
      if ((int64_t)(global_ns() - t0) > budget_ns) return false;
    }
  }
}
// Barrier over all blocks of a cooperative launch (every block resident).
// Bounded: after `budget_ns` the block records WKV_ERR_TIMEOUT and goes on.
// The counter is reset by the launch's last finish_block (every block has
// left the barrier by then).
__device__ __forceinline__ void grid_barrier(WsHeader *h, unsigned nblocks, int64_t budget_ns) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(&h->bar, 1u);
    const uint64_t t0 = global_ns();
    unsigned backoff = 64;
    while (ld_acquire(&h->bar) < nblocks) {
      if ((int64_t)(global_ns() - t0) > budget_ns) {
        atomicCAS(&h->status, 0, -5 /* WKV_ERR_TIMEOUT */);
        break;
      }
      __nanosleep(backoff);  // back off: spinning steals issue slots from working warps
      backoff = backoff < 256u ? backoff * 2u : 256u;
    }
  }
  __syncthreads();
}
// Logistic gate sigma(r) = 1 / (1 + 2^{-r log2 e}) from the hardware
// exp2 and reciprocal (saturates to 0 / 1 for large |r|).
__device__ __forceinline__ float gate_sigmoid(float r) { return rcp(1.f + ex2(-r * kLog2e)); }
// The gate and its slope sigma'(r) = sigma (1 - sigma) = e / (1 + e)^2 with
// e = exp(-r), formed without the cancellation of 1 - sigma near sigma = 1;
// e is capped so that e = inf (r -> -inf) gives slope 0, not inf * 0.
__device__ __forceinline__ void gate_sigmoid_slope(float r, float &s, float &ds) {
  const float e = ex2(-r * kLog2e);
  const float q = rcp(1.f + e);
  s = q;
  ds = fminf(e, 1.0e30f) * q * q;
}
// L2 eviction-priority policies for TMA loads (createpolicy).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
// As tma_load_2d, with an L2 eviction-priority hint.
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const void *map, int x, int y,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// 2-D tiled TMA load of box {32 columns, rows} at column x, row y into shared
// memory, completing on `bar` (transaction bytes).  No multicast.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// ---------------------------------------------------- launch descriptors ---
struct FwdArgs {
  int64_t B, T, C;
  const float *w, *u;
  const void *k, *v;
  const float *state_in;  // natural-log exponent, may be null
  void *y;                // may be null (checkpoint-only pass)
  float *state_out;       // natural-log exponent, may be null
  float *ckpt;            // base-2 exponent, [nck][3][B][C], may be null
  WsHeader *hdr;
  unsigned *flags;
  float *desc;
  int64_t nct;      // channel tiles of 32 per batch row
  int64_t nchains;  // B * nct
  int64_t nchunks;  // chunks of the time axis
  int64_t spin_limit;
  int hold_first;
  const void *r;  // output gate input [B, T, C] (y becomes sigma(r) * wkv), or null
};

struct BwdArgs {
  int64_t B, T, C;
  const float *w, *u;
  const void *k, *v, *gy;
  const float *ckpt;  // base-2 exponent checkpoints [nck][3][B][C]
  void *gk, *gv;
  float *part;  // [nchunks][2][B][C] per-chunk partial dL/dw, dL/du
  WsHeader *hdr;
  unsigned *flags;
  float *desc;
  int64_t nct, nchains, nchunks;
  int64_t spin_limit;
  int hold_first;
  const void *r;  // output gate input (grad_y is then the gated output's gradient), or null
  void *gr;       // gradient of the gate input (with r)
  // State terms of a sequence split across calls (all null when unused):
  const float *gs_out;    // [3][B][C] dL/d(a, b, p) of the state after the last token
  const float *p_out;     // [B][C] the p plane of the representation gs_out refers to
  float *gs_in;           // [3][B][C] receives dL/d(a, b, p) of state_in
  const float *state_in;  // the caller's initial state as given (null: empty)
};

// Adjoint of the final sums from dL/d(a, b) of a state representation with
// exponent p (natural log): dL/dA_T = ga e^{-p}, dL/dB_T = gb e^{-p}, held as
// Ahat = ah 2^{-r}, Hhat = hh 2^{-r} (Hhat = -dL/dB) scaled by an exact power
// of two so that |ah| + |hh| lies in [1, 2) (the adjoint joins pick their
// anchor from r and assume normalised values).  Zero gradients and an empty
// state (p = -inf) give the empty adjoint; NaN and inf pass unscaled.
__device__ __forceinline__ void end_adjoint(float ga, float gb, float p, float &ah, float &hh, float &r) {
  const float m = fabsf(ga) + fabsf(gb);
  if (m == 0.f || p == -INFINITY) {
    ah = 0.f;
    hh = 0.f;
    r = kEmptyR;
    return;
  }
  const int e = m < INFINITY ? ilogbf(m) : 0;
  ah = ldexpf(ga, -e);
  hh = -ldexpf(gb, -e);
  r = fmaf(p, kLog2e, -(float)e);
}

// dL/d(a, b, p) of the caller's initial state (a, b, p) from the adjoint of
// the initial sums, Ahat_0 = ah 2^{-r0}, Hhat_0 = hh 2^{-r0}:
// dL/da = Ahat_0 e^p, dL/db = -Hhat_0 e^p, dL/dp = a dL/da + b dL/db.
// s_in null (the empty state) gives zeros.
__device__ __forceinline__ void store_state_grad(float *gs, const float *s_in, int64_t bc, int64_t BC,
                                                 float ah, float hh, float r0) {
  float ga = 0.f, gb = 0.f, gp = 0.f;
  if (s_in) {
    const float a = s_in[bc], b = s_in[BC + bc], p = s_in[2 * BC + bc];
    const float f = ex2(fmaf(p, kLog2e, -r0));
    ga = ah * f;
    gb = -hh * f;
    gp = fmaf(a, ga, b * gb);
  }
  gs[bc] = ga;
  gs[BC + bc] = gb;
  gs[2 * BC + bc] = gp;
}

struct StepArgs {
  int64_t N, C;
  const float *w, *u, *k, *v, *state_in;
  float *y, *state_out;
};

}  // namespace wkv
