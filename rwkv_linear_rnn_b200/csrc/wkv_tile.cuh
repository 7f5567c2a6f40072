// wkv_tile.cuh -- definitions shared by the tile kernels (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "wkv_internal.cuh"

namespace wkv {

constexpr int kTileWarps = 4;   // warps per block (backward)
constexpr int kTileFwdWarps = 3;  // warps per block (forward: three blocks of 3 x 24 KB fit an SM)
constexpr int kTileLF32 = 32;   // tokens per unit, fp32 tensors
constexpr int kTileLBF16 = 64;  // tokens per unit, bf16 tensors (same tile bytes)
constexpr int kTileRB = 16;     // tokens per batch of the fast path
constexpr int kMaxDevices = 64; // per-device launch caches

struct TileFwdArgs {
  FwdArgs f;
  float4 *rec;   // [units][2][32] records: summary, inclusive prefix
  int64_t nseg;  // units per chain
};

// Round a float to the tensor element type (bf16: to nearest, ties to even).
template <typename E>
__device__ __forceinline__ E from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ uint16_t from_f32<uint16_t>(float x) {
  unsigned short h;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(x));
  return h;
}

// Per-lane constants of the batch fast path in the form the tile and chain
// kernels use (see FastC in wkv_math.cuh for the two modes).  The undecayed mode
// carries the state as alpha' = alpha 2^{w2}, which removes one multiply per
// token: alpha' += e0 v, and the bonus factor becomes 2^{u2 + w2}.
struct TileFast {
  float we;    // decay folded into the keys (natural log): w undecayed, 0 decaying
  float ewm;   // per-token multiplicative decay (decaying) or 1
  float cu;    // bonus factor relative to e0: 2^{u2 + w2e}
  float sh;    // w2e: added to the state's scale exponent at batch start
  float nend;  // anchored decay count after a batch: RB - 1 undecayed, 0 decaying
  bool ok;     // the fast path is valid for this lane's decay (no growth)
};
template <int RB>
__device__ __forceinline__ TileFast tile_fast(float w, float w2, float u2) {
  const bool decaying = fabsf(w2) * (float)RB >= 40.f;
  TileFast f;
  f.we = decaying ? 0.f : w;
  const float w2e = decaying ? 0.f : w2;
  f.ewm = decaying ? ex2(w2) : 1.f;
  f.cu = ex2(u2 + w2e);
  f.sh = w2e;
  f.nend = decaying ? 0.f : (float)(RB - 1);
  f.ok = !(decaying && w2 > 0.f) && u2 < 60.f;  // a growing state could overflow within a batch
  return f;
}

// ------------------------------------------------------------- TMA (3-D) ---
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *map, int x, int y, int z, uint32_t bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const void *map, int x, int y, int z, uint32_t src) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(src)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk store of this thread has read its shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every bulk store of this thread is complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Generic-proxy accesses to shared memory ordered before later async-proxy ones.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------- records ---
// The tile kernels join their units through records in the workspace that
// carry their own validity: every 16-byte word of a record holds, in its
// last 32 bits, a tag made of the launch epoch and the record kind, and is
// written and read with single 16-byte accesses (aligned 16-byte vector
// accesses are performed as one access, the property decoupled look-back
// scans rely on).  A reader that sees the expected tag in a word sees that
// word's payload; a word from an earlier launch, or not yet written, shows
// another tag and is read again.  So publishing needs no fence: payload and
// tag travel together.  A per-unit status word (the tag of the latest record
// published) is a hint that tells a reader how far back to look; the words
// themselves decide.
constexpr unsigned kFlagAgg = 1u, kFlagInc = 2u;
__device__ __forceinline__ unsigned tile_flag(unsigned epoch, unsigned what) {
  return (epoch_tag(epoch) << 2) | what;
}
__device__ __forceinline__ void st_relaxed_v4(float4 *p, float4 v) {
  asm volatile("st.relaxed.gpu.global.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}
__device__ __forceinline__ float4 ld_relaxed_v4(const float4 *p) {
  float4 v;
  asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u32(unsigned *p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ float tagf(unsigned t) { return __uint_as_float(t); }
__device__ __forceinline__ bool tag_is(float x, unsigned t) { return __float_as_uint(x) == t; }

// Forward records, 1.5 KB per unit: the unit's summary (a, b, E, tag) at
// rec[unit * 96 + lane] with its exponent evaluated (E = P + n w2, one
// rounding: a summary enters a prefix once, so nothing accumulates), then
// its inclusive prefix in two words, (a, b, P, tag) at +32 and (n, tag, 0, 0)
// at +64, with the anchored exponent kept exact along the chain.
constexpr int kFwdRecWords = 96;
__device__ __forceinline__ void tile_put_agg(float4 *rec, int64_t unit, const St &s, float w2, unsigned tag,
                                             int lane) {
  st_relaxed_v4(rec + unit * kFwdRecWords + lane, make_float4(s.a, s.b, st_exp(s, w2), tagf(tag)));
}
__device__ __forceinline__ void tile_put_inc(float4 *rec, int64_t unit, const St &s, unsigned tag, int lane) {
  float4 *d = rec + unit * kFwdRecWords + lane;
  st_relaxed_v4(d + 32, make_float4(s.a, s.b, s.P, tagf(tag)));
  st_relaxed_v4(d + 64, make_float4(s.n, tagf(tag), 0.f, 0.f));
}

// dL/dw, dL/du partials of the tile backwards: one tagged word (gw, gu, tag,
// 0) per (unit position, b, c).  Sums of n such words spaced `stride` words
// apart, in index order in float64, sixteen loads in flight, re-reading
// words whose tag does not check yet (their stores may still be on the way).
// False if the wait bound ran out.  (Eight loads in flight.)
constexpr int kPartGroup = 16;  // positions per first-level sum
__device__ __forceinline__ bool sum_tagged(const float4 *p, int64_t stride, int n, unsigned tag, double &sx,
                                           double &sy, int64_t budget_ns) {
  sx = 0.0;
  sy = 0.0;
  const uint64_t t0 = global_ns();
  for (int i0 = 0; i0 < n; i0 += 8) {
    float4 r[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j < n) r[j] = ld_relaxed_v4(p + (int64_t)(i0 + j) * stride);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (i0 + j < n) {
        while (!tag_is(r[j].z, tag)) {
          if ((int64_t)(global_ns() - t0) > budget_ns) return false;
          __nanosleep(64);
          r[j] = ld_relaxed_v4(p + (int64_t)(i0 + j) * stride);
        }
        sx += (double)r[j].x;
        sy += (double)r[j].y;
      }
    }
  }
  return true;
}
// The fixed-order sums of one channel's partials, called by the warp that ran
// the unit at position `pos` after it stored its own partial: a unit at a
// position that is a multiple of kPartGroup adds the partials of its group
// (positions pos .. pos + kPartGroup - 1, later in time, so earlier in scan
// order) into a first-level word; the chain's first unit adds the first-level
// words into the chain's sum; the chain of the last batch row of a channel
// tile then adds the chains.  Every word waited on comes from a unit earlier
// in scan order, which never waits on this warp.  part: [nseg][B][C] words,
// l1: [ceil(nseg / kPartGroup)][B][C], chain: [B][C].  Out of line: it runs
// once per kPartGroup units and keeps its registers out of the unit loop.
static __device__ __noinline__ void reduce_partials(const float4 *part, float4 *l1, float4 *chain, float *gw, float *gu,
                                                int pos, int nseg, int64_t b, int64_t B, int64_t c, int64_t C,
                                                unsigned tag, int64_t budget_ns, WsHeader *hdr, unsigned epoch) {
  if (pos % kPartGroup != 0) return;
  const int64_t BC = B * C, bc = b * C + c;
  bool ok = true;
  double sw, su;
  ok = sum_tagged(part + (int64_t)pos * BC + bc, BC, min(kPartGroup, nseg - pos), tag, sw, su, budget_ns) && ok;
  st_relaxed_v4(l1 + (int64_t)(pos / kPartGroup) * BC + bc, make_float4((float)sw, (float)su, tagf(tag), 0.f));
  if (pos == 0) {
    ok = sum_tagged(l1 + bc, BC, (nseg + kPartGroup - 1) / kPartGroup, tag, sw, su, budget_ns) && ok;
    st_relaxed_v4(chain + bc, make_float4((float)sw, (float)su, tagf(tag), 0.f));
    if (b == B - 1) {
      ok = sum_tagged(chain + c, C, (int)B, tag, sw, su, budget_ns) && ok;
      gw[c] = (float)sw;
      gu[c] = (float)su;
    }
  }
  if (!ok) raise_timeout(hdr, epoch);
}

// Tokens per unit of the tile kernels for an element type (0 fp32, 1 bf16).
int tile_fwd_tokens(int dtype);

}  // namespace wkv
