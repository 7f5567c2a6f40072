// wkv_ring.cuh -- per-warp TMA ring of row batches (internal).
#pragma once

#include <cuda.h>

#include "wkv_internal.cuh"

namespace wkv {

// Shared memory of a block of NW warps: all stages first (each warp's S
// stages contiguous, every stage a multiple of 128 bytes, so every TMA
// destination is 128-byte aligned as tensor copies require), then all the
// mbarriers (8 bytes each).  A stage holds ROWS rows of 32 channels of each
// of the NARR tensors.
template <typename E, int S, int NARR, int ROWS>
struct WarpRing {
  static constexpr int ARR_BYTES = ROWS * 32 * (int)sizeof(E);
  static constexpr int STAGE_BYTES = NARR * ARR_BYTES;
  static_assert(ARR_BYTES % 128 == 0, "TMA destinations must stay 128-byte aligned");
  static constexpr int RING_BYTES = S * STAGE_BYTES;
  static constexpr int block_bytes(int nw) { return nw * (RING_BYTES + S * 8); }
};

template <typename E, int S, int NARR, int ROWS>
struct Ring {
  using L = WarpRing<E, S, NARR, ROWS>;
  unsigned char *base;
  uint32_t bar0;
  __device__ __forceinline__ Ring(unsigned char *smem, int wl, int nw) {
    base = smem + (size_t)wl * L::RING_BYTES;
    bar0 = smem_addr(smem + (size_t)nw * L::RING_BYTES) + 8u * S * wl;
  }
  __device__ __forceinline__ const E *stage(int s, int arr) const {
    return reinterpret_cast<const E *>(base + (size_t)s * L::STAGE_BYTES + (size_t)arr * L::ARR_BYTES);
  }
  __device__ __forceinline__ uint32_t bar(int s) const { return bar0 + 8u * s; }
  __device__ __forceinline__ void init(int lane) const {
    if (lane == 0) {
      for (int s = 0; s < S; ++s) mbar_init(bar(s), 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
  }
  // True when every stage of this warp's ring is 128-byte aligned (checked
  // once; issue_stage then skips the per-copy check).
  __device__ __forceinline__ bool aligned() const {
    uint32_t bad = 0;
    for (int s = 0; s < S; ++s)
      for (int a = 0; a < NARR; ++a) bad |= smem_addr(stage(s, a)) & 127u;
    return bad == 0;
  }
  // As issue_stage, loading only the first n of the NARR tensors.
  __device__ __forceinline__ void issue_stage_n(const CUtensorMap *const (&maps)[NARR], int s, int x, int y,
                                                uint64_t policy, int n) const {
    mbar_expect_tx(bar(s), (uint32_t)(n * L::ARR_BYTES));
#pragma unroll
    for (int a = 0; a < NARR; ++a)
      if (a < n) tma_load_2d_hint(smem_addr(stage(s, a)), maps[a], x, y, bar(s), policy);
  }
  // Loads into stage s (the caller tracks stages), with an L2 policy; the
  // ring must have passed aligned().
  __device__ __forceinline__ void issue_stage(const CUtensorMap *const (&maps)[NARR], int s, int x, int y,
                                              uint64_t policy) const {
    mbar_expect_tx(bar(s), (uint32_t)L::STAGE_BYTES);
#pragma unroll
    for (int a = 0; a < NARR; ++a) tma_load_2d_hint(smem_addr(stage(s, a)), maps[a], x, y, bar(s), policy);
  }
};

}  // namespace wkv
