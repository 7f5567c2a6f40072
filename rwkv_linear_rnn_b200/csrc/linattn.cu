// linattn.cu -- causal linear attention with the elu + 1 feature map, on the
// sm_100a tensor cores: chunked products issued with tcgen05.mma, operands
// staged in shared memory by TMA, accumulators in tensor memory.
//
// Linear attention post ("Transformers are RNNs: 선형 어텐션으로 만드는 빠른
// 자기회귀 트랜스포머"): section "인과 마스킹과 누적합" gives the causal form
// with the cumulative states S_i = sum_{j<=i} phi(K_j) V_j^T and
// Z_i = sum_{j<=i} phi(K_j), V'_i = phi(Q_i)^T S_i / (phi(Q_i)^T Z_i);
// section "특징 맵 선택과 계산 비용" the feature map phi(x) = elu(x) + 1;
// section "상수 메모리 기울기 계산" the gradients as a forward cumulative sum
// (for phi(Q)) and reverse cumulative sums (for phi(K) and V).
//
// Chunked form.  Positions are cut into chunks of L = 128; inside chunk c,
// rows i and j are positions c*L + i and c*L + j, and S_prev, Z_prev are the
// sums of phi(K)^T V and phi(K)^T 1 over the chunks before c:
//   forward   A = tril(phi(Q) phi(K)^T)          (j <= i kept)
//             den = A 1 + phi(Q) Z_prev,  out = (A V + phi(Q) S_prev) / den
//   backward  gnum = G / den,  gden = -rowsum(G * out) / den,
//             P = tril(gnum V^T + gden 1^T),
//             dphi(Q) = P phi(K) + gnum S_prev^T + gden Z_prev^T,
//             dphi(K) = P^T phi(Q) + V U_next^T + 1 u_next^T,
//             dV      = A^T gnum + phi(K) U_next,
//   with U_next, u_next the sums of phi(Q)^T gnum, phi(Q)^T gden over the
//   chunks after c, and then the chain rule through phi (phi'(x) = 1 for
//   x > 0, e^x otherwise, which is min(phi(x), 1)).
//
// Every product above is one or a few tcgen05.mma (kind::f16, bfloat16
// operands, float32 accumulation in tensor memory, M = 128).  The chunk
// states are summed over chunks by a separate scan kernel in a fixed order,
// so the results do not depend on scheduling.
//
// Shared-memory tiles are the 128B-atom canonical layouts the MMA reads:
// a [128 x 32] bfloat16 tile (64-byte rows) in the 64-byte swizzle, which is
// also what TMA writes with CU_TENSOR_MAP_SWIZZLE_64B, and the [128 x 128]
// masked score tiles in the 128-byte swizzle as two [128 x 64] halves.  One
// tile serves as a K-major operand and, transposed, as an MN-major one.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/linattn.h"
#include "../../include/wkv.h"
#include "wkv_internal.cuh"
#include "wkv_tile.cuh"

namespace wkv {

bool encode_heads_sw64(CUtensorMap *m, const void *ptr, int64_t BH, int64_t N, int width);

namespace la {

constexpr int kL = 128;                  // positions per chunk (the MMA's M)
constexpr int kD = 32;                   // head size: D = M
constexpr int kDM = kD * kD;             // floats of S
constexpr int kRec = kDM + kD;           // floats of one chunk state (S, then Z)
constexpr uint32_t kTile = kL * kD * 2;  // bytes of a [128 x 32] bf16 tile
constexpr uint32_t kStile = kD * kD * 2; // bytes of a [32 x 32] bf16 tile
constexpr uint32_t kPhalf = kL * 64 * 2; // bytes of one [128 x 64] half of a score tile
constexpr int kWarpgroup = 128;   // threads of one warpgroup: one per tile row
constexpr int kThreads = 256;     // threads per CTA: two warpgroups

struct LaArgs {
  int64_t BH, N;
  int nch;          // chunks per head
  float *rec;       // [BH][nch][kRec]: chunk states, then their exclusive prefix
  float *rec_r;     // [BH][nch][kRec]: reverse chunk states, then exclusive suffix
  float *gden;      // [BH][N]
  float *den;       // [BH][nch * 128]: the forward's denominators (kept for a saved-state backward)
  WsHeader *hdr;
  int64_t budget_ns;
};

// ------------------------------------------------------------ tcgen05 ---
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D (tensor memory) = A B^T (+ D if `acc`), A and B from shared-memory
// descriptors; issued by one thread.
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc)
      : "memory");
}
// Arrive on `bar` once every MMA issued so far by this thread is complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// 32 consecutive columns of this warp's 32 lanes (lane = thread's row).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

// 16 consecutive columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}
// One column of this warp's 32 lanes.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
  return __uint_as_float(r);
}

// Bulk copy (no tensor map) of `bytes` from global memory into shared memory,
// completing on `bar`; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Shared-memory matrix descriptor: start address, leading and stride byte
// offsets, the fixed version bits of sm_100, and the swizzle layout.
constexpr uint32_t kSw128 = 2, kSw64 = 4;
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
// Operand views of the tiles.  K-major: rows are the M (or N) index and the
// contraction runs along a row; MN-major: the transposed view of the same
// bytes.  `k16` is the 16-wide step of the contraction.
__device__ __forceinline__ uint64_t kmaj64(uint32_t tile, int k16) {  // [rows x 32], K along the row
  return sdesc(tile + 32u * k16, 16u, 512u, kSw64);
}
__device__ __forceinline__ uint64_t mnmaj64(uint32_t tile, int k16, uint32_t group_stride) {  // K down the rows
  return sdesc(tile + 1024u * k16, group_stride, 512u, kSw64);
}
__device__ __forceinline__ uint64_t kmaj128(uint32_t tile, int k16) {  // [128 x 128] in two halves
  return sdesc(tile + kPhalf * (k16 >> 2) + 32u * (k16 & 3), 16u, 1024u, kSw128);
}
__device__ __forceinline__ uint64_t mnmaj128(uint32_t tile, int k16) {  // its transpose
  return sdesc(tile + 2048u * k16, kPhalf, 1024u, kSw128);
}
// Instruction descriptor: bf16 x bf16 -> f32, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ elementwise ---
__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : __expf(x); }
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ float lo16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t phi2(uint32_t w) { return pack2(phi(lo16(w)), phi(hi16(w))); }

// Byte offset of the 16-byte unit `u` of row `r` in the two swizzles.
__device__ __forceinline__ uint32_t sw64(int r, int u) { return (uint32_t)(r * 64 + ((u ^ ((r >> 1) & 3)) << 4)); }
__device__ __forceinline__ uint32_t sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// phi in place over a [128 x 32] tile by NT threads; rows >= `valid` become
// 0 if `zero_tail`.
template <int NT = kThreads>
__device__ __forceinline__ void phi_tile(uint8_t *t, int valid, bool zero_tail) {
#pragma unroll
  for (int it = 0; it < 512 / NT; ++it) {
    const int g = it * NT + (int)threadIdx.x;  // 16-byte unit; its row is g / 4
    uint4 *p = reinterpret_cast<uint4 *>(t + 16 * g);
    uint4 x = *p;
    if (zero_tail && (g >> 2) >= valid) {
      x = make_uint4(0u, 0u, 0u, 0u);
    } else {
      x.x = phi2(x.x), x.y = phi2(x.y), x.z = phi2(x.z), x.w = phi2(x.w);
    }
    *p = x;
  }
}
__device__ __forceinline__ void get_row64(const uint8_t *t, int r, float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const uint4 x = *reinterpret_cast<const uint4 *>(t + sw64(r, u));
    v[8 * u + 0] = lo16(x.x), v[8 * u + 1] = hi16(x.x), v[8 * u + 2] = lo16(x.y), v[8 * u + 3] = hi16(x.y);
    v[8 * u + 4] = lo16(x.z), v[8 * u + 5] = hi16(x.z), v[8 * u + 6] = lo16(x.w), v[8 * u + 7] = hi16(x.w);
  }
}
__device__ __forceinline__ void put_row64(uint8_t *t, int r, const float (&v)[32]) {
#pragma unroll
  for (int u = 0; u < 4; ++u)
    *reinterpret_cast<uint4 *>(t + sw64(r, u)) =
        make_uint4(pack2(v[8 * u], v[8 * u + 1]), pack2(v[8 * u + 2], v[8 * u + 3]),
                   pack2(v[8 * u + 4], v[8 * u + 5]), pack2(v[8 * u + 6], v[8 * u + 7]));
}
// 32 columns (block b of 4) of row r of a [128 x 128] score tile.
__device__ __forceinline__ void put_row128(uint8_t *t, int r, int b, const float (&v)[32]) {
  uint8_t *half = t + kPhalf * (b >> 1);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4 *>(half + sw128(r, (b & 1) * 4 + q)) =
        make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                   pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
}
// A [32 x 32] float32 chunk state (row-major) into a bf16 64-byte-swizzle tile.
__device__ __forceinline__ void put_state_tile(uint8_t *t, const float *src, int tid) {
  const int d = tid >> 2, u = tid & 3;  // one warpgroup: tid in 0..127
  const float4 a = *reinterpret_cast<const float4 *>(src + d * kD + 8 * u);
  const float4 b = *reinterpret_cast<const float4 *>(src + d * kD + 8 * u + 4);
  *reinterpret_cast<uint4 *>(t + sw64(d, u)) = make_uint4(pack2(a.x, a.y), pack2(a.z, a.w), pack2(b.x, b.y),
                                                          pack2(b.z, b.w));
}

// ------------------------------------------------------------- control ---
struct Ctl {
  uint64_t bar[2];  // [0] TMA loads, [1] MMA completions
  uint32_t tmem;
  int ok;                    // no wait gave up
  int fail_bar, fail_parity; // the wait that gave up
};
__device__ __forceinline__ void ctl_setup(Ctl *ctl, uint32_t ncols) {
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&ctl->bar[0]), 1);
    mbar_init(smem_addr(&ctl->bar[1]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    ctl->ok = 1;
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_addr(&ctl->tmem), ncols);
    tmem_relinquish();
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
}
// Bounded wait by every thread; a wait that gives up records WKV_ERR_TIMEOUT
// and the CTA skips the rest of its work (the result is then invalid).
__device__ __forceinline__ bool ctl_wait(Ctl *ctl, int which, uint32_t parity, const LaArgs &a) {
  const bool ok = mbar_wait(smem_addr(&ctl->bar[which]), parity, a.budget_ns, nullptr);
  if (!ok) {
    atomicCAS(&a.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    ctl->ok = 0;
    ctl->fail_bar = which;
    ctl->fail_parity = (int)parity;
  }
  return __syncthreads_and(ok) != 0;
}
// End of the CTA: after a wait that gave up, wait once more (bounded) for the
// operation it was waiting for (the loads or the MMAs still in flight), then
// free the tensor memory.
__device__ __forceinline__ void ctl_finish(Ctl *ctl, uint32_t ncols, const LaArgs &a) {
  if (!ctl->ok) mbar_wait(smem_addr(&ctl->bar[ctl->fail_bar]), (uint32_t)ctl->fail_parity, a.budget_ns, nullptr);
  tc_before_sync();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_after_sync();
    tmem_dealloc(ctl->tmem, ncols);
  }
}
__device__ __forceinline__ uint8_t *align1k(uint8_t *p) {
  const uint32_t s = smem_addr(p);
  return p + (((s + 1023u) & ~1023u) - s);
}

// ------------------------------------------------------------- kernels ---
// Chunk states: phi(K)^T V (32 x 32) and phi(K)^T 1 (32) of every chunk,
// each as one MMA chain with M = 128 (rows 32..127 of its A operand are
// other tiles' bytes and their results are not read) and N = 48
// (B = [V | ones]).  Persistent: CTA g takes chunks g, g + G, ... and keeps
// two chunks' loads in flight (a stage is refilled as soon as its MMAs are
// complete).  Shared memory: stages (phi(K), V) at 0 and 16K, the ones tile
// at 32K; the spare rows of stage 1's A operand reach to 48K.
constexpr uint32_t kSStage = 2 * kTile, kSOnes = 2 * kSStage;
__global__ void __launch_bounds__(kThreads) la_state_kernel(const __grid_constant__ CUtensorMap kmap,
                                                            const __grid_constant__ CUtensorMap vmap, LaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_ld[2], bar_mma;
  __shared__ uint32_t tmem_s;
  uint8_t *sm = align1k(smem_raw);
  const uint32_t s0 = smem_addr(sm);
  const int64_t total = a.BH * a.nch;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar_ld[0]), 1);
    mbar_init(smem_addr(&bar_ld[1]), 1);
    mbar_init(smem_addr(&bar_mma), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(&tmem_s), 64);
    tmem_relinquish();
  }
  {
    uint4 *o = reinterpret_cast<uint4 *>(sm + kSOnes);
    for (int g = threadIdx.x; g < (int)(kTile / 16); g += kThreads)
      o[g] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // bf16 1.0
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = tmem_s;
  const uint64_t pol = l2_policy_evict_last();  // read again by the output kernel
  auto issue = [&](int64_t idx, int st) {
    const int h = (int)(idx / a.nch), c = (int)(idx % a.nch);
    const uint32_t dst = s0 + st * kSStage, bar = smem_addr(&bar_ld[st]);
    mbar_expect_tx(bar, 2 * kTile);
    tma_load_3d(dst, &kmap, 0, c * kL, h, bar, pol);
    tma_load_3d(dst + kTile, &vmap, 0, c * kL, h, bar, pol);
  };
  int64_t issued = 0;
  if (threadIdx.x == 0) {
    for (int st = 0; st < 2; ++st)
      if ((int64_t)blockIdx.x + (int64_t)st * gridDim.x < total) {
        issue((int64_t)blockIdx.x + (int64_t)st * gridDim.x, st);
        ++issued;
      }
  }
  uint32_t mma_phase = 0;
  int it = 0;
  bool failed = false, mma_pending = false;  // uniform over the CTA
  for (int64_t idx = blockIdx.x; idx < total; idx += gridDim.x, ++it) {
    const int st = it & 1;
    const int h = (int)(idx / a.nch), c = (int)(idx % a.nch);
    const int64_t rem = a.N - (int64_t)c * kL;
    const int valid = rem < kL ? (int)rem : kL;
    const uint32_t ak = s0 + st * kSStage, av = ak + kTile;
    failed = !__syncthreads_and(mbar_wait(smem_addr(&bar_ld[st]), (uint32_t)(it >> 1) & 1u, a.budget_ns, nullptr));
    if (failed) break;
    phi_tile<kThreads>(sm + st * kSStage, valid, true);
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_after_sync();
      constexpr uint32_t id = idesc(128, 48, true, true);
      const uint32_t ones_off = s0 + kSOnes - av;
#pragma unroll
      for (int k16 = 0; k16 < kL / 16; ++k16)
        mma(tm, mnmaj64(ak, k16, kTile), mnmaj64(av, k16, ones_off), id, k16 > 0);
      mma_commit(smem_addr(&bar_mma));
    }
    mma_pending = true;
    failed = !__syncthreads_and(mbar_wait(smem_addr(&bar_mma), mma_phase, a.budget_ns, nullptr));
    if (failed) break;
    mma_pending = false;
    mma_phase ^= 1u;
    tc_after_sync();
    if (threadIdx.x == 0) {  // this stage's tiles are consumed: load the chunk two ahead into it
      const int64_t nxt = idx + 2 * (int64_t)gridDim.x;
      if (nxt < total) {
        issue(nxt, st);
        ++issued;
      }
    }
    if (warp == 0) {
      float sv[32];
      tmem_ld32(tm, sv);
      const float z = tmem_ld1(tm + 32u);
      float *r = a.rec + ((int64_t)h * a.nch + c) * kRec;
      float4 *row = reinterpret_cast<float4 *>(r + threadIdx.x * kD);
#pragma unroll
      for (int q = 0; q < 8; ++q) row[q] = make_float4(sv[4 * q], sv[4 * q + 1], sv[4 * q + 2], sv[4 * q + 3]);
      r[kDM + threadIdx.x] = z;
    }
    tc_before_sync();
    __syncthreads();  // the accumulator is read before the next chunk's MMAs overwrite it
  }
  if (failed && threadIdx.x == 0) {
    atomicCAS(&a.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
    if (mma_pending) mbar_wait(smem_addr(&bar_mma), mma_phase, a.budget_ns, nullptr);
    for (int64_t m = it; m < issued; ++m)
      mbar_wait(smem_addr(&bar_ld[m & 1]), (uint32_t)(m >> 1) & 1u, a.budget_ns, nullptr);
  }
  tc_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_after_sync();
    tmem_dealloc(tm, 64);
  }
}

// Exclusive prefix (or, reversed, suffix) of the chunk states of every head,
// in place, in chunk order; the totals go to `total` ([BH][32][32] then
// [BH][32]) when it is given.
__global__ void la_scan_kernel(float *rec, int64_t BH, int nch, int reverse, float *total) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= BH * kRec) return;
  const int64_t h = e / kRec;
  const int f = (int)(e % kRec);
  float *base = rec + h * nch * kRec + f;
  float run = 0.f;
  // 16 chunks at a time: their loads are independent, so they are all in
  // flight together; the running sum then goes through them in order
  constexpr int kBatch = 16;
  for (int s0 = 0; s0 < nch; s0 += kBatch) {
    float x[kBatch];
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int s = s0 + t;
      x[t] = s < nch ? base[(int64_t)(reverse ? nch - 1 - s : s) * kRec] : 0.f;
    }
#pragma unroll
    for (int t = 0; t < kBatch; ++t) {
      const int s = s0 + t;
      if (s < nch) {
        base[(int64_t)(reverse ? nch - 1 - s : s) * kRec] = run;
        run += x[t];
      }
    }
  }
  if (total) {
    if (f < kDM)
      total[h * kDM + f] = run;
    else
      total[BH * kDM + h * kD + (f - kDM)] = run;
  }
}

// Masked scores of the thread's row (its warp holds rows 32w..32w+31) into
// a [128 x 128] bf16 tile, for two of the four 32-column blocks: warpgroup 0
// takes blocks 0 and 3, warpgroup 1 blocks 1 and 2 (the causal mask gives
// both about the same work).  Column blocks left of the warp's diagonal
// block need no mask, those right of it are zero (their TMEM columns are
// not read).
template <bool ADD = false>
__device__ __forceinline__ void causal_scores_to_tile(uint32_t tm_row, uint8_t *tile, int i, int wg,
                                                      float add = 0.f) {
  const int w = i >> 5;
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    const int b = wg == 0 ? 3 * q : 1 + q;
    float v[32];
    if (b <= w) {
      tmem_ld32(tm_row + 32u * b, v);
      if (ADD) {
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = (b < w || 32 * b + r <= i) ? v[r] + add : 0.f;
      } else if (b == w) {
#pragma unroll
        for (int r = 0; r < 32; ++r) v[r] = (32 * b + r <= i) ? v[r] : 0.f;
      }
    } else {
#pragma unroll
      for (int r = 0; r < 32; ++r) v[r] = 0.f;
    }
    put_row128(tile, i, b, v);
  }
}

// Forward outputs.  Persistent: CTA g takes chunks g, g + G, ... (G = the
// grid) and double-buffers their Q, K, V tiles, so a chunk's loads run
// while the one before it is computed.  Per chunk: scores phi(Q) phi(K)^T
// (2 MMAs), the masked score tile, then numerators and denominator in one
// accumulator, A [V | 1] + phi(Q) [S_prev | Z_prev] (10 MMAs, N = 48:
// column 32 is the denominator), and out = numerators / denominator; each
// row's denominator also goes to the workspace for the saved-state backward.
// Shared memory: two stages of (phi(Q), phi(K) then the output tile, V) at
// 0 and 24K, a ones tile at 48K, S_prev and Z_prev (bf16) at 56K and 58K,
// the score tile at 64K (32K bytes), and per stage the chunk's float32
// (S_prev, Z_prev) record, copied in with its tiles, at 96K.
constexpr uint32_t kFStage = 3 * kTile, kFOnes = 2 * kFStage, kFS = kFOnes + kTile, kFZ = kFS + kStile,
                   kFP = 8 * kTile, kFRec = 12 * kTile, kRecBytes = kRec * 4;
static_assert(kRecBytes % 128 == 0, "records stay 128-byte aligned in shared memory");
__global__ void __launch_bounds__(kThreads) la_fwd_kernel(const __grid_constant__ CUtensorMap qmap,
                                                          const __grid_constant__ CUtensorMap kmap,
                                                          const __grid_constant__ CUtensorMap vmap,
                                                          const __grid_constant__ CUtensorMap omap, LaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_ld[2], bar_mma;
  __shared__ uint32_t tmem_s;
  uint8_t *sm = align1k(smem_raw);
  const uint32_t s0 = smem_addr(sm);
  const int64_t total = a.BH * a.nch;
  // 8 warps: row i = thread % 128 (warp w % 4 reads TMEM lanes 32(w % 4)..);
  // the two warpgroups split the epilogues' columns
  const int i = threadIdx.x & 127, wg = threadIdx.x >> 7, warp = threadIdx.x >> 5;
  const uint32_t lane_off = (uint32_t)(i & ~31) << 16;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar_ld[0]), 1);
    mbar_init(smem_addr(&bar_ld[1]), 1);
    mbar_init(smem_addr(&bar_mma), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    tmem_alloc(smem_addr(&tmem_s), 128);
    tmem_relinquish();
  }
  {
    uint4 *o = reinterpret_cast<uint4 *>(sm + kFOnes);
    for (int g = threadIdx.x; g < (int)(kTile / 16); g += kThreads)
      o[g] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // bf16 1.0
  }
  tc_before_sync();
  __syncthreads();
  tc_after_sync();
  const uint32_t tm = tmem_s;
  const uint64_t pol = l2_policy_evict_first();
  auto issue = [&](int64_t idx, int st) {
    const int h = (int)(idx / a.nch), c = (int)(idx % a.nch);
    const uint32_t dst = s0 + st * kFStage, bar = smem_addr(&bar_ld[st]);
    mbar_expect_tx(bar, 3 * kTile + kRecBytes);
    tma_load_3d(dst, &qmap, 0, c * kL, h, bar, pol);
    tma_load_3d(dst + kTile, &kmap, 0, c * kL, h, bar, pol);
    tma_load_3d(dst + 2 * kTile, &vmap, 0, c * kL, h, bar, pol);
    bulk_load(s0 + kFRec + st * kRecBytes, a.rec + ((int64_t)h * a.nch + c) * kRec, kRecBytes, bar);
  };
  int64_t issued = 0;  // chunks of this CTA whose loads were issued (thread 0)
  if (threadIdx.x == 0) {
    for (int st = 0; st < 2; ++st)
      if ((int64_t)blockIdx.x + (int64_t)st * gridDim.x < total) {
        issue((int64_t)blockIdx.x + (int64_t)st * gridDim.x, st);
        ++issued;
      }
  }
  uint32_t mma_phase = 0;
  int it = 0;
  bool failed = false, mma_pending = false;  // uniform over the CTA
  for (int64_t idx = blockIdx.x; idx < total; idx += gridDim.x, ++it) {
    const int st = it & 1;
    const int h = (int)(idx / a.nch), c = (int)(idx % a.nch);
    uint8_t *tq = sm + st * kFStage, *tk = tq + kTile;
    const uint32_t aq = s0 + st * kFStage, ak = aq + kTile, av = aq + 2 * kTile;
    failed = !__syncthreads_and(mbar_wait(smem_addr(&bar_ld[st]), (uint32_t)(it >> 1) & 1u, a.budget_ns, nullptr));
    if (failed) break;
    // S_prev and Z_prev of this chunk, from the copy that came with its tiles,
    // as bf16 operand tiles (the previous chunk's MMAs are complete)
    const float *prev = reinterpret_cast<const float *>(sm + kFRec + st * kRecBytes);
    if (threadIdx.x < kWarpgroup) put_state_tile(sm + kFS, prev, threadIdx.x);
    if (threadIdx.x >= kWarpgroup && threadIdx.x < kWarpgroup + kD) {
      const int d = threadIdx.x - kWarpgroup;
      const uint32_t zz = pack2(prev[kDM + d], prev[kDM + d]);
      const uint4 x = make_uint4(zz, zz, zz, zz);
      uint4 *row = reinterpret_cast<uint4 *>(sm + kFZ + 64 * d);
      row[0] = x, row[1] = x, row[2] = x, row[3] = x;
    }
    phi_tile<kThreads>(tq, kL, false);
    phi_tile<kThreads>(tk, kL, false);
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {  // scores phi(Q) phi(K)^T
      tc_after_sync();
      constexpr uint32_t id = idesc(128, 128, false, false);
      mma(tm, kmaj64(aq, 0), kmaj64(ak, 0), id, false);
      mma(tm, kmaj64(aq, 1), kmaj64(ak, 1), id, true);
      mma_commit(smem_addr(&bar_mma));
      // the previous chunk's stage is free once its output store has read
      // it: load the chunk after this one there
      const int64_t nxt = idx + gridDim.x;
      if (it >= 1 && nxt < total) {
        bulk_wait_read_all();
        issue(nxt, st ^ 1);
        ++issued;
      }
    }
    mma_pending = true;
    failed = !__syncthreads_and(mbar_wait(smem_addr(&bar_mma), mma_phase, a.budget_ns, nullptr));
    if (failed) break;
    mma_pending = false;
    mma_phase ^= 1u;
    tc_after_sync();
    causal_scores_to_tile(tm + lane_off, sm + kFP, i, wg);
    tc_before_sync();
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {  // A [V | 1] + phi(Q) [S_prev | Z_prev]
      tc_after_sync();
      constexpr uint32_t id = idesc(128, 48, false, true);
      const uint32_t ones_off = s0 + kFOnes - av;
#pragma unroll
      for (int k16 = 0; k16 < kL / 16; ++k16) mma(tm, kmaj128(s0 + kFP, k16), mnmaj64(av, k16, ones_off), id, k16 > 0);
      mma(tm, kmaj64(aq, 0), mnmaj64(s0 + kFS, 0, kStile), id, true);
      mma(tm, kmaj64(aq, 1), mnmaj64(s0 + kFS, 1, kStile), id, true);
      mma_commit(smem_addr(&bar_mma));
    }
    mma_pending = true;
    failed = !__syncthreads_and(mbar_wait(smem_addr(&bar_mma), mma_phase, a.budget_ns, nullptr));
    if (failed) break;
    mma_pending = false;
    mma_phase ^= 1u;
    tc_after_sync();
    float o[16];  // this warpgroup's 16 of the 32 output columns
    tmem_ld16(tm + lane_off + 16u * wg, o);
    const float den = tmem_ld1(tm + lane_off + 32u);
    const float inv = 1.f / den;
    if (wg == 0) a.den[((int64_t)h * a.nch + c) * kL + i] = den;
#pragma unroll
    for (int u = 0; u < 2; ++u)  // phi(K) is no longer read: the output goes there
      *reinterpret_cast<uint4 *>(tk + sw64(i, 2 * wg + u)) =
          make_uint4(pack2(o[8 * u] * inv, o[8 * u + 1] * inv), pack2(o[8 * u + 2] * inv, o[8 * u + 3] * inv),
                     pack2(o[8 * u + 4] * inv, o[8 * u + 5] * inv), pack2(o[8 * u + 6] * inv, o[8 * u + 7] * inv));
    tc_before_sync();
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tma_store_3d(&omap, 0, c * kL, h, ak);
      bulk_commit();
    }
  }
  if (failed) {
    // a wait gave up (WKV_ERR_TIMEOUT): wait once more, bounded, for what is
    // still in flight before the shared and tensor memory are released
    if (threadIdx.x == 0) {
      atomicCAS(&a.hdr->status, 0, -5 /* WKV_ERR_TIMEOUT */);
      if (mma_pending) mbar_wait(smem_addr(&bar_mma), mma_phase, a.budget_ns, nullptr);
      for (int64_t m = it; m < issued; ++m)
        mbar_wait(smem_addr(&bar_ld[m & 1]), (uint32_t)(m >> 1) & 1u, a.budget_ns, nullptr);
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();
  tc_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_after_sync();
    tmem_dealloc(tm, 128);
  }
}

// Backward, first part, of one chunk: numerators and denominator again (as
// the forward: A [V | 1] + phi(Q) [S_prev | Z_prev]), gnum = G / den (bf16,
// to the workspace) and gden = -rowsum(G * out) / den (float32, to the
// workspace), and the chunk's reverse state phi(Q)^T [gnum | gden].  Two
// warpgroups: row i = thread % 128, the epilogues' columns split between
// them.  Shared memory: phi(Q) 0, gnum 8K, gden (each row filled with its
// value) 16K, phi(K) 24K, V 32K, G 40K, S_prev 48K, Z_prev 50K, scores 64K
// (32K bytes), ones 96K.
constexpr uint32_t kPOnes = 12 * kTile;
__global__ void __launch_bounds__(kThreads) la_bwd_prep_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap,
                                                                  const __grid_constant__ CUtensorMap gmap,
                                                                  const __grid_constant__ CUtensorMap nmap, LaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  __shared__ float gpart[kL];  // warpgroup 1's part of rowsum(G * out)
  uint8_t *sm = align1k(smem_raw);
  const uint32_t s0 = smem_addr(sm);
  uint8_t *tq = sm, *tn = sm + kTile, *tg_den = sm + 2 * kTile, *tk = sm + 3 * kTile, *tgo = sm + 5 * kTile,
          *ts = sm + 6 * kTile, *tz = sm + 6 * kTile + kStile, *tp = sm + 8 * kTile;
  const uint32_t aq = s0, an = s0 + kTile, ak = s0 + 3 * kTile, av = s0 + 4 * kTile, ag = s0 + 5 * kTile,
                 as = s0 + 6 * kTile, ap = s0 + 8 * kTile;
  const int h = (int)(blockIdx.x / a.nch), c = (int)(blockIdx.x % a.nch);
  const int i = threadIdx.x & 127, wg = threadIdx.x >> 7;
  const int64_t rem = a.N - (int64_t)c * kL;
  const int valid = rem < kL ? (int)rem : kL;
  const uint32_t lane_off = (uint32_t)(i & ~31) << 16;
  ctl_setup(&ctl, 128);
  const uint32_t bl = smem_addr(&ctl.bar[0]), bm = smem_addr(&ctl.bar[1]);
  if (threadIdx.x == 0) {
    const uint64_t pol = l2_policy_evict_last();  // read again by the gradient kernel
    mbar_expect_tx(bl, 4 * kTile);
    tma_load_3d(aq, &qmap, 0, c * kL, h, bl, pol);
    tma_load_3d(ak, &kmap, 0, c * kL, h, bl, pol);
    tma_load_3d(av, &vmap, 0, c * kL, h, bl, pol);
    tma_load_3d(ag, &gmap, 0, c * kL, h, bl, l2_policy_evict_first());
  }
  {
    uint4 *o = reinterpret_cast<uint4 *>(sm + kPOnes);
    for (int g = threadIdx.x; g < (int)(kTile / 16); g += kThreads)
      o[g] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);  // bf16 1.0
  }
  const float *prev = a.rec + ((int64_t)h * a.nch + c) * kRec;
  if (wg == 0) put_state_tile(ts, prev, i);
  if (wg == 1 && i < kD) {  // Z_prev[d] across row d
    const uint32_t zz = pack2(prev[kDM + i], prev[kDM + i]);
    const uint4 x = make_uint4(zz, zz, zz, zz);
    uint4 *row = reinterpret_cast<uint4 *>(tz + 64 * i);
    row[0] = x, row[1] = x, row[2] = x, row[3] = x;
  }
  if (ctl_wait(&ctl, 0, 0, a)) {
    phi_tile<kThreads>(tq, kL, false);
    phi_tile<kThreads>(tk, kL, false);
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tc_after_sync();
      constexpr uint32_t id = idesc(128, 128, false, false);
      mma(ctl.tmem, kmaj64(aq, 0), kmaj64(ak, 0), id, false);
      mma(ctl.tmem, kmaj64(aq, 1), kmaj64(ak, 1), id, true);
      mma_commit(bm);
    }
    if (ctl_wait(&ctl, 1, 0, a)) {
      tc_after_sync();
      causal_scores_to_tile(ctl.tmem + lane_off, tp, i, wg);
      tc_before_sync();
      fence_proxy_async_smem();
      __syncthreads();
      if (threadIdx.x == 0) {  // A [V | 1] + phi(Q) [S_prev | Z_prev]: column 32 is den
        tc_after_sync();
        constexpr uint32_t id = idesc(128, 48, false, true);
#pragma unroll
        for (int k16 = 0; k16 < kL / 16; ++k16)
          mma(ctl.tmem, kmaj128(ap, k16), mnmaj64(av, k16, s0 + kPOnes - av), id, k16 > 0);
        mma(ctl.tmem, kmaj64(aq, 0), mnmaj64(as, 0, kStile), id, true);
        mma(ctl.tmem, kmaj64(aq, 1), mnmaj64(as, 1, kStile), id, true);
        mma_commit(bm);
      }
      if (ctl_wait(&ctl, 1, 1, a)) {
        tc_after_sync();
        float o[16], g[16];  // this warpgroup's 16 columns
        tmem_ld16(ctl.tmem + lane_off + 16u * wg, o);
        const float inv = 1.f / tmem_ld1(ctl.tmem + lane_off + 32u);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const uint4 x = *reinterpret_cast<const uint4 *>(tgo + sw64(i, 2 * wg + u));
          g[8 * u + 0] = lo16(x.x), g[8 * u + 1] = hi16(x.x), g[8 * u + 2] = lo16(x.y), g[8 * u + 3] = hi16(x.y);
          g[8 * u + 4] = lo16(x.z), g[8 * u + 5] = hi16(x.z), g[8 * u + 6] = lo16(x.w), g[8 * u + 7] = hi16(x.w);
        }
        float go = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
          go = fmaf(g[m], o[m] * inv, go);
          g[m] *= inv;  // gnum
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
          *reinterpret_cast<uint4 *>(tn + sw64(i, 2 * wg + u)) =
              make_uint4(pack2(g[8 * u], g[8 * u + 1]), pack2(g[8 * u + 2], g[8 * u + 3]),
                         pack2(g[8 * u + 4], g[8 * u + 5]), pack2(g[8 * u + 6], g[8 * u + 7]));
        if (wg == 1) gpart[i] = go;
        __syncthreads();
        if (wg == 0) {
          const float gden = -(go + gpart[i]) * inv;
          const uint32_t w = pack2(gden, gden);
          const uint4 x = make_uint4(w, w, w, w);
#pragma unroll
          for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4 *>(tg_den + 64 * i + 16 * u) = x;
          if (i < valid) a.gden[(int64_t)h * a.N + (int64_t)c * kL + i] = gden;
        }
        tc_before_sync();
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
          tma_store_3d(&nmap, 0, c * kL, h, an);
          bulk_commit();
          // reverse state phi(Q)^T [gnum | gden]: M = 128 over the tiles at
          // 0, 8K, 16K, 24K (rows 32..127 unused), N = 48 over gnum, gden
          tc_after_sync();
          constexpr uint32_t id3 = idesc(128, 48, true, true);
#pragma unroll
          for (int k16 = 0; k16 < kL / 16; ++k16)
            mma(ctl.tmem, mnmaj64(aq, k16, kTile), mnmaj64(an, k16, kTile), id3, k16 > 0);
          mma_commit(bm);
        }
        if (ctl_wait(&ctl, 1, 0, a)) {
          tc_after_sync();
          if (threadIdx.x < 32) {
            float rv[32];
            tmem_ld32(ctl.tmem, rv);
            const float uz = tmem_ld1(ctl.tmem + 32u);
            float *r = a.rec_r + ((int64_t)h * a.nch + c) * kRec;
            float4 *row = reinterpret_cast<float4 *>(r + threadIdx.x * kD);
#pragma unroll
            for (int q = 0; q < 8; ++q) row[q] = make_float4(rv[4 * q], rv[4 * q + 1], rv[4 * q + 2], rv[4 * q + 3]);
            r[kDM + threadIdx.x] = uz;
          }
        }
        if (threadIdx.x == 0) bulk_wait_all();
      }
    }
  }
  ctl_finish(&ctl, 128, a);
}

// Backward, first part, from the forward's saved state: the forward's
// output and denominators give gnum = G / den (bf16, to the workspace) and
// gden = -rowsum(G * out) / den (float32, to the workspace) directly, and
// one MMA chain the chunk's reverse state phi(Q)^T [gnum | gden].  Shared
// memory: phi(Q) 0, gnum 8K, gden (rows filled with their value) 16K, G 24K
// (also the spare rows of the MMA's A operand), out 32K, den 40K.
__global__ void __launch_bounds__(kThreads) la_bwd_prep_saved_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                     const __grid_constant__ CUtensorMap gmap,
                                                                     const __grid_constant__ CUtensorMap omap,
                                                                     const __grid_constant__ CUtensorMap nmap,
                                                                     LaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  __shared__ float gpart[kL];  // warpgroup 1's part of rowsum(G * out)
  uint8_t *sm = align1k(smem_raw);
  const uint32_t s0 = smem_addr(sm);
  uint8_t *tq = sm, *tn = sm + kTile, *tg_den = sm + 2 * kTile, *tgo = sm + 3 * kTile, *tout = sm + 4 * kTile;
  const float *dens = reinterpret_cast<const float *>(sm + 5 * kTile);
  const uint32_t aq = s0, an = s0 + kTile;
  const int h = (int)(blockIdx.x / a.nch), c = (int)(blockIdx.x % a.nch);
  const int i = threadIdx.x & 127, wg = threadIdx.x >> 7;
  const int64_t rem = a.N - (int64_t)c * kL;
  const int valid = rem < kL ? (int)rem : kL;
  ctl_setup(&ctl, 64);
  const uint32_t bl = smem_addr(&ctl.bar[0]), bm = smem_addr(&ctl.bar[1]);
  if (threadIdx.x == 0) {
    const uint64_t pol = l2_policy_evict_first();
    mbar_expect_tx(bl, 3 * kTile + kL * 4);
    tma_load_3d(aq, &qmap, 0, c * kL, h, bl, l2_policy_evict_last());  // read again by the gradient kernel
    tma_load_3d(s0 + 3 * kTile, &gmap, 0, c * kL, h, bl, pol);
    tma_load_3d(s0 + 4 * kTile, &omap, 0, c * kL, h, bl, pol);
    bulk_load(s0 + 5 * kTile, a.den + ((int64_t)h * a.nch + c) * kL, kL * 4, bl);
  }
  if (ctl_wait(&ctl, 0, 0, a)) {
    phi_tile<kThreads>(tq, kL, false);
    float g[16], o[16];  // this warpgroup's 16 columns of G and out
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 x = *reinterpret_cast<const uint4 *>(tgo + sw64(i, 2 * wg + u));
      const uint4 y = *reinterpret_cast<const uint4 *>(tout + sw64(i, 2 * wg + u));
      g[8 * u + 0] = lo16(x.x), g[8 * u + 1] = hi16(x.x), g[8 * u + 2] = lo16(x.y), g[8 * u + 3] = hi16(x.y);
      g[8 * u + 4] = lo16(x.z), g[8 * u + 5] = hi16(x.z), g[8 * u + 6] = lo16(x.w), g[8 * u + 7] = hi16(x.w);
      o[8 * u + 0] = lo16(y.x), o[8 * u + 1] = hi16(y.x), o[8 * u + 2] = lo16(y.y), o[8 * u + 3] = hi16(y.y);
      o[8 * u + 4] = lo16(y.z), o[8 * u + 5] = hi16(y.z), o[8 * u + 6] = lo16(y.w), o[8 * u + 7] = hi16(y.w);
    }
    const float inv = 1.f / dens[i];
    float go = 0.f;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      go = fmaf(g[m], o[m], go);
      g[m] *= inv;  // gnum
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
      *reinterpret_cast<uint4 *>(tn + sw64(i, 2 * wg + u)) =
          make_uint4(pack2(g[8 * u], g[8 * u + 1]), pack2(g[8 * u + 2], g[8 * u + 3]),
                     pack2(g[8 * u + 4], g[8 * u + 5]), pack2(g[8 * u + 6], g[8 * u + 7]));
    if (wg == 1) gpart[i] = go;
    __syncthreads();
    if (wg == 0) {
      const float gden = -(go + gpart[i]) * inv;
      const uint32_t w = pack2(gden, gden);
      const uint4 x = make_uint4(w, w, w, w);
#pragma unroll
      for (int u = 0; u < 4; ++u) *reinterpret_cast<uint4 *>(tg_den + 64 * i + 16 * u) = x;
      if (i < valid) a.gden[(int64_t)h * a.N + (int64_t)c * kL + i] = gden;
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      tma_store_3d(&nmap, 0, c * kL, h, an);
      bulk_commit();
      // reverse state phi(Q)^T [gnum | gden]: M = 128 over the tiles at
      // 0, 8K, 16K, 24K (rows 32..127 unused), N = 48 over gnum, gden
      tc_after_sync();
      constexpr uint32_t id3 = idesc(128, 48, true, true);
#pragma unroll
      for (int k16 = 0; k16 < kL / 16; ++k16) mma(ctl.tmem, mnmaj64(aq, k16, kTile), mnmaj64(an, k16, kTile), id3, k16 > 0);
      mma_commit(bm);
    }
    if (ctl_wait(&ctl, 1, 0, a)) {
      tc_after_sync();
      if (threadIdx.x < 32) {
        float rv[32];
        tmem_ld32(ctl.tmem, rv);
        const float uz = tmem_ld1(ctl.tmem + 32u);
        float *r = a.rec_r + ((int64_t)h * a.nch + c) * kRec;
        float4 *row = reinterpret_cast<float4 *>(r + threadIdx.x * kD);
#pragma unroll
        for (int q = 0; q < 8; ++q) row[q] = make_float4(rv[4 * q], rv[4 * q + 1], rv[4 * q + 2], rv[4 * q + 3]);
        r[kDM + threadIdx.x] = uz;
      }
    }
    if (threadIdx.x == 0) bulk_wait_all();
  }
  ctl_finish(&ctl, 64, a);
}

// Backward, gradients of one chunk.  One score tile and 128 tensor-memory
// columns, so that three CTAs fit per SM (registers capped to match): the
// masked A feeds A^T gnum first, whose result waits in registers, and is
// then overwritten by P = tril(gnum V^T + gden 1^T).  Two warpgroups: row
// i = thread % 128, the epilogues' columns split between them.  Shared
// memory: phi(Q) 0, phi(K) 8K, V 16K, gnum 24K, S_prev 32K, U_next 34K, the
// score tile 36K (32K bytes); the output tiles reuse 36K, 44K, 52K.
__global__ void __launch_bounds__(kThreads, 3) la_bwd_kernel(const __grid_constant__ CUtensorMap qmap,
                                                           const __grid_constant__ CUtensorMap kmap,
                                                           const __grid_constant__ CUtensorMap vmap,
                                                           const __grid_constant__ CUtensorMap nmap,
                                                           const __grid_constant__ CUtensorMap dqmap,
                                                           const __grid_constant__ CUtensorMap dkmap,
                                                           const __grid_constant__ CUtensorMap dvmap, LaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ Ctl ctl;
  __shared__ float zprev[kD], unext[kD], gden_s[kL];
  uint8_t *sm = align1k(smem_raw);
  const uint32_t s0 = smem_addr(sm);
  constexpr uint32_t kT = 4 * kTile + 2 * kStile;  // the score tile (1024-aligned)
  uint8_t *tq = sm, *tk = sm + kTile, *ts = sm + 4 * kTile, *tu = sm + 4 * kTile + kStile, *tt = sm + kT;
  const uint32_t aq = s0, ak = s0 + kTile, av = s0 + 2 * kTile, an = s0 + 3 * kTile, as = s0 + 4 * kTile,
                 au = s0 + 4 * kTile + kStile, at = s0 + kT;
  const int h = (int)(blockIdx.x / a.nch), c = (int)(blockIdx.x % a.nch);
  const int i = threadIdx.x & 127, wg = threadIdx.x >> 7;
  const int64_t rem = a.N - (int64_t)c * kL;
  const int valid = rem < kL ? (int)rem : kL;
  const uint32_t lane_off = (uint32_t)(i & ~31) << 16;
  ctl_setup(&ctl, 128);
  const uint32_t bl = smem_addr(&ctl.bar[0]), bm = smem_addr(&ctl.bar[1]);
  if (threadIdx.x == 0) {
    const uint64_t pol = l2_policy_evict_first();
    mbar_expect_tx(bl, 4 * kTile);
    tma_load_3d(aq, &qmap, 0, c * kL, h, bl, pol);
    tma_load_3d(ak, &kmap, 0, c * kL, h, bl, pol);
    tma_load_3d(av, &vmap, 0, c * kL, h, bl, pol);
    tma_load_3d(an, &nmap, 0, c * kL, h, bl, pol);
  }
  const float *prev = a.rec + ((int64_t)h * a.nch + c) * kRec;
  const float *next = a.rec_r + ((int64_t)h * a.nch + c) * kRec;
  put_state_tile(wg == 0 ? ts : tu, wg == 0 ? prev : next, i);
  if (i < kD) (wg == 0 ? zprev : unext)[i] = (wg == 0 ? prev : next)[kDM + i];
  if (wg == 0) gden_s[i] = i < valid ? a.gden[(int64_t)h * a.N + (int64_t)c * kL + i] : 0.f;
  if (ctl_wait(&ctl, 0, 0, a)) {
    phi_tile<kThreads>(tq, kL, false);
    phi_tile<kThreads>(tk, kL, false);
    fence_proxy_async_smem();
    __syncthreads();
    constexpr uint32_t sq = idesc(128, 128, false, false), kk = idesc(128, 32, false, false),
                       kmn = idesc(128, 32, false, true), mnmn = idesc(128, 32, true, true);
    if (threadIdx.x == 0) {  // scores
      tc_after_sync();
      mma(ctl.tmem, kmaj64(aq, 0), kmaj64(ak, 0), sq, false);
      mma(ctl.tmem, kmaj64(aq, 1), kmaj64(ak, 1), sq, true);
      mma_commit(bm);
    }
    if (ctl_wait(&ctl, 1, 0, a)) {
      tc_after_sync();
      causal_scores_to_tile(ctl.tmem + lane_off, tt, i, wg);  // A
      tc_before_sync();
      fence_proxy_async_smem();
      __syncthreads();
      if (threadIdx.x == 0) {  // A^T gnum, dL/dV's first part, into columns 0..31
        tc_after_sync();
#pragma unroll
        for (int k16 = 0; k16 < kL / 16; ++k16)
          mma(ctl.tmem, mnmaj128(at, k16), mnmaj64(an, k16, kTile), mnmn, k16 > 0);
        mma_commit(bm);
      }
      if (ctl_wait(&ctl, 1, 1, a)) {
        tc_after_sync();
        float dv1[16];  // this warpgroup's 16 columns, kept until the end
        tmem_ld16(ctl.tmem + lane_off + 16u * wg, dv1);
        tc_before_sync();
        __syncthreads();
        if (threadIdx.x == 0) {  // gnum V^T
          tc_after_sync();
          mma(ctl.tmem, kmaj64(an, 0), kmaj64(av, 0), sq, false);
          mma(ctl.tmem, kmaj64(an, 1), kmaj64(av, 1), sq, true);
          mma_commit(bm);
        }
        if (ctl_wait(&ctl, 1, 0, a)) {
          tc_after_sync();
          causal_scores_to_tile<true>(ctl.tmem + lane_off, tt, i, wg, gden_s[i]);  // P over A
          tc_before_sync();
          fence_proxy_async_smem();
          __syncthreads();
          if (threadIdx.x == 0) {
            tc_after_sync();
            // dphi(Q) -> columns 0..31: P phi(K) + gnum S_prev^T
#pragma unroll
            for (int k16 = 0; k16 < kL / 16; ++k16) mma(ctl.tmem, kmaj128(at, k16), mnmaj64(ak, k16, kTile), kmn, k16 > 0);
            mma(ctl.tmem, kmaj64(an, 0), kmaj64(as, 0), kk, true);
            mma(ctl.tmem, kmaj64(an, 1), kmaj64(as, 1), kk, true);
            // dphi(K) -> columns 32..63: P^T phi(Q) + V U_next^T
#pragma unroll
            for (int k16 = 0; k16 < kL / 16; ++k16)
              mma(ctl.tmem + 32u, mnmaj128(at, k16), mnmaj64(aq, k16, kTile), mnmn, k16 > 0);
            mma(ctl.tmem + 32u, kmaj64(av, 0), kmaj64(au, 0), kk, true);
            mma(ctl.tmem + 32u, kmaj64(av, 1), kmaj64(au, 1), kk, true);
            // dL/dV's second part -> columns 64..95: phi(K) U_next
            mma(ctl.tmem + 64u, kmaj64(ak, 0), mnmaj64(au, 0, kTile), kmn, false);
            mma(ctl.tmem + 64u, kmaj64(ak, 1), mnmaj64(au, 1, kTile), kmn, true);
            mma_commit(bm);
          }
          if (ctl_wait(&ctl, 1, 1, a)) {
            tc_after_sync();
            float x[32], f[32];
            uint8_t *oq = tt, *ok = tt + kTile, *ov = tt + 2 * kTile;  // the score tile is no longer read
            tmem_ld32(ctl.tmem + lane_off + 32u * wg, x);
            get_row64(wg == 0 ? tq : tk, i, f);
            if (wg == 0) {
              const float gd = gden_s[i];
#pragma unroll
              for (int d = 0; d < kD; ++d) x[d] = fmaf(gd, zprev[d], x[d]) * fminf(f[d], 1.f);
            } else {
#pragma unroll
              for (int d = 0; d < kD; ++d) x[d] = (x[d] + unext[d]) * fminf(f[d], 1.f);
            }
            put_row64(wg == 0 ? oq : ok, i, x);
            float y[16];
            tmem_ld16(ctl.tmem + lane_off + 64u + 16u * wg, y);
#pragma unroll
            for (int u = 0; u < 2; ++u)
              *reinterpret_cast<uint4 *>(ov + sw64(i, 2 * wg + u)) = make_uint4(
                  pack2(y[8 * u] + dv1[8 * u], y[8 * u + 1] + dv1[8 * u + 1]),
                  pack2(y[8 * u + 2] + dv1[8 * u + 2], y[8 * u + 3] + dv1[8 * u + 3]),
                  pack2(y[8 * u + 4] + dv1[8 * u + 4], y[8 * u + 5] + dv1[8 * u + 5]),
                  pack2(y[8 * u + 6] + dv1[8 * u + 6], y[8 * u + 7] + dv1[8 * u + 7]));
            fence_proxy_async_smem();
            __syncthreads();
            if (threadIdx.x == 0) {
              tma_store_3d(&dqmap, 0, c * kL, h, at);
              tma_store_3d(&dkmap, 0, c * kL, h, at + kTile);
              tma_store_3d(&dvmap, 0, c * kL, h, at + 2 * kTile);
              bulk_commit();
              bulk_wait_all();
            }
          }
        }
      }
    }
  }
  ctl_finish(&ctl, 128, a);
}

// Shared-memory bytes of each kernel (tiles plus the 1 KB alignment slack).
constexpr int kStateSmem = 6 * kTile + 1024;             // 2 x (K, V), ones, spare rows
constexpr int kFwdSmem = 12 * kTile + 2 * kRecBytes + 1024;  // 2 x (Q, K, V), ones, S, Z | scores | 2 records
constexpr int kPrepSmem = 13 * kTile + 1024;             // Q, gnum, gden, K, V, G, S, Z (+pad) | scores | ones
constexpr int kBwdSmem = 8 * kTile + 2 * kStile + 1024;     // Q, K, V, gnum, S, U | one score tile
constexpr int kPrepSavedSmem = 5 * kTile + kL * 4 + 1024;  // Q, gnum, gden, G, out, den

}  // namespace la
}  // namespace wkv

// ---------------------------------------------------------------- host ---

namespace {
using namespace wkv;
using namespace wkv::la;

struct LaLayout {
  size_t rec, den, rec_r, gnum, gden, total;
};
bool la_layout(int op, int64_t BH, int64_t N, LaLayout *L) {
  if (BH < 1 || N < 0 || BH > (int64_t(1) << 31) || N > (int64_t(1) << 31) || BH * N >= (int64_t(1) << 31))
    return false;
  const int64_t nch = (N + kL - 1) / kL;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  size_t off = 256;  // header
  // The forward's regions come first and sit at the same offsets in both
  // layouts, so a backward-sized workspace can carry the forward's state
  // into linattn_backward_saved.
  L->rec = off;
  off = up(off + (size_t)BH * nch * kRec * 4);
  L->den = off;
  off = up(off + (size_t)BH * nch * kL * 4);
  L->rec_r = L->gnum = L->gden = 0;
  if (op == LINATTN_OP_BACKWARD) {
    L->rec_r = off;
    off = up(off + (size_t)BH * nch * kRec * 4);
    L->gnum = off;
    off = up(off + (size_t)BH * N * kD * 2);
    L->gden = off;
    off = up(off + (size_t)BH * N * 4);
  }
  L->total = off;
  return true;
}
bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Grid of a persistent kernel: one wave of resident CTAs, at most one per
// chunk.  Residency is counted from the shared memory per SM and the tensor
// memory each CTA allocates (512 columns per SM); the occupancy calculator
// does not know the latter.
int la_num_sms();
template <typename K>
int64_t persistent_grid(K kern, int smem, int tmem_cols, int64_t units) {
  int dev = 0, per_sm = 0, reserved = 0;
  cudaFuncAttributes fa{};
  int occ = 1;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) == cudaSuccess &&
      cudaFuncGetAttributes(&fa, (const void *)kern) == cudaSuccess)
    occ = per_sm / (smem + (int)fa.sharedSizeBytes + reserved);
  occ = std::max(1, std::min(occ, std::min(512 / tmem_cols, 2048 / kThreads)));
  return std::min<int64_t>(units, (int64_t)occ * la_num_sms());
}
template <typename K>
int prepare(K kern, int smem, int threads = kThreads) {
  int occ = 0;
  return blocks_per_sm((const void *)kern, threads, smem, &occ) == cudaSuccess && occ >= 1 ? 0 : -1;
}
int cuda_rc(cudaError_t e) { return e == cudaSuccess ? WKV_OK : WKV_ERR_CUDA; }
int la_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return n;
}
constexpr int64_t kBudgetNs = 1000000000;  // one second per bounded wait

int check_common(int64_t BH, int64_t N, int D, int M, void *ws, size_t ws_bytes, int op, LaLayout *L) {
  if (!ws) return WKV_ERR_INVALID_ARG;
  if (!la_layout(op, BH, N, L)) return WKV_ERR_INVALID_ARG;
  if (D != kD || M != kD) return WKV_ERR_UNSUPPORTED;
  if (((uintptr_t)ws & 255u) != 0) return WKV_ERR_UNSUPPORTED;
  if (ws_bytes < L->total) return WKV_ERR_WORKSPACE;
  return WKV_OK;
}
}  // namespace

extern "C" size_t linattn_workspace_size(int op, int64_t BH, int64_t N, int D, int M) {
  LaLayout L;
  if ((op != LINATTN_OP_FORWARD && op != LINATTN_OP_BACKWARD) || D != kD || M != kD || !la_layout(op, BH, N, &L))
    return 0;
  return L.total;
}

extern "C" int linattn_forward(int64_t BH, int64_t N, int D, int M, const void *q, const void *k, const void *v,
                               void *out, float *state_out, void *ws, size_t ws_bytes, void *stream) {
  LaLayout L;
  if (N != 0 && (!q || !k || !v || !out)) return WKV_ERR_INVALID_ARG;  // empty tensors may be null
  if (N != 0 && (out == q || out == k || out == v)) return WKV_ERR_INVALID_ARG;
  const int rc = check_common(BH, N, D, M, ws, ws_bytes, LINATTN_OP_FORWARD, &L);
  if (rc != WKV_OK) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(state_out))
    return WKV_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  LaArgs a{};
  a.BH = BH;
  a.N = N;
  a.nch = (int)((N + kL - 1) / kL);
  a.rec = reinterpret_cast<float *>(base + L.rec);
  a.den = reinterpret_cast<float *>(base + L.den);
  a.hdr = reinterpret_cast<WsHeader *>(base);
  a.budget_ns = kBudgetNs;
  const int64_t units = BH * a.nch;
  if (units > 0) {
    CUtensorMap qm, km, vm, om;
    if (!encode_heads_sw64(&qm, q, BH, N, kD) || !encode_heads_sw64(&km, k, BH, N, kD) ||
        !encode_heads_sw64(&vm, v, BH, N, kD) || !encode_heads_sw64(&om, out, BH, N, kD))
      return WKV_ERR_UNSUPPORTED;
    if (prepare(la_state_kernel, kStateSmem, kThreads) || prepare(la_fwd_kernel, kFwdSmem, kThreads)) return WKV_ERR_CUDA;
    cudaError_t e = launch_kernel(la_state_kernel, dim3((unsigned)persistent_grid(la_state_kernel, kStateSmem, 64, units)),
                                  dim3(kThreads), kStateSmem, st, km, vm, a);
    if (e != cudaSuccess) return WKV_ERR_CUDA;
    const int64_t n = BH * kRec;
    e = launch_kernel(la_scan_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, a.rec, BH, a.nch, 0,
                      state_out);
    if (e != cudaSuccess) return WKV_ERR_CUDA;
    return cuda_rc(launch_kernel(la_fwd_kernel, dim3((unsigned)persistent_grid(la_fwd_kernel, kFwdSmem, 128, units)),
                                 dim3(kThreads), kFwdSmem, st, qm, km, vm, om, a));
  }
  if (state_out)  // N = 0: the empty state
    return cuda_rc(cudaMemsetAsync(state_out, 0, (size_t)BH * kRec * sizeof(float), st));
  return WKV_OK;
}

extern "C" int linattn_backward(int64_t BH, int64_t N, int D, int M, const void *q, const void *k, const void *v,
                                const void *grad_out, void *grad_q, void *grad_k, void *grad_v, void *ws,
                                size_t ws_bytes, void *stream) {
  LaLayout L;
  const void *ins[4] = {q, k, v, grad_out};
  const void *outs[3] = {grad_q, grad_k, grad_v};
  if (N != 0) {  // empty tensors may be null
    for (const void *p : ins)
      if (!p) return WKV_ERR_INVALID_ARG;
    for (const void *o : outs) {
      if (!o) return WKV_ERR_INVALID_ARG;
      for (const void *in : ins)
        if (o == in) return WKV_ERR_INVALID_ARG;
    }
    if (grad_q == grad_k || grad_q == grad_v || grad_k == grad_v) return WKV_ERR_INVALID_ARG;
  }
  const int rc = check_common(BH, N, D, M, ws, ws_bytes, LINATTN_OP_BACKWARD, &L);
  if (rc != WKV_OK) return rc;
  for (const void *p : ins)
    if (!aligned16(p)) return WKV_ERR_UNSUPPORTED;
  for (const void *p : outs)
    if (!aligned16(p)) return WKV_ERR_UNSUPPORTED;
  if (N == 0) return WKV_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  LaArgs a{};
  a.BH = BH;
  a.N = N;
  a.nch = (int)((N + kL - 1) / kL);
  a.rec = reinterpret_cast<float *>(base + L.rec);
  a.rec_r = reinterpret_cast<float *>(base + L.rec_r);
  a.gden = reinterpret_cast<float *>(base + L.gden);
  a.hdr = reinterpret_cast<WsHeader *>(base);
  a.budget_ns = kBudgetNs;
  void *gnum = base + L.gnum;
  CUtensorMap qm, km, vm, gm, nm, dqm, dkm, dvm;
  if (!encode_heads_sw64(&qm, q, BH, N, kD) || !encode_heads_sw64(&km, k, BH, N, kD) ||
      !encode_heads_sw64(&vm, v, BH, N, kD) || !encode_heads_sw64(&gm, grad_out, BH, N, kD) ||
      !encode_heads_sw64(&nm, gnum, BH, N, kD) || !encode_heads_sw64(&dqm, grad_q, BH, N, kD) ||
      !encode_heads_sw64(&dkm, grad_k, BH, N, kD) || !encode_heads_sw64(&dvm, grad_v, BH, N, kD))
    return WKV_ERR_UNSUPPORTED;
  if (prepare(la_state_kernel, kStateSmem, kThreads) || prepare(la_bwd_prep_kernel, kPrepSmem, kThreads) ||
      prepare(la_bwd_kernel, kBwdSmem, kThreads))
    return WKV_ERR_CUDA;
  const int64_t units = BH * a.nch;
  const int64_t n = BH * kRec;
  const dim3 sgrid((unsigned)((n + 255) / 256));
  cudaError_t e = launch_kernel(la_state_kernel, dim3((unsigned)persistent_grid(la_state_kernel, kStateSmem, 64, units)),
                                dim3(kThreads), kStateSmem, st, km, vm, a);
  if (e == cudaSuccess) e = launch_kernel(la_scan_kernel, sgrid, dim3(256), 0, st, a.rec, BH, a.nch, 0, (float *)nullptr);
  if (e == cudaSuccess)
    e = launch_kernel(la_bwd_prep_kernel, dim3((unsigned)units), dim3(kThreads), kPrepSmem, st, qm, km, vm, gm, nm,
                      a);
  if (e == cudaSuccess)
    e = launch_kernel(la_scan_kernel, sgrid, dim3(256), 0, st, a.rec_r, BH, a.nch, 1, (float *)nullptr);
  if (e == cudaSuccess)
    e = launch_kernel(la_bwd_kernel, dim3((unsigned)units), dim3(kThreads), kBwdSmem, st, qm, km, vm, nm, dqm, dkm,
                      dvm, a);
  return cuda_rc(e);
}

extern "C" int linattn_backward_saved(int64_t BH, int64_t N, int D, int M, const void *q, const void *k,
                                      const void *v, const void *out, const void *grad_out, void *grad_q,
                                      void *grad_k, void *grad_v, void *ws, size_t ws_bytes, void *stream) {
  LaLayout L;
  const void *ins[5] = {q, k, v, out, grad_out};
  const void *outs[3] = {grad_q, grad_k, grad_v};
  if (N != 0) {  // empty tensors may be null
    for (const void *p : ins)
      if (!p) return WKV_ERR_INVALID_ARG;
    for (const void *o : outs) {
      if (!o) return WKV_ERR_INVALID_ARG;
      for (const void *in : ins)
        if (o == in) return WKV_ERR_INVALID_ARG;
    }
    if (grad_q == grad_k || grad_q == grad_v || grad_k == grad_v) return WKV_ERR_INVALID_ARG;
  }
  const int rc = check_common(BH, N, D, M, ws, ws_bytes, LINATTN_OP_BACKWARD, &L);
  if (rc != WKV_OK) return rc;
  for (const void *p : ins)
    if (!aligned16(p)) return WKV_ERR_UNSUPPORTED;
  for (const void *p : outs)
    if (!aligned16(p)) return WKV_ERR_UNSUPPORTED;
  if (N == 0) return WKV_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  LaArgs a{};
  a.BH = BH;
  a.N = N;
  a.nch = (int)((N + kL - 1) / kL);
  a.rec = reinterpret_cast<float *>(base + L.rec);  // the forward's chunk prefixes
  a.den = reinterpret_cast<float *>(base + L.den);  // and its denominators
  a.rec_r = reinterpret_cast<float *>(base + L.rec_r);
  a.gden = reinterpret_cast<float *>(base + L.gden);
  a.hdr = reinterpret_cast<WsHeader *>(base);
  a.budget_ns = kBudgetNs;
  void *gnum = base + L.gnum;
  CUtensorMap qm, km, vm, om, gm, nm, dqm, dkm, dvm;
  if (!encode_heads_sw64(&qm, q, BH, N, kD) || !encode_heads_sw64(&km, k, BH, N, kD) ||
      !encode_heads_sw64(&vm, v, BH, N, kD) || !encode_heads_sw64(&om, out, BH, N, kD) ||
      !encode_heads_sw64(&gm, grad_out, BH, N, kD) || !encode_heads_sw64(&nm, gnum, BH, N, kD) ||
      !encode_heads_sw64(&dqm, grad_q, BH, N, kD) || !encode_heads_sw64(&dkm, grad_k, BH, N, kD) ||
      !encode_heads_sw64(&dvm, grad_v, BH, N, kD))
    return WKV_ERR_UNSUPPORTED;
  if (prepare(la_bwd_prep_saved_kernel, kPrepSavedSmem, kThreads) || prepare(la_bwd_kernel, kBwdSmem, kThreads))
    return WKV_ERR_CUDA;
  const int64_t units = BH * a.nch;
  const int64_t n = BH * kRec;
  cudaError_t e = launch_kernel(la_bwd_prep_saved_kernel, dim3((unsigned)units), dim3(kThreads), kPrepSavedSmem, st,
                                qm, gm, om, nm, a);
  if (e == cudaSuccess)
    e = launch_kernel(la_scan_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, a.rec_r, BH, a.nch, 1,
                      (float *)nullptr);
  if (e == cudaSuccess)
    e = launch_kernel(la_bwd_kernel, dim3((unsigned)units), dim3(kThreads), kBwdSmem, st, qm, km, vm, nm, dqm, dkm,
                      dvm, a);
  return cuda_rc(e);
}
