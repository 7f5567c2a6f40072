// wkv_api.cu -- C ABI of libwkv (declared in include/wkv.h): argument
// checks, workspace layout and kernel selection.  Every step of the
// operator runs in the kernels of wkv_forward.cu, wkv_backward.cu and
// wkv_step.cu; this file only validates and launches.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/wkv.h"
#include "wkv_internal.cuh"
#include "wkv_tile.cuh"

namespace wkv {
cudaError_t launch_forward(const FwdArgs &a, int dtype, int kind, int num_sms, cudaStream_t st);
bool fwd_tma_eligible(const FwdArgs &a, int dtype);
cudaError_t launch_reduce_wu(const float *part, int64_t nchunks, int64_t B, int64_t C, float *gw,
                             float *gu, cudaStream_t st);
cudaError_t launch_forward_seg(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st);
cudaError_t launch_forward_clu(const FwdArgs &f, int dtype, int num_sms, cudaStream_t st);
cudaError_t launch_backward_seg(const BwdArgs &p, int dtype, float *gw, float *gu, unsigned *tile_cnt,
                                int64_t scratch_doubles, int num_sms, cudaStream_t st);
cudaError_t launch_backward(const BwdArgs &a, int dtype, float *gw, float *gu, cudaStream_t st);
cudaError_t launch_step(const StepArgs &a, bool vec, int num_sms, cudaStream_t st);
cudaError_t launch_gate(int op, int dtype, void *x, const void *go, const void *r, int64_t n, int num_sms,
                        cudaStream_t st);
cudaError_t launch_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int n, const float *mu, const void *x,
                               const void *x_prev, void *out, const void *g, void *gx, void *gx_prev, float *part,
                               float *gmu, bool bwd, bool vec, int num_sms, cudaStream_t st);
int64_t token_shift_rows(int64_t B, int64_t T);
cudaError_t launch_state_grad_t0(const float *gs_out, const float *p_out, const float *s_in, float *gs_in,
                                 int64_t BC, int num_sms, cudaStream_t st);
int64_t fwd_chunk_tokens();
cudaError_t launch_forward_tile(const FwdArgs &f, float4 *rec, int dtype, int num_sms, cudaStream_t st);
cudaError_t launch_backward_tile(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *rec, float4 *chain_sum,
                                 int num_sms, cudaStream_t st);
cudaError_t launch_forward_chain(const FwdArgs &f, int dtype, cudaStream_t st);
cudaError_t launch_backward_chain(const BwdArgs &p, int dtype, float *gw, float *gu, float4 *chain_sum, int num_sms,
                                  cudaStream_t st);
}  // namespace wkv

using namespace wkv;

namespace {

constexpr int kGateApply = 0, kGatePre = 1, kGatePost = 2;  // launch_gate ops

// The cudaError_t behind the calling thread's most recent WKV_ERR_CUDA.
thread_local int t_last_cuda_error = 0;

int cuda_rc(cudaError_t e) {
  if (e == cudaSuccess) return WKV_OK;
  t_last_cuda_error = (int)e;
  return WKV_ERR_CUDA;
}

constexpr int64_t kDefaultSpin = 1000000;  // polls of ~1 us backoff: about one second
constexpr int64_t kSeqMinChains = 148 * 1024;  // chains that fill B200 with one thread each

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
inline size_t esize(int dtype) { return dtype == WKV_BF16 ? 2 : 4; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
  return x < y + nb && y < x + na;
}

// Sizes: B, C >= 1, 0 <= T < 2^31, B*T*C < 2^62 (checked without overflow).
bool sizes_ok(int64_t B, int64_t T, int64_t C) {
  if (B < 1 || C < 1 || T < 0 || T >= (int64_t(1) << 31)) return false;
  const int64_t lim = int64_t(1) << 62;
  if (B > lim / C) return false;
  const int64_t BC = B * C;
  if (T > 0 && BC > lim / T) return false;
  return true;
}

struct Layout {
  size_t flags, desc, desc_bytes, ckpt, part, cnt, rec, sums, total;
  int64_t nct, nchains, nchunks_f, nchunks_b, nck;
};

// Workspace: [256 B header][flags][descriptors][ckpt (backward)][partials
// (backward)].  The flag/descriptor region is sized for the larger of the
// forward and backward tilings so one workspace serves both.
Layout layout(int op, int64_t B, int64_t T, int64_t C) {
  Layout L{};
  L.nct = cdiv(C, 32);
  L.nchains = B * L.nct;
  L.nchunks_f = cdiv(T, fwd_chunk_tokens());
  L.nchunks_b = cdiv(T, 32);  // the backward kernels' records: units of at least 32 tokens
  L.nck = cdiv(T, kCkpt);     // checkpoints
  const int64_t tiles = L.nchains * (L.nchunks_f > L.nchunks_b ? L.nchunks_f : L.nchunks_b);
  size_t off = sizeof(WsHeader);
  L.flags = off;
  off = align_up(off + sizeof(unsigned) * (size_t)tiles, 256);
  L.desc = off;
  L.desc_bytes = sizeof(float) * kDescFloats * (size_t)tiles;
  off = align_up(off + L.desc_bytes, 256);
  // tile kernels: two records per unit of at most 32 tokens, 16 bytes per
  // lane each (forward) or 32 (backward); their flags share the flag region.
  // The region sits at the same offset in the forward and the backward
  // layout: a backward without checkpoints runs the forward on its own
  // workspace, and the forward's records must not reach the regions below.
  L.rec = off;
  off = align_up(off + (op == WKV_OP_BACKWARD ? 2048 : 1536) * (size_t)(L.nchains * L.nchunks_b), 256);
  L.ckpt = L.part = L.cnt = 0;
  if (op == WKV_OP_BACKWARD) {
    L.ckpt = off;
    off = align_up(off + sizeof(float) * 3 * (size_t)(B * C) * (size_t)L.nck, 256);
    L.part = off;  // dL/dw, dL/du partials: 2 floats per (chunk, b, c); the tile kernel's tagged words: 4
    off = align_up(off + sizeof(float) * 4 * (size_t)(B * C) * (size_t)L.nchunks_b, 256);
    L.cnt = off;  // per channel tile counters of the segment backward's reduction (cleared by it)
    off = align_up(off + sizeof(unsigned) * (size_t)L.nct, 256);
    // the tile backward's per-chain sums of dL/dw, dL/du, then its
    // first-level sums (one 16-byte word per (b, c) and group of 16 units)
    L.sums = off;
    off = align_up(off + 16 * (size_t)(B * C) * (size_t)(1 + cdiv(L.nchunks_b, 16)), 256);
  }
  L.total = off;
  return L;
}


// SM count of the current device, looked up once per device.
int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// AUTO picks the tile kernels when a chain has few units in flight at once
// (at most about four of the resident warps per chain): their joins then find
// the records they need published a step earlier.  With more (long chains
// over few batch rows and channels) the segment kernels' longer segments
// amortise their joins better.  warps_per_sm: resident warps of the kernel.
bool tile_pays(int64_t nchains, int warps_per_sm) { return nchains * 4 >= (int64_t)warps_per_sm * num_sms(); }

// AUTO picks the chain kernels when the chains (one per warp scheduler, four
// per SM) occupy at least 60 % of the schedulers; with more chains than one
// wave holds they run in waves.  Measured on B200 (bf16, T 4096, forward /
// backward): 384 chains 128 / 227 us against the tile kernels' 165 / 293;
// 640 chains 222 / 410 against 239 / 439; 1024 chains 222 / 413 against
// 375 / 625.  With fewer chains the idle schedulers cost more than the
// time-parallel kernels' joins (192 chains, fp32 T 1024: 41 / 91 us against
// the segment kernels' 29 / 52).
bool chain_pays(int64_t nchains) {
  const int64_t slots = 4 * (int64_t)num_sms();
  return nchains * 5 >= slots * 3;
}

bool pick_chunked(const wkv_options *opt, int64_t B, int64_t T, int64_t C) {
  const int kernel = opt ? opt->kernel : WKV_KERNEL_AUTO;
  if (kernel == WKV_KERNEL_SEQUENTIAL) return false;
  if (kernel == WKV_KERNEL_CHUNKED || kernel == WKV_KERNEL_CHUNKED_REGS || kernel == WKV_KERNEL_SEGMENT ||
      kernel == WKV_KERNEL_CLUSTER || kernel == WKV_KERNEL_TILE || kernel == WKV_KERNEL_CHAIN)
    return true;
  // Enough independent chains to fill the GPU, or too short to split.
  return !(B * C >= kSeqMinChains || T <= 2 * fwd_chunk_tokens());
}

bool options_ok(const wkv_options *opt) {
  if (!opt) return true;
  const int k = opt->kernel;
  return k == WKV_KERNEL_AUTO || k == WKV_KERNEL_SEQUENTIAL || k == WKV_KERNEL_CHUNKED ||
         k == WKV_KERNEL_CHUNKED_REGS || k == WKV_KERNEL_SEGMENT || k == WKV_KERNEL_CLUSTER ||
         k == WKV_KERNEL_TILE || k == WKV_KERNEL_CHAIN;
}

int64_t spin_of(const wkv_options *opt) {
  return (opt && opt->spin_limit > 0) ? opt->spin_limit : kDefaultSpin;
}

int check_forward_args(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                       const void *k, const void *v, const float *state_in, const void *y,
                       const float *state_out, const float *ckpt) {
  if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_INVALID_ARG;
  if (!sizes_ok(B, T, C)) return WKV_ERR_INVALID_ARG;
  if (!w || !u) return WKV_ERR_INVALID_ARG;
  if (T > 0 && (!k || !v)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype);
  if (!aligned(w, 4) || !aligned(u, 4) || !aligned(k, es) || !aligned(v, es) ||
      !aligned(y, es) || !aligned(state_in, 4) || !aligned(state_out, 4) || !aligned(ckpt, 4))
    return WKV_ERR_UNSUPPORTED;
  const size_t nb = (size_t)(B * T * C) * es;
  if (overlaps(y, nb, k, nb) || overlaps(y, nb, v, nb)) return WKV_ERR_UNSUPPORTED;
  const size_t sb = 3 * sizeof(float) * (size_t)(B * C);
  if (state_in && state_out && state_in != state_out && overlaps(state_in, sb, state_out, sb))
    return WKV_ERR_UNSUPPORTED;
  return WKV_OK;
}

// r: gate input (y receives sigma(r) * wkv), or NULL.  The segment forward
// applies the gate in its store loop; the other kernels write wkv and an
// elementwise pass gates it.
int forward_impl(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                 const void *k, const void *v, const float *state_in, void *y, float *state_out,
                 float *ckpt, void *ws, size_t ws_bytes, cudaStream_t st, const wkv_options *opt,
                 const void *r = nullptr) {
  if (T == 0) {
    // No tokens: the state passes through unchanged (the sequential kernel
    // with T = 0 only converts state_in, or the empty state, to state_out).
    if (!state_out) return WKV_OK;
    FwdArgs a{};
    a.B = B; a.T = 0; a.C = C; a.w = w; a.u = u; a.state_in = state_in; a.state_out = state_out;
    return cuda_rc(launch_forward(a, dtype, 0, 1, st));
  }
  const Layout L = layout(WKV_OP_FORWARD, B, T, C);
  const bool chunked = pick_chunked(opt, B, T, C);
  if (chunked) {
    if (!ws || !aligned(ws, 256)) return WKV_ERR_WORKSPACE;
    if (ws_bytes < L.total) return WKV_ERR_WORKSPACE;
  }
  FwdArgs a{};
  a.B = B; a.T = T; a.C = C; a.w = w; a.u = u; a.k = k; a.v = v;
  a.state_in = state_in; a.y = y; a.state_out = state_out; a.ckpt = ckpt;
  char *base = static_cast<char *>(ws);
  a.hdr = reinterpret_cast<WsHeader *>(base);
  a.flags = base ? reinterpret_cast<unsigned *>(base + L.flags) : nullptr;
  a.desc = base ? reinterpret_cast<float *>(base + L.desc) : nullptr;
  a.nct = L.nct; a.nchains = L.nchains; a.nchunks = L.nchunks_f;
  a.spin_limit = spin_of(opt);
  a.hold_first = opt ? opt->test_hold_first_chunk : 0;
  const int kernel = opt ? opt->kernel : WKV_KERNEL_AUTO;
  const bool tma = chunked && fwd_tma_eligible(a, dtype);
  // chain forward: whole chains per warp, y (and r) loaded and stored by TMA
  if (tma && (kernel == WKV_KERNEL_CHAIN || (kernel == WKV_KERNEL_AUTO && chain_pays(L.nchains))) &&
      aligned(y, 16) && aligned(r, 16)) {
    a.r = r;
    return cuda_rc(launch_forward_chain(a, dtype, st));
  }
  // tile forward: whole units of tokens, y (and r) loaded and stored by TMA
  if (tma && (kernel == WKV_KERNEL_TILE || kernel == WKV_KERNEL_CHAIN ||
              (kernel == WKV_KERNEL_AUTO && tile_pays(L.nchains, r ? 6 : 9))) &&
      T >= tile_fwd_tokens(dtype) && aligned(y, 16) && aligned(r, 16)) {
    a.r = r;
    return cuda_rc(launch_forward_tile(a, reinterpret_cast<float4 *>(base + L.rec), dtype, num_sms(), st));
  }
  const bool seg = tma && (kernel == WKV_KERNEL_AUTO || kernel == WKV_KERNEL_SEGMENT || kernel == WKV_KERNEL_TILE ||
                           kernel == WKV_KERNEL_CHAIN);
  if (seg && (!r || aligned(r, 16))) {
    a.r = r;  // fused gate
    return cuda_rc(launch_forward_seg(a, dtype, num_sms(), st));
  }
  cudaError_t e;
  if (tma && kernel == WKV_KERNEL_CLUSTER) {
    e = launch_forward_clu(a, dtype, num_sms(), st);
  } else if (seg) {
    e = launch_forward_seg(a, dtype, num_sms(), st);
  } else {
    int kind = 0;
    if (chunked) kind = (tma && kernel != WKV_KERNEL_CHUNKED_REGS) ? 2 : 1;
    e = launch_forward(a, dtype, kind, num_sms(), st);
  }
  if (e == cudaSuccess && r) e = launch_gate(kGateApply, dtype, y, nullptr, r, B * T * C, num_sms(), st);
  return cuda_rc(e);
}

// The segment backward runs for AUTO/SEGMENT when the rows of k, v and the
// output gradient are 16-byte aligned.
bool bwd_uses_seg(int64_t B, int64_t T, int64_t C, int dtype, const void *k, const void *v, const void *gy,
                  const wkv_options *opt) {
  const int kernel = opt ? opt->kernel : WKV_KERNEL_AUTO;
  if (kernel != WKV_KERNEL_AUTO && kernel != WKV_KERNEL_SEGMENT && kernel != WKV_KERNEL_TILE &&
      kernel != WKV_KERNEL_CHAIN)
    return false;
  FwdArgs probe{};
  probe.B = B; probe.T = T; probe.C = C; probe.k = k; probe.v = v;
  return fwd_tma_eligible(probe, dtype) && aligned(gy, 16);
}

// Checks shared by the gated and ungated backward (grad_y: the gradient the
// caller passes, of y or of the gated output).
int check_backward_args(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                        const void *k, const void *v, const void *grad_y, const float *state_in,
                        const float *ckpt, float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                        const wkv_options *opt) {
  int rc = check_forward_args(B, T, C, dtype, w, u, k, v, state_in, nullptr, nullptr, ckpt);
  if (rc != WKV_OK) return rc;
  if (!options_ok(opt)) return WKV_ERR_INVALID_ARG;
  if (!grad_w || !grad_u) return WKV_ERR_INVALID_ARG;
  if (T > 0 && (!grad_y || !grad_k || !grad_v)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype);
  if (!aligned(grad_y, es) || !aligned(grad_k, es) || !aligned(grad_v, es) ||
      !aligned(grad_w, 4) || !aligned(grad_u, 4))
    return WKV_ERR_UNSUPPORTED;
  const size_t nb = (size_t)(B * T * C) * es;
  const void *ins[3] = {k, v, grad_y};
  for (const void *in : ins)
    if (overlaps(grad_k, nb, in, nb) || overlaps(grad_v, nb, in, nb)) return WKV_ERR_UNSUPPORTED;
  if (overlaps(grad_k, nb, grad_v, nb) || overlaps(grad_w, 4 * C, grad_u, 4 * C))
    return WKV_ERR_UNSUPPORTED;
  return WKV_OK;
}

// State terms of a backward (all null when unused): the final state's
// gradient with the p plane of the representation it refers to, and the
// output for the initial state's gradient.
struct StateTerms {
  const float *gs_out = nullptr, *p_out = nullptr;
  float *gs_in = nullptr;
};

// Backward after the checks.  r, gr: gate input and its gradient for the
// fused gated segment backward (grad_y is then dL/do), else NULL.
int backward_impl(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                  const void *k, const void *v, const void *grad_y, const float *state_in,
                  const float *ckpt, float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                  void *ws, size_t ws_bytes, cudaStream_t st, const wkv_options *opt,
                  const void *r = nullptr, void *gr = nullptr, const StateTerms &sg = StateTerms()) {
  if (T == 0) {
    int rc = cuda_rc(cudaMemsetAsync(grad_w, 0, sizeof(float) * C, st));
    if (rc == WKV_OK) rc = cuda_rc(cudaMemsetAsync(grad_u, 0, sizeof(float) * C, st));
    if (rc == WKV_OK && sg.gs_in)
      rc = cuda_rc(launch_state_grad_t0(sg.gs_out, sg.p_out, state_in, sg.gs_in, B * C, num_sms(), st));
    return rc;
  }
  const Layout L = layout(WKV_OP_BACKWARD, B, T, C);
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return WKV_ERR_WORKSPACE;
  char *base = static_cast<char *>(ws);
  const float *ck = ckpt;
  if (!ck) {
    // Recompute the per-chunk states with a forward pass that writes only
    // the checkpoints (one extra read of k and v).
    float *ws_ck = reinterpret_cast<float *>(base + L.ckpt);
    int rc = forward_impl(B, T, C, dtype, w, u, k, v, state_in, nullptr, nullptr, ws_ck, ws, ws_bytes, st, opt);
    if (rc != WKV_OK) return rc;
    ck = ws_ck;
  }
  BwdArgs a{};
  a.B = B; a.T = T; a.C = C; a.w = w; a.u = u; a.k = k; a.v = v; a.gy = grad_y;
  a.ckpt = ck; a.gk = grad_k; a.gv = grad_v;
  a.part = reinterpret_cast<float *>(base + L.part);
  a.hdr = reinterpret_cast<WsHeader *>(base);
  a.flags = reinterpret_cast<unsigned *>(base + L.flags);
  a.desc = reinterpret_cast<float *>(base + L.desc);
  a.nct = L.nct; a.nchains = L.nchains; a.nchunks = L.nchunks_b;
  a.spin_limit = spin_of(opt);
  a.hold_first = opt ? opt->test_hold_first_chunk : 0;
  a.r = r;
  a.gr = gr;
  a.gs_out = sg.gs_out;
  a.p_out = sg.p_out;
  a.gs_in = sg.gs_in;
  a.state_in = state_in;
  const int kernel = opt ? opt->kernel : WKV_KERNEL_AUTO;
  const bool bwd_tma = bwd_uses_seg(B, T, C, dtype, k, v, grad_y, nullptr) && aligned(grad_k, 16) &&
                       aligned(grad_v, 16);
  if ((!r || (aligned(r, 16) && aligned(gr, 16))) && bwd_tma && aligned(ck, 16) &&
      (kernel == WKV_KERNEL_CHAIN || (kernel == WKV_KERNEL_AUTO && chain_pays(L.nchains)))) {
    float4 *sums = reinterpret_cast<float4 *>(base + L.sums);
    return cuda_rc(launch_backward_chain(a, dtype, grad_w, grad_u, sums, num_sms(), st));
  }
  if ((!r || (aligned(r, 16) && aligned(gr, 16))) &&
      (kernel == WKV_KERNEL_TILE || kernel == WKV_KERNEL_CHAIN ||
       (kernel == WKV_KERNEL_AUTO && tile_pays(L.nchains, r ? 6 : 8))) &&
      T >= tile_fwd_tokens(dtype) && bwd_uses_seg(B, T, C, dtype, k, v, grad_y, nullptr) && aligned(grad_k, 16) &&
      aligned(grad_v, 16)) {
    // the per-chain sums of dL/dw, dL/du use the descriptor region (16 bytes
    // per (b, c) <= 640 bytes per chain and chunk), idle in the tile kernels
    float4 *rec = reinterpret_cast<float4 *>(base + L.rec), *sums = reinterpret_cast<float4 *>(base + L.sums);
    return cuda_rc(launch_backward_tile(a, dtype, grad_w, grad_u, rec, sums, num_sms(), st));
  }
  if (bwd_uses_seg(B, T, C, dtype, k, v, grad_y, opt)) {
    const int64_t scratch = (int64_t)(L.desc_bytes / sizeof(double));
    return cuda_rc(launch_backward_seg(a, dtype, grad_w, grad_u, reinterpret_cast<unsigned *>(base + L.cnt), scratch,
                               num_sms(), st));
  }
  if (r) return WKV_ERR_UNSUPPORTED;  // callers fuse the gate only into the segment backward
  return cuda_rc(launch_backward(a, dtype, grad_w, grad_u, st));
}

}  // namespace

extern "C" {

size_t wkv_workspace_size(int op, int64_t B, int64_t T, int64_t C, int dtype) {
  if (dtype != WKV_F32 && dtype != WKV_BF16) return 0;
  if (!sizes_ok(B, T, C)) return 0;
  if (op == WKV_OP_STEP) return 0;
  if (op != WKV_OP_FORWARD && op != WKV_OP_BACKWARD) return 0;
  return layout(op, B, T, C).total;
}

int wkv_workspace_init(void *ws, size_t ws_bytes, void *stream) {
  if (!ws) return WKV_ERR_WORKSPACE;
  return cuda_rc(cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream));
}

size_t wkv_ckpt_size(int64_t B, int64_t T, int64_t C) {
  if (!sizes_ok(B, T, C)) return 0;
  return sizeof(float) * 3 * (size_t)(B * C) * (size_t)cdiv(T, kCkpt);
}

int wkv_forward_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                   const void *k, const void *v, const float *state_in, void *y,
                   float *state_out, float *ckpt, void *ws, size_t ws_bytes, void *stream,
                   const wkv_options *opt) {
  int rc = check_forward_args(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt);
  if (rc != WKV_OK) return rc;
  if (T > 0 && !y) return WKV_ERR_INVALID_ARG;
  if (!options_ok(opt)) return WKV_ERR_INVALID_ARG;
  return forward_impl(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes,
                      (cudaStream_t)stream, opt);
}

int wkv_forward(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                const void *k, const void *v, const float *state_in, void *y, float *state_out,
                float *ckpt, void *ws, size_t ws_bytes, void *stream) {
  return wkv_forward_ex(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes,
                        stream, nullptr);
}

int wkv_backward_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                    const void *k, const void *v, const void *grad_y, const float *state_in,
                    const float *ckpt, float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                    void *ws, size_t ws_bytes, void *stream, const wkv_options *opt) {
  const int rc = check_backward_args(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                                     grad_k, grad_v, opt);
  if (rc != WKV_OK) return rc;
  return backward_impl(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k, grad_v,
                       ws, ws_bytes, (cudaStream_t)stream, opt);
}

int wkv_backward(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                 const void *k, const void *v, const void *grad_y, const float *state_in,
                 const float *ckpt, float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                 void *ws, size_t ws_bytes, void *stream) {
  return wkv_backward_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                         grad_k, grad_v, ws, ws_bytes, stream, nullptr);
}

int wkv_backward_state_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                          const void *k, const void *v, const void *grad_y, const float *state_in,
                          const float *ckpt, const float *state_out, const float *grad_state_out,
                          float *grad_w, float *grad_u, void *grad_k, void *grad_v, float *grad_state_in,
                          void *ws, size_t ws_bytes, void *stream, const wkv_options *opt) {
  const int rc = check_backward_args(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                                     grad_k, grad_v, opt);
  if (rc != WKV_OK) return rc;
  if (grad_state_out && !state_out) return WKV_ERR_INVALID_ARG;
  if (!aligned(state_out, 4) || !aligned(grad_state_out, 4) || !aligned(grad_state_in, 4))
    return WKV_ERR_UNSUPPORTED;
  const size_t es = esize(dtype), nb = (size_t)(B * T * C) * es, sb = 3 * sizeof(float) * (size_t)(B * C);
  if (grad_state_in) {
    const void *big[4] = {k, v, grad_y, ckpt};
    for (const void *x : big)
      if (overlaps(grad_state_in, sb, x, x == ckpt ? wkv_ckpt_size(B, T, C) : nb)) return WKV_ERR_UNSUPPORTED;
    const void *st3[3] = {state_in, state_out, grad_state_out};
    for (const void *x : st3)
      if (overlaps(grad_state_in, sb, x, sb)) return WKV_ERR_UNSUPPORTED;
    if (overlaps(grad_state_in, sb, grad_k, nb) || overlaps(grad_state_in, sb, grad_v, nb) ||
        overlaps(grad_state_in, sb, grad_w, 4 * C) || overlaps(grad_state_in, sb, grad_u, 4 * C))
      return WKV_ERR_UNSUPPORTED;
  }
  if (grad_state_out && (overlaps(grad_k, nb, grad_state_out, sb) || overlaps(grad_v, nb, grad_state_out, sb)))
    return WKV_ERR_UNSUPPORTED;
  StateTerms sg;
  sg.gs_out = grad_state_out;
  sg.p_out = grad_state_out ? state_out + 2 * B * C : nullptr;
  sg.gs_in = grad_state_in;
  return backward_impl(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k, grad_v, ws,
                       ws_bytes, (cudaStream_t)stream, opt, nullptr, nullptr, sg);
}

int wkv_backward_state(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                       const void *k, const void *v, const void *grad_y, const float *state_in,
                       const float *ckpt, const float *state_out, const float *grad_state_out, float *grad_w,
                       float *grad_u, void *grad_k, void *grad_v, float *grad_state_in, void *ws,
                       size_t ws_bytes, void *stream) {
  return wkv_backward_state_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, state_out, grad_state_out,
                               grad_w, grad_u, grad_k, grad_v, grad_state_in, ws, ws_bytes, stream, nullptr);
}

int wkv_forward_gated_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                         const void *k, const void *v, const void *r, const float *state_in, void *o,
                         float *state_out, float *ckpt, void *ws, size_t ws_bytes, void *stream,
                         const wkv_options *opt) {
  int rc = check_forward_args(B, T, C, dtype, w, u, k, v, state_in, o, state_out, ckpt);
  if (rc != WKV_OK) return rc;
  if (T > 0 && (!o || !r)) return WKV_ERR_INVALID_ARG;
  if (!options_ok(opt)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype), nb = (size_t)(B * T * C) * es;
  if (!aligned(r, es)) return WKV_ERR_UNSUPPORTED;
  if (overlaps(o, nb, r, nb)) return WKV_ERR_UNSUPPORTED;
  return forward_impl(B, T, C, dtype, w, u, k, v, state_in, o, state_out, ckpt, ws, ws_bytes,
                      (cudaStream_t)stream, opt, T > 0 ? r : nullptr);
}

int wkv_forward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                      const void *k, const void *v, const void *r, const float *state_in, void *o,
                      float *state_out, float *ckpt, void *ws, size_t ws_bytes, void *stream) {
  return wkv_forward_gated_ex(B, T, C, dtype, w, u, k, v, r, state_in, o, state_out, ckpt, ws, ws_bytes,
                              stream, nullptr);
}

int wkv_backward_gated_ex(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                          const void *k, const void *v, const void *r, const void *grad_o,
                          const float *state_in, const float *ckpt, float *grad_w, float *grad_u,
                          void *grad_k, void *grad_v, void *grad_r, void *ws, size_t ws_bytes, void *stream,
                          const wkv_options *opt) {
  int rc = check_backward_args(B, T, C, dtype, w, u, k, v, grad_o, state_in, ckpt, grad_w, grad_u, grad_k,
                               grad_v, opt);
  if (rc != WKV_OK) return rc;
  if (T > 0 && (!r || !grad_r)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype), nb = (size_t)(B * T * C) * es;
  if (!aligned(r, es) || !aligned(grad_r, es)) return WKV_ERR_UNSUPPORTED;
  const void *others[6] = {k, v, r, grad_o, grad_k, grad_v};
  for (const void *x : others)
    if (overlaps(grad_r, nb, x, nb)) return WKV_ERR_UNSUPPORTED;
  if (overlaps(grad_k, nb, r, nb) || overlaps(grad_v, nb, r, nb)) return WKV_ERR_UNSUPPORTED;
  cudaStream_t st = (cudaStream_t)stream;
  if (T > 0 && (!ws || !aligned(ws, 256) || ws_bytes < layout(WKV_OP_BACKWARD, B, T, C).total))
    return WKV_ERR_WORKSPACE;
  // (the fused kernel also reads grad_k's rows back through TMA)
  if (T == 0 || (bwd_uses_seg(B, T, C, dtype, k, v, grad_o, opt) && aligned(r, 16) && aligned(grad_k, 16)))
    return backward_impl(B, T, C, dtype, w, u, k, v, grad_o, state_in, ckpt, grad_w, grad_u, grad_k, grad_v,
                         ws, ws_bytes, st, opt, T > 0 ? r : nullptr, grad_r);
  // Unfused: grad_r first carries dL/dwkv = grad_o sigma(r) into the WKV
  // backward, then wkv itself (a forward into grad_r), and finally
  // dL/dr = grad_o wkv sigma'(r).
  const int64_t n = B * T * C;
  rc = cuda_rc(launch_gate(kGatePre, dtype, grad_r, grad_o, r, n, num_sms(), st));
  if (rc != WKV_OK) return rc;
  rc = backward_impl(B, T, C, dtype, w, u, k, v, grad_r, state_in, ckpt, grad_w, grad_u, grad_k, grad_v, ws,
                     ws_bytes, st, opt);
  if (rc != WKV_OK) return rc;
  rc = forward_impl(B, T, C, dtype, w, u, k, v, state_in, grad_r, nullptr, nullptr, ws, ws_bytes, st, opt);
  if (rc != WKV_OK) return rc;
  return cuda_rc(launch_gate(kGatePost, dtype, grad_r, grad_o, r, n, num_sms(), st));
}

int wkv_backward_gated(int64_t B, int64_t T, int64_t C, int dtype, const float *w, const float *u,
                       const void *k, const void *v, const void *r, const void *grad_o, const float *state_in,
                       const float *ckpt, float *grad_w, float *grad_u, void *grad_k, void *grad_v,
                       void *grad_r, void *ws, size_t ws_bytes, void *stream) {
  return wkv_backward_gated_ex(B, T, C, dtype, w, u, k, v, r, grad_o, state_in, ckpt, grad_w, grad_u, grad_k,
                               grad_v, grad_r, ws, ws_bytes, stream, nullptr);
}

size_t wkv_token_shift_workspace_size(int64_t B, int64_t T, int64_t C, int n) {
  if (n < 1 || n > 4 || !sizes_ok(B, T, C)) return 0;
  const size_t bytes = sizeof(float) * (size_t)token_shift_rows(B, T) * (size_t)n * (size_t)C;
  return align_up(bytes > 0 ? bytes : 1, 256);
}

int wkv_token_shift(int64_t B, int64_t T, int64_t C, int dtype, int n, const float *mu, const void *x,
                    const void *x_prev, void *out, void *stream) {
  if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_INVALID_ARG;
  if (n < 1 || n > 4 || !sizes_ok(B, T, C) || !mu) return WKV_ERR_INVALID_ARG;
  if (T > 0 && (!x || !out)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype), nb = (size_t)(B * T * C) * es, pb = (size_t)(B * C) * es;
  if (!aligned(mu, 4) || !aligned(x, es) || !aligned(x_prev, es) || !aligned(out, es)) return WKV_ERR_UNSUPPORTED;
  if (overlaps(out, n * nb, x, nb) || overlaps(out, n * nb, x_prev, pb) || overlaps(out, n * nb, mu, 4 * n * C))
    return WKV_ERR_UNSUPPORTED;
  if (T == 0) return WKV_OK;
  const size_t va = 4 * es;
  const bool vec = C % 4 == 0 && aligned(x, va) && aligned(x_prev, va) && aligned(out, va);
  return cuda_rc(launch_token_shift(B, T, C, dtype, n, mu, x, x_prev, out, nullptr, nullptr, nullptr, nullptr,
                                    nullptr, false, vec, num_sms(), (cudaStream_t)stream));
}

int wkv_token_shift_backward(int64_t B, int64_t T, int64_t C, int dtype, int n, const float *mu, const void *x,
                             const void *x_prev, const void *grad_out, void *grad_x, float *grad_mu,
                             void *grad_x_prev, void *ws, size_t ws_bytes, void *stream) {
  if (dtype != WKV_F32 && dtype != WKV_BF16) return WKV_ERR_INVALID_ARG;
  if (n < 1 || n > 4 || !sizes_ok(B, T, C) || !mu || !grad_mu) return WKV_ERR_INVALID_ARG;
  if (T > 0 && (!x || !grad_out || !grad_x)) return WKV_ERR_INVALID_ARG;
  const size_t es = esize(dtype), nb = (size_t)(B * T * C) * es, pb = (size_t)(B * C) * es;
  const size_t mb = 4 * (size_t)n * (size_t)C;
  if (!aligned(mu, 4) || !aligned(grad_mu, 4) || !aligned(x, es) || !aligned(x_prev, es) ||
      !aligned(grad_out, es) || !aligned(grad_x, es) || !aligned(grad_x_prev, es))
    return WKV_ERR_UNSUPPORTED;
  // outputs must not overlap the inputs or each other
  struct Span { const void *p; size_t n; };
  const Span ins[4] = {{x, nb}, {x_prev, pb}, {grad_out, n * nb}, {mu, mb}};
  const Span outs[3] = {{grad_x, nb}, {grad_mu, mb}, {grad_x_prev, pb}};
  for (const Span &o : outs) {
    for (const Span &i : ins)
      if (overlaps(o.p, o.n, i.p, i.n)) return WKV_ERR_UNSUPPORTED;
    for (const Span &o2 : outs)
      if (&o2 != &o && overlaps(o.p, o.n, o2.p, o2.n)) return WKV_ERR_UNSUPPORTED;
  }
  cudaStream_t st = (cudaStream_t)stream;
  if (T == 0) {
    int rc = cuda_rc(cudaMemsetAsync(grad_mu, 0, mb, st));
    if (rc == WKV_OK && grad_x_prev) rc = cuda_rc(cudaMemsetAsync(grad_x_prev, 0, pb, st));
    return rc;
  }
  const size_t need = wkv_token_shift_workspace_size(B, T, C, n);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return WKV_ERR_WORKSPACE;
  const size_t va = 4 * es;
  const bool vec = C % 4 == 0 && aligned(x, va) && aligned(x_prev, va) && aligned(grad_out, va) &&
                   aligned(grad_x, va) && aligned(grad_x_prev, va);
  return cuda_rc(launch_token_shift(B, T, C, dtype, n, mu, x, x_prev, nullptr, grad_out, grad_x, grad_x_prev,
                                    static_cast<float *>(ws), grad_mu, true, vec, num_sms(), st));
}

int wkv_step(int64_t N, int64_t C, const float *w, const float *u, const float *k_t,
             const float *v_t, const float *state_in, float *y_t, float *state_out, void *stream) {
  if (!sizes_ok(N, 1, C)) return WKV_ERR_INVALID_ARG;
  if (!w || !u || !k_t || !v_t || !state_in || !y_t || !state_out) return WKV_ERR_INVALID_ARG;
  const void *ptrs[7] = {w, u, k_t, v_t, state_in, y_t, state_out};
  for (const void *p : ptrs)
    if (!aligned(p, 4)) return WKV_ERR_UNSUPPORTED;
  const size_t nb = sizeof(float) * (size_t)(N * C), sb = 3 * nb;
  if (state_in != state_out && overlaps(state_in, sb, state_out, sb)) return WKV_ERR_UNSUPPORTED;
  if (overlaps(y_t, nb, state_in, sb) || overlaps(y_t, nb, state_out, sb) ||
      overlaps(y_t, nb, k_t, nb) || overlaps(y_t, nb, v_t, nb) ||
      overlaps(state_out, sb, k_t, nb) || overlaps(state_out, sb, v_t, nb))
    return WKV_ERR_UNSUPPORTED;
  StepArgs a{N, C, w, u, k_t, v_t, state_in, y_t, state_out};
  bool vec = (C % 4) == 0;
  for (const void *p : ptrs) vec = vec && aligned(p, 16);
  return cuda_rc(launch_step(a, vec, num_sms(), (cudaStream_t)stream));
}

int wkv_get_status(void *ws, void *stream) {
  if (!ws) return WKV_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  int rc = cuda_rc(cudaStreamSynchronize(st));
  if (rc != WKV_OK) return rc;
  int status = 0;
  WsHeader *h = static_cast<WsHeader *>(ws);
  if ((rc = cuda_rc(cudaMemcpy(&status, &h->status, sizeof(int), cudaMemcpyDeviceToHost))) != WKV_OK) return rc;
  if (status != 0 && (rc = cuda_rc(cudaMemset(&h->status, 0, sizeof(int)))) != WKV_OK) return rc;
  return status;
}

const char *wkv_strerror(int status) {
  switch (status) {
    case WKV_OK: return "success";
    case WKV_ERR_INVALID_ARG: return "invalid argument (NULL pointer, size out of range, bad dtype)";
    case WKV_ERR_UNSUPPORTED: return "unsupported layout (misaligned pointer or overlapping buffers)";
    case WKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case WKV_ERR_CUDA: return "CUDA runtime error or failed kernel launch";
    case WKV_ERR_TIMEOUT: return "a bounded device-side wait gave up (results invalid)";
    default: return "unknown status";
  }
}

int wkv_version(void) { return WKV_VERSION; }

int wkv_last_cuda_error(void) { return t_last_cuda_error; }

const char *wkv_cuda_error_name(int err) { return cudaGetErrorName((cudaError_t)err); }

}  // extern "C"
