"""GPU parity: every libwkv entry point against the float64 oracle.

All calls go through the C ABI (the package's tensor helpers only marshal
pointers).  Inputs are the seeded workloads of ``rwkv_linear_rnn_b200.workloads``
at their full sizes, every output element compared (the OpenMP oracle runs
every chain of the largest workloads in seconds), plus small and ragged
shapes that exercise tile edges.
"""
import numpy as np
import pytest
import torch

import oracle
import rwkv_linear_rnn_b200 as W
from rwkv_linear_rnn_b200 import abi, workloads
from gpu_util import (BF16_TOL, F32_FWD_TOL, F32_GRAD_TOL, dev, fwd_err, host,
                      inputs_to_device, rel_l2, state_err)

pytestmark = pytest.mark.gpu

KERNELS = {"seq": W.WKV_KERNEL_SEQUENTIAL, "chunked": W.WKV_KERNEL_CHUNKED,
           "chunked_regs": W.WKV_KERNEL_CHUNKED_REGS, "segment": W.WKV_KERNEL_SEGMENT,
           "cluster": W.WKV_KERNEL_CLUSTER, "tile": W.WKV_KERNEL_TILE, "chain": W.WKV_KERNEL_CHAIN}
BWD_KERNELS = {"chunked": W.WKV_KERNEL_CHUNKED, "segment": W.WKV_KERNEL_SEGMENT, "tile": W.WKV_KERNEL_TILE,
               "chain": W.WKV_KERNEL_CHAIN}


def small_case(B, T, C, seed, dtype="f32", td=(-3.0, 1.0), kstd=1.0, state=False):
    rng = np.random.default_rng(seed)
    w = (-np.exp(rng.uniform(*td, C))).astype(np.float32)
    u = rng.uniform(-1, 1, C).astype(np.float32)
    k = (rng.normal(0, kstd, (B, T, C))).astype(np.float32)
    v = rng.normal(size=(B, T, C)).astype(np.float32)
    g = rng.normal(size=(B, T, C)).astype(np.float32)
    if dtype == "bf16":
        k = workloads.bf16_to_f32(workloads.bf16_round(k))
        v = workloads.bf16_to_f32(workloads.bf16_round(v))
        g = workloads.bf16_to_f32(workloads.bf16_round(g))
    st = None
    if state:
        st = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                       rng.normal(0, 2, (B, C))]).astype(np.float32)
    return w, u, k, v, g, st


def to_dev_kv(x, dtype):
    return dev(x, torch.bfloat16 if dtype == "bf16" else torch.float32)


# ---------------------------------------------------------------- forward ---

@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("shape", [(1, 1, 64), (1, 2, 40), (2, 7, 33), (3, 200, 70),
                                   (2, 129, 64), (1, 1000, 96), (4, 64, 256)])
def test_forward_small_shapes(kernel, shape):
    B, T, C = shape
    w, u, k, v, _, _ = small_case(B, T, C, seed=T * 7 + C)
    y, s, _ = W.forward(dev(w), dev(u), dev(k), dev(v), want_state=True, kernel=KERNELS[kernel])
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v)
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_forward_with_state_in(kernel):
    B, T, C = 2, 300, 64
    w, u, k, v, _, st = small_case(B, T, C, seed=5, state=True)
    y, s, _ = W.forward(dev(w), dev(u), dev(k), dev(v), dev(st), want_state=True,
                        kernel=KERNELS[kernel])
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v, st)
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_forward_tiny_workload(kernel):
    inp = workloads.generate("tiny")
    w, u, k, v, _ = inputs_to_device(inp)
    y, s, _ = W.forward(w, u, k, v, want_state=True, kernel=KERNELS[kernel])
    y_ref = oracle.fwd_direct(inp["w"], inp["u"], inp["k"], inp["v"])
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL


def test_forward_rwkv169m_full():
    inp = workloads.generate("rwkv169m")
    w, u, k, v, _ = inputs_to_device(inp)
    y, s, _ = W.forward(w, u, k, v, want_state=True)
    y_ref, s_ref = oracle.fwd_recur(inp["w"], inp["u"], inp["k"], inp["v"])
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL
    # the defining O(T^2) sum at sampled points
    rng = np.random.default_rng(1)
    pb, pt, pc = (rng.integers(0, 8, 400), rng.integers(0, 1024, 400), rng.integers(0, 768, 400))
    yp = oracle.fwd_points(inp["w"], inp["u"], inp["k"], inp["v"], pb, pt, pc)
    assert fwd_err(host(y)[pb, pt, pc], yp) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", ["auto", "tile"])
def test_forward_rwkv1b5_bf16(kernel):
    inp = workloads.generate("rwkv1b5_bf16", grad=False)
    w, u, k, v, _ = inputs_to_device(inp)
    kid = W.WKV_KERNEL_AUTO if kernel == "auto" else KERNELS[kernel]
    y, s, _ = W.forward(w, u, k, v, want_state=True, kernel=kid)
    y_ref, s_ref = oracle.fwd_recur(inp["w"], inp["u"], inp["k"], inp["v"])
    assert fwd_err(host(y), y_ref) <= BF16_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL * 10


def test_forward_longctx():
    inp = workloads.generate("longctx", grad=False)
    w, u, k, v, _ = inputs_to_device(inp)
    y, s, _ = W.forward(w, u, k, v, want_state=True)
    y_ref, s_ref = oracle.fwd_recur(inp["w"], inp["u"], inp["k"], inp["v"])
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL


def test_sequential_equals_chunked_longctx_slice():
    inp = workloads.generate("longctx", T=8192, C=512, grad=False)
    w, u, k, v, _ = inputs_to_device(inp)
    y1, s1, _ = W.forward(w, u, k, v, want_state=True, kernel=W.WKV_KERNEL_SEQUENTIAL)
    y2, s2, _ = W.forward(w, u, k, v, want_state=True, kernel=W.WKV_KERNEL_CHUNKED)
    assert fwd_err(host(y1), host(y2)) <= 2 * F32_FWD_TOL
    assert state_err(host(s1), host(s2)) <= 2 * F32_FWD_TOL


@pytest.mark.parametrize("kernel", sorted(KERNELS))
def test_split_forward_equals_whole(kernel):
    B, T, C = 2, 700, 64
    w, u, k, v, _, _ = small_case(B, T, C, seed=9)
    W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
    y, s, _ = W.forward(W_, U_, K_, V_, want_state=True, kernel=KERNELS[kernel])
    y1, s1, _ = W.forward(W_, U_, K_[:, :333].contiguous(), V_[:, :333].contiguous(),
                          want_state=True, kernel=KERNELS[kernel])
    y2, s2, _ = W.forward(W_, U_, K_[:, 333:].contiguous(), V_[:, 333:].contiguous(), s1,
                          want_state=True, kernel=KERNELS[kernel])
    assert fwd_err(host(torch.cat([y1, y2], 1)), host(y)) <= 2 * F32_FWD_TOL
    assert state_err(host(s2), host(s)) <= 2 * F32_FWD_TOL


def test_zero_length_forward():
    B, C = 2, 40
    w, u, _, _, _, st = small_case(B, 3, C, seed=10, state=True)
    k = torch.empty((B, 0, C), device="cuda")
    y, s, _ = W.forward(dev(w), dev(u), k, k.clone(), dev(st), want_state=True)
    assert y.shape == (B, 0, C)
    assert state_err(host(s), st) <= 1e-6


# ------------------------------------------------------------------- step ---

def test_steps_equal_forward():
    B, T, C = 3, 40, 68
    w, u, k, v, _, st = small_case(B, T, C, seed=11, state=True)
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v, st)
    s = dev(st)
    W_, U_ = dev(w), dev(u)
    ys = []
    for t in range(T):
        y_t, s = W.step(W_, U_, dev(k[:, t]), dev(v[:, t]), s)
        ys.append(host(y_t))
    assert fwd_err(np.stack(ys, 1), y_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL
    # and against the library's own forward
    yf, sf, _ = W.forward(W_, U_, dev(k), dev(v), dev(st), want_state=True)
    assert fwd_err(np.stack(ys, 1), host(yf)) <= 2 * F32_FWD_TOL


def test_step_scalar_path_and_out_of_place():
    N, C = 5, 7  # C % 4 != 0: scalar kernel
    w, u, k, v, _, st = small_case(N, 1, C, seed=12, state=True)
    s_in = dev(st)
    s_out = torch.empty_like(s_in)
    y, so = W.step(dev(w), dev(u), dev(k[:, 0]), dev(v[:, 0]), s_in, state_out=s_out)
    y_ref, s_ref = oracle.step(w, u, k[:, 0], v[:, 0], st)
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL
    assert state_err(host(so), s_ref) <= F32_FWD_TOL
    assert np.array_equal(host(s_in), st.astype(np.float64))  # input untouched


def test_decode14b_prefill_and_32_steps():
    d = workloads.generate_decode_steps("decode14b")
    N, C = d["N"], d["C"]
    w, u = dev(d["w"]), dev(d["u"])
    _, s, _ = W.forward(w, u, dev(d["k"]), dev(d["v"]), want_state=True)
    _, s_ref = oracle.fwd_recur(d["w"], d["u"], d["k"], d["v"])
    assert state_err(host(s), s_ref) <= F32_FWD_TOL
    worst = 0.0
    for i in range(d["k_steps"].shape[0]):
        y, s = W.step(w, u, dev(d["k_steps"][i]), dev(d["v_steps"][i]), s)
        y_ref, s_ref = oracle.step(d["w"], d["u"], d["k_steps"][i], d["v_steps"][i], s_ref)
        worst = max(worst, fwd_err(host(y), y_ref))
    assert worst <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL


# --------------------------------------------------------------- backward ---

def grads_ref(w, u, k, v, g, st=None):
    return oracle.bwd_recur(w, u, k, v, g, st)


def assert_grads(got, ref, tol):
    """Relative L2 per tensor.  A reference that is zero up to rounding (dL/dw
    and dL/du when T = 1: no past token, and y_0 = v_0) has no relative error;
    there the bound applies to the absolute error instead."""
    names = ("gw", "gu", "gk", "gv")
    for n, a, b in zip(names, got, ref):
        x = host(a)
        if np.linalg.norm(b) <= 1e-9 * np.sqrt(b.size):
            assert np.max(np.abs(x)) <= tol, (n, np.max(np.abs(x)))
            continue
        e = rel_l2(x, b)
        assert e <= tol, (n, e)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
@pytest.mark.parametrize("use_ckpt", [True, False])
@pytest.mark.parametrize("shape", [(1, 1, 64), (2, 7, 33), (3, 200, 70), (2, 129, 64),
                                   (1, 1000, 96), (2, 300, 40)])
def test_backward_small_shapes(shape, use_ckpt, kernel):
    B, T, C = shape
    w, u, k, v, g, _ = small_case(B, T, C, seed=T + 3 * C)
    W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
    ck = None
    if use_ckpt:
        _, _, ck = W.forward(W_, U_, K_, V_, want_ckpt=True)
    got = W.backward(W_, U_, K_, V_, dev(g), ckpt=ck, kernel=BWD_KERNELS[kernel])
    assert_grads(got, grads_ref(w, u, k, v, g), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_backward_with_state_in(kernel):
    B, T, C = 2, 300, 64
    w, u, k, v, g, st = small_case(B, T, C, seed=13, state=True)
    got = W.backward(dev(w), dev(u), dev(k), dev(v), dev(g), dev(st), kernel=BWD_KERNELS[kernel])
    assert_grads(got, grads_ref(w, u, k, v, g, st), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_backward_bf16_small(kernel):
    B, T, C = 2, 333, 64
    w, u, k, v, g, _ = small_case(B, T, C, seed=19, dtype="bf16")
    bf = lambda x: dev(x, torch.bfloat16)
    got = W.backward(dev(w), dev(u), bf(k), bf(v), bf(g), kernel=BWD_KERNELS[kernel])
    assert_grads(got, grads_ref(w, u, k, v, g), BF16_TOL)


# Cases that steer the segment kernels' batch fast path and its fallback:
# keys spread over hundreds of binades (fallback), a dominant early spike
# followed by small keys, and a near-zero decay over a long sequence (the
# undecayed mode, where a repeated decay factor would accumulate rounding).
RANGE_CASES = {
    "wide_keys": dict(B=2, T=700, C=64, td=(-6.0, 3.0), kstd=40.0),
    "near_zero_decay": dict(B=1, T=6000, C=64, td=(-9.0, -6.0), kstd=1.0),
    "strong_decay": dict(B=2, T=500, C=64, td=(1.5, 3.0), kstd=2.0),
}


def _range_case(name, seed):
    c = RANGE_CASES[name]
    w, u, k, v, g, _ = small_case(c["B"], c["T"], c["C"], seed=seed, td=c["td"], kstd=c["kstd"])
    if name == "wide_keys":
        k[:, 5, :] = 60.0   # an early spike that dominates the state for a while
        k[:, 300:340, :] = -80.0
    return w, u, k, v, g


@pytest.mark.parametrize("kernel", ["segment", "cluster", "tile", "chain"])
@pytest.mark.parametrize("name", sorted(RANGE_CASES))
def test_segment_forward_ranges(name, kernel):
    w, u, k, v, g = _range_case(name, seed=41)
    y, _, _ = W.forward(dev(w), dev(u), dev(k), dev(v), kernel=KERNELS[kernel])
    y_ref, _ = oracle.fwd_recur(w, u, k, v)
    assert fwd_err(host(y), y_ref) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", ["segment", "tile", "chain"])
@pytest.mark.parametrize("name", sorted(RANGE_CASES))
def test_segment_backward_ranges(name, kernel):
    w, u, k, v, g = _range_case(name, seed=43)
    W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
    _, _, ck = W.forward(W_, U_, K_, V_, want_ckpt=True, kernel=KERNELS[kernel])
    got = W.backward(W_, U_, K_, V_, dev(g), ckpt=ck, kernel=BWD_KERNELS[kernel])
    assert_grads(got, grads_ref(w, u, k, v, g), F32_GRAD_TOL)


def test_backward_tiny_workload_vs_direct():
    inp = workloads.generate("tiny")
    w, u, k, v, gy = inputs_to_device(inp)
    _, _, ck = W.forward(w, u, k, v, want_ckpt=True)
    got = W.backward(w, u, k, v, gy, ckpt=ck)
    ref = oracle.bwd_direct(inp["w"], inp["u"], inp["k"], inp["v"], inp["gy"])
    assert_grads(got, ref, F32_GRAD_TOL)


def test_backward_rwkv169m_full():
    inp = workloads.generate("rwkv169m")
    w, u, k, v, gy = inputs_to_device(inp)
    _, _, ck = W.forward(w, u, k, v, want_ckpt=True)
    got = W.backward(w, u, k, v, gy, ckpt=ck)
    ref = grads_ref(inp["w"], inp["u"], inp["k"], inp["v"], inp["gy"])
    assert_grads(got, ref, F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", ["auto", "tile"])
def test_backward_rwkv1b5_bf16_full(kernel):
    inp = workloads.generate("rwkv1b5_bf16")
    w, u, k, v, gy = inputs_to_device(inp)
    kid = W.WKV_KERNEL_AUTO if kernel == "auto" else KERNELS[kernel]
    _, _, ck = W.forward(w, u, k, v, want_ckpt=True, kernel=kid)
    got = W.backward(w, u, k, v, gy, ckpt=ck, kernel=kid)
    ref = grads_ref(inp["w"], inp["u"], inp["k"], inp["v"], inp["gy"])
    assert_grads(got, ref, BF16_TOL)
    # every channel of dL/dk and dL/dv, each on its own (a channel-wise fault
    # would hide in the whole tensor's relative L2)
    for name, a, b in (("gk", got[2], ref[2]), ("gv", got[3], ref[3])):
        x = host(a)
        num = np.sqrt(((x - b) ** 2).sum(axis=(0, 1)))
        den = np.sqrt((b ** 2).sum(axis=(0, 1)))
        assert np.max(num / den) <= BF16_TOL, (name, int(np.argmax(num / den)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_chain_kernels_over_more_chains_than_one_wave(dtype):
    """More chains (batch rows x 32-channel tiles) than four warps per SM can
    hold at once: the forward runs its blocks in several waves, the
    backward's warps take several chains each, and the batch rows' dL/dw,
    dL/du sums still meet."""
    B, T, C = 50, 100, 416  # 650 chains, a ragged channel tile
    w, u, k, v, g, _ = small_case(B, T, C, seed=51, dtype=dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K_, V_, G_ = dev(k, tdt), dev(v, tdt), dev(g, tdt)
    W_, U_ = dev(w), dev(u)
    y, s, ck = W.forward(W_, U_, K_, V_, want_state=True, want_ckpt=True, kernel=W.WKV_KERNEL_CHAIN)
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v)
    assert fwd_err(host(y), y_ref) <= (BF16_TOL if dtype == "bf16" else F32_FWD_TOL)
    assert state_err(host(s), s_ref) <= F32_FWD_TOL * (10 if dtype == "bf16" else 1)
    got = W.backward(W_, U_, K_, V_, G_, ckpt=ck, kernel=W.WKV_KERNEL_CHAIN)
    assert_grads(got, grads_ref(w, u, k, v, g), BF16_TOL if dtype == "bf16" else F32_GRAD_TOL)


def test_backward_deterministic():
    B, T, C = 4, 500, 96
    w, u, k, v, g, _ = small_case(B, T, C, seed=14)
    args = (dev(w), dev(u), dev(k), dev(v), dev(g))
    a = W.backward(*args)
    b = W.backward(*args)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_autograd_function_matches_oracle():
    B, T, C = 2, 150, 48
    w, u, k, v, g, _ = small_case(B, T, C, seed=15)
    tw, tu, tk, tv = (dev(x).requires_grad_(True) for x in (w, u, k, v))
    y = W.wkv(tw, tu, tk, tv)
    (y * dev(g)).sum().backward()
    ref = grads_ref(w, u, k, v, g)
    assert_grads((tw.grad, tu.grad, tk.grad, tv.grad), ref, F32_GRAD_TOL)


# -------------------------------------------------- failure and edge paths ---

@pytest.mark.parametrize("kernel", ["chunked", "segment", "tile"])
def test_timeout_is_reported_and_context_survives(kernel):
    """The first chunk (segment) is told never to publish its record: the
    warps that wait on it give up after a short bounded wait, the status word
    reads WKV_ERR_TIMEOUT, and the next normal call works."""
    B, T, C = 1, 1024, 64
    kid = KERNELS[kernel]
    w, u, k, v, _, _ = small_case(B, T, C, seed=16)
    W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
    ws = W.Workspace()
    buf, nb = ws.get(W.WKV_OP_FORWARD, B, T, C, W.WKV_F32)
    y = torch.empty_like(K_)
    opt = abi.Options(kernel=kid, test_hold_first_chunk=1, spin_limit=2000)
    stream = torch.cuda.current_stream().cuda_stream
    rc = abi.wkv_forward_ex(B, T, C, 0, W_.data_ptr(), U_.data_ptr(), K_.data_ptr(), V_.data_ptr(),
                            0, y.data_ptr(), 0, 0, buf.data_ptr(), nb, stream, opt)
    assert rc == 0
    assert ws.status() == abi.WKV_ERR_TIMEOUT
    assert ws.status() == 0  # cleared by the read
    y2, _, _ = W.forward(W_, U_, K_, V_, workspace=ws, kernel=kid)
    assert ws.status() == 0
    y_ref, _ = oracle.fwd_recur(w, u, k, v)
    assert fwd_err(host(y2), y_ref) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", ["segment", "tile"])
def test_backward_timeout_is_reported_and_context_survives(kernel):
    """The backward with the last segment's (unit's) record held back: the
    waits and the grid barrier stay bounded, the status reads WKV_ERR_TIMEOUT,
    and the next call on the same workspace is correct."""
    B, T, C = 1, 1024, 64
    w, u, k, v, g, _ = small_case(B, T, C, seed=18)
    W_, U_, K_, V_, G_ = dev(w), dev(u), dev(k), dev(v), dev(g)
    ws = W.Workspace()
    _, _, ck = W.forward(W_, U_, K_, V_, want_ckpt=True, workspace=ws)
    buf, nb = ws.get(W.WKV_OP_BACKWARD, B, T, C, W.WKV_F32)
    gw = torch.empty(C, device="cuda"); gu = torch.empty(C, device="cuda")
    gk = torch.empty_like(K_); gv = torch.empty_like(V_)
    opt = abi.Options(kernel=BWD_KERNELS[kernel], test_hold_first_chunk=1, spin_limit=2000)
    stream = torch.cuda.current_stream().cuda_stream
    P = lambda t: t.data_ptr()
    rc = abi.wkv_backward_ex(B, T, C, 0, P(W_), P(U_), P(K_), P(V_), P(G_), 0, P(ck), P(gw), P(gu),
                             P(gk), P(gv), P(buf), nb, stream, opt)
    assert rc == 0
    assert ws.status() == abi.WKV_ERR_TIMEOUT
    got = W.backward(W_, U_, K_, V_, G_, ckpt=ck, workspace=ws, kernel=BWD_KERNELS[kernel])
    assert ws.status() == 0
    assert_grads(got, grads_ref(w, u, k, v, g), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", ["segment", "tile", "chain"])
def test_segment_backward_reuses_a_workspace_across_shapes(kernel):
    """One workspace, shapes in decreasing then increasing size: whatever an
    earlier call left in the workspace does not leak into a later result."""
    ws = W.Workspace()
    for (B, T, C) in [(3, 1000, 96), (2, 129, 64), (1, 300, 32), (3, 1000, 96)]:
        w, u, k, v, g, _ = small_case(B, T, C, seed=B + T + C)
        W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
        _, _, ck = W.forward(W_, U_, K_, V_, want_ckpt=True, workspace=ws)
        got = W.backward(W_, U_, K_, V_, dev(g), ckpt=ck, workspace=ws, kernel=BWD_KERNELS[kernel])
        assert ws.status() == 0
        assert_grads(got, grads_ref(w, u, k, v, g), F32_GRAD_TOL)


@pytest.mark.parametrize("fwd_kernel", ["segment", "tile", "chain"])
def test_segment_outputs_stay_inside_their_buffers(fwd_kernel):
    B, T, C = 2, 300, 96
    w, u, k, v, g, _ = small_case(B, T, C, seed=27)
    n = B * T * C
    guard = 4096
    bufs = [torch.full((n + 2 * guard,), 12345.0, device="cuda") for _ in range(3)]
    y, gk, gv = (b_[guard:guard + n].view(B, T, C) for b_ in bufs)
    W_, U_, K_, V_ = dev(w), dev(u), dev(k), dev(v)
    _, _, ck = W.forward(W_, U_, K_, V_, y=y, want_ckpt=True, kernel=KERNELS[fwd_kernel])
    W.backward(W_, U_, K_, V_, dev(g), ckpt=ck, grad_k=gk, grad_v=gv, kernel=BWD_KERNELS[fwd_kernel])
    torch.cuda.synchronize()
    for b_ in bufs:
        assert torch.all(b_[:guard] == 12345.0) and torch.all(b_[guard + n:] == 12345.0)


def test_outputs_do_not_write_outside_their_buffers():
    B, T, C = 2, 300, 70
    w, u, k, v, g, _ = small_case(B, T, C, seed=17)
    n = B * T * C
    guard = 4096
    ybuf = torch.full((n + 2 * guard,), 12345.0, device="cuda")
    y = ybuf[guard:guard + n].view(B, T, C)
    W.forward(dev(w), dev(u), dev(k), dev(v), y=y, kernel=W.WKV_KERNEL_CHUNKED)
    W.forward(dev(w), dev(u), dev(k), dev(v), y=y, kernel=W.WKV_KERNEL_SEQUENTIAL)
    torch.cuda.synchronize()
    assert torch.all(ybuf[:guard] == 12345.0) and torch.all(ybuf[guard + n:] == 12345.0)


def test_argument_errors_launch_nothing():
    C = 64
    w = torch.zeros(C, device="cuda")
    k = torch.zeros((1, 8, C), device="cuda")
    y = torch.zeros_like(k)
    s = torch.cuda.current_stream().cuda_stream
    p = lambda t: t.data_ptr()
    assert abi.wkv_forward(1, 8, C, 5, p(w), p(w), p(k), p(k), 0, p(y), 0, 0, 0, 0, s) == -1
    assert abi.wkv_forward(1, 8, C, 0, p(w), p(w), p(k), p(k), 0, p(k), 0, 0, 0, 0, s) == -2
    assert abi.wkv_forward(1, 8, C, 0, p(w), p(w), p(k) + 1, p(k), 0, p(y), 0, 0, 0, 0, s) == -2
    assert abi.wkv_forward_ex(1, 8, C, 0, p(w), p(w), p(k), p(k), 0, p(y), 0, 0, 0, 0, s,
                              abi.Options(kernel=2)) == -3
    torch.cuda.synchronize()


@pytest.mark.parametrize("kernel", ["tile", "chain"])
def test_tile_results_are_bit_reproducible_at_full_size(kernel):
    """The tile kernels' look-backs take whatever prefix is published first,
    but every prefix is the same left fold of unit records; the chain
    kernels add the batch rows' dL/dw, dL/du in a fixed order whichever
    finishes first: two runs of the RWKV-4 169M-shaped layer give identical
    bits."""
    inp = workloads.generate("rwkv169m")
    w, u, k, v, gy = inputs_to_device(inp)
    runs = []
    for _ in range(2):
        y, s, ck = W.forward(w, u, k, v, want_state=True, want_ckpt=True, kernel=KERNELS[kernel])
        grads = W.backward(w, u, k, v, gy, ckpt=ck, kernel=KERNELS[kernel])
        runs.append((y, s, ck) + tuple(grads))
    for a, b in zip(*runs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("kernel", ["tile", "chain"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [1, 15, 16, 17, 32, 33, 48, 64, 65, 96, 129])
def test_tile_unit_boundaries(T, dtype, kernel):
    """Lengths at and just past one and two tile units (32 fp32 / 64 bf16
    tokens) and the batches inside them (16 tokens): a chain of a single
    unit, a ragged last unit and batch, and the group boundaries of the
    backward's fixed-order sums."""
    kid = KERNELS[kernel]
    B, C = 3, 96
    w, u, k, v, g, _ = small_case(B, T, C, seed=T * 11 + len(dtype), dtype=dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K_, V_, G_ = dev(k, tdt), dev(v, tdt), dev(g, tdt)
    W_, U_ = dev(w), dev(u)
    y, s, ck = W.forward(W_, U_, K_, V_, want_state=True, want_ckpt=True, kernel=kid)
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v)
    tol_f = BF16_TOL if dtype == "bf16" else F32_FWD_TOL
    assert fwd_err(host(y), y_ref) <= tol_f
    assert state_err(host(s), s_ref) <= F32_FWD_TOL * (10 if dtype == "bf16" else 1)
    got = W.backward(W_, U_, K_, V_, G_, ckpt=ck, kernel=kid)
    assert_grads(got, grads_ref(w, u, k, v, g), BF16_TOL if dtype == "bf16" else F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", ["segment", "tile", "chain"])
def test_cached_tensor_maps_follow_shape_changes(kernel):
    """The library remembers encoded tensor maps by (address, shape, dtype,
    box).  One pair of buffers viewed as several shapes in turn (same base
    address, different extents), then the first shape again: every call
    matches the oracle, and the repeated shape gives the same bits as its
    first call."""
    kern = KERNELS[kernel]
    C = 64
    cap = 3 * 400 * C
    kbuf = torch.empty(cap, device="cuda")
    vbuf = torch.empty(cap, device="cuda")
    gbuf = torch.empty(cap, device="cuda")
    seen = {}
    for call, (B, T) in enumerate([(3, 400), (2, 150), (1, 400), (3, 97), (3, 400)]):
        w, u, k, v, g, _ = small_case(B, T, C, seed=200 + B * T)
        n = B * T * C
        K_, V_, G_ = (buf[:n].view(B, T, C) for buf in (kbuf, vbuf, gbuf))
        K_.copy_(dev(k)), V_.copy_(dev(v)), G_.copy_(dev(g))
        W_, U_ = dev(w), dev(u)
        y, _, ck = W.forward(W_, U_, K_, V_, want_ckpt=True, kernel=kern)
        gw, gu, gk, gv = W.backward(W_, U_, K_, V_, G_, ckpt=ck, kernel=BWD_KERNELS[kernel])
        assert fwd_err(host(y), oracle.fwd_recur(w, u, k, v)[0]) <= F32_FWD_TOL, call
        assert_grads((gw, gu, gk, gv), grads_ref(w, u, k, v, g), F32_GRAD_TOL)
        out = (y.clone(), gw.clone(), gu.clone(), gk.clone(), gv.clone())
        if (B, T) in seen:
            for a, b in zip(seen[(B, T)], out):
                assert torch.equal(a, b), call
        seen[(B, T)] = out
