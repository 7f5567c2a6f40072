"""GPU parity of the gated entry points (o = sigma(r) * wkv) against the
float64 oracle's ``fwd_gated`` / ``bwd_gated``.

The gate is the time-mixing block's receptance gate (RWKV paper review,
section "출력 게이팅(Output Gating)").  Covered: every forward kernel (the
segment forward fuses the gate, the others gate in a separate pass), both
backward kernels (the segment backward fuses it), rows that are not 16-byte
aligned (the unfused path under the default selector), bf16, state_in,
checkpoint reuse with the ungated calls, T = 0, buffer guards, the
autograd wrapper and the full rwkv169m workload.
"""
import numpy as np
import pytest
import torch

import oracle
import rwkv_linear_rnn_b200 as W
from rwkv_linear_rnn_b200 import workloads
from gpu_util import (BF16_TOL, F32_FWD_TOL, F32_GRAD_TOL, dev, dev_bf16_bits, fwd_err, host,
                      inputs_to_device, rel_l2, state_err)

pytestmark = pytest.mark.gpu

KERNELS = {"seq": W.WKV_KERNEL_SEQUENTIAL, "chunked": W.WKV_KERNEL_CHUNKED,
           "chunked_regs": W.WKV_KERNEL_CHUNKED_REGS, "segment": W.WKV_KERNEL_SEGMENT,
           "cluster": W.WKV_KERNEL_CLUSTER, "tile": W.WKV_KERNEL_TILE, "chain": W.WKV_KERNEL_CHAIN}
BWD_KERNELS = {"chunked": W.WKV_KERNEL_CHUNKED, "segment": W.WKV_KERNEL_SEGMENT, "tile": W.WKV_KERNEL_TILE, "chain": W.WKV_KERNEL_CHAIN}


def gated_case(B, T, C, seed, dtype="f32", rstd=1.5, state=False):
    rng = np.random.default_rng(seed)
    w = (-np.exp(rng.uniform(-3.0, 1.0, C))).astype(np.float32)
    u = rng.uniform(-1, 1, C).astype(np.float32)
    k, v, r, g = (rng.normal(size=(B, T, C)).astype(np.float32) for _ in range(4))
    r *= np.float32(rstd)
    if dtype == "bf16":
        k, v, r, g = (workloads.bf16_to_f32(workloads.bf16_round(x)) for x in (k, v, r, g))
    st = None
    if state:
        st = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                       rng.normal(0, 2, (B, C))]).astype(np.float32)
    return w, u, k, v, r, g, st


def shifted(x, dtype=torch.float32):
    """A device copy whose data starts one element past a 16-byte boundary."""
    flat = torch.empty(x.size + 1, dtype=dtype, device="cuda")
    flat[1:] = torch.from_numpy(np.ascontiguousarray(x).ravel()).to("cuda").to(dtype)
    return flat[1:].view(x.shape)


def assert_grads5(got, ref, tol):
    for n, a, b in zip(("gw", "gu", "gk", "gv", "gr"), got, ref):
        x = host(a)
        if np.linalg.norm(b) <= 1e-9 * np.sqrt(b.size):
            assert np.max(np.abs(x)) <= tol, (n, np.max(np.abs(x)))
            continue
        e = rel_l2(x, b)
        assert e <= tol, (n, e)


SHAPES = [(1, 1, 64), (2, 7, 33), (3, 200, 70), (2, 129, 64), (1, 1000, 96), (4, 64, 256)]


@pytest.mark.parametrize("kernel", sorted(KERNELS))
@pytest.mark.parametrize("shape", SHAPES)
def test_forward_gated_small_shapes(kernel, shape):
    B, T, C = shape
    w, u, k, v, r, _, _ = gated_case(B, T, C, seed=T * 5 + C)
    o, s, _ = W.forward_gated(dev(w), dev(u), dev(k), dev(v), dev(r), want_state=True,
                              kernel=KERNELS[kernel])
    o_ref, s_ref = oracle.fwd_gated(w, u, k, v, r)
    assert fwd_err(host(o), o_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", ["segment", "chunked", "chain"])
def test_forward_gated_state_in_and_extreme_gate(kernel):
    B, T, C = 2, 300, 64
    w, u, k, v, r, _, st = gated_case(B, T, C, seed=6, rstd=30.0, state=True)
    r[:, :5, :] = 200.0   # open (sigma = 1 exactly in float32)
    r[:, 5:9, :] = -200.0  # shut (e^{200} overflows float32: sigma = 0)
    o, s, _ = W.forward_gated(dev(w), dev(u), dev(k), dev(v), dev(r), dev(st), want_state=True,
                              kernel=KERNELS[kernel])
    o_ref, s_ref = oracle.fwd_gated(w, u, k, v, r, st)
    assert fwd_err(host(o), o_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL
    assert np.all(host(o)[:, 5:9, :] == 0.0)


def test_forward_gated_unaligned_gate_input():
    """r one element off a 16-byte boundary: the default selector gates in a
    separate pass."""
    B, T, C = 2, 257, 64
    w, u, k, v, r, _, _ = gated_case(B, T, C, seed=7)
    o, _, _ = W.forward_gated(dev(w), dev(u), dev(k), dev(v), shifted(r))
    o_ref, _ = oracle.fwd_gated(w, u, k, v, r)
    assert fwd_err(host(o), o_ref) <= F32_FWD_TOL


def test_forward_gated_keeps_the_recurrence():
    """State and checkpoints of the gated forward are the ungated ones, bit
    for bit (the gate does not enter the recurrence)."""
    B, T, C = 3, 500, 96
    w, u, k, v, r, _, _ = gated_case(B, T, C, seed=8)
    a = (dev(w), dev(u), dev(k), dev(v))
    y, s0, c0 = W.forward(*a, want_state=True, want_ckpt=True)
    o, s1, c1 = W.forward_gated(*a, dev(r), want_state=True, want_ckpt=True)
    assert torch.equal(s0, s1) and torch.equal(c0, c1)
    assert fwd_err(host(o), oracle.sigmoid(r) * host(y)) <= F32_FWD_TOL


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
@pytest.mark.parametrize("use_ckpt", [True, False])
@pytest.mark.parametrize("shape", SHAPES[:5] + [(2, 300, 40)])
def test_backward_gated_small_shapes(shape, use_ckpt, kernel):
    B, T, C = shape
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=T + 7 * C)
    W_, U_, K_, V_, R_ = dev(w), dev(u), dev(k), dev(v), dev(r)
    ck = None
    if use_ckpt:
        _, _, ck = W.forward_gated(W_, U_, K_, V_, R_, want_ckpt=True)
    got = W.backward_gated(W_, U_, K_, V_, R_, dev(g), ckpt=ck, kernel=BWD_KERNELS[kernel])
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_backward_gated_state_in(kernel):
    B, T, C = 2, 300, 64
    w, u, k, v, r, g, st = gated_case(B, T, C, seed=9, state=True)
    got = W.backward_gated(dev(w), dev(u), dev(k), dev(v), dev(r), dev(g), dev(st),
                           kernel=BWD_KERNELS[kernel])
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g, st), F32_GRAD_TOL)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gated_chain_kernels_over_more_chains_than_one_wave(dtype):
    """The gated chain forward and backward with more chains than four warps
    per SM hold at once (several waves of blocks forward; several chains per
    warp backward, with the batch rows' dL/dw, dL/du sums meeting)."""
    B, T, C = 50, 100, 416  # 650 chains, a ragged channel tile
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=52, dtype=dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    W_, U_ = dev(w), dev(u)
    K_, V_, R_, G_ = (dev(x, tdt) for x in (k, v, r, g))
    o, s, ck = W.forward_gated(W_, U_, K_, V_, R_, want_state=True, want_ckpt=True,
                               kernel=W.WKV_KERNEL_CHAIN)
    o_ref, s_ref = oracle.fwd_gated(w, u, k, v, r)
    tol = BF16_TOL if dtype == "bf16" else F32_FWD_TOL
    assert fwd_err(host(o), o_ref) <= tol
    assert state_err(host(s), s_ref) <= F32_FWD_TOL * (10 if dtype == "bf16" else 1)
    got = W.backward_gated(W_, U_, K_, V_, R_, G_, ckpt=ck, kernel=W.WKV_KERNEL_CHAIN)
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), BF16_TOL if dtype == "bf16" else F32_GRAD_TOL)


def test_backward_gated_unaligned_gate_input():
    B, T, C = 2, 300, 64
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=10)
    got = W.backward_gated(dev(w), dev(u), dev(k), dev(v), shifted(r), dev(g))
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


def test_backward_gated_unaligned_grad_k():
    """The fused backward reads grad_k's rows back through TMA, so grad_k off
    a 16-byte boundary takes the unfused path."""
    B, T, C = 2, 300, 64
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=18)
    gk = torch.empty(B * T * C + 1, device="cuda")[1:].view(B, T, C)
    got = W.backward_gated(dev(w), dev(u), dev(k), dev(v), dev(r), dev(g), grad_k=gk)
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


def test_backward_gated_wide_keys():
    """Keys over hundreds of binades (the segment kernels' slow path) with a
    saturated gate on part of the sequence."""
    B, T, C = 2, 700, 64
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=11, rstd=20.0)
    k *= 40.0
    k[:, 5, :] = 60.0
    W_, U_, K_, V_, R_ = dev(w), dev(u), dev(k), dev(v), dev(r)
    _, _, ck = W.forward_gated(W_, U_, K_, V_, R_, want_ckpt=True)
    got = W.backward_gated(W_, U_, K_, V_, R_, dev(g), ckpt=ck)
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_gated_bf16_small(kernel):
    B, T, C = 2, 333, 64
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=12, dtype="bf16")
    bf = lambda x: dev(x, torch.bfloat16)
    o, _, _ = W.forward_gated(dev(w), dev(u), bf(k), bf(v), bf(r), kernel=KERNELS[kernel])
    assert fwd_err(host(o), oracle.fwd_gated(w, u, k, v, r)[0]) <= BF16_TOL
    got = W.backward_gated(dev(w), dev(u), bf(k), bf(v), bf(r), bf(g), kernel=BWD_KERNELS[kernel])
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), BF16_TOL)


def test_gated_zero_length():
    B, C = 2, 64
    w, u, _, _, _, _, st = gated_case(B, 1, C, seed=13, state=True)
    e = torch.empty((B, 0, C), device="cuda")
    o, s, _ = W.forward_gated(dev(w), dev(u), e, e, e, dev(st), want_state=True)
    assert o.numel() == 0
    assert state_err(host(s), st.astype(np.float64)) <= F32_FWD_TOL
    gw, gu, gk, gv, gr = W.backward_gated(dev(w), dev(u), e, e, e, e, dev(st))
    assert torch.all(gw == 0) and torch.all(gu == 0) and gr.numel() == 0


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_gated_outputs_stay_inside_their_buffers(kernel):
    B, T, C = 2, 301, 96
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=14)
    n = B * T * C
    pad = 4096
    bufs = [torch.full((n + 2 * pad,), 7.0, device="cuda") for _ in range(4)]
    o, gk, gv, gr = (b[pad:pad + n].view(B, T, C) for b in bufs)
    W_, U_, K_, V_, R_ = dev(w), dev(u), dev(k), dev(v), dev(r)
    _, _, ck = W.forward_gated(W_, U_, K_, V_, R_, o=o, want_ckpt=True, kernel=KERNELS[kernel])
    W.backward_gated(W_, U_, K_, V_, R_, dev(g), ckpt=ck, grad_k=gk, grad_v=gv, grad_r=gr,
                     kernel=BWD_KERNELS[kernel])
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:pad] == 7.0) and torch.all(b[pad + n:] == 7.0)


@pytest.mark.parametrize("form", ["grad_arg", "sum"])
def test_gated_autograd_matches_oracle(form):
    B, T, C = 2, 150, 48
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=15)
    ts = [dev(x).requires_grad_() for x in (w, u, k, v, r)]
    o = W.gated_wkv(*ts)
    if form == "sum":
        (o * dev(g)).sum().backward()
    else:
        o.backward(dev(g))
    assert fwd_err(host(o), oracle.fwd_gated(w, u, k, v, r)[0]) <= F32_FWD_TOL
    assert_grads5([t.grad for t in ts], oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


def test_gated_direct_calls_partial_channel_tile():
    """C = 48: the second 32-channel tile is half outside the rows."""
    B, T, C = 2, 150, 48
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=15)
    W_, U_, K_, V_, R_ = dev(w), dev(u), dev(k), dev(v), dev(r)
    o, _, ck = W.forward_gated(W_, U_, K_, V_, R_, want_ckpt=True)
    assert fwd_err(host(o), oracle.fwd_gated(w, u, k, v, r)[0]) <= F32_FWD_TOL
    got = W.backward_gated(W_, U_, K_, V_, R_, dev(g), ckpt=ck)
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


def test_gated_deterministic():
    B, T, C = 4, 500, 96
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=16)
    args = (dev(w), dev(u), dev(k), dev(v), dev(r), dev(g))
    a = W.backward_gated(*args)
    b = W.backward_gated(*args)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_gated_rwkv169m_full():
    """The full rwkv169m workload (B 8, T 1024, C 768, fp32) with a gate
    input N(0, 1), in the launch configuration the benchmark times."""
    inp = workloads.generate("rwkv169m", gate=True)
    w, u, k, v, go = inputs_to_device(inp)
    r = dev(inp["r"])
    o, s, ck = W.forward_gated(w, u, k, v, r, want_state=True, want_ckpt=True)
    o_ref, s_ref = oracle.fwd_gated(inp["w"], inp["u"], inp["k"], inp["v"], inp["r"])
    assert fwd_err(host(o), o_ref) <= F32_FWD_TOL
    assert state_err(host(s), s_ref) <= F32_FWD_TOL
    got = W.backward_gated(w, u, k, v, r, go, ckpt=ck)
    ref = oracle.bwd_gated(inp["w"], inp["u"], inp["k"], inp["v"], inp["r"], inp["gy"])
    assert_grads5(got, ref, F32_GRAD_TOL)


def test_gated_rwkv1b5_bf16_full():
    inp = workloads.generate("rwkv1b5_bf16", gate=True)
    w, u, k, v, go = inputs_to_device(inp)
    r = dev_bf16_bits(inp["r_bits"])
    o, _, ck = W.forward_gated(w, u, k, v, r, want_ckpt=True)
    got = W.backward_gated(w, u, k, v, r, go, ckpt=ck)
    args = (inp["w"], inp["u"], inp["k"], inp["v"], inp["r"])
    assert fwd_err(host(o), oracle.fwd_gated(*args)[0]) <= BF16_TOL
    assert_grads5(got, oracle.bwd_gated(*args, inp["gy"]), BF16_TOL)


def test_calls_from_a_fresh_thread():
    """A host thread whose first CUDA use is this library has no current
    context until the runtime binds one; the tensor maps the segment kernels
    need are encoded through the driver API, so the library binds it.  (An
    autograd worker thread is such a thread.)  Buffers are allocated here and
    the thread makes only libwkv calls."""
    import threading
    from rwkv_linear_rnn_b200 import abi
    B, T, C = 2, 150, 48
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=17)
    W_, U_, K_, V_, R_, G_ = (dev(x) for x in (w, u, k, v, r, g))
    o, gk, gv, gr = (torch.empty_like(K_) for _ in range(4))
    gw, gu = torch.empty(C, device="cuda"), torch.empty(C, device="cuda")
    ck = torch.empty(W.wkv_ckpt_size(B, T, C) // 4, device="cuda")
    nws = W.wkv_workspace_size(W.WKV_OP_BACKWARD, B, T, C, W.WKV_F32)
    ws = torch.zeros(nws, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    P = lambda t: t.data_ptr()
    rcs = []

    def work():
        rcs.append(abi.wkv_forward_gated(B, T, C, W.WKV_F32, P(W_), P(U_), P(K_), P(V_), P(R_), 0, P(o), 0,
                                         P(ck), P(ws), nws, 0))
        rcs.append(abi.wkv_backward_gated(B, T, C, W.WKV_F32, P(W_), P(U_), P(K_), P(V_), P(R_), P(G_), 0,
                                          P(ck), P(gw), P(gu), P(gk), P(gv), P(gr), P(ws), nws, 0))
        rcs.append(abi.wkv_get_status(P(ws), 0))

    th = threading.Thread(target=work)
    th.start()
    th.join()
    assert rcs == [0, 0, 0]
    assert fwd_err(host(o), oracle.fwd_gated(w, u, k, v, r)[0]) <= F32_FWD_TOL
    assert_grads5((gw, gu, gk, gv, gr), oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)


def test_gated_long_sequence_flag_join():
    """5000 tokens in one chain: more than 32 segments, so both segment
    kernels join through per-record flags instead of the grid barrier.
    (Warps holding several segments, with the gated backward's held
    second-pass loads, run in test_gated_rwkv1b5_bf16_full.)"""
    B, T, C = 1, 5000, 64
    w, u, k, v, r, g, _ = gated_case(B, T, C, seed=33)
    W_, U_, K_, V_, R_ = dev(w), dev(u), dev(k), dev(v), dev(r)
    o, _, ck = W.forward_gated(W_, U_, K_, V_, R_, want_ckpt=True)
    assert fwd_err(host(o), oracle.fwd_gated(w, u, k, v, r)[0]) <= F32_FWD_TOL
    got = W.backward_gated(W_, U_, K_, V_, R_, dev(g), ckpt=ck)
    assert_grads5(got, oracle.bwd_gated(w, u, k, v, r, g), F32_GRAD_TOL)
