"""GPU parity of the state gradients (``wkv_backward_state``) against the
float64 oracle's ``bwd_state``.

A sequence split across calls back-propagates through the recurrent state
(the RNN form of the RWKV paper review, section "RNN-유사추론"): a gradient
arrives at the final state and one leaves through the initial state.  Both
backward kernels are covered, with and without forward checkpoints, on
ragged shapes, wide key ranges, bf16, T = 0, the empty initial state, two
calls chained through the state against one call, the autograd wrapper, and
the full rwkv169m workload.

The final-state gradient refers to a representation (a, b, p) of the final
state; the tests pass the oracle's own final state (rounded to float32), so
no expected value depends on the CUDA path.
"""
import numpy as np
import pytest
import torch

import oracle
import rwkv_linear_rnn_b200 as W
from rwkv_linear_rnn_b200 import workloads
from gpu_util import BF16_TOL, F32_GRAD_TOL, dev, host, inputs_to_device, rel_l2

pytestmark = pytest.mark.gpu

BWD_KERNELS = {"chunked": W.WKV_KERNEL_CHUNKED, "segment": W.WKV_KERNEL_SEGMENT, "tile": W.WKV_KERNEL_TILE, "chain": W.WKV_KERNEL_CHAIN}


def state_case(B, T, C, seed, dtype="f32", kstd=1.0, td=(-3.0, 1.0)):
    rng = np.random.default_rng(seed)
    w = (-np.exp(rng.uniform(*td, C))).astype(np.float32)
    u = rng.uniform(-1, 1, C).astype(np.float32)
    k = (rng.normal(0, kstd, (B, T, C))).astype(np.float32)
    v = rng.normal(size=(B, T, C)).astype(np.float32)
    g = rng.normal(size=(B, T, C)).astype(np.float32)
    if dtype == "bf16":
        k, v, g = (workloads.bf16_to_f32(workloads.bf16_round(x)) for x in (k, v, g))
    s_in = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                     rng.normal(0, 2, (B, C))]).astype(np.float32)
    gso = rng.normal(size=(3, B, C)).astype(np.float32)
    # the final state's representation: the oracle's own, rounded to float32
    _, s_out = oracle.fwd_recur(w, u, k, v, s_in)
    return w, u, k, v, g, s_in, s_out.astype(np.float32), gso


def assert_grads_state(got, ref, tol):
    for n, a, b in zip(("gw", "gu", "gk", "gv", "gs_in"), got, ref):
        x = host(a)
        if np.linalg.norm(b) <= 1e-9 * np.sqrt(max(b.size, 1)):
            assert np.max(np.abs(x), initial=0.0) <= tol, (n, np.max(np.abs(x)))
            continue
        e = rel_l2(x, b)
        assert e <= tol, (n, e)


SHAPES = [(1, 1, 64), (2, 7, 33), (3, 200, 70), (2, 129, 64), (1, 1000, 96), (2, 300, 40)]


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
@pytest.mark.parametrize("use_ckpt", [True, False])
@pytest.mark.parametrize("shape", SHAPES)
def test_backward_state_small_shapes(shape, use_ckpt, kernel):
    B, T, C = shape
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=T + 11 * C)
    a = (dev(w), dev(u), dev(k), dev(v))
    ck = None
    if use_ckpt:
        _, _, ck = W.forward(*a, dev(s_in), want_ckpt=True)
    got = W.backward_state(*a, dev(g), dev(s_in), ck, state_out=dev(s_out), grad_state_out=dev(gso),
                           kernel=BWD_KERNELS[kernel])
    ref = oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso)
    assert_grads_state(got, ref, F32_GRAD_TOL)


@pytest.mark.parametrize("T", [100, 129])
def test_chain_state_backward_over_more_chains_than_one_wave(T):
    """The chain backward's state terms with more chains than four warps per
    SM hold at once: warps run several chains, each starting from its own
    final-state gradient; T = 129 ends in a one-token batch that must not
    sweep the zero-filled rows after it."""
    B, C = 50, 416  # 650 chains, a ragged channel tile
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=T + 3)
    a = (dev(w), dev(u), dev(k), dev(v))
    _, _, ck = W.forward(*a, dev(s_in), want_ckpt=True)
    got = W.backward_state(*a, dev(g), dev(s_in), ck, state_out=dev(s_out), grad_state_out=dev(gso),
                           kernel=W.WKV_KERNEL_CHAIN)
    ref = oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso)
    assert_grads_state(got, ref, F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_state_in_gradient_without_final_state_term(kernel):
    B, T, C = 2, 300, 64
    w, u, k, v, g, s_in, _, _ = state_case(B, T, C, seed=21)
    got = W.backward_state(dev(w), dev(u), dev(k), dev(v), dev(g), dev(s_in), kernel=BWD_KERNELS[kernel])
    assert_grads_state(got, oracle.bwd_state(w, u, k, v, g, s_in), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_empty_initial_state_gets_zero_gradient(kernel):
    B, T, C = 2, 130, 64
    w, u, k, v, g, _, _, gso = state_case(B, T, C, seed=22)
    _, s_out = oracle.fwd_recur(w, u, k, v)
    s_out = s_out.astype(np.float32)
    got = W.backward_state(dev(w), dev(u), dev(k), dev(v), dev(g), None, state_out=dev(s_out),
                           grad_state_out=dev(gso), kernel=BWD_KERNELS[kernel])
    ref = oracle.bwd_state(w, u, k, v, g, None, s_out, gso)
    assert torch.all(got[4] == 0)
    assert_grads_state(got[:4], ref[:4], F32_GRAD_TOL)


def test_backward_state_T0():
    B, C = 2, 64
    w, u, k, v, g, s_in, _, gso = state_case(B, 0, C, seed=23)
    rng = np.random.default_rng(1)
    s_out = np.stack([s_in[0], s_in[1], s_in[2] + rng.uniform(-1, 1, (B, C))]).astype(np.float32)
    e = torch.empty((B, 0, C), device="cuda")
    got = W.backward_state(dev(w), dev(u), e, e, e, dev(s_in), state_out=dev(s_out), grad_state_out=dev(gso))
    ref = oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso)
    assert torch.all(got[0] == 0) and torch.all(got[1] == 0)
    assert rel_l2(host(got[4]), ref[4]) <= 1e-6


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_backward_state_wide_keys(kernel):
    B, T, C = 2, 700, 64
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=24, kstd=40.0, td=(-6.0, 3.0))
    k[:, 5, :] = 60.0
    _, s_out = oracle.fwd_recur(w, u, k, v, s_in)
    s_out = s_out.astype(np.float32)
    got = W.backward_state(dev(w), dev(u), dev(k), dev(v), dev(g), dev(s_in), state_out=dev(s_out),
                           grad_state_out=dev(gso), kernel=BWD_KERNELS[kernel])
    assert_grads_state(got, oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso), F32_GRAD_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_backward_state_bf16(kernel):
    B, T, C = 2, 333, 64
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=25, dtype="bf16")
    bf = lambda x: dev(x, torch.bfloat16)
    got = W.backward_state(dev(w), dev(u), bf(k), bf(v), bf(g), dev(s_in), state_out=dev(s_out),
                           grad_state_out=dev(gso), kernel=BWD_KERNELS[kernel])
    assert_grads_state(got, oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso), BF16_TOL)


@pytest.mark.parametrize("kernel", sorted(BWD_KERNELS))
def test_two_calls_chained_through_the_state(kernel):
    """Forward in two calls (the second starts from the first's state_out),
    backward in reverse order with the second call's grad_state_in fed to the
    first: the gradients match the oracle's one-call backward."""
    B, T, C, t1 = 2, 520, 64, 200
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=26)
    kk = BWD_KERNELS[kernel]
    W_, U_ = dev(w), dev(u)
    K1, V1, G1 = dev(k[:, :t1]), dev(v[:, :t1]), dev(g[:, :t1])
    K2, V2, G2 = dev(k[:, t1:]), dev(v[:, t1:]), dev(g[:, t1:])
    _, S1, ck1 = W.forward(W_, U_, K1, V1, dev(s_in), want_state=True, want_ckpt=True)
    _, _, ck2 = W.forward(W_, U_, K2, V2, S1, want_ckpt=True)
    second = W.backward_state(W_, U_, K2, V2, G2, S1, ck2, state_out=dev(s_out), grad_state_out=dev(gso),
                              kernel=kk)
    first = W.backward_state(W_, U_, K1, V1, G1, dev(s_in), ck1, state_out=S1, grad_state_out=second[4],
                             kernel=kk)
    ref = oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso)
    got = (first[0] + second[0], first[1] + second[1], torch.cat([first[2], second[2]], dim=1),
           torch.cat([first[3], second[3]], dim=1), first[4])
    assert_grads_state(got, ref, F32_GRAD_TOL)


def test_autograd_through_the_state():
    """Two differentiable calls chained through the state, loss on both
    outputs and on the final state's sums."""
    B, T, C, t1 = 2, 150, 48, 64
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=27)
    tw, tu, tk, tv, ts = (dev(x).requires_grad_() for x in (w, u, k, v, s_in))
    y1, S1 = W.wkv_state(tw, tu, tk[:, :t1], tv[:, :t1], ts)
    y2, S2 = W.wkv_state(tw, tu, tk[:, t1:], tv[:, t1:], S1)
    G = dev(g)
    # a loss on the final state through its sums: gA A + gB B with the oracle's p as reference
    P = dev(s_out[2])
    gA, gB = dev(gso[0]), dev(gso[1])
    AT = S2[0] * torch.exp(S2[2] - P)
    BT = S2[1] * torch.exp(S2[2] - P)
    L = (y1 * G[:, :t1]).sum() + (y2 * G[:, t1:]).sum() + (gA * AT).sum() + (gB * BT).sum()
    L.backward()
    ref = oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso)
    assert_grads_state((tw.grad, tu.grad, tk.grad, tv.grad, ts.grad), ref, F32_GRAD_TOL)


def test_backward_state_rwkv169m_full():
    """The full rwkv169m workload (B 8, T 1024, C 768, fp32) with an initial
    state and a final-state gradient."""
    inp = workloads.generate("rwkv169m")
    w, u, k, v, gy = inputs_to_device(inp)
    rng = np.random.default_rng(31)
    B, C = inp["B"], inp["C"]
    s_in = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                     rng.normal(0, 2, (B, C))]).astype(np.float32)
    gso = rng.normal(size=(3, B, C)).astype(np.float32)
    _, s_out = oracle.fwd_recur(inp["w"], inp["u"], inp["k"], inp["v"], s_in)
    s_out = s_out.astype(np.float32)
    _, _, ck = W.forward(w, u, k, v, dev(s_in), want_ckpt=True)
    got = W.backward_state(w, u, k, v, gy, dev(s_in), ck, state_out=dev(s_out), grad_state_out=dev(gso))
    ref = oracle.bwd_state(inp["w"], inp["u"], inp["k"], inp["v"], inp["gy"], s_in, s_out, gso)
    assert_grads_state(got, ref, F32_GRAD_TOL)


def test_backward_state_long_sequence_flag_join():
    """5000 tokens in one chain: more than 32 segments, so the segment
    backward joins through per-record flags (blocks of segments with suffix
    records), the final-state gradient entering the first block's folds."""
    B, T, C = 1, 5000, 64
    w, u, k, v, g, s_in, s_out, gso = state_case(B, T, C, seed=32, td=(-5.0, -1.0))
    got = W.backward_state(dev(w), dev(u), dev(k), dev(v), dev(g), dev(s_in), state_out=dev(s_out),
                           grad_state_out=dev(gso), kernel=W.WKV_KERNEL_SEGMENT)
    assert_grads_state(got, oracle.bwd_state(w, u, k, v, g, s_in, s_out, gso), F32_GRAD_TOL)
