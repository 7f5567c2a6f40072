"""wkv_backward_static: the backward for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run the backward (inside an
allocator or memory-pool callback, in plugin hosts with fixed buffers), so
they cannot pass a workspace.  wkv_backward_static keeps its scratch in a
static device array instead.  These tests call it through the C ABI on a
sequence of problems of different shapes and element types (a larger one,
smaller ones, the larger one again, one with checkpoints from a forward), so
that every call meets the shared scratch as the previous, different call
left it, and check each call's gradients against the float64 oracle within
the suite's tolerances; they also check that the status word reads clean and
that a problem too large for the static scratch is rejected.

This file is collected last on purpose; it must pass both on its own in a
fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import oracle
import rwkv_linear_rnn_b200 as W
from rwkv_linear_rnn_b200 import workloads
from gpu_util import BF16_TOL, F32_GRAD_TOL, dev, host, rel_l2

pytestmark = pytest.mark.gpu


def _case(seed, B, T, C, dtype, state):
    rng = np.random.default_rng(seed)
    w = (-np.exp(rng.uniform(-3, 1, C))).astype(np.float32)
    u = rng.uniform(-1, 1, C).astype(np.float32)
    k = rng.normal(size=(B, T, C)).astype(np.float32)
    v = rng.normal(size=(B, T, C)).astype(np.float32)
    g = rng.normal(size=(B, T, C)).astype(np.float32)
    if dtype == "bf16":  # the oracle runs on the rounded values
        k, v, g = (workloads.bf16_to_f32(workloads.bf16_round(x)) for x in (k, v, g))
    st = None
    if state:
        st = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                       rng.normal(0, 2, (B, C))]).astype(np.float32)
    return w, u, k, v, g, st


def _static_backward(w, u, k, v, g, st, dtype, ckpt=None):
    abi = W.abi
    B, T, C = k.shape
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    K_, V_, G_ = (dev(x).to(tdt) for x in (k, v, g))
    W_, U_ = dev(w), dev(u)
    S_ = dev(st) if st is not None else None
    gw = torch.empty(C, device="cuda")
    gu = torch.empty(C, device="cuda")
    gk = torch.empty_like(K_)
    gv = torch.empty_like(V_)
    p = lambda t: 0 if t is None else t.data_ptr()
    dt = W.WKV_BF16 if dtype == "bf16" else W.WKV_F32
    ck = None
    if ckpt:  # checkpoints from a forward call with a caller workspace
        _, _, ck = W.forward(W_, U_, K_, V_, S_, want_ckpt=True)
    rc = abi.wkv_backward_static(B, T, C, dt, p(W_), p(U_), p(K_), p(V_), p(G_), p(S_), p(ck),
                                 p(gw), p(gu), p(gk), p(gv), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, W.wkv_strerror(rc)
    return gw, gu, gk, gv


# (B, T, C, dtype, initial state, checkpoints passed in)
SEQUENCE = [(3, 1000, 96, "f32", False, False),
            (2, 129, 64, "f32", True, False),
            (1, 300, 32, "bf16", False, True),
            (2, 700, 64, "bf16", True, False),
            (3, 1000, 96, "f32", True, True)]


def test_static_backward_matches_the_oracle_across_calls():
    for call, (B, T, C, dtype, state, ckpt) in enumerate(SEQUENCE):
        w, u, k, v, g, st = _case(100 + call, B, T, C, dtype, state)
        got = _static_backward(w, u, k, v, g, st, dtype, ckpt)
        torch.cuda.synchronize()
        ref = oracle.bwd_recur(w, u, k, v, g, st)
        tol = BF16_TOL if dtype == "bf16" else F32_GRAD_TOL
        for name, a, b in zip(("gw", "gu", "gk", "gv"), got, ref):
            e = rel_l2(host(a), b)
            assert e <= tol, (call, name, e)
        assert W.abi.wkv_backward_static_status(torch.cuda.current_stream().cuda_stream) == 0


def test_static_backward_rejects_sizes_beyond_the_scratch():
    B, T, C = 8, 4096, 2048
    assert W.wkv_workspace_size(W.WKV_OP_BACKWARD, B, T, C, W.WKV_F32) > W.WKV_STATIC_SCRATCH_BYTES
    fake = 1 << 20
    rc = W.abi.wkv_backward_static(B, T, C, W.WKV_F32, fake, fake, fake * 2, fake * 3, fake * 4, 0,
                                   0, fake * 5, fake * 6, fake * 7, fake * 8, 0)
    assert rc == W.abi.WKV_ERR_WORKSPACE
