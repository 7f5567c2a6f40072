"""wkv_backward_static: the backward for callers that cannot allocate.

Some callers cannot call cudaMalloc where they run the backward (inside an
allocator or memory-pool callback, in plugin hosts with fixed buffers), so
they cannot pass a workspace.  wkv_backward_static keeps its scratch in a
static device array instead.  These tests call it through the C ABI and
check that two consecutive calls (different inputs, so the shared scratch
carries the first call's leftovers into the second) give the same gradients
as the ordinary wkv_backward with a caller workspace, and that a problem too
large for the static scratch is rejected.

This file is collected last on purpose; it must pass both on its own in a
fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import rwkv_linear_rnn_b200 as W
from gpu_util import F32_GRAD_TOL, dev, host, rel_l2

pytestmark = pytest.mark.gpu


def _case(seed, B, T, C, state):
    rng = np.random.default_rng(seed)
    w = (-np.exp(rng.uniform(-3, 1, C))).astype(np.float32)
    u = rng.uniform(-1, 1, C).astype(np.float32)
    k = rng.normal(size=(B, T, C)).astype(np.float32)
    v = rng.normal(size=(B, T, C)).astype(np.float32)
    g = rng.normal(size=(B, T, C)).astype(np.float32)
    st = None
    if state:
        st = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 3, (B, C)),
                       rng.normal(0, 2, (B, C))]).astype(np.float32)
    return [dev(x) if x is not None else None for x in (w, u, k, v, g, st)]


def _static_backward(w, u, k, v, g, st):
    abi = W.abi
    B, T, C = k.shape
    gw = torch.empty(C, device="cuda")
    gu = torch.empty(C, device="cuda")
    gk = torch.empty_like(k)
    gv = torch.empty_like(v)
    p = lambda t: 0 if t is None else t.data_ptr()
    rc = abi.wkv_backward_static(B, T, C, W.WKV_F32, p(w), p(u), p(k), p(v), p(g), p(st), 0,
                                 p(gw), p(gu), p(gk), p(gv), torch.cuda.current_stream().cuda_stream)
    assert rc == 0, W.wkv_strerror(rc)
    return gw, gu, gk, gv


@pytest.mark.parametrize("shape", [(2, 300, 64), (3, 1000, 96)])
def test_static_backward_matches_workspace_backward_twice(shape):
    B, T, C = shape
    for call, (seed, state) in enumerate([(41, False), (42, True)]):
        w, u, k, v, g, st = _case(seed + B, B, T, C, state)
        got = _static_backward(w, u, k, v, g, st)
        ref = W.backward(w, u, k, v, g, st)
        torch.cuda.synchronize()
        for name, a, b in zip(("gw", "gu", "gk", "gv"), got, ref):
            e = rel_l2(host(a), host(b))
            assert e <= F32_GRAD_TOL, (call, name, e)


def test_static_backward_rejects_sizes_beyond_the_scratch():
    B, T, C = 8, 4096, 2048
    assert W.wkv_workspace_size(W.WKV_OP_BACKWARD, B, T, C, W.WKV_F32) > W.WKV_STATIC_SCRATCH_BYTES
    fake = 1 << 20
    rc = W.abi.wkv_backward_static(B, T, C, W.WKV_F32, fake, fake, fake * 2, fake * 3, fake * 4, 0,
                                   0, fake * 5, fake * 6, fake * 7, fake * 8, 0)
    assert rc == W.abi.WKV_ERR_WORKSPACE
