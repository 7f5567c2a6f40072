"""GPU parity of the token shift (``wkv_token_shift`` and its backward)
against the float64 oracle ``oracle.tokenshift``.

The interpolation of the current and previous token (RWKV paper review,
section "토큰 변환"): n = 1..4 interpolations, with and without the carried
previous token, the 4-channel vector path and the per-channel path
(C not a multiple of 4, or rows off the vector alignment), strips of 32
tokens with ragged ends, T = 1 and T = 0, bf16, a sequence split across two
calls, autograd, reproducibility, and the rwkv169m layer shape.
"""
import numpy as np
import pytest
import torch

import rwkv_linear_rnn_b200 as W
from oracle import tokenshift as ts
from gpu_util import BF16_TOL, F32_FWD_TOL, F32_GRAD_TOL, dev, fwd_err, host, rel_l2

pytestmark = pytest.mark.gpu


def ts_case(B, T, C, n, seed, dtype="f32"):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(B, T, C)).astype(np.float32)
    mu = rng.uniform(0, 1, (n, C)).astype(np.float32)
    xp = rng.normal(size=(B, C)).astype(np.float32)
    g = rng.normal(size=(n, B, T, C)).astype(np.float32)
    if dtype == "bf16":
        from rwkv_linear_rnn_b200 import workloads
        x, xp, g = (workloads.bf16_to_f32(workloads.bf16_round(a)) for a in (x, xp, g))
    return x, mu, xp, g


def check(B, T, C, n, seed, dtype="f32", with_prev=True, shift_ptr=False):
    x, mu, xp, g = ts_case(B, T, C, n, seed, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    tol_f = BF16_TOL if dtype == "bf16" else F32_FWD_TOL
    tol_g = BF16_TOL if dtype == "bf16" else F32_GRAD_TOL

    def put(a):
        if not shift_ptr:
            return dev(a, tdt)
        flat = torch.empty(a.size + 1, dtype=tdt, device="cuda")  # one element off the vector alignment
        flat[1:] = torch.from_numpy(np.ascontiguousarray(a).ravel()).to("cuda").to(tdt)
        return flat[1:].view(a.shape)

    X, MU, G = put(x), dev(mu), put(g)
    XP = put(xp) if with_prev else None
    out = W.token_shift(X, MU, XP)
    ref = ts.shift(x, mu, xp if with_prev else None)
    assert fwd_err(host(out), ref) <= tol_f
    gx, gmu, gxp = W.token_shift_backward(X, MU, G, XP, want_grad_x_prev=with_prev)
    rgx, rgmu, rgxp = ts.shift_bwd(x, mu, g, xp if with_prev else None)
    assert rel_l2(host(gx), rgx) <= tol_g
    assert rel_l2(host(gmu), rgmu) <= tol_g
    if with_prev:
        assert rel_l2(host(gxp), rgxp) <= tol_g


@pytest.mark.parametrize("n", [1, 2, 3, 4])
@pytest.mark.parametrize("shape", [(1, 1, 8), (2, 31, 64), (3, 33, 36), (2, 100, 768), (1, 65, 33)])
def test_token_shift_shapes(shape, n):
    check(*shape, n, seed=sum(shape) + n)


@pytest.mark.parametrize("with_prev", [True, False])
def test_token_shift_previous_token(with_prev):
    check(2, 70, 128, 3, seed=5, with_prev=with_prev)


def test_token_shift_unaligned_rows_take_the_channel_path():
    check(2, 50, 64, 3, seed=6, shift_ptr=True)


@pytest.mark.parametrize("n", [1, 3])
def test_token_shift_bf16(n):
    check(2, 97, 256, n, seed=7, dtype="bf16")
    check(2, 40, 30, n, seed=8, dtype="bf16")  # per-channel path


def test_token_shift_T0():
    B, C = 2, 64
    X = torch.empty((B, 0, C), device="cuda")
    MU = dev(np.full((3, C), 0.5, np.float32))
    XP = dev(np.ones((B, C), np.float32))
    out = W.token_shift(X, MU, XP)
    assert out.shape == (3, B, 0, C)
    gx, gmu, gxp = W.token_shift_backward(X, MU, torch.empty((3, B, 0, C), device="cuda"), XP,
                                          want_grad_x_prev=True)
    assert torch.all(gmu == 0) and torch.all(gxp == 0)


def test_token_shift_split_across_calls():
    """Two calls with the first call's last token carried equal one call."""
    x, mu, _, _ = ts_case(2, 90, 128, 3, seed=9)
    X, MU = dev(x), dev(mu)
    full = W.token_shift(X, MU)
    a = W.token_shift(X[:, :41].contiguous(), MU)
    b = W.token_shift(X[:, 41:].contiguous(), MU, X[:, 40].contiguous())
    assert torch.equal(torch.cat([a, b], dim=2), full)


def test_token_shift_autograd():
    x, mu, xp, g = ts_case(2, 45, 96, 3, seed=10)
    tx, tmu, txp = (dev(a).requires_grad_() for a in (x, mu, xp))
    out = W.TokenShift.apply(tx, tmu, txp)
    (out * dev(g)).sum().backward()
    rgx, rgmu, rgxp = ts.shift_bwd(x, mu, g, xp)
    assert rel_l2(host(tx.grad), rgx) <= F32_GRAD_TOL
    assert rel_l2(host(tmu.grad), rgmu) <= F32_GRAD_TOL
    assert rel_l2(host(txp.grad), rgxp) <= F32_GRAD_TOL


def test_token_shift_backward_reproducible():
    x, mu, xp, g = ts_case(4, 300, 256, 3, seed=11)
    args = (dev(x), dev(mu), dev(g), dev(xp))
    a = W.token_shift_backward(*args, want_grad_x_prev=True)
    b = W.token_shift_backward(*args, want_grad_x_prev=True)
    for p, q in zip(a, b):
        assert torch.equal(p, q)


def test_token_shift_rwkv169m_shape():
    """The rwkv169m layer shape (B 8, T 1024, C 768) with the three
    time-mixing interpolations (R, K, V)."""
    check(8, 1024, 768, 3, seed=12)
