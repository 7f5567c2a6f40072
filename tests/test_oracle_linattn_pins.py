"""Pins for the causal linear-attention oracle (``oracle.linattn``).

The operator is the causal form of the linear attention post ("Transformers
are RNNs: 선형 어텐션으로 만드는 빠른 자기회귀 트랜스포머", sections "인과
마스킹과 누적합" and "상수 메모리 기울기 계산").  The pins tie the oracle to
things other than itself:

* phi against torch's ``elu`` + 1 (a library routine);
* the O(N^2) definition against the cumulative-state recurrence;
* forward and all three gradients against torch autograd through an O(N^2)
  masked-matmul form written in torch (an independent derivation of the
  gradients from the page's cumulative sums);
* float64 central finite differences;
* N = 1 (V'_0 = V_0), the convex hull of V and equivariance V -> a V + b;
* two calls with the state carried equal one call;
* planted mistakes (copies of the oracle's backward with one line changed)
  must fail the finite-difference pin.
"""
import inspect

import numpy as np
import pytest
import torch

from oracle import linattn as la


def case(seed, lead=(2, 3), N=9, D=4, M=5, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.normal(0, scale, (*lead, N, D))
    k = rng.normal(0, scale, (*lead, N, D))
    v = rng.normal(size=(*lead, N, M))
    g = rng.normal(size=(*lead, N, M))
    return q, k, v, g


def relerr(a, b):
    return np.linalg.norm((np.asarray(a) - b).ravel()) / max(np.linalg.norm(np.ravel(b)), 1e-300)


def test_phi_matches_library_elu():
    x = np.linspace(-50, 50, 20001)
    ref = torch.nn.functional.elu(torch.from_numpy(x)).numpy() + 1.0
    # elu(x) + 1 = (e^x - 1) + 1 cancels for x << 0 (one ulp of 1 absolute);
    # the oracle forms e^x directly, which is also checked on its own
    np.testing.assert_allclose(la.phi(x), ref, rtol=1e-14, atol=4e-16)
    neg = x[x <= 0]
    np.testing.assert_allclose(la.phi(neg), np.exp(neg), rtol=1e-15)
    assert np.all(la.phi(x) > 0)


def test_dphi_by_finite_differences():
    x = np.concatenate([np.linspace(-6, -0.01, 50), np.linspace(0.01, 6, 50)])
    h = 1e-6
    np.testing.assert_allclose(la.dphi(x), (la.phi(x + h) - la.phi(x - h)) / (2 * h), rtol=1e-8)


def test_direct_equals_recurrence():
    q, k, v, _ = case(1, N=40)
    y1 = la.fwd_direct(q, k, v)
    y2, _ = la.fwd_recur(q, k, v)
    assert np.max(np.abs(y1 - y2)) <= 1e-12


def torch_reference(q, k, v, g):
    """Forward and gradients by torch autograd through the O(N^2) masked
    form (float64)."""
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    fq = torch.nn.functional.elu(tq) + 1
    fk = torch.nn.functional.elu(tk) + 1
    s = torch.tril(fq @ fk.transpose(-1, -2))
    y = (s @ tv) / s.sum(-1, keepdim=True)
    (y * torch.tensor(g)).sum().backward()
    return y.detach().numpy(), tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


def test_against_torch_autograd():
    q, k, v, g = case(2, N=30, D=8, M=6, scale=1.5)
    y, gq, gk, gv = torch_reference(q, k, v, g)
    assert np.max(np.abs(la.fwd_direct(q, k, v) - y)) <= 1e-12
    got = la.bwd_recur(q, k, v, g)
    for name, a, b in zip(("gq", "gk", "gv"), got, (gq, gk, gv)):
        assert relerr(a, b) <= 1e-12, (name, relerr(a, b))


def fd_grads(q, k, v, g):
    def L(q_, k_, v_):
        return float(np.sum(g * la.fwd_direct(q_, k_, v_)))

    def num(x, f):
        out = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            h = 1e-6 * max(1.0, abs(x[i]))
            xp = x.copy(); xp[i] += h
            xm = x.copy(); xm[i] -= h
            out[i] = (f(xp) - f(xm)) / (2 * h)
        return out

    return (num(q, lambda x: L(x, k, v)), num(k, lambda x: L(q, x, v)), num(v, lambda x: L(q, k, x)))


def check_fd(bwd):
    q, k, v, g = case(3, lead=(2,), N=7, D=3, M=4)
    ref = fd_grads(q, k, v, g)
    got = bwd(q, k, v, g)
    for name, a, b in zip(("gq", "gk", "gv"), got, ref):
        assert relerr(a, b) < 1e-7, (name, relerr(a, b))


def test_finite_differences():
    check_fd(la.bwd_recur)


def test_single_position_returns_v():
    q, k, v, _ = case(4, N=1)
    np.testing.assert_allclose(la.fwd_direct(q, k, v), v, rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(la.fwd_recur(q, k, v)[0], v, rtol=1e-15, atol=1e-15)


def test_convex_hull_and_equivariance():
    q, k, v, _ = case(5, N=25)
    y = la.fwd_recur(q, k, v)[0]
    cmin = np.minimum.accumulate(v, axis=-2)
    cmax = np.maximum.accumulate(v, axis=-2)
    assert np.all(y >= cmin - 1e-12) and np.all(y <= cmax + 1e-12)
    y2 = la.fwd_recur(q, k, 2.5 * v - 0.75)[0]
    np.testing.assert_allclose(y2, 2.5 * y - 0.75, rtol=1e-12, atol=1e-12)


def test_split_with_state_equals_one_call():
    q, k, v, g = case(6, N=20)
    y, st = la.fwd_recur(q, k, v)
    y1, s1 = la.fwd_recur(q[..., :8, :], k[..., :8, :], v[..., :8, :])
    y2, s2 = la.fwd_recur(q[..., 8:, :], k[..., 8:, :], v[..., 8:, :], s1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=-2), y, rtol=1e-12)
    np.testing.assert_allclose(s2[0], st[0], rtol=1e-12)
    np.testing.assert_allclose(s2[1], st[1], rtol=1e-12)
    # the backward of the second part with the first part's state equals the
    # full backward's rows there
    full = la.bwd_recur(q, k, v, g)
    part = la.bwd_recur(q[..., 8:, :], k[..., 8:, :], v[..., 8:, :], g[..., 8:, :], s1)
    np.testing.assert_allclose(part[0], full[0][..., 8:, :], rtol=1e-10, atol=1e-13)


def _mutant(old, new):
    """A copy of the oracle's backward with one line changed."""
    src = inspect.getsource(la.bwd_recur)
    assert old in src, old
    ns = dict(vars(la))
    exec(src.replace(old, new), ns)
    return ns["bwd_recur"]


MUTANTS = {
    # the normalisation's gradient dropped from phi(Q)
    "no_den_in_q": ("+ Z * gden[..., i, None])", ")"),
    # the reverse sums taken over j > i instead of j >= i
    "strict_reverse_sum": ("gfk[..., i, :] = np.einsum(\"...dm,...m->...d\", U, v[..., i, :]) + u",
                           "gfk[..., i, :] = np.einsum(\"...dm,...m->...d\", U - fq[..., i, :, None] "
                           "* gnum[..., i, None, :], v[..., i, :]) + u"),
    # phi' taken as 1 everywhere (the relu-style slope)
    "unit_slope": ("return gfq * dphi(q), gfk * dphi(k), gv", "return gfq, gfk, gv"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistakes(name):
    with pytest.raises(AssertionError):
        check_fd(_mutant(*MUTANTS[name]))
