"""Pins for the oracle's gated operator o_t = sigma(r_t) * wkv_t.

The gate is the review's output gating ("[논문 리뷰] Reinvention RNNs for the
Transformer Era: RWKV", section "출력 게이팅(Output Gating)", eq.
o_t = W_o (sigma(r_t) * WKV_t)) without the W_o projection.  Each pin ties
the oracle to something other than itself:

* the logistic function against scipy's ``expit`` (a library routine), over
  a range where a naive formula overflows;
* T = 1: wkv_0 = v_0, so o_0 = sigma(r_0) v_0 and the gradients are closed
  forms;
* the gate's limits (r -> +inf passes wkv, r -> -inf closes it, r = 0 halves
  it);
* float64 central finite differences of L = sum(go * o) against all five
  gradients, with o evaluated through the O(T^2) direct sum (not the
  recurrence the gated backward uses);
* planted mistakes in the chain rule must fail the finite-difference pin.
"""
import numpy as np
import pytest
from scipy.special import expit

import oracle


def rand_case(seed, B=2, T=9, C=3, rstd=1.5):
    rng = np.random.default_rng(seed)
    w = -np.exp(rng.uniform(-1.0, 1.0, C))
    u = rng.uniform(-0.5, 0.5, C)
    k = rng.normal(size=(B, T, C))
    v = rng.normal(size=(B, T, C))
    r = rng.normal(0, rstd, (B, T, C))
    go = rng.normal(size=(B, T, C))
    return w, u, k, v, r, go


def relerr(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


def test_sigmoid_matches_library():
    x = np.concatenate([np.linspace(-800, 800, 4001), [-1e-300, 0.0, 1e-300]])
    # below 1e-300 the two differ only in how they round into the subnormal range
    np.testing.assert_allclose(oracle.sigmoid(x), expit(x), rtol=1e-15, atol=1e-300)


def test_T1_closed_form():
    w, u, k, v, r, go = rand_case(1, T=1)
    o, _ = oracle.fwd_gated(w, u, k, v, r)
    s = expit(r)
    np.testing.assert_allclose(o, s * v, rtol=1e-15, atol=1e-300)
    gw, gu, gk, gv, gr = oracle.bwd_gated(w, u, k, v, r, go)
    np.testing.assert_allclose(gv, go * s, rtol=1e-14)
    np.testing.assert_allclose(gr, go * v * s * (1 - s), rtol=1e-14)
    assert np.max(np.abs(gk)) <= 1e-15 and np.max(np.abs(gw)) <= 1e-15
    assert np.max(np.abs(gu)) <= 1e-15


def test_gate_limits():
    w, u, k, v, r, go = rand_case(2, T=20)
    y, _ = oracle.fwd_recur(w, u, k, v)
    o_open, _ = oracle.fwd_gated(w, u, k, v, np.full_like(r, 40.0))
    o_shut, _ = oracle.fwd_gated(w, u, k, v, np.full_like(r, -40.0))
    o_half, _ = oracle.fwd_gated(w, u, k, v, np.zeros_like(r))
    np.testing.assert_allclose(o_open, y, rtol=1e-16, atol=0)
    assert np.max(np.abs(o_shut)) <= 5e-18 * np.max(np.abs(y))
    np.testing.assert_allclose(o_half, 0.5 * y, rtol=1e-16, atol=0)
    gr_half = oracle.bwd_gated(w, u, k, v, np.zeros_like(r), go)[4]
    np.testing.assert_allclose(gr_half, 0.25 * go * y, rtol=1e-15, atol=1e-300)


def gated_direct(w, u, k, v, r):
    return expit(r) * oracle.fwd_direct(w, u, k, v)


def fd_grads(w, u, k, v, r, go):
    def L(w_, u_, k_, v_, r_):
        return float(np.sum(go * gated_direct(w_, u_, k_, v_, r_)))

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

    return (num(w, lambda x: L(x, u, k, v, r)), num(u, lambda x: L(w, x, k, v, r)),
            num(k, lambda x: L(w, u, x, v, r)), num(v, lambda x: L(w, u, k, x, r)),
            num(r, lambda x: L(w, u, k, v, x)))


def check_fd(bwd):
    w, u, k, v, r, go = rand_case(3, B=2, T=10, C=3)
    ref = fd_grads(w, u, k, v, r, go)
    got = bwd(w, u, k, v, r, go)
    for name, a, b in zip(("gw", "gu", "gk", "gv", "gr"), got, ref):
        assert relerr(a, b) < 1e-6, (name, relerr(a, b))


def test_finite_differences():
    check_fd(oracle.bwd_gated)


def _mutant_no_gate_in_wkv_grad(w, u, k, v, r, go):
    """Mistake: the WKV backward fed with grad_o instead of grad_o * sigma(r)."""
    y, _ = oracle.fwd_recur(w, u, k, v)
    s = expit(r)
    gw, gu, gk, gv = oracle.bwd_recur(w, u, k, v, go)
    return gw, gu, gk, gv, go * y * s * (1 - s)


def _mutant_wrong_sigmoid_slope(w, u, k, v, r, go):
    """Mistake: d sigma / dr taken as sigma instead of sigma (1 - sigma)."""
    y, _ = oracle.fwd_recur(w, u, k, v)
    s = expit(r)
    gw, gu, gk, gv = oracle.bwd_recur(w, u, k, v, go * s)
    return gw, gu, gk, gv, go * y * s


@pytest.mark.parametrize("mutant", [_mutant_no_gate_in_wkv_grad, _mutant_wrong_sigmoid_slope])
def test_pins_reject_gate_mistakes(mutant):
    with pytest.raises(AssertionError):
        check_fd(mutant)
