"""Pins for the oracle's state gradients (``oracle.bwd_state``).

A sequence split across calls (the RNN mode of the RWKV paper review, "[논문
리뷰] Reinvention RNNs for the Transformer Era: RWKV", section "RNN-유사추론")
needs two more terms in the backward: the gradient arriving at the final
state, and the gradient leaving through the initial state.  The pins tie the
oracle to things other than its own reverse walk:

* central finite differences of L = sum(g * y) + ga A_T e^{-p*} + gb B_T e^{-p*}
  with y from the O(T^2) defining sum (``fwd_direct``) and A_T, B_T from
  their closed-form sums, against every gradient including the three
  components of the initial state;
* T = 0 and T = 1 closed forms;
* chaining: two calls joined through the state give the one-call gradients;
* planted mistakes in the state terms must fail the finite-difference pin.
"""
import numpy as np
import pytest

import oracle


def case(seed, B=2, T=7, C=3):
    rng = np.random.default_rng(seed)
    w = -np.exp(rng.uniform(-1.0, 1.0, C))
    u = rng.uniform(-0.5, 0.5, C)
    k = rng.normal(size=(B, T, C))
    v = rng.normal(size=(B, T, C))
    g = rng.normal(size=(B, T, C))
    s_in = np.stack([rng.normal(size=(B, C)), rng.uniform(0.5, 2.0, (B, C)),
                     rng.normal(0.0, 1.0, (B, C))])
    # the representation the final-state gradient refers to: any p will do
    p_ref = rng.uniform(-2.0, 3.0, (B, C))
    gso = np.stack([rng.normal(size=(B, C)), rng.normal(size=(B, C)), rng.normal(size=(B, C))])
    return w, u, k, v, g, s_in, p_ref, gso


def closed_form_sums(w, k, v, s_in):
    """A_T = sum_i e^{(T-1-i) w + k_i} v_i + e^{T w} A_0 (and B_T with v = 1):
    the review's hidden sums written out, not advanced token by token."""
    B, T, C = k.shape
    A0 = s_in[0] * np.exp(s_in[2])
    B0 = s_in[1] * np.exp(s_in[2])
    lag = (T - 1 - np.arange(T))[None, :, None]
    e = np.exp(lag * w[None, None, :] + k)
    return (e * v).sum(axis=1) + np.exp(T * w) * A0, e.sum(axis=1) + np.exp(T * w) * B0


def loss(w, u, k, v, g, s_in, p_ref, gso):
    y = oracle.fwd_direct(w, u, k, v, s_in)
    AT, BT = closed_form_sums(w, k, v, s_in)
    return float(np.sum(g * y) + np.sum(gso[0] * AT * np.exp(-p_ref))
                 + np.sum(gso[1] * BT * np.exp(-p_ref)))


def fd(f, x, h0=1e-6):
    out = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        h = h0 * max(1.0, abs(x[i]))
        xp = x.copy(); xp[i] += h
        xm = x.copy(); xm[i] -= h
        out[i] = (f(xp) - f(xm)) / (2 * h)
    return out


def relerr(a, b):
    return np.linalg.norm((np.asarray(a) - b).ravel()) / max(np.linalg.norm(np.ravel(b)), 1e-300)


def state_out_ref(p_ref):
    # only p is read; a, b are set to something that is clearly not used
    return np.stack([np.full_like(p_ref, np.nan), np.full_like(p_ref, np.nan), p_ref])


def check_fd(bwd, seed=3):
    w, u, k, v, g, s_in, p_ref, gso = case(seed)
    L = lambda w_=w, u_=u, k_=k, v_=v, s_=s_in: loss(w_, u_, k_, v_, g, s_, p_ref, gso)
    ref = (fd(lambda x: L(w_=x), w), fd(lambda x: L(u_=x), u), fd(lambda x: L(k_=x), k),
           fd(lambda x: L(v_=x), v), fd(lambda x: L(s_=x), s_in))
    got = bwd(w, u, k, v, g, s_in, state_out_ref(p_ref), gso)
    for name, a, b in zip(("gw", "gu", "gk", "gv", "gs_in"), got, ref):
        assert relerr(a, b) < 1e-6, (name, relerr(a, b))


def test_finite_differences_with_state_terms():
    check_fd(oracle.bwd_state)


def test_without_state_terms_equals_bwd_recur():
    w, u, k, v, g, s_in, _, _ = case(4)
    a = oracle.bwd_recur(w, u, k, v, g, s_in)
    b = oracle.bwd_state(w, u, k, v, g, s_in)
    for x, y in zip(a, b[:4]):
        np.testing.assert_array_equal(x, y)


def test_T0_closed_form():
    w, u, k, v, g, s_in, p_ref, gso = case(5, T=0)
    gw, gu, gk, gv, gs = oracle.bwd_state(w, u, k, v, g, s_in, state_out_ref(p_ref), gso)
    assert np.all(gw == 0) and np.all(gu == 0) and gk.size == 0
    scale = np.exp(s_in[2] - p_ref)
    np.testing.assert_allclose(gs[0], gso[0] * scale, rtol=1e-14)
    np.testing.assert_allclose(gs[1], gso[1] * scale, rtol=1e-14)
    np.testing.assert_allclose(gs[2], s_in[0] * gs[0] + s_in[1] * gs[1], rtol=1e-13)


def test_T1_closed_form_state_term_only():
    """One token, no output gradient: A_1 = e^w A_0 + e^{k_0} v_0."""
    w, u, k, v, g, s_in, p_ref, gso = case(6, T=1)
    g = np.zeros_like(g)
    gw, gu, gk, gv, gs = oracle.bwd_state(w, u, k, v, g, s_in, state_out_ref(p_ref), gso)
    gA, gB = gso[0] * np.exp(-p_ref), gso[1] * np.exp(-p_ref)
    ek = np.exp(k[:, 0, :])
    np.testing.assert_allclose(gv[:, 0, :], ek * gA, rtol=1e-14)
    np.testing.assert_allclose(gk[:, 0, :], ek * (v[:, 0, :] * gA + gB), rtol=1e-13)
    assert np.max(np.abs(gu)) == 0.0
    A0, B0 = s_in[0] * np.exp(s_in[2]), s_in[1] * np.exp(s_in[2])
    np.testing.assert_allclose(gw, np.sum(np.exp(w) * (A0 * gA + B0 * gB), axis=0), rtol=1e-13)
    np.testing.assert_allclose(gs[0], np.exp(w) * gA * np.exp(s_in[2]), rtol=1e-14)


def test_empty_final_state_passes_no_gradient():
    w, u, k, v, g, s_in, p_ref, gso = case(7)
    so = state_out_ref(np.full_like(p_ref, -np.inf))
    a = oracle.bwd_state(w, u, k, v, g, s_in, so, gso)
    b = oracle.bwd_state(w, u, k, v, g, s_in)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_two_calls_chained_through_the_state_equal_one_call():
    """Forward: S0 -> [tokens 0..t1) -> S1 -> [tokens t1..T) -> S2.  The
    second call's state gradient, fed to the first call as its final-state
    gradient (in the representation S1 the first forward returned), gives the
    gradients of the one-call backward."""
    w, u, k, v, g, s_in, p_ref, gso = case(8, T=11)
    t1 = 4
    _, S1 = oracle.fwd_recur(w, u, k[:, :t1], v[:, :t1], s_in)
    _, S2 = oracle.fwd_recur(w, u, k[:, t1:], v[:, t1:], S1)
    so2 = state_out_ref(p_ref)
    full = oracle.bwd_state(w, u, k, v, g, s_in, so2, gso)
    second = oracle.bwd_state(w, u, k[:, t1:], v[:, t1:], g[:, t1:], S1, so2, gso)
    first = oracle.bwd_state(w, u, k[:, :t1], v[:, :t1], g[:, :t1], s_in, S1, second[4])
    np.testing.assert_allclose(first[0] + second[0], full[0], rtol=1e-12)
    np.testing.assert_allclose(first[1] + second[1], full[1], rtol=1e-12)
    np.testing.assert_allclose(np.concatenate([first[2], second[2]], axis=1), full[2], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(np.concatenate([first[3], second[3]], axis=1), full[3], rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(first[4], full[4], rtol=1e-11)


def _mutant_no_rescale(w, u, k, v, g, s_in, so, gso):
    """Mistake: the final-state gradient taken as dL/dA_T itself (no e^{-p})."""
    return oracle.bwd_state(w, u, k, v, g, s_in, np.stack([so[0], so[1], np.zeros_like(so[2])]), gso)


def _mutant_no_p_component(w, u, k, v, g, s_in, so, gso):
    """Mistake: the initial state's p component left at zero."""
    out = list(oracle.bwd_state(w, u, k, v, g, s_in, so, gso))
    out[4] = out[4].copy()
    out[4][2] = 0.0
    return out


def _mutant_sign_of_B(w, u, k, v, g, s_in, so, gso):
    """Mistake: dL/dB_T entered with the wrong sign."""
    gso2 = gso.copy()
    gso2[1] = -gso2[1]
    return oracle.bwd_state(w, u, k, v, g, s_in, so, gso2)


@pytest.mark.parametrize("mutant", [_mutant_no_rescale, _mutant_no_p_component, _mutant_sign_of_B])
def test_pins_reject_state_mistakes(mutant):
    with pytest.raises(AssertionError):
        check_fd(mutant)
