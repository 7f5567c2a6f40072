"""Pins for the float64 oracle: checks against things other than itself.

Each check ties the oracle to a fact the pages or plain mathematics fix:

* hand-computed closed forms of the defining sum (``tests/golden``);
* a library routine: ``torch.softmax`` in float64 over the masked score
  matrix (the review's softmax-attention form with a lag bias);
* special cases: T = 1, strong decay, very large / very small bonus;
* invariants: convex combination, shift of k, affine map of v;
* the two independent derivations (direct sum vs recurrence) agreeing;
* gradient sum rules implied by the invariants, and float64 central finite
  differences;
* RNN-mode consistency: T single steps == one forward; a split forward with
  the state carried == one forward.

The last block plants mistakes in small pure-Python copies of the operator
(wrong lag, wrong sign, dropped bonus, dropped decay in the adjoint, ...) and
checks that at least one pin rejects each of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import load_golden


def rand_case(seed, B=2, T=9, C=3, state=False, td=(-1.0, 1.0), ustd=0.5, kstd=1.0):
    rng = np.random.default_rng(seed)
    w = -np.exp(rng.uniform(*td, C))
    u = rng.uniform(-ustd, ustd, C)
    k = rng.normal(0, kstd, (B, T, C))
    v = rng.normal(size=(B, T, C))
    g = rng.normal(size=(B, T, C))
    st = None
    if state:
        st = np.stack([rng.normal(size=(B, C)), rng.uniform(0.2, 3.0, (B, C)),
                       rng.normal(0, 2, (B, C))])
    return w, u, k, v, g, st


def relerr(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300)


# --------------------------------------------------------------------------
# Checkers, parameterised by the implementation so the mutation tests below
# can reuse them.
# --------------------------------------------------------------------------

def check_golden_forward(fwd):
    for name in ("geometric_decay.txt", "running_mean.txt", "bonus_double.txt"):
        g = load_golden(name)
        T = g["k"].size
        y = fwd(g["w"], g["u"], g["k"].reshape(1, T, 1), g["v"].reshape(1, T, 1), None)
        np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-13, atol=1e-14, err_msg=name)


def check_golden_state(fwd):
    g = load_golden("initial_state.txt")
    T = g["k"].size
    st = g["state"].reshape(3, 1, 1)
    y = fwd(g["w"], g["u"], g["k"].reshape(1, T, 1), g["v"].reshape(1, T, 1), st)
    np.testing.assert_allclose(y.ravel(), g["y"], rtol=1e-13)


def check_golden_grad(bwd):
    g = load_golden("grad_T3.txt")
    T = g["k"].size
    sh = (1, T, 1)
    gw, gu, gk, gv = bwd(g["w"], g["u"], g["k"].reshape(sh), g["v"].reshape(sh),
                         g["g"].reshape(sh), None)
    np.testing.assert_allclose(gw, g["gw"], atol=1e-14)
    np.testing.assert_allclose(gu, g["gu"], atol=1e-14)
    np.testing.assert_allclose(gk.ravel(), g["gk"], atol=1e-14)
    np.testing.assert_allclose(gv.ravel(), g["gv"], atol=1e-14)


def check_T1(fwd):
    w, u, k, v, _, _ = rand_case(11, B=3, T=1, C=5)
    y = fwd(w, u, k, v, None)
    # y_0 = (e^{u+k_0} v_0) / e^{u+k_0}: v_0 up to the rounding of one product
    # and one quotient
    np.testing.assert_allclose(y, v, rtol=3e-16, atol=0, err_msg="T=1 must give y_0 = v_0")


def check_softmax_reduction(fwd):
    """y_t = softmax_i(S_{t,i}) @ v per channel, S the lag-biased scores."""
    w, u, k, v, _, _ = rand_case(12, B=2, T=13, C=3)
    y = fwd(w, u, k, v, None)
    B, T, C = k.shape
    kt = torch.from_numpy(k)
    vt = torch.from_numpy(v)
    t_idx = torch.arange(T, dtype=torch.float64).view(T, 1)
    i_idx = torch.arange(T, dtype=torch.float64).view(1, T)
    for c in range(C):
        lag = (t_idx - 1 - i_idx)
        S = lag * float(w[c]) + kt[:, None, :, c]          # [B, T(t), T(i)]
        diag = float(u[c]) + kt[:, :, c]
        S = S.clone()
        idx = torch.arange(T)
        S[:, idx, idx] = diag
        S = S.masked_fill(i_idx > t_idx, float("-inf"))
        ref = torch.softmax(S, dim=-1) @ vt[:, :, c:c + 1]
        np.testing.assert_allclose(y[:, :, c], ref[..., 0].numpy(), rtol=1e-12, atol=1e-13)


def check_convex_hull(fwd):
    w, u, k, v, _, _ = rand_case(13, B=2, T=40, C=4, td=(-3, 1), kstd=2.0)
    y = fwd(w, u, k, v, None)
    lo = np.minimum.accumulate(v, axis=1)
    hi = np.maximum.accumulate(v, axis=1)
    assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)


def check_invariances(fwd):
    w, u, k, v, _, _ = rand_case(14, B=2, T=21, C=3)
    y = fwd(w, u, k, v, None)
    y_shift = fwd(w, u, k + 3.7, v, None)
    np.testing.assert_allclose(y_shift, y, rtol=1e-12, atol=1e-13)
    y_aff = fwd(w, u, k, -2.5 * v + 0.75, None)
    np.testing.assert_allclose(y_aff, -2.5 * y + 0.75, rtol=1e-12, atol=1e-12)


def check_strong_decay(fwd):
    """w -> -inf keeps only the lag-0 past token and the current token."""
    w, u, k, v, _, _ = rand_case(15, B=2, T=10, C=3)
    w = np.full_like(w, -1e4)
    y = fwd(w, u, k, v, None)
    ek_prev = np.exp(k[:, :-1])
    ecur = np.exp(u + k[:, 1:])
    ref = (ek_prev * v[:, :-1] + ecur * v[:, 1:]) / (ek_prev + ecur)
    np.testing.assert_allclose(y[:, 1:], ref, rtol=1e-13)
    np.testing.assert_array_equal(y[:, 0], v[:, 0])


def check_bonus_limits(fwd):
    w, u, k, v, _, _ = rand_case(16, B=1, T=12, C=2)
    # u -> +inf: the current token dominates
    y = fwd(w, np.full_like(u, 60.0), k, v, None)
    np.testing.assert_allclose(y, v, rtol=1e-12, atol=1e-12)
    # u -> -inf, w = 0, k = 0: the mean of the past tokens (t >= 1)
    z = np.zeros_like(k)
    y = fwd(np.zeros_like(w), np.full_like(u, -60.0), z, v, None)
    past_mean = np.cumsum(v, axis=1)[:, :-1] / np.arange(1, 12).reshape(1, -1, 1)
    np.testing.assert_allclose(y[:, 1:], past_mean, rtol=1e-12, atol=1e-12)


def check_direct_equals_recurrence(fwd_a, fwd_b):
    for seed in range(4):
        for T in (1, 2, 5, 17):
            for state in (False, True):
                w, u, k, v, _, st = rand_case(100 + seed, T=T, state=state)
                ya = fwd_a(w, u, k, v, st)
                yb = fwd_b(w, u, k, v, st)
                assert relerr(ya, yb) < 1e-12, (seed, T, state, relerr(ya, yb))


def fd_grads(fwd, w, u, k, v, g, st):
    """Central finite differences of L = sum g * y (float64)."""
    def L(w_, u_, k_, v_):
        return float(np.sum(g * fwd(w_, u_, k_, v_, st)))

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

    gw = num(w, lambda x: L(x, u, k, v))
    gu = num(u, lambda x: L(w, x, k, v))
    gk = num(k, lambda x: L(w, u, x, v))
    gv = num(v, lambda x: L(w, u, k, x))
    return gw, gu, gk, gv


def check_fd(bwd, fwd, state):
    w, u, k, v, g, st = rand_case(21 if state else 20, B=2, T=12, C=3, state=state)
    ref = fd_grads(fwd, w, u, k, v, g, st)
    got = bwd(w, u, k, v, g, st)
    for name, a, b in zip(("gw", "gu", "gk", "gv"), got, ref):
        assert relerr(a, b) < 1e-6, (name, relerr(a, b))


def check_sum_rules(bwd):
    """k -> k + c leaves y unchanged, v -> v + c shifts y by c (zero state),
    so sum_t dL/dk_t = 0 and sum_t dL/dv_t = sum_t g_t per (b, c)."""
    w, u, k, v, g, _ = rand_case(22, B=2, T=30, C=3, td=(-3, 1))
    _, _, gk, gv = bwd(w, u, k, v, g, None)
    scale = np.abs(gk).sum(axis=1)
    assert np.all(np.abs(gk.sum(axis=1)) <= 1e-12 * scale + 1e-14)
    np.testing.assert_allclose(gv.sum(axis=1), g.sum(axis=1), rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# The oracle against the pins
# --------------------------------------------------------------------------

def o_fwd_direct(w, u, k, v, st):
    return oracle.fwd_direct(w, u, k, v, st)


def o_fwd_recur(w, u, k, v, st):
    return oracle.fwd_recur(w, u, k, v, st)[0]


FWDS = {"direct": o_fwd_direct, "recur": o_fwd_recur}
BWDS = {"direct": oracle.bwd_direct, "recur": oracle.bwd_recur}


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_golden_forward(impl):
    check_golden_forward(FWDS[impl])
    check_golden_state(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(BWDS))
def test_golden_grad(impl):
    check_golden_grad(BWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_T1_gives_v0(impl):
    check_T1(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_softmax_reduction(impl):
    check_softmax_reduction(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_convex_hull(impl):
    check_convex_hull(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_invariances(impl):
    check_invariances(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_strong_decay(impl):
    check_strong_decay(FWDS[impl])


@pytest.mark.parametrize("impl", sorted(FWDS))
def test_bonus_limits(impl):
    check_bonus_limits(FWDS[impl])


def test_direct_equals_recurrence():
    check_direct_equals_recurrence(o_fwd_direct, o_fwd_recur)


@pytest.mark.parametrize("impl", sorted(BWDS))
@pytest.mark.parametrize("state", [False, True])
def test_finite_differences(impl, state):
    check_fd(BWDS[impl], o_fwd_direct, state)


@pytest.mark.parametrize("impl", sorted(BWDS))
def test_gradient_sum_rules(impl):
    check_sum_rules(BWDS[impl])


@pytest.mark.parametrize("state", [False, True])
def test_bwd_direct_equals_recur(state):
    w, u, k, v, g, st = rand_case(30, B=3, T=33, C=4, state=state, td=(-3, 1))
    a = oracle.bwd_direct(w, u, k, v, g, st)
    b = oracle.bwd_recur(w, u, k, v, g, st)
    for x, y in zip(a, b):
        assert relerr(x, y) < 1e-11


def test_points_equal_direct():
    w, u, k, v, _, st = rand_case(31, B=2, T=25, C=3, state=True)
    y = oracle.fwd_direct(w, u, k, v, st)
    rng = np.random.default_rng(0)
    pb, pt, pc = rng.integers(0, 2, 50), rng.integers(0, 25, 50), rng.integers(0, 3, 50)
    yp = oracle.fwd_points(w, u, k, v, pb, pt, pc, st)
    np.testing.assert_allclose(yp, y[pb, pt, pc], rtol=0, atol=0)


def test_steps_equal_forward():
    """T single RNN steps reproduce the time-parallel forward and its state."""
    w, u, k, v, _, st = rand_case(32, B=3, T=15, C=4, state=True)
    y_ref, s_ref = oracle.fwd_recur(w, u, k, v, st)
    s = st
    for t in range(k.shape[1]):
        y_t, s = oracle.step(w, u, k[:, t], v[:, t], s)
        np.testing.assert_allclose(y_t, y_ref[:, t], rtol=1e-13, atol=1e-14)
    for a, b in zip(oracle.canonical_state(s), oracle.canonical_state(s_ref)):
        np.testing.assert_allclose(a, b, rtol=1e-13)
    # and against the direct (non-recurrent) definition
    np.testing.assert_allclose(oracle.fwd_direct(w, u, k, v, st), y_ref, rtol=1e-12, atol=1e-13)


def test_split_forward_equals_whole():
    w, u, k, v, _, _ = rand_case(33, B=2, T=40, C=3)
    y, s = oracle.fwd_recur(w, u, k, v)
    y1, s1 = oracle.fwd_recur(w, u, k[:, :17], v[:, :17])
    y2, s2 = oracle.fwd_recur(w, u, k[:, 17:], v[:, 17:], s1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-13, atol=1e-14)
    for a, b in zip(oracle.canonical_state(s2), oracle.canonical_state(s)):
        np.testing.assert_allclose(a, b, rtol=1e-13)
    # the direct form resumes from the same state
    np.testing.assert_allclose(oracle.fwd_direct(w, u, k[:, 17:], v[:, 17:], s1), y2,
                               rtol=1e-12, atol=1e-13)


def test_state_golden_canonical():
    g = load_golden("initial_state.txt")
    T = g["k"].size
    _, s = oracle.fwd_recur(g["w"], g["u"], g["k"].reshape(1, T, 1), g["v"].reshape(1, T, 1),
                            g["state"].reshape(3, 1, 1))
    ratio, logb = oracle.canonical_state(s)
    np.testing.assert_allclose([ratio.item(), logb.item()], g["state_canonical"], rtol=1e-14)


def test_empty_state_matches_no_state():
    w, u, k, v, _, _ = rand_case(34, B=2, T=8, C=3)
    empty = np.stack([np.zeros((2, 3)), np.zeros((2, 3)), np.full((2, 3), -np.inf)])
    for f in (o_fwd_direct, o_fwd_recur):
        np.testing.assert_array_equal(f(w, u, k, v, empty), f(w, u, k, v, None))


def test_zero_length_sequence():
    w, u, _, _, _, st = rand_case(35, B=2, T=3, C=3, state=True)
    k = np.zeros((2, 0, 3))
    y, s = oracle.fwd_recur(w, u, k, k, st)
    assert y.shape == (2, 0, 3)
    for a, b in zip(oracle.canonical_state(s), oracle.canonical_state(st)):
        np.testing.assert_allclose(a, b, rtol=1e-14)


def test_gradient_determinism():
    w, u, k, v, g, _ = rand_case(36, B=4, T=50, C=8)
    a = oracle.bwd_recur(w, u, k, v, g)
    b = oracle.bwd_recur(w, u, k, v, g)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


# --------------------------------------------------------------------------
# Planted mistakes: each must be rejected by at least one pin.
# --------------------------------------------------------------------------

def _py_fwd(w, u, k, v, st, lag_offset=1, w_sign=1.0, bonus=True, causal=True):
    """Pure-Python direct sum with switchable mistakes (tiny inputs only)."""
    B, T, C = k.shape
    y = np.empty((B, T, C))
    for b in range(B):
        for c in range(C):
            A0 = B0 = 0.0
            if st is not None and np.isfinite(st[2, b, c]):
                A0 = st[0, b, c] * math.exp(st[2, b, c])
                B0 = st[1, b, c] * math.exp(st[2, b, c])
            for t in range(T):
                num = A0 * math.exp(t * w_sign * w[c])
                den = B0 * math.exp(t * w_sign * w[c])
                hi = t + 1 if causal else min(T, t + 2)
                for i in range(hi):
                    if i == t:
                        s = (u[c] if bonus else 0.0) + k[b, t, c]
                    elif i < t:
                        s = (t - lag_offset - i) * w_sign * w[c] + k[b, i, c]
                    else:
                        s = w[c] + k[b, i, c]
                    e = math.exp(s)
                    num += e * v[b, i, c]
                    den += e
                y[b, t, c] = num / den
    return y


def _py_bwd(w, u, k, v, g, st, decay_in_adjoint=True, bh_sign=-1.0, gw_decay=True):
    """Pure-Python recurrent backward with switchable mistakes."""
    B, T, C = k.shape
    gw = np.zeros(C); gu = np.zeros(C)
    gk = np.zeros_like(k); gv = np.zeros_like(v)
    for b in range(B):
        for c in range(C):
            ew = math.exp(w[c])
            A = [0.0]; Bs = [0.0]
            if st is not None and np.isfinite(st[2, b, c]):
                A[0] = st[0, b, c] * math.exp(st[2, b, c])
                Bs[0] = st[1, b, c] * math.exp(st[2, b, c])
            for t in range(T):
                ek = math.exp(k[b, t, c])
                A.append(ew * A[t] + ek * v[b, t, c])
                Bs.append(ew * Bs[t] + ek)
            Ah = Bh = 0.0
            for t in range(T - 1, -1, -1):
                ecur = math.exp(u[c] + k[b, t, c]); ek = math.exp(k[b, t, c])
                D = Bs[t] + ecur
                yt = (A[t] + ecur * v[b, t, c]) / D
                gt = g[b, t, c]
                gv[b, t, c] = gt * ecur / D + ek * Ah
                gk[b, t, c] = gt * ecur * (v[b, t, c] - yt) / D + ek * (v[b, t, c] * Ah + Bh)
                gu[c] += gt * ecur * (v[b, t, c] - yt) / D
                gw[c] += (ew if gw_decay else 1.0) * (A[t] * Ah + Bs[t] * Bh)
                f = ew if decay_in_adjoint else 1.0
                Ah = gt / D + f * Ah
                Bh = bh_sign * gt * yt / D + f * Bh
    return gw, gu, gk, gv


def _rejected(checks):
    for chk in checks:
        try:
            chk()
        except AssertionError:
            return True
    return False


FWD_MUTANTS = {
    "lag (t - i) instead of (t - 1 - i)": dict(lag_offset=0),
    "decay sign flipped": dict(w_sign=-1.0),
    "bonus u dropped": dict(bonus=False),
    "one future token leaks in": dict(causal=False),
}


def test_python_copy_passes_pins():
    """The switchable Python copy itself is correct with no mistake planted."""
    f = lambda w, u, k, v, st: _py_fwd(w, u, k, v, st)
    check_golden_forward(f)
    check_golden_state(f)
    check_softmax_reduction(f)
    b = lambda w, u, k, v, g, st: _py_bwd(w, u, k, v, g, st)
    check_golden_grad(b)
    check_fd(b, o_fwd_direct, state=True)


@pytest.mark.parametrize("name", sorted(FWD_MUTANTS))
def test_pins_reject_forward_mistakes(name):
    kw = FWD_MUTANTS[name]
    f = lambda w, u, k, v, st: _py_fwd(w, u, k, v, st, **kw)
    checks = [lambda: check_golden_forward(f), lambda: check_softmax_reduction(f),
              lambda: check_convex_hull(f), lambda: check_T1(f)]
    assert _rejected(checks), f"planted mistake not caught: {name}"


BWD_MUTANTS = {
    "decay missing in the adjoint walk": dict(decay_in_adjoint=False),
    "sign of the B adjoint flipped": dict(bh_sign=1.0),
    "decay factor missing in dL/dw": dict(gw_decay=False),
}


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_pins_reject_backward_mistakes(name):
    kw = BWD_MUTANTS[name]
    b = lambda w, u, k, v, g, st: _py_bwd(w, u, k, v, g, st, **kw)
    checks = [lambda: check_golden_grad(b), lambda: check_fd(b, o_fwd_direct, False),
              lambda: check_sum_rules(b)]
    assert _rejected(checks), f"planted mistake not caught: {name}"
