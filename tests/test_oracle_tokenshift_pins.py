"""Pins for the token-shift oracle (``oracle.tokenshift``).

The interpolation of the current and previous token (RWKV paper review,
section "토큰 변환") is pinned by its limits (mu = 1 is the identity, mu = 0
the pure shift by one token), a torch reference through ``torch.roll``
with autograd for the gradients, float64 finite differences, splitting a
sequence with the last token carried, and planted mistakes.
"""
import numpy as np
import pytest
import torch

from oracle import tokenshift as ts


def case(seed, B=2, T=6, C=5, n=3):
    rng = np.random.default_rng(seed)
    x = rng.normal(size=(B, T, C))
    mu = rng.uniform(0, 1, (n, C))
    xp = rng.normal(size=(B, C))
    g = rng.normal(size=(n, B, T, C))
    return x, mu, xp, g


def relerr(a, b):
    return np.linalg.norm((np.asarray(a) - b).ravel()) / max(np.linalg.norm(np.ravel(b)), 1e-300)


def test_limits():
    x, mu, xp, _ = case(1)
    out = ts.shift(x, np.stack([np.ones(5), np.zeros(5)]), xp)
    np.testing.assert_array_equal(out[0], x)
    np.testing.assert_array_equal(out[1][:, 1:], x[:, :-1])
    np.testing.assert_array_equal(out[1][:, 0], xp)
    assert np.all(ts.shift(x, np.zeros((1, 5)))[0][:, 0] == 0)


def torch_reference(x, mu, xp, g):
    tx = torch.tensor(x, requires_grad=True)
    tmu = torch.tensor(mu, requires_grad=True)
    txp = torch.tensor(xp, requires_grad=True)
    prev = torch.roll(tx, 1, dims=1).clone()
    prev[:, 0] = txp
    out = torch.stack([m * tx + (1 - m) * prev for m in tmu])
    (out * torch.tensor(g)).sum().backward()
    return out.detach().numpy(), tx.grad.numpy(), tmu.grad.numpy(), txp.grad.numpy()


def test_against_torch_autograd():
    x, mu, xp, g = case(2, T=11, C=7)
    out, gx, gmu, gxp = torch_reference(x, mu, xp, g)
    np.testing.assert_allclose(ts.shift(x, mu, xp), out, rtol=1e-15, atol=1e-15)
    got = ts.shift_bwd(x, mu, g, xp)
    for name, a, b in zip(("gx", "gmu", "gx_prev"), got, (gx, gmu, gxp)):
        assert relerr(a, b) <= 1e-14, name


def fd(f, x, h=1e-6):
    out = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp = x.copy(); xp[i] += h
        xm = x.copy(); xm[i] -= h
        out[i] = (f(xp) - f(xm)) / (2 * h)
    return out


def check_fd(bwd):
    x, mu, xp, g = case(3)
    L = lambda x_=x, mu_=mu, xp_=xp: float(np.sum(g * ts.shift(x_, mu_, xp_)))
    ref = (fd(lambda a: L(x_=a), x), fd(lambda a: L(mu_=a), mu), fd(lambda a: L(xp_=a), xp))
    for name, a, b in zip(("gx", "gmu", "gx_prev"), bwd(x, mu, g, xp), ref):
        assert relerr(a, b) < 1e-8, (name, relerr(a, b))


def test_finite_differences():
    check_fd(ts.shift_bwd)


def test_split_with_last_token_carried():
    x, mu, _, g = case(4, T=9)
    full = ts.shift(x, mu)
    a = ts.shift(x[:, :4], mu)
    b = ts.shift(x[:, 4:], mu, x[:, 3])
    np.testing.assert_array_equal(np.concatenate([a, b], axis=2), full)
    gfull = ts.shift_bwd(x, mu, g)
    gb = ts.shift_bwd(x[:, 4:], mu, g[:, :, 4:], x[:, 3])
    ga = ts.shift_bwd(x[:, :4], mu, g[:, :, :4])
    # the second part's gradient for the carried token adds to the first
    # part's last token
    gx = np.concatenate([ga[0], gb[0]], axis=1)
    gx[:, 3] += gb[2]
    np.testing.assert_allclose(gx, gfull[0], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ga[1] + gb[1], gfull[1], rtol=1e-13)


def _mutant_no_shifted_term(x, mu, g, xp):
    """Mistake: the gradient through x[t-1] (the (1 - mu) g[t+1] term) dropped."""
    gx, gmu, gprev = ts.shift_bwd(x, mu, g, xp)
    for m in range(mu.shape[0]):
        gx[:, :-1, :] -= (1.0 - mu[m]) * g[m][:, 1:, :]
    return gx, gmu, gprev


def _mutant_mu_sign(x, mu, g, xp):
    """Mistake: d out / d mu taken as x[t-1] - x[t]."""
    gx, gmu, gprev = ts.shift_bwd(x, mu, g, xp)
    return gx, -gmu, gprev


@pytest.mark.parametrize("mutant", [_mutant_no_shifted_term, _mutant_mu_sign])
def test_pins_reject_planted_mistakes(mutant):
    with pytest.raises(AssertionError):
        check_fd(mutant)
