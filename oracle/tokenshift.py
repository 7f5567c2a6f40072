"""float64 CPU oracle for the token shift (test infrastructure).

Only the test suite may import this module; the CUDA library never does.
The RWKV paper review ("[논문 리뷰] Reinvention RNNs for the Transformer Era:
RWKV", section "토큰 변환") forms the time-mixing inputs R, K, V (and the
channel-mixing R', K') by linear interpolation between the current and the
previous time step.  Written out per channel, with one mixing vector mu_m
per interpolated input:

    out_m[t] = mu_m * x[t] + (1 - mu_m) * x[t-1],   t = 0..T-1,

where x[-1] is the last token of the previous call (x_prev), or zero for a
sequence that starts here.  Shapes: x [B, T, C], mu [n, C], x_prev [B, C],
out [n, B, T, C].  Pinned by ``tests/test_oracle_tokenshift_pins.py``.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def _previous(x, x_prev):
    """x[t-1] for every t: the sequence shifted by one, x_prev (or 0) first."""
    first = np.zeros_like(x[:, :1, :]) if x_prev is None else _f64(x_prev)[:, None, :]
    return np.concatenate([first, x[:, :-1, :]], axis=1)


def shift(x, mu, x_prev=None):
    """out [n, B, T, C]: the interpolations for every row of mu."""
    x, mu = _f64(x), _f64(mu)
    xp = _previous(x, x_prev)
    return np.stack([m * x + (1.0 - m) * xp for m in mu])


def shift_bwd(x, mu, g, x_prev=None):
    """Gradients of L = sum(g * out): (gx [B, T, C], gmu [n, C], gx_prev [B, C]).

    gx[t] = sum_m (mu_m g_m[t] + (1 - mu_m) g_m[t+1]) (g_m[T] = 0),
    gmu_m = sum_{b, t} g_m[t] (x[t] - x[t-1]),
    gx_prev = sum_m (1 - mu_m) g_m[0].
    """
    x, mu, g = _f64(x), _f64(mu), _f64(g)
    xp = _previous(x, x_prev)
    gx = np.zeros_like(x)
    gmu = np.empty(mu.shape)
    gprev = np.zeros(x[:, 0, :].shape)
    for m in range(mu.shape[0]):
        gx += mu[m] * g[m]
        gx[:, :-1, :] += (1.0 - mu[m]) * g[m][:, 1:, :]
        gprev += (1.0 - mu[m]) * g[m][:, 0, :]
        gmu[m] = np.sum(g[m] * (x - xp), axis=(0, 1))
    return gx, gmu, gprev
