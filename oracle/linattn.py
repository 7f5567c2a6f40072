"""float64 CPU oracle for causal linear attention (test infrastructure).

Only the test suite may import this module; the CUDA library never does and
the two share no code.  Plain numpy in float64, written from the linear
attention post ("Transformers are RNNs: 선형 어텐션으로 만드는 빠른 자기회귀
트랜스포머", juhoplayground):

* ``phi``           -- the feature map of section "특징 맵 선택과 계산 비용":
                       phi(x) = elu(x) + 1, i.e. x + 1 for x > 0 and e^x
                       otherwise (strictly positive);
* ``fwd_direct``    -- section "인과 마스킹과 누적합", the causal form of the
                       generalised attention: V'_i = sum_{j<=i} s_ij V_j /
                       sum_{j<=i} s_ij with s_ij = phi(Q_i)^T phi(K_j), the
                       O(N^2) definition;
* ``fwd_recur``     -- the same section's cumulative states S_i = sum_{j<=i}
                       phi(K_j) V_j^T, Z_i = sum_{j<=i} phi(K_j) and
                       V'_i = phi(Q_i)^T S_i / (phi(Q_i)^T Z_i), advanced one
                       position at a time (the RNN form of section
                       "트랜스포머는 RNN이다"), with the final (S, Z);
* ``bwd_recur``     -- section "상수 메모리 기울기 계산": the numerator's
                       gradients as a forward cumulative sum for phi(Q) and
                       reverse cumulative sums for phi(K) and V, extended by
                       the chain rule through the normalisation and phi.

Conventions: q, k are [..., N, D], v is [..., N, M] (leading axes are
independent problems, e.g. batch and head); positions are 0-based; a state
is the pair (S [..., D, M], Z [..., D]); no epsilon is added to the
denominator (the pages print none, and phi > 0 keeps it positive).

Pinned by ``tests/test_oracle_linattn_pins.py``.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def phi(x):
    """elu(x) + 1."""
    x = _f64(x)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def dphi(x):
    """d phi / dx: 1 for x > 0, e^x otherwise."""
    x = _f64(x)
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


def fwd_direct(q, k, v):
    """O(N^2) causal form; returns V' [..., N, M]."""
    fq, fk, v = phi(q), phi(k), _f64(v)
    s = fq @ np.swapaxes(fk, -1, -2)              # s_ij = phi(Q_i)^T phi(K_j)
    n = s.shape[-1]
    s = s * np.tril(np.ones((n, n)))               # j <= i only
    return (s @ v) / s.sum(axis=-1, keepdims=True)


def fwd_recur(q, k, v, state=None):
    """Cumulative states one position at a time; returns (V', (S, Z))."""
    fq, fk, v = phi(q), phi(k), _f64(v)
    *lead, n, d = fq.shape
    m = v.shape[-1]
    if state is None:
        S = np.zeros((*lead, d, m))
        Z = np.zeros((*lead, d))
    else:
        S, Z = _f64(state[0]).copy(), _f64(state[1]).copy()
    out = np.empty((*lead, n, m))
    for i in range(n):
        S = S + fk[..., i, :, None] * v[..., i, None, :]   # S_i = S_{i-1} + phi(K_i) V_i^T
        Z = Z + fk[..., i, :]
        num = np.einsum("...d,...dm->...m", fq[..., i, :], S)
        den = np.einsum("...d,...d->...", fq[..., i, :], Z)
        out[..., i, :] = num / den[..., None]
    return out, (S, Z)


def bwd_recur(q, k, v, g, state=None):
    """Gradients (gq, gk, gv) of L = sum(g * V') for the causal form.

    With num_i = phi(Q_i)^T S_i and den_i = phi(Q_i)^T Z_i:
    dL/dnum_i = g_i / den_i, dL/dden_i = -(g_i . V'_i) / den_i.  The
    numerator part follows the page's cumulative sums:
      dL/dphi(Q_i) = S_i dL/dnum_i + Z_i dL/dden_i              (forward sum)
      dL/dphi(K_i) = U_i V_i + u_i,   dL/dV_i = U_i^T phi(K_i)   (reverse sums)
    with U_i = sum_{j>=i} phi(Q_j) dL/dnum_j^T and u_i = sum_{j>=i} phi(Q_j)
    dL/dden_j; then dL/dx = dL/dphi(x) * phi'(x).  An initial state enters S
    and Z and receives no gradient.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    fq, fk = phi(q), phi(k)
    *lead, n, d = fq.shape
    m = v.shape[-1]
    out, _ = fwd_recur(q, k, v, state)
    # forward sweep: gradient of phi(Q) from S_i, Z_i
    if state is None:
        S = np.zeros((*lead, d, m))
        Z = np.zeros((*lead, d))
    else:
        S, Z = _f64(state[0]).copy(), _f64(state[1]).copy()
    gnum = np.empty((*lead, n, m))
    gden = np.empty((*lead, n))
    gfq = np.empty((*lead, n, d))
    for i in range(n):
        S = S + fk[..., i, :, None] * v[..., i, None, :]
        Z = Z + fk[..., i, :]
        den = np.einsum("...d,...d->...", fq[..., i, :], Z)
        gnum[..., i, :] = g[..., i, :] / den[..., None]
        gden[..., i] = -np.einsum("...m,...m->...", g[..., i, :], out[..., i, :]) / den
        gfq[..., i, :] = (np.einsum("...dm,...m->...d", S, gnum[..., i, :])
                          + Z * gden[..., i, None])
    # reverse sweep: gradients of phi(K) and V
    U = np.zeros((*lead, d, m))
    u = np.zeros((*lead, d))
    gfk = np.empty((*lead, n, d))
    gv = np.empty((*lead, n, m))
    for i in range(n - 1, -1, -1):
        U = U + fq[..., i, :, None] * gnum[..., i, None, :]
        u = u + fq[..., i, :] * gden[..., i, None]
        gfk[..., i, :] = np.einsum("...dm,...m->...d", U, v[..., i, :]) + u
        gv[..., i, :] = np.einsum("...dm,...d->...m", U, fk[..., i, :])
    return gfq * dphi(q), gfk * dphi(k), gv
