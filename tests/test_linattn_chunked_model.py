"""The chunked form of causal linear attention, checked against the oracle.

The linear attention post ("Transformers are RNNs: 선형 어텐션으로 만드는 빠른
자기회귀 트랜스포머", sections "인과 마스킹과 누적합" and "상수 메모리 기울기
계산") computes the causal product with running sums.  A tensor-core kernel
processes it in chunks of L positions, where every step is a small dense
contraction:

forward, chunk c (rows i of the chunk, A = tril(phiQ phiK^T)):
    num = A V + phiQ S_prev,   den = A 1 + phiQ Z_prev,   out = num / den,
    S = S_prev + phiK^T V,     Z = Z_prev + phiK^T 1;

backward, chunks last to first, with gnum = G / den and
gden = -rowsum(G * out) / den, P = tril(gnum V^T + gden 1^T):
    dphiQ = P phiK + gnum S_prev^T + gden Z_prev^T,
    dphiK = P^T phiQ + V U_next^T + 1 u_next^T,
    dV    = A^T gnum + phiK U_next,
    U = U_next + phiQ^T gnum,  u = u_next + phiQ^T gden,
then the chain rule through phi.  This file holds that blocked model (test
code, not the oracle) and checks it against ``oracle.linattn`` for several
chunk lengths, including ones that do not divide N, so that the algebra a
kernel will implement is settled before the kernel is written.
"""
import numpy as np
import pytest

from oracle import linattn as la


def chunked_fwd(q, k, v, L):
    fq, fk = la.phi(q), la.phi(k)
    *lead, n, d = fq.shape
    m = v.shape[-1]
    S = np.zeros((*lead, d, m))
    Z = np.zeros((*lead, d))
    out = np.empty((*lead, n, m))
    dens = np.empty((*lead, n))
    for c0 in range(0, n, L):
        sl = slice(c0, min(c0 + L, n))
        Q, K, V = fq[..., sl, :], fk[..., sl, :], v[..., sl, :]
        A = np.tril(Q @ np.swapaxes(K, -1, -2))
        num = A @ V + Q @ S
        den = A.sum(-1) + np.einsum("...id,...d->...i", Q, Z)
        out[..., sl, :] = num / den[..., None]
        dens[..., sl] = den
        S = S + np.swapaxes(K, -1, -2) @ V
        Z = Z + K.sum(-2)
    return out, dens


def chunked_bwd(q, k, v, g, L):
    fq, fk = la.phi(q), la.phi(k)
    *lead, n, d = fq.shape
    m = v.shape[-1]
    out, den = chunked_fwd(q, k, v, L)
    gnum = g / den[..., None]
    gden = -(g * out).sum(-1) / den
    # states before each chunk (forward), then the reverse sweep
    starts = list(range(0, n, L))
    S_prev, Z_prev = [], []
    S = np.zeros((*lead, d, m))
    Z = np.zeros((*lead, d))
    for c0 in starts:
        S_prev.append(S)
        Z_prev.append(Z)
        sl = slice(c0, min(c0 + L, n))
        S = S + np.swapaxes(fk[..., sl, :], -1, -2) @ v[..., sl, :]
        Z = Z + fk[..., sl, :].sum(-2)
    U = np.zeros((*lead, d, m))
    u = np.zeros((*lead, d))
    dq = np.empty_like(fq)
    dk = np.empty_like(fk)
    dv = np.empty_like(v)
    for idx in range(len(starts) - 1, -1, -1):
        c0 = starts[idx]
        sl = slice(c0, min(c0 + L, n))
        Q, K, V = fq[..., sl, :], fk[..., sl, :], v[..., sl, :]
        gn, gd = gnum[..., sl, :], gden[..., sl]
        A = np.tril(Q @ np.swapaxes(K, -1, -2))
        P = np.tril(gn @ np.swapaxes(V, -1, -2) + gd[..., :, None])
        dq[..., sl, :] = (P @ K + gn @ np.swapaxes(S_prev[idx], -1, -2)
                          + gd[..., :, None] * Z_prev[idx][..., None, :])
        dk[..., sl, :] = (np.swapaxes(P, -1, -2) @ Q + V @ np.swapaxes(U, -1, -2) + u[..., None, :])
        dv[..., sl, :] = np.swapaxes(A, -1, -2) @ gn + K @ U
        U = U + np.swapaxes(Q, -1, -2) @ gn
        u = u + np.einsum("...id,...i->...d", Q, gd)
    return dq * la.dphi(q), dk * la.dphi(k), dv


def case(seed, lead=(2, 2), N=37, D=8, M=6):
    rng = np.random.default_rng(seed)
    return (rng.normal(0, 1.2, (*lead, N, D)), rng.normal(0, 1.2, (*lead, N, D)),
            rng.normal(size=(*lead, N, M)), rng.normal(size=(*lead, N, M)))


@pytest.mark.parametrize("L", [1, 4, 8, 16, 37, 64])
def test_chunked_forward_matches_oracle(L):
    q, k, v, _ = case(L)
    ref, _ = la.fwd_recur(q, k, v)
    out, _ = chunked_fwd(q, k, v, L)
    assert np.max(np.abs(out - ref)) <= 1e-12


@pytest.mark.parametrize("L", [1, 5, 8, 16, 64])
def test_chunked_backward_matches_oracle(L):
    q, k, v, g = case(100 + L)
    ref = la.bwd_recur(q, k, v, g)
    got = chunked_bwd(q, k, v, g, L)
    for name, a, b in zip(("gq", "gk", "gv"), got, ref):
        err = np.linalg.norm(a - b) / np.linalg.norm(b)
        assert err <= 1e-12, (name, L, err)
