"""float64 CPU oracle for the RWKV-4 WKV operator (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may import this package.  The CUDA library never does, and the two
share no code: this module wraps ``wkv_oracle.c`` (plain C, IEEE double,
OpenMP over independent (batch, channel) chains) through ctypes.

Functions and the passages they follow (see the C file for the formulas):

* ``fwd_direct``   -- eq. wkv_t, "WKV 연산자" section of the RWKV paper review
                      ("[논문 리뷰] Reinvention RNNs for the Transformer Era:
                      RWKV"): the O(T^2) normalised exponential average.
* ``fwd_points``   -- the same sum at sampled (b, t, c) points.
* ``fwd_recur``    -- eq. WKV_t, "RNN-유사추론" section of the same review:
                      the hidden sums A_t, B_t advanced token by token.
* ``step``         -- one token of ``fwd_recur`` ("자기 회귀 디코딩", steps 4, 7).
* ``bwd_direct``   -- the softmax Jacobian of eq. wkv_t.
* ``bwd_recur``    -- back-propagation through the recurrence (reverse-time
                      walk, the structure of the linear-attention post's
                      gradient section).
* ``bwd_state``    -- ``bwd_recur`` with the state terms of a sequence split
                      across calls (truncated back-propagation through the
                      RNN form of "RNN-유사추론"): a loss term on the final
                      state enters as the adjoints of A_T, B_T, and the
                      gradient of the initial state (a, b, p) comes out.
* ``fwd_gated``    -- the review's output gating ("출력 게이팅(Output Gating)"
                      section, eq. o_t = W_o (sigma(r_t) * WKV_t)) without the
                      W_o projection: o_t = sigma(r_t) * wkv_t, elementwise.
* ``bwd_gated``    -- its gradients by the chain rule: the WKV backward fed
                      with grad_o * sigma(r), and grad_r = grad_o * wkv *
                      sigma(r) (1 - sigma(r)).

Conventions: arrays are float64, [B, T, C] row-major with C fastest; ``w``
(the decay itself, normally -exp(time_decay)) and ``u`` are [C]; states are
[3, B, C] planes (a, b, p) meaning A = a e^p, B = b e^p; state outputs are
canonical (A/B, 1, ln B), or (0, 0, -inf) for an empty state.  gw, gu are
summed over the batch.

The submodule ``oracle.linattn`` (numpy) holds the causal linear-attention
operator of the linear attention post, the second workload's checker, and
``oracle.tokenshift`` the token shift of the review's "토큰 변환" section.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``
against closed forms, library routines, invariants and finite differences.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libwkv_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, IEEE semantics, OpenMP)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
           "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_P = ctypes.c_void_p
_I = ctypes.c_int64


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            sigs = {
                "wkv_oracle_fwd_direct": [_I, _I, _I, _P, _P, _P, _P, _P, _P],
                "wkv_oracle_fwd_recur": [_I, _I, _I, _P, _P, _P, _P, _P, _P, _P],
                "wkv_oracle_fwd_points": [_I, _I, _I, _P, _P, _P, _P, _P, _I,
                                          _P, _P, _P, _P],
                "wkv_oracle_step": [_I, _I, _P, _P, _P, _P, _P, _P, _P],
                "wkv_oracle_bwd_direct": [_I, _I, _I, _P, _P, _P, _P, _P, _P,
                                          _P, _P, _P, _P],
                "wkv_oracle_bwd_recur": [_I, _I, _I, _P, _P, _P, _P, _P, _P,
                                         _P, _P, _P, _P],
                "wkv_oracle_bwd_recur_state": [_I, _I, _I] + [_P] * 14,
            }
            for name, args in sigs.items():
                fn = getattr(lib, name)
                fn.argtypes = args
                fn.restype = None
            lib.wkv_oracle_num_threads.restype = ctypes.c_int
            lib.wkv_oracle_set_threads.argtypes = [ctypes.c_int]
            _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _shape3(k):
    if k.ndim != 3:
        raise ValueError("k must be [B, T, C]")
    return k.shape


def num_threads() -> int:
    return _load().wkv_oracle_num_threads()


def set_threads(n: int) -> None:
    _load().wkv_oracle_set_threads(int(n))


def fwd_direct(w, u, k, v, state_in=None):
    """O(T^2) defining sum; returns y [B, T, C]."""
    lib = _load()
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    s = None if state_in is None else _f64(state_in)
    B, T, C = _shape3(k)
    y = np.empty((B, T, C))
    lib.wkv_oracle_fwd_direct(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s), _ptr(y))
    return y


def fwd_points(w, u, k, v, pb, pt, pc, state_in=None):
    """Defining sum at the points (pb[j], pt[j], pc[j]); returns [npts]."""
    lib = _load()
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    s = None if state_in is None else _f64(state_in)
    B, T, C = _shape3(k)
    pb = np.ascontiguousarray(pb, dtype=np.int64)
    pt = np.ascontiguousarray(pt, dtype=np.int64)
    pc = np.ascontiguousarray(pc, dtype=np.int64)
    assert pb.shape == pt.shape == pc.shape
    if pb.size and (pb.min() < 0 or pb.max() >= B or pt.min() < 0 or pt.max() >= T
                    or pc.min() < 0 or pc.max() >= C):
        raise ValueError("point index out of range")
    y = np.empty(pb.shape[0])
    lib.wkv_oracle_fwd_points(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s),
                              pb.shape[0], _ptr(pb), _ptr(pt), _ptr(pc), _ptr(y))
    return y


def fwd_recur(w, u, k, v, state_in=None, want_y=True):
    """Token-by-token recurrence; returns (y or None, state_out [3, B, C])."""
    lib = _load()
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    s = None if state_in is None else _f64(state_in)
    B, T, C = _shape3(k)
    y = np.empty((B, T, C)) if want_y else None
    so = np.empty((3, B, C))
    lib.wkv_oracle_fwd_recur(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s),
                             _ptr(y), _ptr(so))
    return y, so


def step(w, u, k_t, v_t, state_in):
    """One RNN-mode token for N sequences; k_t, v_t [N, C]; returns (y, state)."""
    lib = _load()
    w, u, k_t, v_t, s = _f64(w), _f64(u), _f64(k_t), _f64(v_t), _f64(state_in)
    N, C = k_t.shape
    y = np.empty((N, C))
    so = np.empty((3, N, C))
    lib.wkv_oracle_step(N, C, _ptr(w), _ptr(u), _ptr(k_t), _ptr(v_t), _ptr(s), _ptr(y), _ptr(so))
    return y, so


def _bwd(fn, w, u, k, v, gy, state_in):
    w, u, k, v, gy = _f64(w), _f64(u), _f64(k), _f64(v), _f64(gy)
    s = None if state_in is None else _f64(state_in)
    B, T, C = _shape3(k)
    gw = np.empty(C)
    gu = np.empty(C)
    gk = np.empty((B, T, C))
    gv = np.empty((B, T, C))
    fn(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s), _ptr(gy),
       _ptr(gw), _ptr(gu), _ptr(gk), _ptr(gv))
    return gw, gu, gk, gv


def bwd_direct(w, u, k, v, gy, state_in=None):
    """Softmax-Jacobian backward; returns (gw [C], gu [C], gk, gv)."""
    return _bwd(_load().wkv_oracle_bwd_direct, w, u, k, v, gy, state_in)


def bwd_recur(w, u, k, v, gy, state_in=None):
    """Reverse-time backward of the recurrence; returns (gw, gu, gk, gv)."""
    return _bwd(_load().wkv_oracle_bwd_recur, w, u, k, v, gy, state_in)


def canonical_state(state):
    """(a, b, p) -> (A/B, ln B) with A = a e^p, B = b e^p; empty -> (0, -inf).

    The (a, b, p) form is not unique (any (a e^d, b e^d, p - d) is the same
    state); this pair is.
    """
    st = np.asarray(state, dtype=np.float64)
    a, b, p = st[0], st[1], st[2]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(b > 0, a / np.where(b > 0, b, 1.0), 0.0)
        logb = np.where(b > 0, p + np.log(np.where(b > 0, b, 1.0)), -np.inf)
    return ratio, logb


def sigmoid(x):
    """Logistic function 1 / (1 + e^-x) in float64, without overflow for
    large |x| (e^-x is formed only for x >= 0, e^x only for x < 0)."""
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def fwd_gated(w, u, k, v, r, state_in=None):
    """o_t = sigma(r_t) * wkv_t; returns (o, final state)."""
    y, st = fwd_recur(w, u, k, v, state_in)
    return sigmoid(r) * y, st


def bwd_gated(w, u, k, v, r, go, state_in=None):
    """Gradients of L = sum(go * o) for o = sigma(r) * wkv; returns
    (gw, gu, gk, gv, gr)."""
    y, _ = fwd_recur(w, u, k, v, state_in)
    sr = sigmoid(r)
    gw, gu, gk, gv = bwd_recur(w, u, k, v, _f64(go) * sr, state_in)
    gr = _f64(go) * y * sr * (1.0 - sr)
    return gw, gu, gk, gv, gr


def bwd_state(w, u, k, v, gy, state_in=None, state_out=None, grad_state_out=None):
    """``bwd_recur`` with the recurrent state's gradients; returns
    (gw, gu, gk, gv, grad_state_in [3, B, C]).

    ``grad_state_out`` [3, B, C] is dL/d(a, b, p) of the state after the last
    token in the representation ``state_out`` (any (a, b, p) of that state:
    only its p is read).  The loss is taken to depend on the state only
    through the sums it represents, A = a e^p and B = b e^p, so
    dL/dA_T = ga e^{-p}, dL/dB_T = gb e^{-p}, and the p component (then
    a ga + b gb, no extra information) is not read.  An empty state
    (p = -inf) passes no gradient.  ``grad_state_in`` is dL/d(a, b, p) of
    ``state_in`` exactly as given: (dL/dA_0 e^p, dL/dB_0 e^p,
    A_0 dL/dA_0 + B_0 dL/dB_0); zeros for ``state_in=None`` (the empty
    state, p = -inf).
    """
    w, u, k, v, gy = _f64(w), _f64(u), _f64(k), _f64(v), _f64(gy)
    s = None if state_in is None else _f64(state_in)
    B, T, C = _shape3(k)
    gA_T = gB_T = None
    if grad_state_out is not None:
        if state_out is None:
            raise ValueError("grad_state_out needs the state_out it refers to")
        go, so = _f64(grad_state_out), _f64(state_out)
        p = so[2]
        with np.errstate(over="ignore", invalid="ignore"):
            scale = np.where(np.isneginf(p), 0.0, np.exp(-np.where(np.isneginf(p), 0.0, p)))
        gA_T = np.ascontiguousarray(go[0] * scale)
        gB_T = np.ascontiguousarray(go[1] * scale)
    gw, gu = np.empty(C), np.empty(C)
    gk, gv = np.empty((B, T, C)), np.empty((B, T, C))
    gA_0, gB_0 = np.empty((B, C)), np.empty((B, C))
    _load().wkv_oracle_bwd_recur_state(B, T, C, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(s),
                                       _ptr(gy), _ptr(gA_T), _ptr(gB_T), _ptr(gw), _ptr(gu),
                                       _ptr(gk), _ptr(gv), _ptr(gA_0), _ptr(gB_0))
    gs_in = np.zeros((3, B, C))
    if s is not None:
        a, b, p = s[0], s[1], s[2]
        e = np.exp(p)  # 0 for an empty state
        gs_in[0] = gA_0 * e
        gs_in[1] = gB_0 * e
        gs_in[2] = a * gs_in[0] + b * gs_in[1]  # A_0 dL/dA_0 + B_0 dL/dB_0
    return gw, gu, gk, gv, gs_in
