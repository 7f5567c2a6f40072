"""Seeded synthetic inputs for the WKV operator.

This module only draws random numbers and rounds them to the storage type;
it holds none of the operator's arithmetic, so that the CUDA path and the
float64 oracle can both consume the same host arrays.

Recipe (one ``numpy.random.Generator(PCG64(seed))`` per workload, draws in
this order): time_decay [C], u [C], k [B,T,C], (spike mask and spike values
for the long-context stress case), v [B,T,C], grad_y [B,T,C].  The decay
handed to the operator is ``w = -exp(time_decay)`` rounded to float32 (the
RWKV review writes the decay as a positive rate subtracted per step of lag;
the library takes the signed per-step log-decay).  bf16 workloads round k, v
and grad_y to bfloat16 with round-to-nearest-even; w, u stay float32.

The five workloads are the shapes of RWKV-4 layers and a decode batch:

=====================  =========================================================
``tiny``               B1 T64 C64 fp32, td U(-1,1), u U(-0.5,0.5), seed 0
``rwkv169m``           B8 T1024 C768 fp32, td U(-3,1), u U(-1,1), seed 1
``rwkv1b5_bf16``       B8 T4096 C2048 bf16 I/O, k N(0,1.5), td U(-4,2), seed 2
``longctx``            B1 T65536 C2560 fp32, k N(0,3) with 0.1% of entries set
                       to U(20,30), td U(-6,2), u U(-2,2), seed 3 (forward only)
``decode14b``          512 sequences x C5120 fp32: T128 prefill (k,v N(0,1),
                       td U(-3,1), u U(-1,1)), then 32 steps of fresh k_t, v_t
                       N(0,1), seed 4
=====================  =========================================================
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    C: int
    dtype: str  # "f32" or "bf16": storage type of k, v, y, grad_y, grad_k, grad_v
    td: tuple
    u: tuple
    k_std: float
    seed: int
    ops: tuple
    spike_frac: float = 0.0
    spike_range: tuple = (20.0, 30.0)
    steps: int = 0  # decode steps after the prefill (decode workload only)
    note: str = field(default="", compare=False)

    @property
    def channel_tokens(self) -> int:
        return self.B * self.T * self.C


WORKLOADS = {
    "tiny": Workload("tiny", 1, 64, 64, "f32", (-1.0, 1.0), (-0.5, 0.5), 1.0, 0,
                     ("fwd", "bwd")),
    "rwkv169m": Workload("rwkv169m", 8, 1024, 768, "f32", (-3.0, 1.0), (-1.0, 1.0), 1.0, 1,
                         ("fwd", "bwd")),
    "rwkv1b5_bf16": Workload("rwkv1b5_bf16", 8, 4096, 2048, "bf16", (-4.0, 2.0), (-1.0, 1.0),
                             1.5, 2, ("fwd", "bwd")),
    "longctx": Workload("longctx", 1, 65536, 2560, "f32", (-6.0, 2.0), (-2.0, 2.0), 3.0, 3,
                        ("fwd",), spike_frac=0.001),
    "decode14b": Workload("decode14b", 512, 128, 5120, "f32", (-3.0, 1.0), (-1.0, 1.0), 1.0, 4,
                          ("prefill", "step"), steps=32),
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even).

    Returns the bf16 bit patterns as uint16.  NaN stays NaN.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        rounded[nan] = ((bits[nan] >> 16) | 0x40).astype(np.uint16)
    return rounded


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


def _normal(rng, shape, std):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def _uniform(rng, lo, hi, shape):
    return (lo + (hi - lo) * rng.random(size=shape, dtype=np.float64)).astype(np.float32)


def generate(wl: Workload | str, B: int | None = None, T: int | None = None,
             C: int | None = None, grad: bool = True, seed: int | None = None,
             gate: bool = False):
    """Draw one workload's inputs (host numpy arrays).

    Returns a dict with ``w, u`` (float32 [C]), ``k, v`` and, if ``grad``,
    ``gy`` ([B,T,C] float32 values, already rounded to bf16 for bf16
    workloads), and for bf16 workloads also ``k_bits, v_bits, gy_bits``
    (uint16 bf16 patterns).  B, T, C and seed may be overridden to draw a
    smaller instance with the same distributions.  ``gate`` adds the output
    gate's input ``r`` (N(0, 1), drawn after everything else so the other
    arrays do not change; ``r_bits`` for bf16).
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    C = wl.C if C is None else C
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    td = _uniform(rng, wl.td[0], wl.td[1], (C,))
    u = _uniform(rng, wl.u[0], wl.u[1], (C,))
    w = (-np.exp(td.astype(np.float64))).astype(np.float32)
    k = _normal(rng, (B, T, C), wl.k_std)
    if wl.spike_frac > 0:
        mask = rng.random(size=(B, T, C), dtype=np.float32) < np.float32(wl.spike_frac)
        n = int(mask.sum())
        k[mask] = _uniform(rng, wl.spike_range[0], wl.spike_range[1], (n,))
    v = _normal(rng, (B, T, C), 1.0)
    out = {"w": w, "u": u, "time_decay": td}
    gy = _normal(rng, (B, T, C), 1.0) if grad else None
    if wl.dtype == "bf16":
        out["k_bits"] = bf16_round(k)
        out["v_bits"] = bf16_round(v)
        k = bf16_to_f32(out["k_bits"])
        v = bf16_to_f32(out["v_bits"])
        if gy is not None:
            out["gy_bits"] = bf16_round(gy)
            gy = bf16_to_f32(out["gy_bits"])
    out["k"] = k
    out["v"] = v
    if gy is not None:
        out["gy"] = gy
    if gate:
        r = _normal(rng, (B, T, C), 1.0)
        if wl.dtype == "bf16":
            out["r_bits"] = bf16_round(r)
            r = bf16_to_f32(out["r_bits"])
        out["r"] = r
    out["B"], out["T"], out["C"], out["dtype"] = B, T, C, wl.dtype
    return out


def generate_decode_steps(wl: Workload | str = "decode14b", N: int | None = None,
                          C: int | None = None, steps: int | None = None,
                          seed: int | None = None):
    """Decode workload: prefill inputs and the per-step (k_t, v_t).

    Draw order: time_decay, u, prefill k, prefill v, then for each step
    k_t then v_t.  Returns dict with ``w, u, k, v`` (prefill, [N,T,C]) and
    ``k_steps, v_steps`` ([steps, N, C]).
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    N = wl.B if N is None else N
    C = wl.C if C is None else C
    steps = wl.steps if steps is None else steps
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    td = _uniform(rng, wl.td[0], wl.td[1], (C,))
    u = _uniform(rng, wl.u[0], wl.u[1], (C,))
    w = (-np.exp(td.astype(np.float64))).astype(np.float32)
    k = _normal(rng, (N, wl.T, C), wl.k_std)
    v = _normal(rng, (N, wl.T, C), 1.0)
    ks = np.empty((steps, N, C), np.float32)
    vs = np.empty((steps, N, C), np.float32)
    for s in range(steps):
        ks[s] = _normal(rng, (N, C), 1.0)
        vs[s] = _normal(rng, (N, C), 1.0)
    return {"w": w, "u": u, "time_decay": td, "k": k, "v": v,
            "k_steps": ks, "v_steps": vs, "N": N, "T": wl.T, "C": C}


# ----------------------------------------------- causal linear attention ---
# Shapes of the linear attention post's experiments (section "실험 설정"):
# heads of 32 dimensions (8 heads over a 256-wide embedding); MNIST image
# generation runs 784-position sequences at batch 10, CIFAR-10 3072-position
# sequences at batch 4 for the linear model.  The post states no value
# distributions; q, k, v and the output gradient are drawn N(0, 1) (unit-
# variance projections) and rounded to bfloat16, the operator's storage type.
# ``la_cifar_b32`` is the CIFAR-10 head shape at batch 32, a throughput case
# larger than L2.

@dataclass(frozen=True)
class LinAttnWorkload:
    name: str
    BH: int  # batch x heads
    N: int
    D: int   # = M
    seed: int
    note: str = ""


LINATTN_WORKLOADS = {
    "la_mnist": LinAttnWorkload("la_mnist", 10 * 8, 784, 32, 10, "MNIST: batch 10, 8 heads, N784, D=M=32"),
    "la_cifar": LinAttnWorkload("la_cifar", 4 * 8, 3072, 32, 11, "CIFAR-10: batch 4, 8 heads, N3072, D=M=32"),
    "la_cifar_b32": LinAttnWorkload("la_cifar_b32", 32 * 8, 3072, 32, 12,
                                    "CIFAR-10 head shape at batch 32: 256 heads, N3072, D=M=32"),
}


def generate_linattn(wl: LinAttnWorkload | str, BH: int | None = None, N: int | None = None,
                     grad: bool = True, seed: int | None = None):
    """Draw q, k [BH, N, D], v [BH, N, M] and (if ``grad``) g = dL/dV'.

    Draw order: q, k, v, g, each N(0, 1) float32 rounded to bfloat16.
    Returns a dict with the bf16 bit patterns (``q_bits`` ...) and the same
    values widened to float32 (``q`` ...), plus BH, N, D, M.
    """
    if isinstance(wl, str):
        wl = LINATTN_WORKLOADS[wl]
    BH = wl.BH if BH is None else BH
    N = wl.N if N is None else N
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    out = {"BH": BH, "N": N, "D": wl.D, "M": wl.D}
    for name in ("q", "k", "v", "g") if grad else ("q", "k", "v"):
        bits = bf16_round(_normal(rng, (BH, N, wl.D), 1.0))
        out[name + "_bits"] = bits
        out[name] = bf16_to_f32(bits)
    return out
