"""Helpers for the GPU parity tests: device copies and the error metrics.

Metrics (readings of the tolerances, one per output kind):
* forward outputs and states: max |x - ref| / max(|ref|, 1), since y is a
  convex mix of v ~ N(0, 1) and can cross zero (a pure relative error is
  ill-posed there); fp32 bound 1e-5, bf16 bound 1e-2;
* gradients: relative L2 error per tensor (gk, gv, gw, gu separately); fp32
  bound 1e-4, bf16 bound 1e-2.
"""
import numpy as np
import torch

import oracle
from rwkv_linear_rnn_b200 import workloads

F32_FWD_TOL = 1e-5
F32_GRAD_TOL = 1e-4
BF16_TOL = 1e-2


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype).contiguous()


def dev_bf16_bits(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to("cuda")
    return t.view(torch.bfloat16)


def host(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def fwd_err(x, ref):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    if x.size == 0:
        return 0.0
    return float(np.max(np.abs(x - ref) / np.maximum(np.abs(ref), 1.0)))


def rel_l2(x, ref):
    x = np.asarray(x, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def state_err(s, ref):
    """Compare states through their canonical form (A/B, ln B)."""
    ra, rb = oracle.canonical_state(ref)
    xa, xb = oracle.canonical_state(s)
    return max(fwd_err(xa, ra), fwd_err(xb, rb))


def inputs_to_device(inp):
    """Device tensors (w, u, k, v, gy) for a generated workload dict."""
    w = dev(inp["w"])
    u = dev(inp["u"])
    if inp["dtype"] == "bf16":
        k = dev_bf16_bits(inp["k_bits"])
        v = dev_bf16_bits(inp["v_bits"])
        gy = dev_bf16_bits(inp["gy_bits"]) if "gy_bits" in inp else None
    else:
        k = dev(inp["k"])
        v = dev(inp["v"])
        gy = dev(inp["gy"]) if "gy" in inp else None
    return w, u, k, v, gy

