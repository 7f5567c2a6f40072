"""GPU parity of the causal linear attention kernels against the float64 oracle.

The oracle is ``oracle.linattn`` (the linear attention post: the causal form
with cumulative states of section "인과 마스킹과 누적합" and the gradients of
section "상수 메모리 기울기 계산").  Inputs are bfloat16, the operator's
storage type, and the oracle runs on the same rounded values in float64.

Tolerances: outputs and the final state by the forward metric
(max |x - ref| / max(|ref|, 1)) within 1e-2, gradients by relative L2 per
tensor within 1e-2 -- the bf16-I/O bounds of the WKV operator.  The kernels
round their tensor-core operands (phi(Q), phi(K), the masked scores, the
chunk states) and their outputs to bfloat16, so each output carries a few
bf16 roundings (2^-8 relative each) of positively weighted sums.
"""
import numpy as np
import pytest
import torch

import rwkv_linear_rnn_b200 as W
from oracle import linattn as la
from rwkv_linear_rnn_b200 import workloads
from gpu_util import BF16_TOL, dev_bf16_bits, fwd_err, host, rel_l2

pytestmark = pytest.mark.gpu


def case(BH, N, seed, std=1.0, D=32):
    rng = np.random.default_rng(seed)
    out = {}
    for name in ("q", "k", "v", "g"):
        bits = workloads.bf16_round((rng.normal(0, std if name in "qk" else 1.0, (BH, N, D))).astype(np.float32))
        out[name + "_bits"] = bits
        out[name] = workloads.bf16_to_f32(bits)
    return out


def on_device(inp, names=("q", "k", "v", "g")):
    return [dev_bf16_bits(inp[n + "_bits"]) for n in names]


def check_forward(inp, heads=None):
    q, k, v = on_device(inp, ("q", "k", "v"))
    out, (S, Z) = W.linattn_forward(q, k, v, want_state=True)
    sel = slice(None) if heads is None else heads
    ref, (S_ref, Z_ref) = la.fwd_recur(inp["q"][sel], inp["k"][sel], inp["v"][sel])
    assert fwd_err(host(out)[sel], ref) <= BF16_TOL
    # the state by the same metric, relative to its own scale (sums of N terms)
    scale = max(1.0, float(np.max(np.abs(Z_ref))))
    assert np.max(np.abs(host(S)[sel] - S_ref)) / scale <= BF16_TOL
    assert np.max(np.abs(host(Z)[sel] - Z_ref)) / scale <= BF16_TOL
    return out


def check_backward(inp, heads=None):
    q, k, v, g = on_device(inp)
    got = W.linattn_backward(q, k, v, g)
    sel = slice(None) if heads is None else heads
    ref = la.bwd_recur(inp["q"][sel], inp["k"][sel], inp["v"][sel], inp["g"][sel])
    for name, a, b in zip(("gq", "gk", "gv"), got, ref):
        x = host(a)[sel]
        if np.linalg.norm(b) <= 1e-9 * np.sqrt(b.size):
            # zero up to rounding (N = 1: out_0 = v_0 whatever q and k are, so
            # dL/dq = dL/dk = 0): no relative error; bound the absolute one
            assert np.max(np.abs(x)) <= BF16_TOL, (name, np.max(np.abs(x)))
            continue
        e = rel_l2(x, b)
        assert e <= BF16_TOL, (name, e)
    return got


@pytest.mark.parametrize("BH,N", [(1, 1), (2, 5), (1, 127), (1, 128), (3, 129), (2, 300), (1, 1000)])
def test_forward_small_and_ragged(BH, N):
    """One chunk, a partial chunk, exactly one chunk, one past a chunk, and
    several chunks with a ragged tail."""
    inp = case(BH, N, seed=BH * 1000 + N)
    out = check_forward(inp)
    if N <= 300:  # the O(N^2) definition as well
        ref = la.fwd_direct(inp["q"], inp["k"], inp["v"])
        assert fwd_err(host(out), ref) <= BF16_TOL


def test_forward_wide_inputs():
    """q, k ~ N(0, 3): phi spans e^-9 .. 10, the scores over four decades."""
    check_forward(case(4, 700, seed=5, std=3.0))


@pytest.mark.parametrize("name", ["la_mnist", "la_cifar"])
def test_forward_workloads(name):
    check_forward(workloads.generate_linattn(name, grad=False))


def test_forward_batch32_workload_head_subset():
    inp = workloads.generate_linattn("la_cifar_b32", grad=False)
    check_forward(inp, heads=np.arange(0, inp["BH"], 8))


@pytest.mark.parametrize("BH,N", [(1, 1), (2, 5), (1, 128), (3, 129), (2, 300), (1, 1000)])
def test_backward_small_and_ragged(BH, N):
    check_backward(case(BH, N, seed=7 * BH + N))


def test_backward_wide_inputs():
    check_backward(case(4, 700, seed=6, std=3.0))


@pytest.mark.parametrize("name", ["la_mnist", "la_cifar"])
def test_backward_workloads(name):
    check_backward(workloads.generate_linattn(name))


def test_backward_batch32_workload_head_subset():
    inp = workloads.generate_linattn("la_cifar_b32")
    check_backward(inp, heads=np.arange(3, inp["BH"], 16))


def test_results_are_bit_reproducible():
    """Chunk states are summed in a fixed order: two runs give the same bits."""
    inp = workloads.generate_linattn("la_cifar")
    q, k, v, g = on_device(inp)
    a = (W.linattn_forward(q, k, v)[0],) + W.linattn_backward(q, k, v, g)
    b = (W.linattn_forward(q, k, v)[0],) + W.linattn_backward(q, k, v, g)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_empty_sequence_and_status():
    q = torch.zeros((3, 0, 32), dtype=torch.bfloat16, device="cuda")
    out, (S, Z) = W.linattn_forward(q, q.clone(), q.clone(), want_state=True)
    assert out.shape == (3, 0, 32)
    assert torch.count_nonzero(S) == 0 and torch.count_nonzero(Z) == 0
    gq, gk, gv = W.linattn_backward(q, q.clone(), q.clone(), q.clone())
    assert gq.numel() == 0
    ws = W.Workspace()
    inp = case(2, 300, seed=9)
    qq, kk, vv, gg = on_device(inp)
    W.linattn_forward(qq, kk, vv, workspace=ws)
    W.linattn_backward(qq, kk, vv, gg, workspace=ws)
    assert ws.status() == 0


def test_outputs_stay_inside_their_buffers():
    """Ragged tails are clipped by the tensor maps: guard bytes on both sides
    of every output survive."""
    BH, N, D = 2, 200, 32
    inp = case(BH, N, seed=11)
    q, k, v, g = on_device(inp)
    n = BH * N * D
    guard = 4096
    bufs = [torch.full((n + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    out, gq, gk, gv = (b[guard:guard + n].view(BH, N, D) for b in bufs)
    W.linattn_forward(q, k, v, out=out)
    W.linattn_backward(q, k, v, g, grad_q=gq, grad_k=gk, grad_v=gv)
    torch.cuda.synchronize()
    for b in bufs:
        assert torch.all(b[:guard] == 7.0) and torch.all(b[guard + n:] == 7.0)
    assert fwd_err(host(out), la.fwd_recur(inp["q"], inp["k"], inp["v"])[0]) <= BF16_TOL


def check_backward_saved(inp, heads=None):
    """The backward from the forward's saved state: forward, then the
    gradients with its output, on one workspace."""
    q, k, v, g = on_device(inp)
    ws = W.Workspace()
    out, _ = W.linattn_forward(q, k, v, workspace=ws)
    got = W.linattn_backward(q, k, v, g, out=out, workspace=ws)
    sel = slice(None) if heads is None else heads
    ref = la.bwd_recur(inp["q"][sel], inp["k"][sel], inp["v"][sel], inp["g"][sel])
    for name, a, b in zip(("gq", "gk", "gv"), got, ref):
        x = host(a)[sel]
        if np.linalg.norm(b) <= 1e-9 * np.sqrt(b.size):
            assert np.max(np.abs(x)) <= BF16_TOL, (name, np.max(np.abs(x)))
            continue
        assert rel_l2(x, b) <= BF16_TOL, (name, rel_l2(x, b))
    return got


@pytest.mark.parametrize("BH,N", [(1, 1), (2, 5), (1, 128), (3, 129), (2, 300), (1, 1000)])
def test_backward_saved_small_and_ragged(BH, N):
    check_backward_saved(case(BH, N, seed=11 * BH + N))


@pytest.mark.parametrize("name", ["la_mnist", "la_cifar"])
def test_backward_saved_workloads(name):
    check_backward_saved(workloads.generate_linattn(name))


def test_backward_saved_agrees_with_recompute():
    """The saved-state backward and the recomputing one differ by rounding
    only: the reused state is the forward's own, and dL/d(den) takes the
    bf16 output instead of the float32 one."""
    inp = case(4, 700, seed=21)
    q, k, v, g = on_device(inp)
    ws = W.Workspace()
    out, _ = W.linattn_forward(q, k, v, workspace=ws)
    saved = W.linattn_backward(q, k, v, g, out=out, workspace=ws)
    recomputed = W.linattn_backward(q, k, v, g, workspace=W.Workspace())
    for a, b in zip(saved, recomputed):
        assert rel_l2(host(a), host(b)) <= 5e-3


def test_workspace_reuse_across_shapes():
    """One workspace through calls of different shapes (its regions move
    with BH and N): every forward and saved-state backward matches the
    oracle, and the repeated shape gives the same bits as its first call."""
    ws = W.Workspace()
    seen = {}
    for BH, N in [(3, 700), (1, 129), (5, 40), (3, 700)]:
        inp = case(BH, N, seed=BH * 31 + N)
        q, k, v, g = on_device(inp)
        out, (S, Z) = W.linattn_forward(q, k, v, want_state=True, workspace=ws)
        grads = W.linattn_backward(q, k, v, g, out=out, workspace=ws)
        assert fwd_err(host(out), la.fwd_recur(inp["q"], inp["k"], inp["v"])[0]) <= BF16_TOL
        for name, a, b in zip(("gq", "gk", "gv"), grads, la.bwd_recur(inp["q"], inp["k"], inp["v"], inp["g"])):
            assert rel_l2(host(a), b) <= BF16_TOL, (BH, N, name)
        res = (out.clone(), S.clone(), Z.clone()) + tuple(x.clone() for x in grads)
        if (BH, N) in seen:
            for a, b in zip(seen[(BH, N)], res):
                assert torch.equal(a, b)
        seen[(BH, N)] = res
    assert ws.status() == 0


def test_many_short_heads():
    """600 heads of 40 positions: one ragged chunk per head, far more chunks
    than resident CTAs, so every persistent CTA walks several heads."""
    check_forward(case(600, 40, seed=3))
    check_backward_saved(case(600, 40, seed=4))
