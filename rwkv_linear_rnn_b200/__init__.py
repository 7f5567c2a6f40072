"""libwkv: the RWKV-4 WKV time-mixing operator on NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/wkv.h`` and
``include/linattn.h`` (causal linear attention: ``linattn_forward``,
``linattn_backward``).  The functions in
``abi`` carry the C names and take raw device pointers (ints) -- argument
marshalling only.  The tensor helpers below (``forward``, ``backward``,
``step``, ``WKV``, ``backward_state``, ``token_shift`` and the gated ``forward_gated``, ``backward_gated``,
``GatedWKV``) take torch CUDA tensors, allocate outputs with torch, and
call the same entry points; PyTorch provides memory and streams only, every
step of the operator runs in the library's CUDA kernels.

The library is required: importing this package fails loudly if
``libwkv.so`` is missing (build it with ``python -m rwkv_linear_rnn_b200.build``).
There is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import importlib

from .constants import (WKV_BF16, WKV_F32, WKV_KERNEL_AUTO, WKV_KERNEL_CHUNKED,
                        WKV_KERNEL_CLUSTER, WKV_KERNEL_SEGMENT, WKV_KERNEL_TILE, WKV_KERNEL_CHAIN,
                        WKV_KERNEL_CHUNKED_REGS, WKV_KERNEL_SEQUENTIAL, WKV_OP_BACKWARD,
                        WKV_OP_FORWARD, WKV_OP_STEP, WKV_STATIC_SCRATCH_BYTES)

__all__ = [
    "abi", "WKVError", "WKV_F32", "WKV_BF16", "WKV_OP_FORWARD", "WKV_OP_BACKWARD", "WKV_OP_STEP",
    "WKV_KERNEL_AUTO", "WKV_KERNEL_SEQUENTIAL", "WKV_KERNEL_CHUNKED", "WKV_KERNEL_CHUNKED_REGS",
    "WKV_KERNEL_SEGMENT", "WKV_KERNEL_CLUSTER", "WKV_KERNEL_TILE", "WKV_KERNEL_CHAIN", "WKV_STATIC_SCRATCH_BYTES", "Workspace", "forward", "backward", "backward_state", "step", "token_shift",
    "token_shift_backward", "TokenShift",
    "forward_gated", "backward_gated", "WKV", "wkv", "WKVState", "wkv_state", "GatedWKV", "gated_wkv", "wkv_workspace_size", "wkv_ckpt_size", "wkv_strerror", "wkv_version",
    "library_path", "LINATTN_OP_FORWARD", "LINATTN_OP_BACKWARD", "linattn_workspace_size",
    "linattn_forward", "linattn_backward",
]


def __getattr__(name):
    # The ctypes layer (and with it libwkv.so) loads on first use; it raises
    # ImportError with a build hint if the library has not been built.
    if name in ("abi", "WKVError"):
        abi_mod = importlib.import_module(".abi", __name__)
        return abi_mod if name == "abi" else abi_mod.WKVError
    raise AttributeError(name)


def _abi():
    return importlib.import_module(".abi", __name__)


def wkv_workspace_size(op, B, T, C, dtype):
    return _abi().wkv_workspace_size(op, B, T, C, dtype)


def wkv_ckpt_size(B, T, C):
    return _abi().wkv_ckpt_size(B, T, C)


def wkv_strerror(status):
    return _abi().wkv_strerror(status)


def wkv_version():
    return _abi().wkv_version()


def library_path() -> str:
    return _abi().LIB_PATH


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return WKV_F32
    if t.dtype == torch.bfloat16:
        return WKV_BF16
    raise TypeError(f"k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t):
    return 0 if t is None else t.data_ptr()


def _stream(stream):
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


class Workspace:
    """A zero-initialised device workspace that grows on demand.

    One workspace may serve forward and backward calls of any shape, as long
    as they are ordered on one stream.
    """

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, op, B, T, C, dtype):
        return self.get_bytes(wkv_workspace_size(op, B, T, C, dtype))

    def get_bytes(self, need):
        torch = _torch()
        if need == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < need:
            # zero-filled: the library requires a zeroed workspace before first use
            self.buf = torch.zeros(need + 256, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf, self.buf.numel()

    def status(self, stream=None) -> int:
        """Device-side status of earlier calls (waits for the stream); clears it."""
        if self.buf is None:
            return 0
        return _abi().wkv_get_status(self.buf.data_ptr(), _stream(stream))


_default_ws = {}


def _ws_for(device, ws):
    if ws is not None:
        return ws
    key = str(device)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def forward(w, u, k, v, state_in=None, *, want_state=False, want_ckpt=False, y=None,
            workspace=None, stream=None, kernel=WKV_KERNEL_AUTO):
    """y = WKV(w, u, k, v) for k, v [B, T, C]; optionally the final state and
    the checkpoints for ``backward``.  Returns (y, state_out, ckpt)."""
    torch = _torch()
    _check_cuda(w, u, k, v, state_in, y)
    B, T, C = k.shape
    dt = _dtype_code(k)
    if y is None:
        y = torch.empty_like(k)
    state_out = torch.empty((3, B, C), dtype=torch.float32, device=k.device) if want_state else None
    ckpt = None
    if want_ckpt:
        n = wkv_ckpt_size(B, T, C) // 4
        ckpt = torch.empty(max(n, 1), dtype=torch.float32, device=k.device)
    ws = _ws_for(k.device, workspace)
    buf, nbytes = ws.get(WKV_OP_FORWARD, B, T, C, dt)
    abi = _abi()
    opts = abi.Options(kernel=kernel)
    abi.check(abi.wkv_forward_ex(B, T, C, dt, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(state_in),
                                 _ptr(y), _ptr(state_out), _ptr(ckpt), _ptr(buf), nbytes,
                                 _stream(stream), opts))
    return y, state_out, ckpt


def backward(w, u, k, v, grad_y, state_in=None, ckpt=None, *, grad_k=None, grad_v=None,
             workspace=None, stream=None, kernel=WKV_KERNEL_AUTO):
    """Gradients (grad_w [C], grad_u [C], grad_k, grad_v) of L given grad_y.
    ``grad_k`` / ``grad_v`` may be given as output buffers (shape and dtype of k)."""
    torch = _torch()
    _check_cuda(w, u, k, v, grad_y, state_in, ckpt, grad_k, grad_v)
    B, T, C = k.shape
    dt = _dtype_code(k)
    gw = torch.empty(C, dtype=torch.float32, device=k.device)
    gu = torch.empty(C, dtype=torch.float32, device=k.device)
    gk = torch.empty_like(k) if grad_k is None else grad_k
    gv = torch.empty_like(v) if grad_v is None else grad_v
    ws = _ws_for(k.device, workspace)
    buf, nbytes = ws.get(WKV_OP_BACKWARD, B, T, C, dt)
    abi = _abi()
    opts = abi.Options(kernel=kernel)
    abi.check(abi.wkv_backward_ex(B, T, C, dt, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(grad_y),
                                  _ptr(state_in), _ptr(ckpt), _ptr(gw), _ptr(gu), _ptr(gk),
                                  _ptr(gv), _ptr(buf), nbytes, _stream(stream), opts))
    return gw, gu, gk, gv


def backward_state(w, u, k, v, grad_y, state_in=None, ckpt=None, *, state_out=None,
                   grad_state_out=None, want_grad_state_in=True, grad_k=None, grad_v=None,
                   workspace=None, stream=None, kernel=WKV_KERNEL_AUTO):
    """``backward`` with the state terms of a sequence split across calls.
    ``grad_state_out`` is dL/d(a, b, p) of the state after the last token,
    given in the representation ``state_out`` (only its p is read).  Returns
    (grad_w, grad_u, grad_k, grad_v, grad_state_in); grad_state_in is
    dL/d(a, b, p) of ``state_in`` as given (None unless wanted)."""
    torch = _torch()
    _check_cuda(w, u, k, v, grad_y, state_in, ckpt, state_out, grad_state_out, grad_k, grad_v)
    B, T, C = k.shape
    dt = _dtype_code(k)
    gw = torch.empty(C, dtype=torch.float32, device=k.device)
    gu = torch.empty(C, dtype=torch.float32, device=k.device)
    gk = torch.empty_like(k) if grad_k is None else grad_k
    gv = torch.empty_like(v) if grad_v is None else grad_v
    gs = torch.empty((3, B, C), dtype=torch.float32, device=k.device) if want_grad_state_in else None
    ws = _ws_for(k.device, workspace)
    buf, nbytes = ws.get(WKV_OP_BACKWARD, B, T, C, dt)
    abi = _abi()
    opts = abi.Options(kernel=kernel)
    abi.check(abi.wkv_backward_state_ex(B, T, C, dt, _ptr(w), _ptr(u), _ptr(k), _ptr(v),
                                        _ptr(grad_y), _ptr(state_in), _ptr(ckpt), _ptr(state_out),
                                        _ptr(grad_state_out), _ptr(gw), _ptr(gu), _ptr(gk),
                                        _ptr(gv), _ptr(gs), _ptr(buf), nbytes, _stream(stream),
                                        opts))
    return gw, gu, gk, gv, gs


# ------------------------------------------------ causal linear attention ---

LINATTN_OP_FORWARD, LINATTN_OP_BACKWARD = 0, 1


def linattn_workspace_size(op, BH, N, D, M):
    return _abi().linattn_workspace_size(op, BH, N, D, M)


def _check_linattn(q, k, v, *more):
    torch = _torch()
    _check_cuda(q, k, v, *more)
    for t in (q, k, v) + tuple(x for x in more if x is not None):
        if t.dtype != torch.bfloat16 or t.dim() != 3:
            raise ValueError("linear attention takes bfloat16 [BH, N, D] tensors")
    BH, N, D = q.shape
    if k.shape != q.shape or v.shape[:2] != (BH, N):
        raise ValueError("q, k must be [BH, N, D] and v [BH, N, M]")
    return BH, N, D, v.shape[2]


def linattn_forward(q, k, v, *, want_state=False, out=None, workspace=None, stream=None):
    """Causal linear attention (elu + 1 feature map) for q, k [BH, N, D] and
    v [BH, N, M], bfloat16 (include/linattn.h).  Returns (out [BH, N, M],
    state or None) with state = (S [BH, D, M], Z [BH, D]) float32 after the
    last position."""
    torch = _torch()
    BH, N, D, M = _check_linattn(q, k, v, out)
    if out is None:
        out = torch.empty((BH, N, M), dtype=torch.bfloat16, device=q.device)
    st = torch.empty(BH * (D * M + D), dtype=torch.float32, device=q.device) if want_state else None
    ws = _ws_for(q.device, workspace)
    # backward-sized, so that linattn_backward(..., out=out) can reuse the
    # state this call leaves in the workspace
    buf, nbytes = ws.get_bytes(linattn_workspace_size(LINATTN_OP_BACKWARD, BH, N, D, M))
    abi = _abi()
    abi.check(abi.linattn_forward(BH, N, D, M, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(st),
                                  _ptr(buf), nbytes, _stream(stream)))
    if st is not None:
        st = (st[:BH * D * M].view(BH, D, M), st[BH * D * M:].view(BH, D))
    return out, st


def linattn_backward(q, k, v, grad_out, *, out=None, grad_q=None, grad_k=None, grad_v=None, workspace=None,
                     stream=None):
    """Gradients (grad_q, grad_k, grad_v) of L given grad_out = dL/dV'.

    With ``out`` (the output of the ``linattn_forward`` call on these q, k, v
    that used the same workspace, with no call on it since), the forward's
    saved chunk states and denominators are reused instead of recomputed
    (``linattn_backward_saved``)."""
    torch = _torch()
    BH, N, D, M = _check_linattn(q, k, v, grad_out, out, grad_q, grad_k, grad_v)
    grad_q = torch.empty_like(q) if grad_q is None else grad_q
    grad_k = torch.empty_like(k) if grad_k is None else grad_k
    grad_v = torch.empty_like(v) if grad_v is None else grad_v
    ws = _ws_for(q.device, workspace)
    buf, nbytes = ws.get_bytes(linattn_workspace_size(LINATTN_OP_BACKWARD, BH, N, D, M))
    abi = _abi()
    if out is not None:
        abi.check(abi.linattn_backward_saved(BH, N, D, M, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(grad_out),
                                             _ptr(grad_q), _ptr(grad_k), _ptr(grad_v), _ptr(buf), nbytes,
                                             _stream(stream)))
    else:
        abi.check(abi.linattn_backward(BH, N, D, M, _ptr(q), _ptr(k), _ptr(v), _ptr(grad_out), _ptr(grad_q),
                                       _ptr(grad_k), _ptr(grad_v), _ptr(buf), nbytes, _stream(stream)))
    return grad_q, grad_k, grad_v


def token_shift(x, mu, x_prev=None, *, out=None, stream=None):
    """out[m] = mu[m] * x[t] + (1 - mu[m]) * x[t-1] for x [B, T, C] and
    mu [n, C] (float32); x[-1] = x_prev [B, C] or 0.  Returns out [n, B, T, C]."""
    torch = _torch()
    _check_cuda(x, mu, x_prev, out)
    B, T, C = x.shape
    n = mu.shape[0]
    if out is None:
        out = torch.empty((n, B, T, C), dtype=x.dtype, device=x.device)
    abi = _abi()
    abi.check(abi.wkv_token_shift(B, T, C, _dtype_code(x), n, _ptr(mu), _ptr(x), _ptr(x_prev),
                                  _ptr(out), _stream(stream)))
    return out


def token_shift_backward(x, mu, grad_out, x_prev=None, *, want_grad_x_prev=False, stream=None):
    """Gradients (grad_x, grad_mu, grad_x_prev or None) of L given
    grad_out = dL/dout [n, B, T, C]."""
    torch = _torch()
    _check_cuda(x, mu, grad_out, x_prev)
    B, T, C = x.shape
    n = mu.shape[0]
    gx = torch.empty_like(x)
    gmu = torch.empty((n, C), dtype=torch.float32, device=x.device)
    gxp = torch.empty((B, C), dtype=x.dtype, device=x.device) if want_grad_x_prev else None
    abi = _abi()
    nws = abi.wkv_token_shift_workspace_size(B, T, C, n)
    ws = torch.empty(max(nws, 1), dtype=torch.uint8, device=x.device)
    abi.check(abi.wkv_token_shift_backward(B, T, C, _dtype_code(x), n, _ptr(mu), _ptr(x),
                                           _ptr(x_prev), _ptr(grad_out), _ptr(gx), _ptr(gmu),
                                           _ptr(gxp), _ptr(ws), nws, _stream(stream)))
    return gx, gmu, gxp


def forward_gated(w, u, k, v, r, state_in=None, *, want_state=False, want_ckpt=False, o=None,
                  workspace=None, stream=None, kernel=WKV_KERNEL_AUTO):
    """o = sigmoid(r) * WKV(w, u, k, v) for k, v, r [B, T, C].  Returns
    (o, state_out, ckpt) as ``forward`` does (the state and checkpoints are the
    WKV recurrence's)."""
    torch = _torch()
    _check_cuda(w, u, k, v, r, state_in, o)
    B, T, C = k.shape
    dt = _dtype_code(k)
    if o is None:
        o = torch.empty_like(k)
    state_out = torch.empty((3, B, C), dtype=torch.float32, device=k.device) if want_state else None
    ckpt = None
    if want_ckpt:
        n = wkv_ckpt_size(B, T, C) // 4
        ckpt = torch.empty(max(n, 1), dtype=torch.float32, device=k.device)
    ws = _ws_for(k.device, workspace)
    buf, nbytes = ws.get(WKV_OP_FORWARD, B, T, C, dt)
    abi = _abi()
    opts = abi.Options(kernel=kernel)
    abi.check(abi.wkv_forward_gated_ex(B, T, C, dt, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                       _ptr(state_in), _ptr(o), _ptr(state_out), _ptr(ckpt),
                                       _ptr(buf), nbytes, _stream(stream), opts))
    return o, state_out, ckpt


def backward_gated(w, u, k, v, r, grad_o, state_in=None, ckpt=None, *, grad_k=None, grad_v=None,
                   grad_r=None, workspace=None, stream=None, kernel=WKV_KERNEL_AUTO):
    """Gradients (grad_w, grad_u, grad_k, grad_v, grad_r) of L given
    grad_o = dL/do for o = sigmoid(r) * WKV(w, u, k, v)."""
    torch = _torch()
    _check_cuda(w, u, k, v, r, grad_o, state_in, ckpt, grad_k, grad_v, grad_r)
    B, T, C = k.shape
    dt = _dtype_code(k)
    gw = torch.empty(C, dtype=torch.float32, device=k.device)
    gu = torch.empty(C, dtype=torch.float32, device=k.device)
    gk = torch.empty_like(k) if grad_k is None else grad_k
    gv = torch.empty_like(v) if grad_v is None else grad_v
    gr = torch.empty_like(r) if grad_r is None else grad_r
    ws = _ws_for(k.device, workspace)
    buf, nbytes = ws.get(WKV_OP_BACKWARD, B, T, C, dt)
    abi = _abi()
    opts = abi.Options(kernel=kernel)
    abi.check(abi.wkv_backward_gated_ex(B, T, C, dt, _ptr(w), _ptr(u), _ptr(k), _ptr(v), _ptr(r),
                                        _ptr(grad_o), _ptr(state_in), _ptr(ckpt), _ptr(gw),
                                        _ptr(gu), _ptr(gk), _ptr(gv), _ptr(gr), _ptr(buf), nbytes,
                                        _stream(stream), opts))
    return gw, gu, gk, gv, gr


def step(w, u, k_t, v_t, state, *, y=None, state_out=None, stream=None):
    """One RNN-mode token for N sequences.  ``state_out`` defaults to updating
    ``state`` in place.  Returns (y_t, state_out)."""
    torch = _torch()
    _check_cuda(w, u, k_t, v_t, state, y, state_out)
    N, C = k_t.shape
    if y is None:
        y = torch.empty_like(k_t)
    if state_out is None:
        state_out = state
    abi = _abi()
    abi.check(abi.wkv_step(N, C, _ptr(w), _ptr(u), _ptr(k_t), _ptr(v_t), _ptr(state), _ptr(y),
                           _ptr(state_out), _stream(stream)))
    return y, state_out


class WKV:
    """torch.autograd.Function wrapper: y = WKV.apply(w, u, k, v)."""

    _fn = None

    @classmethod
    def apply(cls, w, u, k, v):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, w, u, k, v):
                    w, u, k, v = (t.contiguous() for t in (w, u, k, v))
                    y, _, ck = forward(w, u, k, v, want_ckpt=True)
                    ctx.save_for_backward(w, u, k, v, ck)
                    return y

                @staticmethod
                def backward(ctx, gy):
                    w, u, k, v, ck = ctx.saved_tensors
                    gw, gu, gk, gv = backward(w, u, k, v, gy.contiguous(), ckpt=ck)
                    return gw, gu, gk, gv

            cls._fn = _F
        return cls._fn.apply(w, u, k, v)


def wkv(w, u, k, v):
    """Differentiable WKV: y [B, T, C] from w, u [C] and k, v [B, T, C]."""
    return WKV.apply(w, u, k, v)


class WKVState:
    """torch.autograd.Function wrapper with the recurrent state:
    (y, state_out) = WKVState.apply(w, u, k, v, state_in).  Gradients reach
    state_in through both y and state_out, so a sequence split across calls
    back-propagates through the state (truncated BPTT)."""

    _fn = None

    @classmethod
    def apply(cls, w, u, k, v, state_in):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, w, u, k, v, state_in):
                    w, u, k, v, state_in = (t.contiguous() for t in (w, u, k, v, state_in))
                    y, s_out, ck = forward(w, u, k, v, state_in, want_state=True, want_ckpt=True)
                    ctx.save_for_backward(w, u, k, v, state_in, s_out, ck)
                    return y, s_out

                @staticmethod
                def backward(ctx, gy, gs):
                    w, u, k, v, state_in, s_out, ck = ctx.saved_tensors
                    gy = torch.zeros_like(k) if gy is None else gy.contiguous()
                    gs = None if gs is None else gs.contiguous()
                    return backward_state(w, u, k, v, gy, state_in, ck, state_out=s_out,
                                          grad_state_out=gs)

            cls._fn = _F
        return cls._fn.apply(w, u, k, v, state_in)


def wkv_state(w, u, k, v, state_in):
    """Differentiable WKV with the state: (y, state_out) from w, u [C],
    k, v [B, T, C] and state_in [3, B, C]."""
    return WKVState.apply(w, u, k, v, state_in)


class TokenShift:
    """torch.autograd.Function wrapper: out = TokenShift.apply(x, mu, x_prev)
    (x_prev may be None)."""

    _fn = None

    @classmethod
    def apply(cls, x, mu, x_prev=None):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, x, mu, x_prev):
                    x, mu = x.contiguous(), mu.contiguous()
                    x_prev = None if x_prev is None else x_prev.contiguous()
                    ctx.save_for_backward(x, mu, x_prev)
                    return token_shift(x, mu, x_prev)

                @staticmethod
                def backward(ctx, g):
                    x, mu, x_prev = ctx.saved_tensors
                    gx, gmu, gxp = token_shift_backward(x, mu, g.contiguous(), x_prev,
                                                        want_grad_x_prev=x_prev is not None)
                    return gx, gmu, gxp

            cls._fn = _F
        return cls._fn.apply(x, mu, x_prev)


class GatedWKV:
    """torch.autograd.Function wrapper: o = GatedWKV.apply(w, u, k, v, r)."""

    _fn = None

    @classmethod
    def apply(cls, w, u, k, v, r):
        if cls._fn is None:
            torch = _torch()

            class _F(torch.autograd.Function):
                @staticmethod
                def forward(ctx, w, u, k, v, r):
                    w, u, k, v, r = (t.contiguous() for t in (w, u, k, v, r))
                    o, _, ck = forward_gated(w, u, k, v, r, want_ckpt=True)
                    ctx.save_for_backward(w, u, k, v, r, ck)
                    return o

                @staticmethod
                def backward(ctx, go):
                    w, u, k, v, r, ck = ctx.saved_tensors
                    return backward_gated(w, u, k, v, r, go.contiguous(), ckpt=ck)

            cls._fn = _F
        return cls._fn.apply(w, u, k, v, r)


def gated_wkv(w, u, k, v, r):
    """Differentiable gated WKV: sigmoid(r) * WKV(w, u, k, v)."""
    return GatedWKV.apply(w, u, k, v, r)
