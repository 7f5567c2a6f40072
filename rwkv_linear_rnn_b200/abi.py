"""ctypes declarations of the libwkv C ABI (``include/wkv.h``, ``include/linattn.h``).

Each function keeps its C name and signature; pointers are passed as Python
ints (device addresses), streams as ``cudaStream_t`` ints.  Loading fails
loudly if ``libwkv.so`` has not been built.
"""
from __future__ import annotations

import ctypes
import os

# LIBWKV_PATH selects another build of the library (e.g. one compiled with
# different tile parameters); by default the in-tree build is used.
LIB_PATH = os.environ.get("LIBWKV_PATH") or os.path.join(os.path.dirname(os.path.abspath(__file__)),
                                                          "libwkv.so")

from .constants import *  # noqa: F401,F403  (codes shared with include/wkv.h)
from .constants import WKV_ERR_CUDA, WKV_OK

# Every symbol the header declares, in declaration order.
EXPORTS = (
    "wkv_workspace_size", "wkv_workspace_init", "wkv_ckpt_size", "wkv_forward", "wkv_forward_ex",
    "wkv_backward", "wkv_backward_ex", "wkv_backward_state", "wkv_backward_state_ex",
    "wkv_forward_gated", "wkv_forward_gated_ex", "wkv_backward_gated", "wkv_backward_gated_ex",
    "wkv_token_shift", "wkv_token_shift_workspace_size", "wkv_token_shift_backward",
    "wkv_step", "wkv_backward_static", "wkv_backward_static_status", "wkv_get_status",
    "wkv_strerror", "wkv_last_cuda_error", "wkv_cuda_error_name", "wkv_version",
    # include/linattn.h
    "linattn_workspace_size", "linattn_forward", "linattn_backward", "linattn_backward_saved",
)


class Options(ctypes.Structure):
    """wkv_options: kernel selector, test hook, look-back wait limit."""
    _fields_ = [("kernel", ctypes.c_int), ("test_hold_first_chunk", ctypes.c_int),
                ("spin_limit", ctypes.c_int64)]


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libwkv.so not found at {LIB_PATH}; build it with "
                      "`python -m rwkv_linear_rnn_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_i64, _int, _sz, _p = ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
_opt = ctypes.POINTER(Options)

_SIGS = {
    "wkv_workspace_size": (_sz, [_int, _i64, _i64, _i64, _int]),
    "wkv_workspace_init": (_int, [_p, _sz, _p]),
    "wkv_ckpt_size": (_sz, [_i64, _i64, _i64]),
    "wkv_forward": (_int, [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "wkv_forward_ex": (_int, [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p,
                              _opt]),
    "wkv_backward": (_int, [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                            _p, _sz, _p]),
    "wkv_backward_ex": (_int, [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                               _p, _p, _sz, _p, _opt]),
    "wkv_backward_state": (_int, [_i64, _i64, _i64, _int] + [_p] * 15 + [_sz, _p]),
    "wkv_backward_state_ex": (_int, [_i64, _i64, _i64, _int] + [_p] * 15 + [_sz, _p, _opt]),
    "wkv_forward_gated": (_int, [_i64, _i64, _i64, _int] + [_p] * 10 + [_sz, _p]),
    "wkv_forward_gated_ex": (_int, [_i64, _i64, _i64, _int] + [_p] * 10 + [_sz, _p, _opt]),
    "wkv_backward_gated": (_int, [_i64, _i64, _i64, _int] + [_p] * 14 + [_sz, _p]),
    "wkv_backward_gated_ex": (_int, [_i64, _i64, _i64, _int] + [_p] * 14 + [_sz, _p, _opt]),
    "wkv_token_shift": (_int, [_i64, _i64, _i64, _int, _int, _p, _p, _p, _p, _p]),
    "wkv_token_shift_workspace_size": (_sz, [_i64, _i64, _i64, _int]),
    "wkv_token_shift_backward": (_int, [_i64, _i64, _i64, _int, _int] + [_p] * 8 + [_sz, _p]),
    "wkv_step": (_int, [_i64, _i64, _p, _p, _p, _p, _p, _p, _p, _p]),
    "wkv_backward_static": (_int, [_i64, _i64, _i64, _int, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                   _p, _p, _p]),
    "wkv_backward_static_status": (_int, [_p]),
    "wkv_get_status": (_int, [_p, _p]),
    "wkv_strerror": (ctypes.c_char_p, [_int]),
    "wkv_last_cuda_error": (_int, []),
    "wkv_cuda_error_name": (ctypes.c_char_p, [_int]),
    "wkv_version": (_int, []),
    "linattn_workspace_size": (_sz, [_int, _i64, _i64, _int, _int]),
    "linattn_forward": (_int, [_i64, _i64, _int, _int, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "linattn_backward": (_int, [_i64, _i64, _int, _int] + [_p] * 7 + [_p, _sz, _p]),
    "linattn_backward_saved": (_int, [_i64, _i64, _int, _int] + [_p] * 8 + [_p, _sz, _p]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class WKVError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        msg = f"libwkv error {status}: {wkv_strerror(status)}"
        if status == WKV_ERR_CUDA:
            err = wkv_last_cuda_error()
            msg += f" ({wkv_cuda_error_name(err)} = {err})"
        super().__init__(msg)


def _opts(o):
    return None if o is None else ctypes.byref(o)


def wkv_workspace_size(op, B, T, C, dtype):
    return lib.wkv_workspace_size(op, B, T, C, dtype)


def wkv_workspace_init(ws, ws_bytes, stream):
    return lib.wkv_workspace_init(ws, ws_bytes, stream)


def wkv_ckpt_size(B, T, C):
    return lib.wkv_ckpt_size(B, T, C)


def wkv_forward(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes, stream):
    return lib.wkv_forward(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes,
                           stream)


def wkv_forward_ex(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes, stream,
                   opt=None):
    return lib.wkv_forward_ex(B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws,
                              ws_bytes, stream, _opts(opt))


def wkv_backward(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k,
                 grad_v, ws, ws_bytes, stream):
    return lib.wkv_backward(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                            grad_k, grad_v, ws, ws_bytes, stream)


def wkv_backward_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u, grad_k,
                    grad_v, ws, ws_bytes, stream, opt=None):
    return lib.wkv_backward_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                               grad_k, grad_v, ws, ws_bytes, stream, _opts(opt))


def wkv_backward_state(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, state_out,
                       grad_state_out, grad_w, grad_u, grad_k, grad_v, grad_state_in, ws, ws_bytes,
                       stream):
    return lib.wkv_backward_state(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, state_out,
                                  grad_state_out, grad_w, grad_u, grad_k, grad_v, grad_state_in, ws,
                                  ws_bytes, stream)


def wkv_backward_state_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, state_out,
                          grad_state_out, grad_w, grad_u, grad_k, grad_v, grad_state_in, ws,
                          ws_bytes, stream, opt=None):
    return lib.wkv_backward_state_ex(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt,
                                     state_out, grad_state_out, grad_w, grad_u, grad_k, grad_v,
                                     grad_state_in, ws, ws_bytes, stream, _opts(opt))


def wkv_forward_gated(B, T, C, dtype, w, u, k, v, r, state_in, o, state_out, ckpt, ws, ws_bytes,
                      stream):
    return lib.wkv_forward_gated(B, T, C, dtype, w, u, k, v, r, state_in, o, state_out, ckpt, ws,
                                 ws_bytes, stream)


def wkv_forward_gated_ex(B, T, C, dtype, w, u, k, v, r, state_in, o, state_out, ckpt, ws,
                         ws_bytes, stream, opt=None):
    return lib.wkv_forward_gated_ex(B, T, C, dtype, w, u, k, v, r, state_in, o, state_out, ckpt,
                                    ws, ws_bytes, stream, _opts(opt))


def wkv_backward_gated(B, T, C, dtype, w, u, k, v, r, grad_o, state_in, ckpt, grad_w, grad_u,
                       grad_k, grad_v, grad_r, ws, ws_bytes, stream):
    return lib.wkv_backward_gated(B, T, C, dtype, w, u, k, v, r, grad_o, state_in, ckpt, grad_w,
                                  grad_u, grad_k, grad_v, grad_r, ws, ws_bytes, stream)


def wkv_backward_gated_ex(B, T, C, dtype, w, u, k, v, r, grad_o, state_in, ckpt, grad_w, grad_u,
                          grad_k, grad_v, grad_r, ws, ws_bytes, stream, opt=None):
    return lib.wkv_backward_gated_ex(B, T, C, dtype, w, u, k, v, r, grad_o, state_in, ckpt,
                                     grad_w, grad_u, grad_k, grad_v, grad_r, ws, ws_bytes, stream,
                                     _opts(opt))


def wkv_token_shift(B, T, C, dtype, n, mu, x, x_prev, out, stream):
    return lib.wkv_token_shift(B, T, C, dtype, n, mu, x, x_prev, out, stream)


def wkv_token_shift_workspace_size(B, T, C, n):
    return lib.wkv_token_shift_workspace_size(B, T, C, n)


def wkv_token_shift_backward(B, T, C, dtype, n, mu, x, x_prev, grad_out, grad_x, grad_mu,
                             grad_x_prev, ws, ws_bytes, stream):
    return lib.wkv_token_shift_backward(B, T, C, dtype, n, mu, x, x_prev, grad_out, grad_x,
                                        grad_mu, grad_x_prev, ws, ws_bytes, stream)


def wkv_step(N, C, w, u, k_t, v_t, state_in, y_t, state_out, stream):
    return lib.wkv_step(N, C, w, u, k_t, v_t, state_in, y_t, state_out, stream)


def wkv_backward_static(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w, grad_u,
                        grad_k, grad_v, stream):
    return lib.wkv_backward_static(B, T, C, dtype, w, u, k, v, grad_y, state_in, ckpt, grad_w,
                                   grad_u, grad_k, grad_v, stream)


def wkv_backward_static_status(stream):
    return lib.wkv_backward_static_status(stream)


def wkv_get_status(ws, stream):
    return lib.wkv_get_status(ws, stream)


def wkv_strerror(status):
    return lib.wkv_strerror(status).decode()


def wkv_last_cuda_error():
    return lib.wkv_last_cuda_error()


def wkv_cuda_error_name(err):
    return lib.wkv_cuda_error_name(err).decode()


def wkv_version():
    return lib.wkv_version()


def linattn_workspace_size(op, BH, N, D, M):
    return lib.linattn_workspace_size(op, BH, N, D, M)


def linattn_forward(BH, N, D, M, q, k, v, out, state_out, ws, ws_bytes, stream):
    return lib.linattn_forward(BH, N, D, M, q, k, v, out, state_out, ws, ws_bytes, stream)


def linattn_backward(BH, N, D, M, q, k, v, grad_out, grad_q, grad_k, grad_v, ws, ws_bytes, stream):
    return lib.linattn_backward(BH, N, D, M, q, k, v, grad_out, grad_q, grad_k, grad_v, ws, ws_bytes,
                                stream)


def linattn_backward_saved(BH, N, D, M, q, k, v, out, grad_out, grad_q, grad_k, grad_v, ws, ws_bytes, stream):
    return lib.linattn_backward_saved(BH, N, D, M, q, k, v, out, grad_out, grad_q, grad_k, grad_v, ws, ws_bytes,
                                      stream)


def check(rc: int) -> None:
    if rc != WKV_OK:
        raise WKVError(rc)
