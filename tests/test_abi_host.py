"""Host-side checks of the C ABI (no GPU needed).

* the library loads and exports every function ``include/*.h`` declares;
* argument validation rejects bad calls with the documented code before any
  CUDA work (these calls never reach a kernel launch);
* workspace and checkpoint sizes follow the documented layout.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def W():
    from rwkv_linear_rnn_b200.build import build_library
    build_library()
    import rwkv_linear_rnn_b200
    return rwkv_linear_rnn_b200


def header_functions():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h), encoding="utf-8").read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*((?:wkv|linattn)_[a-z_]+)\s*\(", src,
                            flags=re.M)
    return names


def test_header_declares_expected(W):
    names = header_functions()
    assert sorted(names) == sorted(W.abi.EXPORTS)


def test_every_declared_symbol_is_exported(W):
    lib = ctypes.CDLL(W.library_path())
    for name in header_functions():
        assert hasattr(lib, name), name


def test_version_and_strerror(W):
    assert W.wkv_version() == 140
    for code in range(0, -6, -1):
        assert W.wkv_strerror(code) != "unknown status"
    assert W.wkv_strerror(7) == "unknown status"


def test_sizes(W):
    B, T, C = 8, 1024, 768
    assert W.wkv_ckpt_size(B, T, C) == 4 * 3 * B * C * (T // 16)  # a checkpoint every 16 tokens
    assert W.wkv_workspace_size(W.WKV_OP_STEP, B, T, C, 0) == 0
    f = W.wkv_workspace_size(W.WKV_OP_FORWARD, B, T, C, 0)
    b = W.wkv_workspace_size(W.WKV_OP_BACKWARD, B, T, C, 0)
    assert 256 < f < b
    assert b >= 256 + W.wkv_ckpt_size(B, T, C) + 4 * 2 * B * C * 16
    assert W.wkv_workspace_size(0, 0, T, C, 0) == 0     # B < 1
    assert W.wkv_workspace_size(0, B, -1, C, 0) == 0    # T < 0
    assert W.wkv_workspace_size(0, B, T, C, 3) == 0     # bad dtype
    assert W.wkv_workspace_size(9, B, T, C, 0) == 0     # bad op
    assert W.wkv_ckpt_size(1 << 40, 1 << 20, 1 << 20) == 0  # overflow


FAKE = 1 << 20  # an aligned non-null address; validation fails before any use


@pytest.mark.parametrize("args,code", [
    # (B, T, C, dtype, w, u, k, v, state_in, y, state_out, ckpt, ws, ws_bytes)
    ((1, 8, 4, 2, FAKE, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),   # bad dtype
    ((0, 8, 4, 0, FAKE, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),   # B = 0
    ((1, -1, 4, 0, FAKE, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),  # T < 0
    ((1, 8, 4, 0, 0, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),      # w NULL
    ((1, 8, 4, 0, FAKE, FAKE, 0, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),      # k NULL
    ((1, 8, 4, 0, FAKE, FAKE, FAKE, FAKE, 0, 0, 0, 0, 0, 0), -1),          # y NULL
    ((1, 8, 4, 0, FAKE + 2, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -2),  # w misaligned
    ((1, 8, 4, 1, FAKE, FAKE, FAKE + 1, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -2),  # bf16 k odd
    ((1, 8, 4, 0, FAKE, FAKE, FAKE, FAKE, 0, FAKE + 16, 0, 0, 0, 0), -2),  # y overlaps k
    ((1, 1 << 31, 4, 0, FAKE, FAKE, FAKE, FAKE, 0, FAKE * 2, 0, 0, 0, 0), -1),  # T too large
])
def test_forward_validation(W, args, code):
    assert W.abi.wkv_forward(*args, 0) == code


def test_forward_chunked_needs_workspace(W):
    opt = W.abi.Options(kernel=W.WKV_KERNEL_CHUNKED)
    base = (1, 1024, 64, 0, FAKE, FAKE, FAKE, FAKE, 0, FAKE * 4, 0, 0)
    assert W.abi.wkv_forward_ex(*base, 0, 0, 0, opt) == -3             # NULL ws
    assert W.abi.wkv_forward_ex(*base, FAKE * 8, 256, 0, opt) == -3    # too small
    assert W.abi.wkv_forward_ex(*base, FAKE * 8 + 16, 1 << 30, 0, opt) == -3  # misaligned


@pytest.mark.parametrize("kernel", [4, 5, 10, -1])
def test_retired_and_unknown_kernel_selectors_are_rejected(W, kernel):
    """Selector values 4 and 5 are retired; unknown values are rejected too,
    before anything is launched."""
    opt = W.abi.Options(kernel=kernel)
    fwd = (1, 64, 32, 0, FAKE, FAKE, FAKE, FAKE * 2, 0, FAKE * 4, 0, 0, FAKE * 8, 1 << 30, 0)
    assert W.abi.wkv_forward_ex(*fwd, opt) == -1
    bwd = (1, 64, 32, 0, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, 0, 0, FAKE * 4, FAKE * 5,
           FAKE * 6, FAKE * 7, FAKE * 8, 1 << 30, 0)
    assert W.abi.wkv_backward_ex(*bwd, opt) == -1


def test_backward_validation(W):
    a = W.abi
    # (B, T, C, dt, w, u, k, v, gy, state_in, ckpt, gw, gu, gk, gv, ws, ws_bytes, stream)
    ok = [1, 64, 32, 0, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, 0, 0, FAKE * 4, FAKE * 5,
          FAKE * 6, FAKE * 7, 0, 0, 0]
    bad = list(ok); bad[11] = 0
    assert a.wkv_backward(*bad) == -1                      # grad_w NULL
    bad = list(ok); bad[13] = FAKE                         # grad_k overlaps k
    assert a.wkv_backward(*bad) == -2
    bad = list(ok); bad[14] = FAKE * 6                     # grad_v overlaps grad_k
    assert a.wkv_backward(*bad) == -2
    assert a.wkv_backward(*ok) == -3                       # no workspace


def test_step_validation(W):
    a = W.abi
    assert a.wkv_step(0, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0) == -1
    assert a.wkv_step(1, 4, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, 0) == -1
    assert a.wkv_step(1, 4, FAKE, FAKE, FAKE, FAKE, FAKE + 1, FAKE, FAKE, 0) == -2
    # state_out partly overlapping state_in
    assert a.wkv_step(2, 4, FAKE, FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, FAKE * 4 + 16, 0) == -2


def test_get_status_null(W):
    assert W.abi.wkv_get_status(0, 0) == -3


def test_forward_gated_validation(W):
    a = W.abi
    # (B, T, C, dt, w, u, k, v, r, state_in, o, state_out, ckpt, ws, ws_bytes, stream)
    ok = [1, 8, 4, 0, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, 0, FAKE * 4, 0, 0, 0, 0, 0]
    bad = list(ok); bad[8] = 0
    assert a.wkv_forward_gated(*bad) == -1                 # r NULL
    bad = list(ok); bad[10] = 0
    assert a.wkv_forward_gated(*bad) == -1                 # o NULL
    bad = list(ok); bad[10] = FAKE * 3 + 16
    assert a.wkv_forward_gated(*bad) == -2                 # o overlaps r
    bad = list(ok); bad[10] = FAKE * 2
    assert a.wkv_forward_gated(*bad) == -2                 # o overlaps v
    bad = list(ok); bad[3] = 1; bad[8] = FAKE * 3 + 1
    assert a.wkv_forward_gated(*bad) == -2                 # bf16 r odd
    opt = a.Options(kernel=5)
    assert a.wkv_forward_gated_ex(*ok, opt) == -1          # retired selector


def test_backward_gated_validation(W):
    a = W.abi
    # (B, T, C, dt, w, u, k, v, r, go, state_in, ckpt, gw, gu, gk, gv, gr, ws, ws_bytes, stream)
    ok = [1, 64, 32, 0, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, FAKE * 4, 0, 0, FAKE * 5, FAKE * 6,
          FAKE * 7, FAKE * 8, FAKE * 9, 0, 0, 0]
    for i in (8, 9, 16):                                   # r, grad_o, grad_r NULL
        bad = list(ok); bad[i] = 0
        assert a.wkv_backward_gated(*bad) == -1, i
    for clash in (FAKE, FAKE * 3, FAKE * 4, FAKE * 7, FAKE * 8):  # grad_r on an input or output
        bad = list(ok); bad[16] = clash
        assert a.wkv_backward_gated(*bad) == -2, clash
    bad = list(ok); bad[14] = FAKE * 3                     # grad_k overlaps r
    assert a.wkv_backward_gated(*bad) == -2
    bad = list(ok); bad[16] = FAKE * 9 + 2
    assert a.wkv_backward_gated(*bad) == -2                # grad_r misaligned
    assert a.wkv_backward_gated(*ok) == -3                 # no workspace


def test_backward_state_validation(W):
    a = W.abi
    # (B, T, C, dt, w, u, k, v, gy, state_in, ckpt, state_out, gso, gw, gu, gk, gv, gsi,
    #  ws, ws_bytes, stream)
    ok = [1, 64, 32, 0, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, FAKE * 10, 0, FAKE * 11, FAKE * 12,
          FAKE * 4, FAKE * 5, FAKE * 6, FAKE * 7, FAKE * 13, 0, 0, 0]
    bad = list(ok); bad[11] = 0
    assert a.wkv_backward_state(*bad) == -1                # grad_state_out without state_out
    bad = list(ok); bad[17] = FAKE * 13 + 2
    assert a.wkv_backward_state(*bad) == -2                # grad_state_in misaligned
    for clash in (FAKE, FAKE * 10, FAKE * 11, FAKE * 12, FAKE * 6):  # on k, state_in, state_out, gso, grad_k
        bad = list(ok); bad[17] = clash
        assert a.wkv_backward_state(*bad) == -2, clash
    bad = list(ok); bad[12] = FAKE * 6                     # grad_state_out inside grad_k
    assert a.wkv_backward_state(*bad) == -2
    assert a.wkv_backward_state(*ok) == -3                 # no workspace
    opt = a.Options(kernel=4)
    assert a.wkv_backward_state_ex(*ok, opt) == -1         # retired selector


def test_token_shift_validation(W):
    a = W.abi
    # (B, T, C, dt, n, mu, x, x_prev, out, stream)
    ok = [2, 8, 16, 0, 3, FAKE, FAKE * 2, 0, FAKE * 4, 0]
    for i, val in ((4, 0), (4, 5), (5, 0), (3, 2)):          # n = 0, n = 5, NULL mu, bad dtype
        bad = list(ok); bad[i] = val
        assert a.wkv_token_shift(*bad) == -1, (i, val)
    bad = list(ok); bad[8] = FAKE * 2 + 64
    assert a.wkv_token_shift(*bad) == -2                     # out overlaps x
    bad = list(ok); bad[6] = FAKE * 2 + 2
    assert a.wkv_token_shift(*bad) == -2                     # x misaligned
    assert a.wkv_token_shift(2, 0, 16, 0, 3, FAKE, 0, 0, 0, 0) == 0  # T = 0: nothing to do
    # 2 strips of 32 tokens: one partial row per batch row (B = 2), n = 3, C = 16,
    # rounded up to 256 bytes
    assert a.wkv_token_shift_workspace_size(2, 33, 16, 3) == 512
    assert a.wkv_token_shift_workspace_size(2, 33, 16, 5) == 0
    # (B, T, C, dt, n, mu, x, x_prev, g, gx, gmu, gx_prev, ws, ws_bytes, stream)
    okb = [2, 8, 16, 0, 3, FAKE, FAKE * 2, 0, FAKE * 3, FAKE * 5, FAKE * 6, 0, FAKE * 8, 1 << 20, 0]
    bad = list(okb); bad[10] = 0
    assert a.wkv_token_shift_backward(*bad) == -1            # NULL grad_mu
    bad = list(okb); bad[9] = FAKE * 3
    assert a.wkv_token_shift_backward(*bad) == -2            # grad_x on grad_out
    bad = list(okb); bad[12] = 0
    assert a.wkv_token_shift_backward(*bad) == -3            # no workspace
    bad = list(okb); bad[13] = 64
    assert a.wkv_token_shift_backward(*bad) == -3            # workspace too small


def test_linattn_sizes_and_argument_checks(W):
    """Linear attention: workspace sizes, and calls rejected before any
    launch (unsupported head size, null or misaligned pointers, a small
    workspace, bad sizes)."""
    abi = W.abi
    f = W.linattn_workspace_size(0, 32, 3072, 32, 32)
    b = W.linattn_workspace_size(1, 32, 3072, 32, 32)
    nch = 3072 // 128
    assert f >= 256 + 32 * nch * (32 * 32 + 32) * 4
    assert b >= f + 32 * nch * (32 * 32 + 32) * 4 + 32 * 3072 * (32 * 2 + 4)
    assert W.linattn_workspace_size(0, 32, 3072, 64, 64) == 0   # head size not supported
    assert W.linattn_workspace_size(0, 0, 3072, 32, 32) == 0    # BH < 1
    assert W.linattn_workspace_size(0, 1, -1, 32, 32) == 0      # N < 0
    assert W.linattn_workspace_size(2, 1, 8, 32, 32) == 0       # bad op
    F = FAKE
    ws = 1 << 24
    big = 1 << 30
    # (BH, N, D, M, q, k, v, out, state_out, ws, ws_bytes) -> code
    cases = [
        ((1, 8, 64, 64, F, F * 2, F * 3, F * 4, 0, ws, big), -2),   # D = 64
        ((1, 8, 32, 32, 0, F * 2, F * 3, F * 4, 0, ws, big), -1),   # q NULL
        ((1, 8, 32, 32, F, F * 2, F * 3, F, 0, ws, big), -1),       # out is q
        ((0, 8, 32, 32, F, F * 2, F * 3, F * 4, 0, ws, big), -1),   # BH = 0
        ((1, 8, 32, 32, F + 2, F * 2, F * 3, F * 4, 0, ws, big), -2),  # q misaligned
        ((1, 8, 32, 32, F, F * 2, F * 3, F * 4, 0, ws, 16), -3),    # workspace too small
        ((1, 8, 32, 32, F, F * 2, F * 3, F * 4, 0, ws + 16, big), -2),  # workspace misaligned
        ((1, 8, 32, 32, F, F * 2, F * 3, F * 4, 0, 0, big), -1),    # no workspace
    ]
    for args, code in cases:
        assert abi.linattn_forward(*args, 0) == code, args
    bargs = (1, 8, 32, 32, F, F * 2, F * 3, F * 4, F * 5, F * 6, F * 7, ws, big, 0)
    assert abi.linattn_backward(*bargs[:4], 0, *bargs[5:]) == -1           # q NULL
    assert abi.linattn_backward(1, 8, 32, 32, F, F * 2, F * 3, F * 4, F, F * 6, F * 7, ws, big, 0) == -1  # grad_q is q
    assert abi.linattn_backward(1, 8, 16, 16, *bargs[4:]) == -2            # head size
    assert abi.linattn_backward(*bargs[:11], ws, 16, 0) == -3              # workspace too small


def test_linattn_backward_saved_argument_checks(W):
    abi = W.abi
    F = FAKE
    ws = 1 << 24
    big = 1 << 30
    # (BH, N, D, M, q, k, v, out, grad_out, grad_q, grad_k, grad_v, ws, ws_bytes, stream)
    ok = (1, 8, 32, 32, F, F * 2, F * 3, F * 4, F * 5, F * 6, F * 7, F * 8, ws, big, 0)
    assert abi.linattn_backward_saved(*ok[:7], 0, *ok[8:]) == -1                  # out NULL
    assert abi.linattn_backward_saved(*ok[:9], F, *ok[10:]) == -1                 # grad_q is q
    assert abi.linattn_backward_saved(1, 8, 64, 64, *ok[4:]) == -2                # head size
    assert abi.linattn_backward_saved(*ok[:12], ws, 16, 0) == -3                  # workspace too small
    assert abi.linattn_backward_saved(*ok[:4], F + 2, *ok[5:]) == -2              # q misaligned
