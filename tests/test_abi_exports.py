"""The C-ABI library builds, loads and exports every symbol its header declares.

CPU only: no call here reaches the GPU.  Argument validation runs before any
CUDA call, so the error paths are checked on the host as well.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
HEADERS = sorted(os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE) if f.endswith(".h"))


@pytest.fixture(scope="module")
def lib():
    from sub_bit_weight_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(lb_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("lb_pack_signs", "lb_layer_create", "lb_linear_forward", "lb_layer_destroy",
                     "lb_stack_create", "lb_stack_forward", "lb_stack_destroy", "lb_layer_bpw",
                     "lb_dual_svid_workspace_bytes", "lb_dual_svid_init", "lb_littlebit2_workspace_bytes",
                     "lb_littlebit2_init"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_side_argument_checks(lib):
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    lib.lb_status_string.restype = ctypes.c_char_p
    assert lib.lb_status_string(0) == b"LB_OK"
    assert b"INVALID" in lib.lb_status_string(1)
    lib.lb_packed_words.restype = ctypes.c_size_t
    lib.lb_packed_words.argtypes = [i64, ctypes.c_int]
    assert lib.lb_packed_words(10, 33) == 20
    assert lib.lb_packed_words(-1, 3) == 0
    lib.lb_pack_signs.argtypes = [vp, i64, ctypes.c_int, vp, vp]
    assert lib.lb_pack_signs(None, -1, 4, None, None) == 1
    assert lib.lb_pack_signs(None, 3, 0, None, None) == 1
    assert lib.lb_pack_signs(None, 0, 4, None, None) == 0          # empty: nothing to do
    assert lib.lb_pack_signs(None, 5, 4, None, None) == 1
    assert lib.lb_pack_signs(vp(2), 5, 4, vp(64), None) == 1       # misaligned F
    out = vp()
    lib.lb_layer_create.argtypes = [ctypes.POINTER(vp)] + [ctypes.c_int] * 4 + [vp] * 6
    assert lib.lb_layer_create(ctypes.byref(out), 8, 8, 4, 3, None, None, None, None, None, None) == 2
    assert lib.lb_layer_create(ctypes.byref(out), 0, 8, 4, 2, None, None, None, None, None, None) == 1
    assert lib.lb_layer_create(ctypes.byref(out), 8, 8, 4096, 2, None, None, None, None, None, None) == 1
    assert lib.lb_layer_create(ctypes.byref(out), 8, 8, 4, 2, None, None, None, None, None, None) == 1
    assert lib.lb_layer_create(None, 8, 8, 4, 2, None, None, None, None, None, None) == 1
    lib.lb_linear_forward.argtypes = [vp, ctypes.c_int, vp, vp, vp]
    assert lib.lb_linear_forward(None, 1, None, None, None) == 1
    lib.lb_stack_create.argtypes = [ctypes.POINTER(vp), vp, ctypes.c_int, vp]
    assert lib.lb_stack_create(ctypes.byref(out), None, 0, None) == 1
    lib.lb_stack_forward.argtypes = [vp, vp, vp, ctypes.c_int, vp]
    assert lib.lb_stack_forward(None, None, None, 1, None) == 1
    lib.lb_layer_bpw.restype = ctypes.c_double
    lib.lb_layer_bpw.argtypes = [vp]
    assert lib.lb_layer_bpw(None) == 0.0
    lib.lb_layer_selftest_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    assert lib.lb_layer_selftest_wait_timeout(None, 10, None) == 1
    lib.lb_layer_destroy.argtypes = [vp]
    lib.lb_layer_destroy(None)
    lib.lb_stack_destroy.argtypes = [vp]
    lib.lb_stack_destroy(None)


def test_initialisation_argument_checks(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.lb_dual_svid_workspace_bytes.restype = ctypes.c_size_t
    lib.lb_dual_svid_workspace_bytes.argtypes = [i, i, i]
    assert lib.lb_dual_svid_workspace_bytes(8, 8, 9) == 0          # r above min(N, K)
    assert lib.lb_dual_svid_workspace_bytes(0, 8, 1) == 0
    ws = lib.lb_dual_svid_workspace_bytes(96, 40, 6)
    assert ws > 96 * 40 * 8
    lib.lb_dual_svid_init.argtypes = [vp, i, i, i, i, i] + [ctypes.POINTER(vp)] * 5 + [vp, vp, ctypes.c_size_t, vp]
    one = (vp * 1)(vp(256))
    args = [one] * 5
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 6, 3, 24, *args, None, vp(256), ws, None) == 2   # npaths
    assert lib.lb_dual_svid_init(None, 96, 40, 6, 1, 24, *args, None, vp(256), ws, None) == 1      # W
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 41, 1, 24, *args, None, vp(256), ws, None) == 1  # rank
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 6, 1, -1, *args, None, vp(256), ws, None) == 1   # iters
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 6, 1, 24, *args, None, vp(256), ws - 8, None) == 1   # small
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 6, 1, 24, *args, None, vp(264), ws, None) == 1   # misaligned
    nulls = (vp * 1)(None)
    assert lib.lb_dual_svid_init(vp(256), 96, 40, 6, 1, 24, nulls, *args[1:], None, vp(256), ws, None) == 1
    # LittleBit-2 (Joint-ITQ) variant: its own workspace size, the same checks plus its own arguments
    lib.lb_littlebit2_workspace_bytes.restype = ctypes.c_size_t
    lib.lb_littlebit2_workspace_bytes.argtypes = [i, i, i]
    assert lib.lb_littlebit2_workspace_bytes(8, 8, 9) == 0
    ws2 = lib.lb_littlebit2_workspace_bytes(96, 40, 6)
    assert ws2 > ws
    P = ctypes.POINTER(vp)
    lib.lb_littlebit2_init.argtypes = [vp, i, i, i, i, i, i] + [P] * 6 + [vp, vp, P, vp, ctypes.c_size_t, vp]
    call = lambda it, R0=None, loss=None, w=ws2, npaths=1: lib.lb_littlebit2_init(
        vp(256), 96, 40, 6, npaths, 24, it, R0, *args, None, loss, None, vp(256), w, None)
    assert call(-1) == 1                                         # itq_iters
    assert call(1001) == 1
    assert call(50, npaths=3) == 2
    assert call(50, w=ws) == 1                                   # the Dual-SVID workspace is too small
    assert call(50, R0=(vp * 1)(vp(260))) == 1                   # misaligned R0
    assert call(50, loss=vp(260)) == 1                           # misaligned loss


def test_backward_argument_checks(lib):
    vp, i = ctypes.c_void_p, ctypes.c_int
    P = ctypes.POINTER(vp)
    one = (vp * 1)(vp(256))
    lib.lb_backward_create.argtypes = [P, i, i, i, i] + [P] * 5 + [vp]
    out = vp()
    assert lib.lb_backward_create(None, 64, 64, 8, 1, one, one, one, one, one, None) == 1
    assert lib.lb_backward_create(ctypes.byref(out), 64, 64, 8, 3, one, one, one, one, one, None) == 2
    assert lib.lb_backward_create(ctypes.byref(out), 64, 60, 8, 1, one, one, one, one, one, None) == 2   # K % 8
    assert lib.lb_backward_create(ctypes.byref(out), 0, 64, 8, 1, one, one, one, one, one, None) == 1
    nulls = (vp * 1)(None)
    assert lib.lb_backward_create(ctypes.byref(out), 64, 64, 8, 1, nulls, one, one, one, one, None) == 1
    lib.lb_layer_backward.argtypes = [vp, vp, vp, i] + [P] * 2 + [vp] + [P] * 5 + [vp]
    assert lib.lb_layer_backward(None, vp(256), vp(256), 4, one, one, vp(256), one, one, one, one, one, None) == 1
    lib.lb_backward_destroy.argtypes = [vp]
    lib.lb_backward_destroy(None)
    from sub_bit_weight_b200 import lib as binding     # the binding declares the same argument counts
    assert len(binding._lib.lb_layer_backward.argtypes) == 13
    assert len(binding._lib.lb_backward_create.argtypes) == 11
    assert len(binding._lib.lb_dual_svid_init.argtypes) == 15
    assert len(binding._lib.lb_littlebit2_init.argtypes) == 19


def test_gemm_argument_checks(lib):
    """lb_gemm_at_b rejects bad arguments before touching the device."""
    vp, i = ctypes.c_void_p, ctypes.c_int
    f = lib.lb_gemm_at_b
    f.argtypes = [vp, i, vp, i, vp, i, i, i, i, vp, vp, vp]
    a = vp(256)
    assert f(None, 64, a, 64, a, 64, 8, 64, 64, a, a, None) == 1            # null A
    assert f(a, 64, a, 64, a, 64, 8, 64, 64, None, a, None) == 1            # null alpha
    assert f(a, 64, a, 64, a, 64, 8, 64, 64, a, None, None) == 1            # null err
    assert f(vp(264), 64, a, 64, a, 64, 8, 64, 64, a, a, None) == 1        # misaligned A
    assert f(a, 32, a, 64, a, 64, 8, 64, 64, a, a, None) == 1               # lda < Mr
    assert f(a, 68, a, 64, a, 64, 8, 64, 64, a, a, None) == 2               # lda not a multiple of 8
    assert f(a, 64, a, 48, a, 48, 8, 64, 48, a, a, None) == 2               # Nc not a multiple of 32
    assert f(a, 64, a, 64, a, 66, 8, 64, 64, a, a, None) == 2               # ldd not a multiple of 4
    assert f(a, 64, a, 64, a, 64, 0, 64, 64, a, a, None) == 2               # Kc = 0
    assert f(a, 64, a, 64, a, 64, 8, 0, 64, a, a, None) == 0                # Mr = 0: nothing to do
    assert f(a, 64, a, 64, a, 64, -1, 64, 64, a, a, None) == 1
    from sub_bit_weight_b200 import lib as binding
    assert len(binding._lib.lb_gemm_at_b.argtypes) == 12
