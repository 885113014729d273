"""CPU oracle for the LittleBit compressed linear layer (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never does; the two share no code.

The arithmetic lives in ``littlebit_oracle.c`` (plain float64 loops in the
order the LittleBit notes give: ``x (.) g -> . V_sign -> (.) l -> . U_sign^T
-> (.) h``, paths summed).  This module compiles it with the host C compiler on
first use and marshals numpy arrays through ctypes; it does no arithmetic of
its own.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "littlebit_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_u16p = ctypes.POINTER(ctypes.c_uint16)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i8p = ctypes.POINTER(ctypes.c_int8)


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        lib.orc_half_to_double.restype = ctypes.c_double
        lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_double.restype = ctypes.c_double
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_packed_words.restype = ctypes.c_int64
        lib.orc_packed_words.argtypes = [ctypes.c_int64, ctypes.c_int]
        lib.orc_pack_signs.restype = None
        lib.orc_pack_signs.argtypes = [_f32p, ctypes.c_int64, ctypes.c_int, _u32p]
        lib.orc_unpack_signs.restype = None
        lib.orc_unpack_signs.argtypes = [_u32p, ctypes.c_int64, ctypes.c_int, _i8p]
        lib.orc_bpw.restype = ctypes.c_double
        lib.orc_bpw.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        pp = ctypes.POINTER
        common = [ctypes.c_int] * 5 + [_u16p, pp(_u32p), pp(_u32p), pp(_u16p), pp(_u16p), pp(_u16p)]
        lib.orc_forward.restype = None
        lib.orc_forward.argtypes = common + [_f64p]
        lib.orc_forward_sampled.restype = None
        lib.orc_forward_sampled.argtypes = common + [
            ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.POINTER(ctypes.c_int64), ctypes.c_int, _f64p]
        lib.orc_dense_weight.restype = None
        lib.orc_dense_weight.argtypes = [ctypes.c_int] * 4 + [pp(_u32p), pp(_u32p), pp(_u16p), pp(_u16p),
                                                               pp(_u16p), _f64p]
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def half_to_double(bits: int) -> float:
    return _load().orc_half_to_double(int(bits))


def bf16_to_double(bits: int) -> float:
    return _load().orc_bf16_to_double(int(bits))


def packed_words(rows: int, r: int) -> int:
    return int(_load().orc_packed_words(rows, r))


def pack_signs(F: np.ndarray) -> np.ndarray:
    """fp32 factor [rows, r] -> canonical packed signs [rows, ceil(r/32)] uint32."""
    F = _c(F, np.float32)
    rows, r = F.shape
    out = np.empty((rows, (r + 31) // 32), dtype=np.uint32)
    _load().orc_pack_signs(_ptr(F, ctypes.c_float), rows, r, _ptr(out, ctypes.c_uint32))
    return out


def unpack_signs(packed: np.ndarray, r: int) -> np.ndarray:
    """Canonical packed signs [rows, ceil(r/32)] -> int8 +-1 [rows, r]."""
    packed = _c(packed, np.uint32)
    rows = packed.shape[0]
    out = np.empty((rows, r), dtype=np.int8)
    _load().orc_unpack_signs(_ptr(packed, ctypes.c_uint32), rows, r, _ptr(out, ctypes.c_int8))
    return out


def bpw(N: int, K: int, r: int, npaths: int = 2) -> float:
    return float(_load().orc_bpw(N, K, r, npaths))


class _Paths:
    """ctypes pointer arrays for the per-path inputs of one layer."""

    def __init__(self, layer):
        self.keep = []
        self.npaths = len(layer["U"])

        def arr(key, dtype, ctype):
            items = [_c(a, dtype) for a in layer[key]]
            self.keep.extend(items)
            p = (ctypes.POINTER(ctype) * self.npaths)(*[_ptr(a, ctype) for a in items])
            self.keep.append(p)
            return p

        self.U = arr("U", np.uint32, ctypes.c_uint32)
        self.V = arr("V", np.uint32, ctypes.c_uint32)
        self.h = arr("h", np.uint16, ctypes.c_uint16)
        self.g = arr("g", np.uint16, ctypes.c_uint16)
        self.l = arr("l", np.uint16, ctypes.c_uint16)


def forward(x_bits: np.ndarray, layer: dict) -> np.ndarray:
    """y [M, N] float64 of one layer.

    ``layer`` holds N, K, r and per-path lists U, V (canonical packed uint32),
    h, g, l (binary16 bit patterns as uint16).  ``x_bits`` is [M, K] bfloat16
    bit patterns (uint16).
    """
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    if K != layer["K"]:
        raise ValueError("x width != K")
    P = _Paths(layer)
    y = np.empty((M, layer["N"]), dtype=np.float64)
    _load().orc_forward(M, layer["N"], K, layer["r"], P.npaths, _ptr(x, ctypes.c_uint16),
                        P.U, P.V, P.h, P.g, P.l, _ptr(y, ctypes.c_double))
    return y


def forward_sampled(x_bits: np.ndarray, layer: dict, ms, ns) -> np.ndarray:
    """y[ms][:, ns] of one layer, computed one sampled element at a time."""
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    ms = np.ascontiguousarray(ms, dtype=np.int32)
    ns = np.ascontiguousarray(ns, dtype=np.int64)
    if ms.size and (ms.min() < 0 or ms.max() >= M):
        raise ValueError("row index out of range")
    if ns.size and (ns.min() < 0 or ns.max() >= layer["N"]):
        raise ValueError("column index out of range")
    P = _Paths(layer)
    out = np.empty((ms.size, ns.size), dtype=np.float64)
    _load().orc_forward_sampled(M, layer["N"], K, layer["r"], P.npaths, _ptr(x, ctypes.c_uint16),
                                P.U, P.V, P.h, P.g, P.l,
                                ms.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), ms.size,
                                ns.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), ns.size,
                                _ptr(out, ctypes.c_double))
    return out


def dense_weight(layer: dict) -> np.ndarray:
    """The effective weight W [N, K] float64 (brute force; small layers only)."""
    P = _Paths(layer)
    W = np.empty((layer["N"], layer["K"]), dtype=np.float64)
    _load().orc_dense_weight(layer["N"], layer["K"], layer["r"], P.npaths, P.U, P.V, P.h, P.g, P.l,
                             _ptr(W, ctypes.c_double))
    return W
