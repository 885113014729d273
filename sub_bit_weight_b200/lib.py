"""Thin Python binding of the C ABI in ``include/littlebit.h``.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of ``liblittlebit.so``.  PyTorch supplies device memory and streams.
Importing this module loads the library and raises ImportError when it has not
been built (``python -m sub_bit_weight_b200.build``); there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblittlebit.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sub_bit_weight_b200.build`")

_lib = ctypes.CDLL(LIB_PATH)

LB_OK, LB_ERR_INVALID_ARG, LB_ERR_UNSUPPORTED, LB_ERR_OOM, LB_ERR_CUDA, LB_ERR_TIMEOUT = range(6)
LB_DECODE_MAX_M = 16
LB_MAX_RANK = 2048
LB_STACK_MAX_LAYERS = 4096

_vp = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_st = ctypes.c_int


def _sig(name, res, args):
    f = getattr(_lib, name)
    f.restype = res
    f.argtypes = args
    return f


_sig("lb_status_string", ctypes.c_char_p, [_st])
_sig("lb_packed_words", ctypes.c_size_t, [_i64, _i])
_sig("lb_pack_signs", _st, [_vp, _i64, _i, _vp, _vp])
_sig("lb_layer_create", _st, [ctypes.POINTER(_vp), _i, _i, _i, _i] + [ctypes.POINTER(_vp)] * 5 + [_vp])
_sig("lb_layer_destroy", None, [_vp])
_sig("lb_layer_shape", _st, [_vp] + [ctypes.POINTER(_i)] * 4)
_sig("lb_layer_bpw", ctypes.c_double, [_vp])
_sig("lb_layer_device_bytes", ctypes.c_size_t, [_vp])
_sig("lb_linear_forward", _st, [_vp, _i, _vp, _vp, _vp])
_sig("lb_linear_forward_noalloc", _st, [_vp, _i, _vp, _vp, _vp])
_sig("lb_stack_create", _st, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp])
_sig("lb_stack_destroy", None, [_vp])
_sig("lb_stack_forward", _st, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(_vp), _i, _vp])
_sig("lb_last_launch_count", _i, [])
_sig("lb_profile_events", _st, [ctypes.POINTER(_vp), _i])
_sig("lb_stack_status", _st, [_vp, _vp])
_sig("lb_layer_status", _st, [_vp, _vp])
_sig("lb_selftest_wait_timeout", _st, [ctypes.c_longlong, _vp])
_sig("lb_layer_selftest_wait_timeout", _st, [_vp, ctypes.c_longlong, _vp])
_sig("lb_dual_svid_workspace_bytes", ctypes.c_size_t, [_i, _i, _i])
_sig("lb_backward_create", _st, [ctypes.POINTER(_vp), _i, _i, _i, _i] + [ctypes.POINTER(_vp)] * 5 + [_vp])
_sig("lb_backward_destroy", None, [_vp])
_sig("lb_layer_backward", _st, [_vp, _vp, _vp, _i] + [ctypes.POINTER(_vp)] * 2 + [_vp] + [ctypes.POINTER(_vp)] * 5 + [_vp])
_sig("lb_backward_status", _st, [_vp, _vp])
_sig("lb_gemm_at_b", _st, [_vp, _i, _vp, _i, _vp, _i, _i, _i, _i, _vp, _vp, _vp])
_sig("lb_dual_svid_init", _st, [_vp, _i, _i, _i, _i, _i] + [ctypes.POINTER(_vp)] * 5 + [_vp, _vp, ctypes.c_size_t, _vp])
_sig("lb_littlebit2_workspace_bytes", ctypes.c_size_t, [_i, _i, _i])
_sig("lb_littlebit2_init", _st, [_vp, _i, _i, _i, _i, _i, _i] + [ctypes.POINTER(_vp)] * 6 +
     [_vp, _vp, ctypes.POINTER(_vp), _vp, ctypes.c_size_t, _vp])


class LittleBitError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {lb_status_string(status)}")


def lb_status_string(status: int) -> str:
    return _lib.lb_status_string(status).decode()


def _check(status: int, where: str):
    if status != LB_OK:
        raise LittleBitError(status, where)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def lb_layer_status(layer, stream=None) -> int:
    """Synchronise and return (and clear) the layer's device-side status: LB_OK or LB_ERR_TIMEOUT."""
    return int(_lib.lb_layer_status(layer.handle, _stream(stream)))


def lb_stack_status(stack, stream=None) -> int:
    return int(_lib.lb_stack_status(stack.handle, _stream(stream)))


def lb_selftest_wait_timeout(cycles: int, stream=None) -> int:
    return int(_lib.lb_selftest_wait_timeout(int(cycles), _stream(stream)))


def lb_layer_selftest_wait_timeout(layer, cycles: int, stream=None) -> int:
    """Run the bounded-wait self-test against the layer's error slot (no synchronisation)."""
    return int(_lib.lb_layer_selftest_wait_timeout(layer.handle, int(cycles), _stream(stream)))


def lb_packed_words(rows: int, r: int) -> int:
    return int(_lib.lb_packed_words(rows, r))


def lb_last_launch_count() -> int:
    return int(_lib.lb_last_launch_count())


def lb_profile_events(events) -> None:
    """Register torch.cuda.Event objects (timing enabled) for the next forward calls; [] clears."""
    n = len(events)
    arr = (_vp * max(1, n))(*[e.cuda_event for e in events]) if n else None
    _check(_lib.lb_profile_events(arr, n), "lb_profile_events")


def lb_pack_signs(F: torch.Tensor, packed: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """fp32 factor [rows, r] (CUDA) -> canonical packed signs, int32 [rows, ceil(r/32)] (bit patterns)."""
    if F.dim() != 2:
        raise ValueError("F must be 2-D [rows, r]")
    rows, r = F.shape
    if packed is None:
        packed = torch.empty((rows, (r + 31) // 32), dtype=torch.int32, device=F.device)
    else:
        _numel(packed, rows * ((r + 31) // 32), "packed")
    _check(_lib.lb_pack_signs(_dev(F, torch.float32, "F"), rows, r, _dev(packed, torch.int32, "packed"),
                              _stream(stream)), "lb_pack_signs")
    return packed


def _u16(t: torch.Tensor, name: str) -> int:
    # binary16 values, or their bit patterns; bfloat16 is refused since its bits read as binary16 are other numbers
    if t.dtype in (torch.float16, torch.int16, torch.uint16):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
        return t.data_ptr()
    raise TypeError(f"{name} must be binary16 (float16, or its bit patterns as int16/uint16), got {t.dtype}")


def _numel(t, n: int, name: str):
    """The library takes bare pointers: a tensor shorter than the layout it stands for would be read or
    written past its end on the device, so every size is checked here, before any call."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.numel() != n:
        raise ValueError(f"{name} must hold {n} elements, got {t.numel()} (shape {tuple(t.shape)})")


def _layer_arrays(N: int, K: int, r: int, U, V, h, g, l):
    """Per-path pointer arrays of lb_layer_create / lb_backward_create: U[p] [N, ceil(r/32)] and
    V[p] [K, ceil(r/32)] int32, h[p] [N], g[p] [K], l[p] [r] binary16, each size checked (invalid shapes
    themselves are left to the library, which rejects them)."""
    npaths = len(U)
    wpr = (r + 31) // 32
    sizes = {"U": N * wpr, "V": K * wpr, "h": N, "g": K, "l": r}
    lists = (("U", U), ("V", V), ("h", h), ("g", g), ("l", l))
    for name, lst in lists:
        if len(lst) != npaths:
            raise ValueError(f"{name} must have one entry per path")
        if min(N, K, r) > 0:
            for p, t in enumerate(lst):
                _numel(t, sizes[name], f"{name}[{p}]")
    arrs = []
    for name, lst in lists:
        ptrs = [_dev(t, torch.int32, f"{name}[{p}]") if name in ("U", "V") else _u16(t, f"{name}[{p}]")
                for p, t in enumerate(lst)]
        arrs.append((_vp * max(1, npaths))(*ptrs))
    return npaths, arrs


class Layer:
    """Owns an ``lb_layer`` handle (see ``lb_layer_create``)."""

    def __init__(self, handle: int, N: int, K: int, r: int, npaths: int):
        self.handle = handle
        self.N, self.K, self.r, self.npaths = N, K, r, npaths

    @property
    def bpw(self) -> float:
        return float(_lib.lb_layer_bpw(self.handle))

    @property
    def device_bytes(self) -> int:
        return int(_lib.lb_layer_device_bytes(self.handle))

    def close(self):
        if self.handle:
            _lib.lb_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lb_layer_create(N: int, K: int, r: int, U, V, h, g, l, stream=None) -> Layer:
    """Per-path lists: U[p] int32 [N, ceil(r/32)], V[p] int32 [K, ceil(r/32)] (canonical packed),
    h[p] [N], g[p] [K], l[p] [r] binary16 (float16 or int16/uint16 bit patterns), all CUDA."""
    npaths, arrs = _layer_arrays(N, K, r, U, V, h, g, l)
    out = _vp()
    _check(_lib.lb_layer_create(ctypes.byref(out), N, K, r, npaths, *arrs, _stream(stream)), "lb_layer_create")
    return Layer(out.value, N, K, r, npaths)


def lb_linear_forward(x: torch.Tensor, layer: Layer, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y[M, N] float32 = x[M, K] (bfloat16) . W_hat^T."""
    if x.dim() != 2 or x.shape[1] != layer.K:
        raise ValueError(f"x must be [M, {layer.K}]")
    M = x.shape[0]
    if y is None:
        y = torch.empty((M, layer.N), dtype=torch.float32, device=x.device)
    elif tuple(y.shape) != (M, layer.N):
        raise ValueError(f"y must be [{M}, {layer.N}]")
    _check(_lib.lb_linear_forward(_dev(x, torch.bfloat16, "x") if M else None, M, layer.handle,
                                  _dev(y, torch.float32, "y") if M else None, _stream(stream)),
           "lb_linear_forward")
    return y


def lb_linear_forward_noalloc(x: torch.Tensor, layer: Layer, y: torch.Tensor, stream=None) -> torch.Tensor:
    """Same result as lb_linear_forward for M <= 16, without allocating: scratch is a static
    device array inside the library and ``y`` must be supplied (see the C header)."""
    if x.dim() != 2 or x.shape[1] != layer.K:
        raise ValueError(f"x must be [M, {layer.K}]")
    M = x.shape[0]
    if tuple(y.shape) != (M, layer.N):
        raise ValueError(f"y must be [{M}, {layer.N}]")
    _check(_lib.lb_linear_forward_noalloc(_dev(x, torch.bfloat16, "x") if M else None, M, layer.handle,
                                          _dev(y, torch.float32, "y") if M else None, _stream(stream)),
           "lb_linear_forward_noalloc")
    return y


class Stack:
    """Owns an ``lb_stack`` handle; keeps its layers alive."""

    def __init__(self, handle: int, layers):
        self.handle = handle
        self.layers = list(layers)

    def close(self):
        if self.handle:
            _lib.lb_stack_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lb_stack_create(layers, stream=None) -> Stack:
    arr = (_vp * len(layers))(*[L.handle for L in layers])
    out = _vp()
    _check(_lib.lb_stack_create(ctypes.byref(out), arr, len(layers), _stream(stream)), "lb_stack_create")
    return Stack(out.value, layers)


class StackIO:
    """Pointer tables of a stack call, marshalled once and reused."""

    def __init__(self, stack: Stack, xs, ys):
        if len(xs) != len(stack.layers) or len(ys) != len(stack.layers):
            raise ValueError("one x and one y per layer")
        M = xs[0].shape[0]
        for L, x, y in zip(stack.layers, xs, ys):
            if tuple(x.shape) != (M, L.K) or tuple(y.shape) != (M, L.N):
                raise ValueError("x/y shapes do not match the layers")
        self.M = M
        self.xs, self.ys = list(xs), list(ys)
        self.xp = (_vp * len(xs))(*[_dev(x, torch.bfloat16, "x") for x in xs])
        self.yp = (_vp * len(ys))(*[_dev(y, torch.float32, "y") for y in ys])


def lb_stack_forward(stack: Stack, xs=None, ys=None, stream=None, io: StackIO | None = None) -> StackIO:
    """Run every layer i: ys[i] = xs[i] . W_hat_i^T.  Pass ``io`` to reuse marshalled pointer tables."""
    if io is None:
        io = StackIO(stack, xs, ys)
    _check(_lib.lb_stack_forward(stack.handle, io.xp, io.yp, io.M, _stream(stream)), "lb_stack_forward")
    return io


# ---------------------------------------------------------------------------
# Initialisation: Dual-SVID + residual compensation (include/littlebit_init.h)
# ---------------------------------------------------------------------------

def lb_dual_svid_workspace_bytes(N: int, K: int, r: int) -> int:
    return int(_lib.lb_dual_svid_workspace_bytes(N, K, r))


class DualSvidResult:
    """Per-path outputs of ``lb_dual_svid_init``: packed signs (int32 bit patterns) and float32 scales."""

    def __init__(self, U, V, h, g, l, sigma):
        self.U, self.V, self.h, self.g, self.l, self.sigma = U, V, h, g, l, sigma

    def layer_args(self):
        """(U, V, h, g, l) lists for lb_layer_create, the scales rounded to binary16."""
        return self.U, self.V, [x.half() for x in self.h], [x.half() for x in self.g], [x.half() for x in self.l]


def lb_dual_svid_init(W: torch.Tensor, r: int, npaths: int = 2, iters: int = 24, workspace: torch.Tensor | None = None,
                      stream=None) -> DualSvidResult:
    """Dual-SVID (+ residual) initialisation of a LittleBit layer from a dense float32 W [N, K] (CUDA).

    Allocates the outputs (and the workspace unless one is passed: a uint8 CUDA tensor of at least
    ``lb_dual_svid_workspace_bytes(N, K, r)`` bytes).  The call waits for its stream.
    """
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    need = lb_dual_svid_workspace_bytes(N, K, r)
    if need == 0:
        raise ValueError(f"invalid shape N={N} K={K} r={r}")
    dev = W.device
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wpr = (r + 31) // 32
    U = [torch.empty((N, wpr), dtype=torch.int32, device=dev) for _ in range(npaths)]
    V = [torch.empty((K, wpr), dtype=torch.int32, device=dev) for _ in range(npaths)]
    h = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(npaths)]
    g = [torch.empty(K, dtype=torch.float32, device=dev) for _ in range(npaths)]
    l = [torch.empty(r, dtype=torch.float32, device=dev) for _ in range(npaths)]
    sigma = torch.empty((npaths, r), dtype=torch.float32, device=dev)

    def arr(lst, dtype, name):
        return (_vp * max(1, len(lst)))(*[_dev(t, dtype, f"{name}[{p}]") for p, t in enumerate(lst)])

    _check(_lib.lb_dual_svid_init(_dev(W, torch.float32, "W"), N, K, r, npaths, iters,
                                  arr(U, torch.int32, "U"), arr(V, torch.int32, "V"), arr(h, torch.float32, "h"),
                                  arr(g, torch.float32, "g"), arr(l, torch.float32, "l"),
                                  _dev(sigma, torch.float32, "sigma"), _dev(workspace, torch.uint8, "workspace"),
                                  workspace.numel(), _stream(stream)), "lb_dual_svid_init")
    return DualSvidResult(U, V, h, g, l, sigma)


def lb_littlebit2_workspace_bytes(N: int, K: int, r: int) -> int:
    return int(_lib.lb_littlebit2_workspace_bytes(N, K, r))


class LittleBit2Result(DualSvidResult):
    """Outputs of ``lb_littlebit2_init``: those of Dual-SVID plus the ITQ loss [npaths, itq_iters + 1] and R."""

    def __init__(self, U, V, h, g, l, sigma, itq_loss, R):
        super().__init__(U, V, h, g, l, sigma)
        self.itq_loss, self.R = itq_loss, R


def lb_littlebit2_init(W: torch.Tensor, r: int, npaths: int = 2, iters: int = 24, itq_iters: int = 50,
                       R0: list | None = None, workspace: torch.Tensor | None = None, stream=None) -> LittleBit2Result:
    """LittleBit-2 initialisation (Joint-ITQ latent rotation, then Dual-SVID + residual) of a dense float32 W (CUDA).

    ``R0``: None (identity starts) or a list of npaths float64 CUDA [r, r] orthogonal matrices (or None entries).
    Allocates the outputs (and the workspace unless one is passed).  The call waits for its stream.
    """
    if W.dim() != 2:
        raise ValueError("W must be 2-D [N, K]")
    N, K = W.shape
    need = lb_littlebit2_workspace_bytes(N, K, r)
    if need == 0:
        raise ValueError(f"invalid shape N={N} K={K} r={r}")
    dev = W.device
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    wpr = (r + 31) // 32
    U = [torch.empty((N, wpr), dtype=torch.int32, device=dev) for _ in range(npaths)]
    V = [torch.empty((K, wpr), dtype=torch.int32, device=dev) for _ in range(npaths)]
    h = [torch.empty(N, dtype=torch.float32, device=dev) for _ in range(npaths)]
    g = [torch.empty(K, dtype=torch.float32, device=dev) for _ in range(npaths)]
    l = [torch.empty(r, dtype=torch.float32, device=dev) for _ in range(npaths)]
    sigma = torch.empty((npaths, r), dtype=torch.float32, device=dev)
    loss = torch.empty((npaths, itq_iters + 1), dtype=torch.float64, device=dev)
    R = [torch.empty((r, r), dtype=torch.float64, device=dev) for _ in range(npaths)]

    def arr(lst, dtype, name):
        return (_vp * max(1, len(lst)))(*[None if t is None else _dev(t, dtype, f"{name}[{p}]")
                                          for p, t in enumerate(lst)])

    r0 = None
    if R0 is not None:
        if len(R0) != npaths or any(t is not None and tuple(t.shape) != (r, r) for t in R0):
            raise ValueError("R0 must hold npaths [r, r] matrices (or None entries)")
        r0 = arr(list(R0), torch.float64, "R0")
    _check(_lib.lb_littlebit2_init(_dev(W, torch.float32, "W"), N, K, r, npaths, iters, itq_iters, r0,
                                   arr(U, torch.int32, "U"), arr(V, torch.int32, "V"), arr(h, torch.float32, "h"),
                                   arr(g, torch.float32, "g"), arr(l, torch.float32, "l"),
                                   _dev(sigma, torch.float32, "sigma"), _dev(loss, torch.float64, "itq_loss"),
                                   arr(R, torch.float64, "R"), _dev(workspace, torch.uint8, "workspace"),
                                   workspace.numel(), _stream(stream)), "lb_littlebit2_init")
    return LittleBit2Result(U, V, h, g, l, sigma, loss, R)


# ---------------------------------------------------------------------------
# QAT backward (include/littlebit_backward.h)
# ---------------------------------------------------------------------------

class Backward:
    """Owns an ``lb_backward`` handle (see ``lb_backward_create``)."""

    def __init__(self, handle: int, N: int, K: int, r: int, npaths: int):
        self.handle = handle
        self.N, self.K, self.r, self.npaths = N, K, r, npaths

    def close(self):
        if self.handle:
            _lib.lb_backward_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lb_backward_create(N: int, K: int, r: int, U, V, h, g, l, stream=None) -> Backward:
    """Per-path lists as lb_layer_create: canonical packed U, V (int32) and binary16 h, g, l (CUDA)."""
    npaths, arrs = _layer_arrays(N, K, r, U, V, h, g, l)
    out = _vp()
    _check(_lib.lb_backward_create(ctypes.byref(out), N, K, r, npaths, *arrs, _stream(stream)), "lb_backward_create")
    return Backward(out.value, N, K, r, npaths)


def lb_layer_backward(B: Backward, x: torch.Tensor, dy: torch.Tensor, U_lat, V_lat, stream=None) -> dict:
    """Gradients for x [M, K] (bfloat16) and dy [M, N] (float32): dx [M, K] and per-path lists dh, dg, dl, dU, dV."""
    if x.dim() != 2 or x.shape[1] != B.K or tuple(dy.shape) != (x.shape[0], B.N):
        raise ValueError(f"x must be [M, {B.K}] and dy [M, {B.N}]")
    M = x.shape[0]
    for name, lst, rows in (("U_lat", U_lat, B.N), ("V_lat", V_lat, B.K)):
        if len(lst) != B.npaths:
            raise ValueError(f"{name} must have one entry per path")
        for p, t in enumerate(lst):
            _numel(t, rows * B.r, f"{name}[{p}]")
    dev = x.device
    P = B.npaths
    out = {"dx": torch.empty((M, B.K), dtype=torch.float32, device=dev),
           "dh": [torch.empty(B.N, dtype=torch.float32, device=dev) for _ in range(P)],
           "dg": [torch.empty(B.K, dtype=torch.float32, device=dev) for _ in range(P)],
           "dl": [torch.empty(B.r, dtype=torch.float32, device=dev) for _ in range(P)],
           "dU": [torch.empty((B.N, B.r), dtype=torch.float32, device=dev) for _ in range(P)],
           "dV": [torch.empty((B.K, B.r), dtype=torch.float32, device=dev) for _ in range(P)]}

    def arr(lst, name):
        return (_vp * max(1, len(lst)))(*[_dev(t, torch.float32, f"{name}[{p}]") for p, t in enumerate(lst)])

    _check(_lib.lb_layer_backward(B.handle, _dev(x, torch.bfloat16, "x"), _dev(dy, torch.float32, "dy"), M,
                                  arr(U_lat, "U_lat"), arr(V_lat, "V_lat"), _dev(out["dx"], torch.float32, "dx"),
                                  arr(out["dh"], "dh"), arr(out["dg"], "dg"), arr(out["dl"], "dl"),
                                  arr(out["dU"], "dU"), arr(out["dV"], "dV"), _stream(stream)), "lb_layer_backward")
    return out


def lb_backward_status(B: Backward, stream=None) -> int:
    return int(_lib.lb_backward_status(B.handle, _stream(stream)))


def lb_gemm_at_b(A: torch.Tensor, B: torch.Tensor, alpha: torch.Tensor, err: torch.Tensor, stream=None) -> torch.Tensor:
    """D = alpha * A^T B for A [Kc, Mr] and B [Kc, Nc] (float16, contiguous), alpha a one-element float32 CUDA tensor
    and err a one-element int32 CUDA tensor (the kernel's bounded waits report there).  Returns D [Mr, Nc] float32."""
    if A.dim() != 2 or B.dim() != 2 or A.shape[0] != B.shape[0]:
        raise ValueError("A must be [Kc, Mr] and B [Kc, Nc]")
    _numel(alpha, 1, "alpha")
    _numel(err, 1, "err")
    Kc, Mr = A.shape
    Nc = B.shape[1]
    D = torch.empty((Mr, Nc), dtype=torch.float32, device=A.device)
    _check(_lib.lb_gemm_at_b(_dev(A, torch.float16, "A"), Mr, _dev(B, torch.float16, "B"), Nc,
                             _dev(D, torch.float32, "D"), Nc, Kc, Mr, Nc, _dev(alpha, torch.float32, "alpha"),
                             _dev(err, torch.int32, "err"), _stream(stream)), "lb_gemm_at_b")
    return D
