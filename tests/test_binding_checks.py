"""The Python binding refuses, before any library call, tensors the C ABI would misread.

The C entry points take bare pointers, so they cannot see a buffer's length or
element type.  A per-path tensor shorter than the layout it stands for would be
read (or, for ``packed``, written) past its end on the device, and bfloat16
scales would be read as binary16 bit patterns, i.e. as other numbers.  These
checks run on the host, so CPU tensors exercise them: a wrong size must give
ValueError naming the tensor, and a correctly sized CPU tensor must get past
the size check and stop at the device check (TypeError / ValueError about
CUDA), never at the library.
"""

import pytest
import torch


@pytest.fixture(scope="module")
def lib():
    from sub_bit_weight_b200 import build
    build.build()
    from sub_bit_weight_b200 import lib as binding
    return binding


def _layer_tensors(N, K, r, npaths=2, scale_dtype=torch.float16):
    wpr = (r + 31) // 32
    U = [torch.zeros((N, wpr), dtype=torch.int32) for _ in range(npaths)]
    V = [torch.zeros((K, wpr), dtype=torch.int32) for _ in range(npaths)]
    h = [torch.zeros(N, dtype=scale_dtype) for _ in range(npaths)]
    g = [torch.zeros(K, dtype=scale_dtype) for _ in range(npaths)]
    l = [torch.zeros(r, dtype=scale_dtype) for _ in range(npaths)]
    return {"U": U, "V": V, "h": h, "g": g, "l": l}


@pytest.mark.parametrize("create", ["lb_layer_create", "lb_backward_create"])
@pytest.mark.parametrize("name,p,bad", [
    ("U", 0, lambda N, K, r: torch.zeros((N - 1, (r + 31) // 32), dtype=torch.int32)),
    ("V", 1, lambda N, K, r: torch.zeros((K, (r + 31) // 32 - 1), dtype=torch.int32)),
    ("h", 1, lambda N, K, r: torch.zeros(N - 1, dtype=torch.float16)),
    ("g", 0, lambda N, K, r: torch.zeros(K + 1, dtype=torch.float16)),
    ("l", 1, lambda N, K, r: torch.zeros(r - 1, dtype=torch.float16)),
])
def test_wrong_sized_layer_inputs_are_refused(lib, create, name, p, bad):
    N, K, r = 40, 72, 40                    # two sign words per row: a dropped word changes the size
    t = _layer_tensors(N, K, r)
    t[name][p] = bad(N, K, r)
    with pytest.raises(ValueError, match=rf"{name}\[{p}\] must hold"):
        getattr(lib, create)(N, K, r, t["U"], t["V"], t["h"], t["g"], t["l"])


@pytest.mark.parametrize("create", ["lb_layer_create", "lb_backward_create"])
def test_correctly_sized_inputs_pass_the_size_check(lib, create):
    # 2-D or 1-D views of the right length are accepted; the CPU tensor then fails the device check
    N, K, r = 40, 72, 40
    t = _layer_tensors(N, K, r)
    t["U"][1] = t["U"][1].reshape(-1)
    with pytest.raises(TypeError, match="CUDA"):
        getattr(lib, create)(N, K, r, t["U"], t["V"], t["h"], t["g"], t["l"])


def test_scale_lists_must_match_the_path_count(lib):
    t = _layer_tensors(16, 16, 8)
    with pytest.raises(ValueError, match="one entry per path"):
        lib.lb_layer_create(16, 16, 8, t["U"], t["V"], t["h"][:1], t["g"], t["l"])


def test_bfloat16_scales_are_refused(lib):
    # the library reads the scales as binary16; the dtype is checked before the device
    for dt in (torch.bfloat16, torch.float32, torch.int32):
        with pytest.raises(TypeError, match="binary16"):
            lib._u16(torch.zeros(4, dtype=dt), "h[0]")
    for dt in (torch.float16, torch.int16, torch.uint16):     # accepted dtypes stop at the device check
        with pytest.raises(ValueError, match="CUDA"):
            lib._u16(torch.zeros(4, dtype=dt), "h[0]")


def test_pack_signs_checks_a_supplied_output(lib):
    F = torch.zeros((5, 40))
    with pytest.raises(ValueError, match="packed must hold 10"):
        lib.lb_pack_signs(F, torch.zeros((5, 1), dtype=torch.int32))
    with pytest.raises(TypeError, match="CUDA"):                # right size: stops at the device check
        lib.lb_pack_signs(F, torch.zeros((5, 2), dtype=torch.int32))


def test_backward_checks_latent_factors_and_shapes(lib):
    N, K, r = 48, 64, 24
    B = lib.Backward(None, N, K, r, 2)       # no handle: every case below is refused before the library
    x = torch.zeros((3, K), dtype=torch.bfloat16)
    dy = torch.zeros((3, N))
    U_lat = [torch.zeros((N, r)) for _ in range(2)]
    V_lat = [torch.zeros((K, r)) for _ in range(2)]
    with pytest.raises(ValueError, match="x must be"):
        lib.lb_layer_backward(B, x[:, :-1], dy, U_lat, V_lat)
    with pytest.raises(ValueError, match="x must be"):
        lib.lb_layer_backward(B, x, dy[:2], U_lat, V_lat)
    with pytest.raises(ValueError, match="x must be"):
        lib.lb_layer_backward(B, x.reshape(-1), dy, U_lat, V_lat)
    with pytest.raises(ValueError, match="one entry per path"):
        lib.lb_layer_backward(B, x, dy, U_lat[:1], V_lat)
    with pytest.raises(ValueError, match=r"U_lat\[1\] must hold"):
        lib.lb_layer_backward(B, x, dy, [U_lat[0], torch.zeros((N, r - 1))], V_lat)
    with pytest.raises(ValueError, match=r"V_lat\[0\] must hold"):
        lib.lb_layer_backward(B, x, dy, U_lat, [torch.zeros((K - 1, r)), V_lat[1]])
