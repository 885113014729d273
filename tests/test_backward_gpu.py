"""Parity of the CUDA QAT backward of a LittleBit layer with the float64 oracle (oracle/qat_backward.py).

Source: LittleBit paper notes page, "Multi-scale compensation" and "Loss /
training strategy" (SmoothSign).  Tolerance, from the arithmetic of the CUDA
path: dy enters as fp16 after an exact power-of-two scaling, the latent
activations are rounded to fp16 between the contractions (at most three
roundings of 2^-11 on the longest chain, the input gradient) and every
product accumulates in float32, so each output is compared as
max|gpu - ref| / max|ref| <= 2e-3, the forward pass's bar.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import qat_backward as qb
from sub_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sub_bit_weight_b200 import lib as _lib
    return _lib


def _inputs(seed, N, K, r, M, npaths, dy_scale=1e-4):
    rng = np.random.default_rng(seed)
    U = [rng.normal(0, 0.02, (N, r)).astype(np.float32) for _ in range(npaths)]
    V = [rng.normal(0, 0.02, (K, r)).astype(np.float32) for _ in range(npaths)]
    h = [synth.scale_vector(seed, 0, p, "h", N) for p in range(npaths)]
    g = [synth.scale_vector(seed, 0, p, "g", K) for p in range(npaths)]
    l = [synth.scale_vector(seed, 0, p, "l", r) for p in range(npaths)]
    xb = synth.activations(seed, 0, M, K)
    dy = (rng.standard_normal((M, N)) * dy_scale).astype(np.float32)
    return U, V, h, g, l, xb, dy


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def _run(lib, N, K, r, M, npaths, seed=1, dy_scale=1e-4):
    U, V, h, g, l, xb, dy = _inputs(seed, N, K, r, M, npaths, dy_scale)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    B = lib.lb_backward_create(N, K, r, [cu(oracle.pack_signs(u).view(np.int32)) for u in U],
                               [cu(oracle.pack_signs(v).view(np.int32)) for v in V],
                               [cu(x.view(np.int16)) for x in h], [cu(x.view(np.int16)) for x in g],
                               [cu(x.view(np.int16)) for x in l])
    out = lib.lb_layer_backward(B, cu(xb.view(np.int16)).view(torch.bfloat16), cu(dy), [cu(u) for u in U],
                                [cu(v) for v in V])
    torch.cuda.synchronize()
    assert lib.lb_backward_status(B) == lib.LB_OK
    f16 = lambda v: v.view(np.float16).astype(np.float64)
    ref = qb.backward(synth.bf16_bits_to_f32(xb), dy, U, V, [f16(v) for v in h], [f16(v) for v in g],
                      [f16(v) for v in l])
    errs = {"dx": _rel(out["dx"].cpu().numpy(), ref["dx"])}
    for key in ("dh", "dg", "dl", "dU", "dV"):
        for p in range(npaths):
            errs[f"{key}{p}"] = _rel(out[key][p].cpu().numpy(), ref[key][p])
    bad = {k: v for k, v in errs.items() if not v <= TOL}
    assert not bad, (bad, errs)
    return errs


@pytest.mark.parametrize("shape", [
    (64, 96, 16, 64, 2),       # one M tile
    (256, 128, 37, 200, 2),    # r not a multiple of 8, M not a multiple of 128
    (512, 384, 40, 300, 1),    # one path
    (1024, 2048, 100, 257, 2),
])
def test_parity_small(lib, shape):
    _run(lib, *shape)


def test_large_dynamic_range_of_dy(lib):
    # dy spanning 1e-9 .. 1e3: the power-of-two scaling keeps it inside fp16
    _run(lib, 256, 256, 32, 128, 2, dy_scale=1e3)
    _run(lib, 256, 256, 32, 128, 2, dy_scale=1e-9)


def test_zero_dy(lib):
    N, K, r, M = 128, 128, 16, 64
    U, V, h, g, l, xb, dy = _inputs(3, N, K, r, M, 2)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    B = lib.lb_backward_create(N, K, r, [cu(oracle.pack_signs(u).view(np.int32)) for u in U],
                               [cu(oracle.pack_signs(v).view(np.int32)) for v in V],
                               [cu(x.view(np.int16)) for x in h], [cu(x.view(np.int16)) for x in g],
                               [cu(x.view(np.int16)) for x in l])
    out = lib.lb_layer_backward(B, cu(xb.view(np.int16)).view(torch.bfloat16), torch.zeros((M, N), device="cuda"),
                                [cu(u) for u in U], [cu(v) for v in V])
    assert float(out["dx"].abs().max()) == 0.0
    for key in ("dh", "dg", "dl", "dU", "dV"):
        assert all(float(t.abs().max()) == 0.0 for t in out[key])


@pytest.mark.parametrize("shape", [(5120, 5120, 368), (13824, 5120, 544)])
def test_parity_at_llama2_13b_layer_sizes(lib, shape):
    # the q and gate projections of the Llama-2-13B-shaped stack at ~0.3 BPW, M = 2048 rows
    N, K, r = shape
    _run(lib, N, K, r, 2048, 2)
