"""Signed and zero scales on every kernel family, against the CPU oracle.

The scales h, g and l are learned real numbers (LittleBit notes page,
"Multi-scale compensation"); nothing bounds their sign, and a scale can be
exactly zero.  Here each path of a layer gets its own mix: about a third of
the entries of h, g and l negated and about an eighth set to zero (+0.0 or
-0.0), with different positions per path.  The shapes take the one- and
two-row streaming kernels (M = 1, 2), the general decode kernels (M = 3..16)
and the tensor-core kernels (M > 16 with K % 8 == 0 and N % 4 == 0, several
128 x 256 tiles), one and two paths.  A non-finite activation row on the
tensor-core path must give NaN in that row only.  The bar is the workload's:
max|y_gpu - y_ref| / max|y_ref| <= 2e-3 per layer.
"""

import numpy as np
import pytest

import oracle
from sub_bit_weight_b200 import synth
from tests._util import TOL, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch
    from sub_bit_weight_b200 import lib, stacks
    assert torch.cuda.is_available()
    return torch, lib, stacks


def _mix_signs(vec_u16, rng):
    """Negate ~1/3 of a binary16 vector and zero ~1/8 (half of those as -0.0)."""
    v = vec_u16.copy()
    n = v.size
    neg = rng.random(n) < 1.0 / 3.0
    v[neg] ^= np.uint16(0x8000)
    zero = rng.random(n) < 1.0 / 8.0
    v[zero] = np.uint16(0)
    negzero = zero & (rng.random(n) < 0.5)
    v[negzero] = np.uint16(0x8000)
    return v


def _signed_layer(seed, shape, npaths):
    L = oracle_layer(seed, 0, shape, npaths)
    rng = np.random.default_rng([seed, 0x5167])
    for key in ("h", "g", "l"):
        L[key] = [_mix_signs(a, rng) for a in L[key]]
    return L


def _device_layer(env, L, shape, npaths):
    torch, lib, stacks = env
    dev = lambda a: stacks.half_on_device(a, "cuda")
    U = [torch.from_numpy(u.view(np.int32)).cuda() for u in L["U"][:npaths]]
    V = [torch.from_numpy(v.view(np.int32)).cuda() for v in L["V"][:npaths]]
    return lib.lb_layer_create(shape.N, shape.K, shape.r, U, V, [dev(a) for a in L["h"][:npaths]],
                               [dev(a) for a in L["g"][:npaths]], [dev(a) for a in L["l"][:npaths]])


DECODE = [(257, 1000, 33, 2), (700, 3000, 184, 2), (96, 4100, 304, 1), (1024, 2048, 128, 2), (65, 33, 800, 2)]


@pytest.mark.parametrize("N,K,r,P", DECODE)
@pytest.mark.parametrize("M", [1, 2, 3, 5, 16])
def test_decode_signed_and_zero_scales(env, N, K, r, P, M):
    torch, lib, stacks = env
    shape = synth.LayerShape("s", N, K, r)
    seed = 3000 + N + K + r
    L = _signed_layer(seed, shape, P)
    layer = _device_layer(env, L, shape, P)
    xb = synth.activations(seed, 1, M, K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    assert rel_err(y.cpu().numpy(), oracle.forward(xb, L)) <= TOL


PREFILL = [(600, 1024, 200, 2, 300), (1000, 512, 37, 2, 129), (520, 768, 64, 1, 257), (1024, 2048, 300, 2, 140)]


@pytest.mark.parametrize("N,K,r,P,M", PREFILL)
def test_prefill_signed_and_zero_scales(env, N, K, r, P, M):
    torch, lib, stacks = env
    shape = synth.LayerShape("s", N, K, r)
    seed = 4000 + N + K + r
    L = _signed_layer(seed, shape, P)
    layer = _device_layer(env, L, shape, P)
    xb = synth.activations(seed, 1, M, K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    assert lib.lb_last_launch_count() == 2          # the two tensor-core kernels
    assert rel_err(y.cpu().numpy(), oracle.forward(xb, L)) <= TOL


def test_prefill_nonfinite_activation_row(env):
    torch, lib, stacks = env
    shape = synth.LayerShape("s", 512, 1024, 96)
    L = _signed_layer(4100, shape, 2)
    layer = _device_layer(env, L, shape, 2)
    M = 200
    xb = synth.activations(4100, 1, M, shape.K).copy()
    bad = [3, 130]                                  # rows in two different 128-row tiles
    xb[3, 17] = 0x7FC0                              # bfloat16 NaN
    xb[130, 900] = 0x7F80                           # bfloat16 +inf
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    assert lib.lb_last_launch_count() == 2
    got = y.cpu().numpy()
    ref = oracle.forward(xb, L)
    for m in bad:
        assert np.all(np.isnan(got[m])) and np.all(np.isnan(ref[m]))
    keep = [m for m in range(M) if m not in bad]
    assert rel_err(got[keep], ref[keep]) <= TOL


def test_13b_gate_layer_every_row_tile(env):
    # 16 seeded rows in every one of the 16 row tiles of a full Llama-2-13B-shaped gate layer at M = 2048
    torch, lib, stacks = env
    shape = synth.LayerShape("gate", 13824, 5120, 544)
    layer = stacks.build_layer(3, 0, shape)
    M = 2048
    xb = synth.activations(3, 1, M, shape.K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2048)
    ms = np.sort(np.concatenate([t * 128 + rng.choice(128, size=16, replace=False) for t in range(M // 128)]))
    ref = oracle.forward_sampled(xb, oracle_layer(3, 0, shape), ms, np.arange(shape.N))
    assert rel_err(y.cpu().numpy()[ms], ref) <= TOL
