"""Decode-path (M <= 16) parity: lb_linear_forward against the CPU oracle.

Element-by-element comparison on the same seeded inputs; the bar is
max|y_gpu - y_ref| / max|y_ref| <= 2e-3.  Shapes span several tiles with
ragged tails (N, K not multiples of 64 / 32, r not a multiple of 16 / 32).
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


def _run(env, seed, shape, M, npaths=2, xseed=None):
    torch, lib, stacks = env
    layer = stacks.build_layer(seed, 0, shape, npaths=npaths)
    xb = synth.activations(seed if xseed is None else xseed, 0, M, shape.K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    ref = oracle.forward(xb, oracle_layer(seed, 0, shape, npaths))
    return y.cpu().numpy(), ref, layer, xb


@pytest.mark.parametrize("M", [1, 8])
def test_single_512_workload(env, M):
    w = synth.WORKLOADS["single_512"]
    y, ref, _, _ = _run(env, w.seed, w.block[0], M)
    err = rel_err(y, ref)
    print(f"single_512 M={M} rel_err={err:.3e}")
    assert err <= TOL


SHAPES = [
    (100, 70, 5, 2), (64, 64, 16, 1), (1, 1, 1, 2), (257, 1000, 33, 2), (130, 2050, 80, 2),
    (1024, 8192, 32, 2), (65, 33, 800, 2), (700, 3000, 184, 2), (96, 4100, 304, 1),
    (100, 300, 1024, 2),   # contraction-2 depth 64 k-blocks: the deepest the one/two-row kernels take
    (80, 200, 1030, 2),    # deeper than 64 k-blocks (generic streaming loop at one or two rows)
    (72, 520, 2048, 2),    # the largest rank, both paths: 128 k-blocks; at 3..16 rows deeper than the general
                           # kernels' shared memory, so the streaming kernels run once per pair of rows
]


@pytest.mark.parametrize("N,K,r,P", SHAPES)
@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 16])
def test_ragged_shapes(env, N, K, r, P, M):
    shape = synth.LayerShape("t", N, K, r)
    y, ref, _, _ = _run(env, 1000 + N + K + r, shape, M, npaths=P)
    err = rel_err(y, ref)
    assert err <= TOL, err


@pytest.mark.parametrize("M", [2, 7, 11, 13])
def test_all_batch_sizes(env, M):
    shape = synth.LayerShape("t", 320, 1536, 96)
    y, ref, _, _ = _run(env, 77, shape, M)
    assert rel_err(y, ref) <= TOL


def test_rows_above_decode_limit(env):
    shape = synth.LayerShape("t", 200, 300, 40)
    for M in (17, 40):
        y, ref, _, _ = _run(env, 78, shape, M)
        assert rel_err(y, ref) <= TOL


@pytest.mark.parametrize("M", [1, 4])
def test_repeatable(env, M):
    torch, lib, stacks = env
    shape = synth.LayerShape("t", 512, 2048, 128)
    layer = stacks.build_layer(5, 0, shape)
    x = stacks.bf16_on_device(synth.activations(5, 0, M, shape.K), "cuda")
    y1 = lib.lb_linear_forward(x, layer).clone()
    y2 = lib.lb_linear_forward(x, layer)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_empty_batch_and_bad_arguments(env):
    torch, lib, stacks = env
    shape = synth.LayerShape("t", 64, 64, 8)
    layer = stacks.build_layer(6, 0, shape)
    y = lib.lb_linear_forward(torch.empty((0, 64), dtype=torch.bfloat16, device="cuda"), layer)
    assert y.shape == (0, 64)
    x = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        lib.lb_linear_forward(x.float(), layer)
    buf = torch.zeros(2 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.LittleBitError) as e:
        lib.lb_linear_forward(buf[1:1 + 128].view(2, 64), layer)      # 2-byte offset: misaligned
    assert e.value.status == lib.LB_ERR_INVALID_ARG


def test_zero_and_negative_scales(env):
    torch, lib, stacks = env
    N, K, r = 96, 160, 24
    L = oracle_layer(9, 0, synth.LayerShape("t", N, K, r))
    L["h"][0] = np.zeros(N, dtype=np.uint16)                               # primary path muted
    L["g"][1] = (L["g"][1].view(np.float16) * np.float16(-1)).view(np.uint16)  # negative g
    L["l"][1][::3] = 0                                                     # some latent dims off
    dev = lambda a: stacks.half_on_device(a, "cuda")
    U = [torch.from_numpy(u.view(np.int32)).cuda() for u in L["U"]]
    V = [torch.from_numpy(v.view(np.int32)).cuda() for v in L["V"]]
    layer = lib.lb_layer_create(N, K, r, U, V, [dev(a) for a in L["h"]], [dev(a) for a in L["g"]],
                                [dev(a) for a in L["l"]])
    xb = synth.activations(9, 1, 3, K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    assert rel_err(y.cpu().numpy(), oracle.forward(xb, L)) <= TOL
    # all h zero -> exact zeros
    L2 = dict(L)
    L2["h"] = [np.zeros(N, dtype=np.uint16)] * 2
    layer2 = lib.lb_layer_create(N, K, r, U, V, [dev(a) for a in L2["h"]], [dev(a) for a in L["g"]],
                                 [dev(a) for a in L["l"]])
    y2 = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer2)
    assert torch.count_nonzero(y2).item() == 0


@pytest.mark.parametrize("M", [1, 2, 3])
def test_nonfinite_activation_row(env, M):
    torch, lib, stacks = env
    shape = synth.LayerShape("t", 128, 256, 32)
    layer = stacks.build_layer(10, 0, shape)
    xb = synth.activations(10, 0, M, shape.K).copy()
    bad = min(1, M - 1)
    xb[bad, 17] = 0x7FC0          # bfloat16 NaN in one row
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer).cpu().numpy()
    assert np.all(np.isnan(y[bad]))
    ref = oracle.forward(xb, oracle_layer(10, 0, shape))
    assert np.all(np.isnan(ref[bad]))
    keep = [m for m in range(M) if m != bad]
    if keep:
        assert rel_err(y[keep], ref[keep]) <= TOL
    # the next call on the same layer is unaffected by the non-finite row
    xg = synth.activations(11, 0, M, shape.K)
    y2 = lib.lb_linear_forward(stacks.bf16_on_device(xg, "cuda"), layer).cpu().numpy()
    assert rel_err(y2, oracle.forward(xg, oracle_layer(10, 0, shape))) <= TOL


@pytest.mark.parametrize("M", [1, 5])
def test_stack_matches_single_layer_calls(env, M):
    torch, lib, stacks = env
    shapes = [synth.LayerShape("a", 192, 320, 40), synth.LayerShape("b", 64, 1024, 16),
              synth.LayerShape("c", 1000, 96, 200), synth.LayerShape("a", 192, 320, 40)]
    layers = [stacks.build_layer(20 + i, i, s) for i, s in enumerate(shapes)]
    layers[3] = layers[0]                       # a layer may repeat in a stack
    S = lib.lb_stack_create(layers)
    xs = [stacks.bf16_on_device(synth.activations(30 + i, i, M, s.K), "cuda") for i, s in enumerate(shapes)]
    ys = [torch.empty((M, s.N), dtype=torch.float32, device="cuda") for s in shapes]
    lib.lb_stack_forward(S, xs, ys)
    assert lib.lb_last_launch_count() == (4 if M <= 2 else 3)
    for i, s in enumerate(shapes):
        single = lib.lb_linear_forward(xs[i], layers[i])
        torch.cuda.synchronize()
        assert torch.equal(single, ys[i])
        seed = 20 if i == 3 else 20 + i
        ref = oracle.forward(synth.activations(30 + i, i, M, s.K), oracle_layer(seed, 0 if i == 3 else i, s))
        assert rel_err(ys[i].cpu().numpy(), ref) <= TOL


@pytest.mark.parametrize("M", [3, 4, 16])
def test_stack_deeper_than_the_general_kernels(env, M):
    """A stack holding a two-path r = 2048 layer (128 contraction-2 k-blocks) at 3..16 rows runs the streaming
    kernels once per pair of rows (4 launches per pair); every layer, deep or shallow, still matches the oracle and
    the single-layer call, and the row pairs' outputs land in the right rows (ragged M = 3: a last single row)."""
    torch, lib, stacks = env
    shapes = [synth.LayerShape("d", 136, 264, 2048), synth.LayerShape("s", 200, 96, 24)]
    layers = [stacks.build_layer(40 + i, i, s) for i, s in enumerate(shapes)]
    S = lib.lb_stack_create(layers)
    xs = [stacks.bf16_on_device(synth.activations(50 + i, i, M, s.K), "cuda") for i, s in enumerate(shapes)]
    ys = [torch.empty((M, s.N), dtype=torch.float32, device="cuda") for s in shapes]
    lib.lb_stack_forward(S, xs, ys)
    assert lib.lb_last_launch_count() == 4 * ((M + 1) // 2)
    for i, s in enumerate(shapes):
        single = lib.lb_linear_forward(xs[i], layers[i])
        torch.cuda.synchronize()
        ref = oracle.forward(synth.activations(50 + i, i, M, s.K), oracle_layer(40 + i, i, s))
        assert rel_err(ys[i].cpu().numpy(), ref) <= TOL
        assert rel_err(single.cpu().numpy(), ref) <= TOL
