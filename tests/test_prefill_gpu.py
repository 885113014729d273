"""Tensor-core (prefill, M > 16) parity: lb_linear_forward against the CPU oracle.

Shapes cover several 128-row / 256-column tiles with ragged tails: M not a
multiple of 128, N not a multiple of 256 (or of 16, or of 4), K not a multiple
of 64, r not a multiple of 8, one and two paths.
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


def _check(env, seed, shape, M, npaths=2, rows=None):
    torch, lib, stacks = env
    layer = stacks.build_layer(seed, 0, shape, npaths=npaths)
    xb = synth.activations(seed, 1, M, shape.K)
    y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
    torch.cuda.synchronize()
    if shape.K % 8 == 0 and shape.N % 4 == 0:
        assert lib.lb_last_launch_count() == 2      # the two tensor-core kernels (16-byte rows for TMA)
    L = oracle_layer(seed, 0, shape, npaths)
    if rows is None:
        ref = oracle.forward(xb, L)
        got = y.cpu().numpy()
    else:
        rng = np.random.default_rng(seed)
        ms = np.sort(rng.choice(M, size=rows, replace=False))
        ns = np.arange(shape.N)
        ref = oracle.forward_sampled(xb, L, ms, ns)
        got = y.cpu().numpy()[ms]
    err = rel_err(got, ref)
    print(f"{shape} M={M} P={npaths} rel_err={err:.3e}")
    assert err <= TOL, err
    return y


@pytest.mark.parametrize("N,K,r,P,M", [
    (384, 512, 40, 2, 17), (384, 512, 40, 2, 128), (1000, 1000, 37, 2, 200),
    (256, 2048, 300, 2, 300), (96, 64, 1, 2, 33), (4100, 768, 64, 2, 140), (1004, 520, 8, 1, 129),
])
def test_ragged_shapes(env, N, K, r, P, M):
    _check(env, 400 + N + r, synth.LayerShape("t", N, K, r), M, npaths=P)


def test_13b_q_shape(env):
    _check(env, 3, synth.LayerShape("q", 5120, 5120, 368), 256, rows=24)


def test_13b_gate_shape_full_rows(env):
    _check(env, 3, synth.LayerShape("gate", 13824, 5120, 544), 2048, rows=16)


def test_13b_down_shape(env):
    _check(env, 3, synth.LayerShape("down", 5120, 13824, 544), 2048, rows=16)


def test_repeatable_and_stack_equal(env):
    torch, lib, stacks = env
    shapes = [synth.LayerShape("a", 640, 1024, 96), synth.LayerShape("b", 300, 2048, 50)]
    layers = [stacks.build_layer(50 + i, i, s) for i, s in enumerate(shapes)]
    M = 260
    xs = [stacks.bf16_on_device(synth.activations(60 + i, i, M, s.K), "cuda") for i, s in enumerate(shapes)]
    singles = [lib.lb_linear_forward(x, L).clone() for x, L in zip(xs, layers)]
    again = [lib.lb_linear_forward(x, L) for x, L in zip(xs, layers)]
    S = lib.lb_stack_create(layers)
    ys = [torch.empty((M, s.N), dtype=torch.float32, device="cuda") for s in shapes]
    lib.lb_stack_forward(S, xs, ys)
    torch.cuda.synchronize()
    for a, b, c in zip(singles, again, ys):
        assert torch.equal(a, b)
        assert torch.equal(a, c)


def test_rows_not_16_byte_multiples_run_as_row_blocks(env):
    # the tensor-core path needs 16-byte rows of x and y; other K / N take the 16-row decode path
    _check(env, 9, synth.LayerShape("t", 200, 300, 40), 40)
    _check(env, 10, synth.LayerShape("t", 1001, 520, 8), 129, npaths=1)
