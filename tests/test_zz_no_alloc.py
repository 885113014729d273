"""lb_linear_forward_noalloc: the decode forward that allocates no memory.

Some callers must not touch the CUDA allocator while they run: a serving loop
whose device memory is planned once at start-up (cudaMalloc/cudaFree may
synchronise the device and break that plan), or a runtime that owns all device
memory itself.  This entry point keeps its scratch in a fixed static array
inside the library instead.  Its output must match lb_linear_forward within
the tolerance of the other parity tests, on consecutive calls that share (and
inherit the contents of) that array.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""

import pytest

from sub_bit_weight_b200 import synth
from tests._util import TOL, rel_err

pytestmark = pytest.mark.gpu


def test_noalloc_matches_forward_on_consecutive_calls():
    import torch
    from sub_bit_weight_b200 import lib, stacks
    assert torch.cuda.is_available()
    a = synth.LayerShape("a", 1000, 2050, 80)
    b = synth.LayerShape("b", 4096, 4096, 184)
    La = stacks.build_layer(71, 0, a)
    Lb = stacks.build_layer(72, 1, b)
    calls = [(La, a, 1, 81), (Lb, b, 5, 82), (La, a, 16, 83)]
    for L, s, M, xs in calls:
        x = stacks.bf16_on_device(synth.activations(xs, 0, M, s.K), "cuda")
        ref = lib.lb_linear_forward(x, L).clone()
        y = torch.full((M, s.N), float("nan"), dtype=torch.float32, device="cuda")
        lib.lb_linear_forward_noalloc(x, L, y)
        # set-up kernel + the decode kernels (quantisation for one or two rows, then for any row count the
        # two contractions and the finish between them)
        assert lib.lb_last_launch_count() == (5 if M <= 2 else 4)
        torch.cuda.synchronize()
        err = rel_err(y.cpu().numpy(), ref.cpu().numpy())
        assert err <= TOL, (s, M, err)


def test_regular_calls_still_work_after_noalloc_calls():
    # the two entry points share kernel launch settings; a larger layer afterwards must still launch
    import torch
    from sub_bit_weight_b200 import lib, stacks
    small = synth.LayerShape("s", 256, 512, 32)
    big = synth.LayerShape("b", 1024, 4096, 800)
    Ls, Lb = stacks.build_layer(74, 0, small), stacks.build_layer(75, 1, big)
    for M in (1, 16):
        xs = stacks.bf16_on_device(synth.activations(84, 0, M, small.K), "cuda")
        lib.lb_linear_forward_noalloc(xs, Ls, torch.empty((M, small.N), dtype=torch.float32, device="cuda"))
        xb = stacks.bf16_on_device(synth.activations(85, 0, M, big.K), "cuda")
        y1 = lib.lb_linear_forward(xb, Lb)
        y2 = lib.lb_linear_forward_noalloc(xb, Lb, torch.empty_like(y1))
        torch.cuda.synchronize()
        assert rel_err(y2.cpu().numpy(), y1.cpu().numpy()) <= TOL


def test_noalloc_rejects_batches_above_the_decode_limit():
    import torch
    from sub_bit_weight_b200 import lib, stacks
    s = synth.LayerShape("c", 64, 64, 8)
    L = stacks.build_layer(73, 0, s)
    x = torch.zeros((17, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((17, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.LittleBitError) as e:
        lib.lb_linear_forward_noalloc(x, L, y)
    assert e.value.status == lib.LB_ERR_UNSUPPORTED
