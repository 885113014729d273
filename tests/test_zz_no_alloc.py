"""lb_linear_forward_noalloc: the decode forward that allocates no memory.

Some callers must not touch the CUDA allocator while they run: a serving loop
whose device memory is planned once at start-up (cudaMalloc/cudaFree may
synchronise the device and break that plan), or a runtime that owns all device
memory itself.  This entry point keeps its scratch in a fixed static array
inside the library instead.  Its output must match lb_linear_forward, and the
oracle, within the tolerance of the other parity tests, on consecutive calls
that share (and inherit the contents of) that array.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""

import pytest

from sub_bit_weight_b200 import synth
from tests._util import TOL, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


def test_noalloc_matches_forward_and_oracle_on_consecutive_calls():
    import torch
    import oracle
    from sub_bit_weight_b200 import lib, stacks
    assert torch.cuda.is_available()
    a = synth.LayerShape("a", 1000, 2050, 80)
    b = synth.LayerShape("b", 4096, 4096, 184)
    La = stacks.build_layer(71, 0, a)
    Lb = stacks.build_layer(72, 1, b)
    refs = {71: oracle_layer(71, 0, a), 72: oracle_layer(72, 1, b)}
    # one and two rows take the streaming kernels (separate template instances), 5 and 16 the general ones
    calls = [(La, a, 71, 1, 81), (Lb, b, 72, 5, 82), (La, a, 71, 2, 86), (Lb, b, 72, 2, 87), (La, a, 71, 16, 83),
             (Lb, b, 72, 1, 88)]
    for L, s, seed, M, xs in calls:
        xb = synth.activations(xs, 0, M, s.K)
        x = stacks.bf16_on_device(xb, "cuda")
        ref = lib.lb_linear_forward(x, L).clone()
        y = torch.full((M, s.N), float("nan"), dtype=torch.float32, device="cuda")
        lib.lb_linear_forward_noalloc(x, L, y)
        # set-up kernel + the decode kernels (quantisation for one or two rows, then for any row count the
        # two contractions and the finish between them)
        assert lib.lb_last_launch_count() == (5 if M <= 2 else 4)
        torch.cuda.synchronize()
        yn = y.cpu().numpy()
        assert rel_err(yn, ref.cpu().numpy()) <= TOL, (s, M)
        assert rel_err(yn, oracle.forward(xb, refs[seed])) <= TOL, (s, M)
        assert lib.lb_layer_status(L) == lib.LB_OK


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


def test_noalloc_scratch_limit():
    # The static array holds the scratch of a two-path layer up to K = 83,328 inputs at r = 1184 (the
    # accumulators, the latent fragments, the input fragments and their exponents fill 1 MiB to within 224
    # bytes); one more 32-input block is refused.
    import torch
    from sub_bit_weight_b200 import lib, stacks
    at = synth.LayerShape("at", 64, 83328, 1184)
    over = synth.LayerShape("over", 64, 83360, 1184)
    L = stacks.build_layer(76, 0, at)
    for M in (1, 2, 16):
        x = stacks.bf16_on_device(synth.activations(89, 0, M, at.K), "cuda")
        y1 = lib.lb_linear_forward(x, L).clone()
        y2 = lib.lb_linear_forward_noalloc(x, L, torch.empty_like(y1))
        y3 = lib.lb_linear_forward_noalloc(x, L, torch.empty_like(y1))
        torch.cuda.synchronize()
        assert rel_err(y2.cpu().numpy(), y1.cpu().numpy()) <= TOL, M
        assert rel_err(y3.cpu().numpy(), y1.cpu().numpy()) <= TOL, M
    del L
    Lo = stacks.build_layer(77, 0, over)
    x = stacks.bf16_on_device(synth.activations(90, 0, 1, over.K), "cuda")
    with pytest.raises(lib.LittleBitError) as e:
        lib.lb_linear_forward_noalloc(x, Lo, torch.empty((1, over.N), dtype=torch.float32, device="cuda"))
    assert e.value.status == lib.LB_ERR_UNSUPPORTED


def test_noalloc_timeouts_reach_the_layer_status():
    # The no-alloc kernels report a bounded wait that gave up to the layer's own error slot; the self-test
    # aimed at that slot must show up in lb_layer_status exactly once, and the layer must still compute.
    import torch
    from sub_bit_weight_b200 import lib, stacks
    s = synth.LayerShape("t", 192, 256, 24)
    L = stacks.build_layer(78, 0, s)
    assert lib.lb_layer_selftest_wait_timeout(L, 100_000) == lib.LB_OK
    assert lib.lb_layer_status(L) == lib.LB_ERR_TIMEOUT
    assert lib.lb_layer_status(L) == lib.LB_OK
    x = stacks.bf16_on_device(synth.activations(91, 0, 1, s.K), "cuda")
    y1 = lib.lb_linear_forward(x, L).clone()
    y2 = lib.lb_linear_forward_noalloc(x, L, torch.empty_like(y1))
    torch.cuda.synchronize()
    assert rel_err(y2.cpu().numpy(), y1.cpu().numpy()) <= TOL
    assert lib.lb_layer_status(L) == lib.LB_OK


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
