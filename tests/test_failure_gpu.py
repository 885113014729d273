"""Failure reporting of the bounded device-side waits (no GPU fault, no hang).

The kernels never wait without a limit: a wait that gives up records an error
code and its kernel returns.  The self-test entry point runs the same wait
helper on an mbarrier that nothing completes, with a short limit, so the
timeout path itself is exercised; afterwards the context must still work.
"""

import pytest

from sub_bit_weight_b200 import synth
from tests._util import TOL, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    import torch
    from sub_bit_weight_b200 import lib
    assert lib.lb_selftest_wait_timeout(200_000) == lib.LB_ERR_TIMEOUT
    assert lib.lb_selftest_wait_timeout(50_000) == lib.LB_ERR_TIMEOUT
    torch.cuda.synchronize()


def test_context_usable_and_status_clean_after_timeout():
    import torch
    import oracle
    from sub_bit_weight_b200 import lib, stacks
    assert lib.lb_selftest_wait_timeout(100_000) == lib.LB_ERR_TIMEOUT
    shape = synth.LayerShape("t", 192, 256, 24)
    layer = stacks.build_layer(90, 0, shape)
    for M in (1, 40):
        xb = synth.activations(91, 0, M, shape.K)
        y = lib.lb_linear_forward(stacks.bf16_on_device(xb, "cuda"), layer)
        assert lib.lb_layer_status(layer) == lib.LB_OK
        assert rel_err(y.cpu().numpy(), oracle.forward(xb, oracle_layer(90, 0, shape))) <= TOL
