"""lb_pack_signs on the GPU is bit-exact against the oracle's packer."""

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import _golden_pack_cases, _special_factor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    import torch
    from sub_bit_weight_b200 import lib
    assert torch.cuda.is_available()
    return lib


def _gpu_pack(L, F):
    import torch
    out = L.lb_pack_signs(torch.from_numpy(F).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("rows,r", [(1, 1), (7, 31), (5, 32), (9, 33), (300, 80), (1000, 184),
                                    (28672, 304), (11, 800), (3, 2048)])
def test_pack_bit_exact(L, rows, r):
    rng = np.random.default_rng(rows + r)
    F = _special_factor(rng, rows, r)
    assert np.array_equal(_gpu_pack(L, F), oracle.pack_signs(F))


@pytest.mark.parametrize("case", range(len(_golden_pack_cases())))
def test_pack_golden(L, case):
    F, W = _golden_pack_cases()[case]
    assert np.array_equal(_gpu_pack(L, F), W)


def test_pack_empty_and_errors(L):
    import torch
    F = torch.empty((0, 5), dtype=torch.float32, device="cuda")
    assert L.lb_pack_signs(F).shape == (0, 1)
    with pytest.raises(TypeError):
        L.lb_pack_signs(torch.zeros((3, 4), dtype=torch.float64, device="cuda"))
