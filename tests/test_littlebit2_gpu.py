"""Parity of the CUDA LittleBit-2 initialisation (Joint-ITQ latent rotation + Dual-SVID) with the float64 oracle.

Source: wiki page on LittleBit and LittleBit-2, section 1 (latent rotation by
joint iterative quantisation before QAT), on top of the LittleBit paper notes
page, "Dual-SVID initialisation" and "Residual compensation".  Both sides
compute in binary64: the oracle takes LAPACK SVDs for the truncated SVD and
for each Procrustes step, the CUDA path subspace iteration and Newton-Schulz
iterations.  On inputs whose leading singular values are separated the
factors agree to ~1e-12, so every sign decision of every ITQ alternation is
the same on both sides: the rotation and the loss sequence agree to 1e-9 and
the sign words bit for bit.  Scales are float32 outputs, compared at 1e-6 of
each vector's largest entry (float32 rounding is 6e-8).
"""

import numpy as np
import pytest
import torch

from oracle import dual_svid as ods
from oracle import littlebit2 as lb2
from sub_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-6
TOL_R = 1e-9


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from sub_bit_weight_b200 import lib as _lib
    return _lib


def _unpack(words: torch.Tensor, r: int) -> np.ndarray:
    w = words.cpu().numpy().view(np.uint32)
    bits = (w[:, :, None] >> np.arange(32, dtype=np.uint32)[None, None, :]) & 1
    return np.where(bits.reshape(w.shape[0], -1)[:, :r] == 1, -1.0, 1.0)


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def _parity(lib, W, r, npaths, itq_iters, R0s=None, iters=24):
    ref = lb2.littlebit2_init(W.astype(np.float64), r, npaths, itq_iters, R0s)
    R0 = None if R0s is None else [torch.from_numpy(np.ascontiguousarray(R)).cuda() for R in R0s]
    res = lib.lb_littlebit2_init(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda(), r, npaths, iters,
                                 itq_iters, R0)
    for p, rp in enumerate(ref):
        np.testing.assert_allclose(res.R[p].cpu().numpy(), rp["R"], rtol=0, atol=TOL_R, err_msg=f"path {p} R")
        np.testing.assert_allclose(res.itq_loss[p].cpu().numpy(), rp["itq_loss"], rtol=0, atol=TOL_R,
                                   err_msg=f"path {p} loss")
        for f, words in (("U_sign", res.U[p]), ("V_sign", res.V[p])):
            np.testing.assert_array_equal(words.cpu().numpy().view(np.uint32), ods.pack_rows(rp[f]),
                                          err_msg=f"path {p} {f}")
        for f in ("h", "g", "l"):
            assert _rel(getattr(res, f)[p].cpu().numpy(), rp[f]) <= TOL, f"path {p} {f}"
        assert _rel(res.sigma[p].cpu().numpy(), rp["sigma"]) <= TOL
        w_hat = ods.effective_weight(_unpack(res.U[p], r), _unpack(res.V[p], r),
                                     res.h[p].cpu().numpy().astype(np.float64),
                                     res.g[p].cpu().numpy().astype(np.float64),
                                     res.l[p].cpu().numpy().astype(np.float64))
        assert _rel(w_hat, rp["W_hat"]) <= TOL, f"path {p} W_hat"
        loss = res.itq_loss[p].cpu().numpy()
        assert np.all(np.diff(loss) <= 1e-12), loss          # ITQ never raises its loss
        Rg = res.R[p].cpu().numpy()
        np.testing.assert_allclose(Rg.T @ Rg, np.eye(r), rtol=0, atol=1e-12)
    return ref, res


@pytest.mark.parametrize("shape", [
    (40, 24, 6, 2, 10),       # subspace = whole space (exact SVD), K < N
    (24, 40, 6, 2, 10),       # K > N
    (300, 200, 7, 2, 30),     # subspace iteration, ragged sizes
    (512, 384, 16, 2, 50),
    (1000, 513, 100, 2, 50),  # odd K, r not a multiple of 32
    (2048, 1024, 128, 1, 50),
    (600, 400, 200, 2, 12),   # r above the one-cluster polar kernel's limit: the grid-wide kernel
    (130, 70, 1, 2, 5),       # r = 1: the rotation is +-1
    (256, 512, 24, 1, 20),    # one path, K > N
])
def test_parity_on_power_law_weights(lib, shape):
    N, K, r, npaths, it = shape
    _parity(lib, synth.dense_weight(31, N, K), r, npaths, it)


def test_parity_from_random_rotations(lib):
    N, K, r = 640, 320, 24
    R0s = [synth.random_rotation(41, r, p) for p in range(2)]
    _parity(lib, synth.dense_weight(32, N, K), r, 2, 40, R0s)


def test_given_rotation_without_iterations_is_applied_as_is(lib):
    N, K, r = 256, 192, 12
    R0s = [synth.random_rotation(42, r, p) for p in range(2)]
    ref, res = _parity(lib, synth.dense_weight(33, N, K), r, 2, 0, R0s)
    for p in range(2):
        np.testing.assert_allclose(res.R[p].cpu().numpy(), R0s[p], rtol=0, atol=1e-15)


def test_no_rotation_is_dual_svid_bit_for_bit(lib):
    W = torch.from_numpy(synth.dense_weight(34, 700, 300)).cuda()
    a = lib.lb_littlebit2_init(W, 40, 2, 24, 0, None)
    b = lib.lb_dual_svid_init(W, 40, 2, 24)
    for p in range(2):
        for f in ("U", "V", "h", "g", "l"):
            assert torch.equal(getattr(a, f)[p], getattr(b, f)[p]), (p, f)
        assert torch.equal(a.R[p].cpu(), torch.eye(40, dtype=torch.float64))


def test_rotation_lowers_the_quantisation_loss_at_llama2_7b_size(lib):
    # the q projection of the Llama-2-7B-shaped stack at ~0.1 BPW (4096 x 4096, r = 80), both paths, 50 alternations
    ref, res = _parity(lib, synth.dense_weight(35, 4096, 4096), 80, 2, 50)
    for p in range(2):
        loss = res.itq_loss[p].cpu().numpy()
        assert loss[-1] < 0.9 * loss[0]
