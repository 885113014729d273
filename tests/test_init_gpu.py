"""Parity of the CUDA Dual-SVID + residual initialisation with the float64 oracle.

Source: LittleBit paper notes page, "Dual-SVID initialisation" and "Residual
compensation".  Both sides compute in binary64; the CUDA path finds the
truncated SVD by subspace iteration + Rayleigh-Ritz, the oracle by LAPACK, so
on inputs whose leading singular values are separated the results agree to
~1e-12 and the sign decisions agree exactly.  The CUDA outputs are float32
scales, compared with a relative tolerance of 1e-6 of each vector's largest
entry (float32 rounding is 6e-8).  Sign words are compared bit for bit except
where the pages' method itself leaves the sign undetermined: columns whose
singular value is zero up to rounding (their factor entries are rounding
residues), and exact ties of the canonical-sign rule (sign products with
constant magnitudes), where only the product W_hat is unique.
"""

import numpy as np
import pytest
import torch

from oracle import dual_svid as ods
from sub_bit_weight_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 1e-6


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


def _w_hat(res, p, r):
    return ods.effective_weight(_unpack(res.U[p], r), _unpack(res.V[p], r), res.h[p].cpu().numpy().astype(np.float64),
                                res.g[p].cpu().numpy().astype(np.float64), res.l[p].cpu().numpy().astype(np.float64))


def _close(a, b, what):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    scale = max(np.abs(b).max(), 1e-300)
    err = np.abs(a - b).max() / scale
    assert err <= TOL, f"{what}: max rel err {err:.3e}"


def _parity(lib, W, r, npaths, iters=24, check_bits=True):
    ref = ods.littlebit_init(W.astype(np.float64), r, npaths)
    res = lib.lb_dual_svid_init(torch.from_numpy(np.ascontiguousarray(W, np.float32)).cuda(), r, npaths, iters)
    for p, rp in enumerate(ref):
        s = rp["sigma"]
        live = s > 1e-10 * max(s[0], 1e-300)       # columns whose sign factors are determined
        _close(res.sigma[p].cpu().numpy(), s, f"path {p} sigma")
        for f in ("h", "g", "l"):
            _close(getattr(res, f)[p].cpu().numpy(), rp[f], f"path {p} {f}")
        if check_bits:
            for f, words in (("U_sign", res.U[p]), ("V_sign", res.V[p])):
                got = _unpack(words, r)
                if live.all():
                    np.testing.assert_array_equal(words.cpu().numpy().view(np.uint32),
                                                  ods.pack_rows(rp[f]), err_msg=f"path {p} {f}")
                else:
                    np.testing.assert_array_equal(got[:, live], rp[f][:, live], err_msg=f"path {p} {f}")
        _close(_w_hat(res, p, r), rp["W_hat"], f"path {p} W_hat")
    return ref, res


def _golden_cases():
    from tests.test_oracle_dual_svid import _parse_golden
    return _parse_golden()


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_derived_cases(lib, case):
    r, npaths = int(case["r"][0][0]), int(case["npaths"][0][0])
    _, res = _parity(lib, case["W"], r, npaths)
    for p in range(npaths):
        _close(_w_hat(res, p, r), case[f"p{p}.W_hat"], f"path {p} hand-derived W_hat")


@pytest.mark.parametrize("shape", [
    (40, 24, 6, 2),        # subspace = whole space (exact path), K < N
    (24, 40, 6, 2),        # K > N: A = W^T
    (64, 64, 64, 1),       # r = min(N, K)
    (300, 200, 7, 2),      # subspace iteration, one 64-column panel, ragged sizes
    (512, 384, 16, 2),
    (384, 512, 32, 2),
    (1000, 513, 100, 2),   # odd K, four panels, ragged last panel
    (2048, 1024, 128, 2),
])
def test_parity_on_power_law_weights(lib, shape):
    N, K, r, npaths = shape
    W = synth.dense_weight(21, N, K)
    _parity(lib, W, r, npaths)


def test_exact_sign_product_is_reproduced(lib):
    # W = c S diag(l) T^T with orthogonal +-1 columns: Dual-SVID is exact and the residual path vanishes.  Every
    # |U'| entry of a column ties, so the sign of each pair is a rounding decision: compare W_hat, and the signs
    # up to one joint flip per column.
    H16 = np.array([[1.0]])
    while H16.shape[0] < 32:
        H16 = np.block([[H16, H16], [H16, -H16]])
    S, T = H16[:16, :16][:, [1, 2, 5, 11]], H16[:, [3, 6, 9, 30]]
    W = 0.91 * (S * np.array([5.0, 3.0, 2.0, 1.5])) @ T.T
    res = lib.lb_dual_svid_init(torch.from_numpy(W.astype(np.float32)).cuda(), 4, 2, 24)
    _close(_w_hat(res, 0, 4), W, "primary W_hat")
    assert np.abs(_w_hat(res, 1, 4)).max() <= 1e-5 * np.abs(W).max()
    U = _unpack(res.U[0], 4)
    flip = np.sign((U * S).sum(axis=0))
    np.testing.assert_array_equal(U, S * flip)
    np.testing.assert_array_equal(_unpack(res.V[0], 4), T * flip)


def test_rank_deficient_weight(lib):
    # rank-1 W with r = 3 and a subspace smaller than the space: the iteration drops the dependent columns; the
    # primary path reproduces W, the two zero singular values give zero scales
    rng = np.random.default_rng(4)
    W = np.outer(rng.standard_normal(300), rng.standard_normal(200)).astype(np.float32)
    res = lib.lb_dual_svid_init(torch.from_numpy(W).cuda(), 3, 1, 24)
    _close(_w_hat(res, 0, 3), W, "rank-1 W_hat")
    s = res.sigma[0].cpu().numpy()
    assert s[1] <= 1e-6 * s[0] and s[2] <= 1e-6 * s[0]


@pytest.mark.parametrize("shape", [(8, 6, 2), (300, 200, 3)])
def test_zero_weight(lib, shape):
    N, K, r = shape
    res = lib.lb_dual_svid_init(torch.zeros((N, K), dtype=torch.float32, device="cuda"), r, 2, 4)
    for p in range(2):
        for t in (res.U[p], res.V[p]):
            assert int(t.abs().sum()) == 0                      # sign(0) = +1 everywhere
        for t in (res.h[p], res.g[p], res.l[p], res.sigma[p]):
            assert float(t.abs().max()) == 0.0


def test_initialised_layer_forward_matches_the_oracle(lib):
    # init -> lb_layer_create (binary16 scales) -> lb_linear_forward, against the oracle's forward of the oracle's
    # own initialisation with the same binary16 rounding
    import oracle
    N, K, r = 768, 1024, 64
    W = synth.dense_weight(22, N, K)
    res = lib.lb_dual_svid_init(torch.from_numpy(W).cuda(), r, 2, 24)
    layer = lib.lb_layer_create(N, K, r, *res.layer_args())
    ref = ods.littlebit_init(W.astype(np.float64), r, 2)
    f16 = lambda v: np.asarray(v, np.float32).astype(np.float16).view(np.uint16)
    olayer = {"N": N, "K": K, "r": r, "U": [ods.pack_rows(p["U_sign"]) for p in ref],
              "V": [ods.pack_rows(p["V_sign"]) for p in ref], "h": [f16(p["h"]) for p in ref],
              "g": [f16(p["g"]) for p in ref], "l": [f16(p["l"]) for p in ref]}
    x = synth.activations(22, 0, 4, K)
    y = lib.lb_linear_forward(torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16), layer).cpu().numpy()
    yref = oracle.forward(x, olayer)
    assert np.abs(y - yref).max() / np.abs(yref).max() <= 2e-3
    # and the two-path layer approximates W better than the primary path alone
    e1 = np.linalg.norm(W - ref[0]["W_hat"])
    e2 = np.linalg.norm(W - ref[0]["W_hat"] - _w_hat(res, 1, r))
    assert e2 < e1


@pytest.mark.parametrize("shape", [(4096, 4096, 80), (4096, 11008, 128)])
def test_parity_at_llama2_7b_layer_sizes(lib, shape):
    # the q/k/v/o and down-projection shapes of the Llama-2-7B stack at ~0.1 BPW (oracle: full LAPACK SVDs)
    N, K, r = shape
    W = synth.dense_weight(23, N, K)
    _parity(lib, W, r, 2)
