"""Pins of the LittleBit-2 Joint-ITQ oracle (oracle/littlebit2.py), from outside the oracle itself.

CPU only.  Source: wiki page on LittleBit and LittleBit-2, section 1 ("What
happened": latent rotation and joint iterative quantisation before QAT, the
initialisation only), on top of the LittleBit paper notes page, "Dual-SVID
initialisation" and "Residual compensation".  Each check rests on something
the oracle does not compute the same way: hand-derived fixtures
(tests/golden/joint_itq_cases.txt), the monotone loss of an alternating
minimisation, the optimality of each half-step checked by brute force, exact
equivariance under a rotation of the input, the invariances of the objective,
and the reduction to plain Dual-SVID when no rotation is made.
"""

import os

import numpy as np
import pytest

from oracle import dual_svid as ods
from oracle import littlebit2 as lb2
from sub_bit_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "joint_itq_cases.txt")


def _parse_golden():
    cases, cur = [], None
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, _, rest = line.partition(" ")
        if key == "case":
            cur = {"name": rest}
        elif key == "end":
            cases.append(cur)
        else:
            cur[key] = np.array([[float(t) for t in part.split()] for part in rest.split(";")])
    return cases


def _factors(seed, N, K, r):
    W = synth.dense_weight(seed, N, K).astype(np.float64)
    Up, Vp, _ = ods.truncated_svd_factors(W, r)
    return Up, Vp


def _loss(X, R):
    Y = X @ R
    return float(np.sum((np.where(Y < 0, -1.0, 1.0) - Y) ** 2)) / Y.size


@pytest.mark.parametrize("case", _parse_golden(), ids=lambda c: c["name"])
def test_hand_derived_cases(case):
    R, loss = lb2.joint_itq(case["Up"], case["Vp"], case["R0"], int(case["iters"][0][0]))
    np.testing.assert_allclose(R, case["R"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(loss, case["loss"][0], rtol=0, atol=1e-14)


@pytest.mark.parametrize("shape", [(96, 64, 8), (200, 120, 24), (64, 300, 16)])
def test_loss_never_increases_and_rotation_is_orthogonal(shape):
    Up, Vp = _factors(3, *shape)
    r = shape[2]
    for R0 in (None, synth.random_rotation(5, r)):
        R, loss = lb2.joint_itq(Up, Vp, R0, 30)
        assert np.all(np.diff(loss) <= 1e-12), loss
        assert loss[-1] < loss[0]
        np.testing.assert_allclose(R.T @ R, np.eye(r), rtol=0, atol=1e-12)


def test_each_half_step_is_optimal():
    # the sign step minimises the loss entrywise; the Procrustes step beats every nearby rotation
    Up, Vp = _factors(4, 120, 80, 6)
    X = lb2.itq_data(Up, Vp)
    R0 = synth.random_rotation(9, 6)
    Y = X @ R0
    B = np.where(Y < 0, -1.0, 1.0)
    rng = np.random.default_rng(0)
    for _ in range(20):   # any other +-1 matrix is no closer to Y
        flip = rng.random(B.shape) < 0.05
        assert np.sum((np.where(flip, -B, B) - Y) ** 2) >= np.sum((B - Y) ** 2)
    R1, _ = lb2.joint_itq(Up, Vp, R0, 1)
    best = np.sum((B - X @ R1) ** 2)
    for _ in range(200):  # R1 against rotations R1 expm(A) and random orthogonal matrices, for the same B
        A = rng.standard_normal((6, 6)) * 1e-3
        A = A - A.T
        Q = np.linalg.qr(np.eye(6) + A)[0]
        Q = Q * np.sign(np.diag(np.linalg.qr(np.eye(6) + A)[1]))[None, :]
        assert np.sum((B - X @ (R1 @ Q)) ** 2) >= best - 1e-9
    for k in range(50):
        assert np.sum((B - X @ synth.random_rotation(100 + k, 6)) ** 2) >= best


def test_rotated_hypercube_is_recovered_in_one_step():
    # X = B0 Q0^T for a +-1 matrix B0 and a small rotation Q0: sign(X) = B0, and the Procrustes step returns Q0
    rng = np.random.default_rng(1)
    r = 5
    Bu = np.where(rng.random((40, r)) < 0.5, -1.0, 1.0)
    Bv = np.where(rng.random((30, r)) < 0.5, -1.0, 1.0)
    A = rng.standard_normal((r, r)) * 0.02
    Q0 = np.linalg.qr(np.eye(r) + (A - A.T))[0]
    Q0 = Q0 * np.sign(np.diag(Q0))[None, :]
    R, loss = lb2.joint_itq(2.0 * Bu @ Q0.T, 0.1 * Bv @ Q0.T, None, 2)
    np.testing.assert_allclose(R, Q0, rtol=0, atol=1e-12)
    assert loss[0] > 0 and loss[1] < 1e-28 and loss[2] < 1e-28


def test_equivariance_under_a_rotation_of_the_latent_space():
    # rotating both factors by Q and the start by Q^T rotates the result: R'(U'Q, V'Q, Q^T R0) = Q^T R(U', V', R0)
    Up, Vp = _factors(6, 150, 100, 12)
    Q = synth.random_rotation(11, 12)
    R0 = synth.random_rotation(12, 12)
    R, loss = lb2.joint_itq(Up, Vp, R0, 10)
    R2, loss2 = lb2.joint_itq(Up @ Q, Vp @ Q, Q.T @ R0, 10)
    np.testing.assert_allclose(R2, Q.T @ R, rtol=0, atol=1e-10)
    np.testing.assert_allclose(loss2, loss, rtol=0, atol=1e-12)


def test_invariances_of_the_objective():
    # scaling either factor, permuting rows and flipping the sign of rows leave the rotation unchanged
    Up, Vp = _factors(7, 90, 70, 8)
    R0 = synth.random_rotation(13, 8)
    R, loss = lb2.joint_itq(Up, Vp, R0, 8)
    rng = np.random.default_rng(2)
    pu, pv = rng.permutation(90), rng.permutation(70)
    su = np.where(rng.random(90) < 0.5, -1.0, 1.0)[:, None]
    for U2, V2 in ((7.0 * Up, 0.01 * Vp), (Up[pu], Vp[pv]), (su * Up, Vp)):
        R2, loss2 = lb2.joint_itq(U2, V2, R0, 8)
        np.testing.assert_allclose(R2, R, rtol=0, atol=1e-10)
        np.testing.assert_allclose(loss2, loss, rtol=0, atol=1e-12)


def test_rotation_preserves_the_rank_r_product():
    W = synth.dense_weight(8, 160, 96).astype(np.float64)
    Up, Vp, _ = ods.truncated_svd_factors(W, 10)
    p = lb2.littlebit2_path(W, 10, synth.random_rotation(14, 10), 20)
    np.testing.assert_allclose(p["U_prime"] @ p["V_prime"].T, Up @ Vp.T, rtol=0, atol=1e-13)
    # the signs are those of the rotated factors, canonical columns
    np.testing.assert_array_equal(p["U_sign"], np.where(p["U_prime"] < 0, -1.0, 1.0))
    for j in range(10):
        col = p["U_prime"][:, j]
        assert col[np.argmax(np.abs(col))] > 0


def test_no_rotation_reduces_to_dual_svid():
    W = synth.dense_weight(9, 128, 96)
    a = lb2.littlebit2_init(W, 12, 2, itq_iters=0)
    b = ods.littlebit_init(W, 12, 2)
    for pa, pb in zip(a, b):
        for f in ("U_sign", "V_sign"):
            np.testing.assert_array_equal(pa[f], pb[f])
        for f in ("h", "g", "l", "W_hat"):
            np.testing.assert_allclose(pa[f], pb[f], rtol=0, atol=1e-15)


def test_rotation_aligns_the_factors_with_the_hypercube():
    # after Joint-ITQ the factors' magnitudes are flatter: the rank-1 magnitude model explains more of |U' R|,
    # and the quantisation loss of the stacked, normalised factors drops well below its starting value
    W = synth.dense_weight(10, 512, 384).astype(np.float64)
    p0 = lb2.littlebit2_path(W, 32, None, 0)
    p1 = lb2.littlebit2_path(W, 32, None, 50)
    assert p1["itq_loss"][-1] < 0.8 * p1["itq_loss"][0]
    X0 = lb2.itq_data(p0["U_prime"], p0["V_prime"])
    X1 = lb2.itq_data(p1["U_prime"], p1["V_prime"])
    assert _loss(X1, np.eye(32)) == pytest.approx(p1["itq_loss"][-1], abs=1e-12)
    assert _loss(X1, np.eye(32)) < _loss(X0, np.eye(32))


def test_random_rotation_generator():
    # the seeded start rotations handed to both sides: orthogonal, reproducible, distinct per path
    for r in (1, 5, 64):
        Q = synth.random_rotation(3, r)
        np.testing.assert_allclose(Q.T @ Q, np.eye(r), rtol=0, atol=1e-13)
        np.testing.assert_array_equal(Q, synth.random_rotation(3, r))
    assert not np.allclose(synth.random_rotation(3, 8, 0), synth.random_rotation(3, 8, 1))
