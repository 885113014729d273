"""Pins of the Dual-SVID / residual-compensation oracle, from outside the oracle itself.

CPU only.  Each check rests on something the oracle's own code does not
compute the same way: hand-derived fixtures (tests/golden/dual_svid_cases.txt),
matrices whose Dual-SVID is exact by construction (Hadamard sign factors),
closed forms (Eckart-Young through a symmetric eigensolver, the rank-1 case),
the defining identities of a leading singular triplet, and the symmetries the
method has (scaling, negation, transposition, permutations, row sign flips).
Source: LittleBit paper notes page, "Dual-SVID initialisation" and "Residual
compensation".
"""

import os

import numpy as np
import pytest

from oracle import dual_svid as ods
from sub_bit_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "dual_svid_cases.txt")


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
            rows = [[float(t) for t in part.split()] for part in rest.split(";")]
            cur[key] = np.array(rows[0] if len(rows) == 1 and key.split(".")[-1] in ("h", "g", "l") else rows)
    return cases


@pytest.mark.parametrize("case", _parse_golden(), ids=lambda c: c["name"])
def test_hand_derived_cases(case):
    r, npaths = int(case["r"][0][0]), int(case["npaths"][0][0])
    paths = ods.littlebit_init(case["W"], r, npaths)
    for k, p in enumerate(paths):
        for f in ("U_sign", "V_sign"):
            np.testing.assert_array_equal(p[f], case[f"p{k}.{f}"], err_msg=f"path {k} {f}")
        for f in ("h", "g", "l", "W_hat"):
            np.testing.assert_allclose(p[f], case[f"p{k}.{f}"], rtol=0, atol=1e-12, err_msg=f"path {k} {f}")
    if npaths == 2:      # the hand-solvable cases with two paths are reproduced exactly
        np.testing.assert_allclose(sum(p["W_hat"] for p in paths), case["W"], rtol=0, atol=1e-12)


def _hadamard(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_exact_when_the_weight_is_a_scaled_sign_product():
    # W = c diag(h) S diag(l) T^T diag(g) with orthogonal +-1 columns and constant h, g: its SVD is
    # (S / sqrt N, c l sqrt(N K), T / sqrt K), |U'| is exactly rank 1, so Dual-SVID reproduces W and the
    # residual path is zero.
    N, K, lat = 16, 32, np.array([5.0, 3.0, 2.0, 1.5])
    S = _hadamard(N)[:, [1, 2, 5, 11]]
    T = _hadamard(K)[:, [3, 6, 9, 30]]
    W = 0.7 * 1.3 * (S * lat) @ T.T
    pri, res = ods.littlebit_init(W, 4, 2)
    np.testing.assert_allclose(pri["W_hat"], W, rtol=0, atol=1e-12 * np.abs(W).max())
    assert np.abs(res["W_hat"]).max() <= 1e-12 * np.abs(W).max()
    # the sign factors are S and T up to one joint sign per column
    flip = np.sign((pri["U_sign"] * S).sum(axis=0))
    np.testing.assert_array_equal(pri["U_sign"], S * flip)
    np.testing.assert_array_equal(pri["V_sign"], T * flip)
    np.testing.assert_allclose(np.sort(pri["l"])[::-1] * pri["h"].max() * pri["g"].max(), 0.91 * lat, rtol=1e-12)


def test_rank_one_path_is_the_leading_singular_term():
    # r = 1: |U'| is a single column, so the path is exactly s1 u1 v1^T; the triplet here comes from the
    # symmetric eigensolver of W^T W, not from the SVD the oracle calls.
    W = synth.dense_weight(11, 9, 6).astype(np.float64)
    p = ods.dual_svid(W, 1)
    lam, vecs = np.linalg.eigh(W.T @ W)
    v = vecs[:, -1]
    s = np.sqrt(lam[-1])
    u = W @ v / s
    np.testing.assert_allclose(p["W_hat"], s * np.outer(u, v), rtol=0, atol=1e-13 * np.abs(W).max())
    np.testing.assert_allclose(p["sigma"], [s], rtol=1e-13)


@pytest.mark.parametrize("shape", [(40, 24, 6), (24, 40, 6), (33, 33, 33)])
def test_truncation_error_is_the_tail_energy(shape):
    N, K, r = shape
    W = synth.dense_weight(12, N, K).astype(np.float64)
    Up, Vp, s = ods.truncated_svd_factors(W, r)
    lam = np.sort(np.linalg.eigvalsh(W.T @ W if K <= N else W @ W.T))[::-1]
    err = np.sum((W - Up @ Vp.T) ** 2)
    assert abs(err - max(lam[r:].sum(), 0.0)) <= 1e-10 * np.sum(W ** 2)
    np.testing.assert_allclose(s ** 2, lam[:r], rtol=1e-10, atol=1e-13 * lam[0])   # eigvalsh: absolute error ~ eps lam_1
    # balanced split: U'^T U' = V'^T V' = diag(s)
    np.testing.assert_allclose(Up.T @ Up, np.diag(s), atol=1e-12 * s[0])
    np.testing.assert_allclose(Vp.T @ Vp, np.diag(s), atol=1e-12 * s[0])
    # canonical sign: each U' column's largest-magnitude entry is positive
    assert np.all(Up[np.argmax(np.abs(Up), axis=0), np.arange(r)] > 0)


def test_rank1_identities_on_a_magnitude_matrix():
    W = synth.dense_weight(13, 50, 30).astype(np.float64)
    Up, _, _ = ods.truncated_svd_factors(W, 7)
    A = np.abs(Up)
    s, a, b = ods.rank1(A)
    np.testing.assert_allclose(A @ b, s * a, atol=1e-13 * s)
    np.testing.assert_allclose(A.T @ a, s * b, atol=1e-13 * s)
    assert abs(np.linalg.norm(a) - 1) < 1e-13 and abs(np.linalg.norm(b) - 1) < 1e-13
    assert a.min() >= -1e-15 and b.min() >= -1e-15
    np.testing.assert_allclose(s ** 2, np.linalg.eigvalsh(A.T @ A)[-1], rtol=1e-12)
    # Frobenius optimality of the leading term
    np.testing.assert_allclose(np.sum((A - s * np.outer(a, b)) ** 2), np.sum(A ** 2) - s ** 2,
                               atol=1e-12 * np.sum(A ** 2))
    assert ods.rank1(np.zeros((4, 3)))[0] == 0.0


def _w_hat(W, r, npaths=2):
    return sum(p["W_hat"] for p in ods.littlebit_init(W, r, npaths))


def test_symmetries():
    rng = np.random.default_rng(5)
    W = synth.dense_weight(14, 24, 40).astype(np.float64)
    r = 5
    ref = _w_hat(W, r)
    tol = 1e-11 * np.abs(ref).max()
    np.testing.assert_allclose(_w_hat(2.0 * W, r), 2.0 * ref, atol=2 * tol, rtol=0)
    np.testing.assert_allclose(_w_hat(-W, r), -ref, atol=tol, rtol=0)
    np.testing.assert_allclose(_w_hat(W.T, r), ref.T, atol=tol, rtol=0)
    P, Q = rng.permutation(24), rng.permutation(40)
    np.testing.assert_allclose(_w_hat(W[P][:, Q], r), ref[P][:, Q], atol=tol, rtol=0)
    D = np.where(rng.random(24) < 0.5, -1.0, 1.0)
    np.testing.assert_allclose(_w_hat(D[:, None] * W, r), D[:, None] * ref, atol=tol, rtol=0)


def test_scales_are_nonnegative_and_the_residual_path_reduces_the_error():
    W = synth.dense_weight(15, 64, 96).astype(np.float64)
    pri, res = ods.littlebit_init(W, 8, 2)
    for p in (pri, res):
        assert p["h"].min() >= -1e-15 and p["g"].min() >= -1e-15 and p["l"].min() >= -1e-15
    e0 = np.linalg.norm(W)
    e1 = np.linalg.norm(W - pri["W_hat"])
    e2 = np.linalg.norm(W - pri["W_hat"] - res["W_hat"])
    assert e2 < e1 < e0


def test_pack_rows_matches_the_bitwise_packer():
    from oracle import pack_signs
    rng = np.random.default_rng(3)
    S = np.where(rng.random((7, 45)) < 0.5, -1.0, 1.0)
    np.testing.assert_array_equal(ods.pack_rows(S).ravel(), pack_signs(S.astype(np.float32)).ravel())


def test_a_planted_unbalanced_split_is_caught(monkeypatch):
    # Planting U' = U S, V' = V (singular values all on one side) in the oracle breaks the transposition symmetry
    # and the hand-derived cases: the pins above would catch that mistake.
    def unbalanced(W, r):
        U, s, Vt = np.linalg.svd(np.asarray(W, np.float64), full_matrices=False)
        return U[:, :r] * s[:r], Vt[:r].T.copy(), s[:r]
    W = synth.dense_weight(14, 24, 40).astype(np.float64)
    good = _w_hat(W.T, 5)
    monkeypatch.setattr(ods, "truncated_svd_factors", unbalanced)
    assert np.abs(_w_hat(W.T, 5) - _w_hat(W, 5).T).max() > 1e-6 * np.abs(good).max()
