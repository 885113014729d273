"""CPU oracle of the LittleBit initialisation: Dual-SVID and residual compensation.

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import it; the CUDA library never does, and the two
share no code.  Plain numpy in float64; the truncated SVD and the rank-1 SVD
are LAPACK's (``numpy.linalg.svd``), used as library steps.

What it computes (LittleBit paper notes page, "Dual-SVID initialisation" and
"Residual compensation"; the framework steps 1-3 of "Overall framework"):

1. Truncated SVD of W (N x K) to rank r gives factors U' (N x r), V' (K x r)
   with U' V'^T the best rank-r approximation of W.
2. The binary factors are the signs: U_sign = sign(U'), V_sign = sign(V').
3. Each magnitude matrix |U'| and |V'| gets its own rank-1 SVD; the singular
   vectors and values become the row scale h, the column scale g and the
   latent scale l, so that
   W_hat = diag(h) U_sign diag(l) V_sign^T diag(g)  approximates  U' V'^T.
4. The residual path runs the same procedure on W - W_hat_pri.

Readings of points the notes leave open (the same readings as the CUDA path):

* U' = U_r diag(sqrt(s)), V' = V_r diag(sqrt(s)): the r singular values are
  split evenly between the two factors, the plainest way to obtain the
  ``W ~ U V^T`` of framework step 1 from an SVD.
* The sign of each singular pair is fixed so that the entry of largest
  magnitude in each column of U' is positive (first such index on ties).
  W_hat does not depend on this choice (flipping a column of both U' and V'
  leaves the product and both magnitudes unchanged); it only makes the sign
  factors unique.
* sign(0) = +1 (the packing convention of the library: bit set <=> value < 0).
* Rank-1 SVD of a magnitude matrix A: A ~ s_A a b^T with unit a, b chosen
  non-negative (the Perron vectors of a non-negative matrix; the pair is
  flipped when its entries sum below zero).  From |U'| ~ s_u a_u b_u^T and
  |V'| ~ s_v a_v b_v^T:  h = a_u, g = a_v, l = s_u s_v (b_u (.) b_v).  When
  A is zero, s_A = 0 and a = b = 0.
* Both paths have the same rank r; r <= min(N, K).
"""

from __future__ import annotations

import numpy as np


def signs(F: np.ndarray) -> np.ndarray:
    """+-1 factor of F with sign(0) = +1 (and -0.0 -> +1): -1 exactly where F < 0."""
    return np.where(np.asarray(F) < 0, -1.0, 1.0)


def truncated_svd_factors(W: np.ndarray, r: int):
    """(U', V', s): top-r singular pairs of W, singular values split evenly, canonical column signs.

    Step 1 of Dual-SVID (paper notes page, "Dual-SVID initialisation").
    """
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    if not 1 <= r <= min(N, K):
        raise ValueError("rank must be in [1, min(N, K)]")
    U, s, Vt = np.linalg.svd(W, full_matrices=False)
    U, s, V = U[:, :r], s[:r], Vt[:r].T
    root = np.sqrt(s)
    Up = U * root
    Vp = V * root
    for j in range(r):
        i = int(np.argmax(np.abs(Up[:, j])))
        if Up[i, j] < 0:
            Up[:, j] = -Up[:, j]
            Vp[:, j] = -Vp[:, j]
    return Up, Vp, s


def rank1(A: np.ndarray):
    """(s, a, b): leading singular triplet of a non-negative matrix, a and b non-negative unit vectors.

    Step 3 of Dual-SVID; A = 0 gives (0, 0, 0).
    """
    A = np.asarray(A, dtype=np.float64)
    U, s, Vt = np.linalg.svd(A, full_matrices=False)
    if s[0] == 0.0:
        return 0.0, np.zeros(A.shape[0]), np.zeros(A.shape[1])
    a, b = U[:, 0].copy(), Vt[0].copy()
    if b.sum() < 0:
        a, b = -a, -b
    return float(s[0]), a, b


def dual_svid(W: np.ndarray, r: int) -> dict:
    """One path: sign factors (+-1 float64), scales h (N), g (K), l (r), the effective weight and diagnostics."""
    Up, Vp, s = truncated_svd_factors(W, r)
    U_sign, V_sign = signs(Up), signs(Vp)
    s_u, a_u, b_u = rank1(np.abs(Up))
    s_v, a_v, b_v = rank1(np.abs(Vp))
    h, g, l = a_u, a_v, s_u * s_v * (b_u * b_v)
    return {"U_sign": U_sign, "V_sign": V_sign, "h": h, "g": g, "l": l, "sigma": s,
            "U_prime": Up, "V_prime": Vp, "W_hat": effective_weight(U_sign, V_sign, h, g, l)}


def effective_weight(U_sign, V_sign, h, g, l) -> np.ndarray:
    """diag(h) U_sign diag(l) V_sign^T diag(g) (paper notes page, "Multi-scale compensation")."""
    U_sign, V_sign = np.asarray(U_sign, np.float64), np.asarray(V_sign, np.float64)
    return (np.asarray(h, np.float64)[:, None] * (U_sign * np.asarray(l, np.float64)[None, :])) @ \
        (V_sign * np.asarray(g, np.float64)[:, None]).T


def littlebit_init(W: np.ndarray, r: int, npaths: int = 2) -> list:
    """Primary path by Dual-SVID of W; the residual path by Dual-SVID of W - W_hat_pri.

    Paper notes page, "Residual compensation".
    """
    if npaths not in (1, 2):
        raise ValueError("npaths must be 1 or 2")
    target = np.asarray(W, dtype=np.float64)
    paths = []
    for _ in range(npaths):
        p = dual_svid(target, r)
        paths.append(p)
        target = target - p["W_hat"]
    return paths


def pack_rows(S: np.ndarray) -> np.ndarray:
    """Canonical packed words of a +-1 matrix (rows x r): word [i, j // 32], bit j % 32 set <=> S[i, j] < 0."""
    S = np.asarray(S)
    rows, r = S.shape
    wpr = (r + 31) // 32
    out = np.zeros((rows, wpr), dtype=np.uint32)
    for j in range(r):
        out[:, j // 32] |= (S[:, j] < 0).astype(np.uint32) << np.uint32(j % 32)
    return out
