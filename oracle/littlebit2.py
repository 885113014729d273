"""CPU oracle of the LittleBit-2 initialisation: latent rotation by Joint-ITQ before Dual-SVID's binarisation.

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import it; the CUDA library never does, and the two
share no code.  Plain numpy in float64; SVDs are LAPACK's
(``numpy.linalg.svd``), used as library steps.

What it computes (wiki page on LittleBit and LittleBit-2, section 1, "What
happened": the second paper rotates the latent space and runs a joint
iterative quantisation (Joint-ITQ) before quantisation-aware training, to
align the factors with the binary hypercube; only the initialisation
changes, inference does not).  The truncated SVD gives U' (N x r) and V'
(K x r) with U' V'^T the rank-r approximation of W (LittleBit paper notes
page, "Dual-SVID initialisation").  For any orthogonal r x r matrix R,
(U' R)(V' R)^T = U' V'^T, so a rotation of the latent space is free; it only
changes which sign patterns the binarisation sees.  Joint-ITQ picks R so that
both rotated factors lie close to the vertices of the hypercube, then the
usual Dual-SVID steps (signs, rank-1 SVDs of the magnitudes, residual path)
run on U' R and V' R.

The pages give no formulas.  Readings (the CUDA path takes the same):

* ITQ is the iterative quantisation of Gong and Lazebnik (CVPR 2011):
  minimise ||B - X R||_F^2 over B in {-1, +1}^(n x r) and orthogonal R by
  alternating (a) B = sign(X R) and (b) the orthogonal Procrustes solution
  R = S T^T for X^T B = S Omega T^T (SVD).  Neither step can raise the loss,
  so the loss sequence never increases.
* "Joint": one R serves both factors (so that the product is preserved),
  and X stacks the two factors' rows, X = [U' / rho_u ; V' / rho_v], each
  factor divided by the root mean square of its entries so that its entries
  compare with the hypercube's +-1 on equal terms and neither factor
  dominates the shared rotation through its size.  A zero factor keeps
  rho = 1.
* sign(0) = +1, as everywhere in this library.
* R starts from a given orthogonal R0 (ITQ's usual start is a random
  rotation; the identity is the deterministic choice); ``iters`` fixed
  alternations.  loss[t] = ||sign(X R_t) - X R_t||_F^2 / ((N + K) r) for the
  rotation R_t after t alternations, t = 0 .. iters.
* After the rotation the column signs are made canonical again (the entry
  of largest magnitude in each column of U' R is positive, first index on
  ties); the effective weight does not depend on this.
"""

from __future__ import annotations

import numpy as np

from . import dual_svid as ods


def procrustes(C: np.ndarray) -> np.ndarray:
    """The orthogonal R maximising trace(R^T C): S T^T for the SVD C = S Omega T^T."""
    S, _, Tt = np.linalg.svd(np.asarray(C, dtype=np.float64))
    return S @ Tt


def itq_data(Up: np.ndarray, Vp: np.ndarray) -> np.ndarray:
    """X = [U' / rho_u ; V' / rho_v]: both factors stacked, each scaled to unit root-mean-square entry."""
    parts = []
    for F in (np.asarray(Up, np.float64), np.asarray(Vp, np.float64)):
        rho = np.sqrt(np.mean(F * F)) if F.size else 0.0
        parts.append(F / rho if rho > 0 else F)
    return np.vstack(parts)


def joint_itq(Up: np.ndarray, Vp: np.ndarray, R0: np.ndarray | None, iters: int):
    """(R, loss): the Joint-ITQ rotation after `iters` alternations from R0 (identity if None) and the loss sequence."""
    X = itq_data(Up, Vp)
    r = X.shape[1]
    R = np.eye(r) if R0 is None else np.array(R0, dtype=np.float64)
    loss = []
    for _ in range(iters):
        Y = X @ R
        B = ods.signs(Y)
        loss.append(float(np.sum((B - Y) ** 2)) / Y.size)
        R = procrustes(X.T @ B)
    Y = X @ R
    loss.append(float(np.sum((ods.signs(Y) - Y) ** 2)) / Y.size)
    return R, np.array(loss)


def canonical_columns(Up: np.ndarray, Vp: np.ndarray):
    """Flip column pairs so that the largest-magnitude entry of each U' column is positive (first index on ties)."""
    Up, Vp = np.array(Up, np.float64), np.array(Vp, np.float64)
    for j in range(Up.shape[1]):
        i = int(np.argmax(np.abs(Up[:, j])))
        if Up[i, j] < 0:
            Up[:, j] = -Up[:, j]
            Vp[:, j] = -Vp[:, j]
    return Up, Vp


def littlebit2_path(W: np.ndarray, r: int, R0: np.ndarray | None, itq_iters: int) -> dict:
    """One path: truncated SVD, Joint-ITQ rotation of both factors, then Dual-SVID's binarisation and scales."""
    Up, Vp, s = ods.truncated_svd_factors(W, r)
    R, loss = joint_itq(Up, Vp, R0, itq_iters)
    Ur, Vr = canonical_columns(Up @ R, Vp @ R)
    U_sign, V_sign = ods.signs(Ur), ods.signs(Vr)
    s_u, a_u, b_u = ods.rank1(np.abs(Ur))
    s_v, a_v, b_v = ods.rank1(np.abs(Vr))
    h, g, l = a_u, a_v, s_u * s_v * (b_u * b_v)
    return {"U_sign": U_sign, "V_sign": V_sign, "h": h, "g": g, "l": l, "sigma": s, "R": R, "itq_loss": loss,
            "U_prime": Ur, "V_prime": Vr, "W_hat": ods.effective_weight(U_sign, V_sign, h, g, l)}


def littlebit2_init(W: np.ndarray, r: int, npaths: int = 2, itq_iters: int = 50, R0s=None) -> list:
    """Primary path from W, residual path from W - W_hat_pri, each rotated by its own Joint-ITQ (R0s[p] or identity).

    LittleBit paper notes page, "Residual compensation", with the rotation of the wiki page's LittleBit-2.
    """
    if npaths not in (1, 2):
        raise ValueError("npaths must be 1 or 2")
    target = np.asarray(W, dtype=np.float64)
    paths = []
    for p in range(npaths):
        path = littlebit2_path(target, r, None if R0s is None else R0s[p], itq_iters)
        paths.append(path)
        target = target - path["W_hat"]
    return paths
