"""CPU oracle of the LittleBit layer's backward pass for quantisation-aware training (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``
may import it; the CUDA library never does, and the two share no code.  Plain
numpy in float64 (matrix products are numpy's, used as library steps).

What it computes.  The forward pass of one path (LittleBit paper notes page,
"Multi-scale compensation") is

    t = x (.) g,  z = t V_s,  zl = z (.) l,  s = zl U_s^T,  y = sum_paths h (.) s,

with U_s = sign(U), V_s = sign(V) of the latent full-precision factors U, V.
QAT trains U, V, h, g, l; the sign's gradient is replaced by SmoothSign's
(same page, "Loss / training strategy": forward sign, backward tanh(100 u)),
i.e. d sign(u)/du := 100 (1 - tanh^2(100 u)).  Given dy = dL/dy the chain rule
through the same sequence gives, per path,

    ds = dy (.) h            dh = sum_m dy (.) s
    dzl = ds U_s             dU_s = ds^T zl          dU = dU_s (.) 100 (1 - tanh^2(100 U))
    dl = sum_m dzl (.) z     dz = dzl (.) l
    dt = dz V_s^T            dV_s = t^T dz           dV = dV_s (.) 100 (1 - tanh^2(100 V))
    dg = sum_m dt (.) x      dx = sum_paths dt (.) g

Readings (the pages give no more): the scales in the backward are the layer's
stored binary16 values (the ones its forward pass used); x is bfloat16 and dy
float32, both widened exactly; sign(0) = +1.
"""

from __future__ import annotations

import numpy as np


def smooth_sign_grad(u: np.ndarray) -> np.ndarray:
    """d/du tanh(100 u) = 100 (1 - tanh^2(100 u)): the SmoothSign surrogate gradient of sign(u)."""
    t = np.tanh(100.0 * np.asarray(u, dtype=np.float64))
    return 100.0 * (1.0 - t * t)


def signs(F: np.ndarray) -> np.ndarray:
    """+-1 with sign(0) = +1 (and -0.0 -> +1): -1 exactly where F < 0."""
    return np.where(np.asarray(F) < 0, -1.0, 1.0)


def forward(x, U_lat, V_lat, h, g, l):
    """y [M, N] and the per-path intermediates (t, z, zl, s) of the forward pass, float64."""
    x = np.asarray(x, dtype=np.float64)
    y = 0.0
    inter = []
    for p in range(len(U_lat)):
        Us, Vs = signs(U_lat[p]), signs(V_lat[p])
        t = x * np.asarray(g[p], np.float64)[None, :]
        z = t @ Vs
        zl = z * np.asarray(l[p], np.float64)[None, :]
        s = zl @ Us.T
        y = y + np.asarray(h[p], np.float64)[None, :] * s
        inter.append({"t": t, "z": z, "zl": zl, "s": s, "Us": Us, "Vs": Vs})
    return y, inter


def backward(x, dy, U_lat, V_lat, h, g, l) -> dict:
    """dx [M, K] and per-path lists dh [N], dg [K], dl [r], dU [N, r], dV [K, r] (also dU_s, dV_s), float64."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    _, inter = forward(x, U_lat, V_lat, h, g, l)
    out = {"dx": np.zeros_like(x), "dh": [], "dg": [], "dl": [], "dU": [], "dV": [], "dU_s": [], "dV_s": []}
    for p, it in enumerate(inter):
        hp, gp, lp = (np.asarray(v[p], np.float64) for v in (h, g, l))
        ds = dy * hp[None, :]
        dh = np.sum(dy * it["s"], axis=0)
        dzl = ds @ it["Us"]
        dU_s = ds.T @ it["zl"]
        dl = np.sum(dzl * it["z"], axis=0)
        dz = dzl * lp[None, :]
        dt = dz @ it["Vs"].T
        dV_s = it["t"].T @ dz
        dg = np.sum(dt * x, axis=0)
        out["dx"] += dt * gp[None, :]
        out["dh"].append(dh)
        out["dg"].append(dg)
        out["dl"].append(dl)
        out["dU_s"].append(dU_s)
        out["dV_s"].append(dV_s)
        out["dU"].append(dU_s * smooth_sign_grad(U_lat[p]))
        out["dV"].append(dV_s * smooth_sign_grad(V_lat[p]))
    return out
