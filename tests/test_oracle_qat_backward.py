"""Pins of the QAT backward oracle (oracle/qat_backward.py), from outside it.

CPU only.  The layer output y is linear in each of x, h, g, l and in each
entry of the sign factors, so for L = <dy, y> a finite difference taken with
the (separately pinned) C forward oracle is exact up to float64 rounding:
replace one binary16 / bfloat16 value by another, or flip one sign bit (a
change of -2 in U_s[n, j]).  The SmoothSign factor is checked against a
central difference of tanh(100 u); dx against the forward pass of the
transposed layer (U <-> V, h <-> g) applied to dy.  Source: LittleBit paper
notes page, "Multi-scale compensation" and "Loss / training strategy".
"""

import numpy as np
import pytest

import oracle
from oracle import qat_backward as qb
from sub_bit_weight_b200 import synth


def _case(seed=3, N=12, K=10, r=3, M=4, npaths=2):
    rng = np.random.default_rng(seed)
    U = [rng.normal(0, 0.02, (N, r)).astype(np.float32) for _ in range(npaths)]
    V = [rng.normal(0, 0.02, (K, r)).astype(np.float32) for _ in range(npaths)]
    U[0][0, 0] = 0.0                       # sign(0) = +1
    h = [rng.lognormal(-3, 0.5, N).astype(np.float16) for _ in range(npaths)]
    g = [rng.lognormal(-3, 0.5, K).astype(np.float16) for _ in range(npaths)]
    l = [rng.lognormal(-3, 0.5, r).astype(np.float16) for _ in range(npaths)]
    xb = synth.f32_to_bf16_bits(rng.standard_normal((M, K)).astype(np.float32))
    dyb = synth.f32_to_bf16_bits(rng.standard_normal((M, N)).astype(np.float32))
    return dict(N=N, K=K, r=r, M=M, U=U, V=V, h=h, g=g, l=l, xb=xb, dyb=dyb)


def _layer(c, U=None, V=None, h=None, g=None, l=None):
    U, V = U or c["U"], V or c["V"]
    h, g, l = h or c["h"], g or c["g"], l or c["l"]
    return {"N": U[0].shape[0], "K": V[0].shape[0], "r": c["r"],
            "U": [oracle.pack_signs(u) for u in U], "V": [oracle.pack_signs(v) for v in V],
            "h": [np.asarray(v, np.float16).view(np.uint16) for v in h],
            "g": [np.asarray(v, np.float16).view(np.uint16) for v in g],
            "l": [np.asarray(v, np.float16).view(np.uint16) for v in l]}


def _loss(c, xb, **kw):
    dy = synth.bf16_bits_to_f32(c["dyb"]).astype(np.float64)
    return float(np.sum(dy * oracle.forward(xb, _layer(c, **kw))))


def _grads(c):
    x = synth.bf16_bits_to_f32(c["xb"])
    dy = synth.bf16_bits_to_f32(c["dyb"])
    f = lambda L: [np.asarray(v, np.float64) for v in L]
    return qb.backward(x, dy, c["U"], c["V"], f(c["h"]), f(c["g"]), f(c["l"]))


def _other_half(v):
    """A different binary16 value near v (the next code up)."""
    return np.float16(np.frombuffer(np.array([np.float16(v).view(np.uint16) + 1], np.uint16).tobytes(), np.float16)[0])


def test_scale_gradients_by_exact_finite_differences():
    c = _case()
    gr = _grads(c)
    base = _loss(c, c["xb"])
    for p in range(2):
        for name, key in (("h", "dh"), ("g", "dg"), ("l", "dl")):
            vec = c[name][p]
            for i in range(vec.size):
                new = [v.copy() for v in c[name]]
                new[p][i] = _other_half(vec[i])
                delta = float(new[p][i]) - float(vec[i])
                fd = (_loss(c, c["xb"], **{name: new}) - base) / delta
                assert abs(fd - gr[key][p][i]) <= 1e-9 * (abs(fd) + 1e-3), (name, p, i, fd, gr[key][p][i])


def test_sign_factor_gradients_by_flipping_one_sign():
    c = _case()
    gr = _grads(c)
    base = _loss(c, c["xb"])
    for p in range(2):
        for name, key in (("U", "dU_s"), ("V", "dV_s")):
            F = c[name][p]
            for i in range(F.shape[0]):
                for j in range(F.shape[1]):
                    new = [v.copy() for v in c[name]]
                    new[p][i, j] = -new[p][i, j] if new[p][i, j] != 0 else np.float32(-1.0)
                    delta = -2.0 if F[i, j] >= 0 else 2.0          # the sign entry moves from +1 to -1 or back
                    fd = (_loss(c, c["xb"], **{name: new}) - base) / delta
                    assert abs(fd - gr[key][p][i, j]) <= 1e-9 * (abs(fd) + 1e-3), (name, p, i, j)
            sg = qb.smooth_sign_grad(F)
            np.testing.assert_allclose(gr["dU" if name == "U" else "dV"][p], gr[key][p] * sg, rtol=1e-15)


def test_input_gradient_by_exact_finite_differences():
    c = _case()
    gr = _grads(c)
    base = _loss(c, c["xb"])
    x = synth.bf16_bits_to_f32(c["xb"])
    for m in range(c["M"]):
        for k in range(c["K"]):
            xb = c["xb"].copy()
            xb[m, k] += 1                                        # next bfloat16 code
            delta = float(synth.bf16_bits_to_f32(xb)[m, k]) - float(x[m, k])
            fd = (_loss(c, xb) - base) / delta
            assert abs(fd - gr["dx"][m, k]) <= 1e-9 * (abs(fd) + 1e-3), (m, k)


def test_input_gradient_is_the_transposed_layer_applied_to_dy():
    c = _case(seed=8, N=20, K=14, r=4, M=5)
    gr = _grads(c)
    lt = _layer(c, U=c["V"], V=c["U"], h=c["g"], g=c["h"])
    lt["N"], lt["K"] = c["K"], c["N"]
    np.testing.assert_allclose(oracle.forward(c["dyb"], lt), gr["dx"], rtol=0, atol=1e-12 * np.abs(gr["dx"]).max())


@pytest.mark.parametrize("u", [0.0, 3e-3, -3e-3, 1e-2, -0.05, 0.3])
def test_smooth_sign_gradient(u):
    e = 1e-7
    fd = (np.tanh(100 * (u + e)) - np.tanh(100 * (u - e))) / (2 * e)
    assert abs(qb.smooth_sign_grad(np.array(u)) - fd) <= 1e-6 * max(1.0, abs(fd))
    assert qb.smooth_sign_grad(np.array(0.0)) == 100.0


def test_zero_output_gradient_gives_zero_gradients():
    c = _case()
    c["dyb"] = np.zeros_like(c["dyb"])
    gr = _grads(c)
    assert np.abs(gr["dx"]).max() == 0.0
    for key in ("dh", "dg", "dl", "dU", "dV"):
        assert all(np.abs(v).max() == 0.0 for v in gr[key])
