"""Seeded synthetic inputs for LittleBit compressed linear layers.

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle: it draws the inputs, and holds none of the layer's arithmetic.

Recipe (the value distributions of the workloads this library is measured on):

* Factor signs: i.i.d. Bernoulli(0.5) over +-1.  Sign bits come from a
  counter-based generator, SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): output n of a stream with key
  k is ``mix64(k + (n + 1) * 0x9E3779B97F4A7C15)``.  Word n of row i covers
  columns ``64 * (n % W64) ... +63`` of that row (``W64 = ceil(r / 64)``), bit b
  of the word is column ``64 * (n % W64) + b``, and a set bit means -1.  Any
  block of rows can therefore be drawn on its own, which lets full-size layers
  be checked element by element.
* Scales h, g, l: lognormal(mu=-3, sigma=0.5), rounded to IEEE binary16 (round
  to nearest even), from ``numpy.random.default_rng([seed, layer, path, kind])``.
* Activations x: N(0, 1) in float32, rounded to bfloat16 (round to nearest
  even), from ``default_rng([seed, layer, 0x7878])``.  The prefill workload
  uses rows of a shared pool (see ``activation_pool``).

Stream keys are derived from (seed, layer index, path, matrix) by chaining
``mix64``; seeds are the workload index unless stated otherwise.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

_GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1

PATH_PRI, PATH_RES = 0, 1
MAT_U, MAT_V = 0, 1
_KIND = {"h": 1, "g": 2, "l": 3}


def _mix64_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z = z * np.uint64(0xBF58476D1CE4E5B9)
    z = z ^ (z >> np.uint64(27))
    z = z * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(*parts: int) -> int:
    k = 0
    for p in parts:
        k = _mix64_int((k ^ (int(p) & _M64)) + _GOLDEN)
    return k


def splitmix64(key: int, counters: np.ndarray) -> np.ndarray:
    """SplitMix64 outputs number ``counters`` of the stream with this key."""
    n = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key) + (n + np.uint64(1)) * np.uint64(_GOLDEN)
        return _mix64(state)


def sign_words(seed: int, layer: int, path: int, mat: int, r: int, row0: int, row1: int) -> np.ndarray:
    """Sign words of rows [row0, row1) of one factor: uint64 [rows, ceil(r/64)]."""
    w64 = (r + 63) // 64
    rows = np.arange(row0, row1, dtype=np.uint64)
    n = rows[:, None] * np.uint64(w64) + np.arange(w64, dtype=np.uint64)[None, :]
    return splitmix64(stream_key(seed, layer, path, mat), n)


def words_to_negative(words: np.ndarray, r: int) -> np.ndarray:
    """Boolean [rows, r]: True where the sign is -1."""
    words = np.ascontiguousarray(words, dtype="<u8")
    bits = np.unpackbits(words.view(np.uint8), axis=1, bitorder="little")
    return bits[:, :r].astype(bool)


def sign_factor(seed: int, layer: int, path: int, mat: int, rows: int, r: int,
                row0: int = 0, row1: int | None = None) -> np.ndarray:
    """float32 +-1 factor rows [row0, row1) (all rows by default), shape [rows, r]."""
    row1 = rows if row1 is None else row1
    neg = words_to_negative(sign_words(seed, layer, path, mat, r, row0, row1), r)
    return np.where(neg, np.float32(-1.0), np.float32(1.0)).astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def scale_vector(seed: int, layer: int, path: int, kind: str, n: int) -> np.ndarray:
    """binary16 bit patterns (uint16) of a lognormal(-3, 0.5) scale vector."""
    rng = np.random.default_rng([seed, layer, path, _KIND[kind]])
    v = rng.lognormal(mean=-3.0, sigma=0.5, size=n)
    return v.astype(np.float16).view(np.uint16)


def activations(seed: int, layer: int, M: int, K: int) -> np.ndarray:
    """bfloat16 bit patterns [M, K] drawn from N(0, 1)."""
    rng = np.random.default_rng([seed, layer, 0x7878])
    return f32_to_bf16_bits(rng.standard_normal(M * K, dtype=np.float32)).reshape(M, K)


def activation_pool(seed: int, K: int, rows: int) -> np.ndarray:
    """A [rows, K] pool of N(0, 1) bfloat16 rows shared by a prefill stack."""
    rng = np.random.default_rng([seed, K, 0x9001])
    return f32_to_bf16_bits(rng.standard_normal(rows * K, dtype=np.float32)).reshape(rows, K)


# ---------------------------------------------------------------------------
# Workload shapes
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerShape:
    name: str
    N: int   # output features (rows of W, rows of U_sign)
    K: int   # input features (columns of W, rows of V_sign)
    r: int   # latent rank of each path


@dataclass(frozen=True)
class Workload:
    key: str
    title: str
    block: tuple          # LayerShape per block
    nblocks: int
    Ms: tuple
    seed: int
    pool_rows: int = 0    # >0: activations are windows of a shared pool
    notes: str = ""
    extra: dict = field(default_factory=dict)

    def layers(self):
        """(layer index, LayerShape) for every layer of the stack, in order."""
        out = []
        for b in range(self.nblocks):
            for s in self.block:
                out.append((len(out), s))
        return out


WORKLOADS = {
    "single_512": Workload(
        "single_512", "single layer 512x512, r=16, two paths",
        (LayerShape("single", 512, 512, 16),), 1, (1, 8), seed=0),
    "llama2_7b_0.1": Workload(
        "llama2_7b_0.1", "Llama-2-7B-shaped decode stack at ~0.1 BPW",
        (LayerShape("q", 4096, 4096, 80), LayerShape("k", 4096, 4096, 80),
         LayerShape("v", 4096, 4096, 80), LayerShape("o", 4096, 4096, 80),
         LayerShape("gate", 11008, 4096, 128), LayerShape("up", 11008, 4096, 128),
         LayerShape("down", 4096, 11008, 128)), 32, (1,), seed=1),
    "llama2_7b_0.55": Workload(
        "llama2_7b_0.55", "Llama-2-7B-shaped stack at ~0.55 BPW",
        (LayerShape("q", 4096, 4096, 544), LayerShape("k", 4096, 4096, 544),
         LayerShape("v", 4096, 4096, 544), LayerShape("o", 4096, 4096, 544),
         LayerShape("gate", 11008, 4096, 800), LayerShape("up", 11008, 4096, 800),
         LayerShape("down", 4096, 11008, 800)), 32, (1, 4, 16), seed=2),
    "llama2_13b_0.3_prefill": Workload(
        "llama2_13b_0.3_prefill", "Llama-2-13B-shaped prefill stack at ~0.3 BPW",
        (LayerShape("q", 5120, 5120, 368), LayerShape("k", 5120, 5120, 368),
         LayerShape("v", 5120, 5120, 368), LayerShape("o", 5120, 5120, 368),
         LayerShape("gate", 13824, 5120, 544), LayerShape("up", 13824, 5120, 544),
         LayerShape("down", 5120, 13824, 544)), 40, (2048,), seed=3, pool_rows=8 * 2048),
    "llama2_70b_0.1": Workload(
        "llama2_70b_0.1", "Llama-2-70B-shaped decode stack at ~0.1 BPW (exceeds L2)",
        (LayerShape("q", 8192, 8192, 184), LayerShape("k", 1024, 8192, 32),
         LayerShape("v", 1024, 8192, 32), LayerShape("o", 8192, 8192, 184),
         LayerShape("gate", 28672, 8192, 304), LayerShape("up", 28672, 8192, 304),
         LayerShape("down", 8192, 28672, 304)), 80, (1,), seed=4),
}


def layer_activations(w: Workload, layer: int, M: int, K: int, pools: dict | None = None) -> np.ndarray:
    """Activations of one layer of a workload.

    Decode stacks draw their own x per layer.  The prefill stack takes rows
    ``[(layer % 8) * M, +M)`` of a pool of ``pool_rows`` rows of width K, so
    consecutive layers read disjoint windows.
    """
    if not w.pool_rows:
        return activations(w.seed, layer, M, K)
    if pools is None or K not in pools:
        pool = activation_pool(w.seed, K, w.pool_rows)
        if pools is not None:
            pools[K] = pool
    else:
        pool = pools[K]
    nwin = max(1, w.pool_rows // M)
    o = (layer % nwin) * M
    return pool[o:o + M]


def layer_inputs(seed: int, layer: int, shape: LayerShape, npaths: int = 2) -> dict:
    """Factors (float32 +-1) and scales (binary16 bits) of one layer."""
    N, K, r = shape.N, shape.K, shape.r
    out = {"N": N, "K": K, "r": r, "F_U": [], "F_V": [], "h": [], "g": [], "l": []}
    for p in range(npaths):
        out["F_U"].append(sign_factor(seed, layer, p, MAT_U, N, r))
        out["F_V"].append(sign_factor(seed, layer, p, MAT_V, K, r))
        out["h"].append(scale_vector(seed, layer, p, "h", N))
        out["g"].append(scale_vector(seed, layer, p, "g", K))
        out["l"].append(scale_vector(seed, layer, p, "l", r))
    return out


def dense_weight(seed: int, N: int, K: int, alpha: float = 1.0, rms: float = 0.02) -> np.ndarray:
    """Synthetic dense weight W [N, K] (float32 holding bfloat16 values) with a power-law spectrum.

    ``W = A diag(s) B`` with A [N, R], B [R, K] i.i.d. N(0, 1) in float32
    (``R = min(N, K)``, from ``default_rng([seed, N, K, 0x5D])``, A drawn
    first) and ``s_i = (i + 1) ** -alpha``; scaled so that the RMS entry is
    ``rms`` (the magnitude of LLM projection weights) and rounded to bfloat16
    (nearest even), the storage type of such weights.  The decaying spectrum
    stands for the low-rank structure of LLM weight matrices that the
    factorisation relies on.
    """
    rng = np.random.default_rng([seed, N, K, 0x5D])
    R = min(N, K)
    A = rng.standard_normal((N, R), dtype=np.float32)
    B = rng.standard_normal((R, K), dtype=np.float32)
    s = (np.arange(1, R + 1, dtype=np.float64) ** -float(alpha)).astype(np.float32)
    W = (A * s[None, :]) @ B
    W *= np.float32(rms / np.sqrt(np.mean(np.square(W, dtype=np.float64))))
    return bf16_bits_to_f32(f32_to_bf16_bits(W))


def random_rotation(seed: int, r: int, path: int = 0) -> np.ndarray:
    """A seeded random orthogonal r x r matrix (float64), the random start of an iterative-quantisation rotation.

    The Q factor of a QR decomposition of an i.i.d. N(0, 1) matrix from
    ``default_rng([seed, r, path, 0x17])``, its columns signed so that R's
    diagonal is positive (Haar-distributed).  A random draw of the method, made
    here and handed to both sides as an input.
    """
    rng = np.random.default_rng([seed, r, path, 0x17])
    Q, Rq = np.linalg.qr(rng.standard_normal((r, r)))
    return np.ascontiguousarray(Q * np.where(np.diag(Rq) < 0, -1.0, 1.0)[None, :])
