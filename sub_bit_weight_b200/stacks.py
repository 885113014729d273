"""Put synthetic LittleBit layers and activations on the device.

Plumbing shared by the benchmark and the GPU tests: inputs come from
``synth`` (the seeded generator), factors are expanded to float32 +-1 on the
device with PyTorch, binarised by ``lb_pack_signs`` and handed to
``lb_layer_create``.
"""

from __future__ import annotations

import numpy as np
import torch

from . import lib, synth

_SHIFTS = {}


def _shifts(device):
    key = str(device)
    if key not in _SHIFTS:
        _SHIFTS[key] = torch.arange(64, dtype=torch.int64, device=device)
    return _SHIFTS[key]


def factor_on_device(seed: int, layer: int, path: int, mat: int, rows: int, r: int, device) -> torch.Tensor:
    """float32 +-1 factor [rows, r] with the generator's signs (bit set = -1)."""
    words = synth.sign_words(seed, layer, path, mat, r, 0, rows).view(np.int64)
    w = torch.from_numpy(np.ascontiguousarray(words)).to(device, non_blocking=False)
    bits = (w.unsqueeze(-1) >> _shifts(device)) & 1                  # [rows, W64, 64]
    bits = bits.reshape(rows, -1)[:, :r]
    return (1.0 - 2.0 * bits.to(torch.float32)).contiguous()


def half_on_device(bits_u16: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).to(device).view(torch.float16)


def bf16_on_device(bits_u16: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits_u16).view(np.int16)).to(device).view(torch.bfloat16)


def build_layer(seed: int, layer: int, shape: synth.LayerShape, npaths: int = 2, device="cuda") -> lib.Layer:
    N, K, r = shape.N, shape.K, shape.r
    U, V, h, g, l = [], [], [], [], []
    for p in range(npaths):
        U.append(lib.lb_pack_signs(factor_on_device(seed, layer, p, synth.MAT_U, N, r, device)))
        V.append(lib.lb_pack_signs(factor_on_device(seed, layer, p, synth.MAT_V, K, r, device)))
        h.append(half_on_device(synth.scale_vector(seed, layer, p, "h", N), device))
        g.append(half_on_device(synth.scale_vector(seed, layer, p, "g", K), device))
        l.append(half_on_device(synth.scale_vector(seed, layer, p, "l", r), device))
    L = lib.lb_layer_create(N, K, r, U, V, h, g, l)
    torch.cuda.current_stream().synchronize()
    return L


def build_workload(w: synth.Workload, device="cuda", nblocks: int | None = None):
    """Layers of a workload (optionally only its first ``nblocks`` blocks) and its shapes."""
    layers, shapes = [], []
    for idx, shape in w.layers():
        if nblocks is not None and idx >= nblocks * len(w.block):
            break
        layers.append(build_layer(w.seed, idx, shape, device=device))
        shapes.append(shape)
    return layers, shapes


def workload_activations(w: synth.Workload, shapes, M: int, device="cuda"):
    """Per-layer x (bfloat16, device) and y (float32, device) buffers."""
    xs, ys = [], []
    if w.pool_rows:
        pools = {}
        dev_pools = {}
        for idx, s in enumerate(shapes):
            if s.K not in dev_pools:
                pool = synth.activation_pool(w.seed, s.K, w.pool_rows)
                pools[s.K] = pool
                dev_pools[s.K] = bf16_on_device(pool, device)
            nwin = max(1, w.pool_rows // M)
            o = (idx % nwin) * M
            xs.append(dev_pools[s.K][o:o + M])
    else:
        for idx, s in enumerate(shapes):
            xs.append(bf16_on_device(synth.layer_activations(w, idx, M, s.K), device))
    for s in shapes:
        ys.append(torch.empty((M, s.N), dtype=torch.float32, device=device))
    return xs, ys

