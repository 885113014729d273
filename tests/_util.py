"""Helpers shared by the tests (oracle inputs, error metric, GPU detection)."""

import numpy as np

import oracle
from sub_bit_weight_b200 import synth

TOL = 2e-3   # max|y_gpu - y_ref| / max|y_ref| per layer (workload definition)


def oracle_layer(seed, layer, shape, npaths=2):
    """Host description of one synthetic layer for the CPU oracle, packed by the oracle's own packer."""
    inp = synth.layer_inputs(seed, layer, shape, npaths)
    inp["U"] = [oracle.pack_signs(F) for F in inp.pop("F_U")]
    inp["V"] = [oracle.pack_signs(F) for F in inp.pop("F_V")]
    return inp


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    num = np.max(np.abs(y - ref))
    return num / den if den > 0 else num
