"""Full-size workloads, in the launch configuration the benchmark times.

Each workload's whole stack runs through lb_stack_forward; the oracle then
computes sampled outputs one by one (every activation row for decode, a seeded
sample of rows for prefill; a seeded sample of output columns) for one layer
of every shape at the first and last block plus a few random layers.
"""

import numpy as np
import pytest

import oracle
from sub_bit_weight_b200 import synth
from tests._util import TOL, oracle_layer, rel_err

pytestmark = pytest.mark.gpu


def _sample_layers(w, rng, extra=4):
    nb = len(w.block)
    idx = set(range(nb)) | set(range((w.nblocks - 1) * nb, w.nblocks * nb))
    total = w.nblocks * nb
    idx |= set(int(i) for i in rng.choice(total, size=min(extra, total), replace=False))
    return sorted(idx)


def _run_workload(key, M):
    import torch
    from sub_bit_weight_b200 import lib, stacks
    w = synth.WORKLOADS[key]
    layers, shapes = stacks.build_workload(w)
    xs, ys = stacks.workload_activations(w, shapes, M)
    S = lib.lb_stack_create(layers)
    for _ in range(2):                       # warm state, then the checked pass
        lib.lb_stack_forward(S, xs, ys)
    torch.cuda.synchronize()
    rng = np.random.default_rng(1234)
    pools = {}
    worst = 0.0
    for idx in _sample_layers(w, rng):
        s = shapes[idx]
        xb = synth.layer_activations(w, idx, M, s.K, pools)
        ms = np.arange(M) if M <= 16 else np.sort(rng.choice(M, size=8, replace=False))
        ns = np.sort(rng.choice(s.N, size=min(s.N, 192), replace=False))
        ref = oracle.forward_sampled(np.ascontiguousarray(xb), oracle_layer(w.seed, idx, s), ms, ns)
        got = ys[idx].cpu().numpy()[np.ix_(ms, ns)]
        err = rel_err(got, ref)
        worst = max(worst, err)
        assert err <= TOL, (key, idx, s, err)
    print(f"{key} M={M}: worst sampled rel_err {worst:.3e}")
    del S, layers, xs, ys
    torch.cuda.empty_cache()


@pytest.mark.parametrize("M", [1, 8])
def test_single_512(M):
    _run_workload("single_512", M)


def test_llama2_7b_0p1_decode():
    _run_workload("llama2_7b_0.1", 1)


@pytest.mark.parametrize("M", [1, 4, 16])
def test_llama2_7b_0p55(M):
    _run_workload("llama2_7b_0.55", M)


def test_llama2_13b_0p3_prefill():
    _run_workload("llama2_13b_0.3_prefill", 2048)


def test_llama2_70b_0p1_decode():
    _run_workload("llama2_70b_0.1", 1)
