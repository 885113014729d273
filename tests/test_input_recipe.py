"""The synthetic inputs follow their stated recipe (CPU).

The workloads are Llama-2-shaped stacks of LittleBit layers (two paths, one
rank per layer) plus one 512 x 512 layer; their shapes are written out below
by hand.  Inputs are seeded draws: factor signs Bernoulli(0.5) over +-1,
scales h, g, l lognormal(mu = -3, sigma = 0.5) rounded to binary16, and
activations N(0, 1) rounded to bfloat16.  These checks pin the generator to
that recipe (shapes exactly, distributions within a few standard errors of
their sample statistics), independently of the layer arithmetic.
"""

import numpy as np
import pytest

from sub_bit_weight_b200 import synth

# (N, K, r) per layer of one block, blocks, batch sizes, seed
EXPECTED = {
    "single_512": ([(512, 512, 16)], 1, (1, 8), 0),
    "llama2_7b_0.1": ([(4096, 4096, 80)] * 4 + [(11008, 4096, 128)] * 2 + [(4096, 11008, 128)], 32, (1,), 1),
    "llama2_7b_0.55": ([(4096, 4096, 544)] * 4 + [(11008, 4096, 800)] * 2 + [(4096, 11008, 800)], 32, (1, 4, 16), 2),
    "llama2_13b_0.3_prefill": ([(5120, 5120, 368)] * 4 + [(13824, 5120, 544)] * 2 + [(5120, 13824, 544)], 40,
                               (2048,), 3),
    "llama2_70b_0.1": ([(8192, 8192, 184), (1024, 8192, 32), (1024, 8192, 32), (8192, 8192, 184),
                        (28672, 8192, 304), (28672, 8192, 304), (8192, 28672, 304)], 80, (1,), 4),
}


@pytest.mark.parametrize("key", sorted(EXPECTED))
def test_workload_shapes(key):
    shapes, nblocks, Ms, seed = EXPECTED[key]
    w = synth.WORKLOADS[key]
    assert [(s.N, s.K, s.r) for s in w.block] == shapes
    assert (w.nblocks, tuple(w.Ms), w.seed) == (nblocks, Ms, seed)
    assert len(w.layers()) == nblocks * len(shapes)
    assert [i for i, _ in w.layers()] == list(range(nblocks * len(shapes)))


def test_sign_bits_are_fair_and_independent_across_factors():
    rows, r = 2048, 304
    neg = {}
    for path in (synth.PATH_PRI, synth.PATH_RES):
        for mat in (synth.MAT_U, synth.MAT_V):
            neg[path, mat] = synth.words_to_negative(synth.sign_words(4, 7, path, mat, r, 0, rows), r)
    n = rows * r
    se = 0.5 / np.sqrt(n)
    for a in neg.values():
        assert abs(a.mean() - 0.5) < 5 * se
        # neighbouring columns and rows agree half of the time (no structure inside a word or across words)
        assert abs((a[:, 1:] == a[:, :-1]).mean() - 0.5) < 6 * se
        assert abs((a[1:] == a[:-1]).mean() - 0.5) < 6 * se
    keys = list(neg)
    for i in range(len(keys)):
        for j in range(i + 1, len(keys)):
            assert abs((neg[keys[i]] == neg[keys[j]]).mean() - 0.5) < 6 * se
    # another layer of the same stack draws other bits
    other = synth.words_to_negative(synth.sign_words(4, 8, 0, synth.MAT_U, r, 0, rows), r)
    assert abs((other == neg[0, synth.MAT_U]).mean() - 0.5) < 6 * se


def test_sign_rows_can_be_drawn_in_any_block():
    r = 200
    full = synth.sign_factor(1, 3, 1, synth.MAT_V, 300, r)
    assert np.array_equal(full[117:245], synth.sign_factor(1, 3, 1, synth.MAT_V, 300, r, 117, 245))
    assert set(np.unique(full)) == {-1.0, 1.0}


@pytest.mark.parametrize("kind", ["h", "g", "l"])
def test_scales_are_lognormal_binary16(kind):
    n = 200_000
    bits = synth.scale_vector(2, 5, 1, kind, n)
    assert bits.dtype == np.uint16 and bits.shape == (n,)
    v = bits.view(np.float16).astype(np.float64)
    assert np.all(np.isfinite(v)) and np.all(v > 0)
    lv = np.log(v)
    # binary16 rounding moves log v by at most 2^-11 relative: far below the tolerances here
    assert abs(lv.mean() - (-3.0)) < 5 * 0.5 / np.sqrt(n)
    assert abs(lv.std() - 0.5) < 5 * 0.5 / np.sqrt(2 * n)
    assert abs(np.median(v) - np.exp(-3.0)) < 0.01 * np.exp(-3.0)
    # the three kinds and the two paths are separate draws
    assert not np.array_equal(bits[:1000], synth.scale_vector(2, 5, 0, kind, 1000))


def test_activations_are_standard_normal_bfloat16():
    M, K = 16, 16384
    xb = synth.activations(4, 11, M, K)
    assert xb.dtype == np.uint16 and xb.shape == (M, K)
    x = synth.bf16_bits_to_f32(xb).astype(np.float64)
    n = M * K
    assert abs(x.mean()) < 5 / np.sqrt(n)
    assert abs(x.std() - 1.0) < 5 / np.sqrt(2 * n)
    # each value is the float32 draw rounded to the nearest bfloat16: off by at most half a unit in the last
    # place, 2^-8 of the value (8 significant bits); truncation would be off by up to twice that
    x32 = np.random.default_rng([4, 11, 0x7878]).standard_normal(n, dtype=np.float32).astype(np.float64)
    assert np.all(np.abs(x.ravel() - x32) <= np.abs(x32) * 2.0 ** -8)
    # every layer draws its own rows
    assert not np.array_equal(xb, synth.activations(4, 12, M, K))


def test_prefill_layers_read_disjoint_pool_windows():
    w = synth.WORKLOADS["llama2_13b_0.3_prefill"]
    M, K = 2048, 64        # the window rule does not depend on the width; a narrow pool keeps this fast
    pools = {}
    wins = [synth.layer_activations(w, i, M, K, pools) for i in range(8)]
    pool = pools[K]
    assert pool.shape == (w.pool_rows, K)
    for i, a in enumerate(wins):
        assert a.shape == (M, K)
        assert np.shares_memory(a, pool)
        assert np.array_equal(a, pool[i * M:(i + 1) * M])
    # the ninth layer wraps to the first window
    assert np.array_equal(synth.layer_activations(w, 8, M, K, pools), wins[0])
