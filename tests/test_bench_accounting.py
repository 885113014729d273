"""The algorithmic work bench.py divides by, pinned to the method's own accounting (CPU).

Bytes per layer are the packed signs and binary16 scales of both paths — the
bits-per-weight formula of the wiki page on LittleBit and LittleBit-2 ("How to
judge an ultra-low-bit scheme", point 1: factors and scales both count),
BPW = sum over paths of (r (N + K) + 16 (N + K + r)) / (N K) — plus the bf16
activations in and the float32 outputs out.  FLOPs per layer are those of the
two binary contractions, 2 M r (K + N) per path (LittleBit paper notes page,
"Multi-scale compensation": x (.) g -> . V_sign -> (.) l -> . U_sign^T -> (.) h);
the dense 2 M N K the method avoids is never counted.
"""

import os
from fractions import Fraction

import pytest

import bench
from sub_bit_weight_b200 import synth


def bpw(N, K, r, npaths=2):
    return Fraction(npaths * (r * (N + K) + 16 * (N + K + r)), N * K)


@pytest.mark.parametrize("wkey", ["single_512", "llama2_7b_0.1", "llama2_7b_0.55", "llama2_13b_0.3_prefill",
                                  "llama2_70b_0.1"])
def test_weight_bytes_follow_the_bits_per_weight_formula(wkey):
    for s in synth.WORKLOADS[wkey].block:
        k1, k2 = bench.layer_bytes(s, 0)          # M = 0: weights and scales only
        assert Fraction(int(8 * (k1 + k2)), s.N * s.K) == bpw(s.N, s.K, s.r)


@pytest.mark.parametrize("wkey,per_layer", [
    # packed signs + scales of both paths per layer, worked out by hand from the formula
    ("single_512", {"t": 8256}),
    ("llama2_7b_0.1", {"q": 196928, "gate": 544256}),
    ("llama2_7b_0.55", {"q": 1149056, "gate": 3084416}),
    ("llama2_13b_0.3_prefill", {"q": 984512, "gate": 2654336}),
    ("llama2_70b_0.1", {"q": 819936, "k": 110720, "gate": 2950336}),
])
def test_weight_bytes_of_the_workload_layers(wkey, per_layer):
    shapes = {s.name: s for s in synth.WORKLOADS[wkey].block}
    for name, want in per_layer.items():
        s = shapes.get(name) or next(iter(shapes.values()))
        assert sum(bench.layer_bytes(s, 0)) == want


def test_stack_totals():
    w = synth.WORKLOADS["llama2_70b_0.1"]
    weights = sum(sum(bench.layer_bytes(s, 0)) for s in w.block) * w.nblocks
    assert weights == pytest.approx(857.0e6, rel=1e-3)          # > L2: the stack streams from HBM
    p = synth.WORKLOADS["llama2_13b_0.3_prefill"]
    flops = sum(bench.layer_flops(s, 2048) for s in p.block) * p.nblocks
    assert flops == pytest.approx(15.07e12, rel=1e-3)


def test_activation_and_output_bytes():
    s = synth.LayerShape("t", 300, 200, 7)
    for M in (1, 5, 16):
        k1, k2 = bench.layer_bytes(s, M)
        k10, k20 = bench.layer_bytes(s, 0)
        assert k1 - k10 == 2 * M * s.K            # x in, bfloat16
        assert k2 - k20 == 4 * M * s.N            # y out, float32


def test_flops_are_the_two_binary_contractions():
    s = synth.LayerShape("t", 300, 200, 7)
    assert bench.layer_flops(s, 3) == 2 * 3 * 2 * 7 * (200 + 300)
    assert bench.layer_flops(s, 3, npaths=1) == 2 * 3 * 7 * (200 + 300)
    st = bench.backward_stage_flops(s, 3)
    assert sum(st.values()) == 2 * 3 * 2 * 7 * (3 * 200 + 2 * 300)


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk = bench.peaks()
    assert pk["src"] == "fallback" and pk["hbm_gbs"] == 6650.0 and pk["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}')
    pk = bench.peaks()
    assert pk["src"] == "measured" and pk["hbm_gbs"] == 6500.0 and pk["bf16_tflops_sustained"] == 1600.0


def test_dram_traffic_is_reported_only_for_the_sources_it_was_captured_with(tmp_path, monkeypatch):
    # profiles/traffic.txt records, per kernel and workload, the DRAM bytes of one launch and a hash of the
    # sources they were captured with; a changed source makes the figure null rather than stale
    for kernel in bench.KERNEL_SOURCES:
        assert all(os.path.exists(os.path.join(bench.CSRC, f)) for f in bench.KERNEL_SOURCES[kernel])
    prof = tmp_path / "profiles"
    prof.mkdir()
    k = "contraction2_ldg_kernel"
    good = bench.source_hash(k)
    (prof / "traffic.txt").write_text("# kernel workload source_sha16 dram_bytes_per_launch note\n"
                                      f"{k} wl_a {good} 123456 x\n"
                                      f"{k} wl_b {'0' * 16} 999 x\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic(k, "wl_a") == 123456.0
    assert bench.measured_traffic(k, "wl_b") is None          # captured with other sources
    assert bench.measured_traffic(k, "wl_c") is None          # never captured
    assert bench.measured_traffic("prefill_kernel<0>", "wl_a") is None
    # the hash covers every listed source: any edit changes it
    src = tmp_path / "csrc"
    src.mkdir()
    for f in bench.KERNEL_SOURCES[k]:
        (src / f).write_bytes(open(os.path.join(bench.CSRC, f), "rb").read())
    monkeypatch.setattr(bench, "CSRC", str(src))
    assert bench.source_hash(k) == good
    last = src / bench.KERNEL_SOURCES[k][-1]
    last.write_bytes(last.read_bytes() + b"\n")
    assert bench.source_hash(k) != good


def test_roofline_denominators():
    """Decode kernels are measured against HBM copy bandwidth; the prefill GEMMs, each timed alone, against the
    burst tensor peak (the sustained one reported beside it)."""
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "src": "measured"}
    p = synth.WORKLOADS["llama2_13b_0.3_prefill"]
    shapes = list(p.block)
    r = bench.roofline_of({"per_launch": (1.0, 2.0)}, shapes, 2048, True, pk, p.key)
    f2 = sum(2.0 * 2048 * 2 * s.r * s.N for s in shapes)
    assert r["kernel"].startswith("prefill_kernel<1>")
    assert r["achieved"] == pytest.approx(f2 / 2e-3 / 1e12, abs=0.1)
    assert r["peak"] == 1600.0 and r["frac"] == pytest.approx(r["achieved"] / 1600.0, abs=1e-4)
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / 1400.0, abs=1e-4)
    w = synth.WORKLOADS["llama2_70b_0.1"]
    shapes = list(w.block)
    q = sum(2.0 * s.K + 2 * 2.0 * s.K for s in shapes)
    k1 = sum(bench.layer_bytes(s, 1)[0] for s in shapes)
    r = bench.roofline_of({"per_launch": (0.01, 0.05, 0.005, 0.02)}, shapes, 1, False, pk, w.key)
    assert r["kernel"] == "contraction1_ldg_kernel"
    assert r["algorithmic_bytes_per_launch"] == pytest.approx(k1 - q)
    assert r["frac"] == pytest.approx((k1 - q) / 0.05e-3 / 1e9 / 6000.0, abs=1e-4)
    r = bench.roofline_of({"per_launch": (0.01, 0.001, 0.02)}, shapes, 4, False, pk, w.key)
    assert r["kernel"] == "contraction2_kernel"
    assert bench.roofline_of({"per_launch": None}, shapes, 4, False, pk, w.key) is None


def test_config_runs_cover_the_other_workloads():
    items = [t.split(":") for t in bench.CONFIGS_DEFAULT.split(",")]
    got = {(t[0], int(t[1]), len(t) > 2) for t in items}
    assert {("single_512", 1, False), ("single_512", 8, False)} <= got
    assert {("llama2_7b_0.1", 1, False), ("llama2_7b_0.1", 1, True)} <= got
    assert {("llama2_7b_0.55", m, False) for m in (1, 4, 16)} <= got
    for name, M, _ in got:
        assert M in synth.WORKLOADS[name].Ms


def test_end_to_end_object():
    """e2e is the same metric through the C-ABI call with host buffers: work over the pipelined step time, the serial
    figure beside it, the bytes copied each way as measured; absent when the run measured none."""
    res = {"e2e": {"ms": 0.5, "serial_ms": 1.0, "h2d": 1000, "d2h": 4000, "steps": 10}}
    e = bench.e2e_of(res, None, 1, 896.0e6, False, "how")
    assert e["unit"] == "GB/s" and e["value"] == pytest.approx(896.0e6 / 0.5e-3 / 1e9, abs=0.01)
    assert e["serial"]["value"] == pytest.approx(896.0e6 / 1.0e-3 / 1e9, abs=0.01)
    assert (e["h2d_bytes_per_step"], e["d2h_bytes_per_step"]) == (1000, 4000)
    p = bench.e2e_of(res, None, 1, 0.376e12, True, "how")
    assert p["unit"] == "TFLOP/s" and p["value"] == pytest.approx(0.376e12 / 0.5e-3 / 1e12, abs=0.01)
    assert bench.e2e_of({"e2e": None}, None, 1, 1.0, False, "how") is None
