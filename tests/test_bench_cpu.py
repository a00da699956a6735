"""Host logic of bench.py (no GPU): the workload layer lists, the split of a
bracketed step into in-step segment times (they sum to the timed step), the
regime checks over the segments whose layers all fall in a regime, the
burst / sustained tensor peak, and the traffic record's source-hash check."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


PEAKS = {"hbm_gbs": 6545.0, "bf16_tflops": 1627.8, "bf16_tflops_sustained": 1395.0}


def test_workload_layers(bench):
    l70 = bench.workload_layers("llama70b", bench.weight_copies("llama70b"))
    assert len(l70) == 52 and sorted({L.M for L in l70}) == [2 ** i for i in range(13)]
    d7 = bench.workload_layers("decode7b", bench.weight_copies("decode7b"))
    assert len(d7) == 12 and len({L.copy for L in d7}) == 3           # one weight copy per M
    nd = bench.workload_layers("nested7b_decode", bench.weight_copies("nested7b_decode"))
    assert {L.M for L in nd} == {1, 16} and len({L.copy for L in nd}) == 6
    for L in nd:                                                        # both modes read the same planes
        assert sum(1 for X in nd if (X.copy, X.shape_idx) == (L.copy, L.shape_idx)) == 2


def test_segments_sum_to_the_step_and_regimes(bench):
    layers = bench.workload_layers("llama70b", 1)
    small = tuple(i for i, L in enumerate(layers) if L.M <= 128)
    large = tuple(i for i, L in enumerate(layers) if L.M > 128)
    marks = [(("group", small), None, 0.0), (("quant", large), None, 1.0), (("gemm", large), None, 0.5),
             (("end", ()), None, 5.0)]
    roof, regimes, segs = bench.analyse_segments(layers, marks, 7.0, PEAKS, None, True)
    assert abs(sum(s["us_in_step"] for s in segs) - 7000.0) < 0.1       # scaled to the timed step
    assert roof["bound"] == "tensor" and roof["peak"] == pytest.approx(2790.0)
    gemm_us = 5.0 * 7.0 / 6.5 * 1e3
    flops = sum(layers[i].flops for i in large)
    assert roof["achieved"] == pytest.approx(flops / (gemm_us * 1e-6) / 1e12, rel=1e-3)
    ws = regimes["weight_streaming_m_le_128"]
    wb = sum(layers[i].weight_bytes for i in small)
    assert ws["weight_gbs"] == pytest.approx(wb / (1.0 * 7.0 / 6.5 * 1e-3) / 1e9, rel=1e-3)
    assert "decode_m_le_16" not in regimes                              # no segment holds only M <= 16 layers
    # a short region without the power cap: the burst figure
    roof_b, _, _ = bench.analyse_segments(layers, marks, 7.0, PEAKS, None, False)
    assert roof_b["peak"] == pytest.approx(2 * 1627.8)


def test_nested_decode_regimes_per_mode(bench):
    layers = bench.workload_layers("nested7b_decode", 6)
    f16 = tuple(i for i, L in enumerate(layers) if L.kind == "nested16")
    f8 = tuple(i for i, L in enumerate(layers) if L.kind == "nested8")
    marks = [(("group", f16), None, 0.0), (("group", f8), None, 0.2), (("end", ()), None, 0.1)]
    _, regimes, _ = bench.analyse_segments(layers, marks, 0.3, PEAKS, None, False)
    wb16 = sum(layers[i].weight_bytes for i in f16)
    assert regimes["decode_m_le_16_fp16_mode"]["weight_gbs"] == pytest.approx(wb16 / 0.2e-3 / 1e9, rel=1e-3)
    assert "decode_m_le_16_fp8_mode" in regimes and regimes["decode_m_le_16"]["target"] == 0.80


def test_traffic_record_follows_the_kernel_sources(bench, monkeypatch):
    t, note = bench.profiled_traffic("decode7b")
    assert t is not None and "algorithmic" in note
    monkeypatch.setattr(bench, "kernel_sources_hash", lambda: "000000000000")
    t, note = bench.profiled_traffic("decode7b")
    assert t is None and "changed" in note
