"""The arithmetic behind bench.py's line: algorithmic work of each call, the
layer roofline and whole-job throughput, checked against figures worked out
independently from the definitions (the FLOP and byte counts of the 380M
and 1.3B layer shapes); the DRAM-traffic record's tie to the source it was
measured on; the clock summary."""
import numpy as np
import pytest

import bench
from mixture_memories_layer_b200 import synth

PEAKS = {"bf16_tflops": 1631.7, "hbm_gbs": 6540.2}


def _close(a, b, rel=5e-4):
    return abs(a - b) <= rel * abs(b)


def test_380m_layer_work_and_roofline():
    w = synth.WORKLOADS["mom380m"]
    sw = bench.step_work(w)
    # projections 2 N D (3Hd + 2H) + 2 N k D 2Hd; recurrence 6 N (1+k) H d^2
    assert _close(sw["proj"]["flops"], 240.8e9, 1e-3)
    assert _close(sw["gdn"]["flops"], 77.3e9, 1e-3)
    flops, bytes_, t = bench.layer_roofline(w, PEAKS)
    assert _close(flops, 318.3e9, 1e-3)
    assert _close(bytes_, 132.4e6, 1e-3)
    assert _close(t, 0.1951e-3, 1e-3)                 # tensor-bound: flops / peak
    assert _close(w.n_tokens / t, 84.0e6, 1e-3)       # roofline tokens/s


def test_1p3b_layer_work():
    w = synth.WORKLOADS["mom1p3b_m16"]
    flops, bytes_, t = bench.layer_roofline(w, PEAKS)
    assert _close(flops, 1771.9e9, 1e-3)
    assert _close(bytes_, 571.1e6, 1e-3)
    assert _close(t, 1.0859e-3, 1e-3)


def test_final_states_are_counted_per_sequence():
    # varlen workloads have no fixed batch: the number of sequences is passed
    w = synth.WORKLOADS["mom380m_skew_varlen"]
    S = len(synth.make_problem(w)["cu_seqlens"]) - 1
    b0 = bench.layer_roofline(w, PEAKS, n_seq=0)[1]
    bS = bench.layer_roofline(w, PEAKS, n_seq=S)[1]
    assert bS - b0 == (1 + w.n_mem) * S * w.heads * w.d_head ** 2 * 4


def test_whole_job_throughput_uses_the_slowest_rank():
    assert bench.aggregate_throughput(16384, 2, 20, 12.4) == pytest.approx(16384 * 2 * 20 / 0.0124)


def test_traffic_record_is_reported_only_for_the_source_it_was_measured_on(monkeypatch):
    # profiles/traffic.json holds a kernel's ncu DRAM bytes with the hash of
    # the source they were measured on; the bench reports them only while that
    # source is unchanged (a scratch tree stands in for the repository here)
    import json
    import os
    from tests.conftest import ROOT
    root = os.path.join(ROOT, "mixture_memories_layer_b200", "_build", "traffic_check")
    os.makedirs(os.path.join(root, "profiles"), exist_ok=True)
    os.makedirs(os.path.join(root, "mixture_memories_layer_b200", "csrc"), exist_ok=True)
    src = os.path.join(root, "mixture_memories_layer_b200", "csrc", "k.cu")
    with open(src, "w") as fh:
        fh.write("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", root)
    rec = {"k": {"source": "k.cu", "source_sha": bench.kernel_source_sha("k.cu"), "bytes_per_launch": 123}}
    with open(os.path.join(root, "profiles", "traffic.json"), "w") as fh:
        json.dump(rec, fh)
    assert bench.measured_traffic("k") == (123, "current")
    assert bench.measured_traffic("other") == (None, "none")
    with open(src, "w") as fh:
        fh.write("// kernel v2\n")
    assert bench.measured_traffic("k") == (None, "stale")


def test_committed_traffic_record_status_is_reported():
    # the repository's own record: either it matches the current GDN source
    # (its bytes are reported) or the bench says it is stale and reports none
    traffic, status = bench.measured_traffic("gdn")
    assert status in ("current", "stale")
    assert (traffic is not None) == (status == "current")


def test_clock_summary_names_every_throttle_reason_seen():
    c = bench.ClockSampler(torch_device=None)
    c.sm_max = 1965
    c.samples = [(1965, 0x0), (1950, 0x4), (1800, 0x8 | 0x4), (1965, 0x40)]
    s = c.summary()
    assert s["sm_mhz"] == 1957.5 and s["sm_max_mhz"] == 1965 and s["samples"] == 4
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]
    empty = bench.ClockSampler(torch_device=None)
    empty.sm_max = None
    assert empty.summary()["reasons"] == ["unsampled"]


def test_load_peaks_measured_partial_and_fallback(tmp_path, monkeypatch):
    import json
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.load_peaks()
    assert p["source"] == "fallback" and p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6540.2, "bf16_tflops": 1631.7, "bf16_tflops_sustained": 1358.8, "clocks": "x"}))
    p = bench.load_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6540.2 and p["bf16_tflops_sustained"] == 1358.8
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"peaks": {"hbm_gbs": 6000.0}}))
    p = bench.load_peaks()
    assert p["hbm_gbs"] == 6000.0 and p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]
    assert p["source"].startswith("measured (hbm_gbs)")
    (tmp_path / "MEASURED_PEAKS.json").write_text("not json")
    assert bench.load_peaks()["source"] == "fallback"


def test_380m_block_roofline():
    """The block adds the output gate's and the output projection's products
    (2 N D Hd each), the convolutions (2 W (3 + 2k) N Hd) and the gated norm
    (8 N Hd) to the layer; its bytes replace the layer's output [N, Hd] by y
    [N, D] and add W_g, W_o and the filters."""
    w = synth.WORKLOADS["mom380m_block"]
    flops, bytes_, t = bench.block_roofline(w, PEAKS)
    N, D, Hd = 16384, 1024, 1024
    assert _close(flops, 318.3e9 + 4 * N * D * Hd + 2 * 4 * 7 * N * Hd + 8 * N * Hd, 1e-3)
    assert _close(flops, 388.1e9, 1e-3)
    assert _close(bytes_, 136.8e6, 2e-3)
    assert _close(t, 388.1e9 / 1631.7e12, 1e-3)        # tensor-bound


def test_backward_roofline_is_twice_the_forward_at_the_bf16_peak():
    """The backward's estimate: 2 x the forward's FLOPs (an input and a
    weight gradient per product) against the bf16 peak; for the 380M layer
    636.6 GFLOP, 0.390 ms at 1631.7 TFLOP/s, so 32 ms is 1.2 %."""
    w = synth.WORKLOADS["mom380m"]
    lf = bench.layer_roofline(w, PEAKS)[0]
    r = bench.backward_roofline(lf, PEAKS, 32.0)
    assert r["flops"] == 2 * lf
    assert _close(r["flops"], 636.6e9, 1e-3)
    assert _close(r["roofline_ms"], 636.6e9 / 1631.7e12 * 1e3, 1e-3)
    assert _close(r["frac"], r["roofline_ms"] / 32.0)
    assert 0.011 < r["frac"] < 0.013
