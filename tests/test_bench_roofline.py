"""bench.py's roofline pieces, on CPU.  The W4A4 layer's bound is the slower of
streaming the packed expert weights at the HBM bandwidth and the layer's flops at the
block-scaled fp4 peak (measured bf16 peak x the nominal fp4/bf16 ratio 4).  A DRAM
traffic figure is reported only while the kernel sources hash to the value recorded
with its ncu capture."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PK = dict(hbm=6441.9, bf16=1640.9, bf16_sus=1416.7, source="measured")


def test_120b_shaped_w4a4_layer_is_weight_stream_bound():
    # 128 experts x (2I*H + H*I) weights at 4.25 bits each; T = 4096, top-4
    wbytes = 128 * (2 * 2880 * 2880 + 2880 * 2880) * (0.5 + 1 / 32)
    assert wbytes == 1_692_057_600
    flops = bench.layer_flops(4096, 4, 2880, 2880)
    assert flops == pytest.approx(0.8154e12, rel=1e-4)
    r = bench.w4a4_roofline(flops, wbytes, 0.8, PK)
    assert r["bound"] == "hbm"
    assert r["mxf4_peak_tflops"] == pytest.approx(4 * 1640.9)
    assert r["hbm_us"] == pytest.approx(262.66, abs=0.01)        # 1.692 GB at 6441.9 GB/s
    assert r["mxf4_us"] == pytest.approx(124.23, abs=0.01)       # 0.8154 TFLOP at 6563.6 TFLOP/s
    assert r["bound_us"] == r["hbm_us"]
    assert r["frac"] == pytest.approx(262.66 / 800.0, abs=1e-4)


def test_flop_heavy_layer_is_mxf4_bound():
    r = bench.w4a4_roofline(1e15, 1e6, 1000.0, PK)
    assert r["bound"] == "mxf4"
    assert r["bound_us"] == pytest.approx(1e15 / (4 * 1640.9e12) * 1e6)
    assert 0 < r["frac"] < 1


def test_traffic_is_reported_only_for_the_captured_source(monkeypatch, tmp_path):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k|w": {"dram_bytes_per_launch": 123.0, "source_sha256_16": "a" * 16}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "a" * 16)
    assert bench.traffic_record("k", "w") == 123.0
    assert bench.traffic_record("k", "other") is None          # not captured
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "b" * 16)
    assert bench.traffic_record("k", "w") is None              # kernel source changed since


def test_committed_traffic_record_is_well_formed():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        recs = json.load(f)
    for key, r in recs.items():
        kernel, workload = key.split("|")
        assert r["dram_bytes_per_launch"] == r["dram_read_bytes"] + r["dram_write_bytes"]
        assert len(r["source_sha256_16"]) == 16 and "ncu" in r["command"]


def test_measured_mma_ratio_sets_the_mxf4_peak():
    # the probe's mxf4 / f16 tensor-pipe rate ratio replaces the nominal 4
    rates = {"f16_tflops": 2100.0, "mxf4_tflops": 8358.0, "mxf4_over_f16": 8358.0 / 2100.0}
    peak, src = bench.mxf4_peak(PK, rates)
    assert peak == pytest.approx(1640.9 * 8358.0 / 2100.0)
    assert "probe" in src
    r = bench.w4a4_roofline(1e15, 1e6, 1000.0, PK, rates)
    assert r["mxf4_peak_tflops"] == pytest.approx(peak)
    assert r["bound_us"] == pytest.approx(1e15 / (peak * 1e12) * 1e6)
    assert bench.mxf4_peak(PK, None)[0] == pytest.approx(4 * 1640.9)
