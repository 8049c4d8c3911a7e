"""CPU checks of bench.py's host-side arithmetic and bookkeeping: the FLOP
count of the metric, the DRAM-traffic record that must go null once a
kernel's source changes, and the peaks fallback."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_flop_count_of_the_metric():
    fwd, bwd = bench.attn_flops(2, 16, 16384, 64)
    pairs = 16384 * 16385 // 2
    assert fwd == 4 * 64 * 2 * 16 * pairs == 1099578736640
    assert bwd == 2.5 * fwd
    f1, _ = bench.attn_flops(1, 1, 1, 64)  # one token sees itself only
    assert f1 == 4 * 64


def test_traffic_record_follows_the_kernel_source():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    for kid, (name, src) in bench.KERNELS.items():
        got = bench.recorded_traffic(kid)
        if name in rec and rec[name]["source_sha"] == bench.source_sha(src):
            assert got == float(rec[name]["bytes_per_launch"])
        else:
            assert got is None


def test_traffic_record_goes_null_when_the_source_differs(monkeypatch):
    monkeypatch.setattr(bench, "source_sha", lambda rel: "0" * 16)
    for kid in bench.KERNELS:
        assert bench.recorded_traffic(kid) is None


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.peaks()
    assert p["source"] == "fallback"
    assert p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}))
    p = bench.peaks()
    assert p["source"] == "measured" and p["bf16_tflops"] == 1600.0
    assert p["bf16_tflops_sustained"] == 1400.0
