"""Host-side arithmetic of bench.py: the algorithmic byte counts behind the
roofline figures, the traffic file's source check, and the clock-sample
time stamps (no GPU)."""

import json

import pytest

import bench
import synth


def test_pass_bytes_all_experts_match_the_per_step_count():
    cfg = synth.config("stack")
    d, F, E, dh = 2816, 704, 128, 256
    layer = 2 * ((16 + 16) * dh * d + d * 16 * dh + E * d) + 2 * (E + 1) * 3 * F * d
    kv = sum(2 * 1 * 8 * (4096 if (l + 1) % 6 == 0 else 1024) * dh * 2 for l in range(30))
    head = 262144 * d * 2
    assert bench.bytes_per_step(cfg) == 30 * layer + kv + head
    assert bench.bytes_per_step(cfg) / 1e9 == pytest.approx(49.98, abs=0.01)


def test_gateup_bytes_per_launch_counts_active_groups_rows_and_h():
    cfg = synth.config("stack")
    d, F, T, k = 2816, 704, 256, 8
    got = bench.gateup_bytes_per_launch(cfg, 33.7375)
    assert got == pytest.approx((33.7375 + 1) * 2 * F * d * 2 + (k + 1) * T * d * 2 + (k + 1) * T * F * 2)
    assert got / 1e6 == pytest.approx(291.68, abs=0.01)
    # every expert active: the weights of all 129 groups
    assert bench.gateup_bytes_per_launch(cfg) > 1.0e9


def test_traffic_scales_the_captured_ratio_and_is_null_when_the_gemm_sources_changed(
        tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"gemm_gateup": {"dram_over_algorithmic": 1.25, "kernel_src_sha": "abc"}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_src_sha", lambda: "abc")
    assert bench.load_traffic("gemm_gateup", 400.0) == 500.0
    monkeypatch.setattr(bench, "kernel_src_sha", lambda: "def")
    assert bench.load_traffic("gemm_gateup", 400.0) is None
    assert bench.load_traffic("gemm_down", 400.0) is None


def test_clock_sample_stamps_parse():
    t = bench.ClockSampler._stamp("2026/12/02 17:10:01.250")
    t2 = bench.ClockSampler._stamp("2026/12/02 17:10:02.000")
    assert t2 - t == pytest.approx(0.75)
    assert bench.ClockSampler._stamp("not a time") is None
