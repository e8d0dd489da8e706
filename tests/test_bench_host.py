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


def test_encoder_flops_count_each_position_once_per_visible_key():
    """Brute force on a small shape: per layer, every position's projections and experts,
    plus causal attention over the positions it sees (window on local layers)."""
    import synth
    cfg = synth.config("tiny", prompt_len=37, window=5, global_every=2)
    d, F, E, k = cfg["d_model"], cfg["d_ff"], cfg["n_experts"], cfg["top_k"]
    dh, Hq, Hkv, P, W = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"], 37, 5
    per_token = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d) + 2 * (k + 1) * 3 * F * d
    want = 0
    for l in range(cfg["n_layers"]):
        glob = (l + 1) % cfg["global_every"] == 0
        for p in range(P):
            seen = p + 1 if glob else min(p + 1, W)
            want += per_token + 4 * Hq * dh * seen
    assert bench.encoder_flops(cfg) == want * cfg["batch"]


def test_encoder_bytes_read_each_chunks_weights_once_and_the_visible_cache():
    """Two chunks of 16 over a 20-token prompt: weights twice per layer, the second chunk
    reads the first chunk's cache (all of it on the global layer, window - 1 on the local)."""
    import synth
    cfg = synth.config("tiny", prompt_len=20, window=5, global_every=2)
    d, F, E = cfg["d_model"], cfg["d_ff"], cfg["n_experts"]
    dh, Hq, Hkv, L, B = cfg["head_dim"], cfg["n_q_heads"], cfg["n_kv_heads"], 2, cfg["batch"]
    dense = 2 * ((Hq + 2 * Hkv) * dh * d + d * Hq * dh + E * d)
    egb = 3 * F * d * 2
    kv_row = 2 * B * Hkv * dh * 2            # one position's K and V, every kv head
    kv = (0 + 16) * kv_row + (4 + 4) * kv_row + (0 + 16) * kv_row + (16 + 4) * kv_row
    want = 2 * L * dense + 2 * L * (3 + 1) * egb + kv + B * 20 * d * 2
    got, n_chunks = bench.encoder_bytes(cfg, 3, chunk=16)
    assert n_chunks == 2 and got == want
