"""The benchmark's measurement model on CPU: the algorithmic bytes and flops that
every roofline figure divides by, hand-counted on a small layer; the fused-launch
entries count the shared gradient rows once; recorded DRAM traffic is dropped as
soon as the GEMM sources change."""
import json
import os

import bench


def test_algorithmic_bytes_and_flops_hand_counted():
    T, k, E, H, I, M, b = 4, 2, 3, 16, 8, 5, 2
    P = T * k
    by, fl = bench.algorithmic(T, k, E, H, I, M, b)
    assert by["score"] == T * H * b + P * I * b + 12 * P            # dY, a, idx+w+score
    assert by["pack"] == 2 * M * (2 * H + I) * b + 8 * M            # X_p, DY_p, A_p read+write
    assert by["wgrad_gu"] == 2 * M * I * b + M * H * b + E * 2 * I * H * 4
    assert by["dgrad_x"] == 2 * M * I * b + E * 2 * I * H * b + M * H * b
    assert by["unpack"] == M * H * b + 4 * P + T * H * b
    assert fl["dgrad_swiglu"] + fl["wgrad_down"] + fl["wgrad_gu"] + fl["dgrad_x"] == 12 * M * H * I
    assert by["dgrad_x+wgrad_gu"] == by["dgrad_x"] + by["wgrad_gu"] - 2 * M * I * b
    assert bench.step_gemms(fl) == ["dgrad_swiglu", "wgrad_down", "wgrad_gu", "dgrad_x"]
    # fp32 path packs G_p, U_p too
    by32, _ = bench.algorithmic(T, k, E, H, I, M, 4)
    assert by32["pack"] == 2 * M * (2 * H + 3 * I) * 4 + 8 * M


def test_recorded_traffic_needs_the_current_gemm_sources(monkeypatch, tmp_path):
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = bench.kernel_source_sha1()
    (prof / "traffic.json").write_text(json.dumps(
        {"wgrad_gu@qwen": {"bytes": 123, "source_sha1": sha}}))
    monkeypatch.setattr(bench, "kernel_source_sha1", lambda: sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("wgrad_gu", "qwen") == 123
    assert bench.recorded_traffic("dgrad_x", "qwen") is None
    monkeypatch.setattr(bench, "kernel_source_sha1", lambda: "0" * 40)
    assert bench.recorded_traffic("wgrad_gu", "qwen") is None


def test_committed_traffic_matches_the_committed_gemm_sources():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    assert {e["source_sha1"] for e in table.values()} == {bench.kernel_source_sha1()}
