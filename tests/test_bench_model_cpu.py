"""The benchmark's measurement model on CPU: the algorithmic bytes and flops that
every roofline figure divides by, hand-counted on a small layer; the fused-launch
entries count the shared gradient rows once; recorded DRAM traffic is dropped as
soon as the kernels' code (comments aside) changes."""
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


def test_recorded_traffic_needs_the_kernels_current_sources(monkeypatch, tmp_path):
    prof = tmp_path / "profiles"
    prof.mkdir()
    sha = bench.kernel_source_sha1("wgrad_gu")
    (prof / "traffic.json").write_text(json.dumps({
        "wgrad_gu@qwen": {"bytes": 123, "source_sha1": sha},
        "unpack@qwen-T2048": {"bytes": 300, "algorithmic_bytes": 200, "source_sha1": "x",
                              "scale_to": ["qwen"]}}))
    assert bench.kernel_source_sha1("score") != bench.kernel_source_sha1("wgrad_gu")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_sha1", lambda k: sha if k == "wgrad_gu" else "x")
    assert bench.recorded_traffic("wgrad_gu", "qwen")[0] == 123
    assert bench.recorded_traffic("dgrad_x", "qwen")[0] is None
    # a capture on a smaller case scales by the algorithmic bytes of the full launch
    assert bench.recorded_traffic("unpack", "qwen", 1000.0)[0] == 1500.0
    assert bench.recorded_traffic("unpack", "glm", 1000.0)[0] is None
    monkeypatch.setattr(bench, "kernel_source_sha1", lambda k: "0" * 40)
    assert bench.recorded_traffic("wgrad_gu", "qwen")[0] is None
    assert bench.recorded_traffic("unpack", "qwen", 1000.0)[0] is None


def test_committed_traffic_entries_are_well_formed():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    for key, e in table.items():
        kernel = key.split("@")[0]
        assert kernel in bench.KERNEL_SOURCES, key
        assert len(e["source_sha1"]) == 40 and e["bytes"] > 0, key
        if "scale_to" in e:
            assert e["algorithmic_bytes"] > 0, key


def test_roofline_bound_follows_the_ridge():
    peaks = dict(bench.FALLBACK_PEAKS)
    T, k, E, H, I = 16384, 8, 128, 4096, 1408
    by, fl = bench.algorithmic(T, k, E, H, I, T * k, 2)       # every pair kept
    r = bench.roofline_of("wgrad_gu", 2.5, by, fl, peaks, "fallback", "sweep100")
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - fl["wgrad_gu"] / 2.5e-3 / 1e12) < 1e-9
    assert abs(r["frac"] - r["achieved"] / peaks["bf16_tflops_sustained"]) < 1e-12
    by, fl = bench.algorithmic(8192, 8, 128, 2048, 768, 20427, 2)   # qwen-shaped, pruned
    r = bench.roofline_of("wgrad_gu", 0.34, by, fl, peaks, "fallback", "qwen")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert bench.roofline_of("unpack", 0.03, by, fl, peaks, "fallback", "qwen")["bound"] == "hbm"


def test_source_hash_ignores_comments_only():
    """The traffic records are keyed to the kernels' code: an edit of comments or
    whitespace keeps the key, an edit of code changes it."""
    code = "int f(int a) {  // doubles\n  /* the\n  result */ return 2 * a;\n}\n"
    same = "int f(int a) {\n  return 2 * a;  // twice a\n}\n"
    other = "int f(int a) {\n  return 3 * a;\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
    assert "//" not in bench._code_only(code) and "/*" not in bench._code_only(code)
