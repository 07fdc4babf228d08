"""Host-side logic of bench.py on CPU: the peak figures' fallback, the committed DRAM-traffic
figure's source check, and the parsing of the clock samples taken during the timed region."""
import json

import bench


def test_measured_peaks_read_and_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()                                   # no file
    assert p["source"] == "fallback" and p["hbm_gbs"] == bench.FALLBACK_PEAKS["hbm_gbs"]
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.measured_peaks()["source"] == "fallback"        # malformed
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": None, "bf16_tflops": 1}))
    assert bench.measured_peaks()["source"] == "fallback"        # a null figure
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 7012.5, "bf16_tflops": 1620}))
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 7012.5
    assert p["bf16_tflops_sustained"] == 1620.0                  # burst figure when no sustained one


def test_committed_traffic_only_for_the_current_source(tmp_path, monkeypatch):
    src = bench.kernel_source_hash()
    assert len(src) == 16 and src == bench.kernel_source_hash()  # deterministic
    real_root = bench.ROOT
    (tmp_path / "profiles").mkdir()
    (tmp_path / "long_context_speculative_kv_b200").symlink_to(
        f"{real_root}/long_context_speculative_kv_b200", target_is_directory=True)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    t = tmp_path / "profiles" / "traffic.txt"
    t.write_text("# comment verify_attn ctx1m 1 " + src + "\n"
                 f"verify_attn ctx1m 2161290082 {src}\n"
                 "verify_attn ctx128k 99 0123456789abcdef\n")
    assert bench.committed_traffic("verify_attn", "ctx1m") == 2161290082.0
    assert bench.committed_traffic("verify_attn", "ctx128k") is None     # taken on another source
    assert bench.committed_traffic("verify_attn", "batch8-tree") is None  # no line
    t.write_text(f"verify_attn ctx1m 2161290082 {'f' * 16}\n")
    assert bench.committed_traffic("verify_attn", "ctx1m") is None


def test_clock_samples_parse():
    rows = ["1590, 1965, 980.1, Not Active, Not Active, Not Active, Active",
            "1605, 1965, 990.0, Not Active, Not Active, Not Active, Active",
            "1575, 1965, 1001.2, Active, Not Active, Not Active, Not Active",
            "[N/A], 1965, 10.0, Not Active, Not Active, Not Active, Not Active",
            "garbage line"]
    c = bench.parse_clock_samples("\n".join(rows))
    assert c["samples"] == 4
    assert c["sm_mhz"] == 1590.0                                 # median of the numeric samples
    assert c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert bench.parse_clock_samples("") is None
