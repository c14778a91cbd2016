"""Host-side logic of bench.py (no GPU): the algorithmic-work model behind the
roofline figures, the source-hash guard on committed ncu traffic, and the
parsing of clock samples that decides whether a run is kept."""
import hashlib

import bench
from combine_moe_route_14_b200 import inputs as I


def test_stage_model_mixtral_matches_the_shapes():
    cfg = I.workload("mixtral")  # T=4096, d=4096, E=8, top-2, f=14336
    m = bench.stage_model(cfg)
    T, d, E, f, R = 4096, 4096, 8, 14336, 8192
    assert cfg.R == R
    # GEMM-1 reads W1 once, the dispatched rows once, and writes H once
    assert m["gemm1"]["bytes"] == E * f * d * 2 + R * d * 2 + R * f * 2 == 1241513984
    assert m["gemm1"]["flops"] == m["gemm2"]["flops"] == 2 * R * d * f
    assert m["dispatch"]["bytes"] == T * d * 2 + R * d * 2 + R * 4
    assert m["combine"]["bytes"] == R * d * 2 + R * 8 + T * d * 2
    assert m["router_logits"]["flops"] == 2 * T * d * E
    assert m["ffn"]["flops"] == 2 * m["gemm1"]["flops"]


def test_stage_model_counts_only_active_experts_weights():
    cfg = I.workload("mixtral")
    counts = [1024] * 6 + [0, 0]  # two experts receive no token: their weights are not read
    full, part = bench.stage_model(cfg), bench.stage_model(cfg, counts=counts)
    w = cfg.f * cfg.d * 2
    assert full["gemm1"]["bytes"] - part["gemm1"]["bytes"] == 2 * w
    assert full["gemm2"]["bytes"] - part["gemm2"]["bytes"] == 2 * w


def test_stage_model_fp8_halves_the_gemm1_operands():
    cfg = I.workload("mixtral")
    bf, q = bench.stage_model(cfg), bench.stage_model(cfg, fp8=True)
    R, d, f, E = cfg.R, cfg.d, cfg.f, cfg.E
    assert bf["gemm1"]["bytes"] - q["gemm1"]["bytes"] == E * f * d + R * d
    assert q["gemm2"] == bf["gemm2"]


def _fake_tree(tmp_path, src_text, recorded_sha, traffic=123456789):
    csrc = tmp_path / "combine_moe_route_14_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "grouped_gemm.cu").write_text(src_text)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "grouped_gemm_gelu_mixtral.md").write_text(
        f"# summary\n\ncode_sha256: {recorded_sha}\n\ntraffic_bytes_per_launch: {traffic}\n")


KERNEL = "__global__ void k(int* p) {\n  p[0] = 1;  // store\n}\n"


def test_ncu_traffic_needs_the_recorded_code(tmp_path, monkeypatch):
    _fake_tree(tmp_path, KERNEL, bench.code_sha256(KERNEL))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("grouped_gemm_gelu", "mixtral") == 123456789.0
    assert bench.ncu_traffic("grouped_gemm_gelu", "fine_grained") is None  # no summary


def test_ncu_traffic_survives_comment_and_layout_edits(tmp_path, monkeypatch):
    edited = "/* a note */\n__global__ void k(int* p)\n{\n    p[0] = 1;   // the store\n}\n"
    _fake_tree(tmp_path, edited, bench.code_sha256(KERNEL))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("grouped_gemm_gelu", "mixtral") == 123456789.0


def test_ncu_traffic_is_void_once_the_kernel_changed(tmp_path, monkeypatch):
    _fake_tree(tmp_path, KERNEL.replace("p[0] = 1", "p[0] = 2"), bench.code_sha256(KERNEL))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("grouped_gemm_gelu", "mixtral") is None
    # the raw file hash (the older record format) no longer matches either
    _fake_tree(tmp_path / "raw", KERNEL, hashlib.sha256(KERNEL.encode()).hexdigest())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path / "raw"))
    assert bench.ncu_traffic("grouped_gemm_gelu", "mixtral") is None


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = list(lines)
    return s.summary()


def test_clock_summary_reports_power_cap_and_median():
    lines = [
        "0, 1965, 1965, 650.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.3, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1850, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    ]
    out = _sampler(lines)
    assert out["sm_mhz"] == 1850.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def test_clock_summary_flags_thermal_and_hardware_slowdown():
    lines = ["0, 1200, 1965, 500.0, 0x0000000000000048, Active, Active, Not Active, Not Active"]
    out = _sampler(lines)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]


def test_clock_summary_without_samples():
    out = _sampler(["garbage", "0, [N/A], 1965, 1, 0x0, a, b, c, d"])
    assert out["sm_mhz"] is None and out["samples"] == 0


def test_peak_choice_follows_the_length_of_the_timed_loop():
    assert not bench.sustained_peak_applies(30.0)     # 20 steps of 1.5 ms: burst
    assert not bench.sustained_peak_applies(999.0)
    assert bench.sustained_peak_applies(1000.0)       # a second or more: sustained


def test_both_arms_print_the_same_config():
    import argparse
    cfg = I.workload("mixtral")
    a = argparse.Namespace(fp8=False, gather=False, fused=False, pipeline=False)
    c = bench.arm_config(cfg, a, 1)
    for key in ("workload", "T", "d", "E", "k", "f", "fp8", "gather_on_load", "fused_ffn",
                "temperature", "min_prob", "renormalize", "score", "router"):
        assert key in c
    assert c == bench.arm_config(cfg, a, 1)


def test_host_cpu_reports_nproc():
    info = bench.host_cpu()
    assert info["nproc"] >= 1 and "cpu_model" in info
