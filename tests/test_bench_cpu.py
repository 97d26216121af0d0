"""Host logic of bench.py that needs no GPU: the clock record taken during the
timed region (nvidia-smi rows, here written by the test) and the JSON line's
shape helpers."""
import os

import pytest

import bench


def _sampler_with(rows, tmp_path):
    s = bench.ClockSampler(0)
    p = tmp_path / "clocks.csv"
    p.write_text("".join(r + "\n" for r in rows))
    s.path = str(p)
    return s


def test_clock_summary_uses_loaded_samples_and_active_reasons(tmp_path):
    idle = "0, 1965, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    busy = "0, 1900, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"
    busy2 = "0, 1800, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active"
    s = _sampler_with([idle, busy, busy2, "garbage line", idle], tmp_path)
    out = s.summary()
    assert out["samples"] == 2                       # idle samples (below half the peak power) left out
    assert out["sm_mhz"] == pytest.approx(1850.0)    # median of the loaded samples
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]        # "Not Active" is not a reason
    assert out["power_w_max"] == 980.0
    assert not os.path.exists(s.path)                # the temporary record is removed


def test_clock_summary_reports_throttling_and_missing_record(tmp_path):
    hot = "0, 1200, 1965, 950.0, 0x48, Active, Not Active, Active, Not Active"
    out = _sampler_with([hot, hot], tmp_path).summary()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    empty = bench.ClockSampler(0)
    assert empty.summary()["reasons"] == ["unsampled"]


def test_workload_config_and_metric_names():
    w = bench.WORKLOAD
    c = bench.workload_config(w["B"], w["T"], 1)
    assert c["tokens_per_step_per_gpu"] == w["B"] * w["T"] and c["parallelism"] == "single-gpu"
    assert bench.workload_config(w["B"], w["T"], 8)["parallelism"].startswith("dp8")
    assert bench.metric_for(w, w["B"], w["T"]) == bench.METRIC
    assert bench.metric_for(bench.MODELS["xl"], 4, 1024) != bench.METRIC
    # 6N + 12 L C T with the tied wte counted once at the padded vocabulary
    assert bench.flops_per_token(w) == pytest.approx(8.601e8, rel=1e-3)


def test_exact_causal_flop_count():
    """The exact causal count of one 124M step: 3 x the forward GEMMs plus 3.5 x
    the causal attention forward, written out per term and against the ~1.32e13
    of the hot-path scope table."""
    w = bench.MODELS["124m"]
    B, T, C, L, V, H = 16, 1024, 768, 12, 50304, 12
    gemm = 3 * (L * 2 * B * T * 12 * C * C + 2 * B * T * C * V)
    attn = L * (2 + 5) * B * H * T * (T + 1) * (C // H)
    assert bench.exact_step_flops(w, B, T) == pytest.approx(gemm + attn, rel=1e-12)
    assert bench.exact_step_flops(w, B, T) == pytest.approx(1.32e13, rel=5e-3)
    # the 6N + 12 L C T convention counts more: non-causal attention and the embeddings' 6N share
    assert bench.flops_per_token(w) * B * T > bench.exact_step_flops(w, B, T)


def test_roofline_traffic_only_for_the_captured_source(tmp_path, monkeypatch):
    """`traffic` comes from the committed ncu record only while the kernel source
    it was captured from is unchanged; any edit of that file turns it into null."""
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "decoder_only_transformer_sm_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k_attention_tc.cu").write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_sha("k_attention_tc.cu")
    assert len(sha) == 16
    (prof / "dram_traffic.json").write_text(
        '{"attention bwd": {"kernel_source_sha": "%s", "bytes_per_launch": 123.0}}' % sha)
    assert bench.traffic_for("attention bwd") == 123.0
    assert bench.traffic_for("attention fwd") is None           # no record for that site
    (src / "k_attention_tc.cu").write_text("// kernel v2\n")
    assert bench.traffic_for("attention bwd") is None           # source changed since the capture
