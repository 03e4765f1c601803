"""Host-side logic of bench.py on CPU: the algorithmic work per token, the clock
record, the recorded-traffic lookup and the peaks it divides by."""

import json
import os
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_attention_la2_b200 import inputs as I  # noqa: E402


def test_work_per_token_matches_the_block_algorithm():
    w64 = I.WORKLOADS["bf16_b4h16_n2k"]
    assert bench.bytes_per_token(w64) == 1024            # read Q, K, V and write O, bf16
    # S (2 Bk d), P V (2 Bk dv), Q KV and the state update (2 d dv each)
    assert bench.flops_per_token(w64) == 2 * 64 * 256 + 4 * 128 * 128 == 98304
    assert bench.flops_per_token(w64, causal=False) == 4 * 128 * 128
    assert bench.flops_per_token(I.sweep_workload(1024, 128)) == 131072
    assert bench.bytes_per_token(I.WORKLOADS["fp32_small"]) == (2 * 64 + 2 * 64) * 4


def test_work_per_token_of_a_forward_backward_step():
    w = I.WORKLOADS["bf16_fwdbwd_b2h32_n8k"]
    # forward 1024 B; backward reads Q, K, V, dO and writes dQ, dK, dV: 1792 B
    assert bench.bytes_per_token(w) == 1024 + 1792 == 2816
    assert bench.flops_per_token(w) == 98304 + 2 * 64 * (3 * 128 + 2 * 128) + 10 * 128 * 128
    assert bench.flops_per_token(w) == 98304 + 245760


def test_op_roofline_counts_every_launch_of_the_step():
    w = I.WORKLOADS["bf16_long_512k"]
    per_kernel = {"main": {"launches": 2, "ms": 1.5}, "state": {"launches": 2, "ms": 0.5}}
    r = bench.op_roofline(w, per_kernel, 2, 6545.0, "measured")
    step_s = (1.5 + 0.5) / 2 / 1e3
    assert r["scope"] == "op" and r["kernel"] == "main"
    assert abs(r["achieved"] - w.tokens * 1024 / step_s / 1e9) < 1e-6
    assert abs(r["frac"] - r["achieved"] / 6545.0) < 1e-12
    assert abs(r["kernels"]["state"]["share"] - 0.25) < 1e-12
    assert r["kernels"]["main"]["launches_per_step"] == 1
    assert r["traffic"] is None  # no capture of these kernels on the current sources
    assert bench.op_roofline(w, {}, 0, 6545.0, "measured") is None


def test_oracle_samples_are_bounded():
    long = I.WORKLOADS["bf16_long_512k"]
    form, n, text = bench.oracle_sample_plan(long)
    assert form == "rnn" and n == bench.RNN_SAMPLE_TOKENS and "RNN form" in text
    form, n, _ = bench.oracle_sample_plan(I.WORKLOADS["bf16_b4h16_n2k"])
    assert (form, n) == ("left", 2048)
    form, n, text = bench.oracle_sample_plan(I.WORKLOADS["bf16_fwdbwd_b2h32_n8k"])
    assert (form, n) == ("left", 8192) and "dQ, dK, dV" in text
    small = I.WORKLOADS["fp32_small"]
    n, t = bench.oracle_sample(small, 0)
    assert n == 256 and t > 0


def test_config_names_the_form():
    w = I.WORKLOADS["bf16_b4h16_n2k"]
    assert bench.config_of(w)["workload"].startswith("bf16_b4h16_n2k: causal forward")
    c = bench.config_of(w, causal=False)
    assert "non-causal forward" in c["workload"] and c["causal"] is False


def _sampler_with(lines):
    s = bench.ClockSampler(0)
    s.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0,
                            "kill": lambda self: None})()
    s.lines = lines
    return s


def test_clock_record_median_reasons_and_window():
    row = "0, {sm}, 1965, 900.5, 0x0, {hw}, Not Active, Not Active, {pc}"
    t = time.monotonic()
    lines = [(t - 5.0, row.format(sm=800, hw="Not Active", pc="Not Active")),   # before the window
             (t + 0.1, row.format(sm=1900, hw="Not Active", pc="Active")),
             (t + 0.2, row.format(sm=1800, hw="Not Active", pc="Active")),
             (t + 0.3, row.format(sm=1860, hw="Active", pc="Active")),
             (t + 9.0, "garbage line")]
    rec = _sampler_with(lines).stop(t, t + 1.0)
    assert rec["sm_mhz"] == 1860.0 and rec["sm_max_mhz"] == 1965.0 and rec["samples"] == 3
    assert rec["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert _sampler_with([(t, "garbage")]).stop() is None


def test_recorded_traffic_needs_the_current_sources(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"k/w": {"source_hash": "abc", "bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_hash", lambda: "abc")
    assert bench.recorded_traffic("k", "w") == 123
    assert bench.recorded_traffic("k", "other") is None
    monkeypatch.setattr(bench, "source_hash", lambda: "changed")
    assert bench.recorded_traffic("k", "w") is None  # counters of older kernels are not reported


def test_committed_traffic_record_shows_no_wasted_rereads():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    e = rec["la2_fwd_sm100/bf16_b4h16_n2k"]
    assert len(e["source_hash"]) == 16
    # DRAM traffic may not be far above the algorithmic bytes (no wasted re-reads)
    w = I.WORKLOADS["bf16_b4h16_n2k"]
    assert e["bytes_per_launch"] <= 1.2 * w.tokens * bench.bytes_per_token(w)


def test_peaks_fall_back_without_measurements(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    hbm, tf, tfs, kind = bench.peaks()
    assert (hbm, tf, kind) == (bench.FALLBACK_HBM_GBS, bench.FALLBACK_BF16_TFLOPS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1370.0}))
    assert bench.peaks() == (6500.0, 1600.0, 1370.0, "measured")
