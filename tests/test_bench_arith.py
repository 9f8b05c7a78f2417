"""bench.py's roofline arithmetic, on CPU: the algorithmic FLOPs of the two
gated kernels against their closed forms on the bench workloads, the achieved
rate and fraction of a roofline line, the choice of peak, and the DRAM traffic
taken from a committed ncu summary only while the kernel's source is unchanged."""
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_lmhead_and_attention_flops_on_longctx(bench):
    fb = bench.flops_bytes(bench.workload_cfg("longctx"))
    # 4 canvases of 256 rows, d = 2816, V = 262,144: 2 M d V
    assert fb["flops_lm"] == 2 * (4 * 256) * 2816 * 262144 == 1_511_828_488_192
    # per request: QK^T and PV, 2 flops per MAC each, 256 queries x (32,768 + 256) keys x 128 x 16 heads
    assert fb["flops_attn"] == 4 * (2 * 2 * 256 * (32768 + 256) * 128 * 16) == 277_025_390_592
    # the weights once (bf16) dominate the LM head's bytes
    assert 262144 * 2816 * 2 <= fb["bytes_lm"] < 262144 * 2816 * 2 * 1.01


def test_fp8_lm_head_counts_one_byte_per_weight(bench):
    bf = bench.flops_bytes(bench.workload_cfg("vocab262k"))
    f8 = bench.flops_bytes(bench.workload_cfg("vocab262k_fp8"))
    assert f8["flops_lm"] == bf["flops_lm"]
    assert abs(f8["bytes_lm"] - bf["bytes_lm"] / 2) < 0.01 * bf["bytes_lm"]


def test_roofline_line_arithmetic(bench):
    peaks = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    flops, bytes_, ms = 1.5e12, 1.5e9, 1.25
    line = bench.kernel_roofline("lmhead", "k", flops, bytes_, ms, peaks, "sustained", None)
    assert line["achieved"] == pytest.approx(flops / (ms / 1e3) / 1e12)
    assert line["peak"] == 1400.0 and line["frac"] == pytest.approx(line["achieved"] / 1400.0)
    assert line["roofline_ms"] == pytest.approx(max(flops / 1590e12, bytes_ / 6650e9) * 1e3)
    burst = bench.kernel_roofline("lmhead", "k", flops, bytes_, ms, peaks, "burst", 123)
    assert burst["peak"] == 1590.0 and burst["traffic"] == 123
    fp8 = bench.kernel_roofline("lmhead", "k", flops, bytes_, ms, peaks, "burst", None, fp8=True)
    assert fp8["peak"] == 2 * 1590.0 and fp8["frac"] == pytest.approx(burst["frac"] / 2)


def test_peak_kind(bench):
    assert bench.peak_kind_of(0.4, {"reasons": ["sw_power_cap"]}) == "sustained"
    assert bench.peak_kind_of(0.4, {"reasons": []}) == "burst"
    assert bench.peak_kind_of(0.4, None) == "burst"
    assert bench.peak_kind_of(1.5, {"reasons": []}) == "sustained"


def test_traffic_only_for_unchanged_sources(bench, tmp_path):
    prof = os.path.join(ROOT, "profiles")
    files = [f for f in os.listdir(prof) if f.startswith("traffic_") and f.endswith(".json")]
    assert files, "no committed traffic summaries"
    for f in files:
        t = json.load(open(os.path.join(prof, f)))
        assert f == f"traffic_{t['kernel']}_{t['workload']}.json" and t["bytes_per_launch"] > 0
        fresh = t["source_sha256_16"] == bench.source_sha(t["source"])
        assert bench.traffic_of(t["kernel"], t["workload"]) == (t["bytes_per_launch"] if fresh else None)
    assert bench.traffic_of("no_such_kernel", "longctx") is None
    # a summary whose recorded hash no longer matches its kernel's source is ignored
    t = json.load(open(os.path.join(prof, files[0])))
    t["source_sha256_16"] = "0" * 16
    stale_root = tmp_path
    os.makedirs(stale_root / "profiles")
    json.dump(t, open(stale_root / "profiles" / files[0], "w"))
    os.makedirs(stale_root / os.path.dirname(t["source"]))
    with open(os.path.join(ROOT, t["source"]), "rb") as src, open(stale_root / t["source"], "wb") as dst:
        dst.write(src.read())
    old = bench.ROOT
    try:
        bench.ROOT = str(stale_root)
        assert bench.traffic_of(t["kernel"], t["workload"]) is None
    finally:
        bench.ROOT = old
