"""Host logic of bench.py that needs no GPU: the committed DRAM-traffic figure is reported
only for the GEMM source it was measured on, the reference arm (the CPU oracle) prints
one JSON line with the contract's keys, and the single-thread oracle quantizer rate is
measured on the requested rows."""
import argparse
import json

import bench
import synth


def test_traffic_only_for_the_measured_gemm_source(monkeypatch):
    with open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        committed = json.load(f)
    entry = committed["nvfp4_attn_1mp"]
    if entry["source_hash"] == bench.gemm_source_hash():
        assert bench.ncu_traffic("nvfp4_attn_1mp") == entry["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "gemm_source_hash", lambda: "0" * 16)
    assert bench.ncu_traffic("nvfp4_attn_1mp") is None         # another source: no figure
    assert bench.ncu_traffic("no_such_workload") is None


def test_reference_arm_line(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "0")
    args = argparse.Namespace(gpus=1, steps=1, warmup=0, impl="reference",
                              workload="nvfp4_tiny", m=0)
    assert bench.run_reference(args) == 0
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC
    assert d["unit"] == "TFLOP/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "nvfp4_tiny"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_single_thread_quantizer_rate():
    wl = synth.WORKLOADS["nvfp4_tiny"]
    r = bench.cpu_quantize_one_thread(wl, 4096)
    assert r["threads"] == 1 and r["unit"] == "GB/s" and r["value"] > 0
    assert r["rows"] == wl.M                                    # clamped to the workload
    wl = synth.WORKLOADS["fp8r_1mp"]
    r = bench.cpu_quantize_one_thread(wl, 64)
    assert r["rows"] == 64 and r["value"] > 0
