"""Host logic of bench.py that needs no GPU: the source-keyed DRAM traffic record,
the peak bandwidth source, the format switch and the clock summary."""
from __future__ import annotations

import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_record_is_reported_only_for_the_captured_sources(monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    key = "quantize_batch_nvfp4_razer_sse"
    if rec[key]["source_sha256"] == bench.kernel_source_sha256(key):
        assert bench.traffic_record(key) == rec[key]["dram_bytes_per_element"]
    assert bench.traffic_record("no_such_kernel") is None
    monkeypatch.setattr(bench, "kernel_source_sha256", lambda k: "0" * 64)
    assert bench.traffic_record(key) is None


def test_traffic_record_hash_covers_every_listed_source(monkeypatch, tmp_path):
    """Changing any one of the listed translation units changes the hash."""
    from activation_quantization_block_b200 import _build
    files = bench.TRAFFIC_SOURCES["quantize_batch"]
    for name in files:
        (tmp_path / name).write_bytes(open(os.path.join(_build.CSRC, name), "rb").read())
    monkeypatch.setattr(_build, "CSRC", str(tmp_path))
    h0 = bench.kernel_source_sha256("quantize_batch_nvfp4_razer_sse")
    for name in files:
        p = tmp_path / name
        orig = p.read_bytes()
        p.write_bytes(orig + b"\n")
        assert bench.kernel_source_sha256("quantize_batch_nvfp4_razer_sse") != h0, name
        p.write_bytes(orig)
    assert bench.kernel_source_sha256("quantize_batch_nvfp4_razer_sse") == h0


def test_peaks_read_the_measured_file_else_the_fallback(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps({"hbm_gbs": 6543.1, "bf16_tflops": 1600}))
    assert bench.peaks() == (6543.1, "measured")
    (tmp_path / "MEASURED_PEAKS.json").write_text("{not json")
    assert bench.peaks() == (bench.FALLBACK_HBM_GBS, "fallback")


def test_set_format_renames_the_workload(monkeypatch):
    monkeypatch.setattr(bench, "FMT", bench.FMT)
    monkeypatch.setattr(bench, "WORKLOAD", bench.WORKLOAD)
    assert "NVFP4_RAZER," in bench.WORKLOAD
    bench.set_format("nvfp4_razer_w")
    assert bench.FMT == "nvfp4_razer_w" and "NVFP4_RAZER_W," in bench.WORKLOAD


@pytest.mark.parametrize("lines,want", [
    ([], {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}),
    (["0, 1965, 1965, 950.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"] * 3,
     {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}),
    (["0, 1800, 1965, 1000.0, 0x4, Not Active, Not Active, Not Active, Active\n",
      "0, 1900, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
      "0, 1300, 1965, 700.0, 0x8, Active, Not Active, Not Active, Not Active\n",
      "garbage line\n"],
     {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 3}),
])
def test_clock_summary(lines, want):
    assert bench.summarize_clock_lines(lines) == want


def test_clock_sampler_reads_a_running_nvidia_smi(monkeypatch, tmp_path):
    """The sampler end to end against a stand-in nvidia-smi on PATH that prints CSV lines."""
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nwhile true; do echo '0, 1965, 1965, 900.0, 0x0, Not Active, Not Active, "
                    "Not Active, Active'; sleep 0.05; done\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = bench.ClockSampler(0)
    s.start()
    import time
    time.sleep(0.5)
    got = s.stop()
    assert got["samples"] >= 2 and got["sm_mhz"] == 1965.0 and got["reasons"] == ["sw_power_cap"]


def test_sha256_of_tensors_is_the_digest_of_their_bytes():
    import hashlib

    import numpy as np
    import torch
    a = torch.arange(12, dtype=torch.float32).to(torch.bfloat16).reshape(3, 4)
    b = torch.arange(6, dtype=torch.uint8)
    want = hashlib.sha256(a.view(torch.int16).numpy().view(np.uint8).tobytes() + b.numpy().tobytes()).hexdigest()
    assert bench.sha256_of([a, b]) == want
    wide = torch.zeros(4, 8, dtype=torch.bfloat16)
    assert bench.sha256_of([wide[:, :4]]) == bench.sha256_of([torch.zeros(4, 4, dtype=torch.bfloat16)])
    assert bench.sha256_of([object()]).startswith("unavailable:")


def test_cpu_baseline_leg_checks_the_gpu_results_against_the_oracle():
    """The oracle leg quantizes the given input bytes and compares the given results with its
    own: equal results report parity, and one changed code byte, scale byte, tensor scale or
    an MSE off by more than 1e-5 is caught.  (Results here come from the oracle itself.)"""
    import numpy as np
    import oracle

    import bench
    from activation_quantization_block_b200 import synthetic
    xs = [synthetic.bf16_bits(synthetic.llm_weight(r, c, seed=70 + i)) for i, (r, c) in enumerate([(32, 64), (8, 256)])]
    layer0 = []
    for xb in xs:
        codes, scales, ts, sse = oracle.quantize(xb, bench.FMT, False)
        layer0.append((xb, codes, scales, float(ts), sse / xb.size))
    base, parity = bench.cpu_baseline_leg(layer0)
    assert base["kind"] == "oracle" and base["value"] > 0 and "own input bytes" in base["sample"]
    assert parity["layer0_codes_scales_equal"] and parity["tensor_scales_equal"] and parity["mse_max_rel"] < 1e-12
    bad_codes = layer0[1][1].copy()
    bad_codes[3, 5] ^= 0x10
    _, p = bench.cpu_baseline_leg([layer0[0], (xs[1], bad_codes) + layer0[1][2:]])
    assert not p["codes_equal"] and p["scales_equal"] and not p["layer0_codes_scales_equal"]
    bad_scales = layer0[0][2].copy()
    bad_scales[0, 0] ^= 1
    _, p = bench.cpu_baseline_leg([(xs[0], layer0[0][1], bad_scales) + layer0[0][3:]])
    assert not p["scales_equal"]
    _, p = bench.cpu_baseline_leg([layer0[0][:3] + (np.nextafter(np.float32(layer0[0][3]), np.float32(1)),
                                                     layer0[0][4])])
    assert not p["tensor_scales_equal"]
    _, p = bench.cpu_baseline_leg([layer0[0][:4] + (layer0[0][4] * (1 + 3e-5),)])
    assert p["mse_max_rel"] > p["mse_tolerance"]
