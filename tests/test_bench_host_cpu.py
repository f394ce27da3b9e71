"""Host logic of bench.py that needs no GPU: the clock sampler's parsing of
nvidia-smi output (fed by a stand-in script on PATH) and the rule that a
profile's DRAM traffic is used only when it was taken on the current kernel
sources."""
import os
import shutil
import stat
import time

import pytest

import bench


def _fake_smi(tmp_path, lines):
    script = tmp_path / "nvidia-smi"
    body = "\n".join(f"echo '{ln}'" for ln in lines)
    script.write_text(f"#!/bin/sh\n{body}\nexec sleep 30\n")
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


@pytest.mark.skipif(shutil.which("sh") is None, reason="needs /bin/sh")
def test_clock_sampler_parses_clocks_and_reasons(tmp_path, monkeypatch):
    lines = [
        "0, 1950, 1965, 640.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 700.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1980, 1965, 701.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ.get("PATH", ""))
    s = bench.ClockSampler("0")
    s.start()
    time.sleep(0.5)
    out = s.stop()
    assert out == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_sampler_reports_throttle_reasons(tmp_path, monkeypatch):
    lines = ["0, 1100, 1965, 990.0, 0x48, Active, Not Active, Active, Not Active"]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ.get("PATH", ""))
    s = bench.ClockSampler("0")
    s.start()
    time.sleep(0.5)
    out = s.stop()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"] and out["sm_mhz"] == 1100.0


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler("0")
    s.start()
    assert s.stop() is None


def test_profiled_traffic_only_for_current_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "bitlinear_bitnet_quant_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("// kernel a\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "profiles" / "linear_x.txt").write_text(
        f"# header: with a colon\nkernel: k\nkernel_source_hash: {h}\ndram_bytes_per_launch: 4485632\n")
    assert bench.profiled_traffic("linear_x") == 4485632.0
    assert bench.profiled_traffic("linear_missing") is None
    # the stacked-layer summaries give the bytes of every linear launch of a step
    (tmp_path / "profiles" / "linear_y.txt").write_text(
        f"kernel: all launches of a step\nkernel_source_hash: {h}\ndram_bytes_per_step: 412703232\n")
    assert bench.profiled_traffic("linear_y") == 412703232.0
    (csrc / "a.cu").write_text("// kernel a, changed\n")
    assert bench.kernel_source_hash() != h
    assert bench.profiled_traffic("linear_x") is None and bench.profiled_traffic("linear_y") is None


def test_targets_cover_the_decode_and_prefill_configs():
    """The decode GEMV (>= 70 % of HBM) and the prefill GEMM (>= 50 % of int8)
    targets are attached to exactly those bench lines."""
    assert set(bench.TARGET_FRAC) == {"decode_m1", "decode_m4", "decode_m16", "prefill"}
    assert all(bench.TARGET_FRAC[k] == 0.70 for k in ("decode_m1", "decode_m4", "decode_m16"))
    assert bench.TARGET_FRAC["prefill"] == 0.50
    assert set(bench.TARGET_FRAC) <= set(bench.WORKLOADS)


def test_all_cores_cpu_baseline_line():
    c = bench.WORKLOADS["tiny"]()
    r = bench.cpu_baseline_omp(c, budget_s=0.2)
    assert r["value"] > 0 and r["unit"] == "tokens/s" and r["cores"] >= 1
    assert r["kind"] == "oracle (C++, OpenMP)" and c["name"] in r["sample"]
