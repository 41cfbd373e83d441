"""Host-side arithmetic of bench.py that feeds its JSON line: the
algorithmic byte count behind the roofline, the nvidia-smi clock parser and
the staleness guard on the committed DRAM-traffic figures.  No GPU."""

import json
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from weight_only_quantized_prologue_b200 import _native  # noqa: E402

WEIGHT_FORMATS = ("int4", "int4_asym", "nvfp4", "mxfp4", "fp8", "fp8_static")


@pytest.mark.parametrize("fmt", WEIGHT_FORMATS)
@pytest.mark.parametrize("K,N", [(128, 16), (3072, 4096), (256, 512)])
def test_weight_bytes_match_abi_storage(fmt, K, N):
    # the weight part of the count is exactly the buffers dqgemm_create reads:
    # packed codes + scales (+ the NVFP4 fp32 global scale, passed by value
    # but still one fp32 per call)
    pshape, pdt, sshape, sdt = _native.storage_shapes(fmt, K, N)
    stored = int(np.prod(pshape)) * np.dtype(pdt).itemsize + int(np.prod(sshape)) * np.dtype(sdt).itemsize
    stored += 4 if fmt == "nvfp4" else 0
    assert bench.algorithmic_bytes(fmt, 0, K, N, bias=False) == stored


@pytest.mark.parametrize("fmt", WEIGHT_FORMATS)
def test_activation_output_bias_terms(fmt):
    K, N = 3072, 4096
    w = bench.algorithmic_bytes(fmt, 0, K, N, bias=False)
    # x bf16 [M, K], y bf16 [M, N], bias bf16 [N]
    assert bench.algorithmic_bytes(fmt, 32, K, N, bias=False) - w == 32 * K * 2 + 32 * N * 2
    assert bench.algorithmic_bytes(fmt, 32, K, N, bias=True) - bench.algorithmic_bytes(fmt, 32, K, N, bias=False) \
        == N * 2


def test_headline_bytes_int4():
    # Linear(3072 -> 4096), M = 32, INT4 g128 with bias: 6291456 packed +
    # 196608 scales + 196608 x + 262144 y + 8192 bias
    assert bench.algorithmic_bytes("int4", 32, 3072, 4096) == 6955008


def test_unknown_format_raises():
    with pytest.raises(ValueError):
        bench.algorithmic_bytes("int3", 32, 3072, 4096)


def test_clock_parser():
    lines = [
        "0, 1965, 1965, 612.40, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "0, 1950, 1965, 701.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active\n",
        "0, 1980, 1965, 655.00, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n",
        "garbage\n",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
    ]
    c = bench.parse_clock_samples(lines)
    assert c["samples"] == 3
    assert c["sm_mhz"] == 1965.0
    assert c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"]


def test_clock_parser_thermal_and_empty():
    lines = ["1, 1200, 1965, 990, 0x48, Active, Not Active, Active, Not Active\n"]
    assert bench.parse_clock_samples(lines)["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clock_samples([]) is None
    assert bench.parse_clock_samples(["x, y\n"]) is None


def test_traffic_guard(tmp_path, monkeypatch):
    # DRAM figures are reported only while the kernel sources hash to the
    # value they were captured on
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(
        json.dumps({"kernel_source_hash": "abc", "per_launch_bytes": {"int4": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "abc")
    assert bench.ncu_traffic() == {"int4": 123}
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "def")
    assert bench.ncu_traffic() is None


def test_source_hash_tracks_csrc():
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0
    assert h == bench.kernel_source_hash()


def test_clock_sampler_with_fake_nvidia_smi(tmp_path, monkeypatch):
    # the sampler process end to end, with a stand-in nvidia-smi that prints
    # two samples and then idles until it is terminated
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    "echo '0, 1965, 1965, 600.0, 0x0, Not Active, Not Active, Not Active, Not Active'\n"
                    "echo '0, 1935, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "exec sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    s = bench.ClockSampler(0)
    s.start()
    assert s.proc is not None
    import time
    deadline = time.time() + 10
    while time.time() < deadline and os.path.getsize(s.path) == 0:
        time.sleep(0.05)
    time.sleep(0.2)
    c = s.stop()
    assert c == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}
    assert not os.path.exists(s.path)


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop() is None
    assert not os.path.exists(s.path)


def test_reference_arm_line():
    # the reference arm times the oracle on the host cores; rank 0 alone
    # prints, other ranks do no work
    import argparse
    from weight_only_quantized_prologue_b200 import synthetic  # noqa: F401

    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args, rank=1, world=2) is None
    res = bench.run_reference(args, rank=0, world=1)
    assert res["impl"] == "reference" and res["dtype"] == "f64" and res["higher_is_better"] is False
    assert res["value"] > 0 and res["unit"] == bench.UNIT and res["metric"] == bench.METRIC
    assert res["cpu_baseline"]["kind"] == "oracle" and res["cpu_baseline"]["value"] == res["value"]
    assert res["e2e"] == {"value": res["value"], "unit": res["unit"], "h2d_bytes_per_step": 0,
                          "d2h_bytes_per_step": 0}
    json.dumps(res)
