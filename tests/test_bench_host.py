"""Host-side arithmetic of bench.py (CPU only): algorithmic bytes and flops,
the roofline fraction, the launch count per step, the gating of the captured
DRAM traffic on the device-code hash, and the parsing of the clock samples."""

import os

import pytest

import bench
from linear_attention_diffusion_phi_b200.inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_and_flops():
    # q, k, v read once and out written once, 2 bytes per bf16 element
    assert bench.algorithmic_bytes(WORKLOADS["flux1024"]) == 4 * 24 * 4608 * 128 * 2 == 113_246_208
    assert bench.algorithmic_bytes(WORKLOADS["causal32k"]) == 4 * 4 * 8 * 32768 * 64 * 2
    # E4M3: one byte per q, k, v element, bf16 out
    assert bench.algorithmic_bytes(WORKLOADS["flux1024"], e4m3=True) == (3 + 2) * 24 * 4608 * 128
    # the projection adds W, one [D, F] matrix per head
    assert bench.algorithmic_bytes(WORKLOADS["proj256"]) == 113_246_208 + 24 * 128 * 256 * 2
    # two contractions of 2 N F D each, plus the two N x D x F projections
    f = 24 * (2 * 2 * 4608 * 256 * 128 + 2 * 2 * 4608 * 128 * 256)
    assert bench.algorithmic_flops(WORKLOADS["proj256"]) == f
    assert bench.algorithmic_flops(WORKLOADS["flux1024"]) == 24 * 2 * 2 * 4608 * 128 * 128


def test_roofline_fraction_and_launches():
    roof, launches = bench.roofline(WORKLOADS["flux1024"], 28.9e-6, 6551.0, 1688.0, "measured", 148)
    assert launches == 1 and roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["achieved"] == pytest.approx(113_246_208 / 28.9e-6 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / 6551.0) and 0.59 < roof["frac"] < 0.61
    roof, launches = bench.roofline(WORKLOADS["proj256"], 54.5e-6, 6551.0, 1688.0, "measured", 148)
    assert launches == 3 and roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["frac"] == pytest.approx(bench.algorithmic_flops(WORKLOADS["proj256"]) / 54.5e-6 / 1e12 / 1688.0)
    assert roof["hbm"]["unit"] == "GB/s"


def test_causal_launch_count_follows_the_segment_plan():
    # 32 heads on 148 SMs: four segments of 64 chunks per head, state + chunk kernels
    assert bench.kernels_per_step(WORKLOADS["causal32k"], 148)[1] == 2
    # as many heads as SMs: one segment per head, the chunk kernel alone
    assert bench.kernels_per_step(WORKLOADS["causal32k"].with_(B=37), 148)[1] == 1


def test_traffic_is_reported_only_for_the_captured_device_code(monkeypatch):
    profiles = ""
    for name in os.listdir(os.path.join(ROOT, "profiles")):
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            profiles += fh.read()
    for name, (nbytes, files, digest) in bench.NCU_TRAFFIC.items():
        # the capture's summary names the code version it measured
        assert digest in profiles, name
        got = bench.captured_traffic(None, name)
        assert got == (nbytes if bench.source_hash(files) == digest else None)
    monkeypatch.setattr(bench, "source_hash", lambda files: "0" * 16)
    assert all(bench.captured_traffic(None, name) is None for name in bench.NCU_TRAFFIC)


class _Proc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def test_clock_samples_median_under_load_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1950, 1965, 990.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle, not counted
        "short, row",
    ]
    path = tmp_path / "clocks.csv"
    path.write_text("\n".join(rows) + "\n")
    cs = bench.ClockSampler(0)
    cs.path, cs.fh, cs.proc = str(path), open(path, "a"), _Proc()
    got = cs.stop()
    assert got["samples"] == 4 and got["sm_max_mhz"] == 1965.0
    # median power 965 W: the 990 W and 980 W samples count (1950, 1800 MHz)
    assert got["sm_mhz"] == 1875.0
    assert got["reasons"] == ["sw_power_cap"]
    assert not path.exists()
    assert bench.ClockSampler(0).stop()["reasons"] == ["nvidia-smi unavailable"]
