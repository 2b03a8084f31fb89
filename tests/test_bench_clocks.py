"""Host logic of the benchmark's clock record, with a stand-in for nvidia-smi.

The record must come from samples taken inside the timed region only, report the
median SM clock of the samples under load, and name every throttle reason seen;
and each rank must sample the GPU it drives."""
import os

import pytest

import bench

IDLE = "0, 1005, 1965, 120.50, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active\n"


class _FakeSmi:
    """Writes one sample at start, as nvidia-smi does shortly after launch."""

    def __init__(self, args, stdout=None, stderr=None):
        assert args[0] == "nvidia-smi" and "--format=csv,noheader,nounits" in args
        stdout.write(IDLE)
        stdout.flush()

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def kill(self):
        pass


def test_only_samples_after_start_count(monkeypatch):
    monkeypatch.setattr(bench.subprocess, "Popen", _FakeSmi)
    s = bench.ClockSampler("0")
    s.start()
    assert s.skip == 1  # the sample taken before the timed region is dropped
    for line in (
        "0, 1935, 1965, 700.00, 0x4, Not Active, Not Active, Not Active, Active\n",
        "0, 1905, 1965, 750.25, 0x4, Not Active, Not Active, Not Active, Active\n",
        "0, 1965, 1965, 300.00, 0x0, Not Active, Not Active, Not Active, Not Active\n",
        "0, 600, 1965, 90.00, 0x0, Not Active, Not Active, Not Active, Not Active\n",  # idle
    ):
        s.fh.write(line)
    rec = s.stop()
    assert rec["samples"] == 3  # samples under load (above 250 W)
    assert rec["sm_mhz"] == 1935.0
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["power_w_max"] == 750.25


def test_thermal_reason_is_reported(monkeypatch):
    monkeypatch.setattr(bench.subprocess, "Popen", _FakeSmi)
    s = bench.ClockSampler("0")
    s.start()
    s.fh.write("0, 1500, 1965, 800.00, 0x40, Not Active, Active, Not Active, Not Active\n")
    rec = s.stop()
    assert rec["reasons"] == ["hw_thermal_slowdown"] and rec["samples"] == 1


def test_missing_nvidia_smi(monkeypatch):
    def _absent(*args, **kwargs):
        raise FileNotFoundError("nvidia-smi")

    monkeypatch.setattr(bench.subprocess, "Popen", _absent)
    s = bench.ClockSampler("0")
    s.start()
    rec = s.stop()
    assert rec["samples"] == 0 and rec["reasons"] == ["nvidia-smi unavailable"]
    assert not os.path.exists(s.path)  # no temporary file left behind


@pytest.mark.parametrize("env,local_rank,want", [
    (None, 0, "0"),
    (None, 3, "3"),                          # nothing set: every rank sees every GPU
    ("4,5,6,7", 0, "4"),
    ("4,5,6,7", 2, "6"),
    ("GPU-aaaa, GPU-bbbb", 1, "GPU-bbbb"),
    ("", 1, "1"),
])
def test_physical_gpu(monkeypatch, env, local_rank, want):
    if env is None:
        monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    else:
        monkeypatch.setenv("CUDA_VISIBLE_DEVICES", env)
    assert bench.physical_gpu(local_rank) == want
