"""Work and byte counts behind the bench line, on the CPU: the forward's
algorithmic bytes of the LongNet-base layer are the kept rows read three times
plus the merged output written once, and the labelled 8 d backward rate is 0.8
of the 10 d one."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_long_sequence_dilated_b200 import flops  # noqa: E402
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS  # noqa: E402


def test_longnet_base_kept_rows_and_bytes():
    wl = WORKLOADS["longnet_base_32k"]
    # r = 1, 2, 4 keep N / r rows per head; r = 6 keeps 2731 + 2731 (segments of 16384,
    # offsets h mod 6) or 2730 + 2730, r = 12 keeps 2731 or 2730 of 32768 (offset h mod 12)
    per_head = [32768 + 16384 + 8192 + sum(flops.segment_counts(32768, 16384, 6, h))
                + sum(flops.segment_counts(32768, 32768, 12, h)) for h in range(12)]
    assert flops.kept_rows(1, 32768, 12, wl.patterns) == sum(per_head) == 786432
    assert flops.fwd_bytes(1, 32768, 12, 64, wl.patterns) == 786432 * 384 + 393216 * 132
    assert (flops.fwd_bytes(1, 32768, 12, 64, wl.patterns, out_res=True)
            - flops.fwd_bytes(1, 32768, 12, 64, wl.patterns)) == 393216 * 128


@pytest.mark.parametrize("name", ["sweep_8192", "sweep_1048576", "wide_128k"])
def test_fwd_bytes_are_the_kept_rows_plus_the_output(name):
    wl = WORKLOADS[name]
    rows = flops.kept_rows(wl.B, wl.N, wl.H, wl.patterns)
    # in the geometric families r divides w, so pattern (w, r) keeps N / r rows per head
    assert rows == sum(wl.B * wl.H * (wl.N // r) for (_, r) in wl.patterns)
    assert flops.fwd_bytes(wl.B, wl.N, wl.H, wl.d, wl.patterns) == \
        rows * 6 * wl.d + wl.B * wl.N * wl.H * (2 * wl.d + 4)


def test_extra_counts():
    wl = WORKLOADS["longnet_base_32k"]
    args = (wl.B, wl.N, wl.H, wl.d, wl.patterns, wl.causal)
    e = bench.extra_counts(*args, 0.5, 1.0, 6500.0, True)
    fb = flops.fwd_bytes(*args[:5], out_res=True)
    assert e["fwd_algorithmic_bytes"] == fb
    assert e["fwd_hbm_gbs"] == pytest.approx(fb / 0.5e-3 / 1e9)
    assert e["fwd_frac_of_hbm"] == pytest.approx(e["fwd_hbm_gbs"] / 6500.0)
    b10 = flops.bwd_flops(*args) / 1e-3 / 1e12
    assert e["bwd_tflops_8d_no_recompute"] == pytest.approx(0.8 * b10)
    assert "bwd_tflops_8d_no_recompute" not in bench.extra_counts(*args, 0.5, None, 6500.0,
                                                                    False)
    assert bench.hbm_peak() > 0
