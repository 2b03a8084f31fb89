"""GPU parity of the forward pass against the float64 oracle (same seeded inputs).

Sizes the oracle finishes in seconds cover several tiles, ragged tails and
degenerate shapes in full; the full-size workloads are compared element by
element in tests/test_gpu_scale.py.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_dilated_b200 import dilattn
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import check_close, check_lse, to_device, to_f64

pytestmark = pytest.mark.gpu


def _run_full(B, N, H, d, pats, causal, dtype, seed=0):
    inp = make_inputs(B, N, H, d, seed, dtype)
    q, k, v = to_device(inp, dtype=dtype)
    out, lse = dilattn.fwd(q, k, v, pats, causal)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    want_o, want_l = oracle.fwd(inp["q"], inp["k"], inp["v"], pats, causal)
    check_close(to_f64(out), want_o, dtype, "out")
    check_lse(to_f64(lse), want_l, 2e-2 if dtype == "bf16" else 1e-4)


def test_tiny_f32_workload():
    wl = WORKLOADS["tiny_f32"]
    _run_full(wl.B, wl.N, wl.H, wl.d, wl.patterns, wl.causal, "f32", wl.seed)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pats", [
    [(256, 1), (512, 2), (1024, 4)],
    [(384, 1), (700, 3), (1000, 6), (1100, 12)],     # ragged: w and r do not divide N
    [(1100, 1)],                                      # one long segment, ragged tail tile
    [(64, 5), (96, 200), (1100, 7)],                  # r > w: empty segments; tiny tiles
    [(256, 1), (1024, 1), (512, 2)],                  # two r = 1 patterns: the shorter merges
    [(100, 1), (37, 3), (1100, 1)],                   # merging tiles cross many short segments
])
def test_bf16_small(pats, causal):
    _run_full(2, 1100, 3, 64, pats, causal, "bf16", seed=1)


# degenerate sizes: one row; one partial tile with w > N; a tail of one row past
# a tile; r > N (heads whose offset h mod r is >= N keep no rows at all)
EDGE = [
    (1, 1, 2, [(1, 1)]),
    (1, 127, 2, [(128, 1), (64, 2), (256, 4)]),
    (3, 129, 1, [(128, 1), (129, 3)]),
    (1, 5, 8, [(5, 8), (4, 1)]),
]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,N,H,pats", EDGE)
def test_bf16_edge_sizes(B, N, H, pats, causal):
    _run_full(B, N, H, 64, pats, causal, "bf16", seed=4)


def test_bf16_d128_small():
    _run_full(1, 1536, 4, 128, [(256, 1), (512, 2), (1536, 4)], True, "bf16", seed=2)


def test_f32_ragged():
    _run_full(1, 700, 3, 64, [(256, 1), (300, 3), (700, 5)], False, "f32", seed=3)


def test_unselected_rows_zero():
    # (w, r) = (40, 16): only every 16th row of a segment is kept; the rest get O = 0, lse = -inf
    inp = make_inputs(1, 300, 16, 64, 5, "bf16")
    q, k, v = to_device(inp)
    pats = [(40, 16)]
    out, lse = dilattn.fwd(q, k, v, pats, True)
    want_o, want_l = oracle.fwd(inp["q"], inp["k"], inp["v"], pats, True)
    check_close(to_f64(out), want_o, "bf16", "out")
    check_lse(to_f64(lse), want_l, 2e-2)


def test_train_check_workload_full():
    wl = WORKLOADS["train_check_2k"]
    _run_full(wl.B, wl.N, wl.H, wl.d, wl.patterns, wl.causal, wl.dtype, wl.seed)


@pytest.mark.parametrize("N,H,pats", [
    (32768, 12, WORKLOADS["longnet_base_32k"].patterns),
    (1100, 3, [(384, 1), (700, 3), (1000, 6), (1100, 12)]),
    (300, 16, [(40, 16), (7, 3), (300, 1)]),
])
def test_selection_bit_exact(N, H, pats):
    sig = dilattn.selection(N, H, pats).cpu().numpy().view(np.uint32)
    want = oracle.selection_signature(N, H, pats)
    assert np.array_equal(sig, want)
