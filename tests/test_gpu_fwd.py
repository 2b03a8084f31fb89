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


# d = 128 runs 64-row key tiles against 128-row query tiles: ragged ends,
# segments shorter than a key tile, tail views, and partial query tiles whose
# causal extent ends inside a query tile
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,pats", [
    (1100, [(384, 1), (700, 3), (1000, 6), (1100, 12)]),
    (1100, [(100, 1), (37, 3), (1100, 1)]),
    (1000, [(64, 5), (96, 200), (1000, 7)]),
    (129, [(128, 1), (129, 3)]),
])
def test_bf16_d128_ragged(N, pats, causal):
    _run_full(2, N, 3, 128, pats, causal, "bf16", seed=6)


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


def _one_key_rows(N, H, pats, causal=True):
    """(n, h) of every row whose attended set is one key (itself) in exactly one
    pattern, from the oracle's kept-row sets: the result there must be that
    key's v, bit for bit (P = 1, l = 1, merge weight 1)."""
    count = np.zeros((H, N), dtype=np.int64)
    for w, r in pats:
        for h in range(H):
            for seg in oracle.kept_rows(N, w, r, h):
                count[h, seg] += np.arange(1, len(seg) + 1) if causal else len(seg)
    h_idx, n_idx = np.nonzero(count == 1)
    return n_idx, h_idx


@pytest.mark.parametrize("N,H,d,pats", [
    (16384, 8, 64, [(2048, 1), (4096, 2), (8192, 4), (16384, 8)]),
    (8192, 4, 128, [(512, 1), (2048, 2), (8192, 4)]),
    (4096, 3, 64, [(1024, 1)]),
])
def test_one_key_rows_return_v_exactly(N, H, d, pats):
    inp = make_inputs(1, N, H, d, 11, "bf16")
    q, k, v = to_device(inp)
    out, lse, res = dilattn.fwd_train(q, k, v, pats, True)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    n, h = _one_key_rows(N, H, pats)
    assert len(n) >= H
    got = out[0].float().cpu().numpy()[n, h]
    assert np.array_equal(got, inp["v"][0][n, h]), "a one-key row's out differs from its v"
    assert np.all(res[0].float().cpu().numpy()[n, h] == 0)
    s = np.einsum("id,id->i", inp["q"][0][n, h].astype(np.float64),
                  inp["k"][0][n, h].astype(np.float64)) / np.sqrt(d)
    np.testing.assert_allclose(lse.cpu().numpy()[0][h, n], s, rtol=0, atol=1e-5)


@pytest.mark.parametrize("d,pats", [
    (64, [(256, 1), (512, 2), (1024, 4)]),
    (128, [(256, 1), (512, 2), (1024, 4)]),
    (128, [(500, 2), (1100, 3)]),          # no r = 1 pattern: the merge pass writes it
])
def test_train_residual(d, pats):
    """dilattn_fwd_train returns the same out as dilattn_fwd; out_res is the
    rounding residual of out (at most half a bf16 unit in the last place of
    out), and out + out_res is closer to the float64 oracle than out alone
    (the residual removes the output rounding; what remains is the kernel's
    own error, P entering PV as bf16)."""
    inp = make_inputs(2, 1100, 3, d, 8, "bf16")
    q, k, v = to_device(inp)
    out, lse, res = dilattn.fwd_train(q, k, v, pats, True)
    out_inf, _ = dilattn.fwd(q, k, v, pats, True)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    assert torch.equal(out, out_inf)
    want_o, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], pats, True)
    o1 = to_f64(out)
    r = to_f64(res)
    o2 = o1 + r
    nz = o1 != 0
    ulp = np.exp2(np.floor(np.log2(np.abs(o1[nz]))) - 7)
    assert np.all(np.abs(r[nz]) <= ulp / 2)
    assert np.any(r != 0)
    rel = lambda x: np.linalg.norm(x - want_o) / np.linalg.norm(want_o)
    assert rel(o2) < rel(o1), (rel(o2), rel(o1))


@pytest.mark.parametrize("d", [64, 128])
def test_forward_is_deterministic(d):
    """No atomic operation touches the forward's data: every partial row is
    written by one tile and the merge adds the patterns in a fixed order, so
    two runs give the same bits (out, out_res and lse)."""
    inp = make_inputs(1, 8192, 4, d, 12, "bf16")
    q, k, v = to_device(inp)
    pats = [(1024, 1), (2048, 2), (4096, 4), (8192, 8)]
    o1, l1, r1 = dilattn.fwd_train(q, k, v, pats, True)
    o2, l2, r2 = dilattn.fwd_train(q, k, v, pats, True)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    assert torch.equal(o1, o2) and torch.equal(r1, r2) and torch.equal(l1, l2)
