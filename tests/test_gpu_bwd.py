"""GPU parity of the backward pass against the float64 oracle.

Full comparisons at sizes the oracle finishes in seconds: the bf16 training
forward (out and its rounding residual) then the backward, whose fp32
gradients are compared with the oracle's derivative of its own float64
forward. The full-size workloads are compared element by element in
tests/test_gpu_scale.py. At N = 1048576, sampled dq rows and dk/dv rows
across whole segments computed one by one by the oracle, plus two identities
that hold at any size: per (batch, head) the dk rows sum to 0
(every query's dS row sums to 0) and the dv rows sum to the dO rows of the
selected queries (every query's probabilities sum to 1).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_dilated_b200 import dilattn
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS, make_inputs
from tests import oracle_pool
from tests.gpu_util import check_close, to_device, to_f64

pytestmark = pytest.mark.gpu
NAMES = ("q", "k", "v", "dout")


def _run_full(B, N, H, d, pats, causal, dtype, seed=0):
    inp = make_inputs(B, N, H, d, seed, dtype, NAMES)
    q, k, v, do = to_device(inp, NAMES, dtype)
    if dtype == "bf16":
        out, lse, res = dilattn.fwd_train(q, k, v, pats, causal)
        dq, dk, dv = dilattn.bwd(q, k, v, out, lse, do, pats, causal, out_res=res)
    else:
        out, lse = dilattn.fwd(q, k, v, pats, causal)
        dq, dk, dv = dilattn.bwd(q, k, v, out, lse, do, pats, causal)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    # the oracle differentiates its own float64 forward
    gq, gk, gv = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["dout"], pats, causal)
    check_close(to_f64(dq), gq, dtype, "dq")
    check_close(to_f64(dk), gk, dtype, "dk")
    check_close(to_f64(dv), gv, dtype, "dv")


def test_train_check_workload():
    wl = WORKLOADS["train_check_2k"]
    _run_full(wl.B, wl.N, wl.H, wl.d, wl.patterns, wl.causal, wl.dtype, wl.seed)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pats", [
    [(384, 1), (700, 3), (1000, 6), (1100, 12)],
    [(64, 5), (96, 200), (1100, 7)],
    [(1100, 1)],
    [(256, 1), (1024, 1), (512, 2)],  # two r = 1 patterns: the shorter merges
])
def test_bf16_small(pats, causal):
    _run_full(2, 1100, 3, 64, pats, causal, "bf16", seed=11)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("B,N,H,pats", [
    (1, 1, 2, [(1, 1)]),                          # one row
    (1, 127, 2, [(128, 1), (64, 2), (256, 4)]),   # w > N, one partial tile
    (3, 129, 1, [(128, 1), (129, 3)]),            # a tail of one row past a tile
    (1, 5, 8, [(5, 8), (4, 1)]),                  # r > N: heads 5..7 keep no rows of (5, 8)
])
def test_bf16_edge_sizes(B, N, H, pats, causal):
    _run_full(B, N, H, 64, pats, causal, "bf16", seed=14)


@pytest.mark.parametrize("causal", [True, False])
def test_f32_small(causal):
    _run_full(1, 600, 3, 64, [(128, 1), (300, 3), (600, 4)], causal, "f32", seed=12)


def test_f32_d128():
    _run_full(1, 300, 2, 128, [(100, 1), (300, 2)], True, "f32", seed=13)


def _identities(inp_do, sig, dk, dv):
    """sum_n dk[b, n, h] = 0 and sum_n dv[b, n, h] = sum of dO over the rows some pattern keeps.

    Each stored element carries at most ~2^-8 relative error (bf16 rounding
    plus fp32 arithmetic), independent across rows, so the sums may deviate
    by a few times 2^-8 * sqrt(sum of squares)."""
    sel = (sig.T[None, :, :, None] != 0)          # [1, N, H, 1]
    want_v = (inp_do * sel).sum(axis=1)
    tol_k = 6 * 2.0 ** -8 * np.sqrt((dk ** 2).sum(axis=1)) + 1e-3
    tol_v = 6 * 2.0 ** -8 * np.sqrt((dv ** 2).sum(axis=1)) + 1e-3
    err_k = np.abs(dk.sum(axis=1))
    err_v = np.abs(dv.sum(axis=1) - want_v)
    assert (err_k <= tol_k).all(), float((err_k / tol_k).max())
    assert (err_v <= tol_v).all(), float((err_v / tol_v).max())


def _key_rows(wl, rng):
    """Key rows spread over whole segments of the r = 1 pattern (w0 rows each):
    for four heads, in the first, a middle and the last segment, a row of key
    tile 0 (every query of the segment reaches it), a random row, the middle
    row and a row at the end. Rows have the other parity than the head index,
    so only the r = 1 pattern keeps them and the oracle's per-row cost stays
    bounded (a key every pattern keeps would need ~20000 query rows)."""
    rows = []
    w0 = wl.patterns[0][0]
    for h in (0, 1, 5, wl.H - 1):
        for seg in (0, wl.N // w0 // 2, wl.N // w0 - 1):
            for rel in (0, int(rng.integers(0, w0 - 2)), w0 // 2, w0 - 2):
                if (rel - h) % 2 == 0:
                    rel += 1
                rows.append((0, h, seg * w0 + rel))
    return sorted(set(rows))


def test_1m_sampled_rows_and_identities():
    """N = 1048576: dq rows and dk / dv rows across whole segments against the
    row-at-a-time oracle, plus the two sum identities over every row."""
    wl = WORKLOADS["sweep_1048576"]
    inp = make_inputs(wl.B, wl.N, wl.H, wl.d, wl.seed, wl.dtype, NAMES)
    q, k, v, do = to_device(inp, NAMES)
    out, lse, res = dilattn.fwd_train(q, k, v, wl.patterns, wl.causal)
    dq, dk, dv = dilattn.bwd(q, k, v, out, lse, do, wl.patterns, wl.causal, out_res=res)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    rng = np.random.default_rng(3)
    qrows = [(0, int(rng.integers(0, wl.H)), int(rng.integers(0, wl.N))) for _ in range(44)]
    qrows += [(0, 0, 0), (0, wl.H - 1, wl.N - 1), (0, 3, 2048), (0, 7, wl.N // 2)]
    krows = _key_rows(wl, rng)
    bits = {n: inp[n + "_bits"] for n in NAMES}
    gq, gk, gv = oracle_pool.bwd_rows(bits, qrows, krows, wl.patterns, wl.causal)
    dq_c, dk_c, dv_c = dq.cpu(), dk.cpu(), dv.cpu()
    sel = lambda t, rows: to_f64(t[[r[0] for r in rows], [r[2] for r in rows], [r[1] for r in rows]])
    check_close(sel(dq_c, qrows), gq, "bf16", "1M dq rows")
    check_close(sel(dk_c, krows), gk, "bf16", "1M dk rows")
    check_close(sel(dv_c, krows), gv, "bf16", "1M dv rows")
    sig = oracle.selection_signature(wl.N, wl.H, wl.patterns)
    _identities(inp["dout"], sig, to_f64(dk_c), to_f64(dv_c))
