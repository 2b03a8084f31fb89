"""Pins for the float64 oracle, checked against things other than itself.

* hand-enumerated kept-row sets and hand-derived merged outputs (tests/golden);
* the special case w = N, r = 1, which must reduce to dense softmax attention,
  checked against torch's scaled_dot_product_attention in float64 on the CPU;
* a brute-force form built from explicit per-pattern multiplicity masks
  (one softmax over the multiset union of attended keys);
* invariants: per-pattern weights and merge weights sum to one, constant
  values pass through, a shift of every key leaves the output unchanged and
  moves lse by tau*q.u, closed-form lse of row 0;
* gradients against float64 central finite differences and against torch
  autograd of the brute-force form;
* planted mistakes in a copy of the oracle are caught by these pins.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import dilated as odl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------------------
# index sets
# ---------------------------------------------------------------------------
def _golden_index_lines():
    with open(os.path.join(GOLDEN, "index_sets.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line


@pytest.mark.parametrize("line", list(_golden_index_lines()))
def test_kept_rows_golden(line):
    head, body = line.split(":")
    fields = head.split()
    if fields[0] == "rows":
        N, w, r, h = map(int, fields[1:])
        want = [[int(x) for x in seg.split()] for seg in body.split("|")]
        got = [list(map(int, s)) for s in oracle.kept_rows(N, w, r, h)]
        assert got == want
    else:
        N, w, r, h, seg = map(int, fields[1:])
        n, first, last = map(int, body.split())
        rows = oracle.kept_rows(N, w, r, h)[seg]
        assert (rows.size, int(rows[0]), int(rows[-1])) == (n, first, last)


def test_selection_signature_matches_rows():
    pats = [(8, 3), (16, 2), (5, 1)]
    sig = oracle.selection_signature(20, 3, pats)
    for h in range(3):
        for i, (w, r) in enumerate(pats):
            rows = set(int(x) for s in oracle.kept_rows(20, w, r, h) for x in s)
            for n in range(20):
                assert bool(sig[h, n] >> i & 1) == (n in rows)


# ---------------------------------------------------------------------------
# hand-derived merged outputs
# ---------------------------------------------------------------------------
def _golden_zero_scores():
    with open(os.path.join(GOLDEN, "zero_scores_merge.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, body = line.split(":")
            causal, h = map(int, head.split())
            outs, sizes = body.split(";")
            yield causal, h, [float(x) for x in outs.split()], [int(x) for x in sizes.split()]


@pytest.mark.parametrize("case", list(_golden_zero_scores()))
def test_zero_score_merge_golden(case):
    causal, h, want_out, want_size = case
    N, H, d = 8, 2, 1
    q = np.zeros((1, N, H, d))
    k = np.ones((1, N, H, d))
    v = np.arange(N, dtype=np.float64)[None, :, None, None].repeat(H, axis=2)
    out, lse = oracle.fwd(q, k, v, [(4, 1), (8, 2)], causal=bool(causal))
    np.testing.assert_allclose(out[0, :, h, 0], want_out, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, h], np.log(want_size), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# reduction to dense attention (library routine)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("N,H,d", [(37, 3, 8), (64, 2, 16)])
def test_single_full_pattern_is_dense_attention(causal, N, H, d):
    q, k, v = (_rand((2, N, H, d), s) for s in (1, 2, 3))
    out, lse = oracle.fwd(q, k, v, [(N, 1)], causal=causal)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))  # B H N d
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    np.testing.assert_allclose(out, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    # lse against torch.logsumexp of the masked score matrix
    S = torch.einsum("bhnd,bhmd->bhnm", tq, tk) / math.sqrt(d)
    if causal:
        S = S.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(S, -1).numpy(), rtol=0, atol=1e-12)


def test_w_smaller_than_N_r1_is_block_diagonal_dense():
    N, H, d, w = 48, 2, 8, 16
    q, k, v = (_rand((1, N, H, d), s) for s in (4, 5, 6))
    out, _ = oracle.fwd(q, k, v, [(w, 1)], causal=True)
    for s in range(0, N, w):
        sl = slice(s, s + w)
        tq, tk, tv = (torch.from_numpy(x[:, sl]).permute(0, 2, 1, 3) for x in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
        np.testing.assert_allclose(out[:, sl], ref.permute(0, 2, 1, 3).numpy(), atol=1e-12)


# ---------------------------------------------------------------------------
# brute force: one softmax over the multiset union
# ---------------------------------------------------------------------------
PATTERN_SETS = [
    [(8, 1), (16, 2), (32, 4)],                 # nested powers of two
    [(8, 1), (12, 2), (20, 3), (30, 6)],        # non-nested, ragged (w does not divide N)
    [(5, 1), (7, 7), (3, 5)],                   # r > w and r = w: some segments empty
    [(16, 2), (16, 2)],                         # duplicated pattern
    [(9, 4)],                                   # some rows selected by no pattern
]


@pytest.mark.parametrize("pats", PATTERN_SETS)
@pytest.mark.parametrize("causal", [True, False])
def test_merge_equals_union_softmax(pats, causal):
    N, H, d = 30, 5, 4
    q, k, v = (_rand((2, N, H, d), s) for s in (7, 8, 9))
    out, lse = oracle.fwd(q, k, v, pats, causal)
    bo, bl = oracle.fwd_bruteforce(q, k, v, pats, causal)
    np.testing.assert_allclose(out, bo, rtol=0, atol=1e-12)
    fin = np.isfinite(bl)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], bl[fin], rtol=0, atol=1e-12)


def test_unselected_rows_are_zero_and_minus_inf():
    N, H, d = 20, 4, 3
    q, k, v = (_rand((1, N, H, d), s) for s in (1, 2, 3))
    pats = [(9, 4)]
    out, lse = oracle.fwd(q, k, v, pats)
    sig = oracle.selection_signature(N, H, pats)
    for h in range(H):
        for n in range(N):
            if sig[h, n] == 0:
                assert lse[0, h, n] == -np.inf
                assert np.all(out[0, n, h] == 0)
            else:
                assert np.isfinite(lse[0, h, n])
    assert np.isfinite(out).all()


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("pats", PATTERN_SETS)
def test_per_pattern_weights_sum_to_one(pats):
    N, H, d = 30, 3, 4
    q, k = _rand((1, N, H, d), 1), _rand((1, N, H, d), 2)
    ones = np.ones((1, N, H, d))
    O_i, lse_i = oracle.fwd_per_pattern(q, k, ones, pats)
    for i in range(len(pats)):
        sel = np.isfinite(lse_i[i, 0]).T          # [N, H]
        np.testing.assert_allclose(O_i[i, 0][sel], 1.0, atol=1e-13)
    # merge weights alpha_i = exp(lse_i - L) sum to one on selected rows
    _, L = oracle.fwd(q, k, ones, pats)
    fin = np.isfinite(L)
    with np.errstate(invalid="ignore"):
        alpha = np.where(np.isfinite(lse_i), np.exp(lse_i - np.where(fin, L, 0)[None]), 0.0)
    np.testing.assert_allclose(alpha.sum(axis=0)[fin], 1.0, atol=1e-13)


def test_constant_values_pass_through():
    N, H, d = 30, 3, 4
    pats = PATTERN_SETS[1]
    q, k = _rand((1, N, H, d), 3), _rand((1, N, H, d), 4)
    c = np.array([0.5, -2.0, 3.0, 1.25])
    v = np.broadcast_to(c, (1, N, H, d)).copy()
    out, lse = oracle.fwd(q, k, v, pats)
    sel = np.isfinite(lse[0]).T
    np.testing.assert_allclose(out[0][sel], np.broadcast_to(c, out[0][sel].shape), atol=1e-13)


def test_key_shift_invariance():
    N, H, d = 30, 3, 4
    pats = PATTERN_SETS[0]
    q, k, v = (_rand((1, N, H, d), s) for s in (5, 6, 7))
    u = np.array([0.3, -1.0, 2.0, 0.7])
    out0, lse0 = oracle.fwd(q, k, v, pats)
    out1, lse1 = oracle.fwd(q, k + u, v, pats)
    np.testing.assert_allclose(out1, out0, atol=1e-12)
    shift = np.einsum("bnhd,d->bhn", q, u) / math.sqrt(d)
    fin = np.isfinite(lse0)
    np.testing.assert_allclose((lse1 - lse0)[fin], shift[fin], atol=1e-12)


def test_lse_of_first_row_closed_form():
    N, H, d = 32, 6, 8
    pats = [(8, 1), (16, 2), (32, 4), (32, 3)]
    q, k, v = (_rand((1, N, H, d), s) for s in (8, 9, 10))
    out, lse = oracle.fwd(q, k, v, pats)
    for h in range(H):
        cnt = sum(1 for (w, r) in pats if h % r == 0)
        if cnt == 0:
            assert lse[0, h, 0] == -np.inf
            continue
        want = float(q[0, 0, h] @ k[0, 0, h]) / math.sqrt(d) + math.log(cnt)
        assert abs(lse[0, h, 0] - want) < 1e-13
        np.testing.assert_allclose(out[0, 0, h], v[0, 0, h], atol=1e-14)


def test_duplicate_pattern_adds_log2():
    N, H, d = 24, 3, 4
    q, k, v = (_rand((1, N, H, d), s) for s in (1, 2, 3))
    o1, l1 = oracle.fwd(q, k, v, [(8, 2)])
    o2, l2 = oracle.fwd(q, k, v, [(8, 2), (8, 2)])
    np.testing.assert_allclose(o2, o1, atol=1e-14)
    fin = np.isfinite(l1)
    np.testing.assert_allclose(l2[fin] - l1[fin], math.log(2), atol=1e-14)


def test_row_form_matches_full_form():
    N, H, d = 40, 4, 5
    pats = PATTERN_SETS[1]
    q, k, v = (_rand((2, N, H, d), s) for s in (11, 12, 13))
    out, lse = oracle.fwd(q, k, v, pats)
    rows = [(b, h, n) for b in range(2) for h in range(H) for n in range(0, N, 3)]
    O, L = oracle.fwd_rows(q, k, v, pats, rows)
    for j, (b, h, n) in enumerate(rows):
        np.testing.assert_allclose(O[j], out[b, n, h], atol=1e-12)
        if np.isfinite(lse[b, h, n]):
            assert abs(L[j] - lse[b, h, n]) < 1e-12
        else:
            assert L[j] == -np.inf


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------
def _torch_bruteforce_loss(q, k, v, dout, pats, causal):
    """sum(out * dout) of the multiplicity-mask form, in torch float64."""
    B, N, H, d = q.shape
    loss = 0.0
    for h in range(H):
        M = torch.from_numpy(oracle.multiplicity(N, pats, h, causal).astype(np.float64))
        S = torch.einsum("bnd,bmd->bnm", q[:, :, h], k[:, :, h]) / math.sqrt(d)
        has = M.sum(1) > 0
        S = S.masked_fill(M[None] == 0, -math.inf)
        S = torch.where(has[None, :, None], S, torch.zeros_like(S))
        P = torch.softmax(S + torch.log(torch.where(M > 0, M, torch.ones_like(M)))[None], dim=-1)
        P = P * has[None, :, None]
        loss = loss + (torch.einsum("bnm,bmd->bnd", P, v[:, :, h]) * dout[:, :, h]).sum()
    return loss


@pytest.mark.parametrize("pats", PATTERN_SETS)
@pytest.mark.parametrize("causal", [True, False])
def test_backward_matches_torch_autograd_of_bruteforce(pats, causal):
    N, H, d = 22, 3, 4
    q, k, v, do = (_rand((2, N, H, d), s) for s in (21, 22, 23, 24))
    dq, dk, dv = oracle.bwd(q, k, v, do, pats, causal)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    loss = _torch_bruteforce_loss(tq, tk, tv, torch.from_numpy(do), pats, causal)
    loss.backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), atol=1e-11)


def test_backward_finite_differences():
    N, H, d = 12, 2, 3
    pats = [(4, 1), (8, 2), (12, 3)]
    q, k, v, do = (_rand((1, N, H, d), s) for s in (31, 32, 33, 34))
    dq, dk, dv = oracle.bwd(q, k, v, do, pats)
    eps = 1e-6

    def loss(q_, k_, v_):
        return float((oracle.fwd(q_, k_, v_, pats)[0] * do).sum())

    rng = np.random.default_rng(0)
    for which, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, s)) for s in q.shape)
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[which][idx] += eps
            lp = loss(args["q"], args["k"], args["v"])
            args[which][idx] -= 2 * eps
            lm = loss(args["q"], args["k"], args["v"])
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def test_backward_unselected_rows_have_zero_gradient():
    N, H, d = 20, 4, 3
    pats = [(9, 4)]
    q, k, v, do = (_rand((1, N, H, d), s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle.bwd(q, k, v, do, pats)
    sig = oracle.selection_signature(N, H, pats)
    for h in range(H):
        for n in range(N):
            if sig[h, n] == 0:
                assert not dq[0, n, h].any() and not dk[0, n, h].any() and not dv[0, n, h].any()


def test_row_form_backward_matches_full_form():
    N, H, d = 26, 3, 4
    pats = PATTERN_SETS[1]
    q, k, v, do = (_rand((1, N, H, d), s) for s in (41, 42, 43, 44))
    dq, dk, dv = oracle.bwd(q, k, v, do, pats)
    rows = [(0, h, n) for h in range(H) for n in range(0, N, 5)]
    rq, rk, rv = oracle.bwd_rows(q, k, v, do, pats, rows, rows)
    for j, (b, h, n) in enumerate(rows):
        np.testing.assert_allclose(rq[j], dq[b, n, h], atol=1e-12)
        np.testing.assert_allclose(rk[j], dk[b, n, h], atol=1e-12)
        np.testing.assert_allclose(rv[j], dv[b, n, h], atol=1e-12)


# ---------------------------------------------------------------------------
# effective pair count (the FLOP numerator) against the multiplicity matrix
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("pats", PATTERN_SETS)
@pytest.mark.parametrize("causal", [True, False])
def test_effective_pairs_equals_multiplicity_total(pats, causal):
    N, H = 30, 5
    want = sum(int(oracle.multiplicity(N, pats, h, causal).sum()) for h in range(H))
    assert oracle.effective_pairs(2, N, H, pats, causal) == 2 * want


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by one of the pins above
# ---------------------------------------------------------------------------
def _zero_score_case_fails(fwd_fn):
    for causal, h, want_out, want_size in _golden_zero_scores():
        N, H = 8, 2
        q = np.zeros((1, N, H, 1))
        k = np.ones((1, N, H, 1))
        v = np.arange(N, dtype=np.float64)[None, :, None, None].repeat(H, axis=2)
        out, lse = fwd_fn(q, k, v, [(4, 1), (8, 2)], bool(causal))
        if not (np.allclose(out[0, :, h, 0], want_out, atol=1e-12)
                and np.allclose(lse[0, h], np.log(want_size), atol=1e-12)):
            return True
    return False


def test_planted_global_residue_offset_is_caught(monkeypatch):
    # mistake: offset counted as a global residue instead of from the segment start
    def bad_kept_rows(N, w, r, h):
        segs = []
        for start in range(0, N, w):
            end = min(start + w, N)
            first = start + ((h - start) % r)
            segs.append(np.arange(first, end, r, dtype=np.int64))
        return segs
    monkeypatch.setattr(odl, "kept_rows", bad_kept_rows)
    monkeypatch.setattr(oracle, "kept_rows", bad_kept_rows)
    line = "count 32768 16384 6 4 1 : 2730 16388 32762"
    with pytest.raises(AssertionError):
        test_kept_rows_golden(line)


def test_planted_unweighted_merge_is_caught(monkeypatch):
    # mistake: average the pattern outputs instead of weighting by Z_i
    def bad_merge(pieces, lse_i, N, d):
        cnt = np.isfinite(lse_i).sum(axis=0)
        O = np.zeros((N, d))
        for segs in pieces:
            for idx, O_seg in segs:
                O[idx] += O_seg / np.maximum(cnt[idx], 1)[:, None]
        return O, lse_i.max(axis=0)
    monkeypatch.setattr(odl, "_merge", bad_merge)
    assert _zero_score_case_fails(odl.fwd)


def test_planted_missing_causal_mask_is_caught(monkeypatch):
    orig = odl._segment_attention
    monkeypatch.setattr(odl, "_segment_attention",
                        lambda Qs, Ks, Vs, tau, causal: orig(Qs, Ks, Vs, tau, False))
    assert _zero_score_case_fails(odl.fwd)


def test_planted_missing_D_term_in_backward_is_caught():
    N, H, d = 10, 2, 3
    pats = [(4, 1), (8, 2)]
    q, k, v, do = (_rand((1, N, H, d), s) for s in (1, 2, 3, 4))
    dq, dk, dv = oracle.bwd(q, k, v, do, pats)
    # recompute dq without the D term: must disagree with torch autograd
    out, lse = oracle.fwd(q, k, v, pats)
    tau = 1 / math.sqrt(d)
    bad = np.zeros_like(dq)
    for (w, r) in pats:
        for h in range(H):
            for idx in oracle.kept_rows(N, w, r, h):
                S = tau * q[0, idx, h] @ k[0, idx, h].T
                P = np.tril(np.exp(S - lse[0, h, idx][:, None]))
                bad[0, idx, h] += tau * ((P * (do[0, idx, h] @ v[0, idx, h].T)) @ k[0, idx, h])
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    _torch_bruteforce_loss(tq, tk, tv, torch.from_numpy(do), pats, True).backward()
    assert np.allclose(dq, tq.grad.numpy(), atol=1e-11)
    assert not np.allclose(bad, tq.grad.numpy(), atol=1e-6)
