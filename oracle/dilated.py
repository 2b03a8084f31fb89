"""Plain float64 CPU oracle for LongNet dilated attention, forward and backward.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path. It shares
no code with the CUDA path; the two meet only at the seeded inputs.

What it computes (sources: the LongNet pages -- the gptget.net summary of
arXiv 2307.02486, sections "方法论" and "方法详解"; the abstract printed on the
same page and on the darcstar.tech, summarizepaper and khansong pages; and the
DarcStar commentary on the darcstar.tech page):

* The sequence of length N is cut into equal segments of length w (the last
  one truncated at N) -- "方法详解", first bullet.
* Inside each segment only every r-th row is kept (the dilation rate r), and
  different heads use different offsets -- "方法详解", second and third
  bullets; "方法论". The offset of head h is h mod r, counted from the start
  of the segment: segment s keeps rows s*w + (h mod r) + k*r below
  min((s+1)*w, N).
* On the kept rows of each segment, ordinary scaled dot-product softmax
  attention runs (the abstract: dilated attention is a drop-in replacement for
  standard attention), causal in position order when ``causal`` is set, with
  scale 1/sqrt(d).
* Several (w, r) patterns are mixed (multi-scale, "方法详解" second and seventh
  bullets). A row's outputs from the patterns that select it are combined as
  O = sum_i alpha_i O_i with alpha_i = Z_i / sum_j Z_j, Z_i being pattern i's
  softmax denominator for that row, carried as a log-sum-exp so the shared
  denominator stays exact (DarcStar commentary, third paragraph). A row that
  no pattern selects gets O = 0 and lse = -inf.
* The backward pass is the full derivative of that function (alpha_i is not
  treated as a constant); it recomputes the probabilities from the merged
  lse.

Every step below is written out in the order above with numpy float64
matmuls as the only library primitive. Readings of points the pages leave
open are listed in the repository's design notes; each is also stated where
it is used here.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Sequence, Tuple

import numpy as np

Pattern = Tuple[int, int]


# ---------------------------------------------------------------------------
# Step 1: which rows a pattern keeps ("方法详解": segments, dilation, per-head
# offsets)
# ---------------------------------------------------------------------------
def kept_rows(N: int, w: int, r: int, h: int) -> List[np.ndarray]:
    """Kept row positions of pattern (w, r) for head h, one array per segment.

    Segment s spans [s*w, min((s+1)*w, N)); it keeps s*w + (h mod r) + k*r for
    k = 0, 1, ... while below the segment end. Reading: the offset is relative
    to the segment start (not a global residue), and when the offset is past
    the segment end the segment keeps nothing.
    """
    if N < 1 or w < 1 or r < 1:
        raise ValueError("N, w, r must be >= 1")
    off = h % r
    segs = []
    for start in range(0, N, w):
        end = min(start + w, N)
        segs.append(np.arange(start + off, end, r, dtype=np.int64))
    return segs


def selection_signature(N: int, H: int, patterns: Sequence[Pattern]) -> np.ndarray:
    """uint32 [H, N]: bit i set when pattern i keeps row n for head h."""
    sig = np.zeros((H, N), dtype=np.uint32)
    for i, (w, r) in enumerate(patterns):
        for h in range(H):
            for idx in kept_rows(N, w, r, h):
                sig[h, idx] |= np.uint32(1 << i)
    return sig


# ---------------------------------------------------------------------------
# Steps 2-3: dense softmax attention inside each sparsified segment
# ---------------------------------------------------------------------------
def _segment_attention(Qs: np.ndarray, Ks: np.ndarray, Vs: np.ndarray, tau: float,
                       causal: bool) -> Tuple[np.ndarray, np.ndarray]:
    """Standard softmax attention on one gathered segment.

    Kept rows are increasing positions, so causal order on positions is the
    lower triangle of the gathered score matrix (diagonal included).
    Returns (O_i rows, lse_i rows).
    """
    S = tau * (Qs @ Ks.T)
    if causal:
        n = S.shape[0]
        S = np.where(np.tril(np.ones((n, n), dtype=bool)), S, -np.inf)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    Z = E.sum(axis=1)
    O = (E @ Vs) / Z[:, None]
    lse = m + np.log(Z)
    return O, lse


def fwd_per_pattern(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                    patterns: Sequence[Pattern], causal: bool = True):
    """Per-pattern outputs before the merge.

    q, k, v: [B, N, H, d] (any float dtype; computed in float64).
    Returns O_i [npat, B, N, H, d] and lse_i [npat, B, H, N]; rows a pattern
    does not keep have O_i = 0 and lse_i = -inf.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    tau = 1.0 / math.sqrt(d)
    npat = len(patterns)
    O_i = np.zeros((npat, B, N, H, d))
    lse_i = np.full((npat, B, H, N), -np.inf)
    for i, (w, r) in enumerate(patterns):
        for b in range(B):
            for h in range(H):
                for idx in kept_rows(N, w, r, h):
                    if idx.size == 0:
                        continue
                    O, lse = _segment_attention(q[b, idx, h], k[b, idx, h], v[b, idx, h],
                                                tau, causal)
                    O_i[i, b, idx, h] = O
                    lse_i[i, b, h, idx] = lse
    return O_i, lse_i


# ---------------------------------------------------------------------------
# Step 4: merge through the log-sum-exp of the denominators (DarcStar
# commentary: the shared denominator must stay exact)
# ---------------------------------------------------------------------------
def _merge(O_i: np.ndarray, lse_i: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """O = sum_i exp(lse_i - L) O_i with L = log sum_i exp(lse_i).

    exp(lse_i - L) = Z_i / sum_j Z_j = alpha_i. Rows with every lse_i = -inf
    (selected by no pattern) get L = -inf and O = 0; the -inf - (-inf) case
    is never evaluated.
    """
    npat, B, H, N = lse_i.shape
    mx = lse_i.max(axis=0)                          # [B, H, N]
    sel = np.isfinite(mx)
    mx_safe = np.where(sel, mx, 0.0)
    with np.errstate(invalid="ignore"):
        wts = np.where(sel[None], np.exp(lse_i - mx_safe[None]), 0.0)   # Z_i / exp(mx)
    tot = wts.sum(axis=0)
    L = np.where(sel, mx_safe + np.log(np.where(sel, tot, 1.0)), -np.inf)
    alpha = np.where(sel[None], wts / np.where(sel, tot, 1.0)[None], 0.0)  # [npat, B, H, N]
    O = np.einsum("pbhn,pbnhd->bnhd", alpha, O_i)
    return O, L


def fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, patterns: Sequence[Pattern],
        causal: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Merged dilated attention: out [B, N, H, d] float64, lse [B, H, N] float64 (natural log)."""
    O_i, lse_i = fwd_per_pattern(q, k, v, patterns, causal)
    return _merge(O_i, lse_i)


# ---------------------------------------------------------------------------
# Step 5: backward, recomputing the probabilities from the merged lse
# ---------------------------------------------------------------------------
def bwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray,
        patterns: Sequence[Pattern], causal: bool = True, out: np.ndarray = None,
        lse: np.ndarray = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients (dq, dk, dv) of sum(out * dout), all [B, N, H, d] float64.

    Because the merged output is one softmax over the multiset union of the
    keys the patterns give a row, the probability of key c for row a under
    pattern i is exp(s_ac - L_a) with the merged L, and
    D_a = sum(dO_a * O_a) is the softmax-backward row term. Per (pattern,
    segment): dV += P^T dO, dP = dO V^T, dS = P * (dP - D), dQ += tau dS K,
    dK += tau dS^T Q.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    if out is None or lse is None:
        out, lse = fwd(q, k, v, patterns, causal)
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    B, N, H, d = q.shape
    tau = 1.0 / math.sqrt(d)
    Drow = np.einsum("bnhd,bnhd->bhn", dout, out)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for (w, r) in patterns:
        for b in range(B):
            for h in range(H):
                for idx in kept_rows(N, w, r, h):
                    if idx.size == 0:
                        continue
                    Qs, Ks, Vs, dOs = q[b, idx, h], k[b, idx, h], v[b, idx, h], dout[b, idx, h]
                    S = tau * (Qs @ Ks.T)
                    Ls = lse[b, h, idx]
                    P = np.exp(S - Ls[:, None])
                    if causal:
                        P = np.tril(P)
                    dv[b, idx, h] += P.T @ dOs
                    dP = dOs @ Vs.T
                    dS = P * (dP - Drow[b, h, idx][:, None])
                    dq[b, idx, h] += tau * (dS @ Ks)
                    dk[b, idx, h] += tau * (dS.T @ Qs)
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Row-at-a-time forms, for sampled checks at full problem sizes
# ---------------------------------------------------------------------------
def _row_keys(N: int, patterns: Sequence[Pattern], h: int, n: int, causal: bool):
    """For query row n of head h: list of (pattern index, key positions) over the
    patterns that keep n; keys are the kept rows of n's segment (<= n if causal)."""
    res = []
    for i, (w, r) in enumerate(patterns):
        start = (n // w) * w
        end = min(start + w, N)
        off = h % r
        rel = n - start - off
        if rel < 0 or rel % r != 0:
            continue
        keys = np.arange(start + off, (n + 1) if causal else end, r, dtype=np.int64)
        res.append((i, keys))
    return res


def fwd_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, patterns: Sequence[Pattern],
             rows: Iterable[Tuple[int, int, int]], causal: bool = True):
    """Merged output and lse for selected (b, h, n) rows, one row at a time.

    Returns (O [len(rows), d], lse [len(rows)]) in float64.
    """
    rows = list(rows)
    B, N, H, d = q.shape
    tau = 1.0 / math.sqrt(d)
    O = np.zeros((len(rows), d))
    L = np.full(len(rows), -np.inf)
    for j, (b, h, n) in enumerate(rows):
        qn = np.asarray(q[b, n, h], dtype=np.float64)
        lses, outs = [], []
        for _, keys in _row_keys(N, patterns, h, n, causal):
            s = tau * (np.asarray(k[b, keys, h], dtype=np.float64) @ qn)
            m = s.max()
            e = np.exp(s - m)
            z = e.sum()
            outs.append((e @ np.asarray(v[b, keys, h], dtype=np.float64)) / z)
            lses.append(m + math.log(z))
        if not lses:
            continue
        lses = np.array(lses)
        mx = lses.max()
        wts = np.exp(lses - mx)
        L[j] = mx + math.log(wts.sum())
        O[j] = (wts[:, None] * np.array(outs)).sum(axis=0) / wts.sum()
    return O, L


def bwd_rows(q, k, v, dout, patterns: Sequence[Pattern], qrows, krows, causal: bool = True,
             out_rows_fn=None):
    """Sampled gradients at full size.

    qrows: list of (b, h, n) -> dq rows; krows: list of (b, h, n) -> (dk, dv) rows.
    The merged O and lse of every query row involved are recomputed with
    ``fwd_rows`` (float64), so the result does not depend on any stored output.
    Returns (dq [len(qrows), d], dk [len(krows), d], dv [len(krows), d]).
    """
    B, N, H, d = q.shape
    tau = 1.0 / math.sqrt(d)
    cache = {}

    def row_stats(b, h, n):
        key = (b, h, n)
        if key not in cache:
            O, L = fwd_rows(q, k, v, patterns, [key], causal)
            Drow = float(np.asarray(dout[b, n, h], dtype=np.float64) @ O[0])
            cache[key] = (L[0], Drow)
        return cache[key]

    dq = np.zeros((len(qrows), d))
    for j, (b, h, n) in enumerate(qrows):
        L, Drow = row_stats(b, h, n)
        if not np.isfinite(L):
            continue
        qn = np.asarray(q[b, n, h], dtype=np.float64)
        dOn = np.asarray(dout[b, n, h], dtype=np.float64)
        for _, keys in _row_keys(N, patterns, h, n, causal):
            Kk = np.asarray(k[b, keys, h], dtype=np.float64)
            Vk = np.asarray(v[b, keys, h], dtype=np.float64)
            p = np.exp(tau * (Kk @ qn) - L)
            ds = p * (Vk @ dOn - Drow)
            dq[j] += tau * (ds @ Kk)

    dk = np.zeros((len(krows), d))
    dv = np.zeros((len(krows), d))
    for j, (b, h, c) in enumerate(krows):
        kc = np.asarray(k[b, c, h], dtype=np.float64)
        vc = np.asarray(v[b, c, h], dtype=np.float64)
        for (w, r) in patterns:
            start = (c // w) * w
            end = min(start + w, N)
            off = h % r
            rel = c - start - off
            if rel < 0 or rel % r != 0:
                continue
            qs = np.arange(c if causal else start + off, end, r, dtype=np.int64)
            for n in qs:
                L, Drow = row_stats(b, h, int(n))
                qn = np.asarray(q[b, n, h], dtype=np.float64)
                dOn = np.asarray(dout[b, n, h], dtype=np.float64)
                p = math.exp(tau * float(qn @ kc) - L)
                dv[j] += p * dOn
                ds = p * (float(dOn @ vc) - Drow)
                dk[j] += tau * ds * qn
    return dq, dk, dv


# ---------------------------------------------------------------------------
# Brute force on tiny inputs: one softmax over the multiset union of keys
# ---------------------------------------------------------------------------
def multiplicity(N: int, patterns: Sequence[Pattern], h: int, causal: bool = True) -> np.ndarray:
    """M[a, c] = number of patterns that keep both a and c in the same segment
    (with c <= a when causal), built from explicit per-pattern masks."""
    M = np.zeros((N, N), dtype=np.int64)
    for (w, r) in patterns:
        for idx in kept_rows(N, w, r, h):
            for a in idx:
                for c in idx:
                    if causal and c > a:
                        continue
                    M[a, c] += 1
    return M


def fwd_bruteforce(q: np.ndarray, k: np.ndarray, v: np.ndarray, patterns: Sequence[Pattern],
                   causal: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """out = (M * e^S) V / rowsum(M * e^S), lse = log rowsum(M * e^S) over the full
    N x N score matrix; rows with an all-zero multiplicity row give 0 / -inf."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    tau = 1.0 / math.sqrt(d)
    out = np.zeros((B, N, H, d))
    lse = np.full((B, H, N), -np.inf)
    for h in range(H):
        M = multiplicity(N, patterns, h, causal).astype(np.float64)
        for b in range(B):
            S = tau * (q[b, :, h] @ k[b, :, h].T)
            for a in range(N):
                if M[a].sum() == 0:
                    continue
                cols = M[a] > 0
                m = S[a, cols].max()
                e = M[a] * np.exp(np.where(cols, S[a] - m, -np.inf))
                z = e.sum()
                out[b, a, h] = (e @ v[b, :, h]) / z
                lse[b, h, a] = m + math.log(z)
    return out, lse


# ---------------------------------------------------------------------------
# Work count used for effective FLOP/s
# ---------------------------------------------------------------------------
def effective_pairs(B: int, N: int, H: int, patterns: Sequence[Pattern], causal: bool = True) -> int:
    """Number of nonzero (query, key) pairs under the causal sparse mask, summed
    over patterns (a key reached through two patterns counts twice)."""
    total = 0
    for (w, r) in patterns:
        for h in range(H):
            off = h % r
            for start in range(0, N, w):
                end = min(start + w, N)
                n = max(0, -(-(end - start - off) // r)) if end - start > off else 0
                total += n * (n + 1) // 2 if causal else n * n
    return B * total
