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
def _merge(pieces, lse_i: np.ndarray, N: int, d: int) -> Tuple[np.ndarray, np.ndarray]:
    """O = sum_i exp(lse_i - L) O_i with L = log sum_i exp(lse_i), for one head.

    pieces[i] lists pattern i's (kept rows, O_i rows) per segment; lse_i is
    [npat, N] with -inf where pattern i keeps no row. exp(lse_i - L) =
    Z_i / sum_j Z_j = alpha_i. Rows with every lse_i = -inf (selected by no
    pattern) get L = -inf and O = 0; the -inf - (-inf) case is never
    evaluated.
    """
    mx = lse_i.max(axis=0)                          # [N]
    sel = np.isfinite(mx)
    mx_safe = np.where(sel, mx, 0.0)
    with np.errstate(invalid="ignore"):
        wts = np.where(sel[None], np.exp(lse_i - mx_safe[None]), 0.0)   # Z_i / exp(mx)
    tot = wts.sum(axis=0)
    L = np.where(sel, mx_safe + np.log(np.where(sel, tot, 1.0)), -np.inf)
    alpha = np.where(sel[None], wts / np.where(sel, tot, 1.0)[None], 0.0)  # [npat, N]
    O = np.zeros((N, d))
    for i, segs in enumerate(pieces):
        for idx, O_seg in segs:
            O[idx] += alpha[i, idx][:, None] * O_seg
    return O, L


def fwd_head(q_h: np.ndarray, k_h: np.ndarray, v_h: np.ndarray, h: int,
             patterns: Sequence[Pattern], causal: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Merged dilated attention of one (batch, head) slice.

    q_h, k_h, v_h: [N, d]; h is the head index, which selects every pattern's
    offset h mod r. Returns out [N, d] and lse [N] (float64, natural log).
    Heads and batches never interact, so this is the whole method for one
    slice: steps 1-3 per pattern and segment, then the step-4 merge.
    """
    q_h = np.asarray(q_h, dtype=np.float64)
    k_h = np.asarray(k_h, dtype=np.float64)
    v_h = np.asarray(v_h, dtype=np.float64)
    N, d = q_h.shape
    tau = 1.0 / math.sqrt(d)
    lse_i = np.full((len(patterns), N), -np.inf)
    pieces = []
    for i, (w, r) in enumerate(patterns):
        segs = []
        for idx in kept_rows(N, w, r, h):
            if idx.size == 0:
                continue
            O, lse = _segment_attention(q_h[idx], k_h[idx], v_h[idx], tau, causal)
            segs.append((idx, O))
            lse_i[i, idx] = lse
        pieces.append(segs)
    return _merge(pieces, lse_i, N, d)


def fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, patterns: Sequence[Pattern],
        causal: bool = True) -> Tuple[np.ndarray, np.ndarray]:
    """Merged dilated attention: out [B, N, H, d] float64, lse [B, H, N] float64 (natural log)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, d = q.shape
    out = np.zeros((B, N, H, d))
    lse = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            out[b, :, h], lse[b, h] = fwd_head(q[b, :, h], k[b, :, h], v[b, :, h], h,
                                               patterns, causal)
    return out, lse


# ---------------------------------------------------------------------------
# Step 5: backward, recomputing the probabilities from the merged lse
# ---------------------------------------------------------------------------
def bwd_head(q_h: np.ndarray, k_h: np.ndarray, v_h: np.ndarray, do_h: np.ndarray, h: int,
             patterns: Sequence[Pattern], causal: bool = True, out_h: np.ndarray = None,
             lse_h: np.ndarray = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients (dq, dk, dv) [N, d] of sum(out * dout) for one (batch, head) slice.

    Because the merged output is one softmax over the multiset union of the
    keys the patterns give a row, the probability of key c for row a under
    pattern i is exp(s_ac - L_a) with the merged L, and
    D_a = sum(dO_a * O_a) is the softmax-backward row term. Per (pattern,
    segment): dV += P^T dO, dP = dO V^T, dS = P * (dP - D), dQ += tau dS K,
    dK += tau dS^T Q. out_h / lse_h default to this oracle's own forward.
    """
    q_h = np.asarray(q_h, dtype=np.float64)
    k_h = np.asarray(k_h, dtype=np.float64)
    v_h = np.asarray(v_h, dtype=np.float64)
    do_h = np.asarray(do_h, dtype=np.float64)
    if out_h is None or lse_h is None:
        out_h, lse_h = fwd_head(q_h, k_h, v_h, h, patterns, causal)
    out_h = np.asarray(out_h, dtype=np.float64)
    lse_h = np.asarray(lse_h, dtype=np.float64)
    N, d = q_h.shape
    tau = 1.0 / math.sqrt(d)
    Drow = np.einsum("nd,nd->n", do_h, out_h)
    dq = np.zeros_like(q_h)
    dk = np.zeros_like(k_h)
    dv = np.zeros_like(v_h)
    for (w, r) in patterns:
        for idx in kept_rows(N, w, r, h):
            if idx.size == 0:
                continue
            Qs, Ks, Vs, dOs = q_h[idx], k_h[idx], v_h[idx], do_h[idx]
            S = tau * (Qs @ Ks.T)
            P = np.exp(S - lse_h[idx][:, None])
            if causal:
                P = np.tril(P)
            dv[idx] += P.T @ dOs
            dP = dOs @ Vs.T
            dS = P * (dP - Drow[idx][:, None])
            dq[idx] += tau * (dS @ Ks)
            dk[idx] += tau * (dS.T @ Qs)
    return dq, dk, dv


def bwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, dout: np.ndarray,
        patterns: Sequence[Pattern], causal: bool = True, out: np.ndarray = None,
        lse: np.ndarray = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Gradients (dq, dk, dv) of sum(out * dout), all [B, N, H, d] float64 (bwd_head per slice)."""
    q = np.asarray(q, dtype=np.float64)
    B, N, H, d = q.shape
    dq = np.zeros((B, N, H, d))
    dk = np.zeros((B, N, H, d))
    dv = np.zeros((B, N, H, d))
    for b in range(B):
        for h in range(H):
            o_h = None if out is None else out[b, :, h]
            l_h = None if lse is None else lse[b, h]
            dq[b, :, h], dk[b, :, h], dv[b, :, h] = bwd_head(
                q[b, :, h], k[b, :, h], v[b, :, h], dout[b, :, h], h, patterns, causal, o_h, l_h)
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
