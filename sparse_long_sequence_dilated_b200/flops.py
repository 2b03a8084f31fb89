"""Work counts for reporting: nonzero (query, key) pairs under the causal
sparse mask, effective FLOPs and algorithmic bytes.

Effective FLOPs count only the pairs the dilated patterns make nonzero:
4 d per pair forward (S = Q K^T and O += P V), 10 d per pair backward
(S recomputed, dP = dO V^T, dV, dK, dQ); 8 d per pair is the backward's
count without the recomputed S, reported beside it under that label.

Algorithmic forward bytes: every pattern reads the Q, K and V rows it keeps
once (3 x 2 d bytes per kept row, bf16), and the merged result is written
once (2 d bytes of out and 4 of lse per row, plus 2 d of out_res for the
training forward).
"""
from __future__ import annotations

from typing import Sequence, Tuple


def segment_counts(N: int, w: int, r: int, h: int):
    """Kept-row count of every segment of pattern (w, r) for head h."""
    off = h % r
    out = []
    for start in range(0, N, w):
        ln = min(start + w, N) - start
        out.append((ln - off + r - 1) // r if ln > off else 0)
    return out


def effective_pairs(B: int, N: int, H: int, patterns: Sequence[Tuple[int, int]],
                    causal: bool = True) -> int:
    total = 0
    for (w, r) in patterns:
        for h in range(H):
            for n in segment_counts(N, w, r, h):
                total += n * (n + 1) // 2 if causal else n * n
    return B * total


def fwd_flops(B, N, H, d, patterns, causal=True) -> int:
    return 4 * d * effective_pairs(B, N, H, patterns, causal)


def bwd_flops(B, N, H, d, patterns, causal=True) -> int:
    return 10 * d * effective_pairs(B, N, H, patterns, causal)


def bwd_flops_no_recompute(B, N, H, d, patterns, causal=True) -> int:
    return 8 * d * effective_pairs(B, N, H, patterns, causal)


def kept_rows(B: int, N: int, H: int, patterns: Sequence[Tuple[int, int]]) -> int:
    """Rows kept, summed over patterns, segments, heads and batches."""
    return B * sum(sum(segment_counts(N, w, r, h)) for (w, r) in patterns for h in range(H))


def fwd_bytes(B, N, H, d, patterns, out_res: bool = False) -> int:
    """Algorithmic HBM bytes of one bf16 forward (see the module docstring)."""
    per_row_out = 2 * d + 4 + (2 * d if out_res else 0)
    return 3 * 2 * d * kept_rows(B, N, H, patterns) + per_row_out * B * N * H
