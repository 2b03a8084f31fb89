"""Work counts for reporting: nonzero (query, key) pairs under the causal
sparse mask, effective FLOPs and algorithmic bytes.

Effective FLOPs count only the pairs the dilated patterns make nonzero:
4 d per pair forward (S = Q K^T and O += P V), 10 d per pair backward
(S recomputed, dP = dO V^T, dV, dK, dQ).
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
