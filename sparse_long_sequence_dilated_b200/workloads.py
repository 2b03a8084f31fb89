"""Workload shapes and seeded synthetic inputs.

This module holds no attention arithmetic: only problem shapes, (w, r)
pattern lists and a seeded Gaussian generator. Both the float64 CPU oracle
and the CUDA path draw their inputs from here, so the two sides see the same
numbers without sharing any code that computes the method.

Inputs stand in for the language-modelling data the LongNet pages train on
(The Stack, named in the gptget.net summary of arXiv 2307.02486, section
"实验设计"); the kernels' cost does not depend on the values, so i.i.d.
N(0, 1) tensors of the right shapes replace it.

Generator recipe: ``numpy.random.default_rng(seed)`` (PCG64); q, k, v and
then dO are drawn in that order as float32 standard normals of shape
[B, N, H, d]. For bf16 workloads each value is rounded to bfloat16
(round-to-nearest-even on the float32 bit pattern) and both the bf16 bit
pattern (uint16) and its exact float32 value are returned.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

Pattern = Tuple[int, int]  # (segment length w, dilation rate r)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    d: int
    dtype: str  # "bf16" or "f32"
    patterns: Tuple[Pattern, ...]
    causal: bool = True
    seed: int = 0
    backward: bool = False

    @property
    def w(self) -> List[int]:
        return [p[0] for p in self.patterns]

    @property
    def r(self) -> List[int]:
        return [p[1] for p in self.patterns]


def geometric_patterns(N: int, w0: int = 2048, wmax: Optional[int] = None) -> Tuple[Pattern, ...]:
    """w = w0 * 2**i, r = 2**i for i = 0, 1, ... while w <= wmax (default N)."""
    wmax = N if wmax is None else wmax
    pats = []
    i = 0
    while w0 * (1 << i) <= wmax:
        pats.append((w0 * (1 << i), 1 << i))
        i += 1
    return tuple(pats)


def _sweep(N: int) -> Workload:
    return Workload(f"sweep_{N}", 1, N, 12, 64, "bf16", geometric_patterns(N), True, 0, True)


WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 case, forward only
    "tiny_f32": Workload("tiny_f32", 1, 512, 4, 64, "f32",
                         ((128, 1), (256, 2), (512, 4)), True, 0, False),
    # LongNet-base layer shape (d_model 768 = 12 heads x 64)
    "longnet_base_32k": Workload("longnet_base_32k", 1, 32768, 12, 64, "bf16",
                                 ((2048, 1), (4096, 2), (8192, 4), (16384, 6), (32768, 12)),
                                 True, 0, True),
    # length sweep
    "sweep_8192": _sweep(8192),
    "sweep_32768": _sweep(32768),
    "sweep_131072": _sweep(131072),
    "sweep_262144": _sweep(262144),
    "sweep_1048576": _sweep(1048576),
    # wide model (d_model 4096 = 32 heads x 128), forward
    "wide_128k": Workload("wide_128k", 2, 131072, 32, 128, "bf16",
                          geometric_patterns(131072), True, 0, False),
    # training step: sweep shapes at B = 4
    "train_b4_32k": Workload("train_b4_32k", 4, 32768, 12, 64, "bf16",
                             geometric_patterns(32768), True, 0, True),
    # gradient check of the training step at N = 2048 with scaled-down patterns
    "train_check_2k": Workload("train_check_2k", 4, 2048, 12, 64, "bf16",
                               ((256, 1), (512, 2), (1024, 4), (2048, 8)), True, 0, True),
}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit pattern (uint16), round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    flat_u = u.reshape(-1)
    flat_o = out.reshape(-1)
    step = 1 << 24
    for s in range(0, flat_u.size, step):
        c = flat_u[s:s + step].astype(np.uint64)
        lsb = (c >> 16) & 1
        flat_o[s:s + step] = ((c + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def make_inputs(B: int, N: int, H: int, d: int, seed: int = 0, dtype: str = "bf16",
                names: Sequence[str] = ("q", "k", "v")) -> Dict[str, np.ndarray]:
    """Seeded i.i.d. N(0, 1) tensors of shape [B, N, H, d] drawn in ``names`` order.

    Returns ``{name: float32 values}`` and, for bf16, also ``{name + "_bits": uint16}``.
    The float32 values of a bf16 workload are exactly the bf16 values.
    """
    rng = np.random.default_rng(seed)
    out: Dict[str, np.ndarray] = {}
    for name in names:
        x = rng.standard_normal((B, N, H, d), dtype=np.float32)
        if dtype == "bf16":
            bits = round_to_bf16_bits(x)
            out[name + "_bits"] = bits
            out[name] = bf16_bits_to_f32(bits)
        elif dtype == "f32":
            out[name] = x
        else:
            raise ValueError(f"unknown dtype {dtype!r}")
    return out


def e4m3_values() -> np.ndarray:
    """The value of every e4m3 code 0..255 (sign, 4 exponent bits with bias 7, 3
    mantissa bits; exponent 0 is subnormal, m * 2^-9; code 0x7F / 0xFF is NaN)."""
    vals = np.zeros(256, dtype=np.float64)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals[c] = -v if s else v
    vals[0x7F] = vals[0xFF] = np.nan
    return vals


def quantize_e4m3(x: np.ndarray, amax: float = 448.0):
    """Per-tensor e4m3 quantisation of an input: scale = max|x| / amax; each
    x / scale rounded to the nearest e4m3 value (ties to even code).

    Returns (codes uint8, scale float32, values float64 = decoded codes * scale,
    exactly the numbers an e4m3 kernel computes on)."""
    x = np.asarray(x, dtype=np.float64)
    scale = np.float32(max(float(np.abs(x).max()), 1e-30) / amax)
    y = x / np.float64(scale)
    table = e4m3_values()
    pos = table[:0x7F]                      # non-negative finite values, increasing
    a = np.minimum(np.abs(y), pos[-1]).ravel()
    hi = np.searchsorted(pos, a)            # first value >= a
    hi = np.minimum(hi, len(pos) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - pos[lo], pos[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(y.ravel() < 0, code | 0x80, code).astype(np.uint8).reshape(x.shape)
    return code, scale, table[code] * np.float64(scale)
