"""The FMA-pipe exp2 used by the forward kernel (ex2_poly in csrc/common.cuh).

Checks, on the CPU: the kernel's constants are the ones the Remez fit script
produces; a float32 emulation of the kernel's steps (1.5 * 2^23 rounding trick,
Horner with fused multiply-adds, exponent-field add) stays within the fit's
error bound of 2^x over the range the kernel uses; and -inf maps to a
negligible value instead of NaN.
"""
import os
import re

import numpy as np

from sparse_long_sequence_dilated_b200.csrc import fit_exp2_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "sparse_long_sequence_dilated_b200", "csrc", "common.cuh")


def kernel_coeffs(fn="float ex2_poly(float x)"):
    text = open(SRC, encoding="utf-8").read()
    body = text[text.index(fn):]
    body = body[:body.index("return")]
    nums = [float(x.rstrip("f")) for x in re.findall(r"[0-9]\.[0-9]+e[-+][0-9]+f", body)]
    nums = list(dict.fromkeys(nums))  # the packed form repeats each constant for both lanes
    # Horner order in the source: c3, c2, c1, c0
    return np.array(nums[::-1], dtype=np.float32)


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_poly_emulated(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma32(fma32(fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2])), f,
                    np.full_like(f, c[1])), f, np.full_like(f, c[0]))
    j = (t.view(np.int32).astype(np.int64) - 0x4B400000).astype(np.int64)
    bits = (p.view(np.uint32).astype(np.int64) + (j << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_kernel_constants_match_fit():
    want = fit_exp2_poly.remez().astype(np.float32)
    for fn in ("float ex2_poly(float x)", "uint64_t ex2_poly2(uint64_t x2)"):
        got = kernel_coeffs(fn)
        assert got.shape == (4,), fn
        np.testing.assert_allclose(got, want, rtol=2e-7, atol=0, err_msg=fn)


def test_exponent_shift_forms_agree():
    # the packed form adds (t_bits << 23) instead of ((t_bits - 0x4B400000) << 23)
    x = np.linspace(-125.0, 126.0, 100001).astype(np.float32)
    t = (x + np.float32(12582912.0)).astype(np.float32).view(np.uint32).astype(np.uint64)
    a = ((t - 0x4B400000) << 23) & 0xFFFFFFFF
    b = (t << 23) & 0xFFFFFFFF
    assert np.array_equal(a, b)


def test_relative_error_bound():
    c = kernel_coeffs()
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), -np.linspace(0, 1, 1001)])
    x = x.astype(np.float32)
    got = ex2_poly_emulated(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 8e-5, rel.max()


def test_minus_infinity_is_negligible():
    c = kernel_coeffs()
    y = ex2_poly_emulated(np.array([-np.inf, -1e30, -200.0], dtype=np.float32), c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 3e-38)
