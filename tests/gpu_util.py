"""Helpers shared by the GPU parity tests: move seeded inputs to the device and
compare against float64 oracle values with the stated tolerances."""
import numpy as np
import torch

# bf16 inputs: max-abs <= 2e-2 and relative L2 <= 5e-3; fp32 inputs: max-abs <= 1e-4
BF16_ATOL = 2e-2
BF16_REL_L2 = 5e-3
F32_ATOL = 1e-4


def to_device(inputs, names=("q", "k", "v"), dtype="bf16"):
    out = []
    for n in names:
        if dtype == "bf16":
            bits = np.ascontiguousarray(inputs[n + "_bits"]).view(np.int16)
            out.append(torch.from_numpy(bits).view(torch.bfloat16).cuda())
        else:
            out.append(torch.from_numpy(np.ascontiguousarray(inputs[n])).cuda())
    return out


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(got, want, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    if dtype == "bf16":
        den = float(np.sqrt((want ** 2).sum()))
        rel = float(np.sqrt((err ** 2).sum()) / den) if den > 0 else float(np.sqrt((err ** 2).sum()))
        assert max_abs <= BF16_ATOL and rel <= BF16_REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
        return max_abs, rel
    assert max_abs <= F32_ATOL, f"{what}: max_abs={max_abs:.3e}"
    return max_abs, None


def check_lse(got, want, atol, what="lse"):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: -inf pattern differs"
    assert np.all(got[~fin] == -np.inf), f"{what}: unselected rows must be -inf"
    if fin.any():
        e = float(np.abs(got[fin] - want[fin]).max())
        assert e <= atol, f"{what}: max_abs={e:.3e}"
