"""The e4m3 input quantiser of the FP8 forward's tests, pinned to torch's
float8_e4m3fn cast (round to nearest even) on the CPU, and its code table to
the format's definition at a few hand-checked points."""
import numpy as np
import torch

from sparse_long_sequence_dilated_b200.workloads import e4m3_values, quantize_e4m3


def test_code_table_points():
    t = e4m3_values()
    assert t[0] == 0.0 and t[1] == 2.0 ** -9 and t[7] == 7 * 2.0 ** -9   # subnormals
    assert t[8] == 2.0 ** -6 and t[0x38] == 1.0 and t[0x7E] == 448.0     # normals, max
    assert t[0x80 | 0x38] == -1.0 and np.isnan(t[0x7F])


def test_quantiser_matches_torch_float8_cast():
    x = np.random.default_rng(3).standard_normal(200000) * 3.0
    codes, scale, vals = quantize_e4m3(x)
    y = torch.from_numpy(x / np.float64(scale)).to(torch.float8_e4m3fn)
    assert np.array_equal(codes, y.view(torch.uint8).numpy())
    assert np.array_equal(vals, y.to(torch.float64).numpy() * np.float64(scale))
    assert np.abs(x / scale).max() <= 448.0 * (1 + 1e-6)
