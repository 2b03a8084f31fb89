"""The seeded input generator both sides share (workloads.py), on the CPU: its
bf16 rounding is round-to-nearest-even exactly as torch's float32 -> bfloat16
cast, the float32 values of a bf16 workload are exactly its bf16 values, and
the draws are fixed by the seed and by the order of the names."""
import numpy as np
import pytest
import torch

from sparse_long_sequence_dilated_b200.workloads import (WORKLOADS, bf16_bits_to_f32,
                                                         geometric_patterns, make_inputs,
                                                         round_to_bf16_bits)


def _torch_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_rounding_matches_torch_on_random_and_extreme_values():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),   # subnormals
        np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38, np.finfo(np.float32).max,
                  np.finfo(np.float32).tiny, np.inf, -np.inf], dtype=np.float32),
    ])
    np.testing.assert_array_equal(round_to_bf16_bits(x), _torch_bits(x))


def test_ties_go_to_even():
    # bits with the low half exactly 0x8000: half-way between two bf16 values
    hi = np.arange(0x3F80, 0x3F90, dtype=np.uint32)
    x = ((hi << 16) | 0x8000).view(np.float32)
    got = round_to_bf16_bits(x).astype(np.uint32)
    want = np.where(hi % 2 == 0, hi, hi + 1)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got, _torch_bits(x))
    # one unit above the tie always rounds up, one below always down
    np.testing.assert_array_equal(round_to_bf16_bits(((hi << 16) | 0x8001).view(np.float32)),
                                  hi + 1)
    np.testing.assert_array_equal(round_to_bf16_bits(((hi << 16) | 0x7FFF).view(np.float32)),
                                  hi)


def test_bf16_workload_values_are_its_bits():
    inp = make_inputs(2, 64, 3, 16, seed=7)
    for n in ("q", "k", "v"):
        np.testing.assert_array_equal(inp[n], bf16_bits_to_f32(inp[n + "_bits"]))
        t = torch.from_numpy(inp[n + "_bits"].view(np.int16)).view(torch.bfloat16).float()
        np.testing.assert_array_equal(t.numpy(), inp[n])


def test_draws_fixed_by_seed_and_name_order():
    a = make_inputs(1, 128, 2, 8, seed=3, names=("q", "k", "v", "dout"))
    b = make_inputs(1, 128, 2, 8, seed=3, names=("q", "k", "v"))
    c = make_inputs(1, 128, 2, 8, seed=4, names=("q",))
    for n in ("q", "k", "v"):
        np.testing.assert_array_equal(a[n + "_bits"], b[n + "_bits"])
    assert not np.array_equal(a["q"], c["q"])
    assert not np.array_equal(a["q"], a["k"])
    f = make_inputs(1, 128, 2, 8, seed=3, dtype="f32", names=("q",))
    np.testing.assert_array_equal(round_to_bf16_bits(f["q"]), a["q_bits"])


def test_draws_are_standard_normal():
    x = make_inputs(1, 4096, 4, 64, seed=0, dtype="f32", names=("q",))["q"]
    assert x.shape == (1, 4096, 4, 64) and x.dtype == np.float32
    assert abs(float(x.mean())) < 0.01 and abs(float(x.std()) - 1.0) < 0.01


def test_unknown_dtype_is_refused():
    with pytest.raises(ValueError):
        make_inputs(1, 8, 1, 8, dtype="f16")


def test_geometric_families():
    assert geometric_patterns(8192) == ((2048, 1), (4096, 2), (8192, 4))
    assert geometric_patterns(1 << 20)[-1] == (1 << 20, 512)
    assert WORKLOADS["sweep_131072"].patterns == geometric_patterns(131072)
    assert WORKLOADS["longnet_base_32k"].patterns == ((2048, 1), (4096, 2), (8192, 4),
                                                      (16384, 6), (32768, 12))
