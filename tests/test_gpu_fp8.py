"""The FP8 forward (e4m3 q and k, bf16 v, d = 128) against the float64 oracle.

q and k are quantised per tensor to e4m3 (tests' input recipe,
workloads.quantize_e4m3); the oracle runs on the dequantised values, so the
quantisation is an input of the forward, as the bf16 rounding of the inputs
is for the bf16 path, and the bounds are the bf16 ones: S = Q K^T is exact
on e4m3 inputs and P, V, PV are as in the bf16 kernel."""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_dilated_b200 import dilattn
from sparse_long_sequence_dilated_b200.workloads import (geometric_patterns, make_inputs,
                                                          quantize_e4m3)
from tests import oracle_pool
from tests.gpu_util import check_close, check_lse, to_f64

pytestmark = pytest.mark.gpu


def _case(B, N, H, seed):
    inp = make_inputs(B, N, H, 128, seed, "bf16")
    q8, qs, qv = quantize_e4m3(inp["q"])
    k8, ks, kv = quantize_e4m3(inp["k"])
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    v = torch.from_numpy(np.ascontiguousarray(inp["v_bits"]).view(np.int16)).view(torch.bfloat16).cuda()
    return (dev(q8), dev(k8), v, float(qs), float(ks)), (qv, kv, inp["v"], inp["v_bits"])


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pats", [
    [(256, 1), (512, 2), (1536, 4)],
    [(500, 2), (1536, 3)],            # no r = 1 pattern: separate merge pass
])
def test_small_full(pats, causal):
    (q8, k8, v, qs, ks), (qv, kv, vv, _) = _case(1, 1536, 4, 41)
    out, lse = dilattn.fwd_fp8(q8, k8, v, pats, qs, ks, causal)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    want_o, want_l = oracle.fwd(qv, kv, vv, pats, causal)
    check_close(to_f64(out), want_o, "bf16", "fp8 out")
    check_lse(to_f64(lse), want_l, 2e-2)


@pytest.mark.parametrize("causal", [True, False])
def test_ragged_full(causal):
    # N and the segments not multiples of the 64-row key tiles or 128-row query tiles
    pats = [(384, 1), (700, 3), (1000, 6), (1100, 12)]
    (q8, k8, v, qs, ks), (qv, kv, vv, _) = _case(2, 1100, 3, 43)
    out, lse = dilattn.fwd_fp8(q8, k8, v, pats, qs, ks, causal)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    want_o, want_l = oracle.fwd(qv, kv, vv, pats, causal)
    check_close(to_f64(out), want_o, "bf16", "fp8 out, ragged")
    check_lse(to_f64(lse), want_l, 2e-2)


def test_16k_every_element():
    N, H = 16384, 8
    pats = geometric_patterns(N)
    (q8, k8, v, qs, ks), (qv, kv, vv, v_bits) = _case(1, N, H, 42)
    out, lse = dilattn.fwd_fp8(q8, k8, v, pats, qs, ks, True)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    got = {"out": out.contiguous().view(torch.int16).cpu().numpy().view(np.uint16),
           "lse": lse.cpu().numpy()}
    stats = oracle_pool.run("fwd", {"q": qv, "k": kv, "v": v_bits}, got, pats, True)
    oracle_pool.check(stats, "bf16", 2e-2, "fp8 16K")
