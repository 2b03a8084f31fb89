"""CPU checks of the parallel oracle harness used by the full-size GPU parity tests:
with the oracle's own results as the "GPU" side it must report zero error on
every slice, keep every head's offsets (a slice checked under the wrong head
index fails), and catch a planted error in one element of one slice."""
import numpy as np
import pytest

import oracle
from sparse_long_sequence_dilated_b200.workloads import make_inputs
from tests import oracle_pool

PATS = [(32, 1), (64, 2), (128, 4)]


def _case(with_dout=False):
    names = ("q", "k", "v", "dout") if with_dout else ("q", "k", "v")
    inp = make_inputs(2, 128, 3, 16, 3, "bf16", names)
    bits = {n: inp[n + "_bits"] for n in names}
    return inp, bits


def test_pool_forward_matches_in_process_oracle():
    inp, bits = _case()
    out, lse = oracle.fwd(inp["q"], inp["k"], inp["v"], PATS, True)
    got = {"out": out.astype(np.float32), "lse": lse.astype(np.float32)}
    stats = oracle_pool.run("fwd", bits, got, PATS, True)
    summ = oracle_pool.check(stats, "f32", 1e-4)
    assert summ["out"][0] < 1e-6 and summ["lse"][0] < 1e-5
    assert len(stats["out"]) == 2 * 3


def test_pool_backward_and_variants():
    inp, bits = _case(with_dout=True)
    gq, gk, gv = oracle.bwd(inp["q"], inp["k"], inp["v"], inp["dout"], PATS, True)
    out, lse = oracle.fwd(inp["q"], inp["k"], inp["v"], PATS, True)
    got = {"out": out.astype(np.float32), "lse": lse.astype(np.float32),
           "dq": gq.astype(np.float32), "dk": gk.astype(np.float32), "dv": gv.astype(np.float32),
           "dq@copy": gq.astype(np.float32)}
    stats = oracle_pool.run("bwd", bits, got, PATS, True)
    summ = oracle_pool.check(stats, "f32", 1e-4)
    assert set(summ) == {"out", "lse", "dq", "dk", "dv", "dq@copy"}


def test_pool_catches_planted_error_and_wrong_head():
    inp, bits = _case()
    out, lse = oracle.fwd(inp["q"], inp["k"], inp["v"], PATS, True)
    bad = out.astype(np.float32).copy()
    bad[1, 77, 2, 5] += 0.05
    stats = oracle_pool.run("fwd", bits, {"out": bad, "lse": lse.astype(np.float32)}, PATS, True)
    with pytest.raises(AssertionError):
        oracle_pool.check(stats, "bf16", 2e-2)
    # heads 1 and 2 swapped on the GPU side: their offsets differ for r = 2, 4
    sw = out.astype(np.float32)[:, :, [0, 2, 1], :]
    stats = oracle_pool.run("fwd", bits, {"out": sw}, PATS, True, pairs=[(0, 1)])
    with pytest.raises(AssertionError):
        oracle_pool.check(stats, "f32", 1e-4)
