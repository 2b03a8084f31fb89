"""The sequence-parallel forward's kernels on one GPU, ranks emulated in turn.

Each emulated rank packs its block's kept rows of k and v with
dilattn_pack_dilated; the packs are concatenated in rank order (what the
all-gather of the multi-GPU path delivers); then every rank's
dilattn_fwd_seqpar runs on its own block, one after another (no rank waits on
another). The assembled out and lse must match the float64 oracle on the
whole sequence, and the single-device dilattn_fwd.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_dilated_b200 import dilattn, seqpar
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS, make_inputs
from tests import oracle_pool
from tests.gpu_util import check_close, check_lse, to_device, to_f64

pytestmark = pytest.mark.gpu


def _emulate(q, k, v, pats, world, causal=True):
    B, N, H, d = q.shape
    L = N // world
    plans = seqpar.plan(N, world, pats)
    blocks = [[x[:, g * L:(g + 1) * L].contiguous() for x in (q, k, v)] for g in range(world)]
    packs = {}
    for p in plans:
        if p.spans:
            packs[p.index] = [
                torch.stack([dilattn.pack_dilated(blocks[g][j], p.r) for g in range(world)])
                for j in (1, 2)]  # [world, B, L/r, H, d] for k, v
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    for g in range(world):
        kg, vg = [None] * len(pats), [None] * len(pats)
        for p in plans:
            if p.spans:
                first = p.segment_ranks(g)[0]
                kg[p.index] = packs[p.index][0][first:first + p.ranks]
                vg[p.index] = packs[p.index][1][first:first + p.ranks]
        o, l = dilattn.fwd_seqpar(*blocks[g], pats, g, world, kg, vg, causal)
        out[:, g * L:(g + 1) * L] = o
        lse[:, :, g * L:(g + 1) * L] = l
    return out, lse


def test_pack_dilated_rows():
    inp = make_inputs(2, 1024, 3, 64, 5, "bf16")
    k, = to_device(inp, ("k",))
    got = to_f64(dilattn.pack_dilated(k, 4))
    for h in range(3):
        np.testing.assert_array_equal(got[:, :, h], inp["k"][:, (h % 4)::4, h])


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("world", [2, 4])
def test_small_against_oracle(world, causal, d):
    N, H = 4096, 4
    pats = [(512, 1), (1024, 2), (2048, 4), (4096, 8)]
    inp = make_inputs(1, N, H, d, 9, "bf16")
    q, k, v = to_device(inp)
    out, lse = _emulate(q, k, v, pats, world, causal)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    want_o, want_l = oracle.fwd(inp["q"], inp["k"], inp["v"], pats, causal)
    check_close(to_f64(out), want_o, "bf16", f"out, {world} ranks, causal={causal}, d={d}")
    check_lse(to_f64(lse), want_l, 2e-2)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_32k_against_oracle_and_single_device(world):
    wl = WORKLOADS["sweep_32768"]
    inp = make_inputs(wl.B, wl.N, wl.H, wl.d, wl.seed, wl.dtype)
    bits = {n: inp[n + "_bits"] for n in ("q", "k", "v")}
    q, k, v = to_device(inp)
    out, lse = _emulate(q, k, v, wl.patterns, world)
    ref_o, ref_l = dilattn.fwd(q, k, v, wl.patterns, True)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    check_close(to_f64(out), to_f64(ref_o), "bf16", "out vs single device")
    got = {"out": out.contiguous().view(torch.int16).cpu().numpy().view(np.uint16),
           "lse": lse.cpu().numpy()}
    stats = oracle_pool.run("fwd", bits, got, wl.patterns, True)
    oracle_pool.check(stats, "bf16", 2e-2, f"32K, {world} ranks")
