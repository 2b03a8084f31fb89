"""The forward entry point that allocates nothing, dilattn_fwd_noalloc.

Some callers cannot hand the library a workspace: a plugin that is given only
its input and output pointers, a server that reserves all device memory at
start-up and forbids cudaMalloc afterwards. For them the library keeps the
forward's scratch (per-pattern partial results) in a fixed 64 MiB array of its
own. These tests run that entry point through the C ABI and compare it with
dilattn_fwd, which takes its scratch from the library's memory pool, on
calls in a row with different shapes, patterns and inputs (with and without
an r = 1 pattern, so both ways of merging run on the shared array), so
scratch read from the wrong place or left over from an earlier call would
show up; and they check that a problem too large for the array is refused.

This file is named to be collected last: a failure here stops a -x run only
after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_long_sequence_dilated_b200 import dilattn
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS, make_inputs
from tests.gpu_util import check_close, check_lse, to_device, to_f64

pytestmark = pytest.mark.gpu

PATS = [(256, 1), (512, 2), (1024, 4), (2048, 8)]


def _noalloc(q, k, v, out, lse, pats):
    B, N, H, d = q.shape
    w, r, n = dilattn._patterns(pats)
    rc = dilattn.load().dilattn_fwd_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
        B, N, H, d, w, r, n, 1, torch.cuda.current_stream().cuda_stream)
    assert rc == 0, (dilattn.status_string(rc), dilattn.last_error())


# two problems with different scratch layouts: the second call reuses the
# array with other pattern counts, segment sizes and row offsets, so an entry
# read from the wrong place (or left over from the first call) shows up
CALLS = [
    (2, 2048, 8, PATS, 21),
    (1, 3000, 6, [(300, 1), (700, 3), (3000, 5)], 22),
    (1, 1500, 4, [(500, 2), (1500, 3)], 23),  # no r = 1 pattern: separate merge pass
]


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_matches_pooled_forward_on_consecutive_calls(d):
    calls = []
    for B, N, H, pats, seed in CALLS:
        assert dilattn.fwd_scratch_size(B, N, H, d, pats) <= dilattn.NOALLOC_SCRATCH_BYTES
        q, k, v = to_device(make_inputs(B, N, H, d, seed, "bf16"))
        out = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        calls.append((q, k, v, out, lse, pats))
    # the calls in a row on the shared scratch
    for q, k, v, out, lse, pats in calls:
        _noalloc(q, k, v, out, lse, pats)
    torch.cuda.synchronize()
    assert dilattn.device_error() == 0
    for q, k, v, out, lse, pats in calls:
        ref_o, ref_l = dilattn.fwd(q, k, v, pats, True)
        torch.cuda.synchronize()
        check_close(to_f64(out), to_f64(ref_o), "bf16", "out vs dilattn_fwd")
        check_lse(to_f64(lse), to_f64(ref_l), 2e-2, "lse vs dilattn_fwd")


def test_noalloc_refuses_problems_larger_than_its_scratch():
    wl = WORKLOADS["longnet_base_32k"]
    need = dilattn.fwd_scratch_size(wl.B, wl.N, wl.H, wl.d, wl.patterns)
    assert need > dilattn.NOALLOC_SCRATCH_BYTES
    w, r, n = dilattn._patterns(wl.patterns)
    base = 1 << 20  # aligned stand-in pointers: a refused call touches no memory
    step = wl.B * wl.N * wl.H * wl.d * 2
    rc = dilattn.load().dilattn_fwd_noalloc(base, base + step, base + 2 * step, base + 3 * step,
                                            None, wl.B, wl.N, wl.H, wl.d, w, r, n, 1, None)
    assert rc == 4  # DILATTN_ERR_WORKSPACE
    assert "scratch" in dilattn.last_error()
