"""Failure detection on the GPU without a GPU fault.

Every wait in the kernels is bounded: on running out it records a code in the
library's device error word, raises the CTA's abort flag so the other warps
stop waiting too, and the kernel returns. dilattn_selftest_wait_timeout makes
one wait run out on purpose (an mbarrier that nothing arrives on, 1 ms
limit) and a second warp wait with the ordinary 4 s limit; this checks that
the kernel returns promptly, that the code is reported once and then
cleared, and that an unread failure does not disturb a later forward call.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_long_sequence_dilated_b200 import dilattn
from sparse_long_sequence_dilated_b200.workloads import make_inputs
from tests.gpu_util import check_close, check_lse, to_device, to_f64

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    assert dilattn.device_error() == 0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    res = dilattn.selftest_wait_timeout(1_000_000)
    ev1.record()
    torch.cuda.synchronize()
    r = res.cpu().tolist()
    assert r[0] == 0 and r[1] == 0, r          # neither wait completed
    assert 1_000_000 <= r[2] < 200_000_000, r  # warp 0 gave up after its 1 ms limit
    assert r[3] < 200_000_000, r               # warp 1 followed the abort, not its 4 s limit
    assert ev0.elapsed_time(ev1) < 1000.0
    assert dilattn.device_error() == 1         # kErrWaitTimeout, read once ...
    assert dilattn.device_error() == 0         # ... and cleared


def test_unread_failure_does_not_disturb_later_calls():
    dilattn.selftest_wait_timeout(1_000_000)   # leaves code 1 unread
    pats = [(256, 1), (512, 2), (1024, 4)]
    inp = make_inputs(1, 1024, 4, 64, 31, "bf16")
    q, k, v = to_device(inp)
    out, lse = dilattn.fwd(q, k, v, pats, True)
    torch.cuda.synchronize()
    want_o, want_l = oracle.fwd(inp["q"], inp["k"], inp["v"], pats, True)
    check_close(to_f64(out), want_o, "bf16", "out after an unread failure")
    check_lse(to_f64(lse), want_l, 2e-2)
    assert dilattn.device_error() == 1
    assert dilattn.device_error() == 0
