"""Host-only checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments with status codes before touching
the GPU (so these run without one)."""
import ctypes
import os
import re

import pytest

from sparse_long_sequence_dilated_b200 import dilattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dilattn.h")

OK, INVALID, UNSUPPORTED, CUDA, WORKSPACE = 0, 1, 2, 3, 4
FAKE = 1 << 20  # 16-byte aligned fake device address; never dereferenced by a rejected call


def header_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dilattn_[a-z0-9_]+)\s*\(", text)))


def test_binding_covers_header_exactly():
    assert header_functions() == sorted(dilattn.SIGNATURES)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(dilattn.LIB_PATH)
    for name in header_functions():
        assert hasattr(lib, name), name


def test_noalloc_scratch_constant_matches_header():
    text = open(HEADER, encoding="utf-8").read()
    m = re.search(r"#define DILATTN_NOALLOC_SCRATCH_BYTES \((\d+)u \* 1024u \* 1024u\)", text)
    assert m is not None
    assert dilattn.NOALLOC_SCRATCH_BYTES == int(m.group(1)) * 1024 * 1024


def test_status_strings():
    assert dilattn.status_string(0) == "DILATTN_OK"
    assert dilattn.status_string(4) == "DILATTN_ERR_WORKSPACE"
    assert dilattn.status_string(99) == "DILATTN_UNKNOWN_STATUS"


def _pats(p):
    return dilattn._patterns(p)


def _fwd(B=1, N=256, H=2, d=64, pats=((128, 1),), causal=1, q=FAKE, k=FAKE + 4096 * 1024,
         v=FAKE + 8192 * 1024, out=FAKE + 16384 * 1024, lse=None, ws=None, wsb=0):
    w, r, n = _pats(pats)
    lib = dilattn.load()
    return lib.dilattn_fwd(q, k, v, out, lse, B, N, H, d, w, r, n, causal, ws, wsb, None)


@pytest.mark.parametrize("kw", [
    dict(B=0), dict(N=0), dict(H=-1), dict(d=0), dict(causal=2),
    dict(pats=()), dict(pats=((0, 1),)), dict(pats=((16, 0),)),
    dict(pats=tuple((8, 1) for _ in range(17))),
    dict(q=0), dict(q=FAKE + 8), dict(out=FAKE),  # null, misaligned, out aliases q
])
def test_fwd_rejects_invalid(kw):
    assert _fwd(**kw) == INVALID


def test_fwd_rejects_unsupported_head_dim():
    assert _fwd(d=96) == UNSUPPORTED


def test_fwd_rejects_missing_or_small_workspace():
    assert _fwd(ws=None) == WORKSPACE
    assert _fwd(ws=FAKE * 64, wsb=16) == WORKSPACE
    assert _fwd(ws=FAKE * 64 + 16, wsb=1 << 30) == WORKSPACE  # not 256-byte aligned


def test_workspace_sizes():
    lib = dilattn.load()
    w, r, n = _pats(((128, 1), (256, 2), (512, 4)))
    # partial rows: sum_i B*H*nseg_i*(128*ceil(ceil(min(w,N)/r)/128)) = 2*3*(4*128 + 2*128 + 1*128)
    rows = 2 * 3 * (512 + 256 + 128)
    align = lambda x: (x + 255) // 256 * 256
    assert lib.dilattn_fwd_workspace_size(1, 1000, 1, 64, *_pats(((1000, 3),))) == \
        384 * 64 * 4 + align(384 * 4) + align(1000 * 64 * 4)  # 334 rows -> 384
    # partial outputs, partial lse, then an fp32 copy of out
    assert lib.dilattn_fwd_workspace_size(2, 512, 3, 64, w, r, n) == \
        align(rows * 64 * 4) + align(rows * 4) + align(2 * 512 * 3 * 64 * 4)
    t = 2 * 512 * 3 * 64 * 4
    # dq, dk, dv accumulators, D, then 256 bytes for the key-tile kernel's unit counter
    assert lib.dilattn_bwd_workspace_size(2, 512, 3, 64, w, r, n) == \
        3 * align(t) + align(2 * 3 * 512 * 4) + 256
    assert lib.dilattn_fwd_workspace_size(0, 512, 3, 64, w, r, n) == 0


def test_valid_call_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    w, r, n = _pats(((128, 1),))
    lib = dilattn.load()
    rc = lib.dilattn_fwd_f32(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, None, 1, 256, 2, 64, w, r, n, 1,
                             None)
    assert rc in (CUDA, UNSUPPORTED)
    assert isinstance(dilattn.last_error(), str)


# ---------------------------------------------------------------------------
# host-side work counts against the oracle's brute-force multiplicity count
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("pats", [[(8, 1), (16, 2), (32, 4)], [(8, 1), (12, 2), (20, 3), (30, 6)],
                                  [(5, 1), (7, 7), (3, 5)], [(9, 4)]])
@pytest.mark.parametrize("causal", [True, False])
def test_effective_pairs_matches_oracle(pats, causal):
    import oracle
    from sparse_long_sequence_dilated_b200 import flops
    assert flops.effective_pairs(2, 30, 5, pats, causal) == oracle.effective_pairs(2, 30, 5, pats, causal)
    want = sum(int(oracle.multiplicity(30, pats, h, causal).sum()) for h in range(5))
    assert flops.effective_pairs(1, 30, 5, pats, causal) == want
