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
         v=FAKE + 8192 * 1024, out=FAKE + 16384 * 1024, lse=None):
    w, r, n = _pats(pats)
    lib = dilattn.load()
    return lib.dilattn_fwd(q, k, v, out, lse, B, N, H, d, w, r, n, causal, None)


def _bwd(ws=FAKE * 64, wsb=1 << 20, **kw):
    B, N, H, d = kw.get("B", 1), 256, 2, 64
    w, r, n = _pats(((128, 1),))
    base = [FAKE + i * (4096 * 1024) for i in range(10)]  # 4 MiB apart: nothing overlaps
    lib = dilattn.load()
    return lib.dilattn_bwd(*base, B, N, H, d, w, r, n, 1, ws, wsb, None)


@pytest.mark.parametrize("kw", [
    dict(B=0), dict(N=0), dict(H=-1), dict(d=0), dict(causal=2),
    dict(pats=()), dict(pats=((0, 1),)), dict(pats=((16, 0),)),
    dict(pats=tuple((8, 1) for _ in range(17))),
    dict(q=0), dict(q=FAKE + 8), dict(out=FAKE),  # null, misaligned, out aliases q
])
def test_fwd_rejects_invalid(kw):
    assert _fwd(**kw) == INVALID


def test_fwd_rejects_lse_overlapping_a_tensor():
    # bf16 tensors of 64 KiB at 4 MiB spacing; lse (2 KiB) starting inside k or out
    assert _fwd(lse=FAKE + 4096 * 1024 + 1024) == INVALID
    assert _fwd(lse=FAKE + 16384 * 1024 + 65536 - 16) == INVALID
    w, r, n = _pats(((128, 1),))
    lib = dilattn.load()
    t = [FAKE + i * (4096 * 1024) for i in range(5)]
    args = (1, 256, 2, 64, w, r, n, 1, None)
    # the fp32 forward: out over q, lse over out, lse over v
    assert lib.dilattn_fwd_f32(t[0], t[1], t[2], t[0] + 4096, t[4], *args) == INVALID
    assert lib.dilattn_fwd_f32(t[0], t[1], t[2], t[3], t[3] + 65536, *args) == INVALID
    assert lib.dilattn_fwd_f32(t[0], t[1], t[2], t[3], t[2] + 16, *args) == INVALID


def test_fwd_rejects_unsupported_head_dim():
    assert _fwd(d=96) == UNSUPPORTED


def test_fwd_train_needs_a_residual_buffer():
    w, r, n = _pats(((128, 1),))
    lib = dilattn.load()
    args = (1, 256, 2, 64, w, r, n, 1, None)
    assert lib.dilattn_fwd_train(FAKE, FAKE + (4 << 20), FAKE + (8 << 20), FAKE + (16 << 20), None,
                                 None, *args) == INVALID
    # out_res overlapping out
    assert lib.dilattn_fwd_train(FAKE, FAKE + (4 << 20), FAKE + (8 << 20), FAKE + (16 << 20),
                                 FAKE + (16 << 20) + 1024, None, *args) == INVALID


def test_bwd_rejects_missing_or_small_workspace():
    assert _bwd(ws=None) == WORKSPACE
    assert _bwd(wsb=16) == WORKSPACE
    assert _bwd(ws=FAKE * 64 + 16) == WORKSPACE  # not 256-byte aligned
    assert _bwd(ws=FAKE) == INVALID               # overlaps the inputs
    base = [FAKE + i * (4096 * 1024) for i in range(10)]
    w, r, n = _pats(((128, 1),))
    lib = dilattn.load()
    # q k v out out_res lse dout, then dq dk dv: dk (fp32, 128 KiB) starting inside dq's
    assert lib.dilattn_bwd(*base[:7], base[7], base[7] + 65536, base[9], 1, 256, 2, 64, w, r, n,
                           1, FAKE * 64, 1 << 20, None) == INVALID
    # out_res missing
    assert lib.dilattn_bwd(*base[:4], None, *base[5:10], 1, 256, 2, 64, w, r, n, 1, FAKE * 64,
                           1 << 20, None) == INVALID


def test_fwd_fp8_rejects_invalid():
    w, r, n = _pats(((128, 1),))
    lib = dilattn.load()
    base = (FAKE, FAKE + (4 << 20), FAKE + (8 << 20), FAKE + (16 << 20), None)

    def call(d=128, qs=1.0, ks=1.0, q=FAKE):
        return lib.dilattn_fwd_fp8(q, *base[1:], 1, 256, 2, d, w, r, n, 1, qs, ks, None)

    assert call(d=64) == UNSUPPORTED                 # built for d = 128 only
    assert call(qs=0.0) == INVALID                    # scales must be positive and finite
    assert call(ks=-1.0) == INVALID
    assert call(qs=float("nan")) == INVALID
    assert call(ks=float("inf")) == INVALID
    assert call(q=FAKE + 8) == INVALID                # misaligned
    assert call(q=FAKE + (16 << 20)) == INVALID       # out aliases q8


def test_seqpar_rejects_splits_it_cannot_run():
    lib = dilattn.load()
    L = 1024
    q, k, v, out = (FAKE + i * (4 << 20) for i in range(4))

    def call(pats, rank=0, world=2, kg=None, vg=None):
        w, r, n = _pats(pats)
        return lib.dilattn_fwd_seqpar(q, k, v, out, None, 1, L, 2, 64, w, r, n, 1, rank, world,
                                      kg, vg, None)

    assert call(((512, 1),), rank=2) == INVALID       # rank outside the group
    assert call(((512, 1),), world=0) == INVALID
    assert call(((384, 1),)) == INVALID               # a local pattern whose w does not tile L
    assert call(((2048, 2),)) == INVALID              # spanning pattern without gathered K, V
    arr = (ctypes.c_void_p * 1)(FAKE + (32 << 20))
    assert call(((2048, 3),), kg=arr, vg=arr) == INVALID   # L not a multiple of r
    assert call(((2048, 16),), kg=arr, vg=arr) == INVALID  # L / r not whole 128-row tiles
    assert call(((3072, 2),), world=4, kg=arr, vg=arr) == INVALID  # N not a multiple of w
    # out (256 KiB at FAKE + 12 MiB) over the gathered rows (2 ranks x 512 rows, 256 KiB)
    inside = (ctypes.c_void_p * 1)(out + (128 << 10))
    assert call(((2048, 2),), kg=inside, vg=arr) == INVALID
    assert call(((2048, 2),), kg=arr, vg=(ctypes.c_void_p * 1)(out - (128 << 10))) == INVALID
    # lse (8 KiB) inside the gathered k rows
    w, r, n = _pats(((2048, 2),))
    assert lib.dilattn_fwd_seqpar(q, k, v, out, FAKE + (32 << 20) + 4096, 1, L, 2, 64, w, r, n,
                                  1, 0, 2, arr, (ctypes.c_void_p * 1)(FAKE + (40 << 20)),
                                  None) == INVALID


def test_pack_dilated_rejects_invalid():
    lib = dilattn.load()
    x, buf = FAKE, FAKE + (8 << 20)
    assert lib.dilattn_pack_dilated(x, buf, 1, 1000, 2, 64, 3, None) == INVALID  # L % r != 0
    assert lib.dilattn_pack_dilated(x, buf, 1, 1024, 2, 96, 4, None) == INVALID  # d
    assert lib.dilattn_pack_dilated(x + 8, buf, 1, 1024, 2, 64, 4, None) == INVALID
    assert lib.dilattn_pack_dilated(x, x + 4096, 1, 1024, 2, 64, 4, None) == INVALID  # overlap


def test_scratch_and_workspace_sizes():
    lib = dilattn.load()
    align = lambda x: (x + 255) // 256 * 256
    w, r, n = _pats(((128, 1), (256, 2), (512, 4)))
    # the r = 1 pattern merges and stores no partials; partial rows of the
    # others: B*H*nseg_i*(128*ceil(ceil(min(w,N)/r)/128)) = 2*3*(2*128 + 1*128)
    rows = 2 * 3 * (256 + 128)
    flags = align((rows // 128 + 1) * 4 + 8)  # one flag per 128-row block, then two counters
    assert lib.dilattn_fwd_scratch_size(2, 512, 3, 64, w, r, n) == \
        align(rows * 64 * 4) + align(rows * 4) + flags
    # no r = 1 pattern: every pattern stores partials (334 rows -> 384)
    assert lib.dilattn_fwd_scratch_size(1, 1000, 1, 64, *_pats(((1000, 3),))) == \
        384 * 64 * 4 + align(384 * 4) + align((384 // 128 + 1) * 4 + 8)
    # of two r = 1 patterns the shorter merges
    w2, r2, n2 = _pats(((512, 1), (256, 1)))
    assert lib.dilattn_fwd_scratch_size(1, 512, 1, 64, w2, r2, n2) == \
        align(512 * 64 * 4) + align(512 * 4) + align((512 // 128 + 1) * 4 + 8)
    # D, 256 bytes for the key-tile kernel's unit counter, fp16 copies of q and k
    # (the fp32 gradients are the caller's outputs)
    assert lib.dilattn_bwd_workspace_size(2, 512, 3, 64) == \
        align(2 * 3 * 512 * 4) + 256 + 2 * align(2 * 512 * 3 * 64 * 2)
    assert lib.dilattn_fwd_scratch_size(0, 512, 3, 64, w, r, n) == 0
    assert lib.dilattn_bwd_workspace_size(0, 512, 3, 64) == 0


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


def test_pattern_limit_agrees_everywhere():
    # the header's limit, the binding's and the kernels' per-pattern arrays
    header = open(HEADER, encoding="utf-8").read()
    common = open(os.path.join(ROOT, "sparse_long_sequence_dilated_b200", "csrc", "common.cuh"),
                  encoding="utf-8").read()
    h = int(re.search(r"#define DILATTN_MAX_PATTERNS (\d+)", header).group(1))
    k = int(re.search(r"constexpr int kMaxPat = (\d+);", common).group(1))
    assert h == k == dilattn.MAX_PATTERNS


def test_bwd_rejects_head_dim_128_as_unsupported():
    w, r, n = _pats(((128, 1),))
    base = [FAKE + i * (4096 * 1024) for i in range(10)]
    lib = dilattn.load()
    assert lib.dilattn_bwd(*base, 1, 256, 2, 128, w, r, n, 1, FAKE * 64, 1 << 22,
                           None) == UNSUPPORTED
