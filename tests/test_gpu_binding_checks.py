"""The binding refuses wrong output, gradient and gathered buffers on the device.

Every case swaps the library for an object that fails the test if any entry
point is reached, so an invalid buffer never gets to a kernel even if a check
were missing: the only device work here is allocating the small tensors."""
import pytest
import torch

from sparse_long_sequence_dilated_b200 import dilattn

pytestmark = pytest.mark.gpu

B, N, H, D = 1, 512, 2, 64
PATS = [(256, 1), (512, 2)]


class _NoLibrary:
    def __getattr__(self, name):
        raise AssertionError(f"{name} was reached with an invalid buffer")


@pytest.fixture(autouse=True)
def nolib(monkeypatch):
    monkeypatch.setattr(dilattn, "load", lambda *a, **k: _NoLibrary())


def bf(*s):
    return torch.zeros(s, dtype=torch.bfloat16, device="cuda")


def f32(*s):
    return torch.zeros(s, dtype=torch.float32, device="cuda")


def _cases():
    q = bf(B, N, H, D)
    lse = f32(B, H, N)
    g = f32(B, N, H, D)
    seq_pats = [(256, 1), (1024, 2)]       # N = 512 over 2 ranks: pattern 1 spans both
    good_kg = bf(2, B, 128, H, D)
    q8 = torch.zeros((B, N, H, 128), dtype=torch.uint8, device="cuda")
    v128 = bf(B, N, H, 128)
    return [
        ("fwd out shape", lambda: dilattn.fwd(q, q, q, PATS, out=bf(B, N, H, 32)), "out: shape"),
        ("fwd lse shape", lambda: dilattn.fwd(q, q, q, PATS, lse=f32(B, H, N // 2)), "lse: shape"),
        ("fwd lse dtype", lambda: dilattn.fwd(q, q, q, PATS, lse=bf(B, H, N)), "lse: dtype"),
        ("fwd out layout", lambda: dilattn.fwd(q, q, q, PATS,
                                               out=bf(B, H, N, D).transpose(1, 2)),
         "out must be contiguous"),
        ("fwd k dtype", lambda: dilattn.fwd(q, g, q, PATS), "k: dtype"),
        ("fwd v on host", lambda: dilattn.fwd(q, q, q.cpu(), PATS), "v must be on cuda"),
        ("fwd_train out_res", lambda: dilattn.fwd_train(q, q, q, PATS, out_res=bf(B, N, H, 32)),
         "out_res: shape"),
        ("bwd dq dtype", lambda: dilattn.bwd(q, q, q, q, lse, q, PATS, out_res=q, dq=q),
         "dq: dtype"),
        ("bwd dk shape", lambda: dilattn.bwd(q, q, q, q, lse, q, PATS, out_res=q,
                                             dk=f32(B, N // 2, H, D)), "dk: shape"),
        ("bwd lse shape", lambda: dilattn.bwd(q, q, q, q, f32(B, N, H), q, PATS, out_res=q),
         "lse: shape"),
        ("bwd no out_res", lambda: dilattn.bwd(q, q, q, q, lse, q, PATS), "takes out_res"),
        ("bwd out_res dtype", lambda: dilattn.bwd(q, q, q, q, lse, q, PATS, out_res=g),
         "out_res: dtype"),
        ("bwd workspace dtype", lambda: dilattn.bwd(q, q, q, q, lse, q, PATS, out_res=q,
                                                    workspace=f32(1024)), "workspace: dtype"),
        ("fwd_noalloc lse", lambda: dilattn.fwd_noalloc(q, q, q, PATS, lse=f32(B, H, 8)),
         "lse: shape"),
        ("pack out shape", lambda: dilattn.pack_dilated(q, 2, out=bf(B, N, H, D)), "out: shape"),
        ("seqpar no gathered rows", lambda: dilattn.fwd_seqpar(q[:, :256].contiguous(),
                                                               q[:, :256].contiguous(),
                                                               q[:, :256].contiguous(),
                                                               seq_pats, 0, 2),
         "needs its gathered rows"),
        ("seqpar gathered shape", lambda: dilattn.fwd_seqpar(
            q[:, :256].contiguous(), q[:, :256].contiguous(), q[:, :256].contiguous(), seq_pats,
            0, 2, [None, bf(2, B, 64, H, D)], [None, good_kg]), r"kg\[1\]: shape"),
        ("seqpar lse shape", lambda: dilattn.fwd_seqpar(
            q[:, :256].contiguous(), q[:, :256].contiguous(), q[:, :256].contiguous(), seq_pats,
            0, 2, [None, good_kg], [None, good_kg], lse=f32(B, H, N)), "lse: shape"),
        ("fp8 q8 dtype", lambda: dilattn.fwd_fp8(v128, q8, v128, [(256, 1)], 1.0, 1.0),
         "q8: dtype"),
        ("fp8 out shape", lambda: dilattn.fwd_fp8(q8, q8, v128, [(256, 1)], 1.0, 1.0,
                                                  out=bf(B, N, H, 64)), "out: shape"),
    ]


@pytest.mark.parametrize("idx", range(20))
def test_invalid_buffer_is_refused_before_the_library(idx):
    cases = _cases()
    assert len(cases) == 20
    _, call, match = cases[idx]
    with pytest.raises(ValueError, match=match):
        call()
