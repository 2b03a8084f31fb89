"""The binding's tensor checks, on the CPU: the C entry points take bare
pointers and cannot see a buffer's size, so every torch-facing function
refuses a tensor of the wrong shape, dtype, layout or device before it calls
the library (no GPU is touched: every case fails in the checks)."""
import pytest
import torch

from sparse_long_sequence_dilated_b200 import dilattn

PATS = [(256, 1), (512, 2)]


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_need_accepts_a_matching_tensor_up_to_the_device():
    t = _bf16(1, 64, 2, 64)
    with pytest.raises(ValueError, match="must be on a CUDA device"):
        dilattn._need(t, "x", (1, 64, 2, 64), (torch.bfloat16,))


@pytest.mark.parametrize("t,match", [
    (_bf16(1, 64, 2, 32), r"x: shape \(1, 64, 2, 32\), expected \(1, 64, 2, 64\)"),
    (torch.zeros((1, 64, 2, 64), dtype=torch.float16), "x: dtype torch.float16"),
    (_bf16(1, 2, 64, 64).transpose(1, 2), "x must be contiguous"),
])
def test_need_rejects(t, match):
    with pytest.raises(ValueError, match=match):
        dilattn._need(t, "x", (1, 64, 2, 64), (torch.bfloat16,))


def test_need_lists_every_allowed_dtype():
    with pytest.raises(ValueError, match="expected torch.uint8 or torch.float8_e4m3fn"):
        dilattn._need(_bf16(4), "q8", (4,), (torch.uint8, torch.float8_e4m3fn))


def _host_calls():
    q = _bf16(1, 512, 2, 64)
    f = torch.zeros((1, 512, 2, 64), dtype=torch.float32)
    lse = torch.zeros((1, 2, 512), dtype=torch.float32)
    q8 = torch.zeros((1, 512, 2, 128), dtype=torch.uint8)
    v128 = _bf16(1, 512, 2, 128)
    return {
        "fwd": lambda: dilattn.fwd(q, q, q, PATS),
        "fwd_f32": lambda: dilattn.fwd(f, f, f, PATS),
        "fwd_train": lambda: dilattn.fwd_train(q, q, q, PATS),
        "bwd": lambda: dilattn.bwd(q, q, q, q, lse, q, PATS, out_res=q),
        "bwd_f32": lambda: dilattn.bwd(f, f, f, f, lse, f, PATS),
        "fwd_noalloc": lambda: dilattn.fwd_noalloc(q, q, q, PATS),
        "pack_dilated": lambda: dilattn.pack_dilated(q, 2),
        "fwd_seqpar": lambda: dilattn.fwd_seqpar(q, q, q, PATS, 0, 2),
        "fwd_fp8": lambda: dilattn.fwd_fp8(q8, q8, v128, [(256, 1)], 1.0, 1.0),
    }


@pytest.mark.parametrize("name", sorted(_host_calls()))
def test_wrappers_refuse_host_tensors(name):
    with pytest.raises(ValueError, match="must be on a CUDA device"):
        _host_calls()[name]()


def test_wrappers_refuse_a_wrong_input_shape_first():
    q = _bf16(1, 512, 2, 64)
    with pytest.raises(ValueError, match="expected a"):
        dilattn.fwd(q[0], q[0], q[0], PATS)
    with pytest.raises(ValueError, match="must be a multiple of r"):
        dilattn.pack_dilated(q, 3)
    with pytest.raises(ValueError, match="q: dtype"):
        dilattn.fwd(q.half(), q.half(), q.half(), PATS)
    q8 = torch.zeros((1, 512, 2, 128), dtype=torch.uint8)
    with pytest.raises(ValueError, match="v: dtype"):
        dilattn.fwd_fp8(q8, q8, torch.zeros((1, 512, 2, 128)), [(256, 1)], 1.0, 1.0)


# ---------------------------------------------------------------------------
# Marshalling: with a recording stand-in for the library and the device check
# relaxed, every wrapper hands the C entry point exactly the tensors' pointers,
# the sizes, the pattern arrays, causal and the stream.
# ---------------------------------------------------------------------------
class _Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return 4096 if name.endswith("_size") else 0
        return fn


@pytest.fixture
def rec(monkeypatch):
    r = _Recorder()
    orig = dilattn._need

    def need_on_host(t, name, shape, dtypes, device=None):
        try:
            orig(t, name, shape, dtypes)
        except ValueError as e:
            if "must be on" not in str(e):
                raise

    monkeypatch.setattr(dilattn, "load", lambda *a, **k: r)
    monkeypatch.setattr(dilattn, "_need", need_on_host)
    monkeypatch.setattr(dilattn, "_stream_handle", lambda s: 1234)
    return r


def _pats(args, i):
    w, r, n = args[i], args[i + 1], args[i + 2]
    return [(w[j], r[j]) for j in range(n)]


def test_fwd_marshalling(rec):
    q, k, v = (_bf16(2, 512, 3, 64) for _ in range(3))
    out, lse = dilattn.fwd(q, k, v, PATS, causal=False)
    name, a = rec.calls[-1]
    assert name == "dilattn_fwd"
    assert a[:5] == (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr())
    assert a[5:9] == (2, 512, 3, 64) and _pats(a, 9) == PATS and a[12:] == (0, 1234)
    assert tuple(lse.shape) == (2, 3, 512) and lse.dtype == torch.float32


def test_fwd_train_and_bwd_marshalling(rec):
    q, k, v, do = (_bf16(1, 512, 2, 64) for _ in range(4))
    out, lse, res = dilattn.fwd_train(q, k, v, PATS)
    name, a = rec.calls[-1]
    assert name == "dilattn_fwd_train"
    assert a[:6] == tuple(t.data_ptr() for t in (q, k, v, out, res, lse))
    assert a[6:10] == (1, 512, 2, 64) and _pats(a, 10) == PATS and a[13:] == (1, 1234)
    dq, dk, dv = dilattn.bwd(q, k, v, out, lse, do, PATS, out_res=res)
    names = [c[0] for c in rec.calls[-2:]]
    assert names == ["dilattn_bwd_workspace_size", "dilattn_bwd"]
    a = rec.calls[-1][1]
    assert a[:10] == tuple(t.data_ptr() for t in (q, k, v, out, res, lse, do, dq, dk, dv))
    assert a[10:14] == (1, 512, 2, 64) and _pats(a, 14) == PATS and a[17] == 1
    assert a[19] == 4096 and a[20] == 1234      # the workspace the library asked for
    assert all(t.dtype == torch.float32 for t in (dq, dk, dv))


def test_f32_paths_marshalling(rec):
    q, k, v, do = (torch.zeros((1, 256, 2, 64)) for _ in range(4))
    out, lse = dilattn.fwd(q, k, v, PATS)
    assert rec.calls[-1][0] == "dilattn_fwd_f32"
    dilattn.bwd(q, k, v, out, lse, do, PATS)
    name, a = rec.calls[-1]
    assert name == "dilattn_bwd_f32" and a[9:13] == (1, 256, 2, 64) and a[-1] == 1234


def test_noalloc_pack_seqpar_fp8_marshalling(rec):
    q = _bf16(1, 512, 2, 64)
    out, lse = dilattn.fwd_noalloc(q, q, q, PATS)
    assert rec.calls[-1][0] == "dilattn_fwd_noalloc" and rec.calls[-1][1][5:9] == (1, 512, 2, 64)
    buf = dilattn.pack_dilated(q, 4)
    name, a = rec.calls[-1]
    assert name == "dilattn_pack_dilated" and tuple(buf.shape) == (1, 128, 2, 64)
    assert a == (q.data_ptr(), buf.data_ptr(), 1, 512, 2, 64, 4, 1234)
    blk = _bf16(1, 256, 2, 64)
    kg = _bf16(2, 1, 128, 2, 64)
    vg = _bf16(2, 1, 128, 2, 64)
    o, l = dilattn.fwd_seqpar(blk, blk, blk, [(256, 1), (1024, 2)], 1, 2, [None, kg],
                              [None, vg])
    name, a = rec.calls[-1]
    assert name == "dilattn_fwd_seqpar" and a[5:9] == (1, 256, 2, 64)
    assert a[12:15] == (1, 1, 2)                # causal, rank, world
    assert [a[15][i] for i in range(2)] == [None, kg.data_ptr()]
    assert [a[16][i] for i in range(2)] == [None, vg.data_ptr()]
    q8 = torch.zeros((1, 512, 2, 128), dtype=torch.uint8)
    v = _bf16(1, 512, 2, 128)
    out, lse = dilattn.fwd_fp8(q8, q8, v, [(256, 1)], 0.5, 0.25)
    name, a = rec.calls[-1]
    assert name == "dilattn_fwd_fp8" and a[5:9] == (1, 512, 2, 128) and a[13:] == (0.5, 0.25, 1234)
