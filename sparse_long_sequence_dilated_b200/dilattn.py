"""Thin ctypes binding of libdilattn (include/dilattn.h).

The ``dilattn_*`` functions mirror the C entry points one to one (integer
device pointers and sizes). The torch-facing functions (``fwd``,
``fwd_train``, ``bwd``, ``fwd_fp8``, ``fwd_noalloc``, ``fwd_seqpar``,
``pack_dilated``, ``selection``) add only argument marshalling for torch
tensors: checks of every tensor's shape, dtype, layout and device (the C
entry points take bare pointers and cannot see a buffer's size), output and
workspace allocation with torch, and the current CUDA stream. Every step of the
computation runs in the library's CUDA kernels; there is no other code path,
and a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdilattn.so")

DILATTN_OK = 0
MAX_PATTERNS = 16

_c = ctypes
_vp = _c.c_void_p
_i = _c.c_int
_sz = _c.c_size_t
_ip = _c.POINTER(_c.c_int)

# name -> (restype, argtypes); exactly the functions include/dilattn.h declares
SIGNATURES = {
    "dilattn_status_string": (_c.c_char_p, [_i]),
    "dilattn_last_error": (_c.c_char_p, []),
    "dilattn_fwd_scratch_size": (_sz, [_i, _i, _i, _i, _ip, _ip, _i]),
    "dilattn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _vp]),
    "dilattn_fwd_train": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _vp]),
    "dilattn_fwd_fp8": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _c.c_float,
                             _c.c_float, _vp]),
    "dilattn_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _vp]),
    "dilattn_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "dilattn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip,
                         _i, _i, _vp, _sz, _vp]),
    "dilattn_fwd_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _vp]),
    "dilattn_bwd_f32": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip,
                             _i, _i, _vp]),
    "dilattn_selection": (_i, [_vp, _i, _i, _ip, _ip, _i, _vp]),
    "dilattn_set_trace_events": (_i, [_vp, _vp]),
    "dilattn_device_error": (_i, [_vp, _ip]),
    "dilattn_selftest_wait_timeout": (_i, [_c.c_ulonglong, _vp, _vp]),
    "dilattn_fwd_seqpar": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _ip, _ip, _i, _i, _i, _i,
                                _c.POINTER(_vp), _c.POINTER(_vp), _vp]),
    "dilattn_pack_dilated": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp]),
}

_lib = None


class DilattnError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


def load(path: str = LIB_PATH):
    """Load libdilattn.so (raises if it is missing or lacks a declared symbol)."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m sparse_long_sequence_dilated_b200.build`")
    lib = _c.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def __getattr__(name):
    if name in SIGNATURES:
        return getattr(load(), name)
    raise AttributeError(name)


def status_string(status: int) -> str:
    return load().dilattn_status_string(status).decode()


def last_error() -> str:
    return load().dilattn_last_error().decode()


def _check(rc: int, what: str):
    if rc != DILATTN_OK:
        raise DilattnError(rc, f"{what}: {status_string(rc)} {last_error()}".strip())


def _patterns(patterns: Sequence[Tuple[int, int]]):
    n = len(patterns)
    w = (_c.c_int * max(n, 1))(*[int(p[0]) for p in patterns])
    r = (_c.c_int * max(n, 1))(*[int(p[1]) for p in patterns])
    return w, r, n


# ---------------------------------------------------------------------------
# torch-tensor convenience wrappers (marshalling only)
# ---------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _shape(q):
    if q.dim() != 4:
        raise ValueError("expected a [B, N, H, d] tensor")
    return tuple(int(x) for x in q.shape)


def _need(t, name, shape, dtypes, device=None):
    """Raise ValueError unless t is a contiguous CUDA tensor of this shape, one of
    these dtypes and (if given) on this device."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {' or '.join(map(str, dtypes))}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda or (device is not None and t.device != device):
        raise ValueError(f"{name} must be on {device if device is not None else 'a CUDA device'}")


def fwd_scratch_size(B, N, H, d, patterns) -> int:
    w, r, n = _patterns(patterns)
    return int(load().dilattn_fwd_scratch_size(B, N, H, d, w, r, n))


def bwd_workspace_size(B, N, H, d) -> int:
    return int(load().dilattn_bwd_workspace_size(B, N, H, d))


def fwd(q, k, v, patterns, causal: bool = True, out=None, lse=None, stream=None):
    """Merged dilated attention. bf16 tensors go to dilattn_fwd, float32 to dilattn_fwd_f32.

    Returns (out [B, N, H, d] in q's dtype, lse [B, H, N] float32).
    """
    torch = _torch()
    B, N, H, d = _shape(q)
    _need(q, "q", (B, N, H, d), (torch.bfloat16, torch.float32))
    for name, t in (("k", k), ("v", v)):
        _need(t, name, (B, N, H, d), (q.dtype,), q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(out, "out", (B, N, H, d), (q.dtype,), q.device)
    _need(lse, "lse", (B, H, N), (torch.float32,), q.device)
    w, r, n = _patterns(patterns)
    s = _stream_handle(stream)
    lib = load()
    if q.dtype == torch.bfloat16:
        rc = lib.dilattn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             lse.data_ptr(), B, N, H, d, w, r, n, int(causal), s)
        _check(rc, "dilattn_fwd")
    elif q.dtype == torch.float32:
        rc = lib.dilattn_fwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), B, N, H, d, w, r, n, int(causal), s)
        _check(rc, "dilattn_fwd_f32")
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return out, lse


def fwd_train(q, k, v, patterns, causal: bool = True, out=None, lse=None, out_res=None,
              stream=None):
    """dilattn_fwd_train on bf16 tensors: (out, lse, out_res), out_res the bf16
    rounding residual of out that the backward forms its row term from."""
    torch = _torch()
    B, N, H, d = _shape(q)
    if q.dtype != torch.bfloat16:
        raise ValueError("fwd_train takes bf16 tensors (the fp32 path needs no residual)")
    _need(q, "q", (B, N, H, d), (torch.bfloat16,))
    for name, t in (("k", k), ("v", v)):
        _need(t, name, (B, N, H, d), (torch.bfloat16,), q.device)
    out = torch.empty_like(q) if out is None else out
    out_res = torch.empty_like(q) if out_res is None else out_res
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    for name, t in (("out", out), ("out_res", out_res)):
        _need(t, name, (B, N, H, d), (torch.bfloat16,), q.device)
    _need(lse, "lse", (B, H, N), (torch.float32,), q.device)
    w, r, n = _patterns(patterns)
    rc = load().dilattn_fwd_train(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                  out_res.data_ptr(), lse.data_ptr(), B, N, H, d, w, r, n,
                                  int(causal), _stream_handle(stream))
    _check(rc, "dilattn_fwd_train")
    return out, lse, out_res


def bwd(q, k, v, out, lse, dout, patterns, causal: bool = True, out_res=None, dq=None, dk=None,
        dv=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv), float32, of sum(O * dout) for the forward that produced
    out, lse (and, for bf16, out_res: use fwd_train)."""
    torch = _torch()
    B, N, H, d = _shape(q)
    _need(q, "q", (B, N, H, d), (torch.bfloat16, torch.float32))
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout)):
        _need(t, name, (B, N, H, d), (q.dtype,), q.device)
    _need(lse, "lse", (B, H, N), (torch.float32,), q.device)
    gdt = torch.float32  # the bf16 path returns fp32 gradients, the fp32 path fp32 too
    dq = torch.empty(q.shape, dtype=gdt, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=gdt, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=gdt, device=q.device) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _need(t, name, (B, N, H, d), (gdt,), q.device)
    w, r, n = _patterns(patterns)
    if q.dtype == torch.bfloat16:
        if out_res is None:
            raise ValueError("the bf16 backward takes out_res from fwd_train")
        _need(out_res, "out_res", (B, N, H, d), (torch.bfloat16,), q.device)
        if workspace is not None:
            _need(workspace, "workspace", (workspace.numel(),), (torch.uint8,), q.device)
    s = _stream_handle(stream)
    lib = load()
    if q.dtype == torch.bfloat16:
        need = int(lib.dilattn_bwd_workspace_size(B, N, H, d))
        if workspace is None:
            workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
        rc = lib.dilattn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             out_res.data_ptr(), lse.data_ptr(), dout.data_ptr(), dq.data_ptr(),
                             dk.data_ptr(), dv.data_ptr(), B, N, H, d, w, r, n, int(causal),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(), s)
        _check(rc, "dilattn_bwd")
    elif q.dtype == torch.float32:
        rc = lib.dilattn_bwd_f32(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), dout.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                 dv.data_ptr(), B, N, H, d, w, r, n, int(causal), s)
        _check(rc, "dilattn_bwd_f32")
    else:
        raise ValueError(f"unsupported dtype {q.dtype}")
    return dq, dk, dv


def selection(N: int, H: int, patterns, device="cuda", stream=None):
    """uint32-bit selection map [H, N] (returned as int32 tensor bits) from dilattn_selection."""
    torch = _torch()
    sig = torch.empty((H, N), dtype=torch.int32, device=device)
    w, r, n = _patterns(patterns)
    rc = load().dilattn_selection(sig.data_ptr(), N, H, w, r, n, _stream_handle(stream))
    _check(rc, "dilattn_selection")
    return sig


def device_error(stream=None) -> int:
    code = _c.c_int(0)
    rc = load().dilattn_device_error(_stream_handle(stream), _c.byref(code))
    _check(rc, "dilattn_device_error")
    return int(code.value)


def selftest_wait_timeout(limit_ns: int, stream=None):
    """Run the failure-path self-test; returns the device int[4] result tensor."""
    torch = _torch()
    res = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    rc = load().dilattn_selftest_wait_timeout(int(limit_ns), res.data_ptr(), _stream_handle(stream))
    _check(rc, "dilattn_selftest_wait_timeout")
    return res


def set_trace_events(begin=None, end=None):
    """Record two torch.cuda.Event objects around the next calls' tile kernel (None, None: off).

    The events must already exist on the device (record each once first)."""
    b = int(begin.cuda_event) if begin is not None else None
    e = int(end.cuda_event) if end is not None else None
    _check(load().dilattn_set_trace_events(b, e), "dilattn_set_trace_events")


NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


def fwd_noalloc(q, k, v, patterns, causal: bool = True, out=None, lse=None, stream=None):
    """dilattn_fwd_noalloc on bf16 tensors: the forward with the library's built-in
    scratch instead of a workspace, for callers that cannot allocate device memory.
    (This wrapper itself still lets torch allocate ``out``/``lse`` when they are not
    given; pass them in to allocate nothing.)"""
    torch = _torch()
    B, N, H, d = _shape(q)
    _need(q, "q", (B, N, H, d), (torch.bfloat16,))
    for name, t in (("k", k), ("v", v)):
        _need(t, name, (B, N, H, d), (torch.bfloat16,), q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    _need(out, "out", (B, N, H, d), (torch.bfloat16,), q.device)
    _need(lse, "lse", (B, H, N), (torch.float32,), q.device)
    w, r, n = _patterns(patterns)
    rc = load().dilattn_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, N, H, d, w, r, n, int(causal),
                                    _stream_handle(stream))
    _check(rc, "dilattn_fwd_noalloc")
    return out, lse


def pack_dilated(x, r: int, out=None, stream=None):
    """dilattn_pack_dilated: [B, L/r, H, d] with row m of head h = x[:, (h mod r) + m r, h]."""
    torch = _torch()
    B, L, H, d = _shape(x)
    if r < 1 or L % r != 0:
        raise ValueError(f"the block length {L} must be a multiple of r = {r}")
    _need(x, "x", (B, L, H, d), (torch.bfloat16,))
    if out is None:
        out = torch.empty((B, L // r, H, d), dtype=x.dtype, device=x.device)
    _need(out, "out", (B, L // r, H, d), (torch.bfloat16,), x.device)
    rc = load().dilattn_pack_dilated(x.data_ptr(), out.data_ptr(), B, L, H, d, int(r),
                                     _stream_handle(stream))
    _check(rc, "dilattn_pack_dilated")
    return out


def fwd_seqpar(q, k, v, patterns, rank: int, world: int, kg=None, vg=None, causal: bool = True,
               out=None, lse=None, stream=None):
    """dilattn_fwd_seqpar on this rank's block; kg / vg: per pattern the gathered
    [ranks, B, L/r, H, d] buffer or None."""
    from . import seqpar

    torch = _torch()
    B, L, H, d = _shape(q)
    _need(q, "q", (B, L, H, d), (torch.bfloat16,))
    for name, t in (("k", k), ("v", v)):
        _need(t, name, (B, L, H, d), (torch.bfloat16,), q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _need(out, "out", (B, L, H, d), (torch.bfloat16,), q.device)
    _need(lse, "lse", (B, H, L), (torch.float32,), q.device)
    # the gathered rows of every pattern whose segments span ranks
    for p in seqpar.plan(L * world, world, patterns):
        for name, bufs in (("kg", kg), ("vg", vg)):
            t = bufs[p.index] if bufs is not None and p.index < len(bufs) else None
            if p.spans:
                if t is None:
                    raise ValueError(f"{name}[{p.index}]: pattern {p.index} spans ranks and "
                                     "needs its gathered rows")
                _need(t, f"{name}[{p.index}]", (p.ranks, B, p.rank_rows, H, d),
                      (torch.bfloat16,), q.device)
    w, r, n = _patterns(patterns)
    ptr = lambda t: t.data_ptr() if t is not None else None
    kga = (_vp * max(n, 1))(*[ptr(t) for t in (kg or [None] * n)])
    vga = (_vp * max(n, 1))(*[ptr(t) for t in (vg or [None] * n)])
    rc = load().dilattn_fwd_seqpar(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr(), B, L, H, d, w, r, n, int(causal), int(rank),
                                   int(world), kga, vga, _stream_handle(stream))
    _check(rc, "dilattn_fwd_seqpar")
    return out, lse


def fwd_fp8(q8, k8, v, patterns, q_scale: float, k_scale: float, causal: bool = True, out=None,
            lse=None, stream=None):
    """dilattn_fwd_fp8: q8, k8 e4m3 codes (uint8 or float8 tensors [B, N, H, 128]) with
    per-tensor scales; v bf16. Returns (out bf16, lse)."""
    torch = _torch()
    B, N, H, d = _shape(v)
    _need(v, "v", (B, N, H, d), (torch.bfloat16,))
    codes = (torch.uint8, torch.float8_e4m3fn)
    _need(q8, "q8", (B, N, H, d), codes, v.device)
    _need(k8, "k8", (B, N, H, d), codes, v.device)
    out = torch.empty_like(v) if out is None else out
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=v.device)
    _need(out, "out", (B, N, H, d), (torch.bfloat16,), v.device)
    _need(lse, "lse", (B, H, N), (torch.float32,), v.device)
    w, r, n = _patterns(patterns)
    rc = load().dilattn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, N, H, d, w, r, n, int(causal), float(q_scale),
                                float(k_scale), _stream_handle(stream))
    _check(rc, "dilattn_fwd_fp8")
    return out, lse
