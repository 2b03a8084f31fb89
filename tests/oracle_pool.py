"""The float64 oracle over (batch, head) slices in parallel worker processes.

Full-size parity tests compare every output element of the CUDA path with the
oracle. The oracle is plain float64 NumPy and treats every (batch, head)
slice on its own (``oracle.fwd_head`` / ``oracle.bwd_head``), so one slice is
one task here. Workers are started with the ``spawn`` method: a process that
holds a CUDA context must never be forked.

Inputs and GPU results are placed once in named shared-memory blocks (bf16
tensors as their uint16 bit patterns, float32 tensors as they are). Each
worker reads its slice, runs the oracle, compares and returns only error
sums, which ``check`` turns into the same bounds as ``gpu_util.check_close``:
max-abs <= 2e-2 and relative L2 <= 5e-3 over the whole tensor for bf16,
max-abs <= 1e-4 for float32, and for lse the -inf pattern exactly and
max-abs on the finite entries.

Test infrastructure only; the product never imports it.
"""
from __future__ import annotations

import contextlib
import math
import multiprocessing as mp
import os
from multiprocessing import shared_memory
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

BF16_ATOL = 2e-2
BF16_REL_L2 = 5e-3
F32_ATOL = 1e-4


class _Shared:
    """One numpy array copied into a named shared-memory block."""

    def __init__(self, arr: np.ndarray):
        arr = np.ascontiguousarray(arr)
        self.shm = shared_memory.SharedMemory(create=True, size=max(arr.nbytes, 1))
        view = np.ndarray(arr.shape, arr.dtype, buffer=self.shm.buf)
        view[...] = arr
        del view
        self.spec = (self.shm.name, arr.shape, arr.dtype.str)

    def close(self):
        self.shm.close()
        self.shm.unlink()


def _attach(spec):
    name, shape, dt = spec
    shm = shared_memory.SharedMemory(name=name)
    return shm, np.ndarray(shape, np.dtype(dt), buffer=shm.buf)


def as_f64(a: np.ndarray) -> np.ndarray:
    """float64 values of a bf16 bit-pattern (uint16) or float array."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def _err(got: np.ndarray, want: np.ndarray):
    """(max-abs, sum err^2, sum want^2, non-finite count, (row, col, got, want) at the max)."""
    fin = np.isfinite(got)
    e = np.abs(np.where(fin, got, 0.0) - want)
    if not e.size:
        return 0.0, 0.0, float((want * want).sum()), int((~fin).sum()), None
    i = int(np.argmax(e))
    at = (i // e.shape[-1], i % e.shape[-1], float(got.ravel()[i]), float(want.ravel()[i]))
    return float(e.max()), float((e * e).sum()), float((want * want).sum()), int((~fin).sum()), at


def _lse_err(got: np.ndarray, want: np.ndarray):
    fin = np.isfinite(want)
    pattern = int((np.isfinite(got) != fin).sum()) + int((got[~fin] != -np.inf).sum())
    both = fin & np.isfinite(got)
    e = float(np.abs(got[both] - want[both]).max()) if both.any() else 0.0
    return pattern, e


def _task(args):
    kind, specs, b, h, patterns, causal = args
    held = {}
    try:
        arrs = {}
        for name, spec in specs.items():
            held[name], arrs[name] = _attach(spec)
        sl = lambda name: as_f64(arrs[name][b, :, h, :])
        q, k, v = sl("q"), sl("k"), sl("v")
        import oracle  # noqa: WPS433 (imported in the worker, after the thread limits are set)
        want_o, want_l = oracle.fwd_head(q, k, v, h, patterns, causal)
        want = {"out": want_o}
        if kind == "bwd":
            gq, gk, gv = oracle.bwd_head(q, k, v, sl("dout"), h, patterns, causal, want_o, want_l)
            want.update(dq=gq, dk=gk, dv=gv)
        stats = {}
        for name in specs:
            if not name.startswith("got:"):
                continue
            what = name[4:].split("@")[0]
            if what == "lse":
                stats[name] = _lse_err(as_f64(arrs[name][b, h]), want_l)
            else:
                stats[name] = _err(as_f64(arrs[name][b, :, h, :]), want[what])
        return b, h, {k: (v + ((b, h),) if len(v) == 5 else v) for k, v in stats.items()}
    finally:
        for shm in held.values():
            shm.close()


def usable_cpus() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _mem_cap(N: int, d: int, kind: str) -> int:
    """Workers that fit in 60% of the available memory (a float64 slice costs ~N*d*8)."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        return 1 << 30
    per = N * d * 8 * (14 if kind == "bwd" else 8) + 4 * 2731 * 2731 * 8
    return max(1, int(avail * 0.6 // per))


@contextlib.contextmanager
def _blas_threads(n: int):
    keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    old = {k: os.environ.get(k) for k in keys}
    for k in keys:
        os.environ[k] = str(n)
    try:
        yield
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v


def run(kind: str, inputs: Dict[str, np.ndarray], got: Dict[str, np.ndarray],
        patterns: Sequence[Tuple[int, int]], causal: bool,
        pairs: Optional[List[Tuple[int, int]]] = None):
    """Oracle vs GPU on the given (batch, head) pairs (default: all).

    kind: "fwd" or "bwd". inputs: q, k, v (and dout for "bwd") [B, N, H, d].
    got: GPU results keyed "out", "lse", "dq", "dk", "dv", optionally with a
    "@variant" suffix; [B, N, H, d] except lse [B, H, N]. Returns
    {name: [per-pair stats]}.
    """
    B, N, H, d = inputs["q"].shape
    pairs = pairs if pairs is not None else [(b, h) for b in range(B) for h in range(H)]
    shared = {}
    try:
        for name, arr in inputs.items():
            shared[name] = _Shared(arr)
        for name, arr in got.items():
            shared["got:" + name] = _Shared(arr)
        specs = {name: s.spec for name, s in shared.items()}
        nproc = max(1, min(len(pairs), usable_cpus(), _mem_cap(N, d, kind)))
        threads = max(1, usable_cpus() // nproc)
        ctx = mp.get_context("spawn")
        with _blas_threads(threads):
            pool = ctx.Pool(nproc)
        try:
            res = pool.map(_task, [(kind, specs, b, h, tuple(map(tuple, patterns)), causal)
                                   for (b, h) in pairs], chunksize=1)
        finally:
            pool.close()
            pool.join()
    finally:
        for s in shared.values():
            s.close()
    out: Dict[str, list] = {}
    for _, _, stats in res:
        for name, st in stats.items():
            out.setdefault(name[4:], []).append(st)
    return out


def check(stats: Dict[str, list], dtype: str, lse_atol: float, what: str = ""):
    """Assert the bounds over all pairs; returns {name: (max_abs, rel_l2)} for reporting."""
    summary = {}
    for name, rows in sorted(stats.items()):
        label = f"{what} {name}".strip()
        if name.split("@")[0] == "lse":
            pattern = sum(r[0] for r in rows)
            e = max(r[1] for r in rows)
            assert pattern == 0, f"{label}: -inf pattern differs at {pattern} rows"
            assert e <= lse_atol, f"{label}: max_abs={e:.3e}"
            summary[name] = (e, None)
            continue
        nonfinite = sum(r[3] for r in rows)
        assert nonfinite == 0, f"{label}: {nonfinite} non-finite values"
        worst = max(rows, key=lambda r: r[0])
        max_abs = worst[0]
        err2 = sum(r[1] for r in rows)
        want2 = sum(r[2] for r in rows)
        rel = math.sqrt(err2 / want2) if want2 > 0 else math.sqrt(err2)
        where = ""
        if len(worst) > 5 and worst[4] is not None:
            (b, h), (n, c, g, w) = worst[5], worst[4]
            where = f" at (b={b}, n={n}, h={h}, c={c}): got {g:.6f}, want {w:.6f}"
        if dtype == "bf16":
            assert max_abs <= BF16_ATOL and rel <= BF16_REL_L2, \
                f"{label}: max_abs={max_abs:.3e} rel_l2={rel:.3e}{where}"
        else:
            assert max_abs <= F32_ATOL, f"{label}: max_abs={max_abs:.3e}{where}"
        summary[name] = (max_abs, rel)
    return summary


class _Bf16Array:
    """Read-only float64 view of a bf16 bit-pattern array (converted per index)."""

    def __init__(self, bits: np.ndarray):
        self.bits = bits
        self.shape = bits.shape

    def __getitem__(self, idx):
        return as_f64(self.bits[idx])


def _row_task(args):
    specs, kind, row, patterns, causal = args
    held = {}
    try:
        arrs = {}
        for name, spec in specs.items():
            held[name], a = _attach(spec)
            arrs[name] = _Bf16Array(a)
        import oracle  # noqa: WPS433
        qrows, krows = ([row], []) if kind == "q" else ([], [row])
        gq, gk, gv = oracle.bwd_rows(arrs["q"], arrs["k"], arrs["v"], arrs["dout"], patterns,
                                     qrows, krows, causal)
        return (gq[0],) if kind == "q" else (gk[0], gv[0])
    finally:
        for shm in held.values():
            shm.close()


def bwd_rows(inputs: Dict[str, np.ndarray], qrows, krows, patterns, causal: bool):
    """oracle.bwd_rows on bf16 bit-pattern inputs, one row per worker task.

    Returns (dq [len(qrows), d], dk [len(krows), d], dv [len(krows), d])."""
    shared = {n: _Shared(a) for n, a in inputs.items()}
    try:
        specs = {n: s.spec for n, s in shared.items()}
        pats = tuple(map(tuple, patterns))
        tasks = [(specs, "q", r, pats, causal) for r in qrows]
        tasks += [(specs, "k", r, pats, causal) for r in krows]
        nproc = max(1, min(len(tasks), usable_cpus()))
        ctx = mp.get_context("spawn")
        with _blas_threads(1):
            pool = ctx.Pool(nproc)
        try:
            res = pool.map(_row_task, tasks, chunksize=1)
        finally:
            pool.close()
            pool.join()
    finally:
        for s in shared.values():
            s.close()
    d = inputs["q"].shape[-1]
    dq = np.array([r[0] for r in res[:len(qrows)]]).reshape(len(qrows), d)
    dk = np.array([r[0] for r in res[len(qrows):]]).reshape(len(krows), d)
    dv = np.array([r[1] for r in res[len(qrows):]]).reshape(len(krows), d)
    return dq, dk, dv
