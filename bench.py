"""Benchmark: dilated attention forward + backward on the LongNet-base layer shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is the whole hot path on one batch: dilattn_fwd_train (tile kernel
with the cross-pattern merge fused into the r = 1 pattern's tiles; out and its
rounding residual) then dilattn_bwd (preprocess + tile kernel, fp32
gradients) on B=1, N=32768, H=12, d=64
bf16 inputs with patterns w = 2048..32768, r = 1, 2, 4, 6, 12, causal.
Effective FLOPs count only the nonzero pairs of the causal sparse mask: 4 d
per pair forward, 10 d backward.

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush
(a 256 MB device write, outside the step's events) and timed with CUDA
events on the launching stream; barrier + synchronize on both sides; the
max over ranks. With N > 1 every rank runs its own batch (weak scaling, no
collective on the data path). The tile kernels are also timed alone through
the library's trace hook for the roofline line. e2e repeats the step through
the public API with the step's inputs copied from pinned host memory and the
results copied back inside the timed region; copy-in, compute and copy-out of
consecutive steps overlap on three streams (two device buffer sets), as a
training loop with a prefetching data loader would run them. Clocks are
sampled through NVML every few milliseconds during the timed steps.

The JSON detail adds the other workloads the metric is quoted on: the
training step at B = 4, N = 32768 (forward + backward), the length sweep
N = 8K .. 1M (forward + backward), the wide d = 128 forward (bf16, and FP8
with e4m3 q and k), and the N = 8K step replayed back to back from a CUDA
graph.

cpu_baseline: the float64 CPU oracle on the whole LongNet-base layer, one
worker process per (batch, head) slice, one BLAS thread each, on the host's
cores, plus the one-core figures.

--impl reference times that oracle instead (rank 0 only), each step a bounded
sample of the same workload: every head, positions [0, N') with N' sized so
that the run takes a few minutes.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_long_sequence_dilated_b200 import flops  # noqa: E402
from sparse_long_sequence_dilated_b200.workloads import WORKLOADS, make_inputs  # noqa: E402

METRIC = "dilated-attn fwd/bwd effective TFLOP/s & tokens/s at N=32K–1M; % of BF16 peak"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "longnet_base_32k"
PEAK_FALLBACK = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
# device-code files each tile kernel is built from (the DRAM-traffic record of a
# kernel stays valid while these are unchanged)
KERNEL_SOURCES = {"fwd_tile_kernel": ("common.cuh", "fwd_tc.cuh"),
                  "bwd_tile_kernel": ("common.cuh", "bwd_tc.cuh")}
NAMES = ("q", "k", "v", "dout")
# kernels of the library launched per step of a family with an r = 1 pattern:
# fwd_tile_kernel, bwd_prep_kernel, bwd_tile_kernel
LAUNCHES_PER_STEP = 3


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_long_sequence_dilated_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return PEAK_FALLBACK, "fallback"


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel, {}).get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def _summarise(rows, all_rows=None):
    """rows: (sm_mhz, max_mhz, power_w, set of reasons) taken in the timed region."""
    all_rows = all_rows if all_rows is not None else rows
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(r[0] for r in rows),
            "sm_max_mhz": max(r[1] for r in all_rows),
            "reasons": sorted(set().union(*[r[3] for r in rows])),
            "samples": len(rows), "power_w_max": max(r[2] for r in all_rows)}


class NvmlClockSampler:
    """SM clock, power and throttle reasons read through NVML by a background
    thread every `interval` seconds, from start() to stop()."""

    def __init__(self, gpu_index: str, interval: float = 0.002):
        self.gpu = int(gpu_index)
        self.interval = interval
        self.rows = []
        self.source = "nvml"

    def start(self):
        import pynvml
        pynvml.nvmlInit()
        self.nv = pynvml
        self.h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.bits = {"sw_power_cap": pynvml.nvmlClocksThrottleReasonSwPowerCap,
                     "hw_slowdown": pynvml.nvmlClocksThrottleReasonHwSlowdown,
                     "hw_thermal_slowdown": pynvml.nvmlClocksThrottleReasonHwThermalSlowdown,
                     "sw_thermal_slowdown": pynvml.nvmlClocksThrottleReasonSwThermalSlowdown}
        self.stop_ev = threading.Event()
        self.sample()  # one sample before the thread starts, so even a short region has one
        self.th = threading.Thread(target=self._loop, daemon=True)
        self.th.start()

    def sample(self):
        nv, h = self.nv, self.h
        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        self.rows.append((sm, self.max_mhz, pw, {n for n, b in self.bits.items() if rs & b}))

    def _loop(self):
        while not self.stop_ev.is_set():
            self.sample()
            time.sleep(self.interval)

    def stop(self):
        self.stop_ev.set()
        self.th.join(timeout=5)
        self.sample()
        self.nv.nvmlShutdown()
        rec = _summarise(self.rows)
        rec["source"] = "nvml, every 2 ms"
        return rec


class ClockSampler:
    """nvidia-smi -lms 50 in the background; only samples taken after start() count."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.path = tempfile.mktemp(prefix="dilattn_clocks_", suffix=".csv")
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            self.fh.close()
            os.unlink(self.path)
            return
        # nvidia-smi takes a moment to start: let its first sample land, and
        # keep only the samples taken after this point (the timed region)
        self.skip = 0
        t_end = time.time() + 3.0
        while time.time() < t_end:
            self.fh.flush()
            with open(self.path) as f:
                n = sum(1 for line in f if line.count(",") >= 8)
            if n > 0:
                self.skip = n
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for i, line in enumerate(f):
                if i < self.skip:
                    continue
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]),
                                 {REASONS[j] for j, v in enumerate(parts[5:9]) if v == "Active"}))
                except ValueError:
                    continue
        os.unlink(self.path)
        loaded = [r for r in rows if r[2] > 250.0] or rows
        rec = _summarise(loaded, rows)
        rec["source"] = "nvidia-smi, every 50 ms"
        return rec


def physical_gpu(local_rank: int) -> str:
    """The GPU this rank drives, as nvidia-smi and NVML name it: entry local_rank of
    CUDA_VISIBLE_DEVICES when that lists the node's GPUs, else the local rank."""
    vis = [x.strip() for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    return vis[local_rank] if local_rank < len(vis) else str(local_rank)


def make_clock_sampler(gpu_index: str):
    try:
        import pynvml
        pynvml.nvmlInit()
        pynvml.nvmlShutdown()
        return NvmlClockSampler(gpu_index)
    except Exception:
        return ClockSampler(gpu_index)


# ---------------------------------------------------------------------------
# CPU oracle legs: one worker process per (batch, head) slice
# ---------------------------------------------------------------------------
def usable_cpus() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_task(args):
    """Worker: the oracle forward (+ backward) of one slice; returns compute seconds."""
    q, k, v, do, h, patterns, causal = args
    import oracle
    t0 = time.perf_counter()
    out, lse = oracle.fwd_head(q, k, v, h, patterns, causal)
    if do is not None:
        oracle.bwd_head(q, k, v, do, h, patterns, causal, out, lse)
    return time.perf_counter() - t0


def _noop(_):
    return 0


class OraclePool:
    """Spawn-started workers with one BLAS thread each (never forked: the parent
    may hold a CUDA context)."""

    def __init__(self, nproc: int):
        keys = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
        old = {k_: os.environ.get(k_) for k_ in keys}
        for k_ in keys:
            os.environ[k_] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(nproc)
        finally:
            for k_, v_ in old.items():
                if v_ is None:
                    os.environ.pop(k_, None)
                else:
                    os.environ[k_] = v_
        self.nproc = nproc
        self.pool.map(_noop, range(nproc))  # workers started and warm before any timing
        self.pool.map(_oracle_task, [_tiny_task()] * nproc)  # oracle and numpy imported

    def run(self, wl, n_prefix: int, with_bwd: bool, seed: int = 0):
        """Oracle over every (batch, head) slice of positions [0, n_prefix).

        Returns (wall seconds, sum of per-slice compute seconds, effective FLOPs)."""
        names = NAMES if with_bwd else NAMES[:3]
        inp = make_inputs(wl.B, n_prefix, wl.H, wl.d, seed, wl.dtype, names)
        tasks = [(inp["q"][b, :, h], inp["k"][b, :, h], inp["v"][b, :, h],
                  inp["dout"][b, :, h] if with_bwd else None, h,
                  tuple(map(tuple, wl.patterns)), wl.causal)
                 for b in range(wl.B) for h in range(wl.H)]
        t0 = time.perf_counter()
        secs = self.pool.map(_oracle_task, tasks, chunksize=1)
        wall = time.perf_counter() - t0
        work = flops.fwd_flops(wl.B, n_prefix, wl.H, wl.d, wl.patterns, wl.causal)
        if with_bwd:
            work += flops.bwd_flops(wl.B, n_prefix, wl.H, wl.d, wl.patterns, wl.causal)
        return wall, sum(secs), work

    def close(self):
        self.pool.close()
        self.pool.join()


def _tiny_task():
    import numpy as np
    z = np.zeros((4, 8))
    return (z, z, z, z, 0, ((4, 1),), True)


def affinity_note() -> str:
    try:
        return ",".join(str(c) for c in sorted(os.sched_getaffinity(0)))
    except AttributeError:
        return "n/a"


def cpu_baseline(wl):
    """The oracle on the whole workload over its (batch, head) slices, one process per
    core, plus one-core figures (a slice's own compute time, and the tiny fp32 case)."""
    import threadpoolctl

    import oracle
    nslices = wl.B * wl.H
    nproc = max(1, min(nslices, usable_cpus()))
    pool = OraclePool(nproc)
    try:
        wall, cpu_s, work = pool.run(wl, wl.N, wl.backward, wl.seed)
    finally:
        pool.close()
    tiny = WORKLOADS["tiny_f32"]
    ti = make_inputs(tiny.B, tiny.N, tiny.H, tiny.d, tiny.seed, tiny.dtype)
    with threadpoolctl.threadpool_limits(1):
        t0 = time.perf_counter()
        oracle.fwd(ti["q"], ti["k"], ti["v"], tiny.patterns, tiny.causal)
        t_tiny = time.perf_counter() - t0
    tiny_work = flops.fwd_flops(tiny.B, tiny.N, tiny.H, tiny.d, tiny.patterns, tiny.causal)
    what = "fwd+bwd" if wl.backward else "fwd"
    return {"value": work / wall / 1e12, "unit": UNIT, "cores": nproc, "kind": "oracle",
            "sample": f"float64 oracle {what} of all {nslices} (batch, head) slices of {wl.name} "
                      f"(the whole workload), one spawn-started process per slice, {nproc} at "
                      f"a time, one BLAS thread each: {work:.3e} effective FLOP in {wall:.2f} s",
            "os_cpu_count": os.cpu_count(), "affinity": affinity_note(),
            "one_core": {"per_slice_tflops": work / cpu_s / 1e12,
                         "note": f"{wl.name} {what}: the slices' own compute seconds, each on one "
                                 f"core ({cpu_s:.2f} s in all)",
                         "tiny_f32_fwd_tflops": tiny_work / t_tiny / 1e12,
                         "tiny_f32_fwd_s": t_tiny}}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    nproc = max(1, min(wl.B * wl.H, usable_cpus()))
    pool = OraclePool(nproc)
    try:
        # size each step so that warm-up + timed steps take about --reference-seconds
        budget_s = args.reference_seconds / max(1, args.steps + args.warmup)
        cal_n = min(wl.N, 4096)
        wall, _, _ = pool.run(wl, cal_n, wl.backward, wl.seed)
        n_prefix = int(min(wl.N, max(2048, cal_n * budget_s / max(wall, 1e-3))))
        n_prefix = min(wl.N, max(2048, (n_prefix // 2048) * 2048))
        for _ in range(args.warmup):
            pool.run(wl, n_prefix, wl.backward, wl.seed)
        tot_t, tot_w = 0.0, 0
        for _ in range(args.steps):
            wall, _, w = pool.run(wl, n_prefix, wl.backward, wl.seed)
            tot_t += wall
            tot_w += w
    finally:
        pool.close()
    value = tot_w / tot_t / 1e12
    what = "fwd+bwd" if wl.backward else "fwd"
    sample = (f"float64 oracle {what} of every (batch, head) slice, positions [0, {n_prefix}) of "
              f"{wl.name} (same patterns), one spawn-started process per slice on {nproc} cores")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "N": wl.N, "H": wl.H, "d": wl.d,
                       "patterns": [list(p) for p in wl.patterns], "causal": wl.causal},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nproc, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# multi-rank host logic (one process per GPU; also run with gloo on CPU in tests)
# ---------------------------------------------------------------------------
def rank_seed(base_seed: int, rank: int) -> int:
    """Every rank draws its own batch: the workload's seed plus the rank."""
    return base_seed + rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of the ranks' values of x (a time): the job ends with its slowest rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(world: int, work_per_rank: float, ms: float, calls: int = 1) -> float:
    """Whole-job throughput: all ranks' effective FLOPs over the max-over-ranks time."""
    return world * work_per_rank * calls / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# GPU detail: the other workloads of the metric
# ---------------------------------------------------------------------------
SWEEP = ("sweep_8192", "sweep_32768", "sweep_131072", "sweep_262144", "sweep_1048576")
TRAIN = "train_b4_32k"                                      # B = 4 training step, fwd + bwd
WIDE = "wide_128k"                                          # d = 128, forward


def extra_counts(B, N, H, d, pats, causal, fwd_ms: float, bwd_ms, hbm_gbs: float,
                 out_res: bool) -> dict:
    """The forward's algorithmic HBM bytes and rate (against the measured copy
    bandwidth), and the backward's rate under the 8 d count without the
    recomputed S (labelled; the headline counts 10 d)."""
    fb = flops.fwd_bytes(B, N, H, d, pats, out_res)
    gbs = fb / (fwd_ms * 1e-3) / 1e9
    ent = {"fwd_algorithmic_bytes": fb, "fwd_hbm_gbs": gbs, "fwd_frac_of_hbm": gbs / hbm_gbs}
    if bwd_ms is not None:
        b8 = flops.bwd_flops_no_recompute(B, N, H, d, pats, causal)
        ent["bwd_tflops_8d_no_recompute"] = b8 / (bwd_ms * 1e-3) / 1e12
    return ent


def hbm_peak() -> float:
    return float(load_peaks()[0].get("hbm_gbs", PEAK_FALLBACK["hbm_gbs"]))


def time_workload(dilattn, dev, name: str, flush_buf, peak: float, steps: int = 20,
                  warmup: int = 5):
    """Whole-call and tile-kernel times of one workload on i.i.d. N(0, 1) bf16 inputs
    drawn on the device (the kernels' cost does not depend on the values), L2
    flushed before every call; medians of `steps` timed calls after `warmup`."""
    import torch

    wl = WORKLOADS[name]
    B, N, H, d, pats = wl.B, wl.N, wl.H, wl.d, wl.patterns
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    q, k, v, do = (torch.randn((B, N, H, d), generator=gen, device=dev, dtype=torch.float32)
                   .to(torch.bfloat16) for _ in range(4))
    with_bwd = wl.backward and d == 64
    ws_b = torch.empty(max(dilattn.bwd_workspace_size(B, N, H, d), 256), dtype=torch.uint8,
                       device=dev) if with_bwd else None
    ev = lambda: torch.cuda.Event(enable_timing=True)
    tiles = [ev() for _ in range(4)]
    for e in tiles:
        e.record()
    ftile, btile, fwhole, bwhole = [], [], [], []
    for i in range(warmup + steps):
        a, b, c = ev(), ev(), ev()
        flush_buf.fill_(1)
        a.record()
        dilattn.set_trace_events(tiles[0], tiles[1])
        if with_bwd:
            out, lse, res = dilattn.fwd_train(q, k, v, pats, wl.causal)
        else:
            out, lse = dilattn.fwd(q, k, v, pats, wl.causal)
        b.record()
        if with_bwd:
            dilattn.set_trace_events(tiles[2], tiles[3])
            dilattn.bwd(q, k, v, out, lse, do, pats, wl.causal, out_res=res, workspace=ws_b)
        c.record()
        dilattn.set_trace_events(None, None)
        torch.cuda.synchronize()
        if i >= warmup:
            ftile.append(tiles[0].elapsed_time(tiles[1]))
            fwhole.append(a.elapsed_time(b))
            if with_bwd:
                btile.append(tiles[2].elapsed_time(tiles[3]))
                bwhole.append(b.elapsed_time(c))
    fw = flops.fwd_flops(B, N, H, d, pats, wl.causal)
    fm = statistics.median(fwhole)
    ent = {"workload": name, "B": B, "N": N, "H": H, "d": d, "npat": len(pats),
           "fwd_ms": fm, "fwd_tflops": fw / fm / 1e9, "fwd_frac_of_peak": fw / fm / 1e9 / peak,
           "fwd_tokens_per_s": B * N / (fm * 1e-3),
           "fwd_tile_ms": statistics.median(ftile),
           "fwd_tile_tflops": fw / statistics.median(ftile) / 1e9}
    if with_bwd:
        bw = flops.bwd_flops(B, N, H, d, pats, wl.causal)
        bm = statistics.median(bwhole)
        ent.update({"bwd_ms": bm, "bwd_tflops": bw / bm / 1e9,
                    "bwd_frac_of_peak": bw / bm / 1e9 / peak,
                    "bwd_tokens_per_s": B * N / (bm * 1e-3),
                    "bwd_tile_ms": statistics.median(btile),
                    "bwd_tile_tflops": bw / statistics.median(btile) / 1e9,
                    "step_tflops": (fw + bw) / (fm + bm) / 1e9,
                    "step_frac_of_peak": (fw + bw) / (fm + bm) / 1e9 / peak,
                    "tokens_per_s": B * N / ((fm + bm) * 1e-3)})
    ent.update(extra_counts(B, N, H, d, pats, wl.causal, fm,
                            statistics.median(bwhole) if with_bwd else None, hbm_peak(),
                            with_bwd))
    del q, k, v, do, ws_b
    torch.cuda.empty_cache()
    return ent


def time_fp8(dilattn, dev, flush_buf, peak: float, name: str = WIDE, steps: int = 20,
             warmup: int = 5):
    """The FP8 forward (e4m3 q and k, bf16 v) of a d = 128 workload next to the bf16
    forward of the same inputs. Peak: S runs at the FP8 rate (twice bf16, the
    nominal ratio) and PV at the bf16 rate, half of the FLOPs each, so the
    kernel's ceiling is 4/3 of the bf16 peak."""
    import torch

    wl = WORKLOADS[name]
    B, N, H, d, pats = wl.B, wl.N, wl.H, wl.d, wl.patterns
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    q, k, v = (torch.randn((B, N, H, d), generator=gen, device=dev, dtype=torch.float32)
               .to(torch.bfloat16) for _ in range(3))
    q8, k8 = [], []
    scales = []
    for x, dst in ((q, q8), (k, k8)):
        sc = float(x.float().abs().max()) / 448.0
        dst.append((x.float() / sc).to(torch.float8_e4m3fn))
        scales.append(sc)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    t8, tb = [], []
    for i in range(warmup + steps):
        for fn, acc in ((lambda: dilattn.fwd_fp8(q8[0], k8[0], v, pats, scales[0], scales[1],
                                                   wl.causal), t8),
                        (lambda: dilattn.fwd(q, k, v, pats, wl.causal), tb)):
            a, b = ev(), ev()
            flush_buf.fill_(1)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= warmup:
                acc.append(a.elapsed_time(b))
    fw = flops.fwd_flops(B, N, H, d, pats, wl.causal)
    m8, mb = statistics.median(t8), statistics.median(tb)
    peak8 = peak * 4.0 / 3.0
    del q, k, v, q8, k8
    torch.cuda.empty_cache()
    return {"workload": name, "fp8_fwd_ms": m8, "fp8_fwd_tflops": fw / m8 / 1e9,
            "fp8_peak_tflops": peak8, "fp8_frac_of_peak": fw / m8 / 1e9 / peak8,
            "peak_note": "S at the FP8 rate (2x bf16, nominal ratio), PV at bf16: 4/3 of bf16",
            "bf16_fwd_ms": mb, "bf16_fwd_tflops": fw / mb / 1e9, "speedup": mb / m8}


def graph_step(dilattn, dev, name: str = "sweep_8192", replays: int = 50):
    """The N = 8192 step captured once in a CUDA graph and replayed back to back,
    without L2 flushes: the launch-bound regime. The training step
    (dilattn_fwd_train + dilattn_bwd; the forward's pooled scratch becomes an
    allocation node of the graph) when the capture takes it, else the forward
    alone through dilattn_fwd_noalloc (scratch in the library's fixed array)."""
    try:
        return _graph_step(dilattn, dev, name, replays, train=True)
    except Exception as e:  # noqa: BLE001 (reported in the JSON detail)
        import torch
        torch.cuda.synchronize()
        ent = _graph_step(dilattn, dev, name, replays, train=False)
        ent["training_step_capture"] = f"not taken: {type(e).__name__}: {e}"[:300]
        return ent


def _graph_step(dilattn, dev, name, replays, train):
    import torch

    wl = WORKLOADS[name]
    B, N, H, d, pats = wl.B, wl.N, wl.H, wl.d, wl.patterns
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    q, k, v, do = (torch.randn((B, N, H, d), generator=gen, device=dev, dtype=torch.float32)
                   .to(torch.bfloat16) for _ in range(4))
    out, res = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((B, N, H, d), dtype=torch.float32, device=dev) for _ in range(3))
    ws_b = torch.empty(dilattn.bwd_workspace_size(B, N, H, d), dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)

    def body():
        if train:
            dilattn.fwd_train(q, k, v, pats, wl.causal, out=out, lse=lse, out_res=res, stream=s)
            dilattn.bwd(q, k, v, out, lse, do, pats, wl.causal, out_res=res, dq=dq, dk=dk, dv=dv,
                        workspace=ws_b, stream=s)
        else:
            dilattn.fwd_noalloc(q, k, v, pats, wl.causal, out=out, lse=lse, stream=s)

    with torch.cuda.stream(s):
        for _ in range(3):  # the first call looks up the fixed array, outside the capture
            body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        body()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(replays):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / replays
    work = flops.fwd_flops(B, N, H, d, pats, wl.causal)
    if train:
        work += flops.bwd_flops(B, N, H, d, pats, wl.causal)
    del g
    return {"workload": name, "replays": replays,
            "step": "dilattn_fwd_train + dilattn_bwd" if train else "dilattn_fwd_noalloc",
            "ms_per_step": ms, "tflops": work / ms / 1e9, "tokens_per_s": B * N / (ms * 1e-3),
            "l2": "not flushed (back-to-back replays)"}


def e2e_pipelined(dilattn, host, dev, pats, causal, ws_b, K: int, W: int):
    """K training steps through the public API, each with its own copies.

    Step i copies q, k, v, dout in from pinned host memory, runs dilattn.fwd_train
    and dilattn.bwd, and copies out, lse, dq, dk, dv back to pinned host memory.
    Copy-in, compute and copy-out run on three streams with two device buffer
    sets, so step i + 1's inputs cross PCIe while step i computes and step
    i - 1's results cross back (PCIe is full duplex); a buffer set is reused
    only once the step that last used it is done with it. Returns the device
    time of the K steps (first copy-in to last copy-out) and the bytes each
    step moves in and out."""
    import torch
    shp, bf = host["q"].shape, host["q"].dtype
    B, N, H, _ = shp
    s_in, s_c, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    din = [{n: torch.empty(shp, dtype=bf, device=dev) for n in NAMES} for _ in range(2)]
    dres = [{"out": torch.empty(shp, dtype=bf, device=dev)} for _ in range(2)]
    for r_ in dres:
        r_["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        for n in ("dq", "dk", "dv"):
            r_[n] = torch.empty(shp, dtype=torch.float32, device=dev)
    res = [torch.empty(shp, dtype=bf, device=dev) for _ in range(2)]  # stays on the device
    hres = [{n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in r_.items()}
            for r_ in dres]
    h2d = sum(host[n].numel() * host[n].element_size() for n in NAMES)
    d2h = sum(t.numel() * t.element_size() for t in hres[0].values())
    in_free, res_free = [None, None], [None, None]
    torch.cuda.synchronize()

    def issue(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if in_free[b] is not None:
                s_in.wait_event(in_free[b])  # compute of step i - 2 has read these inputs
            for n in NAMES:
                din[b][n].copy_(host[n], non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(e_in)
            if res_free[b] is not None:
                s_c.wait_event(res_free[b])  # step i - 2's results have left the device
            x, r_ = din[b], dres[b]
            dilattn.fwd_train(x["q"], x["k"], x["v"], pats, causal, out=r_["out"],
                              lse=r_["lse"], out_res=res[b])
            dilattn.bwd(x["q"], x["k"], x["v"], r_["out"], r_["lse"], x["dout"], pats, causal,
                        out_res=res[b], dq=r_["dq"], dk=r_["dk"], dv=r_["dv"], workspace=ws_b)
            e_c = torch.cuda.Event()
            e_c.record(s_c)
            in_free[b] = e_c
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_c)
            for n, t in dres[b].items():
                hres[b][n].copy_(t, non_blocking=True)
            e_o = torch.cuda.Event()
            e_o.record(s_out)
            res_free[b] = e_o

    for i in range(max(1, min(W, 3))):
        issue(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(K):
        issue(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), h2d, d2h


def run_ours(args, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sparse_long_sequence_dilated_b200 import dilattn

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    wl = WORKLOADS[args.workload]
    B, N, H, d = wl.B, wl.N, wl.H, wl.d
    pats = wl.patterns
    causal = wl.causal

    inp = make_inputs(B, N, H, d, rank_seed(wl.seed, rank), wl.dtype, NAMES)
    host = {n: torch.from_numpy(np.ascontiguousarray(inp[n + "_bits"]).view(np.int16))
            .view(torch.bfloat16).pin_memory() for n in NAMES}
    q, k, v, do = (host[n].to(dev) for n in NAMES)
    out, res = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty((B, N, H, d), dtype=torch.float32, device=dev) for _ in range(3))
    ws_b = torch.empty(dilattn.bwd_workspace_size(B, N, H, d), dtype=torch.uint8, device=dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(trace=None, fwd_ev=None):
        if trace is not None:
            dilattn.set_trace_events(trace[0], trace[1])
        dilattn.fwd_train(q, k, v, pats, causal, out=out, lse=lse, out_res=res)
        if fwd_ev is not None:
            fwd_ev.record(stream)
        if trace is not None:
            dilattn.set_trace_events(trace[2], trace[3])
        dilattn.bwd(q, k, v, out, lse, do, pats, causal, out_res=res, dq=dq, dk=dk, dv=dv,
                    workspace=ws_b)
        if trace is not None:
            dilattn.set_trace_events(None, None)

    K, W = args.steps, args.warmup
    ev = lambda: torch.cuda.Event(enable_timing=True)
    step_ev = [(ev(), ev(), ev()) for _ in range(K)]   # start, forward done, step done
    tile_ev = [tuple(ev() for _ in range(4)) for _ in range(K)]
    for tev in tile_ev:  # create the underlying CUDA events before handing them to the library
        for e in tev:
            e.record(stream)

    for _ in range(W):
        flush_buf.fill_(1)
        step()
    torch.cuda.synchronize()
    if dilattn.device_error() != 0:
        raise RuntimeError("a kernel reported a device-side error during warm-up")

    sampler = make_clock_sampler(physical_gpu(local_rank))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(K):
        flush_buf.fill_(1)
        step_ev[i][0].record(stream)
        step(tile_ev[i], step_ev[i][1])
        step_ev[i][2].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    step_ms = sum(a.elapsed_time(c) for a, _, c in step_ev)
    fwd_ms = sum(a.elapsed_time(b) for a, b, _ in step_ev) / K
    bwd_ms = sum(b.elapsed_time(c) for _, b, c in step_ev) / K
    fwd_tile_ms = sum(t[0].elapsed_time(t[1]) for t in tile_ev) / K
    bwd_tile_ms = sum(t[2].elapsed_time(t[3]) for t in tile_ev) / K
    step_ms = max_over_ranks(step_ms, world, dev)
    ms_per_step = step_ms / K

    # e2e through the public API: every step copies its inputs in from pinned
    # host memory and its results back out, inside the timed region
    e2e_total_ms, h2d, d2h = e2e_pipelined(dilattn, host, dev, pats, causal, ws_b, K, W)
    if world > 1:
        dist.barrier()
    e2e_ms = max_over_ranks(e2e_total_ms, world, dev)
    if dilattn.device_error() != 0:
        raise RuntimeError("a kernel reported a device-side error")

    fwd_work = flops.fwd_flops(B, N, H, d, pats, causal)
    bwd_work = flops.bwd_flops(B, N, H, d, pats, causal)
    step_work = fwd_work + bwd_work
    value = job_tflops(world, step_work, ms_per_step)
    e2e_value = job_tflops(world, step_work, e2e_ms, K)
    peaks, peak_src = load_peaks()
    peak = float(peaks["bf16_tflops"])
    fwd_tile_tf = fwd_work / (fwd_tile_ms * 1e-3) / 1e12
    bwd_tile_tf = bwd_work / (bwd_tile_ms * 1e-3) / 1e12
    if bwd_tile_ms >= fwd_tile_ms:
        dom, dom_tf = "bwd_tile_kernel", bwd_tile_tf
    else:
        dom, dom_tf = "fwd_tile_kernel", fwd_tile_tf
    fwd_tf = fwd_work / (fwd_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "N": N, "H": H, "d": d,
                   "patterns": [list(p) for p in pats], "causal": causal,
                   "step": "dilattn_fwd_train + dilattn_bwd (fp32 gradients)",
                   "l2": "flushed between timed steps (256 MB device write outside the events)",
                   "parallelism": f"independent batch per GPU x{world}"},
        "tokens_per_s": world * B * N / (ms_per_step * 1e-3),
        "frac_of_bf16_peak": value / world / peak,
        "detail": {
            "fwd_effective_flop": fwd_work, "bwd_effective_flop": bwd_work,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "fwd_tflops": fwd_tf, "bwd_tflops": bwd_work / (bwd_ms * 1e-3) / 1e12,
            "fwd_tokens_per_s": B * N / (fwd_ms * 1e-3),
            "bwd_tokens_per_s": B * N / (bwd_ms * 1e-3),
            "fwd_tile_ms": fwd_tile_ms, "bwd_tile_ms": bwd_tile_ms,
            "fwd_tile_tflops": fwd_tile_tf, "bwd_tile_tflops": bwd_tile_tf,
            "peak_source": peak_src,
            **extra_counts(B, N, H, d, pats, causal, fwd_ms, bwd_ms, hbm_peak(), True),
        },
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": dom_tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": dom_tf / peak,
                     "peak_note": f"bf16_tflops (burst) of {peak_src} peaks",
                     "traffic": load_traffic(dom, wl.name)},
        "roofline_fwd": {"bound": "tensor", "kernel": "dilattn_fwd_train (whole call)",
                         "achieved": fwd_tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": fwd_tf / peak,
                         "traffic": load_traffic("fwd_tile_kernel", wl.name)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                "overlap": "copy-in, compute, copy-out of consecutive steps on three streams"},
        "gpu_launches": LAUNCHES_PER_STEP * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_sweep:
        det = line["detail"]
        det["training_step_b4"] = time_workload(dilattn, dev, TRAIN, flush_buf, peak)
        det["length_sweep"] = [time_workload(dilattn, dev, n, flush_buf, peak) for n in SWEEP]
        det["wide_d128"] = time_workload(dilattn, dev, WIDE, flush_buf, peak)
        det["graph_8k"] = graph_step(dilattn, dev)
        det["fp8_wide_d128"] = time_fp8(dilattn, dev, flush_buf, peak)
        if dilattn.device_error() != 0:
            raise RuntimeError("a kernel reported a device-side error in the detail runs")
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-seconds", type=float, default=180.0,
                    help="--impl reference: host time the warm-up and timed steps aim for")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the detail runs (B = 4 step, length sweep, wide d = 128, graph)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        print(f"note: WORLD_SIZE={world} differs from --gpus {args.gpus}", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
