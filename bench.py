"""Benchmark: dilated attention forward + backward on the LongNet-base layer shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is the whole hot path on one batch: dilattn_fwd (tile kernel +
merge) then dilattn_bwd (preprocess + tile kernel + convert) on B=1,
N=32768, H=12, d=64 bf16 inputs with patterns w = 2048..32768,
r = 1, 2, 4, 6, 12, causal. Effective FLOPs count only the nonzero pairs of
the causal sparse mask: 4 d per pair forward, 10 d backward.

Timing: W untimed warm-up steps; then K steps, each preceded by an L2 flush
(a 256 MB device write, outside the step's events) and timed with CUDA
events on the launching stream; barrier + synchronize on both sides; the
max over ranks. With N > 1 every rank runs its own batch (weak scaling, no
collective on the data path). The tile kernels are also timed alone through
the library's trace hook for the roofline line. e2e repeats the step through
the public API with the step's inputs copied from pinned host memory and the
results copied back inside the timed region; copy-in, compute and copy-out of
consecutive steps overlap on three streams (two device buffer sets), as a
training loop with a prefetching data loader would run them.

--impl reference times the float64 CPU oracle instead (rank 0 only), each
step a bounded sample of the same workload: the first N' positions of head 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
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
class ClockSampler:
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
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r[2] > 250.0] or rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(loaded), "power_w_max": max(r[2] for r in rows)}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(wl, n_prefix: int):
    """The oracle forward + backward on head 0 of the first n_prefix positions.

    Returns (seconds, effective FLOPs of the sample)."""
    import oracle
    inp = make_inputs(1, n_prefix, 1, wl.d, wl.seed, wl.dtype, NAMES)
    t0 = time.perf_counter()
    out, lse = oracle.fwd(inp["q"], inp["k"], inp["v"], wl.patterns, wl.causal)
    oracle.bwd(inp["q"], inp["k"], inp["v"], inp["dout"], wl.patterns, wl.causal, out=out, lse=lse)
    dt = time.perf_counter() - t0
    work = (flops.fwd_flops(1, n_prefix, 1, wl.d, wl.patterns, wl.causal)
            + flops.bwd_flops(1, n_prefix, 1, wl.d, wl.patterns, wl.causal))
    return dt, work


def cpu_baseline(wl):
    dt, work = oracle_sample(wl, wl.N)
    return {"value": work / dt / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 oracle fwd+bwd, batch 0 head 0 of {wl.name} (N={wl.N}, all "
                      f"{len(wl.patterns)} patterns): {work:.3e} effective FLOP in {dt:.2f} s"}


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    # size each step so that warm-up + timed steps take about two minutes
    budget_s = 120.0 / max(1, args.steps + args.warmup)
    cal_n = min(wl.N, 4096)
    dt, _ = oracle_sample(wl, cal_n)
    n_prefix = int(min(wl.N, max(2048, cal_n * budget_s / max(dt, 1e-3))))
    n_prefix = max(2048, (n_prefix // 2048) * 2048)
    for _ in range(args.warmup):
        oracle_sample(wl, n_prefix)
    tot_t, tot_w = 0.0, 0
    for _ in range(args.steps):
        dt, w = oracle_sample(wl, n_prefix)
        tot_t += dt
        tot_w += w
    value = tot_w / tot_t / 1e12
    sample = (f"float64 oracle fwd+bwd on head 0, positions [0, {n_prefix}) of {wl.name} "
              f"(same patterns), one sample per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "N": wl.N, "H": wl.H, "d": wl.d,
                       "patterns": [list(p) for p in wl.patterns], "causal": wl.causal},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU leg
# ---------------------------------------------------------------------------
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


SWEEP = ("sweep_8192", "sweep_131072", "sweep_1048576")  # the length sweep, fwd + bwd
WIDE = "wide_128k"                                         # d = 128, forward


def sweep_detail(dilattn, dev, steps: int = 3, warmup: int = 2):
    """Tile-kernel and whole-call times for the length sweep (N = 8K, 128K, 1M; fwd + bwd)
    and the wide d = 128 forward, each on i.i.d. N(0, 1) bf16 inputs drawn on the device
    (the kernels' cost does not depend on the values), L2 flushed before every call."""
    import torch

    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    res = []
    for name in SWEEP + (WIDE,):
        wl = WORKLOADS[name]
        B, N, H, d, pats = wl.B, wl.N, wl.H, wl.d, wl.patterns
        t = [torch.randn((B, N, H, d), generator=gen, device=dev, dtype=torch.float32)
             .to(torch.bfloat16) for _ in range(4)]
        q, k, v, do = t
        ws_f = torch.empty(dilattn.fwd_workspace_size(B, N, H, d, pats), dtype=torch.uint8,
                           device=dev)
        with_bwd = wl.backward and d == 64
        tiles = [ev() for _ in range(4)]
        for e in tiles:
            e.record()
        ftile, btile, fwhole, bwhole = [], [], [], []
        for i in range(warmup + steps):
            a, b, c = ev(), ev(), ev()
            flush_buf.fill_(1)
            a.record()
            dilattn.set_trace_events(tiles[0], tiles[1])
            out, lse = dilattn.fwd(q, k, v, pats, wl.causal, workspace=ws_f)
            b.record()
            if with_bwd:
                dilattn.set_trace_events(tiles[2], tiles[3])
                dilattn.bwd(q, k, v, out, lse, do, pats, wl.causal, fwd_workspace=ws_f)
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
        ent = {"workload": name, "B": B, "N": N, "H": H, "d": d,
               "fwd_tile_ms": statistics.median(ftile), "fwd_ms": statistics.median(fwhole),
               "fwd_tile_tflops": fw / statistics.median(ftile) / 1e9,
               "fwd_tflops": fw / statistics.median(fwhole) / 1e9}
        if with_bwd:
            bw = flops.bwd_flops(B, N, H, d, pats, wl.causal)
            ent.update({"bwd_tile_ms": statistics.median(btile), "bwd_ms": statistics.median(bwhole),
                        "bwd_tile_tflops": bw / statistics.median(btile) / 1e9,
                        "step_tflops": (fw + bw) / (statistics.median(fwhole)
                                                    + statistics.median(bwhole)) / 1e9,
                        "tokens_per_s": B * N / ((statistics.median(fwhole)
                                                  + statistics.median(bwhole)) * 1e-3)})
        res.append(ent)
        del q, k, v, do, t, ws_f
        torch.cuda.empty_cache()
    if dilattn.device_error() != 0:
        raise RuntimeError("a kernel reported a device-side error in the length sweep")
    return res


def e2e_pipelined(dilattn, host, dev, pats, causal, ws_f, ws_b, K: int, W: int):
    """K training steps through the public API, each with its own copies.

    Step i copies q, k, v, dout in from pinned host memory, runs dilattn.fwd and
    dilattn.bwd, and copies out, lse, dq, dk, dv back to pinned host memory.
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
    dres = [{n: torch.empty(shp, dtype=bf, device=dev) for n in ("out", "dq", "dk", "dv")}
            for _ in range(2)]
    for r_ in dres:
        r_["lse"] = torch.empty((B, H, N), dtype=torch.float32, device=dev)
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
            dilattn.fwd(x["q"], x["k"], x["v"], pats, causal, out=r_["out"], lse=r_["lse"],
                        workspace=ws_f)
            dilattn.bwd(x["q"], x["k"], x["v"], r_["out"], r_["lse"], x["dout"], pats, causal,
                        dq=r_["dq"], dk=r_["dk"], dv=r_["dv"], workspace=ws_b, fwd_workspace=ws_f)
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
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_f = torch.empty(dilattn.fwd_workspace_size(B, N, H, d, pats), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(dilattn.bwd_workspace_size(B, N, H, d, pats), dtype=torch.uint8, device=dev)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(trace=None):
        if trace is not None:
            dilattn.set_trace_events(trace[0], trace[1])
        dilattn.fwd(q, k, v, pats, causal, out=out, lse=lse, workspace=ws_f)
        if trace is not None:
            dilattn.set_trace_events(trace[2], trace[3])
        dilattn.bwd(q, k, v, out, lse, do, pats, causal, dq=dq, dk=dk, dv=dv, workspace=ws_b,
                    fwd_workspace=ws_f)
        if trace is not None:
            dilattn.set_trace_events(None, None)

    K, W = args.steps, args.warmup
    ev = lambda: torch.cuda.Event(enable_timing=True)
    step_ev = [(ev(), ev()) for _ in range(K)]
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

    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[local_rank]
    sampler = ClockSampler(gpu_index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    for i in range(K):
        flush_buf.fill_(1)
        step_ev[i][0].record(stream)
        step(tile_ev[i])
        step_ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    step_ms = sum(a.elapsed_time(b) for a, b in step_ev)
    fwd_tile_ms = sum(t[0].elapsed_time(t[1]) for t in tile_ev) / K
    bwd_tile_ms = sum(t[2].elapsed_time(t[3]) for t in tile_ev) / K
    step_ms = max_over_ranks(step_ms, world, dev)
    ms_per_step = step_ms / K

    # e2e through the public API: every step copies its inputs in from pinned
    # host memory and its results back out, inside the timed region
    e2e_total_ms, h2d, d2h = e2e_pipelined(dilattn, host, dev, pats, causal, ws_f, ws_b, K, W)
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
        dom, dom_tf, dom_work = "bwd_tile_kernel", bwd_tile_tf, bwd_work
    else:
        dom, dom_tf, dom_work = "fwd_tile_kernel", fwd_tile_tf, fwd_work
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "B": B, "N": N, "H": H, "d": d,
                   "patterns": [list(p) for p in pats], "causal": causal,
                   "step": "dilattn_fwd + dilattn_bwd",
                   "l2": "flushed between timed steps (256 MB device write outside the events)",
                   "parallelism": f"independent batch per GPU x{world}"},
        "tokens_per_s": world * B * N / (ms_per_step * 1e-3),
        "frac_of_bf16_peak": value / world / peak,
        "detail": {
            "fwd_effective_flop": fwd_work, "bwd_effective_flop": bwd_work,
            "fwd_tile_ms": fwd_tile_ms, "bwd_tile_ms": bwd_tile_ms,
            "fwd_tile_tflops": fwd_tile_tf, "bwd_tile_tflops": bwd_tile_tf,
            "fwd_tokens_per_s": B * N / (fwd_tile_ms * 1e-3),
            "peak_source": peak_src,
        },
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": dom_tf, "peak": peak,
                     "unit": "TFLOP/s", "frac": dom_tf / peak,
                     "peak_note": f"bf16_tflops (burst) of {peak_src} peaks",
                     "traffic": load_traffic(dom, wl.name)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / K,
                "overlap": "copy-in, compute, copy-out of consecutive steps on three streams"},
        "gpu_launches": 5 * K,
        "clocks": clocks,
    }
    if world == 1 and not args.no_sweep:
        line["detail"]["length_sweep"] = sweep_detail(dilattn, dev)
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
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the length sweep (N = 8K, 128K, 1M) and the wide d = 128 forward")
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
