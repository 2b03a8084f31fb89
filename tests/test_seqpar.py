"""Host logic of the sequence-parallel forward, on the CPU.

The plan decides which patterns stay inside a rank's block and how spanning
patterns are gathered; two and four gloo ranks then run the exchange the GPU
path runs (each rank sends the rows dilattn_pack_dilated extracts, the ranks
all-gather in rank order, each keeps its segment's slice) and check the
result against the oracle's kept rows: the gathered sequence of every head
must be the segment's kept rows in order, and each rank's query rows must sit
at the tile offset the kernel is given. A second set of gloo ranks carries
the decomposition through in float64: each rank attends its block's local
patterns, attends its kept query rows of every spanning pattern to the
gathered rows (causal from the tile offset the plan gives), merges through
the log-sum-exp of the denominators, and must reproduce the oracle's merged
rows of its block. A third set runs seqpar.forward itself (its packing calls,
its all-gather and its slicing of the gathered buffers) with the two library
calls replaced by host stand-ins, batch 2, against the oracle. The kernels of
that path are checked on the GPU against the oracle (tests/test_gpu_seqpar.py)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import math

import oracle
from sparse_long_sequence_dilated_b200 import seqpar

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = {
    2: (2048, [(256, 1), (512, 2), (2048, 4), (1024, 8)]),
    4: (4096, [(512, 1), (1024, 2), (2048, 4), (4096, 8)]),
}


@pytest.fixture(autouse=True)
def _one_blas_thread_per_rank(monkeypatch):
    """The gloo ranks are processes on the same cores: one BLAS thread each
    (they inherit the environment when spawned)."""
    for name in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        monkeypatch.setenv(name, "1")


def test_plan_local_and_spanning_patterns():
    pl = seqpar.plan(32768, 4, [(2048, 1), (4096, 2), (8192, 4), (16384, 8), (32768, 16)])
    assert [p.spans for p in pl] == [False, False, False, True, True]
    assert (pl[3].ranks, pl[3].rank_rows) == (2, 1024)
    assert (pl[4].ranks, pl[4].rank_rows) == (4, 512)
    assert pl[3].segment_ranks(3) == [2, 3] and pl[4].segment_ranks(1) == [0, 1, 2, 3]
    assert pl[3].tile_offset(3) == 8 and pl[4].tile_offset(2) == 8 and pl[0].tile_offset(2) == 0
    # w larger than N: one segment over every rank
    pl = seqpar.plan(8192, 2, [(1 << 20, 2)])
    assert pl[0].spans and pl[0].ranks == 2
    # segments of 2 blocks of 3072 tile N = 4 blocks
    assert seqpar.plan(12288, 4, [(6144, 1)])[0].ranks == 2


@pytest.mark.parametrize("N,world,pats", [
    (1000, 3, [(100, 1)]),            # N not a multiple of the ranks
    (4096, 2, [(1000, 1)]),           # the block is not a multiple of w
    (4096, 2, [(4096, 3)]),           # L not a multiple of r
    (4096, 2, [(4096, 32)]),          # L / r not whole tiles
    (12288, 4, [(9216, 1)]),          # a segment of 3 blocks does not tile 4 blocks
])
def test_plan_rejects_splits_the_kernels_do_not_take(N, world, pats):
    with pytest.raises(ValueError):
        seqpar.plan(N, world, pats)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        N, pats = CASES[world]
        H, d = 3, 4
        L = N // world
        # every rank draws the same full tensor and keeps its block; the value
        # of a row encodes its position and head, so a misplaced row shows
        k_full = (np.arange(N)[None, :, None, None] * 10 + np.arange(H)[None, None, :, None]
                  + 0.25 * np.arange(d)[None, None, None, :]).astype(np.float64)
        block = torch.from_numpy(k_full[:, rank * L:(rank + 1) * L].copy())
        bad = []
        for p in seqpar.plan(N, world, pats):
            if not p.spans:
                continue
            send = torch.empty((1, L // p.r, H, d), dtype=torch.float64)
            for h in range(H):
                loc = [x - rank * L for x in seqpar.packed_positions(p, L, rank, h)]
                send[0, :, h] = block[0, loc, h]
            recv = [torch.empty_like(send) for _ in range(world)]
            dist.all_gather(recv, send)
            seg = p.segment_ranks(rank)
            gathered = torch.cat([recv[g] for g in seg], dim=1)  # [1, ranks * L / r, H, d]
            s_idx = (rank * L) // p.w if p.w < N else 0
            for h in range(H):
                want = oracle.kept_rows(N, p.w, p.r, h)[s_idx]
                if not np.array_equal(gathered[0, :, h].numpy(), k_full[0, want, h]):
                    bad.append(("gathered", p.index, h))
                # this rank's kept rows sit at the tile offset the kernel gets
                mine = [x for x in want if rank * L <= x < (rank + 1) * L]
                first = int(np.searchsorted(want, mine[0]))
                if first != p.tile_offset(rank) * seqpar.BM or len(mine) != p.rank_rows:
                    bad.append(("offset", p.index, h))
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(bad))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_gather_the_segments_kept_rows(tmp_path, world):
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        assert (tmp_path / f"r{r}.txt").read_text() == "[]"


# (N, world, patterns): local and spanning patterns, one with w > N
MATH_CASES = [
    (2048, 2, [(256, 1), (512, 2), (2048, 4), (1024, 8)]),
    (4096, 4, [(512, 1), (1024, 2), (2048, 4), (4096, 8)]),
    (2048, 2, [(512, 1), (4096, 8)]),
]


def _attend(Q, K, V, tau, causal, q0):
    """Softmax attention of rows Q, which sit at positions q0, q0 + 1, ... of
    the key sequence K (causal: a row sees keys up to its own position)."""
    S = tau * (Q @ K.T)
    if causal:
        pos = q0 + np.arange(Q.shape[0])[:, None]
        S = np.where(np.arange(K.shape[0])[None, :] <= pos, S, -np.inf)
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    Z = E.sum(axis=1)
    return (E @ V) / Z[:, None], m + np.log(Z)


def _block_rows(qb, kb, vb, pats, plans, rank, gathered, causal):
    """This rank's merged rows in float64: qb, kb, vb [L, H, d] its block;
    gathered[i] = (K, V), each [rows, H, d], the kept rows of this rank's
    segment of spanning pattern i in sequence order. Returns out [L, H, d] and
    lse [H, L]."""
    L, H, d = qb.shape
    tau = 1.0 / math.sqrt(d)
    outs, lses = [], []
    local = [p for p in plans if not p.spans]
    if local:
        O_i, lse_i = oracle.fwd_per_pattern(qb[None], kb[None], vb[None],
                                            [(p.w, p.r) for p in local], causal)
        outs += [O_i[j, 0] for j in range(len(local))]
        lses += [lse_i[j, 0] for j in range(len(local))]
    for p in plans:
        if not p.spans:
            continue
        K, V = gathered[p.index]
        O = np.zeros((L, H, d))
        lse = np.full((H, L), -np.inf)
        for h in range(H):
            rows = [x - rank * L for x in seqpar.packed_positions(p, L, rank, h)]
            O[rows, h], lse[h, rows] = _attend(qb[rows, h], K[:, h], V[:, h], tau, causal,
                                               p.tile_offset(rank) * seqpar.BM)
        outs.append(O)
        lses.append(lse)
    # merge through the denominators, row by row of this block
    lse_all = np.stack(lses)                        # [P, H, L]
    mx = lse_all.max(axis=0)
    sel = np.isfinite(mx)
    mx0 = np.where(sel, mx, 0.0)
    wts = np.exp(lse_all - mx0[None])               # exp(-inf) = 0 for rows not kept
    tot = np.where(sel, wts.sum(axis=0), 1.0)
    lse_m = np.where(sel, mx0 + np.log(tot), -np.inf)
    out = sum(np.transpose(wts[i] / tot, (1, 0))[:, :, None] * outs[i] for i in range(len(outs)))
    return out, lse_m


def _errors(out, lse, want_o, want_l):
    """(max |out error|, max |lse error| over finite rows, same -inf rows, kept rows)."""
    err_o = float(np.abs(out - want_o).max())
    same_inf = bool(np.array_equal(np.isinf(lse), np.isinf(want_l)))
    fin = np.isfinite(lse)
    err_l = float(np.abs(lse[fin] - want_l[fin]).max()) if fin.any() else 0.0
    return err_o, err_l, same_inf, int(fin.sum())


def _init_gloo(rank, world, port):
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    return dist


def _full_inputs(N, H, d):
    rng = np.random.default_rng(23)
    return [rng.standard_normal((1, N, H, d)) for _ in range(3)]


def _rank_math(rank: int, world: int, port: int, out_dir: str, case: int, causal: bool):
    dist = _init_gloo(rank, world, port)
    try:
        N, _, pats = MATH_CASES[case]
        H, d = 3, 8
        L = N // world
        q_full, k_full, v_full = _full_inputs(N, H, d)
        blk = slice(rank * L, (rank + 1) * L)
        qb, kb, vb = (x[0, blk] for x in (q_full, k_full, v_full))   # [L, H, d]
        plans = seqpar.plan(N, world, pats)
        gathered = {}
        for p in plans:
            if not p.spans:
                continue
            send = torch.empty((2, L // p.r, H, d), dtype=torch.float64)
            for h in range(H):
                rows = [x - rank * L for x in seqpar.packed_positions(p, L, rank, h)]
                send[0, :, h] = torch.from_numpy(kb[rows, h])
                send[1, :, h] = torch.from_numpy(vb[rows, h])
            recv = [torch.empty_like(send) for _ in range(world)]
            dist.all_gather(recv, send)
            g = torch.cat([recv[r_] for r_ in p.segment_ranks(rank)], dim=1).numpy()
            gathered[p.index] = (g[0], g[1])
        out, lse = _block_rows(qb, kb, vb, pats, plans, rank, gathered, causal)
        want_o, want_l = oracle.fwd(q_full, k_full, v_full, pats, causal)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(_errors(out, lse, want_o[0, blk], want_l[0, :, blk])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("case", range(len(MATH_CASES)))
def test_gloo_ranks_reproduce_the_merged_rows(tmp_path, case, causal):
    world = MATH_CASES[case][1]
    port = _free_port()
    mp.start_processes(_rank_math, args=(world, port, str(tmp_path), case, causal),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        err_o, err_l, same_inf, kept = eval((tmp_path / f"r{r}.txt").read_text())
        assert same_inf and kept > 0
        assert err_o < 1e-12 and err_l < 1e-12, (r, err_o, err_l)


def _rank_forward(rank: int, world: int, port: int, out_dir: str, case: int, causal: bool):
    """seqpar.forward as a user calls it, on gloo ranks: its packing calls, its
    all-gather and its slicing of the gathered buffers run as written; the two
    library calls are replaced by host stand-ins (the packing rule, and the
    float64 decomposition on the buffers forward hands over)."""
    dist = _init_gloo(rank, world, port)
    try:
        from sparse_long_sequence_dilated_b200 import dilattn

        N, _, pats = FORWARD_CASES[case]
        B, H, d = 2, 3, 8
        L = N // world
        rng = np.random.default_rng(29)
        q_full, k_full, v_full = (rng.standard_normal((B, N, H, d)) for _ in range(3))
        blk = slice(rank * L, (rank + 1) * L)
        plans = seqpar.plan(N, world, pats)
        seen = []

        def pack_dilated(x, r, out=None, stream=None):
            Bx, Lx, Hx, dx = x.shape
            buf = torch.empty((Bx, Lx // r, Hx, dx), dtype=x.dtype)
            for h in range(Hx):
                buf[:, :, h] = x[:, (h % r)::r, h]
            return buf

        def fwd_seqpar(q, k, v, patterns, rank_, world_, kg, vg, causal_, out, lse, stream):
            seen.append((rank_, world_, causal_, [g is None for g in kg], [g is None for g in vg]))
            out = torch.empty_like(q)
            lse = torch.empty((q.shape[0], q.shape[2], q.shape[1]), dtype=torch.float64)
            for b in range(q.shape[0]):
                gathered = {}
                for p in plans:
                    if p.spans:
                        assert tuple(kg[p.index].shape) == (p.ranks, q.shape[0], p.rank_rows, H, d)
                        gathered[p.index] = tuple(
                            t[:, b].reshape(p.ranks * p.rank_rows, H, d).numpy() for t in
                            (kg[p.index], vg[p.index]))
                o_b, l_b = _block_rows(q[b].numpy(), k[b].numpy(), v[b].numpy(), patterns, plans,
                                       rank_, gathered, causal_)
                out[b], lse[b] = torch.from_numpy(o_b), torch.from_numpy(l_b)
            return out, lse

        dilattn.pack_dilated = pack_dilated
        dilattn.fwd_seqpar = fwd_seqpar
        blocks = [torch.from_numpy(np.ascontiguousarray(x[:, blk])) for x in (q_full, k_full, v_full)]
        out, lse = seqpar.forward(*blocks, pats, causal)
        want_o, want_l = oracle.fwd(q_full, k_full, v_full, pats, causal)
        errs = [_errors(out[b].numpy(), lse[b].numpy(), want_o[b, blk], want_l[b, :, blk])
                for b in range(B)]
        spans = [not p.spans for p in plans]
        ok_calls = seen == [(rank, world, causal, spans, spans)]
        # segments over fewer ranks than the group gather inside their own subgroup
        sub = sorted({p.ranks for p in plans if p.spans and p.ranks < world})
        ok_calls = ok_calls and sorted(seqpar._SEGMENT_GROUPS) == sub
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr((errs, ok_calls)))
    finally:
        dist.destroy_process_group()


# the decomposition cases, and 8 ranks whose segments span 2, 4 and 8 of them
FORWARD_CASES = MATH_CASES + [(8192, 8, [(512, 1), (2048, 2), (4096, 4), (8192, 8)])]


@pytest.mark.parametrize("case,causal", [(c, x) for c in range(len(MATH_CASES))
                                         for x in (True, False)] + [(len(MATH_CASES), True)])
def test_seqpar_forward_on_gloo_ranks(tmp_path, case, causal):
    world = FORWARD_CASES[case][1]
    port = _free_port()
    mp.start_processes(_rank_forward, args=(world, port, str(tmp_path), case, causal),
                       nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        errs, ok_calls = eval((tmp_path / f"r{r}.txt").read_text())
        assert ok_calls, r
        for err_o, err_l, same_inf, kept in errs:
            assert same_inf and kept > 0
            assert err_o < 1e-12 and err_l < 1e-12, (r, err_o, err_l)
