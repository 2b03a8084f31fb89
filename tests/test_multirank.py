"""Host logic of the multi-GPU bench path, run as two gloo ranks on the CPU.

With N > 1 GPUs every rank runs its own batch with no data-path exchange; the
only collective is the reduction of the timings, so the job's time is the
slowest rank's and its throughput counts every rank's work. These checks run
that logic with world_size 2 over gloo (no GPU needed)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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

    import bench
    from sparse_long_sequence_dilated_b200.workloads import make_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        job_ms = bench.max_over_ranks(local_ms, world)
        inp = make_inputs(1, 64, 2, 64, bench.rank_seed(0, rank), "bf16", ("q",))
        digests = [None] * world
        dist.all_gather_object(digests, int(np.asarray(inp["q_bits"]).astype(np.int64).sum()))
        tflops = bench.job_tflops(world, 2.0e12, job_ms)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([job_ms, tflops, digests[0], digests[1]], dtype=np.float64))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_all_work(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    res = [np.load(os.path.join(tmp_path, f"rank{r}.npy")) for r in range(world)]
    for r in res:
        assert r[0] == pytest.approx(15.0)          # max over ranks, on every rank
        assert r[1] == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)  # both ranks' work / slowest time
        assert r[2] != r[3]                         # each rank draws its own batch
    assert res[0][2] == res[1][2] and res[0][3] == res[1][3]


def test_single_rank_helpers_need_no_process_group():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.rank_seed(7, 0) == 7 and bench.rank_seed(7, 3) == 10
    assert bench.job_tflops(1, 1.0e12, 1000.0, calls=4) == pytest.approx(4.0)
