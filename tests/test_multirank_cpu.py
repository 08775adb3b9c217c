"""The multi-GPU path of bench.py, on CPU: world_size-2 `gloo` ranks check the
pieces a replicated run relies on -- the timed seconds are the max over ranks,
the job throughput counts every rank's units, and ranks draw disjoint input
seeds (independent batches, no collective on the data path)."""
import datetime
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        sec = bench.reduce_max_over_ranks(torch, dist, 0.25 * (rank + 1), "cpu")
        # every rank contributes the seeds of each workload's rotating input
        # sets (as many as bench.py draws); the union must have no repeats
        seeds = {}
        for name in bench.W.WORKLOADS:
            n = bench.n_sets_for(name)
            seeds[name] = [bench.rank_seed0(rank, n) + i for i in range(n)]
        gathered = [None] * world
        dist.all_gather_object(gathered, seeds)
        out.put((rank, sec, gathered))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_disjoint_seeds():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, sec, gathered in res:
        assert sec == pytest.approx(0.5)          # the slower rank's seconds
        for name in gathered[0]:
            flat = [s for seeds in gathered for s in seeds[name]]
            assert len(flat) == len(set(flat)), name   # independent batches per rank


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 256 tokens per rank-step, 100 steps, 4 ranks, 0.5 s (the slowest rank)
    assert bench.job_throughput(256, 100, 4, 0.5) == pytest.approx(204800.0)
