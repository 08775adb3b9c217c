"""Tensor-parallel decomposition on CPU: the shard helpers of
adapter_lora_serving_b200.tp, and two `gloo` ranks that run the fp64 oracle on
their shards -- column-parallel (each rank's columns of every slice, no
communication) and row-parallel (each rank's input features, h summed by an
all-reduce) -- and reproduce the unsharded fold."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from adapter_lora_serving_b200 import tp  # noqa: E402


def test_column_shares_cover_every_slice():
    out_slices = (4096, 1024, 1024)
    for world in (1, 2, 4, 8):
        cols = [set() for _ in out_slices]
        for rank in range(world):
            for i, (start, width) in enumerate(tp.column_shares(out_slices, world, rank)):
                assert width == out_slices[i] // world and width % 8 == 0
                cols[i].update(range(start, start + width))
        assert [len(c) for c in cols] == list(out_slices)
    assert tp.column_widths(out_slices, 4, 3) == (1024, 256, 256)
    with pytest.raises(ValueError):
        tp.column_shares((24,), 2, 0)            # a share of 12 is not whole uint4 rows


def test_row_range_partitions_the_features():
    got = [tp.row_range(4096, 4, r) for r in range(4)]
    assert got == [(0, 1024), (1024, 2048), (2048, 3072), (3072, 4096)]
    with pytest.raises(ValueError):
        tp.row_range(100, 2, 0)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from adapter_lora_serving_b200 import tp as TP
    from adapter_lora_serving_b200 import workloads as W
    from oracle import lora_oracle as O
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p = W.random_linear(77, 60, 256, (64, 32, 32), 5, 16, dead_frac=0.1)
        f = W.bf16_to_f64
        x, y, a, b = f(p.x), f(p.y), f(p.a), f(p.b)
        # row-parallel: this rank's features, partial h, sum over the ranks
        k0, k1 = TP.row_range(p.n_in, world, rank)
        h, mask, _ = O.shrink(x[:, k0:k1], a[:, :, k0:k1], p.token_order, p.slot_indptr,
                              p.ranks, p.R, p.num_slices)
        ht = torch.from_numpy(np.where(mask, h, 0.0))
        dist.all_reduce(ht, op=dist.ReduceOp.SUM)
        y_row, _, _ = O.expand(y, ht.numpy(), b, p.token_order, p.slot_indptr, p.ranks,
                               p.scalings, p.out_slices, p.R)
        # column-parallel: this rank's columns of every slice, its rows of B
        shares = TP.column_shares(p.out_slices, world, rank)
        offs = np.concatenate([[0], np.cumsum(p.out_slices)])
        cols = np.concatenate([np.arange(offs[i] + s0, offs[i] + s0 + w)
                               for i, (s0, w) in enumerate(shares)])
        y_col, _, _ = O.apply_linear(x, y[:, cols], a, b[:, cols, :], p.token_order,
                                     p.slot_indptr, p.ranks, p.scalings,
                                     TP.column_widths(p.out_slices, world, rank), p.R)
        gathered = [None] * world
        dist.all_gather_object(gathered, (cols, y_col))
        out.put((rank, y_row, gathered))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_unsharded_fold():
    import torch.multiprocessing as mp
    from adapter_lora_serving_b200 import workloads as W
    from oracle import lora_oracle as O
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
    p = W.random_linear(77, 60, 256, (64, 32, 32), 5, 16, dead_frac=0.1)
    f = W.bf16_to_f64
    ref, _, _ = O.apply_linear(f(p.x), f(p.y), f(p.a), f(p.b), p.token_order, p.slot_indptr,
                               p.ranks, p.scalings, p.out_slices, p.R)
    for rank, y_row, gathered in res:
        # every rank's replica after the all-reduce of h: the whole fold
        assert np.allclose(y_row, ref, rtol=1e-12, atol=1e-12)
        full = np.full_like(ref, np.nan)
        for cols, y_col in gathered:
            full[:, cols] = y_col
        # the ranks' columns together: the whole fold, each column once
        assert np.allclose(full, ref, rtol=1e-12, atol=1e-12)
