"""Tensor-parallel shards on the GPU (the library's kernels on each rank's
share): column-parallel shares of every slice, row-parallel feature shares
whose partial h are summed, and the row-parallel entry point with a
one-rank NCCL group.  Checked against the unsharded fp64 oracle:
|y_dev - y_ref| <= 1e-2 + 1.6e-2 |y_ref|."""
import datetime
import os
import socket

import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import tp
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import LinearDev, assert_close, dev_bf16, host_bits, torch

pytestmark = pytest.mark.gpu

f64 = W.bf16_to_f64


def _ref(p):
    ref, _, _ = O.apply_linear(f64(p.x), f64(p.y), f64(p.a), f64(p.b), p.token_order,
                               p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)
    return ref


@pytest.mark.parametrize("world", [2, 4])
def test_column_parallel_shares(world):
    t = torch()
    p = W.decode_qkv(3)
    d = LinearDev(p)
    out = np.empty_like(p.y)
    offs = np.concatenate([[0], np.cumsum(p.out_slices)])
    for rank in range(world):
        shares = tp.column_shares(p.out_slices, world, rank)
        cols = np.concatenate([np.arange(offs[i] + s0, offs[i] + s0 + w)
                               for i, (s0, w) in enumerate(shares)])
        y_local = dev_bf16(p.y[:, cols])
        b_local = tp.shard_b_columns(d.b, p.out_slices, world, rank)
        tp.apply_linear_column_parallel(d.x, y_local, d.a, b_local, d.ranks, d.scalings,
                                        d.token_order, d.slot_indptr, p.T, p.n_in, p.slots, p.R,
                                        p.out_slices, world, rank)
        out[:, cols] = host_bits(y_local)
    assert_close(f64(out), _ref(p), "column-parallel")


@pytest.mark.parametrize("regime", [L.LORA_REGIME_BGMV, L.LORA_REGIME_SGMV])
def test_row_parallel_feature_shares(regime):
    """Each share's shrink on the GPU, the partial h summed (what the
    all-reduce does across ranks), then the expand."""
    t = torch()
    p = W.random_linear(88, 1500, 512, (128, 64), 4, 16, ranks=[16, 8, 16, 16])
    d = LinearDev(p)
    world = 2
    h = t.zeros((p.T, p.num_slices * p.R), dtype=t.float32, device="cuda")
    for rank in range(world):
        k0, k1 = tp.row_range(p.n_in, world, rank)
        x_r = dev_bf16(np.ascontiguousarray(p.x[:, k0:k1]))
        a_r = dev_bf16(np.ascontiguousarray(p.a[:, :, k0:k1]))
        h_r = t.zeros_like(h)
        L.lora_shrink(x_r, h_r, a_r, d.ranks, d.token_order, d.slot_indptr, p.T, k1 - k0,
                      p.slots, p.R, p.num_slices, regime=regime)
        h += h_r
    L.lora_expand(d.y, h, d.b, d.ranks, d.scalings, d.token_order, d.slot_indptr, p.T, p.slots,
                  p.R, p.out_slices, regime=regime)
    assert_close(f64(host_bits(d.y)), _ref(p), "row-parallel shares")


def test_row_parallel_entry_point_one_rank_group():
    t = torch()
    import torch.distributed as dist
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        p = W.decode_qkv(4)
        d = LinearDev(p)
        tp.apply_linear_row_parallel(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order,
                                     d.slot_indptr, p.T, p.n_in, p.slots, p.R, p.out_slices)
        t.cuda.synchronize()
        assert_close(f64(host_bits(d.y)), _ref(p), "row-parallel, one rank")
    finally:
        dist.destroy_process_group()
