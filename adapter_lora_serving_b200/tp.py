"""Tensor-parallel use of the delta path: one process per GPU, the shards of a
projection held by the ranks of a torch.distributed group.

Sources: mstar.engine.resources.lora.backend, module text ("out_slices are
this rank's widths of a fused projection's outputs") and
mstar.model.components.linear (FusedColumnLinear is the non-sharded form of
the TP-aware QKVParallelLinear / MergedColumnParallelLinear).

* Column-parallel (the QKV and gate/up projections): every rank holds its
  contiguous share of every output slice, its rows of B, and the whole A.
  The delta of its columns needs nothing from the other ranks: it is the fused
  apply with this rank's widths (`apply_linear_column_parallel`).
* Row-parallel (the reading for the projections that split the input
  features, e.g. o_proj / down_proj): every rank holds its share of the input
  features of x and of A, and the whole B; the shrink of each rank is a
  partial h over its features, the ranks' partials are summed with one fp32
  all-reduce of T x S*R values, and every rank expands the full h onto its
  replica of y (`apply_linear_row_parallel`).

Only argument marshalling and the one collective live here; the arithmetic is
the library's kernels.
"""
from __future__ import annotations

from . import lora as L


def column_shares(out_slices, world, rank):
    """This rank's (start, width) in every slice of a column-parallel fused
    projection: slice i splits into `world` equal contiguous shares."""
    out = []
    for w in out_slices:
        w = int(w)
        if w % world:
            raise ValueError(f"slice width {w} does not split into {world} shares")
        share = w // world
        if share % 8:
            raise ValueError(f"share width {share} is not a multiple of 8")
        out.append((rank * share, share))
    return out


def column_widths(out_slices, world, rank):
    """The out_slices this rank passes to the fused apply."""
    return tuple(w for _, w in column_shares(out_slices, world, rank))


def row_range(in_features, world, rank):
    """[k0, k1): this rank's share of the input features of a row-parallel
    projection (contiguous, equal, multiples of 8)."""
    if in_features % (8 * world):
        raise ValueError(f"in_features {in_features} does not split into {world} shares of 8k")
    share = in_features // world
    return rank * share, (rank + 1) * share


def shard_b_columns(b, out_slices, world, rank):
    """This rank's rows of a full B [slots, out, R] under column-parallel
    sharding, contiguous (setup helper: in a deployment every rank loads only
    its own rows)."""
    import torch
    parts = []
    off = 0
    for (start, width), w in zip(column_shares(out_slices, world, rank), out_slices):
        parts.append(b[:, off + start:off + start + width, :])
        off += int(w)
    return torch.cat(parts, dim=1).contiguous()


def apply_linear_column_parallel(x, y_local, a, b_local, ranks, scalings, token_order,
                                 slot_indptr, T, in_features, slots, R, out_slices, world, rank,
                                 regime=L.LORA_REGIME_AUTO, workspace=None, workspace_bytes=0,
                                 err_flags=None, stream=None):
    """y_local [T, sum of this rank's widths] += the delta of this rank's
    columns; b_local holds this rank's rows of B.  No communication."""
    L.lora_apply_linear(x, y_local, a, b_local, ranks, scalings, token_order, slot_indptr, T,
                        in_features, slots, R, column_widths(out_slices, world, rank),
                        regime=regime, workspace=workspace, workspace_bytes=workspace_bytes,
                        err_flags=err_flags, stream=stream)


def apply_linear_row_parallel(x_local, y, a_local, b, ranks, scalings, token_order,
                              slot_indptr, T, in_local, slots, R, out_slices, h=None,
                              group=None, regime=L.LORA_REGIME_AUTO, err_flags=None):
    """y [T, out] (this rank's replica) += the delta of the whole projection,
    from this rank's input features (x_local [T, in_local], a_local
    [slots, S*R, in_local]): shrink, all-reduce of h (fp32, sum), expand.
    h: an fp32 [T, S*R] device buffer to use (zeroed here), or None.  Runs on
    the current stream; every rank of `group` must call it."""
    import torch
    import torch.distributed as dist
    S = len(out_slices)
    if h is None:
        h = torch.zeros((T, S * R), dtype=torch.float32, device=x_local.device)
    else:
        h.zero_()        # entries no live token writes stay 0 through the sum
    L.lora_shrink(x_local, h, a_local, ranks, token_order, slot_indptr, T, in_local, slots, R,
                  S, regime=regime, err_flags=err_flags)
    dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
    L.lora_expand(y, h, b, ranks, scalings, token_order, slot_indptr, T, slots, R, out_slices,
                  regime=regime, err_flags=err_flags)
    return h
