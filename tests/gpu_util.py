"""Helpers for the GPU parity tests: move seeded problems to the device, call the
library through the C ABI, bring results back as exact float64 values."""
import numpy as np

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W


def torch():
    import torch as _t
    return _t


def dev_bf16(bits):
    t = torch()
    arr = np.ascontiguousarray(bits, dtype=np.uint16)
    return t.from_numpy(arr.view(np.int16).copy()).view(t.bfloat16).cuda()


def dev_i32(v):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(v, dtype=np.int32).copy()).cuda()


def dev_f32(v):
    t = torch()
    return t.from_numpy(np.ascontiguousarray(v, dtype=np.float32).copy()).cuda()


def host_bits(tensor):
    t = torch()
    return tensor.detach().view(t.int16).cpu().numpy().view(np.uint16)


def host_f64(tensor):
    return W.bf16_to_f64(host_bits(tensor))


def flags_buf():
    t = torch()
    return t.zeros(1, dtype=t.int32, device="cuda")


def read_flags(buf):
    return int(buf.cpu().numpy().view(np.uint32)[0])


class LinearDev:
    """A LinearProblem on the device."""

    def __init__(self, p, y_bits=None):
        self.p = p
        self.x = dev_bf16(p.x) if p.x is not None else None
        self.ids = dev_i32(p.ids) if p.ids is not None else None
        self.a = dev_bf16(p.a)
        self.b = dev_bf16(p.b)
        self.y = dev_bf16(p.y if y_bits is None else y_bits)
        self.ranks = dev_i32(p.ranks)
        self.scalings = dev_f32(p.scalings)
        self.token_order = dev_i32(p.token_order)
        self.slot_indptr = dev_i32(p.slot_indptr)
        self.flags = flags_buf()

    def apply_linear(self, regime=L.LORA_REGIME_AUTO, workspace=None, out_slices=None,
                     use_workspace=True):
        """lora_apply_linear with a zeroed workspace of lora_workspace_bytes (the
        BGMV split kernel, or SGMV), or with none (use_workspace=False: the BGMV
        cluster kernel)."""
        p = self.p
        ws_bytes = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R,
                                          p.num_slices, regime) if use_workspace else 0
        if ws_bytes and workspace is None:
            t = torch()
            workspace = t.zeros(ws_bytes // 4 + 4, dtype=t.float32, device="cuda")
        L.lora_apply_linear(self.x, self.y, self.a, self.b, self.ranks, self.scalings,
                            self.token_order, self.slot_indptr, p.T, p.n_in, p.slots, p.R,
                            out_slices or p.out_slices, regime=regime, workspace=workspace,
                            workspace_bytes=ws_bytes, err_flags=self.flags)

    def apply_router(self, regime=L.LORA_REGIME_AUTO):
        """lora_apply_router on a one-slice problem (y = the routing logits)."""
        p = self.p
        assert p.num_slices == 1
        ws_bytes = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R, 1, regime)
        workspace = None
        if ws_bytes:
            t = torch()
            workspace = t.zeros(ws_bytes // 4 + 4, dtype=t.float32, device="cuda")
        L.lora_apply_router(self.x, self.y, self.a, self.b, self.ranks, self.scalings,
                            self.token_order, self.slot_indptr, p.T, p.n_in, p.slots, p.R,
                            p.out, regime=regime, workspace=workspace, workspace_bytes=ws_bytes,
                            err_flags=self.flags)

    def shrink(self, h, regime=L.LORA_REGIME_AUTO):
        p = self.p
        L.lora_shrink(self.x, h, self.a, self.ranks, self.token_order, self.slot_indptr, p.T,
                      p.n_in, p.slots, p.R, p.num_slices, regime=regime, err_flags=self.flags)

    def expand(self, h, regime=L.LORA_REGIME_AUTO):
        p = self.p
        L.lora_expand(self.y, h, self.b, self.ranks, self.scalings, self.token_order,
                      self.slot_indptr, p.T, p.slots, p.R, p.out_slices, regime=regime,
                      err_flags=self.flags)

    def gather_shrink(self, h):
        p = self.p
        L.lora_gather_shrink(self.ids, h, self.a, self.ranks, self.token_order, self.slot_indptr,
                             p.T, p.n_in, p.slots, p.R, p.num_slices, err_flags=self.flags)

    def apply_embedding(self, regime=L.LORA_REGIME_AUTO):
        p = self.p
        L.lora_apply_embedding(self.ids, self.y, self.a, self.b, self.ranks, self.scalings,
                               self.token_order, self.slot_indptr, p.T, p.n_in, p.slots, p.R,
                               p.out_slices, regime=regime, err_flags=self.flags)


class MoEDev:
    def __init__(self, m, y_bits=None):
        self.m = m
        self.x = dev_bf16(m.x)
        self.y = dev_bf16(m.y if y_bits is None else y_bits)
        self.a = dev_bf16(m.a)
        self.b = dev_bf16(m.b)
        self.pair_index = dev_i32(m.pair_index)
        self.ranks = dev_i32(m.ranks)
        self.scalings = dev_f32(m.scalings)
        self.row_slot = dev_i32(m.row_slot)
        self.offsets = dev_i32(m.expert_offsets)
        self.flags = flags_buf()

    def apply(self, grouped=False, workspace=None):
        """lora_expert_apply: without a workspace (the per-chunk BGMV kernel)
        or, grouped=True, with a workspace of lora_workspace_bytes (the fold
        grouped by (slot, expert) on the tensor-core kernels)."""
        m = self.m
        ws_bytes = 0
        if grouped:
            ws_bytes = L.lora_workspace_bytes(L.LORA_OP_EXPERT_APPLY, m.rows_cap, m.num_experts,
                                              m.R, m.num_slices)
            assert ws_bytes > 0
            if workspace is None:
                t = torch()
                workspace = t.empty(ws_bytes // 4 + 4, dtype=t.int32, device="cuda")
        L.lora_expert_apply(self.x, self.y, self.a, self.b, self.pair_index, self.ranks,
                            self.scalings, self.row_slot, self.offsets, m.rows_cap, m.n_in,
                            m.num_experts, m.slots, m.num_pairs, m.R, m.out_slices,
                            workspace=workspace if grouped else None,
                            workspace_bytes=ws_bytes, err_flags=self.flags)


def assert_close(y_dev, y_ref, what=""):
    from oracle import lora_oracle as O
    ok = O.within_tolerance(y_dev, y_ref)
    ok |= np.isnan(y_dev) & np.isnan(y_ref)          # NaN placed in y stays NaN
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} of {ok.size} elements out of tolerance; "
                             f"first at {i}: dev={y_dev[i]!r} ref={y_ref[i]!r}")


def assert_rows_bit_identical(bits_out, bits_in, rows, what=""):
    rows = np.asarray(rows)
    if rows.dtype == bool:
        rows = np.nonzero(rows)[0]
    diff = bits_out[rows] != bits_in[rows]
    if diff.any():
        r = rows[np.argwhere(diff)[0][0]]
        raise AssertionError(f"{what}: untouched row {r} changed")
