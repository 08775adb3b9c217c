"""Thin Python binding of ``liblora_delta.so`` (the C ABI in ``include/lora_delta.h``).

Argument marshalling only: every function here has the C name, passes device
pointers, sizes and the stream straight through, and raises ``LoraError`` on a
non-OK status.  Tensors are ``torch`` tensors on the CUDA device (torch is used
for device memory and streams only); integers are accepted as raw device
pointers.  There is no fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblora_delta.so")

LORA_OK = 0
LORA_ERR_INVALID = 1
LORA_ERR_UNSUPPORTED = 2
LORA_ERR_WORKSPACE = 3
LORA_ERR_CUDA = 4

LORA_FLAG_BAD_INDPTR = 1
LORA_FLAG_BAD_TOKEN = 2
LORA_FLAG_BAD_RANK = 4
LORA_FLAG_BAD_SLOT = 8
LORA_FLAG_BAD_PAIR = 16
LORA_FLAG_BAD_OFFSETS = 32
LORA_FLAG_TIMEOUT = 64

LORA_REGIME_AUTO = 0
LORA_REGIME_BGMV = 1
LORA_REGIME_SGMV = 2
LORA_REGIME_BGMV_SPLIT = 3
LORA_REGIME_STREAM = 4

LORA_OP_SHRINK = 0
LORA_OP_EXPAND = 1
LORA_OP_APPLY_LINEAR = 2
LORA_OP_GATHER_SHRINK = 3
LORA_OP_APPLY_EMBEDDING = 4
LORA_OP_EXPERT_APPLY = 5

LORA_STATIC_SCRATCH_BYTES = 16 << 20

# (name, restype, argtypes) of every exported symbol.
_P = ctypes.c_void_p
_I = ctypes.c_int32
_Z = ctypes.c_size_t
_SIGS = [
    ("lora_shrink", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P]),
    ("lora_expand", _I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _I, _I, _P, _P]),
    ("lora_apply_linear", _I,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P, _Z, _P, _P]),
    ("lora_apply_linear_noalloc", _I,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P, _P]),
    ("lora_apply_router", _I,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z, _P, _P]),
    ("lora_gather_shrink", _I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P]),
    ("lora_apply_embedding", _I,
     [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _I, _I, _P, _P]),
    ("lora_expert_apply", _I,
     [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _I, _P, _Z, _P, _P]),
    ("lora_workspace_bytes", _Z, [_I, _I, _I, _I, _I, _I]),
    ("lora_resolve_regime", _I, [_I, _I, _I, _I, _I]),
    ("lora_plan_tile", _I, [_I, _I]),
    ("lora_plan_linear", _I, [_P, _P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P]),
    ("lora_plan_expert", _I, [_P, _P, _I, _I, _I, _I, _P, _I, _P, _P, _P]),
    ("lora_set_launch_overlap", _I, [_I]),
    ("lora_set_wait_limit_ns", ctypes.c_uint64, [ctypes.c_uint64]),
    ("lora_status_string", ctypes.c_char_p, [_I]),
    ("lora_last_error", ctypes.c_char_p, []),
    ("lora_version", ctypes.c_char_p, []),
]
EXPORTED = [s[0] for s in _SIGS]

_lib = None


class LoraError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{message} ({status})")
        self.status = status


def load(path: str | None = None):
    """Load the library once; raises if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(f"{p} is missing: build it with python -m adapter_lora_serving_b200.build")
    lib = ctypes.CDLL(p)
    for name, res, args in _SIGS:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _slices(out_slices):
    arr = (ctypes.c_int32 * len(out_slices))(*[int(v) for v in out_slices])
    return arr


def _check(status):
    if status != LORA_OK:
        lib = load()
        raise LoraError(lib.lora_status_string(status).decode(),
                        lib.lora_last_error().decode())


def lora_shrink(x, h, a, ranks, token_order, slot_indptr, T, in_features, slots, R,
                num_slices, regime=LORA_REGIME_AUTO, err_flags=None, stream=None):
    _check(load().lora_shrink(_ptr(x), _ptr(h), _ptr(a), _ptr(ranks), _ptr(token_order),
                              _ptr(slot_indptr), T, in_features, slots, R, num_slices, regime,
                              _ptr(err_flags), _stream(stream)))


def lora_expand(y, h, b, ranks, scalings, token_order, slot_indptr, T, slots, R, out_slices,
                regime=LORA_REGIME_AUTO, err_flags=None, stream=None):
    _check(load().lora_expand(_ptr(y), _ptr(h), _ptr(b), _ptr(ranks), _ptr(scalings),
                              _ptr(token_order), _ptr(slot_indptr), T, slots, R,
                              _slices(out_slices), len(out_slices), regime, _ptr(err_flags),
                              _stream(stream)))


def lora_apply_linear(x, y, a, b, ranks, scalings, token_order, slot_indptr, T, in_features,
                      slots, R, out_slices, regime=LORA_REGIME_AUTO, workspace=None,
                      workspace_bytes=0, err_flags=None, stream=None):
    _check(load().lora_apply_linear(_ptr(x), _ptr(y), _ptr(a), _ptr(b), _ptr(ranks),
                                    _ptr(scalings), _ptr(token_order), _ptr(slot_indptr), T,
                                    in_features, slots, R, _slices(out_slices), len(out_slices),
                                    regime, _ptr(workspace), workspace_bytes, _ptr(err_flags),
                                    _stream(stream)))


def lora_apply_linear_noalloc(x, y, a, b, ranks, scalings, token_order, slot_indptr, T,
                              in_features, slots, R, out_slices, regime=LORA_REGIME_AUTO,
                              err_flags=None, stream=None):
    """lora_apply_linear without a workspace, for callers that cannot allocate
    device memory: the library's fixed scratch array is used instead."""
    _check(load().lora_apply_linear_noalloc(_ptr(x), _ptr(y), _ptr(a), _ptr(b), _ptr(ranks),
                                            _ptr(scalings), _ptr(token_order),
                                            _ptr(slot_indptr), T, in_features, slots, R,
                                            _slices(out_slices), len(out_slices), regime,
                                            _ptr(err_flags), _stream(stream)))


def lora_apply_router(router_in, gate_logits, a, b, ranks, scalings, token_order, slot_indptr,
                      T, hidden, slots, R, num_experts, regime=LORA_REGIME_AUTO, workspace=None,
                      workspace_bytes=0, err_flags=None, stream=None):
    _check(load().lora_apply_router(_ptr(router_in), _ptr(gate_logits), _ptr(a), _ptr(b),
                                    _ptr(ranks), _ptr(scalings), _ptr(token_order),
                                    _ptr(slot_indptr), T, hidden, slots, R, num_experts, regime,
                                    _ptr(workspace), workspace_bytes, _ptr(err_flags),
                                    _stream(stream)))


def lora_gather_shrink(ids, h, a, ranks, token_order, slot_indptr, T, vocab, slots, R,
                       num_slices, err_flags=None, stream=None):
    _check(load().lora_gather_shrink(_ptr(ids), _ptr(h), _ptr(a), _ptr(ranks),
                                     _ptr(token_order), _ptr(slot_indptr), T, vocab, slots, R,
                                     num_slices, _ptr(err_flags), _stream(stream)))


def lora_apply_embedding(ids, y, a, b, ranks, scalings, token_order, slot_indptr, T, vocab,
                         slots, R, out_slices, regime=LORA_REGIME_AUTO, err_flags=None,
                         stream=None):
    _check(load().lora_apply_embedding(_ptr(ids), _ptr(y), _ptr(a), _ptr(b), _ptr(ranks),
                                       _ptr(scalings), _ptr(token_order), _ptr(slot_indptr), T,
                                       vocab, slots, R, _slices(out_slices), len(out_slices),
                                       regime, _ptr(err_flags), _stream(stream)))


def lora_expert_apply(x_sorted, y_sorted, a, b, pair_index, ranks, scalings, row_slot,
                      expert_offsets, rows_cap, in_features, num_experts, slots, num_pairs, R,
                      out_slices, workspace=None, workspace_bytes=0, err_flags=None,
                      stream=None):
    _check(load().lora_expert_apply(_ptr(x_sorted), _ptr(y_sorted), _ptr(a), _ptr(b),
                                    _ptr(pair_index), _ptr(ranks), _ptr(scalings),
                                    _ptr(row_slot), _ptr(expert_offsets), rows_cap, in_features,
                                    num_experts, slots, num_pairs, R, _slices(out_slices),
                                    len(out_slices), _ptr(workspace), workspace_bytes,
                                    _ptr(err_flags), _stream(stream)))


def lora_workspace_bytes(op, T, slots, R, num_slices, regime=LORA_REGIME_AUTO):
    return int(load().lora_workspace_bytes(op, T, slots, R, num_slices, regime))


def lora_resolve_regime(op, T, slots, R, num_slices):
    return int(load().lora_resolve_regime(op, T, slots, R, num_slices))


def lora_plan_tile(op, regime):
    return int(load().lora_plan_tile(op, regime))


def lora_plan_linear(slot_indptr, ranks, scalings, T, slots, R, tile, plan_out, plan_cap,
                     plan_count, err_flags=None, stream=None):
    _check(load().lora_plan_linear(_ptr(slot_indptr), _ptr(ranks), _ptr(scalings), T, slots, R,
                                   tile, _ptr(plan_out), plan_cap, _ptr(plan_count),
                                   _ptr(err_flags), _stream(stream)))


def lora_plan_expert(expert_offsets, pair_index, rows_cap, num_experts, slots, max_rows,
                     plan_out, plan_cap, plan_count, err_flags=None, stream=None):
    _check(load().lora_plan_expert(_ptr(expert_offsets), _ptr(pair_index), rows_cap,
                                   num_experts, slots, max_rows, _ptr(plan_out), plan_cap,
                                   _ptr(plan_count), _ptr(err_flags), _stream(stream)))


def lora_set_launch_overlap(enable):
    """Opt in or out of overlapping the fused few-tokens kernel's start with
    the preceding kernel in the stream; returns the previous setting."""
    return int(load().lora_set_launch_overlap(1 if enable else 0))


def lora_set_wait_limit_ns(ns):
    """Limit (ns) of the split kernel's bounded device waits; 0 = the default
    of one second.  Returns the previous setting."""
    return int(load().lora_set_wait_limit_ns(int(ns)))


def lora_version():
    return load().lora_version().decode()
