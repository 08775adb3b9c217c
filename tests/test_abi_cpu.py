"""The C-ABI library on a host without a GPU: it loads, exports every symbol the
header declares, and rejects host-checkable mistakes before any CUDA call."""
import os
import re

import pytest

from adapter_lora_serving_b200 import lora as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_delta.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(L.LIB_PATH):
        from adapter_lora_serving_b200 import build
        build.build()
    return L.load()


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lora_[a-z_]+)\s*\(", txt)))


def test_header_symbols_exported(lib):
    declared = _declared()
    assert "lora_apply_linear" in declared and "lora_expert_apply" in declared
    for name in declared:
        assert hasattr(lib, name), name
    assert sorted(L.EXPORTED) == declared


def test_version(lib):
    assert "sm_100a" in L.lora_version()


FAKE = 1 << 20          # a 16-byte aligned, never dereferenced address


def _apply(lib, **kw):
    args = dict(x=FAKE, y=FAKE, a=FAKE, b=FAKE, ranks=FAKE, scalings=FAKE, token_order=FAKE,
                slot_indptr=FAKE, T=16, in_features=64, slots=2, R=16, out_slices=(32,),
                regime=L.LORA_REGIME_BGMV, ws=None, ws_bytes=0, flags=None)
    args.update(kw)
    sl = L._slices(args["out_slices"])
    return lib.lora_apply_linear(args["x"], args["y"], args["a"], args["b"], args["ranks"],
                                 args["scalings"], args["token_order"], args["slot_indptr"],
                                 args["T"], args["in_features"], args["slots"], args["R"], sl,
                                 len(args["out_slices"]), args["regime"], args["ws"],
                                 args["ws_bytes"], args["flags"], None)


@pytest.mark.parametrize("kw", [
    dict(R=12),                       # not a multiple of 8
    dict(R=0),
    dict(in_features=60),
    dict(out_slices=(20,)),
    dict(out_slices=()),
    dict(out_slices=(8,) * 9),        # more than LORA_MAX_SLICES
    dict(T=-1),
    dict(slots=-2),
    dict(x=None),
    dict(x=FAKE + 8),                 # not 16-byte aligned
    dict(ranks=FAKE + 2),             # not 4-byte aligned
    dict(flags=FAKE + 1),
])
def test_apply_linear_rejects(lib, kw):
    assert _apply(lib, **kw) == L.LORA_ERR_INVALID
    assert lib.lora_last_error().decode().startswith("lora_apply_linear")


def test_limits_unsupported(lib):
    assert _apply(lib, slots=5000) == L.LORA_ERR_UNSUPPORTED
    # 3 slices of R=128 exceed the BGMV shared-memory tile
    assert _apply(lib, R=128, out_slices=(8, 8, 8)) == L.LORA_ERR_UNSUPPORTED


def test_empty_calls_launch_nothing(lib):
    assert _apply(lib, T=0) == L.LORA_OK
    assert _apply(lib, slots=0) == L.LORA_OK


def test_other_entry_points_validate(lib):
    sl = L._slices((16,))
    assert lib.lora_expand(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 2, 10, sl, 1, 0, None,
                           None) == L.LORA_ERR_INVALID
    assert lib.lora_shrink(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 12, 2, 8, 1, 0, None,
                           None) == L.LORA_ERR_INVALID
    assert lib.lora_gather_shrink(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, 0, 2, 8, 1, None,
                                  None) == L.LORA_ERR_INVALID
    assert lib.lora_apply_embedding(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 8, -5, 2, 8,
                                    sl, 1, 0, None, None) == L.LORA_ERR_INVALID
    assert lib.lora_expert_apply(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 64,
                                 -1, 2, 4, 8, sl, 1, None, 0, None, None) == L.LORA_ERR_INVALID
    assert lib.lora_expert_apply(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, 64,
                                 5000, 2, 4, 8, sl, 1, None, 0, None,
                                 None) == L.LORA_ERR_UNSUPPORTED
    assert lib.lora_plan_linear(FAKE, FAKE, None, 8, 2, 8, 0, FAKE, 4, FAKE, None,
                                None) == L.LORA_ERR_INVALID
    assert lib.lora_plan_expert(FAKE, FAKE, 8, 2, 2, 0, FAKE, 4, FAKE, None,
                                None) == L.LORA_ERR_INVALID


def test_router_validates(lib):
    # router_in, gate_logits, a, b, ranks, scalings, token_order, slot_indptr,
    # T, hidden, slots, R, num_experts, regime, workspace, bytes, flags, stream
    def router(**kw):
        args = dict(T=16, hidden=64, slots=2, R=16, num_experts=64)
        args.update(kw)
        return lib.lora_apply_router(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, args["T"],
                                     args["hidden"], args["slots"], args["R"],
                                     args["num_experts"], L.LORA_REGIME_BGMV, None, 0, None,
                                     None)
    assert router(num_experts=60) == L.LORA_ERR_INVALID
    assert "num_experts" in lib.lora_last_error().decode()
    assert router(num_experts=0) == L.LORA_ERR_INVALID
    assert router(hidden=100) == L.LORA_ERR_INVALID
    assert lib.lora_last_error().decode().startswith("lora_apply_router")
    assert router(R=12) == L.LORA_ERR_INVALID
    assert router(T=0) == L.LORA_OK


def test_status_strings(lib):
    for code, name in [(0, "LORA_OK"), (1, "LORA_ERR_INVALID"), (2, "LORA_ERR_UNSUPPORTED"),
                       (3, "LORA_ERR_WORKSPACE"), (4, "LORA_ERR_CUDA")]:
        assert lib.lora_status_string(code).decode() == name


def test_host_queries(lib):
    assert L.lora_plan_tile(L.LORA_OP_APPLY_LINEAR, L.LORA_REGIME_BGMV) == 32
    assert L.lora_plan_tile(L.LORA_OP_EXPERT_APPLY, L.LORA_REGIME_AUTO) == 32
    # the cluster kernel keeps h on chip
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 256, 32, 16, 3,
                                  L.LORA_REGIME_BGMV) == 0
    # the split kernel: 4096 bytes of counters, then one fp32 partial h tile of
    # 32 tokens x S*R per (work item, CTA) pair: at most min(T, slots) +
    # ceil(T/32) items, 256 CTAs
    items = min(256, 32) + 256 // 32
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 256, 32, 16, 3,
                                  L.LORA_REGIME_BGMV_SPLIT) == \
        4096 + (items + 256) * 32 * 3 * 16 * 4
    # beyond its limits it takes nothing (the call is refused)
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 2000, 64, 16, 3,
                                  L.LORA_REGIME_BGMV_SPLIT) == 0
    # SGMV: the counter header, then up to four fp32 partial h buffers
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 8192, 16, 64, 2,
                                  L.LORA_REGIME_SGMV) == 4096 + 4 * 8192 * 64 * 2 * 4
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_LINEAR, 256, 32, 16, 3) == L.LORA_REGIME_BGMV
    # the embedding streams its output rows under AUTO (R up to 64)
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_EMBEDDING, 4096, 8, 16, 1) == \
        L.LORA_REGIME_STREAM
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_EMBEDDING, 64, 8, 64, 2) == \
        L.LORA_REGIME_STREAM
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_EMBEDDING, 64, 8, 72, 1) != \
        L.LORA_REGIME_STREAM
    assert L.lora_plan_tile(L.LORA_OP_APPLY_EMBEDDING, L.LORA_REGIME_STREAM) == 16
    assert L.lora_plan_tile(L.LORA_OP_APPLY_LINEAR, L.LORA_REGIME_STREAM) == 16
    # the fused apply in STREAM: the counter header, then one fp32 partial h
    # per 512 input features, sized for in_features = 4096
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 256, 32, 16, 3,
                                  L.LORA_REGIME_STREAM) == 4096 + 8 * 256 * 3 * 16 * 4
    # AUTO streams 512 <= T <= 8192 with T * in_features <= 2^25 when the
    # workspace holds it: lora_workspace_bytes covers eight partial buffers
    # there (more than SGMV's four), nothing below T = 512, and SGMV's beyond
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 1024, 4, 16, 1) == \
        4096 + 8 * 1024 * 16 * 4
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 8192, 4, 16, 1) == \
        4096 + 8 * 8192 * 16 * 4
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 512, 8, 16, 3) == \
        4096 + 8 * 512 * 3 * 16 * 4
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 256, 32, 16, 3) == 0
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, 16384, 4, 16, 1) == \
        4096 + 4 * 16384 * 16 * 4
    # lora_resolve_regime does not know in_features: SGMV's shapes answer SGMV
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_LINEAR, 2048, 4, 16, 1) == L.LORA_REGIME_SGMV
    # the grouped expert fold: token_order, the group tables (4096 groups x 4
    # ints), then eight fp32 partial h buffers; nothing for the per-chunk kernel
    rows, R, S = 16384, 16, 2
    assert L.lora_workspace_bytes(L.LORA_OP_EXPERT_APPLY, rows, 128, R, S) == \
        rows * 4 + 4 * 4096 * 4 + 8 * rows * R * S * 4
    assert L.lora_workspace_bytes(L.LORA_OP_EXPERT_APPLY, rows, 128, R, S,
                                  L.LORA_REGIME_BGMV) == 0
    assert L.lora_workspace_bytes(L.LORA_OP_EXPERT_APPLY, rows, 128, 8, 1) == 0


def test_wait_limit_setting_roundtrip(lib):
    # a process-wide setting: returns the previous value, launches nothing
    prev = L.lora_set_wait_limit_ns(5_000_000)
    assert L.lora_set_wait_limit_ns(0) == 5_000_000
    assert L.lora_set_wait_limit_ns(prev) == 0


def test_launch_overlap_setting_roundtrip(lib):
    # a process-wide flag: returns the previous setting, launches nothing
    prev = L.lora_set_launch_overlap(1)
    assert L.lora_set_launch_overlap(0) == 1
    assert L.lora_set_launch_overlap(prev) == 0


def test_split_regime_refuses_shapes_beyond_its_limits(lib):
    # 2000 tokens is past the split kernel's token limit: refused before launch
    ws = 1 << 20
    assert _apply(lib, T=2000, regime=L.LORA_REGIME_BGMV_SPLIT, ws=ws, ws_bytes=1 << 30) == \
        L.LORA_ERR_UNSUPPORTED
    assert "BGMV_SPLIT" in lib.lora_last_error().decode()
    # within its limits but without a workspace: refused before launch
    assert _apply(lib, regime=L.LORA_REGIME_BGMV_SPLIT) == L.LORA_ERR_WORKSPACE


def test_stream_regime_refuses_before_launch(lib):
    S = L.LORA_REGIME_STREAM
    ws = 1 << 20
    # S*R outside {16, 32, 48, 64}, or in_features past 4096: unsupported
    assert _apply(lib, R=32, out_slices=(32, 32, 32), regime=S, ws=ws, ws_bytes=1 << 30) == \
        L.LORA_ERR_UNSUPPORTED
    assert "STREAM" in lib.lora_last_error().decode()
    assert _apply(lib, in_features=4104, regime=S, ws=ws, ws_bytes=1 << 30) == \
        L.LORA_ERR_UNSUPPORTED
    # the counter header and one chunk of partials are needed: one byte short
    need = 4096 + 4 * 16 * 16
    assert _apply(lib, regime=S, ws=ws, ws_bytes=need - 1) == L.LORA_ERR_WORKSPACE
    assert _apply(lib, regime=S) == L.LORA_ERR_WORKSPACE
    # a workspace that is not 16-byte aligned
    assert _apply(lib, regime=S, ws=ws + 4, ws_bytes=need) == L.LORA_ERR_INVALID
