"""lora_apply_linear_noalloc: the fused shrink + expand for callers that cannot
hand the library device memory (a plugin inside a runtime that owns all device
memory, code that must not call cudaMalloc where it applies the delta).  It runs
on a scratch array compiled into the library instead of a caller workspace.

The GPU test calls it through the C ABI on the same inputs as lora_apply_linear
(the entry point that takes a workspace): the two must agree bit for bit, since
they run the same kernels, and both must match the fp64 oracle within the
parity tolerance used everywhere in these tests.  Consecutive calls share the
scratch.  This file is named so pytest collects it last.
"""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O


def _problems():
    # Shapes of the tensor-core regime and of the few-tokens split kernel (both
    # take scratch; the split kernel's counters must start at zero, which the
    # scratch does and every call leaves them) and a decode batch, each seeded;
    # shapes again after the scratch held another call's data.
    a = W.random_linear(301, 1500, 256, (136, 64), 3, 16, ranks=[16, 8, 12], dead_frac=0.05)
    b = W.random_linear(302, 1200, 128, (128, 128), 4, 64, ranks=[64, 16, 40, 32],
                        dead_frac=0.05)
    c = W.random_linear(303, 90, 512, (64, 32, 32), 5, 16, dead_frac=0.1)
    return [(a, L.LORA_REGIME_SGMV), (b, L.LORA_REGIME_SGMV), (c, L.LORA_REGIME_BGMV_SPLIT),
            (W.decode_qkv(4), L.LORA_REGIME_AUTO), (c, L.LORA_REGIME_BGMV_SPLIT),
            (a, L.LORA_REGIME_SGMV)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_and_oracle():
    from gpu_util import LinearDev, assert_close, host_bits, read_flags

    for p, regime in _problems():
        ref = LinearDev(p)
        ref.apply_linear(regime)                 # lora_apply_linear with a workspace
        got = LinearDev(p)
        L.lora_apply_linear_noalloc(got.x, got.y, got.a, got.b, got.ranks, got.scalings,
                                    got.token_order, got.slot_indptr, p.T, p.n_in, p.slots, p.R,
                                    p.out_slices, regime=regime, err_flags=got.flags)
        out = host_bits(got.y)
        assert np.array_equal(out, host_bits(ref.y)), f"{p.T} tokens, R={p.R}: not bit-exact"
        y_ref, _, flags = O.apply_linear(W.bf16_to_f64(p.x), W.bf16_to_f64(p.y),
                                         W.bf16_to_f64(p.a), W.bf16_to_f64(p.b), p.token_order,
                                         p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)
        assert_close(W.bf16_to_f64(out), y_ref, f"noalloc {p.T} tokens, R={p.R}")
        assert read_flags(got.flags) == read_flags(ref.flags) == flags == 0


@pytest.mark.gpu
def test_noalloc_sizes_scratch_for_the_regime_that_runs():
    """in_features < 64 keeps an AUTO call with many tokens per slot in the
    few-tokens regime (the tensor-core shrink needs 64): it needs no scratch and
    must be accepted, though the tensor-core workspace for these shapes would
    exceed the library's scratch."""
    from gpu_util import LinearDev, assert_close, host_bits, read_flags
    T, slots, R, S = 8192, 16, 64, 2
    assert L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, T, slots, R, S,
                                  L.LORA_REGIME_SGMV) > L.LORA_STATIC_SCRATCH_BYTES
    p = W.random_linear(304, T, 32, (64, 64), slots, R, ranks=[64, 32] * 8, dead_frac=0.02)
    got = LinearDev(p)
    L.lora_apply_linear_noalloc(got.x, got.y, got.a, got.b, got.ranks, got.scalings,
                                got.token_order, got.slot_indptr, p.T, p.n_in, p.slots, p.R,
                                p.out_slices, regime=L.LORA_REGIME_AUTO, err_flags=got.flags)
    y_ref, _, flags = O.apply_linear(W.bf16_to_f64(p.x), W.bf16_to_f64(p.y), W.bf16_to_f64(p.a),
                                     W.bf16_to_f64(p.b), p.token_order, p.slot_indptr, p.ranks,
                                     p.scalings, p.out_slices, p.R)
    assert_close(W.bf16_to_f64(host_bits(got.y)), y_ref, "noalloc in_features=32")
    assert read_flags(got.flags) == flags == 0


def test_noalloc_rejects_shapes_beyond_the_scratch():
    lib = L.load()
    fake = 1 << 20
    T, slots, R, S = 16384, 16, 64, 2
    need = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, T, slots, R, S, L.LORA_REGIME_SGMV)
    assert need > L.LORA_STATIC_SCRATCH_BYTES
    st = lib.lora_apply_linear_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, T, 4096,
                                       slots, R, L._slices((14336, 14336)), S,
                                       L.LORA_REGIME_SGMV, None, None)
    assert st == L.LORA_ERR_UNSUPPORTED
    assert "static scratch" in lib.lora_last_error().decode()
