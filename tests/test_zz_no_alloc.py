"""lora_apply_linear_noalloc: the fused shrink + expand for callers that cannot
hand the library device memory (a plugin inside a runtime that owns all device
memory, code that must not call cudaMalloc where it applies the delta).  It runs
on a scratch array compiled into the library instead of a caller workspace.

The GPU test compares it, through the C ABI, with lora_apply_linear (the entry
point that takes a workspace) on the same inputs, within the parity tolerance
used everywhere in these tests, over consecutive calls that share the scratch.
This file is named so pytest collects it last.
"""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O


def _problems():
    # Shapes of the tensor-core regime (it needs scratch), then one of the
    # cluster regime (it needs none), each seeded.
    a = W.random_linear(301, 1500, 256, (136, 64), 3, 16, ranks=[16, 8, 12], dead_frac=0.05)
    b = W.random_linear(302, 1200, 128, (128, 128), 4, 64, ranks=[64, 16, 40, 32],
                        dead_frac=0.05)
    c = W.random_linear(303, 90, 512, (64, 32, 32), 5, 16, dead_frac=0.1)
    return [(a, L.LORA_REGIME_SGMV), (b, L.LORA_REGIME_SGMV), (c, L.LORA_REGIME_BGMV),
            (a, L.LORA_REGIME_SGMV)]


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point():
    from gpu_util import LinearDev, host_bits, read_flags

    for p, regime in _problems():
        ref = LinearDev(p)
        ref.apply_linear(regime)                 # lora_apply_linear with a workspace
        got = LinearDev(p)
        L.lora_apply_linear_noalloc(got.x, got.y, got.a, got.b, got.ranks, got.scalings,
                                    got.token_order, got.slot_indptr, p.T, p.n_in, p.slots, p.R,
                                    p.out_slices, regime=regime, err_flags=got.flags)
        y_ref = W.bf16_to_f64(host_bits(ref.y))
        y_got = W.bf16_to_f64(host_bits(got.y))
        ok = O.within_tolerance(y_got, y_ref) | (np.isnan(y_got) & np.isnan(y_ref))
        assert ok.all(), f"{p.T} tokens, R={p.R}: {np.count_nonzero(~ok)} elements differ"
        assert read_flags(got.flags) == read_flags(ref.flags) == 0


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
