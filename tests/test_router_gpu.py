"""GPU parity of the router LoRA fold (lora_apply_router) against the fp64
oracle: the routing logits take each token's router adapter delta before top-k
(spark_model/lora/expert_apply.rs, apply_router_lora).  Tolerance as for every
fold: |y_dev - y_ref| <= 1e-2 + 1.6e-2 |y_ref|; untouched rows bit-exact."""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import LinearDev, assert_close, assert_rows_bit_identical, host_bits, read_flags

pytestmark = pytest.mark.gpu

f64 = W.bf16_to_f64


def _oracle(p):
    return O.apply_router(f64(p.x), f64(p.y), f64(p.a), f64(p.b), p.token_order,
                          p.slot_indptr, p.ranks, p.scalings, p.R)


def _check(p, regime, what):
    d = LinearDev(p)
    d.apply_router(regime)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(p)
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, what)
    assert_rows_bit_identical(out, p.y, ~touched, what)
    return out


@pytest.mark.parametrize("regime", [pytest.param(L.LORA_REGIME_AUTO, id="auto"),
                                    pytest.param(L.LORA_REGIME_BGMV, id="bgmv"),
                                    pytest.param(L.LORA_REGIME_SGMV, id="sgmv")])
def test_router_workload_full(regime):
    """The MoE layer's router at full size: logits [2048, 128], hidden 2048,
    every element against the oracle."""
    p = W.moe_router(0)
    _check(p, regime, "moe_router")


ROUTER_SHAPES = [
    # T, hidden, num_experts, slots, R, dead_frac
    (8, 4096, 8, 2, 16, 0.0),          # a Mixtral-sized router: 8 experts
    (77, 2048, 64, 3, 16, 0.2),        # 64 experts, ragged token count
    (256, 7168, 256, 8, 16, 0.1),      # a 256-expert router on a wide hidden size
    (130, 1024, 160, 5, 8, 0.3),       # R = 8, 160 experts (ten 16-column tiles)
    (1100, 2048, 128, 4, 32, 0.0),     # enough tokens per slot for the SGMV regime
]


@pytest.mark.parametrize("shape", ROUTER_SHAPES)
def test_router_random_shapes(shape):
    T, hidden, E, slots, R, dead = shape
    p = W.random_linear(700 + T, T, hidden, (E,), slots, R, dead_frac=dead)
    _check(p, L.LORA_REGIME_AUTO, f"router {shape}")


def test_router_is_the_one_slice_linear_fold():
    """The router entry point runs the fused kernels with one slice of
    num_experts columns: bit-identical to lora_apply_linear on the same inputs."""
    p = W.moe_router(1)
    for regime in (L.LORA_REGIME_BGMV, L.LORA_REGIME_SGMV):
        d1, d2 = LinearDev(p), LinearDev(p)
        d1.apply_router(regime)
        d2.apply_linear(regime)
        assert np.array_equal(host_bits(d1.y), host_bits(d2.y))


def test_router_fold_changes_the_selection():
    """With a large scaling the delta decides some tokens' top-1 expert: the
    device logits give the oracle's selection wherever the oracle's top two are
    well apart (elsewhere both choices are within rounding of each other)."""
    p = W.moe_router(2)
    p.scalings = np.full(p.slots, 400.0, dtype=np.float32)
    out = _check(p, L.LORA_REGIME_AUTO, "router, large scaling")
    ref, _, _ = _oracle(p)
    base_top = np.argmax(f64(p.y), axis=1)
    ref_top = np.argmax(ref, axis=1)
    dev_top = np.argmax(f64(out), axis=1)
    srt = np.sort(ref, axis=1)
    clear = (srt[:, -1] - srt[:, -2]) > 0.1 + 0.05 * np.abs(srt[:, -1])
    assert (ref_top != base_top).mean() > 0.1
    assert np.array_equal(dev_top[clear], ref_top[clear])
