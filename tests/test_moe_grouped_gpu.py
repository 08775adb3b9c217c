"""GPU parity of the MoE expert fold grouped by (slot, expert): with a
workspace, lora_expert_apply sorts each adapted expert's rows by slot on the
device and runs the tensor-core shrink and expand over the groups.  Checked
against the fp64 oracle's per-expert loop: |y_dev - y_ref| <= 1e-2 +
1.6e-2 |y_ref|, untouched rows and flags bit-exact."""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import MoEDev, assert_close, assert_rows_bit_identical, host_bits, read_flags

pytestmark = pytest.mark.gpu

f64 = W.bf16_to_f64


def _oracle(m, y_bits=None, **kw):
    fields = {**m.__dict__, **kw}
    y = m.y if y_bits is None else y_bits
    return O.expert_apply(f64(m.x), f64(y), f64(m.a), f64(m.b), fields["pair_index"],
                          fields["ranks"], fields["scalings"], fields["row_slot"],
                          fields["expert_offsets"], m.R, m.out_slices, m.slots, m.num_experts,
                          m.num_pairs)


def _check(m, y_bits=None, what="moe grouped"):
    d = MoEDev(m, y_bits)
    d.apply(grouped=True)
    y_in = m.y if y_bits is None else y_bits
    y_ref, touched, flags = _oracle(m, y_bits)
    out = host_bits(d.y)
    assert read_flags(d.flags) == flags
    assert_close(f64(out), y_ref, what)
    assert_rows_bit_identical(out, y_in, ~touched, what + " untouched")
    return out


def test_workload_moe_full_grouped():
    """Both folds of the MoE layer (gate/up 2048 -> 768+768, down 768 -> 2048,
    16384 sorted rows, 128 experts) at full size, every element."""
    gu, dn = W.moe_expert(0)
    for m in (gu, dn):
        _check(m, what=m.name)
        _check(m, y_bits=np.zeros_like(m.y), what=m.name + " y=0")


SHAPES = [
    # rows per expert max, experts, in, out_slices, slots, R, ranks
    (40, 9, 136, (24, 32), 3, 16, None),          # ragged experts, two slices
    (300, 5, 256, (128,), 4, 32, [32, 16, 0, 32]),  # a rank-0 slot, R = 32, big groups
    (150, 12, 64, (64,), 2, 64, [64, 48]),        # R = 64, rank below R
    (7, 40, 512, (16, 16, 16, 16), 5, 16, None),  # many small experts, four slices
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("seed", [0, 1])
def test_moe_grouped_random(shape, seed):
    rmax, E, n_in, outs, slots, R, ranks = shape
    m = W.random_moe(60 + seed + 10 * E, rmax, E, n_in, outs, slots, R, ranks=ranks)
    _check(m, what=f"moe grouped {shape}")


def test_moe_grouped_bad_rows_flagged():
    m = W.random_moe(31, 20, 6, 64, (16,), 3, 16, ranks=[16, 16, 16])
    rs = m.row_slot.copy()
    rs[::7] = 9                                  # slot out of range
    pi = m.pair_index.copy()
    idx = np.nonzero(m.pair_index >= 0)[0][:2]
    pi[idx] = m.num_pairs + 4                    # pair out of range
    ranks = m.ranks.copy()
    ranks[2] = 17                                # rank above R
    q = W.MoEProblem(**{**m.__dict__, "row_slot": rs, "pair_index": pi, "ranks": ranks})
    _check(q, what="moe grouped flags")
    _, _, flags = _oracle(q)
    assert flags == O.FLAG_BAD_SLOT | O.FLAG_BAD_PAIR | O.FLAG_BAD_RANK


def test_moe_grouped_bad_offsets_skip_the_expert():
    """Malformed offsets of the first and the last expert (start < 0, end past
    rows_cap) skip those experts and raise the flag; the others fold."""
    m = W.random_moe(32, 30, 8, 128, (32,), 2, 16, ranks=[16, 16], adapted_frac=1.0)
    off = m.expert_offsets.copy()
    off[0] = -3
    off[-1] = m.rows_cap + 2
    q = W.MoEProblem(**{**m.__dict__, "expert_offsets": off})
    _check(q, what="moe grouped offsets")
    _, _, flags = _oracle(q)
    assert flags & O.FLAG_BAD_OFFSETS


def test_moe_grouped_rerun_bit_exact():
    """Rows land in their group in no fixed order; every row's fold is
    independent of its place, so reruns give identical bits."""
    gu, _ = W.moe_expert(1)
    first = _check(gu)
    d = MoEDev(gu)
    d.apply(grouped=True)
    assert np.array_equal(host_bits(d.y), first)


def test_moe_too_many_groups_falls_back():
    """slots * num_experts above the grouped fold's table: the workspace is
    left unused and the per-chunk kernel runs (same results within tolerance)."""
    m = W.random_moe(33, 3, 1100, 64, (16,), 4, 16, ranks=[16, 8, 16, 16], adapted_frac=0.05)
    _check(m, what="moe fallback")
