"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle on the
same seeded inputs.  Tolerance for floating point: |y_dev - y_ref| <=
1e-2 + 1.6e-2 |y_ref| elementwise; untouched rows, plans and flags bit-exact."""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import (LinearDev, MoEDev, assert_close, assert_rows_bit_identical, dev_i32,
                      dev_f32, host_bits, host_f64, read_flags, torch)

pytestmark = pytest.mark.gpu

class Path:
    """A kernel path of lora_apply_linear: the regime hint, and whether the call
    gets the workspace lora_workspace_bytes asks for."""

    def __init__(self, regime, workspace):
        self.regime = regime
        self.workspace = workspace

    def __eq__(self, other):        # compares as its regime
        return self.regime == (other.regime if isinstance(other, Path) else other)

    def __int__(self):
        return self.regime


SPLIT = Path(L.LORA_REGIME_BGMV_SPLIT, True)
CLUSTER = Path(L.LORA_REGIME_BGMV, True)
SGMV = Path(L.LORA_REGIME_SGMV, True)
REGIMES = [pytest.param(SPLIT, id="bgmv_split"),
           pytest.param(CLUSTER, id="bgmv_cluster"),
           pytest.param(SGMV, id="sgmv")]


def _apply(d, path, **kw):
    path = path if isinstance(path, Path) else Path(path, True)
    d.apply_linear(path.regime, use_workspace=path.workspace, **kw)


def split_takes(p):
    """The shapes the BGMV_SPLIT kernel takes (it refuses the others)."""
    items = min(p.T, p.slots) + -(-p.T // 32)
    return (p.T <= 1024 and p.slots <= 1024 and items <= 512 and p.n_in <= 65536 and
            p.out <= 262144 and p.num_slices * (-(-p.R // 16) * 16) <= 128)


def _skip_unsupported(p, regime, shrink=True):
    """The SGMV kernels take R in {16, 32, 64}, num_slices * R <= 128 and (for the
    shrink) in_features >= 64; the BGMV_SPLIT kernel the shapes of split_takes;
    other shapes are the BGMV regime's."""
    if int(regime) == L.LORA_REGIME_BGMV_SPLIT:
        if not split_takes(p):
            pytest.skip("shape outside the BGMV_SPLIT kernel's limits")
        return
    if int(regime) != L.LORA_REGIME_SGMV:
        return
    if p.R not in (16, 32, 64) or p.num_slices * p.R > 128:
        pytest.skip("shape outside the SGMV regime")
    if shrink and p.n_in < 64:
        pytest.skip("in_features < 64 is outside the SGMV shrink")


def _f64(bits):
    return W.bf16_to_f64(bits)


def _oracle_linear(p, y_bits=None, token_order=None):
    y = _f64(p.y if y_bits is None else y_bits)
    return O.apply_linear(_f64(p.x), y, _f64(p.a), _f64(p.b),
                          p.token_order if token_order is None else token_order,
                          p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)


def _check_linear(p, regime, y_bits=None, what=""):
    _skip_unsupported(p, regime)
    d = LinearDev(p, y_bits)
    _apply(d, regime)
    y_in = p.y if y_bits is None else y_bits
    out = host_bits(d.y)
    y_ref, touched, flags = _oracle_linear(p, y_in)
    assert read_flags(d.flags) == flags
    assert_close(_f64(out), y_ref, what)
    assert_rows_bit_identical(out, y_in, ~touched, what)
    return out


# ---------------------------------------------------------------------------
# Linear target
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("regime", REGIMES)
def test_tiny_linear(regime):
    p = W.tiny_linear(0)
    out = _check_linear(p, regime, what="tiny")
    # slot 0 has rank 0: its tokens are bit-identical
    assert_rows_bit_identical(out, p.y, p.slot_of == 0, "rank-0 slot")


SHAPES = [
    # T, in, out_slices, slots, R, dead_frac
    (37, 24, (8,), 3, 8, 0.2),              # in not a multiple of the stage width
    (100, 200, (48, 16), 3, 16, 0.1),       # several tiles per slot, ragged tails
    (64, 512, (64, 32, 32), 4, 16, 0.0),    # three slices
    (50, 1032, (136,), 5, 32, 0.3),         # R=32, k split ragged across the cluster
    (33, 256, (128, 128), 2, 64, 0.0),      # R=64, two slices
    (300, 64, (8, 8, 8), 7, 8, 0.5),        # many sparse slots
    (90, 128, (24, 40, 8), 3, 16, 0.1),     # 16-column tiles straddling slice edges
]


@pytest.mark.parametrize("regime", REGIMES)
@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("seed", [0, 1])
def test_random_linear(regime, shape, seed):
    T, n_in, outs, slots, R, dead = shape
    p = W.random_linear(100 + seed, T, n_in, outs, slots, R, dead_frac=dead)
    _check_linear(p, regime, what=f"{shape}")


LIMIT_SHAPES = [
    # T, in, out_slices, slots, R, ranks
    (40, 64, (8,) * 8, 3, 16, [16, 9, 1]),     # eight slices (the limit), ranks not a multiple of 4
    (48, 96, (32,), 2, 128, [128, 72]),         # R = 128 in one slice: 8 k-steps per expand tile
    (70, 136, (16, 24), 4, 8, [8, 0, 5, 8]),    # R = 8 (half a k-step), a rank-0 slot
]


@pytest.mark.parametrize("shape", LIMIT_SHAPES)
def test_limit_shapes_bgmv(shape):
    """The BGMV regime at its shape limits (num_slices * roundup(R, 16) = 128),
    with ranks that end inside a group of four columns."""
    T, n_in, outs, slots, R, ranks = shape
    p = W.random_linear(500, T, n_in, outs, slots, R, ranks=ranks, dead_frac=0.1)
    _check_linear(p, L.LORA_REGIME_BGMV, what=f"{shape}")


@pytest.mark.parametrize("regime", REGIMES)
def test_max_slots(regime):
    """LORA_MAX_SLOTS slots (the planner's largest prefix and item caches),
    most of them empty, a few hundred tokens spread over the rest."""
    p = W.random_linear(600, 300, 64, (16, 32), 4096, 16, dead_frac=0.1)
    _check_linear(p, regime, what="4096 slots")


SGMV_SHAPES = [
    # T, in, out_slices, slots, R, ranks
    (700, 256, (136, 64), 3, 16, [16, 8, 12]),       # 3+ tiles per slot, ragged chunks
    (520, 192, (256,), 2, 32, [32, 20]),            # R=32 (64-byte rows)
    (400, 128, (128, 128), 3, 64, [64, 16, 40]),    # R=64, two slices
    (300, 64, (24, 40, 8), 2, 16, [16, 16]),        # chunks straddling slice edges
]


@pytest.mark.parametrize("regime", REGIMES)
@pytest.mark.parametrize("shape", SGMV_SHAPES)
def test_tile_shapes(regime, shape):
    T, n_in, outs, slots, R, ranks = shape
    p = W.random_linear(200 + T, T, n_in, outs, slots, R, ranks=ranks, dead_frac=0.05)
    _check_linear(p, regime, what=f"{shape}")
    _check_linear(p, regime, y_bits=np.zeros_like(p.y), what=f"{shape} y=0")


@pytest.mark.parametrize("regime", REGIMES)
def test_delta_visible_with_zero_y(regime):
    for p in (W.tiny_linear(1), W.random_linear(7, 80, 256, (32, 16), 4, 16, dead_frac=0.1)):
        zero = np.zeros_like(p.y)
        _check_linear(p, regime, y_bits=zero, what=f"{p.name} y=0")


@pytest.mark.parametrize("regime", REGIMES)
def test_noops_bit_exact_and_poison_ignored(regime):
    p = W.random_linear(11, 90, 128, (16, 16), 5, 16, ranks=[0, 8, 16, 5, 16],
                        scalings=[1.0, 0.0, 0.5, 2.0, 1.0], dead_frac=0.2)
    _skip_unsupported(p, regime)
    y = p.y.copy()
    y[:, 0] = 0x8000          # -0.0
    y[:, 1] = 0x7FC1          # NaN payload
    clean = _check_linear(p, regime, y_bits=y, what="noops")
    for s in (0, 1):
        assert_rows_bit_identical(clean, y, p.slot_of == s, f"slot {s}")
    assert_rows_bit_identical(clean, y, p.slot_of == -1, "dead tokens")
    # NaN in A rows and B columns past each slot's rank must not matter
    a = p.a.copy()
    b = p.b.copy()
    for s, r in enumerate(p.ranks):
        a[s, [i * p.R + q for i in range(p.num_slices) for q in range(r, p.R)], :] = 0x7FC0
        b[s, :, r:] = 0x7FC0
    p2 = W.LinearProblem(**{**p.__dict__, "a": a, "b": b})
    d = LinearDev(p2, y)
    _apply(d, regime)
    assert np.array_equal(host_bits(d.y), clean)


@pytest.mark.parametrize("regime", REGIMES)
def test_position_permutation_and_rerun_bit_exact(regime):
    p = W.random_linear(12, 120, 256, (32,), 3, 16, ranks=[16, 8, 16])
    _skip_unsupported(p, regime)
    d = LinearDev(p)
    _apply(d, regime)
    first = host_bits(d.y)
    d2 = LinearDev(p)
    _apply(d2, regime)
    assert np.array_equal(host_bits(d2.y), first)
    rng = np.random.default_rng(3)
    to = p.token_order.copy()
    for s in range(p.slots):
        lo, hi = p.slot_indptr[s], p.slot_indptr[s + 1]
        to[lo:hi] = rng.permutation(to[lo:hi])
    d3 = LinearDev(W.LinearProblem(**{**p.__dict__, "token_order": to}))
    _apply(d3, regime)
    assert np.array_equal(host_bits(d3.y), first)


@pytest.mark.parametrize("regime", REGIMES)
def test_shrink_and_expand(regime):
    t = torch()
    p = W.random_linear(13, 70, 320, (24, 40), 4, 16, ranks=[16, 8, 0, 12], dead_frac=0.1)
    _skip_unsupported(p, regime)
    d = LinearDev(p)
    SR = p.num_slices * p.R
    h = t.full((p.T, SR), float("nan"), dtype=t.float32, device="cuda")
    d.shrink(h, min(int(regime), L.LORA_REGIME_SGMV))
    h_dev = h.cpu().numpy().astype(np.float64)
    h_ref, mask, flags = O.shrink(_f64(p.x), _f64(p.a), p.token_order, p.slot_indptr, p.ranks,
                                  p.R, p.num_slices)
    assert read_flags(d.flags) == flags
    bound = 1e-5 + 1e-3 * np.abs(_f64(p.x)) @ np.abs(_f64(p.a)).reshape(-1, p.n_in).T
    bound = bound.reshape(p.T, p.slots, SR)[np.arange(p.T), np.maximum(p.slot_of, 0)]
    assert np.all(np.abs(h_dev[mask] - h_ref[mask]) <= bound[mask])
    assert np.all(np.isnan(h_dev[~mask]))      # nothing else written
    # expand from an fp32 h
    h32 = np.where(mask, h_ref, 0.0).astype(np.float32)
    h_in = t.from_numpy(h32).cuda()
    d.expand(h_in, min(int(regime), L.LORA_REGIME_SGMV))
    y_ref, touched, f2 = O.expand(_f64(p.y), h32.astype(np.float64), _f64(p.b), p.token_order,
                                  p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)
    out = host_bits(d.y)
    assert_close(_f64(out), y_ref, "expand")
    assert_rows_bit_identical(out, p.y, ~touched, "expand untouched")


# ---------------------------------------------------------------------------
# Embedding target
# ---------------------------------------------------------------------------

def test_gather_shrink_exact():
    t = torch()
    p = W.random_linear(14, 77, None, (16,), 3, 16, ranks=[16, 8, 0], embedding_vocab=1000,
                        bad_id_frac=0.1, dead_frac=0.1)
    d = LinearDev(p)
    h = t.full((p.T, p.R), float("nan"), dtype=t.float32, device="cuda")
    d.gather_shrink(h)
    h_ref, mask, flags = O.gather_shrink(p.ids, _f64(p.a), p.token_order, p.slot_indptr,
                                         p.ranks, p.R, 1, p.n_in)
    h_dev = h.cpu().numpy().astype(np.float64)
    assert read_flags(d.flags) == flags
    assert np.array_equal(h_dev[mask], h_ref[mask])
    assert np.all(np.isnan(h_dev[~mask]))


@pytest.mark.parametrize("regime", REGIMES)
@pytest.mark.parametrize("seed", [0, 1])
def test_apply_embedding(regime, seed):
    p = W.random_linear(15 + seed, 150, None, (64, 32), 5, 16, embedding_vocab=3000,
                        bad_id_frac=0.1, dead_frac=0.05)
    _skip_unsupported(p, regime, shrink=False)
    d = LinearDev(p)
    d.apply_embedding(min(int(regime), L.LORA_REGIME_SGMV))
    y_ref, touched, flags = O.apply_embedding(p.ids, _f64(p.y), _f64(p.a), _f64(p.b),
                                              p.token_order, p.slot_indptr, p.ranks, p.scalings,
                                              p.out_slices, p.R, p.n_in)
    out = host_bits(d.y)
    assert read_flags(d.flags) == flags
    assert_close(_f64(out), y_ref, "embedding")
    assert_rows_bit_identical(out, p.y, ~touched, "embedding untouched")
    zero = np.zeros_like(p.y)
    d0 = LinearDev(p, zero)
    d0.apply_embedding(min(int(regime), L.LORA_REGIME_SGMV))
    y0, _, _ = O.apply_embedding(p.ids, _f64(zero), _f64(p.a), _f64(p.b), p.token_order,
                                 p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R, p.n_in)
    assert_close(_f64(host_bits(d0.y)), y0, "embedding y=0")


# ---------------------------------------------------------------------------
# Addressing: plans and flags
# ---------------------------------------------------------------------------

def _plan_linear_dev(indptr, ranks, scalings, T, R, tile, cap=4096):
    t = torch()
    out = t.full((cap * 3,), -7, dtype=t.int32, device="cuda")
    cnt = t.zeros(1, dtype=t.int32, device="cuda")
    fl = t.zeros(1, dtype=t.int32, device="cuda")
    L.lora_plan_linear(dev_i32(indptr), dev_i32(ranks),
                       None if scalings is None else dev_f32(scalings), T, len(indptr) - 1, R,
                       tile, out, cap, cnt, err_flags=fl)
    n = int(cnt.item())
    items = out.cpu().numpy()[:3 * min(n, cap)].reshape(-1, 3)
    return [tuple(int(v) for v in r) for r in items], n, read_flags(fl)


@pytest.mark.parametrize("tile", [1, 5, 16, 128])
def test_plan_linear_bit_exact(tile):
    p = W.decode_qkv(0)
    for scal in (None, p.scalings):
        items, n, fl = _plan_linear_dev(p.slot_indptr, p.ranks, scal, p.T, p.R, tile)
        ref = O.plan_segments(p.slot_indptr, p.ranks, p.T, p.R, tile, scalings=scal)
        assert n == len(ref) and items == ref and fl == 0
    # malformed segments and ranks
    indptr = [0, 5, 3, 9, 9, 20]
    ranks = [8, 8, 8, 17, 8]
    items, n, fl = _plan_linear_dev(indptr, ranks, None, 12, 16, tile)
    assert items == O.plan_segments(indptr, ranks, 12, 16, tile)
    assert fl == O.FLAG_BAD_INDPTR | O.FLAG_BAD_RANK


def test_plan_expert_bit_exact():
    t = torch()
    gu, _ = W.moe_expert(0)
    cases = [(gu.expert_offsets, gu.pair_index, gu.rows_cap, gu.num_experts, gu.slots)]
    bad_off = gu.expert_offsets.copy()
    bad_off[5] = bad_off[7] + 3              # expert 4 ends after expert 5 starts: malformed
    cases.append((bad_off, gu.pair_index, gu.rows_cap, gu.num_experts, gu.slots))
    for off, pi, rows_cap, E, slots in cases:
        for tile in (16, 128):
            out = t.full((8192 * 3,), -7, dtype=t.int32, device="cuda")
            cnt = t.zeros(1, dtype=t.int32, device="cuda")
            fl = t.zeros(1, dtype=t.int32, device="cuda")
            L.lora_plan_expert(dev_i32(off), dev_i32(pi), rows_cap, E, slots, tile, out, 8192,
                               cnt, err_flags=fl)
            n = int(cnt.item())
            items = [tuple(int(v) for v in r) for r in out.cpu().numpy()[:3 * n].reshape(-1, 3)]
            ref, rflags = O.plan_expert(off, pi, slots, E, rows_cap, tile)
            assert items == ref
            assert read_flags(fl) == rflags


@pytest.mark.parametrize("regime", REGIMES)
def test_bad_addressing_flags(regime):
    p = W.random_linear(16, 40, 64, (16,), 4, 16, ranks=[16, 16, 16, 16])
    to = p.token_order.copy()
    indptr = p.slot_indptr.copy()
    ranks = p.ranks.copy()
    to[indptr[0]] = 1000                     # bad token in slot 0
    ranks[2] = 17                            # rank > R
    indptr[3] = indptr[4] + 1                # slot 3: lo > hi
    q = W.LinearProblem(**{**p.__dict__, "token_order": to, "slot_indptr": indptr,
                           "ranks": ranks})
    _skip_unsupported(q, regime)
    d = LinearDev(q)
    _apply(d, regime)
    y_ref, touched, flags = O.apply_linear(_f64(q.x), _f64(q.y), _f64(q.a), _f64(q.b), to,
                                           indptr, ranks, q.scalings, q.out_slices, q.R)
    out = host_bits(d.y)
    assert read_flags(d.flags) == flags
    assert flags == O.FLAG_BAD_TOKEN | O.FLAG_BAD_RANK | O.FLAG_BAD_INDPTR
    assert_close(_f64(out), y_ref, "bad addressing")
    assert_rows_bit_identical(out, q.y, ~touched, "bad addressing untouched")


def test_empty_and_zero_token_calls():
    p = W.random_linear(17, 16, 64, (16,), 2, 8, slot_of=np.full(16, -1))
    d = LinearDev(p)
    d.apply_linear(L.LORA_REGIME_BGMV)
    assert np.array_equal(host_bits(d.y), p.y)


# ---------------------------------------------------------------------------
# MoE expert fold
# ---------------------------------------------------------------------------

def _check_moe(m, y_bits=None, what="moe"):
    d = MoEDev(m, y_bits)
    d.apply()
    y_in = m.y if y_bits is None else y_bits
    y_ref, touched, flags = O.expert_apply(_f64(m.x), _f64(y_in), _f64(m.a), _f64(m.b),
                                           m.pair_index, m.ranks, m.scalings, m.row_slot,
                                           m.expert_offsets, m.R, m.out_slices, m.slots,
                                           m.num_experts, m.num_pairs)
    out = host_bits(d.y)
    assert read_flags(d.flags) == flags
    assert_close(_f64(out), y_ref, what)
    assert_rows_bit_identical(out, y_in, ~touched, what + " untouched")
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_moe_random(seed):
    m = W.random_moe(20 + seed, 40, 9, 136, (24, 32), 3, 16)
    _check_moe(m)
    _check_moe(m, y_bits=np.zeros_like(m.y), what="moe y=0")


def test_moe_bad_rows_flagged():
    m = W.random_moe(30, 20, 6, 64, (16,), 3, 8, ranks=[8, 8, 8])
    rs = m.row_slot.copy()
    rs[::7] = 9                                  # slot out of range
    pi = m.pair_index.copy()
    pi[pi >= 0][:1] = m.num_pairs + 4
    idx = np.nonzero(m.pair_index >= 0)[0][:2]
    pi[idx] = m.num_pairs + 4                    # pair out of range
    q = W.MoEProblem(**{**m.__dict__, "row_slot": rs, "pair_index": pi})
    _check_moe(q, what="moe flags")


# ---------------------------------------------------------------------------
# The five workloads at full size
# ---------------------------------------------------------------------------

def test_workload_decode_qkv_full():
    p = W.decode_qkv(0)
    _check_linear(p, L.LORA_REGIME_AUTO, what="decode")
    _check_linear(p, L.LORA_REGIME_AUTO, y_bits=np.zeros_like(p.y), what="decode y=0")


def _oracle_rows(p, tokens, y_bits):
    """The oracle on a subset of tokens, as a problem of its own: their x and y
    rows, their slots, the same adapters.  Returns y_ref for those rows."""
    tokens = np.asarray(tokens)
    to, ip = W.csr_by_slot(p.slot_of[tokens], p.slots)
    y_ref, _, _ = O.apply_linear(_f64(p.x[tokens]), _f64(y_bits[tokens]), _f64(p.a), _f64(p.b),
                                 to, ip, p.ranks, p.scalings, p.out_slices, p.R)
    return y_ref


def test_workload_prefill_gate_up_full():
    """Every row of y at the full prefill size (8192 tokens, out 28672) against
    the fp64 oracle, element by element, in chunks of 1024 tokens."""
    p = W.prefill_gate_up(0)
    d = LinearDev(p)
    d.apply_linear(L.LORA_REGIME_AUTO)
    out = host_bits(d.y)
    assert read_flags(d.flags) == 0
    for c0 in range(0, p.T, 1024):
        rows = np.arange(c0, min(p.T, c0 + 1024))
        assert_close(_f64(out[rows]), _oracle_rows(p, rows, p.y), f"prefill rows {c0}..")


def test_workload_embedding_full():
    p = W.embedding(0)
    d = LinearDev(p)
    d.apply_embedding(L.LORA_REGIME_AUTO)
    y_ref, touched, flags = O.apply_embedding(p.ids, _f64(p.y), _f64(p.a), _f64(p.b),
                                              p.token_order, p.slot_indptr, p.ranks, p.scalings,
                                              p.out_slices, p.R, p.n_in)
    out = host_bits(d.y)
    assert read_flags(d.flags) == flags == 0
    assert_close(_f64(out), y_ref, "embedding")
    assert_rows_bit_identical(out, p.y, ~touched, "embedding untouched (id -1)")
    zero = np.zeros_like(p.y)
    d0 = LinearDev(p, zero)
    d0.apply_embedding(L.LORA_REGIME_AUTO)
    y0, _, _ = O.apply_embedding(p.ids, _f64(zero), _f64(p.a), _f64(p.b), p.token_order,
                                 p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R, p.n_in)
    assert_close(_f64(host_bits(d0.y)), y0, "embedding y=0")


def test_workload_moe_full():
    gu, dn = W.moe_expert(0)
    for m in (gu, dn):
        _check_moe(m, what=m.name)


# ---------------------------------------------------------------------------
# Launch overlap (programmatic dependent launch) between dependent calls
# ---------------------------------------------------------------------------

def _chain_problems(regime):
    # Three fused calls on one y: each reads the y the previous call wrote,
    # with its own x, adapters and slot layout.
    if int(regime) == L.LORA_REGIME_SGMV:
        return [W.random_linear(910 + k, 1200, 256, (128, 64), 4, 32, ranks=[32, 16, 8, 32],
                                dead_frac=0.05) for k in range(3)]
    return [W.random_linear(900 + k, 256, 512, (256, 128, 64), 12, 16, ranks=None,
                            dead_frac=0.1) for k in range(3)]


def _oracle_chain(ps, y0):
    y = y0
    for p in ps:
        y_ref, _, _ = _oracle_linear(p, y)
        y = W.f32_to_bf16_bits(y_ref)
    return y


@pytest.mark.parametrize("regime", REGIMES)
@pytest.mark.parametrize("graph", [False, True], ids=["stream", "graph"])
def test_launch_overlap_dependent_chain(regime, graph):
    """With the overlap on, each call still sees the y its predecessor wrote
    (x, y and h are read only after the preceding kernel completed), and calls
    sharing one workspace do not overwrite h while it is being read."""
    t = torch()
    ps = _chain_problems(regime)
    devs = [LinearDev(p) for p in ps]
    ws_bytes = max(L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R,
                                          p.num_slices, int(regime)) for p in ps)
    if not regime.workspace:
        ws_bytes = 0
    ws = t.zeros(max(ws_bytes, 16) // 4, dtype=t.float32, device="cuda")
    y = devs[0].y
    y0 = host_bits(y).copy()
    prev = L.lora_set_launch_overlap(1)
    try:
        def run():
            for d in devs:
                p = d.p
                L.lora_apply_linear(d.x, y, d.a, d.b, d.ranks, d.scalings, d.token_order,
                                    d.slot_indptr, p.T, p.n_in, p.slots, p.R, p.out_slices,
                                    regime=int(regime), workspace=ws if ws_bytes else None,
                                    workspace_bytes=ws_bytes, err_flags=d.flags)
        if graph:
            run()                                   # warm the launch caches outside capture
            t.cuda.synchronize()
            y.copy_(t.from_numpy(y0.view(np.int16).copy()).view(t.bfloat16).cuda())
            g = t.cuda.CUDAGraph()
            with t.cuda.graph(g):
                run()
            y.copy_(t.from_numpy(y0.view(np.int16).copy()).view(t.bfloat16).cuda())
            g.replay()
        else:
            run()
        t.cuda.synchronize()
    finally:
        L.lora_set_launch_overlap(prev)
    ref = _oracle_chain(ps, y0)
    assert_close(_f64(host_bits(y)), _f64(ref), "chain")
    assert all(read_flags(d.flags) == 0 for d in devs)



# ---------------------------------------------------------------------------
# The split kernel's bounded wait
# ---------------------------------------------------------------------------

def test_split_wait_runs_out_and_is_flagged():
    """The BGMV_SPLIT kernel's bounded wait, made to run out without any fault:
    the host sets the first work item's counter
    in the workspace so that it never equals that item's number of shrink
    pieces.  With a 2 ms limit every expand piece of that item gives up,
    LORA_FLAG_TIMEOUT is raised, those rows of y are left as they were, every
    other row is right, the call returns, and the counters end zeroed: the same
    workspace then gives the oracle's result."""
    t = torch()
    p = W.decode_qkv(3)
    ws_bytes = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R, p.num_slices,
                                      L.LORA_REGIME_BGMV_SPLIT)
    ws = t.zeros(ws_bytes // 4, dtype=t.int32, device="cuda")
    ws[0] = 1 << 30                    # item 0's counter: out of reach
    d = LinearDev(p)
    prev = L.lora_set_wait_limit_ns(2_000_000)
    try:
        d.apply_linear(L.LORA_REGIME_BGMV_SPLIT, workspace=ws)
        t.cuda.synchronize()
    finally:
        L.lora_set_wait_limit_ns(prev)
    assert read_flags(d.flags) == L.LORA_FLAG_TIMEOUT
    # item 0: the 32 smallest token ids of the first slot with tokens
    s0 = next(s for s in range(p.slots) if p.slot_indptr[s + 1] > p.slot_indptr[s])
    toks0 = np.sort(p.token_order[p.slot_indptr[s0]:p.slot_indptr[s0 + 1]])[:32]
    out = host_bits(d.y)
    assert_rows_bit_identical(out, p.y, toks0, "timed-out item")
    y_ref, touched, _ = _oracle_linear(p)
    rest = np.setdiff1d(np.nonzero(touched)[0], toks0)
    assert_close(_f64(out[rest]), y_ref[rest], "other items")
    assert int(ws[:1024].abs().sum().item()) == 0     # counters zeroed again
    d2 = LinearDev(p)
    d2.apply_linear(L.LORA_REGIME_BGMV_SPLIT, workspace=ws)
    assert read_flags(d2.flags) == 0
    assert_close(_f64(host_bits(d2.y)), y_ref, "rerun on the same workspace")
