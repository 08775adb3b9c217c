"""Pins for the fp64 oracle (CPU only).

The oracle is trusted only because it is tied here to things other than
itself: hand-derived worked examples (``tests/golden``), an independent
algorithm the pages describe (every token against every slot, then its own
selected), brute force on tiny inputs, closed forms (the gather is the shrink
of a one-hot) and invariants (low rank, bit-identical no-ops, slice and
chunk independence).  A few tests plant a mistake in a copy of the oracle and
check that a pin catches it.
"""
import json
import os

import numpy as np
import pytest

from oracle import lora_oracle as O
from adapter_lora_serving_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f64(p, name):
    v = getattr(p, name)
    return None if v is None else W.bf16_to_f64(v)


def _lin_args(p):
    return dict(x=_f64(p, "x"), y=_f64(p, "y"), a=_f64(p, "a"), b=_f64(p, "b"),
                token_order=p.token_order, slot_indptr=p.slot_indptr, ranks=p.ranks,
                scalings=p.scalings, out_slices=p.out_slices, R=p.R)


# ---------------------------------------------------------------------------
# Hand-derived worked examples
# ---------------------------------------------------------------------------

def test_linear_hand_example():
    g = _load("linear_hand.json")
    x = np.array(g["x"], float)
    a = np.array(g["a"], float)
    b = np.array(g["b"], float)
    y = np.array(g["y"], float)
    args = (g["token_order"], g["slot_indptr"], g["ranks"], g["scalings"],
            g["out_slices"], g["R"])
    y_ref, touched, flags = O.apply_linear(x, y, a, b, *args)
    assert flags == 0
    assert np.array_equal(y_ref, np.array(g["expected_y"], float))
    assert list(touched) == g["expected_touched"]
    yb, fb = O.brute_apply_linear(x, y, a, b, *args)
    assert np.array_equal(yb, np.array(g["expected_y"], float))
    h, mask, _ = O.shrink(x, a, g["token_order"], g["slot_indptr"], g["ranks"], g["R"],
                          len(g["out_slices"]))
    exp_h = g["expected_h"]
    for t in range(g["T"]):
        for c in range(len(exp_h[t])):
            if exp_h[t][c] is None:
                assert not mask[t, c]
            else:
                assert mask[t, c] and h[t, c] == exp_h[t][c]
    y2, t2, _ = O.expand(y, np.nan_to_num(h, nan=1e300), b, g["token_order"],
                         g["slot_indptr"], g["ranks"], g["scalings"], g["out_slices"],
                         g["R"])
    assert np.array_equal(y2, np.array(g["expected_y"], float))


def test_embedding_hand_example():
    g = _load("embedding_hand.json")
    a = np.array(g["a"], float)
    b = np.array(g["b"], float)
    y = np.array(g["y"], float)
    h, mask, flags = O.gather_shrink(g["ids"], a, g["token_order"], g["slot_indptr"],
                                     g["ranks"], g["R"], 1, g["vocab"])
    assert flags == 0 and mask.all()
    assert np.array_equal(h, np.array(g["expected_h"], float))
    y_ref, touched, flags = O.apply_embedding(g["ids"], y, a, b, g["token_order"],
                                              g["slot_indptr"], g["ranks"], g["scalings"],
                                              g["out_slices"], g["R"], g["vocab"])
    assert np.array_equal(y_ref, np.array(g["expected_y"], float))
    assert list(touched) == g["expected_touched"]


def test_expert_plan_hand_example():
    g = _load("expert_plan_hand.json")
    work, flags = O.expert_workitems(g["expert_offsets"], g["adapted"], g["rows_cap"])
    assert [list(w) for w in work] == g["expected_work"]
    assert flags == g["expected_flags"]
    chunks = O.chunk_workitems(work, g["max_rows"])
    assert [list(c) for c in chunks] == g["expected_chunks"]


def test_adapted_experts_hand_example():
    g = _load("adapted_experts_hand.json")
    assert O.adapted_experts(g["pair_index"], g["slots"], g["num_experts"]) == \
        g["expected_adapted"]
    chunks, flags = O.plan_expert(g["expert_offsets"], g["pair_index"], g["slots"],
                                  g["num_experts"], g["rows_cap"], g["max_rows"])
    assert [list(c) for c in chunks] == g["expected_chunks"]
    assert flags == g["expected_flags"]


def test_router_hand_example():
    g = _load("router_hand.json")
    args = dict(router_in=np.array(g["router_in"], float), logits=np.array(g["logits"], float),
                a=np.array(g["a"], float), b=np.array(g["b"], float),
                token_order=g["token_order"], slot_indptr=g["slot_indptr"], ranks=g["ranks"],
                scalings=g["scalings"], R=g["R"])
    out, touched, flags = O.apply_router(**args)
    assert flags == 0
    assert np.array_equal(out, np.array(g["expected_logits"], float))
    assert list(touched) == g["expected_touched"]
    # the element-by-element definition agrees
    brute, bflags = O.brute_apply_linear(args["router_in"], args["logits"], args["a"],
                                         args["b"], g["token_order"], g["slot_indptr"],
                                         g["ranks"], g["scalings"], (g["num_experts"],), g["R"])
    assert bflags == 0 and np.array_equal(brute, out)
    # the fold comes before top-k: it changes token 0's choice
    assert O.top_k_experts(args["logits"], 2) == g["expected_top2_before"]
    assert O.top_k_experts(out, 2) == g["expected_top2_after"]


def test_expert_fold_hand_example():
    g = _load("expert_fold_hand.json")
    args = dict(x=np.array(g["x"], float), y=np.array(g["y"], float),
                a=np.array(g["a"], float), b=np.array(g["b"], float),
                pair_index=np.array(g["pair_index"]).reshape(-1), ranks=g["ranks"],
                scalings=g["scalings"], row_slot=g["row_slot"],
                expert_offsets=g["expert_offsets"], R=g["R"], out_slices=g["out_slices"],
                slots=g["slots"], num_experts=g["num_experts"], num_pairs=g["num_pairs"])
    y_ref, touched, flags = O.expert_apply(**args)
    assert flags == 0
    assert np.array_equal(y_ref, np.array(g["expected_y"], float))
    assert list(touched) == g["expected_touched"]
    assert np.array_equal(O.brute_expert_apply(**args), np.array(g["expected_y"], float))


# ---------------------------------------------------------------------------
# Brute force and an independent algorithm from the pages
# ---------------------------------------------------------------------------

SMALL_SHAPES = [
    # T, in, out_slices, slots, R
    (9, 16, (8,), 3, 8),
    (13, 24, (8, 16), 4, 8),
    (16, 32, (16, 8, 8), 5, 16),
    (7, 8, (24,), 2, 16),
]


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("shape", SMALL_SHAPES)
def test_brute_equals_fast(shape, seed):
    T, n_in, outs, slots, R = shape
    p = W.random_linear(seed, T, n_in, outs, slots, R, dead_frac=0.2)
    p.scalings[0] = 0.0
    args = _lin_args(p)
    y_fast, touched, f1 = O.apply_linear(**args)
    y_brute, f2 = O.brute_apply_linear(**args)
    assert f1 == f2 == 0
    np.testing.assert_allclose(y_fast, y_brute, rtol=1e-12, atol=1e-12)


def _every_slot_then_select(x, y, a, b, slot_of, ranks, scalings, out_slices, R):
    """The pages' reference design (``shrink_reference``): every token against every
    slot, then its own selected; zeros where the expand does not read (dead
    tokens, columns past the rank); then ``expand_reference_``."""
    T = x.shape[0]
    slots = a.shape[0]
    S = len(out_slices)
    h_all = np.einsum("tk,sck->tsc", x, a)                 # [T, slots, S*R]
    live = slot_of >= 0
    sel = np.where(live, slot_of, 0)
    h = h_all[np.arange(T), sel]                           # [T, S*R]
    col_rank = np.tile(np.arange(R), S)[None, :]
    keep = live[:, None] & (col_rank < np.asarray(ranks)[sel][:, None])
    h = np.where(keep, h, 0.0)
    offs = O.slice_offsets(out_slices)
    y2 = y.copy()
    for i, w in enumerate(out_slices):
        bsel = b[sel][:, offs[i]:offs[i] + w, :]            # [T, w, R]
        d = np.einsum("tr,tjr->tj", h[:, i * R:(i + 1) * R], bsel)
        sc = np.where(live, np.asarray(scalings, float)[sel], 0.0)
        y2[:, offs[i]:offs[i] + w] += sc[:, None] * d
    return y2


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_every_slot_then_select_design(seed):
    p = W.random_linear(seed, 40, 64, (16, 8), 6, 16, dead_frac=0.15)
    args = _lin_args(p)
    y_ref, _, _ = O.apply_linear(**args)
    y_alt = _every_slot_then_select(args["x"], args["y"], args["a"], args["b"], p.slot_of,
                                    p.ranks, p.scalings, p.out_slices, p.R)
    np.testing.assert_allclose(y_ref, y_alt, rtol=1e-12, atol=1e-12)


def test_tiny_config_brute():
    p = W.tiny_linear(0)
    args = _lin_args(p)
    y_fast, touched, flags = O.apply_linear(**args)
    y_brute, _ = O.brute_apply_linear(**args)
    assert flags == 0
    np.testing.assert_allclose(y_fast, y_brute, rtol=1e-12, atol=1e-12)
    rank0 = p.slot_of == 0                      # slot 0 has rank 0
    assert not touched[rank0].any()


# ---------------------------------------------------------------------------
# Invariants
# ---------------------------------------------------------------------------

def test_delta_is_low_rank_and_ignores_columns_past_rank():
    p = W.random_linear(3, 48, 32, (24,), 3, 16, ranks=[4, 9, 16])
    args = _lin_args(p)
    y_ref, _, _ = O.apply_linear(**args)
    # poison A rows and B columns past each slot's rank
    a = args["a"].copy()
    b = args["b"].copy()
    for s, r in enumerate(p.ranks):
        a[s, r:, :] = np.nan
        b[s, :, r:] = 1e300
    y_p, _, _ = O.apply_linear(**{**args, "a": a, "b": b})
    assert np.array_equal(y_ref, y_p)
    delta = y_ref - args["y"]
    for s, r in enumerate(p.ranks):
        toks = p.slot_of == s
        if toks.sum() > r:
            assert np.linalg.matrix_rank(delta[toks], tol=1e-9) <= r


def test_no_op_cases_are_bit_identical():
    p = W.random_linear(4, 20, 16, (8, 8), 4, 8, ranks=[0, 8, 8, 8],
                        scalings=[1.0, 0.0, 1.0, 1.0], dead_frac=0.3)
    args = _lin_args(p)
    y = args["y"].copy()
    y[:, 0] = -0.0
    y[:, 1] = np.nan
    y_ref, touched, _ = O.apply_linear(**{**args, "y": y})
    for t in range(p.T):
        s = p.slot_of[t]
        if s in (-1, 0, 1):
            assert not touched[t]
            assert np.array_equal(y_ref[t].view(np.uint64), y[t].view(np.uint64))
        else:
            assert touched[t]


def test_linear_in_scaling():
    p = W.random_linear(5, 30, 32, (16,), 3, 8, ranks=[8, 8, 8])
    args = _lin_args(p)
    y1, _, _ = O.apply_linear(**args)
    y2, _, _ = O.apply_linear(**{**args, "scalings": np.asarray(p.scalings) * 2})
    np.testing.assert_allclose(y2 - args["y"], 2 * (y1 - args["y"]), rtol=1e-9, atol=1e-12)


def test_slices_are_independent():
    """A fused S-slice call equals S single-slice calls on the matching A row block
    and B row block."""
    outs = (16, 8, 24)
    R = 8
    p = W.random_linear(6, 25, 32, outs, 4, R, ranks=[8, 4, 0, 8])
    args = _lin_args(p)
    y_fused, _, _ = O.apply_linear(**args)
    offs = O.slice_offsets(outs)
    for i, w in enumerate(outs):
        y_i, _, _ = O.apply_linear(**{**args, "y": args["y"][:, offs[i]:offs[i] + w],
                                      "a": args["a"][:, i * R:(i + 1) * R, :],
                                      "b": args["b"][:, offs[i]:offs[i] + w, :],
                                      "out_slices": (w,)})
        assert np.array_equal(y_i, y_fused[:, offs[i]:offs[i] + w])


def test_permuting_positions_within_a_slot():
    p = W.random_linear(7, 30, 16, (8,), 3, 8, ranks=[8, 8, 8])
    args = _lin_args(p)
    y_ref, _, _ = O.apply_linear(**args)
    to = p.token_order.copy()
    rng = np.random.default_rng(0)
    for s in range(p.slots):
        lo, hi = p.slot_indptr[s], p.slot_indptr[s + 1]
        to[lo:hi] = rng.permutation(to[lo:hi])
    y_p, _, _ = O.apply_linear(**{**args, "token_order": to})
    assert np.array_equal(y_ref, y_p)


def test_gather_is_shrink_of_one_hot():
    vocab, R = 40, 8
    p = W.random_linear(8, 30, None, (16,), 3, R, ranks=[8, 4, 8], embedding_vocab=vocab,
                        bad_id_frac=0.2)
    a = _f64(p, "a")
    h_g, m_g, _ = O.gather_shrink(p.ids, a, p.token_order, p.slot_indptr, p.ranks, R, 1,
                                  vocab)
    x1 = np.zeros((p.T, vocab))
    for t, v in enumerate(p.ids):
        if 0 <= v < vocab:
            x1[t, v] = 1.0
    h_s, m_s, _ = O.shrink(x1, a, p.token_order, p.slot_indptr, p.ranks, R, 1)
    assert np.array_equal(m_g, m_s)
    assert np.array_equal(h_g[m_g], h_s[m_s])
    y = _f64(p, "y")
    b = _f64(p, "b")
    y_e, t_e, _ = O.apply_embedding(p.ids, y, a, b, p.token_order, p.slot_indptr, p.ranks,
                                    p.scalings, p.out_slices, R, vocab)
    y_l, t_l, _ = O.apply_linear(x1, y, a, b, p.token_order, p.slot_indptr, p.ranks,
                                 p.scalings, p.out_slices, R)
    np.testing.assert_allclose(y_e, y_l, rtol=0, atol=0)
    bad = np.array([not (0 <= v < vocab) for v in p.ids])
    assert not t_e[bad].any()


# ---------------------------------------------------------------------------
# Addressing rules and flags
# ---------------------------------------------------------------------------

def test_plan_segments_hand_example():
    # slot 0: positions 0..4 (5), slot 1: empty, slot 2: 5..6, slot 3 rank 0
    indptr = [0, 5, 5, 7, 9]
    ranks = [8, 8, 8, 0]
    assert O.plan_segments(indptr, ranks, 9, 8, 2) == [(0, 0, 2), (0, 2, 2), (0, 4, 1),
                                                       (2, 5, 2)]
    # scaling 0 removes slot 2 from the scaled plan only
    assert O.plan_segments(indptr, ranks, 9, 8, 4, scalings=[1, 1, 0, 1]) == [(0, 0, 4),
                                                                              (0, 4, 1)]
    # malformed segments and ranks are skipped
    assert O.plan_segments([0, 3, 2, 9], [8, 8, 8], 8, 8, 16) == [(0, 0, 3)]
    assert O.plan_segments([0, 3, 6], [8, 9], 6, 8, 16) == [(0, 0, 3)]


def test_malformed_addressing_is_skipped_and_flagged():
    x = np.ones((4, 2))
    a = np.ones((3, 1, 2))
    b = np.ones((3, 1, 1))
    y = np.zeros((4, 1))
    # slot 0: [0,2) tokens (0, 7->bad); slot 1: [2,1) bad segment; slot 2: rank 5 > R
    y_ref, touched, flags = O.apply_linear(x, y, a, b, [0, 7, 2, 3], [0, 2, 1, 4],
                                           [1, 1, 5], [1.0, 1.0, 1.0], (1,), 1)
    assert flags == O.FLAG_BAD_TOKEN | O.FLAG_BAD_INDPTR | O.FLAG_BAD_RANK
    assert list(touched) == [True, False, False, False]
    assert y_ref[0, 0] == 2.0


def test_duplicate_token_rejected():
    with pytest.raises(O.DuplicateTokenError):
        O.resolve_slots([1, 1, 0], [0, 1, 2], [4, 4], 3, 8)


# ---------------------------------------------------------------------------
# MoE fold
# ---------------------------------------------------------------------------

def _moe_args(m):
    return dict(x=W.bf16_to_f64(m.x), y=W.bf16_to_f64(m.y), a=W.bf16_to_f64(m.a),
                b=W.bf16_to_f64(m.b), pair_index=m.pair_index, ranks=m.ranks,
                scalings=m.scalings, row_slot=m.row_slot, expert_offsets=m.expert_offsets,
                R=m.R, out_slices=m.out_slices, slots=m.slots, num_experts=m.num_experts,
                num_pairs=m.num_pairs)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_expert_loop_equals_row_brute_force(seed):
    m = W.random_moe(seed, 5, 6, 12, (8, 8), 3, 8)
    args = _moe_args(m)
    y_loop, _, flags = O.expert_apply(**args, max_rows=3)
    assert flags == 0
    np.testing.assert_allclose(y_loop, O.brute_expert_apply(**args), rtol=1e-12,
                               atol=1e-12)


def test_expert_chunking_is_identical():
    m = W.random_moe(3, 9, 5, 16, (8,), 2, 8)
    args = _moe_args(m)
    ys = [O.expert_apply(**args, max_rows=mr)[0] for mr in (1, 2, 4, 128)]
    for y in ys[1:]:
        assert np.array_equal(ys[0], y)


def test_expert_fold_reduces_to_linear():
    """One expert and one slot: the fold is the linear apply over the row list."""
    rows, n_in, R = 11, 16, 8
    p = W.random_linear(9, rows, n_in, (8, 8), 1, R, ranks=[8], scalings=[1.5],
                        slot_of=np.zeros(rows, int))
    args = _lin_args(p)
    y_lin, _, _ = O.apply_linear(**args)
    y_moe, _, _ = O.expert_apply(args["x"], args["y"], args["a"], args["b"],
                                 np.array([0]), p.ranks, p.scalings,
                                 np.zeros(rows, np.int32), np.array([0, rows]), R,
                                 p.out_slices, 1, 1, 1, max_rows=4)
    np.testing.assert_allclose(y_moe, y_lin, rtol=1e-12, atol=0)


def test_expert_flags():
    m = W.random_moe(4, 4, 4, 8, (8,), 2, 8)
    args = _moe_args(m)
    assert m.rows_cap > 2
    rs = m.row_slot.copy()
    rs[0] = 5                                   # slot out of range
    rs[1] = 0
    pi = np.full_like(m.pair_index, 99)         # every expert adapted, pair out of range
    _, _, flags = O.expert_apply(**{**args, "row_slot": rs, "pair_index": pi})
    assert flags == O.FLAG_BAD_SLOT | O.FLAG_BAD_PAIR
    off = m.expert_offsets.copy()
    off[2] = off[-1] + 5                         # past rows_cap
    _, _, f2 = O.expert_apply(**{**args, "expert_offsets": off})
    assert f2 & O.FLAG_BAD_OFFSETS


def test_moe_workload_shapes():
    gu, dn = W.moe_expert(0)
    assert gu.rows_cap == 16384 and gu.expert_offsets[-1] == 16384
    assert np.all(np.diff(gu.expert_offsets) >= 0)
    assert gu.num_pairs == 4 * 32
    items, flags = O.plan_expert(gu.expert_offsets, gu.pair_index, gu.slots,
                                 gu.num_experts, gu.rows_cap, 128)
    assert flags == 0 and len(items) > 0
    assert dn.out == 2048 and gu.out == 1536


# ---------------------------------------------------------------------------
# Planted mistakes: a copy of the oracle with one error must fail a pin
# ---------------------------------------------------------------------------

def test_planted_wrong_slice_offset_fails_golden(monkeypatch):
    g = _load("linear_hand.json")
    monkeypatch.setattr(O, "slice_offsets", lambda outs: [0] * (len(outs) + 1))
    y_ref, _, _ = O.apply_linear(np.array(g["x"], float), np.array(g["y"], float),
                                 np.array(g["a"], float), np.array(g["b"], float),
                                 g["token_order"], g["slot_indptr"], g["ranks"],
                                 g["scalings"], g["out_slices"], g["R"])
    assert not np.array_equal(y_ref, np.array(g["expected_y"], float))


def test_planted_transposed_gather_fails_closed_form():
    vocab, R = 16, 16
    p = W.random_linear(10, 12, None, (8,), 2, R, ranks=[16, 16], embedding_vocab=vocab)
    a = _f64(p, "a")
    wrong = a.transpose(0, 2, 1)[:, :R, :vocab]           # rows and ids swapped
    h_w, m_w, _ = O.gather_shrink(p.ids, wrong, p.token_order, p.slot_indptr, p.ranks, R,
                                  1, vocab)
    x1 = np.zeros((p.T, vocab))
    x1[np.arange(p.T), p.ids] = 1.0
    h_s, m_s, _ = O.shrink(x1, a, p.token_order, p.slot_indptr, p.ranks, R, 1)
    assert not np.array_equal(h_w[m_w], h_s[m_s])


def test_planted_unsorted_adapted_list_fails_golden(monkeypatch):
    # experts in the order the pairs are met (slot by slot), not sorted
    g = _load("adapted_experts_hand.json")

    def first_seen(pair_index, slots, num_experts):
        pi = np.asarray(pair_index).reshape(slots, num_experts)
        out = []
        for s in range(slots):
            for e in range(num_experts):
                if pi[s, e] != -1 and e not in out:
                    out.append(e)
        return out
    monkeypatch.setattr(O, "adapted_experts", first_seen)
    chunks, _ = O.plan_expert(g["expert_offsets"], g["pair_index"], g["slots"],
                              g["num_experts"], g["rows_cap"], g["max_rows"])
    assert [list(c) for c in chunks] != g["expected_chunks"]
