"""GPU parity of the embedding target in the STREAM regime (lora_apply_embedding,
the y rows streamed through shared memory) against the fp64 oracle.  Tolerance
|y_dev - y_ref| <= 1e-2 + 1.6e-2 |y_ref| elementwise; untouched rows (ids
outside the vocabulary, rank-0 or scaling-0 slots, tokens in no segment) and
flags bit-exact."""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import LinearDev, assert_close, assert_rows_bit_identical, host_bits, read_flags, torch

pytestmark = pytest.mark.gpu

STREAM = L.LORA_REGIME_STREAM
f64 = W.bf16_to_f64


def _oracle(p, y_bits=None, token_order=None, slot_indptr=None, ranks=None, a=None, b=None):
    return O.apply_embedding(p.ids, f64(p.y if y_bits is None else y_bits),
                             f64(p.a if a is None else a), f64(p.b if b is None else b),
                             p.token_order if token_order is None else token_order,
                             p.slot_indptr if slot_indptr is None else slot_indptr,
                             p.ranks if ranks is None else ranks, p.scalings, p.out_slices,
                             p.R, p.n_in)


def _check(p, regime=STREAM, what=""):
    d = LinearDev(p)
    d.apply_embedding(regime)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(p)
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, what)
    assert_rows_bit_identical(out, p.y, ~touched, what + " untouched")
    return out


def test_auto_resolves_to_stream():
    assert L.lora_resolve_regime(L.LORA_OP_APPLY_EMBEDDING, 4096, 8, 16, 1) == STREAM
    assert L.lora_plan_tile(L.LORA_OP_APPLY_EMBEDDING, STREAM) == 16


@pytest.mark.parametrize("regime", [pytest.param(STREAM, id="stream"),
                                    pytest.param(L.LORA_REGIME_AUTO, id="auto")])
def test_workload_embedding_full_stream(regime):
    """The embedding workload at full size (vocab 128256, T=4096, out 4096),
    every element, and again with y = 0 so the delta alone is compared."""
    p = W.embedding(0)
    out = _check(p, regime, "embedding")
    zero = np.zeros_like(p.y)
    d0 = LinearDev(p, zero)
    d0.apply_embedding(regime)
    y0, _, _ = _oracle(p, zero)
    assert_close(f64(host_bits(d0.y)), y0, "embedding y=0")
    assert out.shape == p.y.shape


SHAPES = [
    # T, vocab, out_slices, slots, R, dead_frac, bad_id_frac
    (150, 3000, (64, 32), 5, 16, 0.05, 0.1),        # two slices, ragged groups
    (37, 1000, (8,), 3, 8, 0.2, 0.2),               # one 8-column piece, R = 8
    (300, 5000, (8, 72, 16), 5, 8, 0.1, 0.05),      # three slices, pieces of 8..64 columns
    (64, 320, (256,), 4, 32, 0.0, 0.0),             # R = 32: two k-steps
    (1000, 2000, (520,), 7, 64, 0.1, 0.1),          # R = 64: 128-column units, ragged tail
    (2000, 129, (4096, 1024), 6, 16, 0.05, 0.05),   # wide slices, many pieces per group
    (5, 50, (1032,), 2, 16, 0.0, 0.0),              # fewer tokens than one group
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("seed", [0, 1])
def test_random_embedding_stream(shape, seed):
    T, vocab, outs, slots, R, dead, bad = shape
    p = W.random_linear(900 + 7 * seed + T, T, None, outs, slots, R, embedding_vocab=vocab,
                        bad_id_frac=bad, dead_frac=dead)
    _check(p, STREAM, f"embedding {shape}")


def test_ids_at_the_vocab_edges():
    """ids 0 and vocab-1 gather the first and last columns of A; ids -1, vocab
    and INT_MIN contribute nothing (their rows stay bit-identical)."""
    p = W.random_linear(31, 64, None, (128,), 2, 16, ranks=[16, 16], embedding_vocab=777)
    ids = p.ids.copy()
    ids[:8] = 0
    ids[8:16] = 776
    ids[16:20] = -1
    ids[20:24] = 777
    ids[24:28] = np.iinfo(np.int32).min
    q = W.LinearProblem(**{**p.__dict__, "ids": ids})
    _check(q, STREAM, "vocab edges")


def test_rank_zero_scaling_zero_and_poison_past_rank():
    """Rank-0 and scaling-0 slots leave y bit-identical; NaN in A rows and B
    columns past a slot's rank is never read."""
    p = W.random_linear(32, 200, None, (96, 64), 4, 16, ranks=[0, 8, 16, 5],
                        scalings=[2.0, 0.0, 1.5, 3.0], embedding_vocab=999)
    a = p.a.copy()
    b = p.b.copy()
    nan = np.uint16(0x7fc0)
    for s in range(p.slots):
        r = int(p.ranks[s])
        for i in range(p.num_slices):
            a[s, i * p.R + r:(i + 1) * p.R, :] = nan
        b[s, :, r:] = nan
    q = W.LinearProblem(**{**p.__dict__, "a": a, "b": b})
    d = LinearDev(q)
    d.apply_embedding(STREAM)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(q)
    assert read_flags(d.flags) == flags == 0
    assert not np.isnan(f64(out)).any()
    assert_close(f64(out), ref, "poison")
    assert_rows_bit_identical(out, q.y, ~touched, "rank 0 / scaling 0")
    assert_rows_bit_identical(out, q.y, np.isin(q.slot_of, [0, 1]), "rank 0 / scaling 0 slots")


def test_bad_addressing_flags_stream():
    p = W.random_linear(33, 60, None, (64,), 4, 16, ranks=[16, 16, 16, 16],
                        embedding_vocab=500)
    to = p.token_order.copy()
    indptr = p.slot_indptr.copy()
    ranks = p.ranks.copy()
    to[indptr[0]] = 1000                     # bad token in slot 0
    ranks[2] = 17                            # rank > R
    indptr[3] = indptr[4] + 1                # slot 3: lo > hi
    q = W.LinearProblem(**{**p.__dict__, "token_order": to, "slot_indptr": indptr,
                           "ranks": ranks})
    d = LinearDev(q)
    d.apply_embedding(STREAM)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(q)
    assert flags == O.FLAG_BAD_TOKEN | O.FLAG_BAD_RANK | O.FLAG_BAD_INDPTR
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, "bad addressing")
    assert_rows_bit_identical(out, q.y, ~touched, "bad addressing untouched")


def test_permutation_and_rerun_bit_exact():
    """Each row's result depends only on its own token: reruns and any order of
    the positions inside each slot give identical bits."""
    p = W.random_linear(34, 500, None, (256, 64), 5, 16, embedding_vocab=4000,
                        bad_id_frac=0.05)
    d = LinearDev(p)
    d.apply_embedding(STREAM)
    first = host_bits(d.y)
    d2 = LinearDev(p)
    d2.apply_embedding(STREAM)
    assert np.array_equal(host_bits(d2.y), first)
    rng = np.random.default_rng(5)
    to = p.token_order.copy()
    for s in range(p.slots):
        lo, hi = p.slot_indptr[s], p.slot_indptr[s + 1]
        to[lo:hi] = rng.permutation(to[lo:hi])
    d3 = LinearDev(W.LinearProblem(**{**p.__dict__, "token_order": to}))
    d3.apply_embedding(STREAM)
    assert np.array_equal(host_bits(d3.y), first)


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
def test_launch_overlap_dependent_chain_stream(graph):
    """Five dependent calls on one y with the launch overlap on (eagerly and in
    a CUDA graph) give the bits of the same calls with it off: every call reads
    y only after the previous one has written it."""
    t = torch()
    p = W.random_linear(35, 1200, None, (1024,), 6, 16, embedding_vocab=5000,
                        bad_id_frac=0.05)
    results = []
    prev = L.lora_set_launch_overlap(0)
    try:
        for overlap in (0, 1):
            L.lora_set_launch_overlap(overlap)
            d = LinearDev(p)
            stream = t.cuda.Stream()
            if graph and overlap:
                g = t.cuda.CUDAGraph()
                with t.cuda.graph(g, stream=stream):
                    for _ in range(5):
                        L.lora_apply_embedding(d.ids, d.y, d.a, d.b, d.ranks, d.scalings,
                                               d.token_order, d.slot_indptr, p.T, p.n_in,
                                               p.slots, p.R, p.out_slices, regime=STREAM,
                                               err_flags=d.flags, stream=stream)
                g.replay()
                t.cuda.synchronize()
                del g
            else:
                with t.cuda.stream(stream):
                    for _ in range(5):
                        L.lora_apply_embedding(d.ids, d.y, d.a, d.b, d.ranks, d.scalings,
                                               d.token_order, d.slot_indptr, p.T, p.n_in,
                                               p.slots, p.R, p.out_slices, regime=STREAM,
                                               err_flags=d.flags, stream=stream)
                t.cuda.synchronize()
            assert read_flags(d.flags) == 0
            results.append(host_bits(d.y))
    finally:
        L.lora_set_launch_overlap(prev)
    assert np.array_equal(results[0], results[1])
    # and five oracle folds agree with the chain
    y = p.y
    ref = f64(y)
    for _ in range(5):
        ref, _, _ = O.apply_embedding(p.ids, ref, f64(p.a), f64(p.b), p.token_order,
                                      p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R,
                                      p.n_in)
        ref = f64(W.f32_to_bf16_bits(ref.astype(np.float32)))
    assert_close(f64(results[0]), ref, "chain of five")
