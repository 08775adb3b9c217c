"""GPU parity of the fused linear fold in the STREAM regime (lora_apply_linear:
the short-segment shrink into per-chunk fp32 partial h, then the streamed
expand) against the fp64 oracle.  Tolerance |y_dev - y_ref| <= 1e-2 + 1.6e-2 |y_ref| elementwise;
untouched rows (tokens in no segment, rank-0 or scaling-0 slots) and flags
bit-exact."""
import numpy as np
import pytest

from adapter_lora_serving_b200 import lora as L
from adapter_lora_serving_b200 import workloads as W
from oracle import lora_oracle as O

from gpu_util import LinearDev, assert_close, assert_rows_bit_identical, host_bits, read_flags, torch

pytestmark = pytest.mark.gpu

STREAM = L.LORA_REGIME_STREAM
f64 = W.bf16_to_f64


def _oracle(p, y_bits=None):
    return O.apply_linear(f64(p.x), f64(p.y if y_bits is None else y_bits), f64(p.a), f64(p.b),
                          p.token_order, p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)


def _nan_workspace(p):
    """A workspace of the bytes lora_workspace_bytes asks for, every word NaN:
    the fold reads no partial it has not written, and needs no initialisation."""
    t = torch()
    n = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R, p.num_slices, STREAM)
    assert n >= 4096 + 4 * p.T * p.num_slices * p.R * ((p.n_in + 511) // 512)
    return t.full((n // 4,), float("nan"), dtype=t.float32, device="cuda"), n


def _apply(d, ws=None):
    p = d.p
    if ws is None:
        ws = _nan_workspace(p)
    L.lora_apply_linear(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order, d.slot_indptr,
                        p.T, p.n_in, p.slots, p.R, p.out_slices, regime=STREAM, workspace=ws[0],
                        workspace_bytes=ws[1], err_flags=d.flags)


def _check(p, what=""):
    d = LinearDev(p)
    ws = _nan_workspace(p)
    _apply(d, ws)
    # the first 4096 bytes (the BGMV_SPLIT counters of a shared workspace) are left alone
    assert bool(ws[0][:1024].isnan().all()), "counter header written"
    out = host_bits(d.y)
    ref, touched, flags = _oracle(p)
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, what)
    assert_rows_bit_identical(out, p.y, ~touched, what + " untouched")
    return out


def test_workload_decode_full_stream():
    """Decode over the fused QKV projection at full size (T=256, in=4096,
    out 4096+1024+1024, 32 slots), every element, and again with y = 0."""
    p = W.decode_qkv(0)
    _check(p, "decode_qkv")
    zero = np.zeros_like(p.y)
    d0 = LinearDev(p, zero)
    _apply(d0)
    y0, _, _ = _oracle(p, zero)
    assert_close(f64(host_bits(d0.y)), y0, "decode_qkv y=0")


def test_router_workload_stream():
    """The MoE layer's router (logits [2048, 128], hidden 2048) through
    lora_apply_router in the STREAM regime."""
    p = W.moe_router(0)
    d = LinearDev(p)
    n = L.lora_workspace_bytes(L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R, 1, STREAM)
    t = torch()
    ws = t.full((n // 4,), float("nan"), dtype=t.float32, device="cuda")
    L.lora_apply_router(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order, d.slot_indptr,
                        p.T, p.n_in, p.slots, p.R, p.out, regime=STREAM, workspace=ws,
                        workspace_bytes=n, err_flags=d.flags)
    out = host_bits(d.y)
    ref, touched, flags = O.apply_router(f64(p.x), f64(p.y), f64(p.a), f64(p.b), p.token_order,
                                         p.slot_indptr, p.ranks, p.scalings, p.R)
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, "router stream")
    assert_rows_bit_identical(out, p.y, ~touched, "router stream untouched")


SHAPES = [
    # T, in, out_slices, slots, R, dead_frac
    (64, 256, (256,), 4, 16, 0.0),               # one chunk, S*R = 16
    (150, 1000, (64, 32), 5, 16, 0.05),          # S*R = 32, ragged last chunk
    (37, 8, (8,), 3, 16, 0.2),                   # in = 8: one k-step partly filled
    (300, 4096, (8, 72, 16), 3, 16, 0.1),        # S*R = 48, eight chunks, narrow slices
    (257, 520, (1032,), 7, 32, 0.1),             # R = 32: two k-steps, 17 row groups
    (500, 2048, (520,), 6, 64, 0.0),             # R = 64, S*R = 64
    (2000, 1536, (4096, 1024), 6, 16, 0.05),     # wide slices, many column blocks
    (5, 4000, (1032,), 2, 16, 0.0),              # fewer tokens than one row group
    (1024, 2048, (2048, 2048, 2048, 2048), 32, 16, 0.0),   # S*R = 64 over four slices
    (150, 264, (48, 40), 4, 24, 0.1),            # R = 24 (two k-steps, rank padded), S*R = 48
    (200, 512, (96,), 3, 48, 0.0),               # R = 48: three k-steps
    (300, 1024, (128, 64, 64, 64, 64, 64, 64, 64), 5, 8, 0.1),   # R = 8 over eight slices
    (8500, 256, (64,), 3, 16, 0.05),             # 535 row groups over 148 CTAs
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("seed", [0, 1])
def test_random_linear_stream(shape, seed):
    T, n_in, outs, slots, R, dead = shape
    p = W.random_linear(1300 + 7 * seed + T, T, n_in, outs, slots, R, dead_frac=dead)
    _check(p, f"linear stream {shape}")


def test_rank_zero_scaling_zero_and_poison_past_rank():
    """Rank-0 and scaling-0 slots leave their rows bit-identical; NaN in A rows
    and B columns past a slot's rank is never used."""
    p = W.random_linear(41, 200, 712, (96, 64), 4, 16, ranks=[0, 8, 16, 5],
                        scalings=[2.0, 0.0, 1.5, 3.0])
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
    _apply(d)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(q)
    assert read_flags(d.flags) == flags == 0
    assert not np.isnan(f64(out)).any()
    assert_close(f64(out), ref, "poison")
    assert_rows_bit_identical(out, q.y, np.isin(q.slot_of, [0, 1]), "rank 0 / scaling 0 slots")


def test_bad_addressing_flags_stream():
    p = W.random_linear(42, 60, 512, (64,), 4, 16, ranks=[16, 16, 16, 16])
    to = p.token_order.copy()
    indptr = p.slot_indptr.copy()
    ranks = p.ranks.copy()
    to[indptr[0]] = 1000                     # bad token in slot 0
    ranks[2] = 17                            # rank > R
    indptr[3] = indptr[4] + 1                # slot 3: lo > hi
    q = W.LinearProblem(**{**p.__dict__, "token_order": to, "slot_indptr": indptr,
                           "ranks": ranks})
    d = LinearDev(q)
    _apply(d)
    out = host_bits(d.y)
    ref, touched, flags = _oracle(q)
    assert flags == O.FLAG_BAD_TOKEN | O.FLAG_BAD_RANK | O.FLAG_BAD_INDPTR
    assert read_flags(d.flags) == flags
    assert_close(f64(out), ref, "bad addressing")
    assert_rows_bit_identical(out, q.y, ~touched, "bad addressing untouched")


def test_permutation_and_rerun_bit_exact():
    """Each row's result depends only on its own token: reruns and any order of
    the positions inside each slot give identical bits."""
    p = W.random_linear(43, 500, 1504, (256, 64), 5, 16, dead_frac=0.05)
    d = LinearDev(p)
    _apply(d)
    first = host_bits(d.y)
    d2 = LinearDev(p)
    _apply(d2)
    assert np.array_equal(host_bits(d2.y), first)
    rng = np.random.default_rng(6)
    to = p.token_order.copy()
    for s in range(p.slots):
        lo, hi = p.slot_indptr[s], p.slot_indptr[s + 1]
        to[lo:hi] = rng.permutation(to[lo:hi])
    d3 = LinearDev(W.LinearProblem(**{**p.__dict__, "token_order": to}))
    _apply(d3)
    assert np.array_equal(host_bits(d3.y), first)


def test_agrees_with_the_other_regimes():
    """STREAM, BGMV and SGMV on the decode workload: each within the oracle's
    tolerance, so within twice of one another."""
    p = W.decode_qkv(1)
    ref, _, _ = _oracle(p)
    for regime in (L.LORA_REGIME_BGMV, L.LORA_REGIME_SGMV):
        d = LinearDev(p)
        d.apply_linear(regime)
        assert_close(f64(host_bits(d.y)), ref, f"regime {regime}")
    _check(p, "stream")


@pytest.mark.parametrize("graph", [False, True], ids=["eager", "graph"])
def test_launch_overlap_dependent_chain_stream(graph):
    """Five dependent calls on one y sharing one workspace, with the launch
    overlap on (eagerly and in a CUDA graph), give the bits of the same calls
    with it off: each shrink writes the partials only after the previous
    expand has read them, and each expand reads y only after the previous one
    wrote it."""
    t = torch()
    p = W.random_linear(44, 1200, 2048, (1024, 256), 6, 16, dead_frac=0.05)
    results = []
    prev = L.lora_set_launch_overlap(0)
    try:
        for overlap in (0, 1):
            L.lora_set_launch_overlap(overlap)
            d = LinearDev(p)
            ws = _nan_workspace(p)
            stream = t.cuda.Stream()

            def chain():
                for _ in range(5):
                    L.lora_apply_linear(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order,
                                        d.slot_indptr, p.T, p.n_in, p.slots, p.R, p.out_slices,
                                        regime=STREAM, workspace=ws[0], workspace_bytes=ws[1],
                                        err_flags=d.flags, stream=stream)
            if graph and overlap:
                g = t.cuda.CUDAGraph()
                with t.cuda.graph(g, stream=stream):
                    chain()
                g.replay()
                t.cuda.synchronize()
                del g
            else:
                with t.cuda.stream(stream):
                    chain()
                t.cuda.synchronize()
            assert read_flags(d.flags) == 0
            results.append(host_bits(d.y))
    finally:
        L.lora_set_launch_overlap(prev)
    assert np.array_equal(results[0], results[1])
    # Against five oracle folds: a fold moves a difference already in y
    # through unchanged (y + delta, then one rounding), so each of the five
    # adds at most its own per-fold bound and the chain is held to five times
    # it (a rounding of y that one side takes up and the other down, repeated
    # five times, reaches five bf16 ulps of y).
    ref = f64(p.y)
    for _ in range(5):
        ref, _, _ = O.apply_linear(f64(p.x), ref, f64(p.a), f64(p.b), p.token_order,
                                   p.slot_indptr, p.ranks, p.scalings, p.out_slices, p.R)
        ref = f64(W.f32_to_bf16_bits(ref.astype(np.float32)))
    err = np.abs(f64(results[0]) - ref)
    assert (err <= 5 * (O.ATOL + O.RTOL * np.abs(ref))).all(), float(err.max())


def test_unsupported_shapes_and_small_workspace():
    """S*R outside {16, 32, 48, 64} or in > 4096 is refused with
    LORA_ERR_UNSUPPORTED; a workspace below the need with LORA_ERR_WORKSPACE;
    y is untouched either way."""
    t = torch()
    for (n_in, outs, R) in ((512, (64, 64, 64), 32), (4104, (64,), 16)):
        p = W.random_linear(45, 40, n_in, outs, 2, R)
        d = LinearDev(p)
        ws = t.zeros(1 << 20, dtype=t.float32, device="cuda")
        with pytest.raises(L.LoraError) as e:
            L.lora_apply_linear(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order,
                                d.slot_indptr, p.T, p.n_in, p.slots, p.R, p.out_slices,
                                regime=STREAM, workspace=ws, workspace_bytes=4 << 20,
                                err_flags=d.flags)
        assert e.value.status == "LORA_ERR_UNSUPPORTED"
        assert np.array_equal(host_bits(d.y), p.y)
    p = W.random_linear(46, 40, 1024, (64,), 2, 16)
    d = LinearDev(p)
    need = 4096 + 4 * p.T * 16 * 2     # the counter header, two chunks of partials
    ws = t.zeros(need // 4, dtype=t.float32, device="cuda")
    with pytest.raises(L.LoraError) as e:
        L.lora_apply_linear(d.x, d.y, d.a, d.b, d.ranks, d.scalings, d.token_order,
                            d.slot_indptr, p.T, p.n_in, p.slots, p.R, p.out_slices,
                            regime=STREAM, workspace=ws, workspace_bytes=need - 4,
                            err_flags=d.flags)
    assert e.value.status == "LORA_ERR_WORKSPACE"
    assert np.array_equal(host_bits(d.y), p.y)


def test_no_live_slot_and_the_slot_limit():
    """Every slot at rank 0 (or scaling 0): no row group, y bit-identical.  Then
    LORA_MAX_SLOTS (4096) slots over 600 tokens: most slots empty, the plan's
    tables at their largest in shared memory."""
    p = W.random_linear(48, 300, 512, (64, 64), 5, 16, ranks=[0, 0, 0, 0, 0])
    d = LinearDev(p)
    _apply(d)
    assert read_flags(d.flags) == 0
    assert np.array_equal(host_bits(d.y), p.y)
    q = W.random_linear(49, 600, 256, (128,), 4096, 16, dead_frac=0.05)
    _check(q, "4096 slots")
