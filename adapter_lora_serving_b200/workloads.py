"""Seeded synthetic inputs for the LoRA delta path.

This module only draws inputs: random tensors rounded to bf16, slot
assignments, CSR-by-slot addressing, MoE routing.  It holds none of the delta
arithmetic, so the CUDA library's tests and the CPU oracle can both be fed
from it without sharing any of the method.

bf16 tensors are returned as ``uint16`` bit patterns (numpy has no bf16);
``bf16_to_f64`` gives their exact values.  All draws use
``numpy.random.default_rng(seed)``.

The five workloads follow the shapes and distributions of the pages' use
cases (a small linear target, decode over a fused QKV projection, prefill over
a fused gate/up projection, an embedding target, and a routed-expert MoE
layer); the values the pages leave open are fixed here and listed in the
design notes.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


# ---------------------------------------------------------------------------
# bf16 encoding
# ---------------------------------------------------------------------------

def f32_to_bf16_bits(v):
    """Round float32 values to bf16 (round to nearest even), as uint16 bits."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits):
    return bf16_to_f32(bits).astype(np.float64)


def _normal_bf16(rng, shape, std=1.0, chunk=1 << 24):
    """N(0, std^2) draws rounded to bf16, generated in chunks to bound memory."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        v = rng.standard_normal(m, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[i:i + m] = f32_to_bf16_bits(v)
    return out.reshape(shape)


# ---------------------------------------------------------------------------
# Addressing from a per-token slot assignment
# ---------------------------------------------------------------------------

def csr_by_slot(slot_of, slots):
    """``token_order`` / ``slot_indptr`` from ``slot_of[t]`` (-1 = no adapter).

    token_order lists live tokens grouped by slot (stable, so each slot's
    tokens keep token order), followed by the dead tokens as padding."""
    slot_of = np.asarray(slot_of, dtype=np.int64)
    T = len(slot_of)
    live = np.nonzero(slot_of >= 0)[0]
    order = live[np.argsort(slot_of[live], kind="stable")]
    dead = np.nonzero(slot_of < 0)[0]
    token_order = np.concatenate([order, dead]).astype(np.int32)
    counts = np.bincount(slot_of[live], minlength=slots)[:slots]
    slot_indptr = np.zeros(slots + 1, dtype=np.int32)
    slot_indptr[1:] = np.cumsum(counts)
    assert token_order.shape == (T,)
    return token_order, slot_indptr


# ---------------------------------------------------------------------------
# Problem containers
# ---------------------------------------------------------------------------

@dataclass
class LinearProblem:
    """A linear (or embedding, when ``ids`` is set) target for one step."""
    name: str
    T: int
    n_in: int
    out_slices: tuple
    slots: int
    R: int
    x: np.ndarray | None          # uint16 [T, in]   (None for embedding)
    a: np.ndarray                 # uint16 [slots, S*R, in]
    b: np.ndarray                 # uint16 [slots, out, R]
    y: np.ndarray                 # uint16 [T, out]
    ranks: np.ndarray             # int32 [slots]
    scalings: np.ndarray          # float32 [slots]
    token_order: np.ndarray       # int32 [T]
    slot_indptr: np.ndarray       # int32 [slots+1]
    slot_of: np.ndarray           # int64 [T], -1 = dead
    ids: np.ndarray | None = None  # int32 [T] for an embedding target
    meta: dict = field(default_factory=dict)

    @property
    def num_slices(self):
        return len(self.out_slices)

    @property
    def out(self):
        return int(sum(self.out_slices))


@dataclass
class MoEProblem:
    """One MoE layer's expert fold inputs for one projection."""
    name: str
    rows_cap: int
    n_in: int
    out_slices: tuple
    slots: int
    num_experts: int
    num_pairs: int
    R: int
    x: np.ndarray                 # uint16 [rows_cap, in]   (sorted rows)
    y: np.ndarray                 # uint16 [rows_cap, out]  (sorted rows)
    a: np.ndarray                 # uint16 [P, S*R, in]
    b: np.ndarray                 # uint16 [P, out, R]
    pair_index: np.ndarray        # int32 [slots*E], -1 = not adapted
    ranks: np.ndarray             # int32 [slots]
    scalings: np.ndarray          # float32 [slots]
    row_slot: np.ndarray          # int32 [rows_cap], -1 = no adapter
    expert_offsets: np.ndarray    # int32 [E+1]
    meta: dict = field(default_factory=dict)

    @property
    def num_slices(self):
        return len(self.out_slices)

    @property
    def out(self):
        return int(sum(self.out_slices))


# ---------------------------------------------------------------------------
# Generic small problems (tests)
# ---------------------------------------------------------------------------

def random_linear(seed, T, n_in, out_slices, slots, R, ranks=None, scalings=None,
                  slot_of=None, dead_frac=0.0, x_std=1.0, ab_std=0.05, y_std=1.0,
                  embedding_vocab=None, bad_id_frac=0.0, name="random"):
    rng = np.random.default_rng(seed)
    out_slices = tuple(int(w) for w in out_slices)
    S = len(out_slices)
    out = sum(out_slices)
    if ranks is None:
        ranks = rng.choice([r for r in (0, 8, 16, 24, 32, 48, 64) if r <= R] or [R],
                           size=slots)
    ranks = np.asarray(ranks, dtype=np.int32)
    if scalings is None:
        scalings = np.where(ranks > 0, 2.0 / np.maximum(ranks, 1), 0.0)
    scalings = np.asarray(scalings, dtype=np.float32)
    if slot_of is None:
        slot_of = rng.integers(0, slots, size=T)
        if dead_frac > 0:
            slot_of[rng.random(T) < dead_frac] = -1
    slot_of = np.asarray(slot_of, dtype=np.int64)
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    vocab = embedding_vocab
    k_in = vocab if vocab is not None else n_in
    a = _normal_bf16(rng, (slots, S * R, k_in), ab_std)
    b = _normal_bf16(rng, (slots, out, R), ab_std)
    y = _normal_bf16(rng, (T, out), y_std)
    x = None
    ids = None
    if vocab is None:
        x = _normal_bf16(rng, (T, n_in), x_std)
    else:
        ids = rng.integers(0, vocab, size=T).astype(np.int32)
        if bad_id_frac > 0:
            ids[rng.random(T) < bad_id_frac] = -1
    return LinearProblem(name, T, k_in, out_slices, slots, R, x, a, b, y, ranks,
                         scalings, token_order, slot_indptr, slot_of, ids)


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------

def tiny_linear(seed=0):
    """T=64, in=256, out=256 (one slice), 4 slots of ranks (0,4,8,8), R=8,
    scaling 16/rank (0 for the rank-0 slot), slot(t) uniform;
    x ~ N(0,1), A,B ~ N(0,1)*0.05, y ~ N(0,1)."""
    rng = np.random.default_rng(1000 + seed)
    T, n_in, out, slots, R = 64, 256, 256, 4, 8
    ranks = np.array([0, 4, 8, 8], dtype=np.int32)
    scalings = np.array([0.0, 16 / 4, 16 / 8, 16 / 8], dtype=np.float32)
    slot_of = rng.integers(0, slots, size=T)
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    x = _normal_bf16(rng, (T, n_in), 1.0)
    a = _normal_bf16(rng, (slots, R, n_in), 0.05)
    b = _normal_bf16(rng, (slots, out, R), 0.05)
    y = _normal_bf16(rng, (T, out), 1.0)
    return LinearProblem("tiny_linear", T, n_in, (out,), slots, R, x, a, b, y, ranks,
                         scalings, token_order, slot_indptr, slot_of)


def zipf_slots(rng, T, slots, exponent=1.1):
    """slot(t) with P(s) proportional to (s+1)^-exponent on s = 0..slots-1."""
    p = (np.arange(1, slots + 1, dtype=np.float64)) ** (-exponent)
    p /= p.sum()
    return rng.choice(slots, size=T, p=p)


def decode_qkv(seed=0):
    """Decode over a fused QKV projection: T=256 (one token per request),
    in=4096, out_slices=(4096,1024,1024), 32 slots, R=16, rank per slot uniform
    in {8,16}, slot(t) Zipf(1.1), scaling 32/rank; x,y ~ N(0,1), A,B ~ N(0,0.02)."""
    rng = np.random.default_rng(2000 + seed)
    T, n_in, slots, R = 256, 4096, 32, 16
    out_slices = (4096, 1024, 1024)
    S, out = 3, 6144
    ranks = rng.choice([8, 16], size=slots).astype(np.int32)
    scalings = (32.0 / ranks).astype(np.float32)
    slot_of = zipf_slots(rng, T, slots)
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    x = _normal_bf16(rng, (T, n_in), 1.0)
    a = _normal_bf16(rng, (slots, S * R, n_in), 0.02)
    b = _normal_bf16(rng, (slots, out, R), 0.02)
    y = _normal_bf16(rng, (T, out), 1.0)
    return LinearProblem("decode_qkv", T, n_in, out_slices, slots, R, x, a, b, y, ranks,
                         scalings, token_order, slot_indptr, slot_of)


def geometric_requests(rng, T, mean_len, slots):
    """Requests with lengths ~ Geometric(1/mean_len) on {1,2,...} drawn until they
    cover T tokens (the last one clipped); each request's slot is uniform."""
    lens = []
    total = 0
    while total < T:
        n = int(rng.geometric(1.0 / mean_len))
        n = min(n, T - total)
        lens.append(n)
        total += n
    req_slot = rng.integers(0, slots, size=len(lens))
    slot_of = np.repeat(req_slot, lens)
    return slot_of, lens


def prefill_gate_up(seed=0, T=8192):
    """Prefill over a fused gate/up projection: T=8192 tokens of requests with
    geometric lengths (mean 512), in=4096, out_slices=(14336,14336), 16 slots,
    R=64, rank per slot uniform in {16,32,64}, scaling 32/rank;
    x,y ~ N(0,1), A,B ~ N(0,0.02)."""
    rng = np.random.default_rng(3000 + seed)
    n_in, slots, R = 4096, 16, 64
    out_slices = (14336, 14336)
    S, out = 2, 28672
    ranks = rng.choice([16, 32, 64], size=slots).astype(np.int32)
    scalings = (32.0 / ranks).astype(np.float32)
    slot_of, lens = geometric_requests(rng, T, 512, slots)
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    x = _normal_bf16(rng, (T, n_in), 1.0)
    a = _normal_bf16(rng, (slots, S * R, n_in), 0.02)
    b = _normal_bf16(rng, (slots, out, R), 0.02)
    y = _normal_bf16(rng, (T, out), 1.0)
    return LinearProblem("prefill_gate_up", T, n_in, out_slices, slots, R, x, a, b, y,
                         ranks, scalings, token_order, slot_indptr, slot_of,
                         meta={"request_lengths": lens})


def embedding(seed=0):
    """Embedding target: vocab 128256, out=4096, T=4096 ids uniform in
    [0, vocab) with 5% set to -1, 8 slots, slot(t) uniform, R=16, rank per slot
    uniform in {8,16}, scaling 2; A,B ~ N(0,0.02), y ~ N(0,1)."""
    rng = np.random.default_rng(4000 + seed)
    T, vocab, out, slots, R = 4096, 128256, 4096, 8, 16
    ranks = rng.choice([8, 16], size=slots).astype(np.int32)
    scalings = np.full(slots, 2.0, dtype=np.float32)
    slot_of = rng.integers(0, slots, size=T)
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    ids = rng.integers(0, vocab, size=T).astype(np.int32)
    ids[rng.random(T) < 0.05] = -1
    a = _normal_bf16(rng, (slots, R, vocab), 0.02)
    b = _normal_bf16(rng, (slots, out, R), 0.02)
    y = _normal_bf16(rng, (T, out), 1.0)
    return LinearProblem("embedding", T, vocab, (out,), slots, R, None, a, b, y, ranks,
                         scalings, token_order, slot_indptr, slot_of, ids)


def moe_routing(rng, T, num_experts, top_k, alpha=0.3):
    """Expert load p ~ Dirichlet(alpha); each token draws top_k distinct experts
    by Gumbel-top-k on log p.  Rows are (token, expert) pairs sorted by expert,
    stable by token.  Returns (row_token, row_expert, expert_offsets)."""
    p = rng.dirichlet(np.full(num_experts, alpha))
    logp = np.log(np.maximum(p, 1e-300))
    g = rng.gumbel(size=(T, num_experts))
    choice = np.argsort(-(logp[None, :] + g), axis=1)[:, :top_k]
    tok = np.repeat(np.arange(T), top_k)
    exp = choice.reshape(-1)
    order = np.lexsort((tok, exp))             # by expert, then token
    row_token = tok[order]
    row_expert = exp[order]
    counts = np.bincount(row_expert, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return row_token, row_expert, offsets.astype(np.int32)


def moe_expert(seed=0, T=2048, num_experts=128, top_k=8, hidden=2048, inter=768,
               slots=4, requests=16, adapted_frac=0.25, R=16, rank=16, scaling=2.0):
    """MoE expert fold for one layer: 128 experts, hidden 2048, moe_inter 768,
    top-8 of T=2048 tokens -> 16384 rows sorted by expert (Dirichlet(0.3) load).
    16 requests of 128 tokens, each with a slot uniform in 4 slots; every slot
    adapts an independent random 25% of the experts (gate, up and down);
    R = rank = 16, scaling 2; x, y ~ N(0,1), A,B ~ N(0,0.02).

    Returns ``(gate_up, down)``: the gate/up fold (in=hidden,
    out_slices=(inter, inter)) and the down fold (in=inter, out=hidden)."""
    rng = np.random.default_rng(5000 + seed)
    E = num_experts
    row_token, row_expert, offsets = moe_routing(rng, T, E, top_k)
    rows = len(row_token)
    per_req = T // requests
    req_slot = rng.integers(0, slots, size=requests)
    tok_slot = np.repeat(req_slot, per_req)
    if len(tok_slot) < T:
        tok_slot = np.concatenate([tok_slot, np.full(T - len(tok_slot), req_slot[-1])])
    row_slot = tok_slot[row_token].astype(np.int32)
    n_adapt = int(round(adapted_frac * E))
    pair_index = np.full((slots, E), -1, dtype=np.int32)
    P = 0
    for s in range(slots):
        for e in np.sort(rng.choice(E, size=n_adapt, replace=False)):
            pair_index[s, e] = P
            P += 1
    ranks = np.full(slots, rank, dtype=np.int32)
    scalings = np.full(slots, scaling, dtype=np.float32)
    hidden_states = _normal_bf16(rng, (T, hidden), 1.0)
    x_gu = hidden_states[row_token]
    y_gu = _normal_bf16(rng, (rows, 2 * inter), 1.0)
    a_gu = _normal_bf16(rng, (P, 2 * R, hidden), 0.02)
    b_gu = _normal_bf16(rng, (P, 2 * inter, R), 0.02)
    x_dn = _normal_bf16(rng, (rows, inter), 1.0)
    y_dn = _normal_bf16(rng, (rows, hidden), 1.0)
    a_dn = _normal_bf16(rng, (P, R, inter), 0.02)
    b_dn = _normal_bf16(rng, (P, hidden, R), 0.02)
    meta = {"row_token": row_token, "row_expert": row_expert}
    gu = MoEProblem("moe_gate_up", rows, hidden, (inter, inter), slots, E, P, R, x_gu,
                    y_gu, a_gu, b_gu, pair_index.reshape(-1).copy(), ranks, scalings,
                    row_slot, offsets, meta)
    dn = MoEProblem("moe_down", rows, inter, (hidden,), slots, E, P, R, x_dn, y_dn,
                    a_dn, b_dn, pair_index.reshape(-1).copy(), ranks, scalings, row_slot,
                    offsets, meta)
    return gu, dn


def moe_router(seed=0, T=2048, num_experts=128, hidden=2048, slots=4, requests=16, R=16,
               scaling=2.0):
    """Router LoRA on the MoE layer above: the routing logits [T=2048, 128 experts]
    of hidden 2048 take each token's router (mlp.gate) adapter delta before
    top-k.  16 requests of 128 tokens, each with a slot uniform in 4 slots;
    R = 16, rank per slot uniform in {8, 16}, scaling 2; router input and
    logits ~ N(0,1), A,B ~ N(0,0.02).  One output slice of 128 columns."""
    rng = np.random.default_rng(6000 + seed)
    per_req = T // requests
    req_slot = rng.integers(0, slots, size=requests)
    slot_of = np.repeat(req_slot, per_req)
    if len(slot_of) < T:
        slot_of = np.concatenate([slot_of, np.full(T - len(slot_of), req_slot[-1])])
    token_order, slot_indptr = csr_by_slot(slot_of, slots)
    ranks = rng.choice([8, 16], size=slots).astype(np.int32)
    scalings = np.full(slots, scaling, dtype=np.float32)
    x = _normal_bf16(rng, (T, hidden), 1.0)
    a = _normal_bf16(rng, (slots, R, hidden), 0.02)
    b = _normal_bf16(rng, (slots, num_experts, R), 0.02)
    y = _normal_bf16(rng, (T, num_experts), 1.0)
    return LinearProblem("moe_router", T, hidden, (num_experts,), slots, R, x, a, b, y, ranks,
                         scalings, token_order, slot_indptr, slot_of)


def random_moe(seed, rows_per_expert_max, num_experts, n_in, out_slices, slots, R,
               ranks=None, adapted_frac=0.5, no_slot_frac=0.1):
    """A small MoE fold problem with ragged expert row blocks (tests)."""
    rng = np.random.default_rng(seed)
    E = num_experts
    counts = rng.integers(0, rows_per_expert_max + 1, size=E)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    rows = int(offsets[-1])
    out_slices = tuple(int(w) for w in out_slices)
    S, out = len(out_slices), sum(out_slices)
    row_slot = rng.integers(0, slots, size=rows).astype(np.int32)
    row_slot[rng.random(rows) < no_slot_frac] = -1
    pair_index = np.full((slots, E), -1, dtype=np.int32)
    P = 0
    for s in range(slots):
        for e in range(E):
            if rng.random() < adapted_frac:
                pair_index[s, e] = P
                P += 1
    if ranks is None:
        ranks = rng.choice([r for r in (0, 8, 16) if r <= R], size=slots)
    ranks = np.asarray(ranks, dtype=np.int32)
    scalings = np.where(ranks > 0, 2.0, 0.0).astype(np.float32)
    x = _normal_bf16(rng, (max(rows, 1), n_in), 1.0)[:rows]
    y = _normal_bf16(rng, (max(rows, 1), out), 1.0)[:rows]
    a = _normal_bf16(rng, (max(P, 1), S * R, n_in), 0.05)
    b = _normal_bf16(rng, (max(P, 1), out, R), 0.05)
    return MoEProblem("random_moe", rows, n_in, out_slices, slots, E, P, R, x, y, a, b,
                      pair_index.reshape(-1).copy(), ranks, scalings, row_slot, offsets)


WORKLOADS = {
    "tiny_linear": tiny_linear,
    "decode_qkv": decode_qkv,
    "prefill_gate_up": prefill_gate_up,
    "embedding": embedding,
    "moe_expert": moe_expert,
    "moe_router": moe_router,
}
