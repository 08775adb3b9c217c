"""Plain fp64 CPU oracle for the batched multi-LoRA delta path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, links or runs
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA library (it does not import the package, and the package
does not import it).  Inputs arrive as float64 arrays holding the exact values
of the bf16 tensors (bf16 -> fp64 is exact); every sum is taken in fp64.

What it computes, and where each rule comes from (page title, section):

* ``mstar.engine.resources.lora.backend`` (module text): shrink is
  ``h = x @ A^T`` and expand is ``y += s * h @ B^T``; shapes
  ``x [T, in]``, ``y [T, out]`` (in place), ``h [T, slices*R]``,
  ``a [slots, slices*R, in]``, ``b [slots, out, R]``, ranks/scalings ``[slots]``;
  slice i reads ``h[:, i*R:(i+1)*R]`` and writes its own columns of y.
* same page, ``LoraBackend.shrink``: rows of rank-0 slots and columns past a
  slot's rank are unspecified (the expand never reads them).
* same page, ``LoraBackend.expand_fused``:
  ``y[t, slice i] += scalings[slot(t)] * h[t, slice i] @ b[slot(t), slice i]^T``
  over the first ``rank`` columns of the slice.
* same page, ``LoraBackend.gather_shrink``: ``h[t] = a[slot(t)][:, ids[t]]``;
  an id outside ``[0, in)`` contributes nothing.
* same page, ``expand_reference_`` / ``shrink_reference`` signatures: the
  addressing is ``(token_order, slot_indptr)``, read here as CSR by slot.
* ``mstar.model.components.linear``, ``FusedColumnLinear`` (``shard_sizes``):
  the output columns of a fused projection are the shards in the given order,
  so slice i starts at the exclusive prefix sum of ``out_slices``.
* ``spark_model/lora/target.rs``, ``ExpertLoraLayer::adapted_experts``: the
  adapted experts are the sorted, de-duplicated expert ids of the stored pairs.
* ``spark_model/lora/expert_apply.rs``, ``expert_delta_workitems``: one work
  item ``(expert, row_off, rows)`` per adapted expert with routed rows, in
  adapted-list order; experts out of range, empty or malformed are skipped.
* same page, ``fold_chunked``: a work item longer than ``max_rows`` is folded as
  ``ceil(rows/max_rows)`` consecutive disjoint row blocks; each row is
  independent, so the result equals one fold.
* same page, ``apply_expert_lora_sorted``: the expert fold adds each adapted
  expert's delta onto its contiguous row block of the sorted output, in place.
* same page, ``apply_router_lora`` and its module text: the router (``mlp.gate``)
  adapter's delta is one delta fold onto the ``[n, num_experts]`` routing
  logits, in place, before top-k selection; ``spark_model/lora/target.rs``,
  ``router_dims``: the router projection is ``[num_experts, hidden]``.

Readings where the pages are silent (each one is listed with its reason in the
design notes of the repository):

* addressing: slot s owns slot-sorted positions
  ``[slot_indptr[s], slot_indptr[s+1])`` and ``token_order[p]`` is the token at
  position p.  A segment is valid iff ``0 <= lo <= hi <= T``; an invalid one is
  skipped and raises ``FLAG_BAD_INDPTR``.  A rank outside ``[0, R]`` skips the
  slot and raises ``FLAG_BAD_RANK``.  A token outside ``[0, T)`` is skipped and
  raises ``FLAG_BAD_TOKEN``.  Tokens listed nowhere ("dead") are untouched.
* a slot takes part only if its rank is > 0 and, for the operations that scale
  (expand, fused apply, fused embedding, expert fold), its scaling is != 0;
  otherwise y stays bit-identical.
* ``h`` is fp32 on the device; entries outside the live columns of live tokens
  are unspecified (returned here as NaN together with a mask).
* MoE: ``row_slot[row]`` is the slot of the row's request (-1 = none); the pair
  is ``pair_index[slot, expert]`` (-1 = not adapted); ranks and scalings are per
  slot.  A row slot outside ``[-1, slots)`` raises ``FLAG_BAD_SLOT``, a pair
  outside ``[-1, num_pairs)`` raises ``FLAG_BAD_PAIR``; offsets with
  ``start < 0``, ``end > rows_cap`` or ``end < start`` raise ``FLAG_BAD_OFFSETS``
  and skip the expert.

Parity pins for every function here live in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import numpy as np

# Error-flag bits reported by the device, restated here from the contract.
FLAG_BAD_INDPTR = 1
FLAG_BAD_TOKEN = 2
FLAG_BAD_RANK = 4
FLAG_BAD_SLOT = 8
FLAG_BAD_PAIR = 16
FLAG_BAD_OFFSETS = 32


class DuplicateTokenError(ValueError):
    """A token appears at more than one live position: the result is undefined."""


def slice_offsets(out_slices):
    """Column offset of each slice: exclusive prefix sum of ``out_slices`` in the
    given order (``FusedColumnLinear``: shards laid out in iteration order)."""
    offs = [0]
    for w in out_slices:
        offs.append(offs[-1] + int(w))
    return offs


# ---------------------------------------------------------------------------
# Addressing and planning
# ---------------------------------------------------------------------------

def resolve_slots(token_order, slot_indptr, ranks, T, R, scalings=None):
    """Per-slot lists of live tokens that take part, in slot then position order.

    ``scalings is None`` selects the unscaled operations (shrink and gather),
    for which a zero scaling does not matter.  Returns ``(groups, flags)`` with
    ``groups = [(slot, [token, ...]), ...]``.
    """
    flags = 0
    slots = len(slot_indptr) - 1
    groups = []
    seen = set()
    for s in range(slots):
        lo = int(slot_indptr[s])
        hi = int(slot_indptr[s + 1])
        r = int(ranks[s])
        seg_ok = 0 <= lo <= hi <= T
        rank_ok = 0 <= r <= R
        if not seg_ok:
            flags |= FLAG_BAD_INDPTR
        if not rank_ok:
            flags |= FLAG_BAD_RANK
        if not (seg_ok and rank_ok) or r == 0:
            continue
        if scalings is not None and float(scalings[s]) == 0.0:
            continue
        toks = []
        for p in range(lo, hi):
            t = int(token_order[p])
            if 0 <= t < T:
                if t in seen:
                    raise DuplicateTokenError(f"token {t} is listed twice")
                seen.add(t)
                toks.append(t)
            else:
                flags |= FLAG_BAD_TOKEN
        groups.append((s, toks))
    return groups, flags


def plan_segments(slot_indptr, ranks, T, R, tile, scalings=None):
    """Work items ``(slot, first_position, count)`` over the slots that take part:
    each slot's positions cut into consecutive tiles of at most ``tile``
    positions, slots in ascending order.  A tile may contain positions whose
    token is out of range; those are skipped when the tile is processed."""
    items = []
    slots = len(slot_indptr) - 1
    for s in range(slots):
        lo = int(slot_indptr[s])
        hi = int(slot_indptr[s + 1])
        r = int(ranks[s])
        if not (0 <= lo <= hi <= T) or not (0 < r <= R):
            continue
        if scalings is not None and float(scalings[s]) == 0.0:
            continue
        p = lo
        while p < hi:
            n = min(tile, hi - p)
            items.append((s, p, n))
            p += n
    return items


# ---------------------------------------------------------------------------
# Linear target: shrink, expand, fused apply (vectorised per slot)
# ---------------------------------------------------------------------------

def shrink(x, a, token_order, slot_indptr, ranks, R, num_slices):
    """``h[t, i*R + r] = sum_k x[t, k] * a[s, i*R + r, k]`` for r < rank[s].

    Returns ``(h, mask, flags)``: h is fp64 ``[T, S*R]`` with NaN where the
    value is unspecified, mask is True where it is specified."""
    T = x.shape[0]
    S = int(num_slices)
    h = np.full((T, S * R), np.nan)
    mask = np.zeros((T, S * R), dtype=bool)
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R)
    for s, toks in groups:
        if not toks:
            continue
        r = int(ranks[s])
        X = x[toks]                                 # [n, in]
        for i in range(S):
            rows = slice(i * R, i * R + r)
            h[np.ix_(toks, range(i * R, i * R + r))] = X @ a[s, rows, :].T
            mask[np.ix_(toks, range(i * R, i * R + r))] = True
    return h, mask, flags


def expand(y, h, b, token_order, slot_indptr, ranks, scalings, out_slices, R):
    """``y[t, off_i + j] += scal[s] * sum_{r<rank} h[t, i*R + r] * b[s, off_i + j, r]``.

    Returns ``(y_ref, touched, flags)``: y_ref is fp64; rows not touched are
    copies of the input (bit-identical)."""
    T = y.shape[0]
    offs = slice_offsets(out_slices)
    y_ref = np.array(y, dtype=np.float64, copy=True)
    touched = np.zeros(T, dtype=bool)
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R, scalings)
    for s, toks in groups:
        if not toks:
            continue
        r = int(ranks[s])
        sc = float(scalings[s])
        for i, w in enumerate(out_slices):
            H = h[np.ix_(toks, range(i * R, i * R + r))]          # [n, r]
            Bs = b[s, offs[i]:offs[i] + w, :r]                   # [w, r]
            y_ref[np.ix_(toks, range(offs[i], offs[i] + w))] += sc * (H @ Bs.T)
        touched[toks] = True
    return y_ref, touched, flags


def apply_linear(x, y, a, b, token_order, slot_indptr, ranks, scalings, out_slices, R):
    """Shrink then expand into y (``LoraBackend.apply_linear_``)."""
    S = len(out_slices)
    T = x.shape[0]
    h = np.zeros((T, S * R))
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R, scalings)
    for s, toks in groups:
        if toks:
            h[toks] = x[toks] @ a[s].T
    y_ref, touched, f2 = expand(y, h, b, token_order, slot_indptr, ranks, scalings,
                                out_slices, R)
    return y_ref, touched, flags | f2


# ---------------------------------------------------------------------------
# Embedding target: gather_shrink and the fused gather + expand
# ---------------------------------------------------------------------------

def gather_shrink(ids, a, token_order, slot_indptr, ranks, R, num_slices, vocab):
    """``h[t, i*R + r] = a[s, i*R + r, ids[t]]``; an id outside ``[0, vocab)`` gives
    a zero row (the shrink of an all-zero one-hot).  Returns ``(h, mask, flags)``."""
    T = len(ids)
    S = int(num_slices)
    h = np.full((T, S * R), np.nan)
    mask = np.zeros((T, S * R), dtype=bool)
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R)
    for s, toks in groups:
        r = int(ranks[s])
        for t in toks:
            v = int(ids[t])
            for i in range(S):
                cols = range(i * R, i * R + r)
                h[t, cols] = a[s, i * R:i * R + r, v] if 0 <= v < vocab else 0.0
                mask[t, cols] = True
    return h, mask, flags


def apply_embedding(ids, y, a, b, token_order, slot_indptr, ranks, scalings,
                    out_slices, R, vocab):
    """Gather then expand (``LoraBackend.apply_`` with ``embedding=True``).  A token
    whose id is outside ``[0, vocab)`` contributes nothing, so its row of y is
    left bit-identical."""
    T = len(ids)
    S = len(out_slices)
    offs = slice_offsets(out_slices)
    y_ref = np.array(y, dtype=np.float64, copy=True)
    touched = np.zeros(T, dtype=bool)
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R, scalings)
    for s, toks in groups:
        r = int(ranks[s])
        sc = float(scalings[s])
        live = [t for t in toks if 0 <= int(ids[t]) < vocab]
        if not live:
            continue
        v = np.array([int(ids[t]) for t in live])
        for i, w in enumerate(out_slices):
            H = a[s, i * R:i * R + r, :][:, v].T                # [n, r]
            Bs = b[s, offs[i]:offs[i] + w, :r]
            y_ref[np.ix_(live, range(offs[i], offs[i] + w))] += sc * (H @ Bs.T)
        touched[live] = True
    return y_ref, touched, flags


# ---------------------------------------------------------------------------
# MoE expert fold
# ---------------------------------------------------------------------------

def adapted_experts(pair_index, slots, num_experts):
    """Sorted, de-duplicated experts that hold a pair for any slot
    (``ExpertLoraLayer::adapted_experts``)."""
    pi = np.asarray(pair_index).reshape(slots, num_experts)
    keys = []
    for s in range(slots):
        for e in range(num_experts):
            if int(pi[s, e]) != -1:
                keys.append(e)
    keys.sort()
    out = []
    for e in keys:                       # dedup of consecutive equal keys
        if not out or out[-1] != e:
            out.append(e)
    return out


def expert_workitems(expert_offsets, adapted, rows_cap):
    """``(expert, row_off, rows)`` per adapted expert with routed rows, in the
    adapted list's order (``expert_delta_workitems``).  Returns ``(work, flags)``."""
    n_experts = max(len(expert_offsets) - 1, 0)
    work = []
    flags = 0
    for e in adapted:
        e = int(e)
        if e < 0 or e >= n_experts:
            continue                      # not in this layer's routing table
        start = int(expert_offsets[e])
        end = int(expert_offsets[e + 1])
        if start < 0 or end > rows_cap or end < start:
            flags |= FLAG_BAD_OFFSETS
            continue
        if end == start:
            continue                      # no rows routed to this expert
        work.append((e, start, end - start))
    return work, flags


def chunk_workitems(work, max_rows):
    """Split each item into ``ceil(rows/max_rows)`` consecutive row blocks
    (``fold_chunked``)."""
    step = max(int(max_rows), 1)
    out = []
    for e, off, rows in work:
        done = 0
        while done < rows:
            m = min(rows - done, step)
            out.append((e, off + done, m))
            done += m
    return out


def plan_expert(expert_offsets, pair_index, slots, num_experts, rows_cap, max_rows):
    """The chunked work-item list of the expert fold."""
    work, flags = expert_workitems(expert_offsets,
                                   adapted_experts(pair_index, slots, num_experts),
                                   rows_cap)
    return chunk_workitems(work, max_rows), flags


def _fold_rows(x, y_ref, touched, rows, e, a, b, pair_index, ranks, scalings,
               row_slot, slots, num_experts, num_pairs, R, out_slices):
    """Fold expert e's delta onto the given sorted rows; returns flags."""
    flags = 0
    offs = slice_offsets(out_slices)
    pi = np.asarray(pair_index).reshape(slots, num_experts)
    for rho in rows:
        s = int(row_slot[rho])
        if s == -1:
            continue
        if s < -1 or s >= slots:
            flags |= FLAG_BAD_SLOT
            continue
        p = int(pi[s, e])
        if p == -1:
            continue
        if p < -1 or p >= num_pairs:
            flags |= FLAG_BAD_PAIR
            continue
        r = int(ranks[s])
        if r < 0 or r > R:
            flags |= FLAG_BAD_RANK
            continue
        sc = float(scalings[s])
        if r == 0 or sc == 0.0:
            continue
        hx = a[p] @ x[rho]                                  # [S*R]
        for i, w in enumerate(out_slices):
            hi = hx[i * R:i * R + r]
            y_ref[rho, offs[i]:offs[i] + w] += sc * (b[p, offs[i]:offs[i] + w, :r] @ hi)
        touched[rho] = True
    return flags


def expert_apply(x, y, a, b, pair_index, ranks, scalings, row_slot, expert_offsets,
                 R, out_slices, slots, num_experts, num_pairs, max_rows=128):
    """The expert fold as the per-expert loop over chunked work items
    (``apply_expert_lora_sorted`` with a per-row slot).  Returns
    ``(y_ref, touched, flags)``."""
    rows_cap = x.shape[0]
    y_ref = np.array(y, dtype=np.float64, copy=True)
    touched = np.zeros(rows_cap, dtype=bool)
    items, flags = plan_expert(expert_offsets, pair_index, slots, num_experts,
                               rows_cap, max_rows)
    for e, off, m in items:
        flags |= _fold_rows(x, y_ref, touched, range(off, off + m), e, a, b,
                            pair_index, ranks, scalings, row_slot, slots,
                            num_experts, num_pairs, R, out_slices)
    return y_ref, touched, flags


# ---------------------------------------------------------------------------
# Router fold
# ---------------------------------------------------------------------------

def apply_router(router_in, logits, a, b, token_order, slot_indptr, ranks, scalings, R):
    """The router adapter's delta onto the routing logits, before top-k
    (``apply_router_lora``): ``logits [T, E] += s * (router_in @ A^T) @ B^T`` per
    token's slot, with ``a [slots, R, hidden]`` and ``b [slots, E, R]``.  The
    page folds it with the same delta routine as a dense projection, so it is
    the fused apply with a single output slice of ``E`` columns.  Returns
    ``(logits_ref, touched, flags)``."""
    E = logits.shape[1]
    return apply_linear(router_in, logits, a, b, token_order, slot_indptr, ranks, scalings,
                        (E,), R)


def top_k_experts(logits, k):
    """The ``k`` experts with the largest logits per token, largest first (ties
    to the lower expert id): the selection that follows the router fold."""
    out = []
    for row in np.asarray(logits, dtype=np.float64):
        order = sorted(range(len(row)), key=lambda e: (-row[e], e))
        out.append(order[:k])
    return out


# ---------------------------------------------------------------------------
# Brute-force forms (pure Python loops, tiny inputs only)
# ---------------------------------------------------------------------------

def brute_apply_linear(x, y, a, b, token_order, slot_indptr, ranks, scalings,
                       out_slices, R):
    """Token by token, element by element: the definition with no matmul."""
    T, n_in = x.shape
    offs = slice_offsets(out_slices)
    y_ref = np.array(y, dtype=np.float64, copy=True)
    groups, flags = resolve_slots(token_order, slot_indptr, ranks, T, R, scalings)
    for s, toks in groups:
        r = int(ranks[s])
        sc = float(scalings[s])
        for t in toks:
            for i, w in enumerate(out_slices):
                hv = []
                for rr in range(r):
                    acc = 0.0
                    for k in range(n_in):
                        acc += float(x[t, k]) * float(a[s, i * R + rr, k])
                    hv.append(acc)
                for j in range(w):
                    d = 0.0
                    for rr in range(r):
                        d += hv[rr] * float(b[s, offs[i] + j, rr])
                    y_ref[t, offs[i] + j] += sc * d
    return y_ref, flags


def brute_expert_apply(x, y, a, b, pair_index, ranks, scalings, row_slot,
                       expert_offsets, R, out_slices, slots, num_experts, num_pairs):
    """Row by row with no planner: each row finds its expert by scanning the
    offsets (well-formed, non-overlapping offsets only)."""
    rows_cap, n_in = x.shape
    offs = slice_offsets(out_slices)
    y_ref = np.array(y, dtype=np.float64, copy=True)
    pi = np.asarray(pair_index).reshape(slots, num_experts)
    for rho in range(rows_cap):
        e = -1
        for ee in range(num_experts):
            if int(expert_offsets[ee]) <= rho < int(expert_offsets[ee + 1]):
                e = ee
        if e < 0:
            continue
        s = int(row_slot[rho])
        if not (0 <= s < slots):
            continue
        p = int(pi[s, e])
        if not (0 <= p < num_pairs):
            continue
        r = int(ranks[s])
        sc = float(scalings[s])
        if r == 0 or sc == 0.0:
            continue
        for i, w in enumerate(out_slices):
            hv = []
            for rr in range(r):
                acc = 0.0
                for k in range(n_in):
                    acc += float(x[rho, k]) * float(a[p, i * R + rr, k])
                hv.append(acc)
            for j in range(w):
                d = 0.0
                for rr in range(r):
                    d += hv[rr] * float(b[p, offs[i] + j, rr])
                y_ref[rho, offs[i] + j] += sc * d
    return y_ref


# ---------------------------------------------------------------------------
# Comparison helpers used by the parity tests
# ---------------------------------------------------------------------------

ATOL = 1e-2
RTOL = 1.6e-2


def within_tolerance(y_dev, y_ref):
    """Elementwise ``|y_dev - y_ref| <= 1e-2 + 1.6e-2 * |y_ref|``."""
    y_dev = np.asarray(y_dev, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    return np.abs(y_dev - y_ref) <= ATOL + RTOL * np.abs(y_ref)
