"""Benchmark of the batched multi-LoRA delta path on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One JSON line on rank 0.  A step is one pass of the workload's whole delta path
over one batch (decode: one fused shrink+expand call over 256 tokens).  Inputs
are seeded and synthetic, resident in HBM before the timed region, and rotate
over enough independent sets (x, y, A, B, addressing) that the step's data is
never in L2 when it is reused.  Steps are replayed from CUDA graphs; time is
taken with CUDA events on the launching stream, max over ranks.  Each rank runs
its own batch (data-parallel replicas, no collective on the data path).

--impl reference times the fp64 CPU oracle (the parity reference) on the
host's cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from adapter_lora_serving_b200 import workloads as W  # noqa: E402

METRIC = "LoRA-apply tokens/s and achieved HBM GB/s (% of B200 roofline) per config"
L2_BYTES = 126 * 1024 * 1024
DESCR = {
    "tiny_linear": "tiny linear: T=64, in=256, out=256, slots=4 ranks (0,4,8,8), R=8",
    "decode_qkv": "decode BGMV fused QKV: T=256 (1 token/request), in=4096, "
                  "out_slices=(4096,1024,1024), slots=32 Zipf(1.1), R=16, ranks {8,16}",
    "prefill_gate_up": "prefill SGMV fused gate/up: T=8192 (geometric segments, mean 512), "
                       "in=4096, out_slices=(14336,14336), slots=16, R=64, ranks {16,32,64}",
    "embedding": "embedding gather_shrink+expand: vocab=128256, out=4096, T=4096 (5% id -1), "
                 "slots=8, R=16, ranks {8,16}",
    "moe_expert": "MoE expert LoRA: 128 experts, hidden=2048, moe_inter=768, top-8 of T=2048 "
                  "-> 16384 sorted rows, 4 slots, 25% experts adapted, R=16; gate/up + down folds",
    "moe_router": "MoE router LoRA: routing logits [T=2048, 128 experts], hidden=2048, "
                  "4 slots, R=16, ranks {8,16}; fold before top-k",
}


# ---------------------------------------------------------------------------
# Algorithmic bytes and FLOPs (what the method must move / compute)
# ---------------------------------------------------------------------------

def linear_cost(p, embedding=False):
    """(bytes, flops, live tokens) of one linear / embedding step."""
    S, out = p.num_slices, p.out
    bytes_ = (p.T + p.slots + 1) * 4 + p.slots * 8          # addressing, ranks, scalings
    flops = 0
    live = 0
    for s in range(p.slots):
        lo, hi = int(p.slot_indptr[s]), int(p.slot_indptr[s + 1])
        r = int(p.ranks[s])
        if hi <= lo or r == 0 or p.scalings[s] == 0:
            continue
        toks = p.token_order[lo:hi]
        if embedding:
            toks = toks[(p.ids[toks] >= 0) & (p.ids[toks] < p.n_in)]
            n = len(toks)
            if n == 0:
                continue
            bytes_ += n * S * r * 2 + n * 4                 # gathered A elements + ids
            flops += n * 2 * r * out
        else:
            n = len(toks)
            bytes_ += n * p.n_in * 2 + S * r * p.n_in * 2    # x rows, live A rows
            flops += n * 2 * r * (S * p.n_in + out)
        bytes_ += out * r * 2 + n * out * 4                   # live B columns, y read+write
        live += n
    return bytes_, flops, live


def moe_cost(m):
    S, out = m.num_slices, m.out
    pi = m.pair_index.reshape(m.slots, m.num_experts)
    bytes_ = (m.rows_cap + m.num_experts + 1 + m.slots * m.num_experts) * 4 + m.slots * 8
    flops = 0
    rows = 0
    used = set()
    for e in range(m.num_experts):
        lo, hi = int(m.expert_offsets[e]), int(m.expert_offsets[e + 1])
        for rho in range(lo, hi):
            s = int(m.row_slot[rho])
            if s < 0 or pi[s, e] < 0 or m.ranks[s] == 0 or m.scalings[s] == 0:
                continue
            r = int(m.ranks[s])
            rows += 1
            used.add((int(pi[s, e]), r))
            bytes_ += m.n_in * 2 + out * 4
            flops += 2 * r * (S * m.n_in + out)
    for _, r in used:
        bytes_ += S * r * m.n_in * 2 + out * r * 2
    return bytes_, flops, rows


# ---------------------------------------------------------------------------
# Workloads on the device
# ---------------------------------------------------------------------------

class Workload:
    """Rotating device input sets and the library call of one step."""

    def __init__(self, name, n_sets, seed0, torch, L, regime=None):
        self.name = name
        self.torch = torch
        self.L = L
        self.regime = L.LORA_REGIME_AUTO if regime is None else regime
        self.sets = []
        self.host_sets = []
        gen = W.WORKLOADS[name]
        for i in range(n_sets):
            prob = gen(seed0 + i)
            self.host_sets.append(prob)
            self.sets.append(self._to_device(prob))
        self.bytes, self.flops, self.tokens = self._cost(self.host_sets[0])

    # --- helpers
    def _bf16(self, bits):
        t = self.torch
        return t.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(t.bfloat16).cuda()

    def _i32(self, v):
        return self.torch.from_numpy(np.ascontiguousarray(v, dtype=np.int32)).cuda()

    def _f32(self, v):
        return self.torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).cuda()

    def _lin(self, p):
        d = dict(p=p, a=self._bf16(p.a), b=self._bf16(p.b), y=self._bf16(p.y),
                 ranks=self._i32(p.ranks), scalings=self._f32(p.scalings),
                 token_order=self._i32(p.token_order), slot_indptr=self._i32(p.slot_indptr))
        if p.x is not None:
            d["x"] = self._bf16(p.x)
        if p.ids is not None:
            d["ids"] = self._i32(p.ids)
        ws = self.L.lora_workspace_bytes(self.L.LORA_OP_APPLY_LINEAR, p.T, p.slots, p.R,
                                         p.num_slices, self.regime)
        d["ws_bytes"] = ws
        # zeroed once: the library keeps its counter header zeroed between calls
        d["ws"] = self.torch.zeros(max(ws, 16) // 4, dtype=self.torch.float32,
                                   device="cuda") if ws else None
        return d

    def _moe(self, m):
        # the workspace selects the fold grouped by (slot, expert); it needs
        # no initialisation
        ws = self.L.lora_workspace_bytes(self.L.LORA_OP_EXPERT_APPLY, m.rows_cap, m.num_experts,
                                         m.R, m.num_slices)
        return dict(m=m, x=self._bf16(m.x), y=self._bf16(m.y), a=self._bf16(m.a),
                    b=self._bf16(m.b), pair_index=self._i32(m.pair_index),
                    ranks=self._i32(m.ranks), scalings=self._f32(m.scalings),
                    row_slot=self._i32(m.row_slot), offsets=self._i32(m.expert_offsets),
                    ws=self.torch.empty(max(ws, 16) // 4, dtype=self.torch.int32,
                                        device="cuda") if ws else None,
                    ws_bytes=ws)

    def _to_device(self, prob):
        if self.name == "moe_expert":
            return [self._moe(m) for m in prob]
        return self._lin(prob)

    def _cost(self, prob):
        if self.name == "moe_expert":
            costs = [moe_cost(m) for m in prob]
            return (sum(c[0] for c in costs), sum(c[1] for c in costs),
                    prob[0].meta["row_token"].size // 8)
        if self.name == "embedding":
            b, f, _ = linear_cost(prob, embedding=True)
            return b, f, prob.T
        b, f, _ = linear_cost(prob)
        return b, f, prob.T

    @property
    def set_bytes(self):
        tot = 0
        for d in (self.sets[0] if isinstance(self.sets[0], list) else [self.sets[0]]):
            for v in d.values():
                if hasattr(v, "element_size"):
                    tot += v.numel() * v.element_size()
        return tot

    @property
    def launches_per_step(self):
        if self.name == "moe_expert":
            # per fold: the (slot, expert) grouping, the shrink and the expand
            return 6 if self.sets[0][0]["ws"] is not None else 2
        p = self.host_sets[0]
        op = self.L.LORA_OP_APPLY_EMBEDDING if self.name == "embedding" else \
            self.L.LORA_OP_APPLY_LINEAR
        reg = self.L.lora_resolve_regime(op, p.T, p.slots, p.R, p.num_slices) \
            if self.regime == self.L.LORA_REGIME_AUTO else self.regime
        if reg in (self.L.LORA_REGIME_SGMV, self.L.LORA_REGIME_STREAM) and self.name != "embedding":
            return 2
        return 1

    def step(self, i, stream=None):
        L = self.L
        d = self.sets[i % len(self.sets)]
        if self.name == "moe_expert":
            for q in d:
                m = q["m"]
                L.lora_expert_apply(q["x"], q["y"], q["a"], q["b"], q["pair_index"], q["ranks"],
                                    q["scalings"], q["row_slot"], q["offsets"], m.rows_cap,
                                    m.n_in, m.num_experts, m.slots, m.num_pairs, m.R,
                                    m.out_slices, workspace=q["ws"],
                                    workspace_bytes=q["ws_bytes"], stream=stream)
            return
        p = d["p"]
        if self.name == "embedding":
            L.lora_apply_embedding(d["ids"], d["y"], d["a"], d["b"], d["ranks"], d["scalings"],
                                   d["token_order"], d["slot_indptr"], p.T, p.n_in, p.slots, p.R,
                                   p.out_slices, regime=self.regime, stream=stream)
            return
        if self.name == "moe_router":
            L.lora_apply_router(d["x"], d["y"], d["a"], d["b"], d["ranks"], d["scalings"],
                                d["token_order"], d["slot_indptr"], p.T, p.n_in, p.slots, p.R,
                                p.out, regime=self.regime, workspace=d["ws"],
                                workspace_bytes=d["ws_bytes"], stream=stream)
            return
        L.lora_apply_linear(d["x"], d["y"], d["a"], d["b"], d["ranks"], d["scalings"],
                            d["token_order"], d["slot_indptr"], p.T, p.n_in, p.slots, p.R,
                            p.out_slices, regime=self.regime, workspace=d["ws"],
                            workspace_bytes=d["ws_bytes"], stream=stream)


def n_sets_for(name):
    """Input sets so that one rotation is larger than twice the L2."""
    per = {"tiny_linear": 0.13e6, "decode_qkv": 21.6e6, "prefill_gate_up": 1.2e9,
           "embedding": 70e6, "moe_expert": 110e6, "moe_router": 9.2e6}[name]
    return max(1, min(64, int(math.ceil(2.2 * L2_BYTES / per))))


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if not (t0 <= ts <= t1 + 0.05):
                continue
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# Timing
# ---------------------------------------------------------------------------

def capture(torch, wl, first, count, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(first, first + count):
            wl.step(i)
    return g


def rank_seed0(rank, n_sets):
    """First input seed of a rank's workload sets: rank r draws seeds
    [r * n_sets, (r + 1) * n_sets), so every replica runs its own batches."""
    return rank * n_sets


def reduce_max_over_ranks(torch, dist, value, device):
    """Max of a per-rank float over the default process group: the timed
    region of a multi-GPU run is the slowest rank's."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, world, sec):
    """Whole-job throughput: the units all ranks processed over the (max over
    ranks) timed seconds."""
    return units_per_rank_step * steps * world / sec


def graph_counts(total, inner):
    """Step counts of the graphs that run `total` steps in chunks of `inner`."""
    out = []
    if total >= inner:
        out.append(inner)
    if total % inner:
        out.append(total % inner)
    return out


def time_steps(torch, wl, steps, warmup, dist=None, sampler=None, load_s=0.0):
    """Run `warmup` steps, then time exactly `steps` steps replayed from CUDA
    graphs.  Every graph the timed region replays is captured (and replayed
    once) before the start event, and a short device-side delay is queued
    ahead of that event so that the host's graph submissions are not timed.
    With `load_s` > 0 the step is also replayed untimed for about that many
    seconds just before the timed region while `sampler` records the clocks.
    Returns (seconds for the timed steps (max over ranks), clock window)."""
    stream = torch.cuda.Stream()
    nset = len(wl.sets)
    # steps per graph: a whole number of rotations, so no set is reused early
    per = 256 if wl.tokens < 1024 else 16
    inner = nset * max(1, per // nset)
    warm = max(warmup, 3)
    # eager warm-up call (sets kernel attributes before any capture)
    with torch.cuda.stream(stream):
        wl.step(0)
    torch.cuda.synchronize()
    graphs = {}
    for c in sorted(set(graph_counts(steps, inner) + graph_counts(warm, inner) + [inner])):
        graphs[c] = capture(torch, wl, 0, c, stream)

    def run(total):
        done = 0
        while done < total:
            c = min(inner, total - done)
            graphs[c].replay()
            done += c

    with torch.cuda.stream(stream):
        for g in graphs.values():      # every graph runs once before timing
            g.replay()
        run(warm)
    torch.cuda.synchronize()
    t_load0 = time.time()
    if load_s > 0:
        with torch.cuda.stream(stream):
            t_end = time.time() + load_s
            while time.time() < t_end:
                graphs[inner].replay()
                torch.cuda.synchronize()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(200000)      # keeps the device busy while the graphs are queued
        e0.record(stream)
        run(steps)
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    sec = e0.elapsed_time(e1) / 1e3
    if dist is not None:
        sec = reduce_max_over_ranks(torch, dist, sec, "cuda")
    graphs.clear()
    return sec, (t_load0, t_wall1)


def time_e2e(torch, wl, steps):
    """Same metric through the public C-ABI calls with host buffers: every step
    copies its inputs from pinned host memory to the device and its result back."""
    L = wl.L
    p = wl.host_sets[0]
    stream = torch.cuda.Stream()
    if wl.name == "moe_expert":
        return None
    d = wl.sets[0]
    pin = {}
    names = ["y", "token_order", "slot_indptr"] + (["ids"] if wl.name == "embedding" else ["x"])
    for k in names:
        pin[k] = d[k].cpu().pin_memory()
    out = torch.empty_like(pin["y"]).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = out.numel() * out.element_size()
    dev = {k: torch.empty_like(d[k]) for k in names}
    torch.cuda.synchronize()

    def one():
        for k in names:
            dev[k].copy_(pin[k], non_blocking=True)
        if wl.name == "embedding":
            L.lora_apply_embedding(dev["ids"], dev["y"], d["a"], d["b"], d["ranks"],
                                   d["scalings"], dev["token_order"], dev["slot_indptr"], p.T,
                                   p.n_in, p.slots, p.R, p.out_slices, regime=wl.regime)
        elif wl.name == "moe_router":
            L.lora_apply_router(dev["x"], dev["y"], d["a"], d["b"], d["ranks"], d["scalings"],
                                dev["token_order"], dev["slot_indptr"], p.T, p.n_in, p.slots,
                                p.R, p.out, regime=wl.regime, workspace=d["ws"],
                                workspace_bytes=d["ws_bytes"])
        else:
            L.lora_apply_linear(dev["x"], dev["y"], d["a"], d["b"], d["ranks"], d["scalings"],
                                dev["token_order"], dev["slot_indptr"], p.T, p.n_in, p.slots,
                                p.R, p.out_slices, regime=wl.regime, workspace=d["ws"],
                                workspace_bytes=d["ws_bytes"])
        out.copy_(dev["y"], non_blocking=True)

    # plain calls with the library's defaults: every kernel follows this step's
    # host-to-device copies, so there is no kernel to overlap with
    prev = L.lora_set_launch_overlap(0)
    with torch.cuda.stream(stream):
        for _ in range(3):
            one()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(steps):
            one()
        e1.record(stream)
    torch.cuda.synchronize()
    L.lora_set_launch_overlap(prev)
    sec = e0.elapsed_time(e1) / 1e3
    return {"value": wl.tokens * steps / sec, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "launches": "eager calls from one host thread, launch overlap off"}


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

def oracle_step_fn(name, prob, frac=1.0, rng=None):
    """A callable running the fp64 oracle on a token sample of `prob`; returns tokens."""
    from oracle import lora_oracle as O
    f = W.bf16_to_f64
    if name == "moe_expert":
        gu, dn = prob
        args = []
        for m in (gu, dn):
            args.append((f(m.x), f(m.y), f(m.a), f(m.b), m))
        n_tok = gu.meta["row_token"].size // 8

        def run():
            keep = None
            if frac < 1.0:
                keep = (rng or np.random.default_rng(0)).random(gu.rows_cap) < frac
            for x, y, a, b, m in args:
                rs = m.row_slot if keep is None else np.where(keep, m.row_slot, -1)
                O.expert_apply(x, y, a, b, m.pair_index, m.ranks, m.scalings, rs,
                               m.expert_offsets, m.R, m.out_slices, m.slots, m.num_experts,
                               m.num_pairs)
            return n_tok * (1.0 if keep is None else keep.mean())
        return run
    x = f(prob.x) if prob.x is not None else None
    y, a, b = f(prob.y), f(prob.a), f(prob.b)

    def run():
        if frac < 1.0:
            k = max(1, int(round(prob.T * frac)))
            toks = (rng or np.random.default_rng(0)).choice(prob.T, size=k, replace=False)
            keep = np.zeros(prob.T, bool)
            keep[toks] = True
            to, ip = W.csr_by_slot(np.where(keep, prob.slot_of, -1), prob.slots)
        else:
            k, to, ip = prob.T, prob.token_order, prob.slot_indptr
        if name == "embedding":
            O.apply_embedding(prob.ids, y, a, b, to, ip, prob.ranks, prob.scalings,
                              prob.out_slices, prob.R, prob.n_in)
        elif name == "moe_router":
            O.apply_router(x, y, a, b, to, ip, prob.ranks, prob.scalings, prob.R)
        else:
            O.apply_linear(x, y, a, b, to, ip, prob.ranks, prob.scalings, prob.out_slices,
                           prob.R)
        return k
    return run


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def time_oracle(name, prob, budget_s=12.0, min_s=10.0):
    """Oracle throughput over a bounded sample: repeat the full step (or a token
    sample of it when one step alone exceeds the budget) for about min_s seconds."""
    run = oracle_step_fn(name, prob)
    t0 = time.perf_counter()
    tok = run()
    t1 = time.perf_counter() - t0
    frac = 1.0
    if t1 > budget_s:
        frac = budget_s / t1 / 4
        run = oracle_step_fn(name, prob, frac, np.random.default_rng(1))
    done_tok, reps = 0.0, 0
    t0 = time.perf_counter()
    while True:
        done_tok += run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_s or el > 3 * budget_s:
            break
    sample = (f"{reps} oracle step(s) of the full batch" if frac == 1.0 else
              f"{reps} oracle step(s) over a {frac:.3%} token sample of the batch")
    return done_tok / el, sample, el


# ---------------------------------------------------------------------------
# Profiles: DRAM traffic of the dominant kernel from a committed ncu summary
# ---------------------------------------------------------------------------

# Sources each kernel is built from: stored DRAM counters stay valid while
# these files are unchanged.
KERNEL_SOURCES = {
    "bgmv_kernel": ["bgmv.cu", "common.cuh", "kernels.h", "expand_tile.cuh"],
    "sgmv_expand_kernel": ["sgmv.cu", "sgmv.h", "tcgen05.cuh", "common.cuh", "kernels.h"],
    "sgmv_shrink_kernel": ["sgmv.cu", "sgmv.h", "tcgen05.cuh", "common.cuh", "kernels.h"],
    "stream_kernel": ["stream.cu", "common.cuh", "kernels.h", "expand_tile.cuh"],
    "group_shrink_kernel": ["group_shrink.cu", "common.cuh", "kernels.h"],
}


def source_digest(kernel):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "adapter_lora_serving_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# The kernel with the largest share of each workload's step under AUTO (the
# launch lists under profiles/).
DOMINANT = {"tiny_linear": "bgmv_kernel", "decode_qkv": "bgmv_kernel",
            "prefill_gate_up": "sgmv_expand_kernel", "embedding": "stream_kernel",
            "moe_expert": "stream_kernel", "moe_router": "group_shrink_kernel"}


def measured_traffic(name):
    """DRAM bytes per launch of the workload's dominant kernel from one ncu
    capture (profiles/traffic.json), or None when there is none or that
    kernel's sources differ from the ones the capture was taken at."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(name)
    except (OSError, ValueError):
        return None, DOMINANT.get(name)
    if not rec:
        return None, DOMINANT.get(name)
    kernel = rec.get("kernel")
    if kernel != DOMINANT.get(name) or kernel not in KERNEL_SOURCES or \
            rec.get("source_digest") != source_digest(kernel):
        return None, DOMINANT.get(name)
    return rec.get("dram_bytes_per_launch"), kernel


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), float(pk["bf16_tflops"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="decode_qkv", choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload table")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch each step's kernel only after the previous one has finished")
    ap.add_argument("--profile", action="store_true",
                    help="timed steps only (no e2e, CPU baseline or table): for ncu captures")
    ap.add_argument("--regime", default="auto",
                    choices=["auto", "bgmv", "sgmv", "bgmv_split", "stream"],
                    help="the headline workload's regime (the other rows of the table: auto)")
    ap.add_argument("--clock-window", type=float, default=0.4,
                    help="seconds of untimed replay of the step, under the clock sampler, "
                         "directly before the timed steps")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return reference_arm(args, world, rank)

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    from adapter_lora_serving_b200 import lora as L
    L.load()
    # consecutive steps overlap the few-tokens kernel's planning and A loads
    # with the previous step's tail (the library's opt-in launch overlap)
    if not args.no_overlap:
        L.lora_set_launch_overlap(1)

    name = args.workload
    nset = n_sets_for(name)
    regime = getattr(L, "LORA_REGIME_" + args.regime.upper())
    wl = Workload(name, nset, rank_seed0(rank, nset), torch, L, regime)
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        uuid = local
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.2)
    sec, (w0, w1) = time_steps(torch, wl, args.steps, args.warmup, dist, load_s=args.clock_window)
    sampler.stop()
    clocks = sampler.summary(w0, w1)
    clocks["window"] = (f"nvidia-smi every 50 ms over an untimed {args.clock_window:.1f} s replay "
                        f"of the same step directly before the timed steps, and the timed steps")

    ms_per_step = sec / args.steps * 1e3
    value = job_throughput(wl.tokens, args.steps, world, sec)
    hbm_peak, tf_peak, peak_kind = load_peaks()
    kernel_s = sec / (args.steps * wl.launches_per_step) if wl.launches_per_step == 1 else None
    step_gbs = wl.bytes / (sec / args.steps) / 1e9
    traffic, kname = measured_traffic(name)
    if args.regime != "auto":
        # the captures behind traffic.json are of the AUTO regime's kernel
        traffic, kname = None, None
    roofline = {"bound": "hbm", "achieved": round(step_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(step_gbs / hbm_peak, 4), "traffic": traffic,
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                "algorithmic_bytes_per_step": int(wl.bytes),
                "kernel": kname,
                "per_launch_us": round(kernel_s * 1e6, 3) if kernel_s else None}

    e2e = time_e2e(torch, wl, args.e2e_steps) if rank == 0 and not args.profile else None

    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded numpy draws, random-init adapters)",
           "config": {"workload": DESCR[name], "tokens_per_step_per_gpu": wl.tokens,
                      "global_batch": wl.tokens * world,
                      "parallelism": f"replicas x{world} (independent batches, no collective)",
                      "l2": f"inputs rotate over {len(wl.sets)} independent sets "
                            f"({len(wl.sets) * wl.set_bytes / 1e6:.0f} MB > 2x L2)",
                      "timing": "CUDA-graph replay (every graph captured and replayed once "
                                "before the start event; a device-side delay queued ahead of "
                                "it), CUDA events on the launching stream",
                      "launch_overlap": "off" if args.no_overlap else
                      "programmatic dependent launch between consecutive steps"},
           "roofline": roofline, "clocks": clocks,
           "gpu_launches": args.steps * wl.launches_per_step, "e2e": e2e}

    if rank == 0 and world == 1 and not args.profile:
        rate, sample, el = time_oracle(name, wl.host_sets[0])
        out["cpu_baseline"] = {"value": round(rate, 2), "unit": "tokens/s",
                               "cores": cpu_threads(), "kind": "oracle",
                               "sample": f"{sample} ({el:.1f} s, fp64 numpy oracle)"}
    if rank == 0 and world == 1 and not (args.no_configs or args.profile):
        out["configs"] = config_table(torch, L, name, wl, sec / args.steps, hbm_peak)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def config_table(torch, L, headline, wl_head, head_step_s, hbm_peak):
    """Per-workload throughput (the other configs are measured the same way,
    with fewer steps)."""
    rows = {}
    for name in W.WORKLOADS:
        if name == headline:
            wl, step_s = wl_head, head_step_s
        else:
            wl = Workload(name, n_sets_for(name), 100, torch, L)
            steps = 2000 if wl.tokens <= 512 else 200
            sec, _ = time_steps(torch, wl, steps, 20)
            step_s = sec / steps
        gbs = wl.bytes / step_s / 1e9
        rows[name] = {"tokens_per_s": round(wl.tokens / step_s, 1),
                      "us_per_step": round(step_s * 1e6, 3),
                      "algorithmic_MB": round(wl.bytes / 1e6, 3),
                      "GBps": round(gbs, 1), "frac_hbm": round(gbs / hbm_peak, 4),
                      "TFLOPps": round(wl.flops / step_s / 1e12, 3),
                      "launches_per_step": wl.launches_per_step}
        if name != headline:
            del wl
            torch.cuda.empty_cache()
    return rows


def reference_arm(args, world, rank):
    """The oracle (the parity reference) timed on the host's cores."""
    if rank != 0:
        return
    name = args.workload
    prob = W.WORKLOADS[name](0)
    run = oracle_step_fn(name, prob)
    t0 = time.perf_counter()
    run()
    t1 = time.perf_counter() - t0
    budget = 90.0
    total = max(args.steps, 1) + max(args.warmup, 0)
    frac = min(1.0, budget / (total * t1)) if t1 > 0 else 1.0
    run = oracle_step_fn(name, prob, frac, np.random.default_rng(2)) if frac < 1.0 else run
    for _ in range(args.warmup):
        run()
    tok = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        tok += run()
    el = time.perf_counter() - t0
    value = tok / el
    sample = (f"{args.steps} oracle steps of the full batch" if frac == 1.0 else
              f"{args.steps} oracle steps over a {frac:.3%} token sample each")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(el / max(args.steps, 1) * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": DESCR[name]},
           "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cpu_threads(),
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
