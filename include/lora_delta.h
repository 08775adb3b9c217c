/*
 * lora_delta.h -- C ABI of the B200 (sm_100a) batched multi-LoRA delta library.
 *
 * Each token (or sorted MoE row) carries an adapter slot.  The library adds
 * the slot's low-rank delta to a projection's output in place:
 *
 *   shrink  h[t, i*R + r] = sum_k x[t, k] * a[slot, i*R + r, k]      (r < rank)
 *   expand  y[t, off_i + j] += scaling[slot] * sum_{r<rank} h[t, i*R + r] * b[slot, off_i + j, r]
 *
 * Sources (page title, section):
 *   mstar.engine.resources.lora.backend -- module text (shapes, slices),
 *     LoraBackend.shrink / expand_fused / apply_linear_ / apply_ / gather_shrink,
 *     and the addressing (token_order, slot_indptr) of shrink_reference,
 *     expand_reference_ and gather_shrink_reference.
 *   mstar.model.components.linear -- FusedColumnLinear (shards laid out in order).
 *   spark_model/lora/expert_apply.rs -- expert_delta_workitems, fold_chunked,
 *     apply_expert_lora_sorted (the expert fold over expert_offsets).
 *   spark_model/lora/target.rs -- ExpertLoraLayer (sparse per-expert pairs,
 *     adapted_experts), expert_router_bytes (uint4-aligned packed rank stride).
 *
 * Conventions for every entry point:
 *   - Pointers are DEVICE pointers unless marked "host".  bf16 tensors are
 *     passed as void* and are row-major and contiguous.  Every device pointer
 *     must be 16-byte aligned.
 *   - The caller owns every buffer.  The library never allocates device
 *     memory and keeps no state between calls except a per-device cache of
 *     kernel attributes (SM count, occupancy), the process-wide launch
 *     overlap and wait-limit settings (lora_set_launch_overlap,
 *     lora_set_wait_limit_ns) and the fixed scratch array of
 *     lora_apply_linear_noalloc, which is part of the library image.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises with the host.  The launch shape
 *     depends only on the scalar arguments, so calls can be captured in a CUDA
 *     graph.
 *   - Host-checkable errors return a non-LORA_OK status before anything is
 *     launched.  lora_last_error() then gives a message (thread-local).
 *   - Bad addressing that is only visible on the device is skipped, never
 *     trapped, and ORed into *err_flags when err_flags is not NULL (bits
 *     LORA_FLAG_*).  err_flags is never cleared by the library.
 *   - Shape rules (uint4 = 16-byte packing of bf16 rows, after the packed rank
 *     stride of expert_router_bytes): in_features % 8 == 0, R % 8 == 0,
 *     every out_slices[i] % 8 == 0, 1 <= num_slices <= LORA_MAX_SLICES.
 *
 * Addressing (CSR by slot): slot s owns slot-sorted positions
 * [slot_indptr[s], slot_indptr[s+1]); token_order[p] is the token at position p.
 * A segment is used only if 0 <= lo <= hi <= T (else LORA_FLAG_BAD_INDPTR) and
 * the slot's rank is in [0, R] (else LORA_FLAG_BAD_RANK).  Positions whose
 * token is outside [0, T) are skipped (LORA_FLAG_BAD_TOKEN).  Tokens listed in
 * no segment are untouched.  A slot with rank 0 -- or, for the operations
 * that scale, scaling 0 -- leaves y bit-identical.  A token listed twice gives
 * an unspecified result.
 */
#ifndef LORA_DELTA_H
#define LORA_DELTA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LORA_API __attribute__((visibility("default")))
#else
#define LORA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LORA_OK = 0,
  LORA_ERR_INVALID = 1,      /* a host-checkable argument is wrong; nothing launched */
  LORA_ERR_UNSUPPORTED = 2,  /* valid, but beyond this library's limits */
  LORA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
  LORA_ERR_CUDA = 4          /* a CUDA runtime call or a launch failed */
} lora_status;

/* Device-side error flags, ORed into *err_flags. */
#define LORA_FLAG_BAD_INDPTR  1u   /* a slot segment outside 0 <= lo <= hi <= T */
#define LORA_FLAG_BAD_TOKEN   2u   /* token_order entry outside [0, T) */
#define LORA_FLAG_BAD_RANK    4u   /* rank outside [0, R] */
#define LORA_FLAG_BAD_SLOT    8u   /* MoE row_slot outside [-1, slots) */
#define LORA_FLAG_BAD_PAIR   16u   /* MoE pair_index outside [-1, num_pairs) */
#define LORA_FLAG_BAD_OFFSETS 32u  /* MoE expert offsets with start < 0, end > rows_cap or end < start */
#define LORA_FLAG_TIMEOUT    64u   /* a bounded device wait expired; the call's output is incomplete */

/* Regime hint.  AUTO picks from the scalar shapes only (tokens per slot). */
#define LORA_REGIME_AUTO 0
#define LORA_REGIME_BGMV 1   /* few tokens per slot: thread-block-cluster kernel, h kept on chip */
#define LORA_REGIME_SGMV 2   /* many tokens per slot: tcgen05/TMEM tiles over slot segments */
#define LORA_REGIME_BGMV_SPLIT 3  /* few tokens per slot, the work split by bytes over every SM
                                     (lora_apply_linear only; needs a zeroed workspace) */
#define LORA_REGIME_STREAM 4 /* output rows streamed in 16-row groups by every SM, the delta
                                from warp MMAs (lora_apply_embedding: AUTO's choice there;
                                lora_apply_linear: after a short-segment shrink, AUTO's
                                choice for mid-size batches) */

#define LORA_MAX_SLICES 8
#define LORA_MAX_SLOTS 4096
#define LORA_MAX_EXPERTS 4096

/* Operation ids for lora_plan_tile / lora_workspace_bytes. */
#define LORA_OP_SHRINK 0
#define LORA_OP_EXPAND 1
#define LORA_OP_APPLY_LINEAR 2
#define LORA_OP_GATHER_SHRINK 3
#define LORA_OP_APPLY_EMBEDDING 4
#define LORA_OP_EXPERT_APPLY 5

/*
 * lora_shrink -- LoraBackend.shrink (mstar.engine.resources.lora.backend):
 *   h[t] = x[t] @ a[slot(t)]^T over num_slices*R columns.
 * x [T, in_features] bf16; a [slots, num_slices*R, in_features] bf16;
 * h [T, num_slices*R] fp32 (written).  Only h[t, i*R + r] with r < rank of a
 * live token's slot is written; every other entry is left as it was (the page
 * allows anything there: the expand never reads it).
 */
LORA_API lora_status lora_shrink(const void* x, float* h, const void* a, const int32_t* ranks,
                        const int32_t* token_order, const int32_t* slot_indptr,
                        int32_t T, int32_t in_features, int32_t slots, int32_t R,
                        int32_t num_slices, int32_t regime, uint32_t* err_flags,
                        void* stream);

/*
 * lora_expand -- LoraBackend.expand_fused:
 *   y[t, slice i] += scalings[slot(t)] * h[t, slice i cols < rank] @ b[slot(t), slice i]^T
 * h [T, num_slices*R] fp32; b [slots, out, R] bf16 with out = sum(out_slices);
 * y [T, out] bf16, in place: y = bf16_rne(float(y) + scaling * acc), acc in fp32.
 * out_slices (host, num_slices entries): widths of the fused projection's
 * outputs in column order (e.g. q, k, v).
 */
LORA_API lora_status lora_expand(void* y, const float* h, const void* b, const int32_t* ranks,
                        const float* scalings, const int32_t* token_order,
                        const int32_t* slot_indptr, int32_t T, int32_t slots, int32_t R,
                        const int32_t* out_slices, int32_t num_slices, int32_t regime,
                        uint32_t* err_flags, void* stream);

/*
 * lora_apply_linear -- LoraBackend.apply_linear_ (shrink then expand, fused):
 * same arguments as lora_shrink + lora_expand.
 *   BGMV: one launch, one thread-block cluster per work item (up to 32 tokens
 *     of one slot), h kept in distributed shared memory; no workspace.
 *   SGMV: a tensor-core shrink writes fp32 partial h (one buffer per split of
 *     the input features) into the workspace and the expand sums them.
 *   STREAM: two launches over every SM: a shrink over 16-row groups of each
 *     slot's tokens writes fp32 partial h per 512 input features into the
 *     workspace, then the streamed expand sums them (rows in 16-row groups,
 *     y by 16-byte loads and stores).  Takes num_slices*R in {16, 32, 48,
 *     64}, roundup(R, 16) <= 64 and in_features <= 4096 (else
 *     LORA_ERR_UNSUPPORTED).  AUTO takes it for those shapes with
 *     512 <= T <= 8192, T * in_features <= 2^25 and T * out <= 2^26 when the
 *     workspace given holds what STREAM needs, else it keeps its BGMV or
 *     SGMV choice (lora_resolve_regime, which knows neither in_features nor
 *     the workspace, answers with that choice).
 *   BGMV_SPLIT (only when asked for): one launch over every SM; the shrink is
 *     cut along the input features and the expand along the output columns
 *     into equal shares, and fp32 partial h pass through the workspace (each
 *     work item's expand waits, bounded, for its partials; lora_set_wait_limit_ns).
 *     Shapes beyond its limits (T > 1024, slots > 1024, more than 512 work
 *     items possible, in_features > 65536, out > 262144) return
 *     LORA_ERR_UNSUPPORTED.
 * workspace must hold lora_workspace_bytes(LORA_OP_APPLY_LINEAR, T, slots, R,
 * num_slices, regime) bytes and be 16-byte aligned (may be NULL when that is
 * 0); for AUTO that covers whichever regime the call resolves to, STREAM
 * included.  Its first 4096 bytes are the BGMV_SPLIT counters: a workspace that
 * BGMV_SPLIT calls use must be ZEROED before its first use (e.g. one
 * cudaMemsetAsync); every call leaves them zeroed again (zero them again after a
 * call that raised LORA_FLAG_TIMEOUT).  The rest needs no initialisation.
 * Calls sharing one workspace must be ordered (one stream, with the launch
 * overlap on too).
 */
LORA_API lora_status lora_apply_linear(const void* x, void* y, const void* a, const void* b,
                              const int32_t* ranks, const float* scalings,
                              const int32_t* token_order, const int32_t* slot_indptr,
                              int32_t T, int32_t in_features, int32_t slots, int32_t R,
                              const int32_t* out_slices, int32_t num_slices, int32_t regime,
                              void* workspace, size_t workspace_bytes, uint32_t* err_flags,
                              void* stream);

/*
 * lora_apply_router -- the router LoRA fold (spark_model/lora/expert_apply.rs,
 * apply_router_lora and its module text; router shape from
 * spark_model/lora/target.rs, router_dims and the Router target): a MoE
 * layer's routing logits take the delta of the router (mlp.gate) adapter of
 * each token's slot, BEFORE top-k expert selection, so the selection sees
 *   gate_logits[t, e] += scalings[slot] * sum_{r<rank} (router_in[t] @ a[slot, r]^T) * b[slot, e, r].
 * router_in [T, hidden] bf16 (the router's input); gate_logits [T, num_experts]
 * bf16, updated in place; a [slots, R, hidden] bf16; b [slots, num_experts, R]
 * bf16; addressing, ranks and scalings as for lora_apply_linear.  It is
 * lora_apply_linear with in_features = hidden and one output slice of
 * num_experts columns, run by the same kernels (regime, workspace and flags
 * behave the same: size the workspace with lora_workspace_bytes(
 * LORA_OP_APPLY_LINEAR, T, slots, R, 1, regime)).  hidden and num_experts must
 * be positive multiples of 8 (LORA_ERR_INVALID otherwise).
 */
LORA_API lora_status lora_apply_router(const void* router_in, void* gate_logits, const void* a,
                                       const void* b, const int32_t* ranks,
                                       const float* scalings, const int32_t* token_order,
                                       const int32_t* slot_indptr, int32_t T, int32_t hidden,
                                       int32_t slots, int32_t R, int32_t num_experts,
                                       int32_t regime, void* workspace, size_t workspace_bytes,
                                       uint32_t* err_flags, void* stream);

/*
 * lora_gather_shrink -- LoraBackend.gather_shrink:
 *   h[t, i*R + r] = a[slot(t), i*R + r, ids[t]]  (r < rank)
 * ids [T] int32 token ids; a [slots, num_slices*R, vocab] bf16; h [T, num_slices*R]
 * fp32.  An id outside [0, vocab) (e.g. -1 for an image position) contributes
 * nothing: its h row is written as zeros.
 */
LORA_API lora_status lora_gather_shrink(const int32_t* ids, float* h, const void* a,
                               const int32_t* ranks, const int32_t* token_order,
                               const int32_t* slot_indptr, int32_t T, int32_t vocab,
                               int32_t slots, int32_t R, int32_t num_slices,
                               uint32_t* err_flags, void* stream);

/*
 * lora_apply_embedding -- LoraBackend.apply_ with embedding=True (gather, then
 * expand; fused, h kept on chip).  A token whose id is outside [0, vocab)
 * contributes nothing and its row of y stays bit-identical.
 * Regimes: AUTO and STREAM run one launch over every SM that streams the y rows
 * of every live token in 16-row groups, 16-byte loads and stores in flight in
 * registers (roundup(R, 16) <= 64, else AUTO takes one of the others); the
 * rows of ids outside the vocabulary are not read.  BGMV and SGMV run those
 * regimes' kernels.
 */
LORA_API lora_status lora_apply_embedding(const int32_t* ids, void* y, const void* a, const void* b,
                                 const int32_t* ranks, const float* scalings,
                                 const int32_t* token_order, const int32_t* slot_indptr,
                                 int32_t T, int32_t vocab, int32_t slots, int32_t R,
                                 const int32_t* out_slices, int32_t num_slices,
                                 int32_t regime, uint32_t* err_flags, void* stream);

/*
 * lora_expert_apply -- the MoE expert fold (spark_model/lora/expert_apply.rs,
 * apply_expert_lora_sorted, with the per-request slot routing the page plans
 * for its grouped (slot, expert) kernel):
 *   for every adapted expert e (ascending) with rows [expert_offsets[e],
 *   expert_offsets[e+1]), for every row rho there whose slot s = row_slot[rho]
 *   is >= 0 and whose pair p = pair_index[s*num_experts + e] is >= 0:
 *     y_sorted[rho, slice i] += scalings[s] * (x_sorted[rho] @ a[p, slice i rows < rank]^T) @ b[p, slice i]^T
 * The fold runs after the base grouped GEMM and before unpermute: for gate/up
 * call it on the gate/up output (before silu_mul), for down on the down output.
 * x_sorted [rows_cap, in_features] bf16; y_sorted [rows_cap, out] bf16 in place;
 * a [num_pairs, num_slices*R, in_features]; b [num_pairs, out, R];
 * pair_index [slots*num_experts] (-1 = not adapted); ranks, scalings [slots];
 * row_slot [rows_cap] (-1 = no adapter); expert_offsets [num_experts+1].
 * Planning happens on the device (no copy of expert_offsets to the host).
 * Row blocks of different experts that overlap give an unspecified result for
 * the shared rows.
 * Without a workspace the fold runs one CTA per chunk of an expert's rows.
 * With a workspace of lora_workspace_bytes(LORA_OP_EXPERT_APPLY, rows_cap,
 * num_experts, R, num_slices, LORA_REGIME_AUTO) bytes (16-byte aligned, no
 * initialisation needed; 0 when the shapes are outside the SGMV rule R in
 * {16, 32, 64}, num_slices * R <= 128) and slots * num_experts <= 4096 and
 * in_features >= 64, it is grouped by (slot, expert): a device pass sorts
 * each adapted expert's rows by slot, then a shrink over 16-row groups
 * (num_slices * R <= 64 and in_features <= 4096; else the tensor-core shrink)
 * writes fp32 partial h into the workspace and the streamed expand folds it
 * into every (slot, expert) group's rows (three launches).  Otherwise the
 * workspace is left unused.
 */
LORA_API lora_status lora_expert_apply(const void* x_sorted, void* y_sorted, const void* a,
                              const void* b, const int32_t* pair_index, const int32_t* ranks,
                              const float* scalings, const int32_t* row_slot,
                              const int32_t* expert_offsets, int32_t rows_cap,
                              int32_t in_features, int32_t num_experts, int32_t slots,
                              int32_t num_pairs, int32_t R, const int32_t* out_slices,
                              int32_t num_slices, void* workspace, size_t workspace_bytes,
                              uint32_t* err_flags, void* stream);

/*
 * lora_apply_linear_noalloc -- lora_apply_linear for callers that cannot give
 * the library any device memory.  The pages have no counterpart: it exists for
 * this library's users.  Some callers cannot allocate where they apply the
 * delta (a plugin inside a runtime that owns all device memory and offers no
 * allocator, code running where cudaMalloc must not be called); this entry
 * point takes the lora_apply_linear arguments without the workspace and uses
 * a scratch array of LORA_STATIC_SCRATCH_BYTES compiled into the library
 * (every GPU that loads the library holds it until the process exits).
 * Shapes whose workspace (lora_workspace_bytes) exceeds that size return
 * LORA_ERR_UNSUPPORTED.  The first call on each device looks up the array's
 * device address with cudaGetSymbolAddress, so make that first call outside
 * stream capture.  It never allocates.  All calls share the array and it keeps
 * the last call's contents (nothing needs clearing); calls that can overlap on
 * the GPU race on it.
 */
#define LORA_STATIC_SCRATCH_BYTES (16u << 20)
LORA_API lora_status lora_apply_linear_noalloc(const void* x, void* y, const void* a, const void* b,
                                               const int32_t* ranks, const float* scalings,
                                               const int32_t* token_order,
                                               const int32_t* slot_indptr, int32_t T,
                                               int32_t in_features, int32_t slots, int32_t R,
                                               const int32_t* out_slices, int32_t num_slices,
                                               int32_t regime, uint32_t* err_flags, void* stream);

/*
 * Workspace bytes an operation needs for these shapes and regime (0 if none).
 * For LORA_OP_EXPERT_APPLY pass rows_cap as T and num_experts as slots.
 */
LORA_API size_t lora_workspace_bytes(int32_t op, int32_t T, int32_t slots, int32_t R,
                            int32_t num_slices, int32_t regime);

/* The regime LORA_REGIME_AUTO resolves to for these scalar shapes. */
LORA_API int32_t lora_resolve_regime(int32_t op, int32_t T, int32_t slots, int32_t R,
                            int32_t num_slices);

/* Positions (or sorted rows) per work item of an operation's kernel in a regime. */
LORA_API int32_t lora_plan_tile(int32_t op, int32_t regime);

/*
 * lora_plan_linear -- runs the device work-item planner the kernels use and
 * writes its plan: plan_out[3*i .. 3*i+2] = (slot, first position, count) for
 * i < min(*plan_count, plan_cap); *plan_count (device int32) = number of items.
 * scalings may be NULL (the unscaled operations: shrink, gather).  Slots are in
 * ascending order, each cut into consecutive tiles of `tile` positions.
 */
LORA_API lora_status lora_plan_linear(const int32_t* slot_indptr, const int32_t* ranks,
                             const float* scalings, int32_t T, int32_t slots, int32_t R,
                             int32_t tile, int32_t* plan_out, int32_t plan_cap,
                             int32_t* plan_count, uint32_t* err_flags, void* stream);

/*
 * lora_plan_expert -- the device expert planner (expert_delta_workitems then
 * fold_chunked): plan_out[3*i..] = (expert, row_off, rows) per chunk of at most
 * `max_rows` rows, experts ascending over the adapted set (experts holding a
 * pair for any slot); *plan_count = number of chunks.
 */
LORA_API lora_status lora_plan_expert(const int32_t* expert_offsets, const int32_t* pair_index,
                             int32_t rows_cap, int32_t num_experts, int32_t slots,
                             int32_t max_rows, int32_t* plan_out, int32_t plan_cap,
                             int32_t* plan_count, uint32_t* err_flags, void* stream);

/*
 * lora_set_launch_overlap -- opt in (enable != 0) or out of overlapping the
 * start of a kernel with the end of the kernel that precedes it in the stream
 * (CUDA programmatic dependent launch; captured into CUDA graphs as a
 * programmatic edge), for lora_apply_linear (both regimes) and
 * lora_apply_embedding / lora_shrink / lora_expand in the SGMV regime.  With it
 * on, a kernel plans its work items and starts loading adapter rows before the
 * preceding kernel has finished; it reads x, y, h and ids, and writes any
 * output or workspace, only after that kernel has finished and its writes are
 * visible.  Contract while enabled: the kernel preceding such a call in its
 * stream does not write a, b, ranks, scalings, token_order or slot_indptr of
 * that call.  Process-wide; off by default; takes effect for launches issued
 * after the call.  Returns the previous setting.
 */
LORA_API int32_t lora_set_launch_overlap(int32_t enable);

/*
 * lora_set_wait_limit_ns -- the limit of every bounded device wait of the
 * BGMV_SPLIT kernel (an expand waiting for its item's partial h), in
 * nanoseconds; 0 restores the default of one second.  A wait that runs out
 * raises LORA_FLAG_TIMEOUT, skips that work item's update of y and lets the
 * call finish.  Process-wide; takes effect for launches issued after the
 * call.  Returns the previous setting (0 = the default).
 */
LORA_API uint64_t lora_set_wait_limit_ns(uint64_t ns);

LORA_API const char* lora_status_string(lora_status status);
LORA_API const char* lora_last_error(void);
/* Library version, e.g. "lora_delta 0.1.0 sm_100a". */
LORA_API const char* lora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LORA_DELTA_H */
