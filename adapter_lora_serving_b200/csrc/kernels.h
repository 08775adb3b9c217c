// Internal interface between the C-ABI entry points (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/lora_delta.h"

namespace lora {

// ---------------------------------------------------------------------------
// BGMV regime: one thread-block cluster of kGroup CTAs per work item of at
// most kTT tokens of one slot.  Each CTA reduces over 1/kGroup of the input
// features (shrink), the cluster sums the partial h through distributed shared
// memory, and each CTA then expands 1/kGroup of the output columns.
// ---------------------------------------------------------------------------

constexpr int kBgmvThreads = 256;
constexpr int kTT = 32;          // tokens (sorted rows) per work item, at most
constexpr int kFusedTile = 32;   // positions per work item of the fused linear path
constexpr int kGroup = 8;        // CTAs per work item (cluster size)
constexpr int kMaxKB = 512;      // input features per pipeline stage (upper bound)
constexpr int kRingBudget = 120 * 1024;  // shared-memory bytes for the staging ring
constexpr int kMaxCombosPerWarp = 4;  // (16-row tile, 8-token tile) pairs per warp:
                                      // (kMaxSRp/16) * (kTT/8) / 8 warps
constexpr int kMaxSRp = 128;     // num_slices * roundup(R, 16) limit of this regime
static_assert((kMaxSRp / 16) * (kTT / 8) <= kMaxCombosPerWarp * (kBgmvThreads / 32),
              "every (row tile, token tile) pair of the shrink has a warp slot");
constexpr int kExStageMax = 96 * 1024;  // largest staged expand the ring is grown for

enum BgmvMode : int {
  kModeFused = 0,   // shrink + expand (apply_linear)
  kModeShrink = 1,  // shrink only, h written to global
  kModeExpand = 2,  // expand only, h read from global
  kModeEmbed = 3,   // gather + expand (apply_embedding)
  kModeGather = 4,  // gather only (gather_shrink)
  kModeExpertSolo = 6,  // MoE fold: one CTA per expert chunk, shrink over all of in
};

// Ring budget of the one-CTA-per-chunk MoE fold (two CTAs per SM).
constexpr int kSoloRingBudget = 80 * 1024;

struct BgmvParams {
  const void* x;               // bf16 [rows, in]
  void* y;                     // bf16 [rows, out]
  const void* a;               // bf16 [W, S*R, in]
  const void* b;               // bf16 [W, out, R]
  float* h;                    // fp32 [T, S*R]
  const int* ids;              // [T]
  const int* ranks;            // [slots]
  const float* scalings;       // [slots] (nullptr for unscaled operations)
  const int* token_order;      // [T]
  const int* slot_indptr;      // [slots+1]
  const int* pair_index;       // [slots*E]
  const int* row_slot;         // [rows_cap]
  const int* expert_offsets;   // [E+1]
  uint32_t* flags;
  int T;          // tokens, or rows_cap for the expert fold
  int in;         // input features (vocab for the embedding modes)
  int slots;
  int R;
  int S;
  int out;
  int num_experts;
  int num_pairs;
  int kchunk;     // input features one CTA reduces over (multiple of 8)
  int kb;         // input features per stage (multiple of 8)
  int nst;        // stages in the ring (1 or 2)
  int ex_stage;   // 1: the expand operands of an item fit the ring and are staged there
  int bulk_stage; // 1: shrink stages are staged by bulk copies, 0: by cp.async
  int ex_cw;      // MoE fold: output columns per staged expand chunk (0: unstaged)
  int tile;       // positions per work item of the linear modes (<= kTT)
  int slice_off[LORA_MAX_SLICES + 1];
};

struct BgmvLayout {
  int prefix_off;
  int misc_off;
  int ring_off;
  int hpart_off;
  int hhi_off;      // bf16 [S][kTT][hst]: h rounded to bf16
  int hlo_off;      // bf16 [S][kTT][hst]: h - hi rounded to bf16
  int hst;          // row stride of the bf16 h tiles (elements): roundup(R,16) + 8
  int total;
  int srp;          // S * roundup(R, 16): h row stride in shared memory (floats)
  int row_stride;   // bytes per staged row: kb bf16 + 16 bytes of padding
  int stage_bytes;  // bytes per pipeline stage
};

__host__ __device__ inline int ceil_div_i(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int round_up_i(int a, int b) { return ceil_div_i(a, b) * b; }

// Output columns each CTA of a cluster expands (multiple of 16).
__host__ __device__ inline int bgmv_ochunk(int out) { return round_up_i(ceil_div_i(out, kGroup), 16); }

// Bytes of the ring that the staged expand operands of one item take: this
// CTA's B columns ([cols][R] bf16) and kTT rows of y over them, each row
// padded by 16 bytes.
__host__ __device__ inline int bgmv_ex_stage_bytes(int out, int R) {
  const int oc = bgmv_ochunk(out);
  return round_up_i(oc * R * 2, 128) + kTT * (oc * 2 + 16);
}

// Items per CTA whose addressing the planner caches in shared memory (linear
// modes, in the sub-batch arrays the expert mode uses otherwise).
constexpr int kItemCache = 8;

// Misc shared region (ints): tok[kTT], id[kTT], ctrl[8], scratch[8],
// sub_s[kTT], sub_p[kTT], sub_cnt[kTT], sub_rows[kTT*kTT].
constexpr int kMiscInts = kTT + kTT + 8 + 8 + 3 * kTT + kTT * kTT;

// Input features each CTA of a cluster reduces over (multiple of 8).
__host__ __device__ inline int bgmv_kchunk(int in) { return round_up_i(ceil_div_i(in, kGroup), 8); }

// ring_min: bytes the ring must hold besides its stages (the staged expand
// operands), 0 when the expand is not staged.
__host__ __device__ inline BgmvLayout bgmv_layout(int mode, int npref, int S, int R, int kb,
                                                  int nst, int ring_min) {
  BgmvLayout L;
  L.srp = S * round_up_i(R, 16);
  L.row_stride = kb * 2 + 16;
  L.stage_bytes = round_up_i((L.srp + kTT) * L.row_stride, 128);
  int off = 128;  // mbarriers
  L.prefix_off = off;
  off += round_up_i((npref + 1) * 4, 128);
  L.misc_off = off;
  off += round_up_i(kMiscInts * 4, 128);
  L.ring_off = off;
  const bool ring = (mode == kModeFused || mode == kModeShrink || mode == kModeExpertSolo);
  if (ring) off += round_up_i(max(nst * L.stage_bytes, ring_min), 128);
  L.hpart_off = off;
  if (ring) off += 2 * kTT * L.srp * 4;
  L.hst = round_up_i(R, 16) + 8;
  L.hhi_off = off;
  off += round_up_i(S * kTT * L.hst * 2, 128);
  L.hlo_off = off;
  off += round_up_i(S * kTT * L.hst * 2, 128);
  L.total = off;
  return L;
}

// Stage width and depth of the staging ring for a CTA reducing over kchunk
// input features (host side).
inline void bgmv_pick_stages(int kchunk, int S, int R, int budget, int* kb, int* nst) {
  const int rows = S * round_up_i(R, 16) + kTT;
  int k = kchunk < kMaxKB ? kchunk : kMaxKB;
  for (;;) {
    const int n = ceil_div_i(kchunk, k) > 1 ? 2 : 1;
    if (k <= 64 || n * rows * (2 * k + 16) <= budget) {
      *kb = k;
      *nst = n;
      return;
    }
    k -= 64;
  }
}

// Process-wide opt-in to programmatic dependent launch of the fused BGMV
// kernel and the SGMV kernels (lora_set_launch_overlap).
int bgmv_set_overlap(int enable);
bool launch_overlap_enabled();
// Process-wide limit of every bounded device wait of the split kernel
// (lora_set_wait_limit_ns); 0 restores the default of one second.
uint64_t set_wait_limit_ns(uint64_t ns);
uint64_t wait_limit_ns();

// ---------------------------------------------------------------------------
// BGMV regime, split kernel (fused apply_linear with a workspace): one CTA per
// SM.  The shrink of every work item (<= kTT tokens of one slot) is cut along
// the input features and the expand along the output columns, both into
// contiguous byte ranges of equal size, one range per CTA.  Shrink pieces
// publish fp32 partial h through the workspace and count themselves on a
// per-item counter; the expand of an item waits (bounded) for its count and
// sums the partials in piece order.
// ---------------------------------------------------------------------------

constexpr int kSpKQ = 64;         // input features per block of the shrink split
constexpr int kSpCQ = 64;         // output columns per block of the expand split
constexpr int kSpMaxGrid = 256;   // CTAs of one launch at most (workspace bound)
constexpr int kSpMaxT = 1024;     // tokens (token_order is held in shared memory)
constexpr int kSpMaxSlots = 1024;
constexpr int kSpMaxItems = 512;  // work items a call may plan
constexpr int kSpMaxIn = 65536;   // keeps every byte count of the split in 32 bits
constexpr int kSpMaxOut = 262144;
constexpr int kSpRingMin = 64 * 1024;   // staging ring of larger shapes (two per SM no longer fit)
// Leading bytes of an apply_linear workspace that hold the split kernel's
// counters; the SGMV kernels use the bytes after them.
constexpr size_t kWsCounterBytes = 4096;

struct SplitParams {
  const void* x;               // bf16 [T, in]
  void* y;                     // bf16 [T, out]
  const void* a;               // bf16 [slots, S*R, in]
  const void* b;               // bf16 [slots, out, R]
  const int* ranks;
  const float* scalings;
  const int* token_order;
  const int* slot_indptr;
  uint32_t* cnt;               // [item_cap] shrink pieces published per item
  uint32_t* cons;              // [item_cap] expand pieces that consumed an item
  float* part;                 // [(item_cap + kSpMaxGrid) * kTT * S * R] partial h
  uint32_t* flags;
  unsigned long long wait_ns;  // bounded-wait limit
  int T, in, slots, R, S, out;
  int item_cap;                // items planned at most (workspace capacity)
  int ring;                    // bytes of the staging ring (split_ring_bytes)
  int slice_off[LORA_MAX_SLICES + 1];
};

struct SplitLayout {
  int tok_off;    // int [T]: token_order, each slot's tokens in canonical order
  int meta_off;   // int4 [item_cap]: slot, first position, slot tokens, rank|tile|count
  int wcum_off;   // u32 [item_cap + 1]: exclusive prefix of shrink units
  int vcum_off;   // u32 [item_cap + 1]: exclusive prefix of expand units
  int cand_off;   // int [kSpMaxGrid]: the shrink pieces of the current expand item
  int wst_off;    // u32 [kSpMaxGrid + 1]: first shrink unit of every CTA
  int vst_off;    // u32 [kSpMaxGrid + 1]: first expand unit of every CTA
  int ctrl_off;   // int [64]: scan scratch and broadcast words
  int xtab_off;   // int [256]: the current expand round's job and piece tables
  int ring_off;   // staging ring: shrink rounds, then expand jobs (and their pieces' h)
  int total;
};

__host__ __device__ inline int split_fixed_bytes(int T, int item_cap) {
  return round_up_i(T * 4, 128) + round_up_i(item_cap * 16, 128) +
         2 * round_up_i((item_cap + 1) * 4, 128) + kSpMaxGrid * 4 +
         2 * round_up_i((kSpMaxGrid + 1) * 4, 128) + 64 * 4 + 256 * 4;
}

__host__ __device__ inline SplitLayout split_layout(int T, int item_cap, int ring) {
  SplitLayout L;
  int off = 0;
  L.tok_off = off;
  off += round_up_i(T * 4, 128);
  L.meta_off = off;
  off += round_up_i(item_cap * 16, 128);
  L.wcum_off = off;
  off += round_up_i((item_cap + 1) * 4, 128);
  L.vcum_off = off;
  off += round_up_i((item_cap + 1) * 4, 128);
  L.cand_off = off;
  off += kSpMaxGrid * 4;
  L.wst_off = off;
  off += round_up_i((kSpMaxGrid + 1) * 4, 128);
  L.vst_off = off;
  off += round_up_i((kSpMaxGrid + 1) * 4, 128);
  L.ctrl_off = off;
  off += 64 * 4;
  L.xtab_off = off;
  off += 256 * 4;
  L.ring_off = off;
  off += ring;
  L.total = off;
  return L;
}

// Row stride (floats) of the fp32 h rows an expand piece keeps in the ring.
__host__ __device__ inline int split_hst(int R) { return round_up_i(R, 16); }

// The staging ring: what keeps a CTA within `budget` bytes of shared memory
// (so that two CTAs fit one SM: one of this launch and one of the next, which
// starts early under the launch overlap), at least kSpRingMin.
inline int split_ring_bytes(int T, int item_cap, int budget) {
  const int r = (budget - split_fixed_bytes(T, item_cap)) & ~127;
  return r > kSpRingMin ? r : kSpRingMin;
}

// Items a call with these shapes can plan at most: every used slot has one
// item per kTT of its tokens.
inline int split_item_cap(int T, int slots) {
  const long long c = (long long)(T < slots ? T : slots) + ceil_div_i(T, kTT);
  return (int)(c > (1 << 30) ? (1 << 30) : c);
}
// Whether the split kernel takes these shapes (else the cluster kernel runs).
inline bool split_eligible(int T, int in, int slots, int R, int S, int out) {
  return T <= kSpMaxT && slots <= kSpMaxSlots && in <= kSpMaxIn && out <= kSpMaxOut &&
         S * round_up_i(R, 16) <= kMaxSRp && split_item_cap(T, slots) <= kSpMaxItems;
}
// Workspace bytes of the split kernel: counters, then the partial h of every
// (item, CTA) piece.
inline size_t split_workspace_bytes(int T, int slots, int R, int S) {
  const size_t cap = (size_t)split_item_cap(T, slots);
  return kWsCounterBytes + (cap + kSpMaxGrid) * kTT * (size_t)S * R * sizeof(float);
}

cudaError_t split_launch(const SplitParams& p, cudaStream_t stream, const char** why);

// ---------------------------------------------------------------------------
// Streamed expand (stream.cu): the embedding target (h gathered from A by token
// id) and the expand of a computed h (fp32 partial buffers, e.g. the grouped
// MoE fold).  The positions of every slot that takes part are cut into row
// groups of kStRows and the output columns into blocks of at most W columns
// (one slice each); the (row group, block) units, row group by row group, are
// split into equal runs, one per CTA (one per SM).  A producer warp
// bulk-copies a B block into a ring of kStBBufs buffers whenever the (slot,
// block) changes; consumer warps hold their B fragments in registers, keep
// the y rows of the next kStDepth units in flight in registers, apply h with
// warp MMAs and store y.
// ---------------------------------------------------------------------------
constexpr int kStRows = 16;       // positions per group (one MMA row tile)
constexpr int kStConsumers = 16;  // consumer warps (one 32-column chunk each)
constexpr int kStThreads = 32 * (1 + kStConsumers);
constexpr int kStDepth = 4;       // units of y in flight per consumer warp
constexpr int kStBBufs = 4;       // B blocks in flight
constexpr int kStMaxRp = 64;      // roundup(R, 16) limit
constexpr int kStMaxGroups = 64;  // groups per table window
constexpr int kStSpec = 2048;     // token_order entries a CTA reads ahead at most

struct StreamParams {
  const int* ids;             // embedding: token ids (h gathered from a)
  const float* h;             // or: h partial buffers [ksplit][T][S*R] (fp32)
  size_t h_split;             // elements between the partial buffers
  int ksplit;
  void* y;
  const void* a;
  const void* b;
  const int* ranks;
  const float* scalings;
  const int* token_order;
  const int* slot_indptr;
  const int* seg_hi;          // grouped addressing: segment ends, or nullptr
  const int* slot_map;        // grouped addressing: b pair of each group, or nullptr
  uint32_t* flags;
  uint64_t wait_ns;
  int T, vocab, slots, R, S, out;
  int slice_off[LORA_MAX_SLICES + 1];
  int block_off[LORA_MAX_SLICES + 1];  // exclusive prefix of column blocks per slice
  int nblocks;                         // column blocks of all slices
  int W;                               // columns per block at most
  int gtab;                            // groups per table window
  int bbytes;                          // bytes of one B buffer (W * R * 2)
  int off_prefix, off_segs, off_scratch, off_spec, off_ctok, off_cval, off_gmeta, off_htab;
  int off_bbuf;
  int smem;
};

// The streamed kernels take roundup(R, 16) <= kStMaxRp.
inline bool stream_supported(int R) { return round_up_i(R, 16) <= kStMaxRp; }
// Fills the layout fields of p (from T, slots, R, S and slice_off) and launches
// (the programmatic edge to the preceding kernel only when allow_overlap).
cudaError_t stream_launch(StreamParams& p, cudaStream_t stream, bool allow_overlap,
                          const char** why);

// Shrink over short segments (group_shrink.cu): row groups of 16, the input
// features in at most kGsMaxParts chunks of group_shrink_chunk(in) = 256 << k
// features, fp32 partial h per chunk; S*R in {16, 32, 48, 64}, 8 <= in <=
// kGsMaxIn.  Segments [seg_lo[s], seg_hi[s]), or CSR by slot [seg_lo[s],
// seg_lo[s+1]) when seg_hi is null; A of pair slot_map[s] (s when null).
// *ksplit_out = the number of chunks.  allow_overlap: the programmatic edge to
// the preceding kernel (x read and h written after it).
constexpr int kGsMaxIn = 4096;
constexpr int kGsMaxParts = 8;
bool group_shrink_supported(int S, int R, int in);
cudaError_t group_shrink_launch(const void* x, const void* a, float* h, const int* token_order,
                                const int* seg_lo, const int* seg_hi, const int* slot_map,
                                const int* ranks, const float* scalings, int T, int in,
                                int slots, int R, int S, int* ksplit_out, cudaStream_t stream,
                                bool allow_overlap);
int group_shrink_chunk(int in);
int group_shrink_chunks(int in);

// The MoE fold grouped by (slot, expert) (moe_group.cu): per adapted expert,
// its rows sorted by slot into token_order, group g = s * num_experts + e owning
// [seg_lo[g], seg_hi[g]) with rank g_rank[g] and scaling g_scal[g].
constexpr int kMoeMaxGroups = 4096;   // slots * num_experts of the grouped fold
cudaError_t moe_group_launch(const int* expert_offsets, const int* pair_index, const int* row_slot,
                             const int* ranks, const float* scalings, int rows_cap,
                             int num_experts, int slots, int num_pairs, int R, int* token_order,
                             int* seg_lo, int* seg_hi, int* g_rank, float* g_scal,
                             uint32_t* flags, cudaStream_t stream);

// Workspace bytes lora_apply_linear needs for these shapes in `regime` (AUTO
// resolved with the real in_features, out and a workspace of ws_bytes), 0 if
// none (api.cu).
size_t apply_linear_workspace(int regime, int T, int in_features, int slots, int R, int S,
                              int out, size_t ws_bytes);

// Launchers (bgmv.cu).  Return a cudaError_t from the launch.
cudaError_t bgmv_launch(int mode, const BgmvParams& p, int max_items, cudaStream_t stream,
                        const char** why);

// Device planners exposed for plan dumps (plan.cu).
cudaError_t plan_linear_launch(const int* slot_indptr, const int* ranks, const float* scalings,
                               int T, int slots, int R, int tile, int* plan_out, int plan_cap,
                               int* plan_count, uint32_t* flags, cudaStream_t stream);
cudaError_t plan_expert_launch(const int* offsets, const int* pair_index, int rows_cap, int E,
                               int slots, int max_rows, int* plan_out, int plan_cap,
                               int* plan_count, uint32_t* flags, cudaStream_t stream);

}  // namespace lora
