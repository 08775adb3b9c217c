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
constexpr int kTT = 32;          // tokens (sorted rows) per work item
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
