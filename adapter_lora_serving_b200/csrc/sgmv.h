// SGMV regime (many tokens per slot): tcgen05 / TMEM tensor-core tiles over
// slot-sorted segments.  Interface used by the C-ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lora {

constexpr int kSgmvTileM = 128;  // positions (tokens) per work item

// Shapes the SGMV kernels take: R in {16, 32, 64}, num_slices * R <= 128.
bool sgmv_supported(int S, int R);
// The same rule as text, for error messages.
constexpr const char* kSgmvShapeRule =
    "the SGMV regime needs R in {16, 32, 64} and num_slices * R <= 128";
// Workspace of lora_apply_linear in this regime (partial h buffers).
size_t sgmv_workspace_bytes(int T, int R, int S);
// Splits of the input features the shrink uses for these shapes.
int sgmv_shrink_splits(int T, int slots, int in);

// Grouped addressing (the MoE fold's (slot, expert) groups): group s owns
// positions [slot_indptr[s], seg_hi[s]) of token_order and uses the adapter
// pair slot_map[s] of a and b, which hold ab_slots pairs.  Its kernels follow
// a kernel that writes that addressing, so they launch without the
// programmatic edge.
struct SgmvGroups {
  const int* seg_hi;
  const int* slot_map;
  int ab_slots;
};

// h[ks][t, i*R + r] = x[t, k-range ks] . a[slot, i*R + r, k-range ks] for the
// live columns of live tokens; ksplit = min(ksplit_max, sgmv_shrink_splits()).
// scalings == nullptr plans every slot of nonzero rank; otherwise slots of
// scaling 0 are skipped too.
cudaError_t sgmv_shrink_launch(const void* x, const void* a, float* h, const int* ranks,
                               const int* token_order, const int* slot_indptr, int T, int in,
                               int slots, int R, int S, uint32_t* flags, cudaStream_t stream,
                               const char** why, int ksplit_max, const float* scalings,
                               const SgmvGroups* groups = nullptr);

// y += scal * h B^T, h = sum of `ksplit` partial buffers of `h` (fp32
// [ksplit][T][S*R]) or, when h is null, gathered from `a` at `ids`
// (embedding target, `vocab` columns).
cudaError_t sgmv_expand_launch(void* y, const float* h, int ksplit, const int* ids, const void* a,
                               const void* b, const int* ranks, const float* scalings,
                               const int* token_order, const int* slot_indptr, int T, int vocab,
                               int slots, int R, int S, const int* slice_off, int out,
                               uint32_t* flags, cudaStream_t stream, const char** why,
                               const SgmvGroups* groups = nullptr);

}  // namespace lora
