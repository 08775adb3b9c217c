// SGMV regime (many tokens per slot): tcgen05 / TMEM tensor-core tiles over
// slot-sorted segments.  Interface used by the C-ABI entry points.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lora {

constexpr int kSgmvTileM = 128;  // positions (tokens) per work item

bool sgmv_supported(int S, int R);
size_t sgmv_workspace_bytes(int T, int R, int S);

// h[t, i*R + r] = x[t] . a[slot, i*R + r] for the live columns of live tokens.
cudaError_t sgmv_shrink_launch(const void* x, const void* a, float* h, const int* ranks,
                               const int* token_order, const int* slot_indptr, int T, int in,
                               int slots, int R, int S, uint32_t* flags, cudaStream_t stream,
                               const char** why);

// y += scal * h B^T.  h comes from `h` (fp32 [T, S*R]) or, when h is null,
// is gathered from `a` at `ids` (embedding target, vocab columns).
cudaError_t sgmv_expand_launch(void* y, const float* h, const int* ids, const void* a,
                               const void* b, const int* ranks, const float* scalings,
                               const int* token_order, const int* slot_indptr, int T, int vocab,
                               int slots, int R, int S, const int* slice_off, int out,
                               uint32_t* flags, cudaStream_t stream, const char** why);

}  // namespace lora
