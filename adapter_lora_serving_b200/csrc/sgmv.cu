// SGMV regime: placeholder until the tcgen05 kernels land; the entry points
// route every call to the BGMV regime while sgmv_supported() is false.
#include "sgmv.h"

namespace lora {

bool sgmv_supported(int, int) { return false; }
size_t sgmv_workspace_bytes(int T, int R, int S) { return (size_t)T * R * S * sizeof(float); }

cudaError_t sgmv_shrink_launch(const void*, const void*, float*, const int*, const int*,
                               const int*, int, int, int, int, int, uint32_t*, cudaStream_t,
                               const char** why) {
  *why = "the SGMV regime is not available in this build";
  return cudaErrorNotSupported;
}

cudaError_t sgmv_expand_launch(void*, const float*, const int*, const void*, const void*,
                               const int*, const float*, const int*, const int*, int, int, int,
                               int, int, const int*, int, uint32_t*, cudaStream_t,
                               const char** why) {
  *why = "the SGMV regime is not available in this build";
  return cudaErrorNotSupported;
}

}  // namespace lora
