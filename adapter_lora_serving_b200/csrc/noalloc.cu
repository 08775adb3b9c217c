// lora_apply_linear_noalloc: the fused shrink + expand for callers that have
// no way to hand the library a device allocation.
//
// Some callers cannot obtain device memory at the point where they apply the
// delta: a plugin inside a serving runtime that owns every byte of device
// memory and exposes no allocator, code that runs from a host callback or
// under a driver-level restriction where cudaMalloc must not be called, or an
// embedding whose only interface is "pointers to inputs and outputs".  For
// them this entry point takes the same arguments as lora_apply_linear minus the
// workspace, and uses a fixed scratch array that lives in the library image on
// every device that loads it.
//
// The scratch is a file-scope __device__ array of LORA_STATIC_SCRATCH_BYTES.
// Host code cannot pass its name to a kernel (on the host it is only a
// stand-in), so the first call on each device looks up its device address
// with cudaGetSymbolAddress while that device is current and caches it; make
// that first call outside any stream capture.  Nothing here allocates or frees
// device memory.  Every call shares the one array, and it keeps what the last
// call wrote: calls that may overlap on the GPU (different streams without an
// ordering between them) race on it.  The kernels write every scratch value
// they later read, so nothing needs clearing between calls.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/lora_delta.h"

namespace lora {
void set_last_error(const char* msg);  // api.cu
size_t apply_linear_workspace(int regime, int T, int in_features, int slots, int R, int S,
                              int out, size_t ws_bytes);  // api.cu
}

namespace {

static __device__ __align__(256) unsigned char g_lora_static_scratch[LORA_STATIC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

}  // namespace

extern "C" {

lora_status lora_apply_linear_noalloc(const void* x, void* y, const void* a, const void* b,
                                      const int32_t* ranks, const float* scalings,
                                      const int32_t* token_order, const int32_t* slot_indptr,
                                      int32_t T, int32_t in_features, int32_t slots, int32_t R,
                                      const int32_t* out_slices, int32_t num_slices,
                                      int32_t regime, uint32_t* err_flags, void* stream) {
  char msg[256];
  long long out = 0;
  if (out_slices != nullptr && num_slices >= 1 && num_slices <= LORA_MAX_SLICES)
    for (int i = 0; i < num_slices; ++i) out += out_slices[i];
  // the scratch these shapes take in the regime lora_apply_linear resolves
  // them to (argument errors are left to lora_apply_linear to report)
  const size_t need =
      (out > 0 && out < (1LL << 30))
          ? lora::apply_linear_workspace(regime, T, in_features, slots, R, num_slices, (int)out,
                                         LORA_STATIC_SCRATCH_BYTES)
          : 0;
  if (need > (size_t)LORA_STATIC_SCRATCH_BYTES) {
    snprintf(msg, sizeof(msg),
             "lora_apply_linear_noalloc: these shapes need %zu bytes of scratch; the static "
             "scratch holds %u bytes (use lora_apply_linear with a workspace)",
             need, (unsigned)LORA_STATIC_SCRATCH_BYTES);
    lora::set_last_error(msg);
    return LORA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  if (need > 0) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err == cudaSuccess && (dev < 0 || dev >= 64)) err = cudaErrorInvalidDevice;
    if (err != cudaSuccess) {
      snprintf(msg, sizeof(msg), "lora_apply_linear_noalloc: %s", cudaGetErrorString(err));
      lora::set_last_error(msg);
      return LORA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      err = cudaGetSymbolAddress(&p, g_lora_static_scratch);
      if (err != cudaSuccess || p == nullptr) {
        snprintf(msg, sizeof(msg), "lora_apply_linear_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(err));
        lora::set_last_error(msg);
        return LORA_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    ws = g_scratch_ptr[dev];
  }
  return lora_apply_linear(x, y, a, b, ranks, scalings, token_order, slot_indptr, T, in_features,
                           slots, R, out_slices, num_slices, regime, ws,
                           ws ? (size_t)LORA_STATIC_SCRATCH_BYTES : 0, err_flags, stream);
}

}  // extern "C"
