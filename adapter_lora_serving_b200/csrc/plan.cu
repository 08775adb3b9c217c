// Plan dumps: run the same device planners the kernels run (one CTA) and write
// the work items out, so the plan can be compared word for word with the CPU
// planner.  Sources: mstar.engine.resources.lora.backend (addressing by
// token_order / slot_indptr) and spark_model/lora/expert_apply.rs
// (expert_delta_workitems, fold_chunked).
#include "common.cuh"
#include "kernels.h"

namespace lora {

constexpr int kPlanThreads = 256;

__global__ void __launch_bounds__(kPlanThreads)
plan_linear_kernel(const int* slot_indptr, const int* ranks, const float* scalings, int T,
                   int slots, int R, int tile, int* plan_out, int plan_cap, int* plan_count,
                   uint32_t* flags) {
  extern __shared__ __align__(16) int plan_smem[];
  int* scratch = plan_smem;
  int* prefix = plan_smem + kPlanThreads / 32;
  const int total = plan_linear<kPlanThreads>(slot_indptr, ranks, scalings, slots, T, R, tile,
                                              prefix, scratch, flags, true);
  if (threadIdx.x == 0) *plan_count = total;
  for (int item = threadIdx.x; item < min(total, plan_cap); item += kPlanThreads) {
    const int s = find_segment(prefix, slots, item);
    const int j = item - prefix[s];
    const int p0 = slot_indptr[s] + j * tile;
    plan_out[3 * item + 0] = s;
    plan_out[3 * item + 1] = p0;
    plan_out[3 * item + 2] = min(tile, slot_indptr[s + 1] - p0);
  }
}

__global__ void __launch_bounds__(kPlanThreads)
plan_expert_kernel(const int* offsets, const int* pair_index, int rows_cap, int E, int slots,
                   int max_rows, int* plan_out, int plan_cap, int* plan_count, uint32_t* flags) {
  extern __shared__ __align__(16) int plan_smem[];
  int* scratch = plan_smem;
  int* prefix = plan_smem + kPlanThreads / 32;
  const int total = plan_expert<kPlanThreads>(offsets, pair_index, E, slots, rows_cap, max_rows,
                                              prefix, scratch, flags, true);
  if (threadIdx.x == 0) *plan_count = total;
  for (int item = threadIdx.x; item < min(total, plan_cap); item += kPlanThreads) {
    const int e = find_segment(prefix, E, item);
    const int c = item - prefix[e];
    const int start = offsets[e] + c * max_rows;
    plan_out[3 * item + 0] = e;
    plan_out[3 * item + 1] = start;
    plan_out[3 * item + 2] = min(max_rows, offsets[e + 1] - start);
  }
}

cudaError_t plan_linear_launch(const int* slot_indptr, const int* ranks, const float* scalings,
                               int T, int slots, int R, int tile, int* plan_out, int plan_cap,
                               int* plan_count, uint32_t* flags, cudaStream_t stream) {
  const size_t smem = (size_t)(kPlanThreads / 32 + slots + 1) * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(plan_linear_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  plan_linear_kernel<<<1, kPlanThreads, smem, stream>>>(slot_indptr, ranks, scalings, T, slots, R,
                                                        tile, plan_out, plan_cap, plan_count,
                                                        flags);
  return cudaGetLastError();
}

cudaError_t plan_expert_launch(const int* offsets, const int* pair_index, int rows_cap, int E,
                               int slots, int max_rows, int* plan_out, int plan_cap,
                               int* plan_count, uint32_t* flags, cudaStream_t stream) {
  const size_t smem = (size_t)(kPlanThreads / 32 + E + 1) * sizeof(int);
  cudaError_t err = cudaFuncSetAttribute(plan_expert_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  plan_expert_kernel<<<1, kPlanThreads, smem, stream>>>(offsets, pair_index, rows_cap, E, slots,
                                                        max_rows, plan_out, plan_cap, plan_count,
                                                        flags);
  return cudaGetLastError();
}

}  // namespace lora
