// The MoE expert fold grouped by (slot, expert): a planner that sorts each
// adapted expert's sorted rows by slot, so that the rows of one (slot, expert)
// pair -- one adapter pair, one rank, one scaling -- form a contiguous segment
// the tensor-core (SGMV) kernels tile like a slot's tokens.
//
// Sources: spark_model/lora/expert_apply.rs, apply_expert_lora_sorted and the
// module text (the fold is applied per expert over its contiguous row block
// of expert_offsets, before unpermute; the planned grouped kernel routes each
// (slot, expert)); expert_delta_workitems (experts out of range, empty or
// with malformed offsets are skipped); spark_model/lora/target.rs,
// ExpertLoraLayer (an expert is adapted when a pair is stored for it).
//
// One CTA per expert e.  If some slot holds a pair for e and its row block
// [off[e], off[e+1]) is valid, every row rho of the block is classified the
// way the fold's rules read: row_slot[rho] == -1 (no adapter) or no pair for
// (slot, e) leaves it out; a slot outside [-1, slots), a pair outside
// [-1, num_pairs) or a rank outside [0, R] raise their flags and leave it out;
// rank 0 or scaling 0 leave it out.  The remaining rows of slot s are group
// g = s * num_experts + e: they are written, in no particular order, to
// token_order[seg_lo[g], seg_hi[g]) inside the block, the rows left out after
// them; g_rank[g] / g_scal[g] are the slot's rank and scaling (0 for an empty
// group).  Each row's fold does not depend on the order inside its group.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace lora {
namespace {

constexpr int kMgThreads = 256;
constexpr int kMgCache = 4096;   // rows whose class is kept in shared memory between the passes

struct MoeGroupParams {
  const int* expert_offsets;
  const int* pair_index;
  const int* row_slot;
  const int* ranks;
  const float* scalings;
  int* token_order;
  int* seg_lo;
  int* seg_hi;
  int* g_rank;
  float* g_scal;
  uint32_t* flags;
  int rows_cap, num_experts, slots, num_pairs, R;
};

// The row's group slot, or -1 when the row is left out (flags in *bad).
// srank / sscal / spair: the slots' ranks, scalings and pairs for expert e,
// read once into shared memory.
LORA_DEV int classify_row(const MoeGroupParams& p, const int* srank, const float* sscal,
                          const int* spair, int rho, uint32_t* bad) {
  const int s = p.row_slot[rho];
  if (s == -1) return -1;
  if (s < -1 || s >= p.slots) {
    *bad |= LORA_FLAG_BAD_SLOT;
    return -1;
  }
  const int pi = spair[s];
  if (pi == -1) return -1;
  if (pi < -1 || pi >= p.num_pairs) {
    *bad |= LORA_FLAG_BAD_PAIR;
    return -1;
  }
  const int r = srank[s];
  if (r < 0 || r > p.R) {
    *bad |= LORA_FLAG_BAD_RANK;
    return -1;
  }
  if (r == 0 || sscal[s] == 0.0f) return -1;
  return s;
}

__global__ void __launch_bounds__(kMgThreads) moe_group_kernel(const MoeGroupParams p) {
  extern __shared__ int sm[];
  int* cnt = sm;               // [slots] rows per slot
  int* cur = sm + p.slots;     // [slots] next position per slot
  int* srank = cur + p.slots;  // [slots]
  float* sscal = reinterpret_cast<float*>(srank + p.slots);   // [slots]
  int* spair = reinterpret_cast<int*>(sscal + p.slots);       // [slots] pair of (slot, e)
  int* cls = spair + p.slots;                                 // [kMgCache] row classes
  __shared__ int scratch[kMgThreads / 32];
  __shared__ int dead_cur;
  __shared__ uint32_t bad_all;
  const int e = blockIdx.x;
  const int E = p.num_experts;
  const int tid = threadIdx.x;
  if (tid == 0) {
    dead_cur = 0;
    bad_all = 0u;
  }
  // everything the classification needs besides the rows, in one round trip
  const int off0 = p.expert_offsets[e];
  const int off1 = p.expert_offsets[e + 1];
  int mine = 0;   // this thread saw a pair for expert e
  for (int s = tid; s < p.slots; s += kMgThreads) {
    cnt[s] = 0;
    srank[s] = p.ranks[s];
    sscal[s] = p.scalings[s];
    const int pi = p.pair_index[(size_t)s * E + e];
    spair[s] = pi;
    if (pi != -1) mine = 1;
  }
  const int adapted = __syncthreads_or(mine);
  int start = 0, end = 0;
  if (adapted) {
    start = off0;
    end = off1;
    if (start < 0 || end > p.rows_cap || end < start) {
      if (tid == 0) bad_all |= LORA_FLAG_BAD_OFFSETS;
      start = end = 0;
    }
  }
  uint32_t bad = 0;
  for (int rho = start + tid; rho < end; rho += kMgThreads) {
    const int s = classify_row(p, srank, sscal, spair, rho, &bad);
    if (rho - start < kMgCache) cls[rho - start] = s;
    if (s >= 0) atomicAdd(&cnt[s], 1);
  }
  if (bad) atomicOr(&bad_all, bad);
  __syncthreads();
  // segments: slot by slot inside the block, the left-out rows last
  int carry = 0;
  for (int base = 0; base < p.slots; base += kMgThreads) {
    const int s = base + tid;
    const int c = s < p.slots ? cnt[s] : 0;
    int tot;
    const int inc = block_inclusive_scan<kMgThreads>(c, scratch, &tot);
    if (s < p.slots) {
      const int lo = start + carry + inc - c;
      const size_t g = (size_t)s * E + e;
      cur[s] = lo;
      p.seg_lo[g] = lo;
      p.seg_hi[g] = lo + c;
      p.g_rank[g] = c > 0 ? p.ranks[s] : 0;
      p.g_scal[g] = c > 0 ? p.scalings[s] : 0.0f;
    }
    carry += tot;
  }
  __syncthreads();
  const int dead_lo = start + carry;
  for (int rho = start + tid; rho < end; rho += kMgThreads) {
    uint32_t unused = 0;
    const int s = rho - start < kMgCache ? cls[rho - start]
                                         : classify_row(p, srank, sscal, spair, rho, &unused);
    const int pos = s >= 0 ? atomicAdd(&cur[s], 1) : dead_lo + atomicAdd(&dead_cur, 1);
    p.token_order[pos] = rho;
  }
  __syncthreads();
  if (tid == 0) raise_flag(p.flags, bad_all);
}

}  // namespace

cudaError_t moe_group_launch(const int* expert_offsets, const int* pair_index, const int* row_slot,
                             const int* ranks, const float* scalings, int rows_cap,
                             int num_experts, int slots, int num_pairs, int R, int* token_order,
                             int* seg_lo, int* seg_hi, int* g_rank, float* g_scal,
                             uint32_t* flags, cudaStream_t stream) {
  MoeGroupParams p = {};
  p.expert_offsets = expert_offsets; p.pair_index = pair_index; p.row_slot = row_slot;
  p.ranks = ranks; p.scalings = scalings; p.token_order = token_order; p.seg_lo = seg_lo;
  p.seg_hi = seg_hi; p.g_rank = g_rank; p.g_scal = g_scal; p.flags = flags;
  p.rows_cap = rows_cap; p.num_experts = num_experts; p.slots = slots; p.num_pairs = num_pairs;
  p.R = R;
  const size_t smem = (size_t)5 * slots * sizeof(int) + (size_t)kMgCache * sizeof(int);
  if (smem > 48 * 1024) {
    const cudaError_t err = cudaFuncSetAttribute(
        moe_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
  }
  moe_group_kernel<<<num_experts, kMgThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace lora
