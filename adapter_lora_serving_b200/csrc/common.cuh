// Device helpers shared by the sm_100a LoRA delta kernels: PTX wrappers for
// mbarriers, bulk copies (TMA), thread-block clusters and warp MMAs, bounded
// waits, bf16 helpers and the work-item planners that every kernel runs on the
// device (no host round trip, so calls stay graph-capturable).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lora_delta.h"

#define LORA_DEV __device__ __forceinline__

namespace lora {

constexpr int kMaxSlices = LORA_MAX_SLICES;
// Upper bound for any single device wait (mbarrier phase, flag): 1 second.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// ---------------------------------------------------------------------------
// Small utilities
// ---------------------------------------------------------------------------

LORA_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// A load that acquires at GPU scope (pairs with a release or fence + atomic).
LORA_DEV uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

LORA_DEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

LORA_DEV void raise_flag(uint32_t* flags, uint32_t bits) {
  if (flags != nullptr && bits != 0) atomicOr(flags, bits);
}

LORA_DEV float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
LORA_DEV float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

LORA_DEV uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ---------------------------------------------------------------------------
// mbarrier (shared::cta) with bounded waits
// ---------------------------------------------------------------------------

LORA_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

LORA_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

LORA_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// Raises the expected transaction bytes of the current phase without arriving.
LORA_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

LORA_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

LORA_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the given phase parity; returns false if the limit expired.
LORA_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// Bulk copies (the TMA engine, untiled form)
// ---------------------------------------------------------------------------

// global -> this CTA's shared memory; completion is counted on `bar` in bytes.
// dst, src and bytes must all be multiples of 16.
LORA_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// shared -> global, tracked by the issuing thread's bulk group.
LORA_DEV void bulk_s2g(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}
// Hint: pull [src, src + bytes) into L2 (src and bytes multiples of 16).
LORA_DEV void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
LORA_DEV void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
LORA_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
LORA_DEV void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
LORA_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// 16-byte asynchronous copies global -> shared (per-thread groups)
// ---------------------------------------------------------------------------

LORA_DEV void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
LORA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
LORA_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch (no-ops when the launch has no such edge)
// ---------------------------------------------------------------------------

// Lets the next kernel in the stream start launching its CTAs.
LORA_DEV void grid_dep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Waits until the preceding kernel has completed and its writes are visible.
LORA_DEV void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Thread-block clusters
// ---------------------------------------------------------------------------

LORA_DEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
LORA_DEV uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
LORA_DEV uint32_t num_clusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Every thread of every CTA of the cluster must call this (hardware barrier).
LORA_DEV void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
LORA_DEV uint32_t dsmem_addr(const void* local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(local)), "r"(rank));
  return r;
}
LORA_DEV float dsmem_ld_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
LORA_DEV float4 dsmem_ld_f32x4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
LORA_DEV int dsmem_ld_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// Warp-level MMA (m16n8k16, bf16 x bf16 -> fp32) fed by ldmatrix
// ---------------------------------------------------------------------------

LORA_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
LORA_DEV void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}
LORA_DEV void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan helper (blockDim.x == NT, multiple of 32)
// ---------------------------------------------------------------------------

// Returns the inclusive prefix of `v` over the block and writes the block total
// to *total.  `scratch` holds NT/32 ints.  All threads must call it.
template <int NT>
LORA_DEV int block_inclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  int warp_prefix = 0;
  int tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    int s = scratch[w];
    if (w < warp) warp_prefix += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return x + warp_prefix;
}

// ---------------------------------------------------------------------------
// Work-item planners
// ---------------------------------------------------------------------------

// Linear / embedding targets.  Slot s takes part when its segment is valid
// (0 <= lo <= hi <= T), its rank is in (0, R] and, for the scaled operations
// (scalings != nullptr), its scaling is nonzero.  Its positions are cut into
// consecutive tiles of `tile`.  Writes prefix[0..slots] (exclusive prefix of
// tile counts) to shared memory and returns the item count.  Flags for bad
// segments and ranks are raised when `report` is set.  The segment of slot s
// is [slot_indptr[s], slot_indptr[s+1]), or [slot_indptr[s], seg_hi[s]) when
// seg_hi is given (segments that need not abut, e.g. the MoE fold's
// (slot, expert) groups).  seg_out (optional, shared memory): every slot's
// (lo, hi, rank, scaling bits) as read.
template <int NT>
LORA_DEV int plan_linear(const int* __restrict__ slot_indptr, const int* __restrict__ ranks,
                         const float* __restrict__ scalings, int slots, int T, int R, int tile,
                         int* prefix, int* scratch, uint32_t* flags, bool report,
                         const int* __restrict__ seg_hi = nullptr, int4* seg_out = nullptr) {
  uint32_t bad = 0;
  int carry = 0;
  if (threadIdx.x == 0) prefix[0] = 0;
  for (int base = 0; base < slots; base += NT) {
    const int s = base + threadIdx.x;
    int cnt = 0;
    if (s < slots) {
      const int lo = slot_indptr[s];
      const int hi = seg_hi != nullptr ? seg_hi[s] : slot_indptr[s + 1];
      const int r = ranks[s];
      const float sc = scalings != nullptr ? scalings[s] : 1.0f;
      // shared memory: the bounds, rank and scaling as read
      if (seg_out != nullptr) seg_out[s] = make_int4(lo, hi, r, __float_as_int(sc));
      const bool seg_ok = lo >= 0 && lo <= hi && hi <= T;
      const bool rank_ok = r >= 0 && r <= R;
      if (!seg_ok) bad |= LORA_FLAG_BAD_INDPTR;
      if (!rank_ok) bad |= LORA_FLAG_BAD_RANK;
      bool take = seg_ok && rank_ok && r > 0;
      if (take && sc == 0.0f) take = false;
      if (take) cnt = (hi - lo + tile - 1) / tile;
    }
    int tot;
    const int inc = block_inclusive_scan<NT>(cnt, scratch, &tot);
    if (s < slots) prefix[s + 1] = carry + inc;
    carry += tot;
  }
  if (report) raise_flag(flags, bad);
  __syncthreads();
  return carry;
}

// Largest s in [0, n) with prefix[s] <= item (prefix non-decreasing, prefix[0]=0).
LORA_DEV int find_segment(const int* prefix, int n, int item) {
  int lo = 0, hi = n;  // invariant: prefix[lo] <= item < prefix[hi] (prefix[n] = total)
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= item) lo = mid; else hi = mid;
  }
  return lo;
}

// MoE expert fold.  Expert e is adapted when any slot holds a pair for it
// (pair_index[s*E + e] != -1).  Its row block [off[e], off[e+1]) is used when
// valid (start >= 0, end <= rows_cap, end >= start; else BAD_OFFSETS) and
// non-empty, cut into chunks of `tile` rows.  Writes prefix[0..E].
template <int NT>
LORA_DEV int plan_expert(const int* __restrict__ offsets, const int* __restrict__ pair_index,
                         int E, int slots, int rows_cap, int tile, int* prefix, int* scratch,
                         uint32_t* flags, bool report) {
  uint32_t bad = 0;
  int carry = 0;
  if (threadIdx.x == 0) prefix[0] = 0;
  for (int base = 0; base < E; base += NT) {
    const int e = base + threadIdx.x;
    int cnt = 0;
    if (e < E) {
      bool adapted = false;
      for (int s = 0; s < slots && !adapted; ++s) adapted = pair_index[(size_t)s * E + e] != -1;
      if (adapted) {
        const int start = offsets[e];
        const int end = offsets[e + 1];
        if (start < 0 || end > rows_cap || end < start) {
          bad |= LORA_FLAG_BAD_OFFSETS;
        } else {
          cnt = (end - start + tile - 1) / tile;
        }
      }
    }
    int tot;
    const int inc = block_inclusive_scan<NT>(cnt, scratch, &tot);
    if (e < E) prefix[e + 1] = carry + inc;
    carry += tot;
  }
  if (report) raise_flag(flags, bad);
  __syncthreads();
  return carry;
}

}  // namespace lora
