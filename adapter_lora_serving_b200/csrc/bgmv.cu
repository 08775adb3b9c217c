// BGMV regime of the LoRA delta path (few tokens per slot): one thread-block
// cluster per work item of at most kTT tokens of one slot (or of one MoE
// expert chunk and slot).
//
// Shrink: each CTA of the cluster owns 1/kGroup of the input features.  The
// slot's live A rows and the item's x rows stream through a kNST-stage ring
// of shared memory by bulk copies (the TMA engine) and feed m16n8k16 warp MMAs
// (fp32 accumulate).  The kGroup partial h tiles are summed in a fixed order
// through distributed shared memory, so every CTA holds the same full h and
// h never leaves the chip.
// Expand: each CTA owns 1/kGroup of the output columns; a thread owns a column
// pair and does the rank-r dot products for every token of the item in fp32,
// then y = bf16_rne(y + scaling * acc) with coalesced 4-byte stores.
//
// Sources: mstar.engine.resources.lora.backend (LoraBackend.shrink,
// expand_fused, apply_linear_, gather_shrink, apply_) and
// spark_model/lora/expert_apply.rs (apply_expert_lora_sorted, with the
// per-(slot, expert) grouping the page plans as its grouped BGMV kernel).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace lora {

namespace {

struct Smem {
  uint64_t* bars;
  int* prefix;
  int* tok;
  int* ids;
  int* ctrl;     // [0..1] item count, [2..3] sub-batch count (by parity), [4] abort
  int* scratch;
  int* sub_s;
  int* sub_p;
  int* sub_cnt;
  int* sub_rows;
  uint8_t* ring;
  float* hpart;  // 2 buffers of kTT * srp
  float* hfull;  // kTT * srp
};

LORA_DEV Smem carve(uint8_t* base, const BgmvLayout& L) {
  Smem s;
  s.bars = reinterpret_cast<uint64_t*>(base);
  s.prefix = reinterpret_cast<int*>(base + L.prefix_off);
  int* m = reinterpret_cast<int*>(base + L.misc_off);
  s.tok = m;
  s.ids = m + kTT;
  s.ctrl = m + 2 * kTT;
  s.scratch = m + 2 * kTT + 8;
  s.sub_s = m + 2 * kTT + 16;
  s.sub_p = s.sub_s + kTT;
  s.sub_cnt = s.sub_p + kTT;
  s.sub_rows = s.sub_cnt + kTT;
  s.ring = base + L.ring_off;
  s.hpart = reinterpret_cast<float*>(base + L.hpart_off);
  s.hfull = reinterpret_cast<float*>(base + L.hfull_off);
  return s;
}

// Shrink of one item over this CTA's share of the input features into
// hpart[t * srp + i*Rpad + r] (t < kTT, every 16-row tile that holds a live
// row).  kbc counts ring stages consumed so far (same in every thread).
LORA_DEV void shrink_partial(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                             uint32_t& kbc, int w, int rank, int n, int nvalid, uint32_t crank,
                             float* hpart) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int Rpad = round_up_i(p.R, 16);
  const int kchunk = round_up_i(ceil_div_i(p.in, kGroup), kKB);
  const int k0 = min(p.in, (int)crank * kchunk);
  const int k1 = min(p.in, k0 + kchunk);
  const int nkb = ceil_div_i(k1 - k0, kKB);
  const int tps = ceil_div_i(rank, 16);
  const int RT = p.S * tps;
  const int NTt = ceil_div_i(n, 8);
  const int combos = RT * NTt;
  const int nrows_a = p.S * rank;
  const __nv_bfloat16* abase =
      reinterpret_cast<const __nv_bfloat16*>(p.a) + (size_t)w * p.S * p.R * p.in;
  const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(p.x);

  float acc[kMaxCombosPerWarp][4];
#pragma unroll
  for (int c = 0; c < kMaxCombosPerWarp; ++c)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[c][q] = 0.f;

  auto issue = [&](int kb, int st) {  // warp 0, converged
    const int kbase = k0 + kb * kKB;
    const int kv = min(kKB, k1 - kbase);
    const uint32_t rowbytes = (uint32_t)kv * 2u;
    uint8_t* stage = sm.ring + (size_t)st * L.stage_bytes;
    if (lane == 0) mbar_arrive_expect_tx(&sm.bars[st], (uint32_t)(nrows_a + nvalid) * rowbytes);
    __syncwarp();
    for (int q = lane; q < nrows_a + n; q += 32) {
      if (q < nrows_a) {
        const int i = q / rank;
        const int r = q - i * rank;
        bulk_g2s(stage + (size_t)(i * Rpad + r) * kRowStride,
                 abase + (size_t)(i * p.R + r) * p.in + kbase, rowbytes, &sm.bars[st]);
      } else {
        const int t = q - nrows_a;
        const int tk = sm.tok[t];
        if (tk >= 0)
          bulk_g2s(stage + (size_t)(L.srp + t) * kRowStride, xb + (size_t)tk * p.in + kbase,
                   rowbytes, &sm.bars[st]);
      }
    }
  };

  volatile int* abort_flag = &sm.ctrl[4];
  if (warp == 0 && *abort_flag == 0) {
    for (int kb = 0; kb < min(nkb, kNST); ++kb) issue(kb, (int)((kbc + kb) % kNST));
  }
  for (int kb = 0; kb < nkb; ++kb) {
    const uint32_t g = kbc + kb;
    const int st = (int)(g % kNST);
    const uint32_t parity = (g / kNST) & 1u;
    bool ok = (*abort_flag == 0);
    if (ok && !mbar_wait(&sm.bars[st], parity)) {
      ok = false;
      *abort_flag = 1;
      raise_flag(p.flags, LORA_FLAG_TIMEOUT);
    }
    if (ok) {
      const int kv = min(kKB, k1 - (k0 + kb * kKB));
      const int nks = ceil_div_i(kv, 16);
      const uint32_t stage_addr = smem_u32(sm.ring + (size_t)st * L.stage_bytes);
#pragma unroll
      for (int ci = 0; ci < kMaxCombosPerWarp; ++ci) {
        const int combo = warp + ci * (kBgmvThreads / 32);
        if (combo < combos) {
          const int rt = combo / NTt;
          const int nt = combo - rt * NTt;
          const int i = rt / tps;
          const int r0 = (rt - i * tps) * 16;
          const uint32_t a_addr =
              stage_addr + (uint32_t)(i * Rpad + r0 + (lane & 15)) * kRowStride + (lane >> 4) * 16;
          const uint32_t x_addr = stage_addr +
                                  (uint32_t)(L.srp + nt * 8 + (lane & 7)) * kRowStride +
                                  ((lane >> 3) & 1) * 16;
          for (int ks = 0; ks < nks; ++ks) {
            uint32_t a0, a1, a2, a3, b0, b1;
            ldsm_x4(a_addr + ks * 32, a0, a1, a2, a3);
            ldsm_x2(x_addr + ks * 32, b0, b1);
            if (kv - ks * 16 < 16) {  // only 8 valid input features in this step
              a2 = 0u;
              a3 = 0u;
              b1 = 0u;
            }
            mma_bf16_16816(acc[ci], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
    __syncthreads();
    if (warp == 0 && kb + kNST < nkb && *abort_flag == 0) issue(kb + kNST, st);
  }
  kbc += (uint32_t)nkb;

  // Scatter the warp tiles into hpart.
  const int g8 = lane >> 2;
  const int c4 = lane & 3;
#pragma unroll
  for (int ci = 0; ci < kMaxCombosPerWarp; ++ci) {
    const int combo = warp + ci * (kBgmvThreads / 32);
    if (combo < combos) {
      const int rt = combo / NTt;
      const int nt = combo - rt * NTt;
      const int i = rt / tps;
      const int row = i * Rpad + (rt - i * tps) * 16 + g8;
      const int t0 = nt * 8 + 2 * c4;
      hpart[t0 * L.srp + row] = acc[ci][0];
      hpart[(t0 + 1) * L.srp + row] = acc[ci][1];
      hpart[t0 * L.srp + row + 8] = acc[ci][2];
      hpart[(t0 + 1) * L.srp + row + 8] = acc[ci][3];
    }
  }
}

// Sum the kGroup partial tiles (fixed order) into this CTA's hfull.
LORA_DEV void cluster_reduce(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                             const float* hpart, int rank, int n) {
  const int Rpad = round_up_i(p.R, 16);
  const int live = p.S * rank;
  for (int e = threadIdx.x; e < n * live; e += kBgmvThreads) {
    const int t = e / live;
    const int q = e - t * live;
    const int i = q / rank;
    const int col = i * Rpad + (q - i * rank);
    const float* src = hpart + t * L.srp + col;
    float s = 0.f;
#pragma unroll
    for (int c = 0; c < kGroup; ++c) s += dsmem_ld_f32(dsmem_addr(src, (uint32_t)c));
    sm.hfull[t * L.srp + col] = s;
  }
}

// Expand of one item over this CTA's share of the output columns:
// y[row, j] = bf16(y + scal * sum_{r<rank} hfull[t, i*Rpad + r] * b[w, j, r]).
LORA_DEV void expand_part(const BgmvParams& p, const BgmvLayout& L, const Smem& sm, int w,
                          int rank, float scal, int n, uint32_t rowmask, uint32_t crank) {
  const int out = p.out;
  const int Rpad = round_up_i(p.R, 16);
  const int ochunk = round_up_i(ceil_div_i(out, kGroup), 8);
  const int j0 = min(out, (int)crank * ochunk);
  const int j1 = min(out, j0 + ochunk);
  const int npairs = (j1 - j0) >> 1;
  const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(p.b) + (size_t)w * out * p.R;
  uint32_t* y32 = reinterpret_cast<uint32_t*>(p.y);
  int rowoff[kTT];
#pragma unroll
  for (int t = 0; t < kTT; ++t) rowoff[t] = (t < n && ((rowmask >> t) & 1u)) ? sm.tok[t] : -1;

  for (int cp = threadIdx.x; cp < npairs; cp += kBgmvThreads) {
    const int j = j0 + 2 * cp;
    int i = 0;
    while (i + 1 < p.S && p.slice_off[i + 1] <= j) ++i;
    const float* hbase = sm.hfull + i * Rpad;
    uint32_t yv[kTT];
#pragma unroll
    for (int t = 0; t < kTT; ++t)
      yv[t] = rowoff[t] >= 0 ? y32[((size_t)rowoff[t] * out + j) >> 1] : 0u;
    float acc0[kTT], acc1[kTT];
#pragma unroll
    for (int t = 0; t < kTT; ++t) { acc0[t] = 0.f; acc1[t] = 0.f; }
    const __nv_bfloat16* b0p = bb + (size_t)j * p.R;
    for (int rc = 0; rc < rank; rc += 8) {
      const uint4 u0 = __ldg(reinterpret_cast<const uint4*>(b0p + rc));
      const uint4 u1 = __ldg(reinterpret_cast<const uint4*>(b0p + p.R + rc));
      float bv0[8], bv1[8];
      bv0[0] = bf16_lo(u0.x); bv0[1] = bf16_hi(u0.x); bv0[2] = bf16_lo(u0.y); bv0[3] = bf16_hi(u0.y);
      bv0[4] = bf16_lo(u0.z); bv0[5] = bf16_hi(u0.z); bv0[6] = bf16_lo(u0.w); bv0[7] = bf16_hi(u0.w);
      bv1[0] = bf16_lo(u1.x); bv1[1] = bf16_hi(u1.x); bv1[2] = bf16_lo(u1.y); bv1[3] = bf16_hi(u1.y);
      bv1[4] = bf16_lo(u1.z); bv1[5] = bf16_hi(u1.z); bv1[6] = bf16_lo(u1.w); bv1[7] = bf16_hi(u1.w);
      const int ql = min(8, rank - rc);
#pragma unroll
      for (int t = 0; t < kTT; ++t) {
        if (t < n) {
          const float* hp = hbase + t * L.srp + rc;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            if (q < ql) {
              const float hv = hp[q];
              acc0[t] = fmaf(hv, bv0[q], acc0[t]);
              acc1[t] = fmaf(hv, bv1[q], acc1[t]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kTT; ++t) {
      if (rowoff[t] >= 0) {
        const float lo = fmaf(scal, acc0[t], bf16_lo(yv[t]));
        const float hi = fmaf(scal, acc1[t], bf16_hi(yv[t]));
        y32[((size_t)rowoff[t] * out + j) >> 1] = pack_bf16x2(lo, hi);
      }
    }
  }
}

// Write the live columns of hfull to global h (tokens t with t % kGroup == crank).
LORA_DEV void store_h(const BgmvParams& p, const BgmvLayout& L, const Smem& sm, int rank, int n,
                      uint32_t rowmask_any, uint32_t crank) {
  const int Rpad = round_up_i(p.R, 16);
  const int live = p.S * rank;
  const int SR = p.S * p.R;
  for (int e = threadIdx.x; e < n * live; e += kBgmvThreads) {
    const int t = e / live;
    if ((t % kGroup) != (int)crank || !((rowmask_any >> t) & 1u)) continue;
    const int q = e - t * live;
    const int i = q / rank;
    const int r = q - i * rank;
    p.h[(size_t)sm.tok[t] * SR + i * p.R + r] = sm.hfull[t * L.srp + i * Rpad + r];
  }
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kBgmvThreads) bgmv_kernel(const BgmvParams p) {
  constexpr bool kClustered = (MODE == kModeFused || MODE == kModeShrink || MODE == kModeExpert);
  constexpr bool kScaled = (MODE == kModeFused || MODE == kModeExpand || MODE == kModeEmbed ||
                            MODE == kModeExpert);
  extern __shared__ __align__(128) uint8_t smem_raw[];
  const int npref = (MODE == kModeExpert) ? p.num_experts : p.slots;
  const BgmvLayout L = bgmv_layout(MODE, npref, p.S, p.R);
  const Smem sm = carve(smem_raw, L);
  const int tid = threadIdx.x;

  uint32_t crank, group, ngroups;
  if (kClustered) {
    crank = cluster_ctarank();
    group = cluster_id_x();
    ngroups = num_clusters_x();
  } else {
    crank = blockIdx.x % kGroup;
    group = blockIdx.x / kGroup;
    ngroups = gridDim.x / kGroup;
  }

  if (tid == 0) {
    for (int st = 0; st < kNST; ++st) mbar_init(&sm.bars[st], 1);
    fence_mbar_init();
    sm.ctrl[4] = 0;
  }
  __syncthreads();

  const bool report = (blockIdx.x == 0);
  int total;
  if (MODE == kModeExpert) {
    total = plan_expert<kBgmvThreads>(p.expert_offsets, p.pair_index, p.num_experts, p.slots, p.T,
                                      kTT, sm.prefix, sm.scratch, p.flags, report);
  } else {
    total = plan_linear<kBgmvThreads>(p.slot_indptr, p.ranks, kScaled ? p.scalings : nullptr,
                                      p.slots, p.T, p.R, kTT, sm.prefix, sm.scratch, p.flags,
                                      report);
  }
  if (kClustered) {
    // The trip count of every loop that contains a cluster barrier comes from
    // rank 0, so all CTAs of a cluster take the same barriers.
    if (tid == 0) sm.ctrl[0] = total;
    cluster_sync();
    total = dsmem_ld_s32(dsmem_addr(&sm.ctrl[0], 0));
  }

  uint32_t kbc = 0;
  int hpar = 0;
  int iter = 0;
  for (int item = (int)group; item < total; item += (int)ngroups, ++iter) {
    if (MODE != kModeExpert) {
      // ---- linear / embedding item: (slot, tile) ----
      const int s = find_segment(sm.prefix, p.slots, item);
      const int j = item - sm.prefix[s];
      const int p0 = p.slot_indptr[s] + j * kTT;
      const int n = max(0, min(kTT, p.slot_indptr[s + 1] - p0));
      const int rank = p.ranks[s];
      const float scal = kScaled ? p.scalings[s] : 0.f;
      const bool emb = (MODE == kModeEmbed || MODE == kModeGather);
      if (tid < kTT) {
        int t = -1;
        int id = -1;
        if (tid < n && p0 + tid >= 0 && p0 + tid < p.T) {
          t = p.token_order[p0 + tid];
          if (t < 0 || t >= p.T) {
            if (crank == 0) raise_flag(p.flags, LORA_FLAG_BAD_TOKEN);
            t = -1;
          }
          if (emb && t >= 0) {
            id = p.ids[t];
            if (id < 0 || id >= p.in) id = -1;
          }
        }
        sm.tok[tid] = t;
        sm.ids[tid] = id;
      }
      __syncthreads();
      uint32_t tokmask = 0, idmask = 0;
      int nvalid = 0;
#pragma unroll
      for (int t = 0; t < kTT; ++t) {
        if (sm.tok[t] >= 0) { tokmask |= 1u << t; ++nvalid; }
        if (sm.ids[t] >= 0) idmask |= 1u << t;
      }
      const int Rpad = round_up_i(p.R, 16);
      if (MODE == kModeFused || MODE == kModeShrink) {
        float* hp = sm.hpart + (size_t)hpar * kTT * L.srp;
        shrink_partial(p, L, sm, kbc, s, rank, n, nvalid, crank, hp);
        cluster_sync();
        cluster_reduce(p, L, sm, hp, rank, n);
        hpar ^= 1;
        __syncthreads();
      } else {
        // gather or load h for every live column of every token of the item
        const int live = p.S * rank;
        for (int e = tid; e < n * live; e += kBgmvThreads) {
          const int t = e / live;
          const int q = e - t * live;
          const int i = q / rank;
          const int r = q - i * rank;
          float v = 0.f;
          if (MODE == kModeExpand) {
            if ((tokmask >> t) & 1u) v = p.h[(size_t)sm.tok[t] * p.S * p.R + i * p.R + r];
          } else {
            if ((idmask >> t) & 1u) {
              const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(p.a);
              v = __bfloat162float(ab[((size_t)s * p.S * p.R + i * p.R + r) * p.in + sm.ids[t]]);
            }
          }
          sm.hfull[t * L.srp + i * Rpad + r] = v;
        }
        __syncthreads();
      }
      if (MODE == kModeShrink || MODE == kModeGather) {
        store_h(p, L, sm, rank, n, tokmask, crank);
      } else {
        const uint32_t rowmask = (MODE == kModeEmbed) ? (tokmask & idmask) : tokmask;
        expand_part(p, L, sm, s, rank, scal, n, rowmask, crank);
      }
      __syncthreads();
    } else {
      // ---- MoE item: chunk of one expert's rows, split by slot ----
      const int E = p.num_experts;
      const int e = find_segment(sm.prefix, E, item);
      const int chunk = item - sm.prefix[e];
      const int start = p.expert_offsets[e] + chunk * kTT;
      const int m = max(0, min(kTT, p.expert_offsets[e + 1] - start));
      int* nsub_slot = &sm.ctrl[2 + (iter & 1)];
      if (tid == 0) {
        uint32_t bad = 0;
        int rs[kTT];
        int rp[kTT];
        for (int q = 0; q < kTT; ++q) {
          rs[q] = -1;
          rp[q] = -1;
          if (q >= m) continue;
          const int rho = start + q;
          if (rho < 0 || rho >= p.T) continue;
          const int s = p.row_slot[rho];
          if (s == -1) continue;
          if (s < -1 || s >= p.slots) { bad |= LORA_FLAG_BAD_SLOT; continue; }
          const int pi = p.pair_index[(size_t)s * E + e];
          if (pi == -1) continue;
          if (pi < -1 || pi >= p.num_pairs) { bad |= LORA_FLAG_BAD_PAIR; continue; }
          const int r = p.ranks[s];
          if (r < 0 || r > p.R) { bad |= LORA_FLAG_BAD_RANK; continue; }
          if (r == 0 || p.scalings[s] == 0.0f) continue;
          rs[q] = s;
          rp[q] = pi;
        }
        // sub-batches in ascending slot order, rows in row order
        int nsub = 0;
        int last = -1;
        while (true) {
          int best = 0x7fffffff;
          for (int q = 0; q < kTT; ++q)
            if (rs[q] > last && rs[q] < best) best = rs[q];
          if (best == 0x7fffffff) break;
          int cnt = 0;
          for (int q = 0; q < kTT; ++q) {
            if (rs[q] == best) {
              sm.sub_rows[nsub * kTT + cnt] = start + q;
              sm.sub_p[nsub] = rp[q];
              ++cnt;
            }
          }
          sm.sub_s[nsub] = best;
          sm.sub_cnt[nsub] = cnt;
          ++nsub;
          last = best;
        }
        *nsub_slot = nsub;
        if (crank == 0) raise_flag(p.flags, bad);
      }
      __syncthreads();
      const int my_nsub = *nsub_slot;
      cluster_sync();
      const int nsub = dsmem_ld_s32(dsmem_addr(nsub_slot, 0));
      for (int q = 0; q < nsub; ++q) {
        const bool mine = q < my_nsub;
        const int s = mine ? sm.sub_s[q] : 0;
        const int w = mine ? sm.sub_p[q] : 0;
        const int n = mine ? sm.sub_cnt[q] : 0;
        const int rank = mine ? p.ranks[s] : 0;
        const float scal = mine ? p.scalings[s] : 0.f;
        if (tid < kTT) sm.tok[tid] = (tid < n) ? sm.sub_rows[q * kTT + tid] : -1;
        __syncthreads();
        const uint32_t mask = (n >= 32) ? 0xffffffffu : ((1u << n) - 1u);
        float* hp = sm.hpart + (size_t)hpar * kTT * L.srp;
        shrink_partial(p, L, sm, kbc, w, rank, n, n, crank, hp);
        cluster_sync();
        cluster_reduce(p, L, sm, hp, rank, n);
        hpar ^= 1;
        __syncthreads();
        expand_part(p, L, sm, w, rank, scal, n, mask, crank);
        __syncthreads();
      }
    }
  }
  if (kClustered) cluster_sync();  // peers may still read this CTA's shared memory
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------

namespace {

// Per (device, mode, shared-memory size): the number of work groups one launch
// uses.  Filled on the first call with those shapes; later calls (and calls
// during stream capture) only read it.
struct LaunchCacheEntry {
  int dev, mode, smem, groups;
};
std::mutex g_cache_mu;
LaunchCacheEntry g_cache[64];
int g_cache_n = 0;

template <int MODE>
cudaError_t launch_mode(const BgmvParams& p, int max_items, cudaStream_t stream,
                        const char** why) {
  constexpr bool kClustered = (MODE == kModeFused || MODE == kModeShrink || MODE == kModeExpert);
  const int npref = (MODE == kModeExpert) ? p.num_experts : p.slots;
  const BgmvLayout L = bgmv_layout(MODE, npref, p.S, p.R);
  auto kern = bgmv_kernel<MODE>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.blockDim = dim3(kBgmvThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  if (kClustered) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kGroup;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }

  int groups = -1;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    for (int i = 0; i < g_cache_n; ++i)
      if (g_cache[i].dev == dev && g_cache[i].mode == MODE && g_cache[i].smem == L.total)
        groups = g_cache[i].groups;
  }
  if (groups < 0) {
    int max_optin = 0;
    err = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err != cudaSuccess) return err;
    if (L.total > max_optin) {
      *why = "shared memory needed by the BGMV kernel exceeds the device limit";
      return cudaErrorInvalidConfiguration;
    }
    // Allow the device maximum once: a later call with a smaller layout must
    // not lower the limit a cached larger layout relies on.
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin);
    if (err != cudaSuccess) return err;
    int sms = 0;
    err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    if (kClustered) {
      cfg.gridDim = dim3(kGroup * 64, 1, 1);
      int active = 0;
      err = cudaOccupancyMaxActiveClusters(&active, kern, &cfg);
      if (err != cudaSuccess) return err;
      if (active <= 0) {
        *why = "no thread-block cluster of the BGMV kernel fits on this device";
        return cudaErrorInvalidConfiguration;
      }
      groups = active;
    } else {
      int per_sm = 0;
      err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kBgmvThreads, L.total);
      if (err != cudaSuccess) return err;
      if (per_sm <= 0) {
        *why = "the BGMV kernel does not fit on one SM";
        return cudaErrorInvalidConfiguration;
      }
      groups = max(1, per_sm * sms / kGroup);
    }
    std::lock_guard<std::mutex> lk(g_cache_mu);
    if (g_cache_n < 64) g_cache[g_cache_n++] = {dev, MODE, L.total, groups};
  }
  groups = max(1, min(groups, max_items));
  cfg.gridDim = dim3((unsigned)(groups * kGroup), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t bgmv_launch(int mode, const BgmvParams& p, int max_items, cudaStream_t stream,
                        const char** why) {
  switch (mode) {
    case kModeFused: return launch_mode<kModeFused>(p, max_items, stream, why);
    case kModeShrink: return launch_mode<kModeShrink>(p, max_items, stream, why);
    case kModeExpand: return launch_mode<kModeExpand>(p, max_items, stream, why);
    case kModeEmbed: return launch_mode<kModeEmbed>(p, max_items, stream, why);
    case kModeGather: return launch_mode<kModeGather>(p, max_items, stream, why);
    case kModeExpert: return launch_mode<kModeExpert>(p, max_items, stream, why);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lora
