// BGMV regime of the LoRA delta path (few tokens per slot): one thread-block
// cluster of kGroup CTAs per work item of at most kTT tokens of one slot; the
// MoE fold runs one CTA per kTT-row chunk of an expert instead.
//
// Shrink: each CTA of the cluster owns 1/kGroup of the input features.  The
// slot's live A rows and the item's x rows are staged in padded shared-memory
// rows (16-byte cp.async, or one bulk copy per 1 KB row) and feed m16n8k16
// warp MMAs (fp32 accumulate).  The kGroup partial h tiles are summed in a
// fixed order through distributed shared memory, so every CTA holds the same
// full h and h never leaves the chip.
// Expand: each CTA owns 1/kGroup of the output columns.  For the fused path
// the slot's B columns and the item's y rows are bulk-copied into the idle
// staging ring while the cluster reduces h; m16n8k16 MMAs (columns as M,
// tokens as N, h = hi + lo in bf16) update y in shared memory, which is then
// written back with coalesced 16-byte stores.  y = bf16_rne(y + scaling * acc).
//
// Sources: mstar.engine.resources.lora.backend (LoraBackend.shrink,
// expand_fused, apply_linear_, gather_shrink, apply_) and
// spark_model/lora/expert_apply.rs (apply_expert_lora_sorted, with the
// per-(slot, expert) grouping the page plans as its grouped BGMV kernel).
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "expand_tile.cuh"
#include "kernels.h"

namespace lora {

static_assert(kTT == 32, "token masks are warp ballots: one token per lane of warp 0");

namespace {

struct Smem {
  int* prefix;
  int* tok;
  int* ids;
  int* ctrl;     // [0] item count, [2..3] sub-batch count (by parity)
  int* scratch;
  int* sub_s;
  int* sub_p;
  int* sub_cnt;
  int* sub_rows;
  uint8_t* ring;
  float* hpart;     // 2 buffers of kTT * srp (cluster partial sums)
  uint16_t* hhi;    // [S][kTT][hst]
  uint16_t* hlo;    // [S][kTT][hst]
};

LORA_DEV Smem carve(uint8_t* base, const BgmvLayout& L) {
  Smem s;
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
  s.hhi = reinterpret_cast<uint16_t*>(base + L.hhi_off);
  s.hlo = reinterpret_cast<uint16_t*>(base + L.hlo_off);
  return s;
}

// Geometry of the shrink of one item on this CTA.
struct ShrinkGeom {
  int k0, k1, nkb;   // this CTA's input features [k0, k1), in stages of p.kb
  int nrows_a;       // live A rows: S * rank
};

LORA_DEV ShrinkGeom shrink_geom(const BgmvParams& p, int rank, uint32_t crank) {
  ShrinkGeom G;
  G.k0 = min(p.in, (int)crank * p.kchunk);
  G.k1 = min(p.in, G.k0 + p.kchunk);
  G.nkb = ceil_div_i(G.k1 - G.k0, p.kb);
  G.nrows_a = p.S * rank;
  return G;
}

// Which staged rows of a stage an issue covers.
enum RowSet : int { kRowsA = 1, kRowsX = 2, kRowsAll = 3 };

// Every thread issues its share of the 16-byte asynchronous copies of stage kb
// into ring slot st and commits them as one group: the live A rows of adapter
// w (rows below nrows_a, at i*Rpad + r) and/or the item's x rows (tokens
// t < n with a valid token, at srp + t), kv input features each; a warp copies
// a row.  (Measured on B200: a round of small per-row copies lands sooner
// through cp.async than through the bulk-copy engine, and the shrink's stages
// are latency bound.)
LORA_DEV void issue_rows(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                         const ShrinkGeom& G, int w, int rank, int n, int kb, int st, int set) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int kbase = G.k0 + kb * p.kb;
  const int cpr = min(p.kb, G.k1 - kbase) >> 3;   // 16-byte chunks per row
  const int Rpad = round_up_i(p.R, 16);
  const uint32_t stage = smem_u32(sm.ring) + (uint32_t)(st * L.stage_bytes);
  if ((set & kRowsA) != 0 && G.nrows_a > 0) {
    // (slice, rank row) of this warp's first A row, advanced 8 rows per step
    int ai = warp / rank;
    int ar = warp - ai * rank;
    for (int row = warp; row < G.nrows_a; row += kBgmvThreads / 32) {
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.a) +
                                 ((size_t)w * p.S * p.R + ai * p.R + ar) * p.in + kbase;
      const uint32_t dst = stage + (uint32_t)((ai * Rpad + ar) * L.row_stride);
      for (int c = lane; c < cpr; c += 32) cp_async16(dst + c * 16, src + c * 8);
      ar += kBgmvThreads / 32;
      while (ar >= rank) {
        ar -= rank;
        ++ai;
      }
    }
  }
  if ((set & kRowsX) != 0) {
    for (int t = warp; t < n; t += kBgmvThreads / 32) {
      const int tk = sm.tok[t];
      if (tk < 0) continue;
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.x) + (size_t)tk * p.in + kbase;
      const uint32_t dst = stage + (uint32_t)((L.srp + t) * L.row_stride);
      for (int c = lane; c < cpr; c += 32) cp_async16(dst + c * 16, src + c * 8);
    }
  }
  cp_async_commit();
}

// Warp 0 issues the same rows as bulk copies (the TMA engine), completing on
// bar: kRowsA only raises the expected bytes, the other sets also arrive (one
// arrival per phase).  Used when stage rows are wide (p.bulk_stage): one copy
// per 1 KB row issues far fewer instructions than 16-byte copies.  Every
// address and size is a multiple of 16 bytes.
LORA_DEV void issue_rows_bulk(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                              const ShrinkGeom& G, int w, int rank, int n, int kb, int st,
                              int set, uint64_t* bar) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const int kbase = G.k0 + kb * p.kb;
  const uint32_t rbytes = (uint32_t)(min(p.kb, G.k1 - kbase) * 2);
  const int Rpad = round_up_i(p.R, 16);
  uint8_t* stage = sm.ring + st * L.stage_bytes;
  const bool want_a = (set & kRowsA) != 0 && G.nrows_a > 0;
  const bool xrow = (set & kRowsX) != 0 && lane < n && sm.tok[lane] >= 0;
  const uint32_t xmask = __ballot_sync(0xffffffffu, xrow);
  if (lane == 0) {
    fence_proxy_async_smem();
    const uint32_t bytes =
        ((want_a ? (uint32_t)G.nrows_a : 0u) + (uint32_t)__popc(xmask)) * rbytes;
    if (set == kRowsA)
      mbar_expect_tx(bar, bytes);
    else
      mbar_arrive_expect_tx(bar, bytes);
  }
  __syncwarp();
  if (want_a) {
    int ai = lane / rank;
    int ar = lane - ai * rank;
    for (int row = lane; row < G.nrows_a; row += 32) {
      const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(p.a) +
                                 ((size_t)w * p.S * p.R + ai * p.R + ar) * p.in + kbase;
      bulk_g2s(stage + (ai * Rpad + ar) * L.row_stride, src, rbytes, bar);
      ar += 32;
      while (ar >= rank) {
        ar -= rank;
        ++ai;
      }
    }
  }
  if (xrow) {
    const __nv_bfloat16* src =
        reinterpret_cast<const __nv_bfloat16*>(p.x) + (size_t)sm.tok[lane] * p.in + kbase;
    bulk_g2s(stage + (L.srp + lane) * L.row_stride, src, rbytes, bar);
  }
}

// Warp-uniform bounded wait for phase `parity` of bar; on timeout raises
// LORA_FLAG_TIMEOUT and waits once more (bounded) so that no copy is still in
// flight when the shared memory is reused.
LORA_DEV void wait_stage(uint64_t* bar, uint32_t parity, uint32_t* flags) {
  if ((threadIdx.x & 31) == 0) {
    if (!mbar_wait(bar, parity)) {
      raise_flag(flags, LORA_FLAG_TIMEOUT);
      mbar_wait(bar, parity);
    }
  }
  __syncwarp();
}

// Copies of the shrink's stages: per-thread cp.async groups, or bulk copies
// on the ring slots' mbarriers (sbar, phase parity bit st of sph).
struct StageCopies {
  bool bulk;
  uint64_t* sbar;
  uint32_t sph;
};

LORA_DEV void issue_stage(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                          const ShrinkGeom& G, int w, int rank, int n, int kb, int st, int set,
                          StageCopies& sc) {
  if (sc.bulk)
    issue_rows_bulk(p, L, sm, G, w, rank, n, kb, st, set, &sc.sbar[st]);
  else
    issue_rows(p, L, sm, G, w, rank, n, kb, st, set);
}

// MMAs of the shrink over this CTA's input features into hpart[t * srp +
// i*Rpad + r] (every 16-row tile holding a live row, t < 8*ceil(n/8)).  The
// caller has issued the A rows of stage 0 (kRowsA); this issues the rest.
LORA_DEV void shrink_partial(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                             const ShrinkGeom& G, int w, int rank, int n, float* hpart,
                             StageCopies& sc) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int Rpad = round_up_i(p.R, 16);
  const int tps = ceil_div_i(rank, 16);
  const int RT = p.S * tps;
  const int NTt = ceil_div_i(n, 8);
  const int combos = RT * NTt;
  const int stride = L.row_stride;

  float acc[kMaxCombosPerWarp][4];
#pragma unroll
  for (int c = 0; c < kMaxCombosPerWarp; ++c)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[c][q] = 0.f;

  if (G.nkb > 0) {
    issue_stage(p, L, sm, G, w, rank, n, 0, 0, kRowsX, sc);
    if (G.nkb > 1 && p.nst == 2) issue_stage(p, L, sm, G, w, rank, n, 1, 1, kRowsAll, sc);
  }
  for (int kb = 0; kb < G.nkb; ++kb) {
    const int st = kb % p.nst;
    if (sc.bulk) {
      wait_stage(&sc.sbar[st], (sc.sph >> st) & 1u, p.flags);
      sc.sph ^= 1u << st;
    } else {
      if (kb + 1 < G.nkb && p.nst == 2) cp_async_wait<1>(); else cp_async_wait<0>();
      __syncthreads();
    }
    const int kv = min(p.kb, G.k1 - (G.k0 + kb * p.kb));
    const int nks = ceil_div_i(kv, 16);
    const uint32_t stage_addr = smem_u32(sm.ring) + (uint32_t)(st * L.stage_bytes);
#pragma unroll
    for (int ci = 0; ci < kMaxCombosPerWarp; ++ci) {
      const int combo = warp + ci * (kBgmvThreads / 32);
      if (combo < combos) {
        const int rt = combo / NTt;
        const int nt = combo - rt * NTt;
        const int i = rt / tps;
        const int r0 = (rt - i * tps) * 16;
        const uint32_t a_addr =
            stage_addr + (uint32_t)((i * Rpad + r0 + (lane & 15)) * stride + (lane >> 4) * 16);
        const uint32_t x_addr =
            stage_addr + (uint32_t)((L.srp + nt * 8 + (lane & 7)) * stride + ((lane >> 3) & 1) * 16);
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
    __syncthreads();
    if (kb + p.nst < G.nkb) issue_stage(p, L, sm, G, w, rank, n, kb + p.nst, st, kRowsAll, sc);
  }

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

// Where the h of an item comes from.
enum HSource : int { kFromCluster = 0, kFromGlobal = 1, kFromGather = 2, kFromLocal = 3 };

// Produce h for every (token t < kTT, slice i, column r < roundup16(rank)) of
// the item -- the value for live tokens and r < rank, 0 elsewhere -- four
// columns per thread.  Writes the bf16 hi/lo tiles the expand MMAs read and/or
// the fp32 global h (tokens t % kGroup == crank).  Cluster partials are summed
// in the fixed order 0..kGroup-1, so every CTA of the cluster holds the same h.
template <int SRC>
LORA_DEV void produce_h(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                        const float* hpart, int w, int rank, int n, uint32_t rowmask,
                        bool want_tiles, bool want_global, uint32_t crank) {
  const int Rpad = round_up_i(p.R, 16);
  const int q4 = ceil_div_i(rank, 16) * 4;     // groups of 4 columns per slice
  const int per_t = p.S * q4;
  // rows of the token tiles the expand reads (8 * ceil(n / 8) <= kTT)
  const int total = round_up_i(n, 8) * per_t;
  for (int e = threadIdx.x; e < total; e += kBgmvThreads) {
    const int t = e / per_t;
    const int q = e - t * per_t;
    const int i = q / q4;
    const int r0 = (q - i * q4) * 4;
    const bool row_live = t < n && ((rowmask >> t) & 1u);
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (row_live && r0 < rank) {
      if (SRC == kFromCluster) {
        const float* src = hpart + t * L.srp + i * Rpad + r0;
#pragma unroll
        for (int c = 0; c < kGroup; ++c) {
          const float4 f = dsmem_ld_f32x4(dsmem_addr(src, (uint32_t)c));
          v[0] += f.x; v[1] += f.y; v[2] += f.z; v[3] += f.w;
        }
      } else if (SRC == kFromLocal) {
        const float4 f = *reinterpret_cast<const float4*>(hpart + t * L.srp + i * Rpad + r0);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
      } else if (SRC == kFromGlobal) {
        const float* hg = p.h + (size_t)sm.tok[t] * p.S * p.R + i * p.R + r0;
#pragma unroll
        for (int k = 0; k < 4; ++k) v[k] = (r0 + k < rank) ? hg[k] : 0.f;
      } else {
        const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(p.a) +
                                  ((size_t)w * p.S * p.R + i * p.R + r0) * p.in + sm.ids[t];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          v[k] = (r0 + k < rank) ? __bfloat162float(ab[(size_t)k * p.in]) : 0.f;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (r0 + k >= rank) v[k] = 0.f;
    }
    if (want_tiles) {
      uint32_t hi2[2], lo2[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
        const float2 hf = __bfloat1622float2(h2);
        const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * k] - hf.x, v[2 * k + 1] - hf.y);
        hi2[k] = *reinterpret_cast<const uint32_t*>(&h2);
        lo2[k] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      const int o = (i * kTT + t) * L.hst + r0;
      *reinterpret_cast<uint2*>(sm.hhi + o) = make_uint2(hi2[0], hi2[1]);
      *reinterpret_cast<uint2*>(sm.hlo + o) = make_uint2(lo2[0], lo2[1]);
    }
    if (want_global && t < n && (t % kGroup) == (int)crank) {
      const int tk = sm.tok[t];
      if (tk >= 0) {
        float* hg = p.h + (size_t)tk * p.S * p.R + i * p.R + r0;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (r0 + k < rank) hg[k] = v[k];
      }
    }
  }
}

// Zero the four B elements k0..k0+3 (bf16 pairs lo = (k0, k0+1), hi =
// (k0+2, k0+3)) at or past the rank.
LORA_DEV uint2 mask_rank4(uint2 v, int k0, int rank) {
  if (k0 + 3 < rank) return v;
  const uint32_t m0 = (k0 < rank ? 0xffffu : 0u) | (k0 + 1 < rank ? 0xffff0000u : 0u);
  const uint32_t m1 = (k0 + 2 < rank ? 0xffffu : 0u) | (k0 + 3 < rank ? 0xffff0000u : 0u);
  return make_uint2(v.x & m0, v.y & m1);
}

// Expand of one item over the output columns [j0, j1) with
// m16n8k16 MMAs: D[16 columns, 8 tokens] = B[16 columns, 16 ranks] H^T.
// MMA row m < 8 is column 2m and row m + 8 is column 2m + 1 of the tile, and
// MMA k (2c + e) / (2c + 8 + e) is rank 4c + e / 4c + 2 + e, so each lane
// loads 8 contiguous bytes per operand and owns a bf16 column pair of two
// tokens.  H = hi + lo in bf16 (two MMAs, fp32 accumulate); then
// y = bf16_rne(y + scal * D) on the live rows.
LORA_DEV void expand_mma(const BgmvParams& p, const BgmvLayout& L, const Smem& sm, int w,
                         int rank, float scal, int n, uint32_t rowmask, int j0, int j1) {
  constexpr int kMT = 3;              // 16-column tiles per warp per pass
  constexpr int kNT = kTT / 8;        // 8-token tiles
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int out = p.out;
  const int R = p.R;
  const int mtiles = ceil_div_i(j1 - j0, 16);
  const int ksteps = ceil_div_i(rank, 16);
  const int ntn = ceil_div_i(n, 8);
  uint32_t* y32 = reinterpret_cast<uint32_t*>(p.y);
  const uint16_t* bb = reinterpret_cast<const uint16_t*>(p.b) + (size_t)w * out * R;
  // rows (tokens) 2c and 2c+1 of every token tile
  size_t yoff[kNT][2];
  bool yok[kNT][2];
#pragma unroll
  for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int t = nt * 8 + 2 * c + e;
      yok[nt][e] = t < n && ((rowmask >> t) & 1u);
      yoff[nt][e] = yok[nt][e] ? (size_t)sm.tok[t] * out : 0;
    }

  for (int base = warp; base < mtiles; base += kMT * (kBgmvThreads / 32)) {
    uint2 bl[kMT], bh[kMT];                 // columns 2g and 2g+1, ranks 4c..4c+3 (k-step 0)
    uint32_t yv[kMT][kNT][2];
#pragma unroll
    for (int q = 0; q < kMT; ++q) {
      const int mt = base + q * (kBgmvThreads / 32);
      bl[q] = bh[q] = make_uint2(0u, 0u);
      const int j = j0 + mt * 16 + 2 * g;   // this lane's column pair
      const bool col_ok = mt < mtiles && j < j1;
      if (col_ok && 4 * c < R) {
        const uint16_t* brow = bb + (size_t)j * R + 4 * c;
        bl[q] = *reinterpret_cast<const uint2*>(brow);
        bh[q] = *reinterpret_cast<const uint2*>(brow + R);
      }
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          yv[q][nt][e] = (col_ok && nt < ntn && yok[nt][e]) ? y32[(yoff[nt][e] + j) >> 1] : 0u;
    }
#pragma unroll
    for (int q = 0; q < kMT; ++q) {
      const int mt = base + q * (kBgmvThreads / 32);
      if (mt >= mtiles) continue;
      const int j = j0 + mt * 16 + 2 * g;
      const bool col_ok = j < j1;
      // A 16-column tile holds at most two slices (slice edges are multiples
      // of 8): one pass per slice, each lane keeping the pass of its column.
      const int jt = j0 + mt * 16;
      const int jl = min(jt + 15, j1 - 1);
      int ia = 0;
      while (ia + 1 < p.S && p.slice_off[ia + 1] <= jt) ++ia;
      int ib = ia;
      while (ib + 1 < p.S && p.slice_off[ib + 1] <= jl) ++ib;
      const int my_i = (ib != ia && j >= p.slice_off[ib]) ? ib : ia;
      float acc[kNT][4];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[nt][k] = 0.f;
      for (int i = ia; i <= ib; ++i) {
        float part[kNT][4];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
          for (int k = 0; k < 4; ++k) part[nt][k] = 0.f;
        for (int ks = 0; ks < ksteps; ++ks) {
          uint2 b0 = bl[q], b1 = bh[q];
          const int k0 = ks * 16 + 4 * c;
          if (ks > 0) {
            b0 = b1 = make_uint2(0u, 0u);
            if (col_ok && k0 < R) {
              const uint16_t* brow = bb + (size_t)j * R + k0;
              b0 = *reinterpret_cast<const uint2*>(brow);
              b1 = *reinterpret_cast<const uint2*>(brow + R);
            }
          }
          b0 = mask_rank4(b0, k0, rank);
          b1 = mask_rank4(b1, k0, rank);
          const int hrow = i * kTT;
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt) {
            if (nt < ntn) {
              const int ho = (hrow + nt * 8 + g) * L.hst + k0;
              const uint2 hh = *reinterpret_cast<const uint2*>(sm.hhi + ho);
              const uint2 hl = *reinterpret_cast<const uint2*>(sm.hlo + ho);
              mma_bf16_16816(part[nt], b0.x, b1.x, b0.y, b1.y, hh.x, hh.y);
              mma_bf16_16816(part[nt], b0.x, b1.x, b0.y, b1.y, hl.x, hl.y);
            }
          }
        }
        if (i == my_i) {
#pragma unroll
          for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[nt][k] = part[nt][k];
        }
      }
      if (col_ok) {
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
          if (nt < ntn) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              if (yok[nt][e]) {
                const uint32_t yo = yv[q][nt][e];
                y32[(yoff[nt][e] + j) >> 1] =
                    pack_bf16x2(fmaf(scal, acc[nt][e], bf16_lo(yo)),
                                fmaf(scal, acc[nt][2 + e], bf16_hi(yo)));
              }
            }
          }
        }
      }
    }
  }
}

// The expand operands of one item, staged in the ring once the shrink no
// longer needs it: this CTA's B columns [j0, j1) of adapter w as stored
// ([cols][R] bf16) at the ring's start, then the y row of every live token of
// the item over the same columns (row stride ystride bytes).
struct ExStage {
  uint8_t* bs;
  uint8_t* ys;
  int ystride;
};

LORA_DEV ExStage ex_stage_carve(const Smem& sm, const BgmvParams& p) {
  const int oc = bgmv_ochunk(p.out);
  ExStage X;
  X.bs = sm.ring;
  X.ys = sm.ring + round_up_i(oc * p.R * 2, 128);
  X.ystride = oc * 2 + 16;
  return X;
}

// Warp 0 issues the bulk copies of the staged operands of adapter w for the
// live rows of the item; their bytes complete on bar.  Every address and size
// is a multiple of 16 bytes: out, R and the slice edges are multiples of 8 and
// j0 a multiple of 16.
LORA_DEV void stage_expand(const BgmvParams& p, const Smem& sm, const ExStage& X, int w, int n,
                           uint32_t rowmask, uint32_t crank, uint64_t* bar) {
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const int oc = bgmv_ochunk(p.out);
  const int j0 = min(p.out, (int)crank * oc);
  const int cols = min(p.out, j0 + oc) - j0;
  const uint32_t live = (n >= 32 ? 0xffffffffu : ((1u << n) - 1u)) & rowmask;
  const bool any = cols > 0 && live != 0u;
  const uint32_t bbytes = (uint32_t)(cols * p.R * 2);
  const uint32_t rbytes = (uint32_t)(cols * 2);
  if (lane == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, any ? bbytes + (uint32_t)__popc(live) * rbytes : 0u);
  }
  __syncwarp();
  if (!any) return;
  if (lane == 0)
    bulk_g2s(X.bs, reinterpret_cast<const uint16_t*>(p.b) + ((size_t)w * p.out + j0) * p.R,
             bbytes, bar);
  if ((live >> lane) & 1u)
    bulk_g2s(X.ys + lane * X.ystride,
             reinterpret_cast<const uint16_t*>(p.y) + (size_t)sm.tok[lane] * p.out + j0, rbytes,
             bar);
}

// L2 prefetch of what stage_expand will copy (issued when the item starts, so
// the copies after the shrink find their bytes in L2).
LORA_DEV void prefetch_expand(const BgmvParams& p, const Smem& sm, int w, int n, uint32_t rowmask,
                              uint32_t crank) {
  const int lane = threadIdx.x & 31;
  const int oc = bgmv_ochunk(p.out);
  const int j0 = min(p.out, (int)crank * oc);
  const int cols = min(p.out, j0 + oc) - j0;
  const uint32_t live = (n >= 32 ? 0xffffffffu : ((1u << n) - 1u)) & rowmask;
  if (cols <= 0 || live == 0u) return;
  if (lane == 0)
    bulk_prefetch_l2(reinterpret_cast<const uint16_t*>(p.b) + ((size_t)w * p.out + j0) * p.R,
                     (uint32_t)(cols * p.R * 2));
  if ((live >> lane) & 1u)
    bulk_prefetch_l2(reinterpret_cast<const uint16_t*>(p.y) + (size_t)sm.tok[lane] * p.out + j0,
                     (uint32_t)(cols * 2));
}

// Expand of a staged item with the m16n8k16 MMAs of expand_mma (same operands,
// same order, so the same results): D[16 columns, 8 tokens] = B H^T per 16-column
// tile of one slice, H = hi + lo.  B comes from the staged copy and y = bf16_rne(
// y + scal * D) is written in place into the staged y rows (write_back_staged
// stores them).  A 16-column tile may reach past the end of its slice (slice
// edges are multiples of 8); those lanes are masked and the next slice
// computes their columns.
LORA_DEV void expand_staged(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                            const ExStage& X, int rank, float scal, int n, uint32_t rowmask,
                            int j0, int j1) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane >> 2;
  const int c = lane & 3;
  const int ksteps = ceil_div_i(rank, 16);
  const int ntn = ceil_div_i(n, 8);
  const bool one = ksteps <= 1;
  const uint16_t* bs = reinterpret_cast<const uint16_t*>(X.bs);
  // live y rows of the item; this lane updates tokens 2c + e of each tile,
  // whose rows start at (8 nt + 2c + e) * ystride in the staged copy
  const uint32_t live = (n >= 32 ? 0xffffffffu : ((1u << n) - 1u)) & rowmask;
  uint8_t* ylane = X.ys + 2 * c * X.ystride;
  const uint2 m0 = rank_mask4(4 * c, rank);

#pragma unroll 1
  for (int i = 0; i < p.S; ++i) {
    const int ls0 = max(j0, p.slice_off[i]) - j0;
    const int ls1 = min(j1, p.slice_off[i + 1]) - j0;
    if (ls0 >= ls1) continue;
#pragma unroll 1
    for (int nt = 0; nt < ntn; ++nt) {
      const int hrow = (i * kTT + nt * 8 + g) * L.hst;
      uint2 hh = make_uint2(0u, 0u), hl = make_uint2(0u, 0u);
      if (one) {
        hh = *reinterpret_cast<const uint2*>(sm.hhi + hrow + 4 * c);
        hl = *reinterpret_cast<const uint2*>(sm.hlo + hrow + 4 * c);
      }
      const uint32_t lv = live >> (nt * 8 + 2 * c);
      uint8_t* yt = ylane + nt * 8 * X.ystride;
#pragma unroll 1
      for (int jt = ls0 + warp * 16; jt < ls1; jt += kExGroup * (kBgmvThreads / 2)) {
        if (one)
          expand_step<true>(bs, sm.hhi, sm.hlo, yt, X.ystride, p.R, hrow, ksteps, rank, m0, hh,
                            hl, jt, ls1, g, c, lv, scal);
        else
          expand_step<false>(bs, sm.hhi, sm.hlo, yt, X.ystride, p.R, hrow, ksteps, rank, m0, hh,
                             hl, jt, ls1, g, c, lv, scal);
      }
    }
  }
}

// Stores the updated staged y rows of the live tokens: warp w copies rows
// w, w + 8, ... with 16-byte loads and stores (a warp instruction moves 512
// contiguous bytes of a row).  Every thread must call it after its
// expand_staged.
LORA_DEV void write_back_staged(const BgmvParams& p, const Smem& sm, const ExStage& X, int n,
                                uint32_t rowmask, int j0, int j1) {
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int cpr = (j1 - j0) >> 3;   // 16-byte chunks per row
  const uint32_t live = (n >= 32 ? 0xffffffffu : ((1u << n) - 1u)) & rowmask;
  for (int t = warp; t < n; t += kBgmvThreads / 32) {
    if (!((live >> t) & 1u)) continue;
    const uint4* src = reinterpret_cast<const uint4*>(X.ys + t * X.ystride);
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.y) +
                                          (size_t)sm.tok[t] * p.out + j0);
    for (int ch = lane; ch < cpr; ch += 32) dst[ch] = src[ch];
  }
}

// Expand of one MoE group on one CTA over every output column, in chunks of
// p.ex_cw columns: the pair's B rows and the group's y rows over a chunk are
// staged through the (idle) ring by 16-byte cp.async copies, then updated by
// expand_staged and written back.  Every thread must call it.
LORA_DEV void expand_chunked(const BgmvParams& p, const BgmvLayout& L, const Smem& sm, int w,
                             int rank, float scal, int n, uint32_t rowmask) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int cw = p.ex_cw;
  ExStage X;
  X.bs = sm.ring;
  X.ys = sm.ring + round_up_i(cw * p.R * 2, 128);
  X.ystride = cw * 2 + 16;
  const uint32_t live = (n >= 32 ? 0xffffffffu : ((1u << n) - 1u)) & rowmask;
  const uint16_t* bg = reinterpret_cast<const uint16_t*>(p.b) + (size_t)w * p.out * p.R;
  const uint16_t* yg = reinterpret_cast<const uint16_t*>(p.y);
  for (int j0 = 0; j0 < p.out; j0 += cw) {
    const int j1 = min(p.out, j0 + cw);
    const int bchunks = (j1 - j0) * p.R / 8;   // B rows [j0, j1) are contiguous
    for (int i = threadIdx.x; i < bchunks; i += kBgmvThreads)
      cp_async16(smem_u32(X.bs) + i * 16, bg + (size_t)j0 * p.R + i * 8);
    const int ypr = (j1 - j0) / 8;             // 16-byte chunks of a y row
    for (int t = warp; t < n; t += kBgmvThreads / 32) {
      if (!((live >> t) & 1u)) continue;
      const uint16_t* src = yg + (size_t)sm.tok[t] * p.out + j0;
      const uint32_t dst = smem_u32(X.ys + t * X.ystride);
      for (int c = lane; c < ypr; c += 32) cp_async16(dst + c * 16, src + c * 8);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    expand_staged(p, L, sm, X, rank, scal, n, rowmask, j0, j1);
    write_back_staged(p, sm, X, n, rowmask, j0, j1);
    __syncthreads();   // the ring is refilled for the next chunk
  }
}

// Waits (bounded, warp-uniform) for the staged expand operands.
LORA_DEV bool wait_staged(uint64_t* bar, uint32_t parity) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Expand of a staged item.  If the copies do not land within the wait limit
// the warp raises LORA_FLAG_TIMEOUT, skips its columns and waits once more
// (bounded) so that no copy is still writing the ring when it is reused; the
// rows are then not stored.  Every thread of the CTA must call it.
LORA_DEV void expand_after_stage(const BgmvParams& p, const BgmvLayout& L, const Smem& sm,
                                 const ExStage& X, uint64_t* bar, uint32_t parity, int rank,
                                 float scal, int n, uint32_t rowmask, uint32_t crank) {
  const int oc = bgmv_ochunk(p.out);
  const int j0 = min(p.out, (int)crank * oc);
  const int j1 = min(p.out, j0 + oc);
  const bool ok = wait_staged(bar, parity);
  if (ok) {
    expand_staged(p, L, sm, X, rank, scal, n, rowmask, j0, j1);
  } else {
    if ((threadIdx.x & 31) == 0) raise_flag(p.flags, LORA_FLAG_TIMEOUT);
    wait_staged(bar, parity);
  }
  // the rows are stored only when every warp saw its copies land
  if (__syncthreads_or(ok ? 0 : 1) == 0) {
    write_back_staged(p, sm, X, n, rowmask, j0, j1);
  }
}

// k-th work item of group g of ng.  Linear targets: passes over the groups
// alternate in direction, so the groups that drew the first (in slot order,
// under a skewed slot load the largest) items of a pass draw the last of the
// next one.  MoE chunks: round robin (measured better there).
LORA_DEV int item_of(bool snake, int k, int g, int ng) {
  return k * ng + ((snake && (k & 1)) ? (ng - 1 - g) : g);
}

}  // namespace

template <int MODE>
__global__ void __launch_bounds__(kBgmvThreads, 2) bgmv_kernel(const BgmvParams p) {
  constexpr bool kClustered = (MODE == kModeFused || MODE == kModeShrink);
  constexpr bool kSolo = (MODE == kModeExpertSolo);
  constexpr bool kMoE = kSolo;
  constexpr bool kScaled = (MODE == kModeFused || MODE == kModeExpand || MODE == kModeEmbed || kMoE);
  constexpr bool kExpands = kScaled;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  // With a programmatic launch edge (fused mode only) the next kernel may
  // start its CTAs as ours finish, and ours read x and y only after the
  // preceding kernel completed (grid_dep_wait below); without one both are
  // no-ops.
  if (MODE == kModeFused) grid_dep_launch_dependents();
  const int npref = kMoE ? p.num_experts : p.slots;
  const BgmvLayout L = bgmv_layout(MODE, npref, p.S, p.R, p.kb, p.nst,
                                   p.ex_stage ? bgmv_ex_stage_bytes(p.out, p.R) : 0);
  const Smem sm = carve(smem_raw, L);
  const int tid = threadIdx.x;
  // Staged expand: B and y of an item are bulk-copied into the idle ring while
  // the cluster reduces h; ebar counts their bytes (one phase per use).
  const bool staged = kExpands && kClustered && p.ex_stage != 0;
  uint64_t* ebar = reinterpret_cast<uint64_t*>(smem_raw);
  const ExStage X = ex_stage_carve(sm, p);
  uint32_t ephase = 0;
  // Shrink stage copies: bulk copies complete on the ring slots' barriers.
  StageCopies sc;
  sc.bulk = p.bulk_stage != 0;
  sc.sbar = ebar + 1;
  sc.sph = 0;
  if (tid == 0 && (staged || sc.bulk)) {
    mbar_init(ebar, 1);
    mbar_init(&sc.sbar[0], 1);
    mbar_init(&sc.sbar[1], 1);
    fence_mbar_init();
  }

  uint32_t crank, group, ngroups;
  if (kClustered) {
    crank = cluster_ctarank();
    group = cluster_id_x();
    ngroups = num_clusters_x();
  } else if (kSolo) {
    crank = 0;
    group = blockIdx.x;
    ngroups = gridDim.x;
  } else {
    crank = blockIdx.x % kGroup;
    group = blockIdx.x / kGroup;
    ngroups = gridDim.x / kGroup;
  }

  // token_order of the first kTokCache positions, loaded while the planner's
  // reads are in flight and kept in shared memory (the expert mode uses that
  // region for its sub-batches instead).
  constexpr int kTokCache = kTT * kTT;
  constexpr int kTokPerThread = kTokCache / kBgmvThreads;
  const int tokc_n = kMoE ? 0 : min(p.T, kTokCache);
  int tv[kTokPerThread];
#pragma unroll
  for (int q = 0; q < kTokPerThread; ++q) {
    const int i = tid + q * kBgmvThreads;
    tv[q] = i < tokc_n ? p.token_order[i] : -1;
  }

  const bool report = (blockIdx.x == 0);
  int total;
  if (kMoE) {
    total = plan_expert<kBgmvThreads>(p.expert_offsets, p.pair_index, p.num_experts, p.slots, p.T,
                                      kTT, sm.prefix, sm.scratch, p.flags, report);
  } else {
    total = plan_linear<kBgmvThreads>(p.slot_indptr, p.ranks, kScaled ? p.scalings : nullptr,
                                      p.slots, p.T, p.R, p.tile, sm.prefix, sm.scratch, p.flags,
                                      report);
  }
#pragma unroll
  for (int q = 0; q < kTokPerThread; ++q) {
    const int i = tid + q * kBgmvThreads;
    if (i < tokc_n) sm.sub_rows[i] = tv[q];
  }
  if (!kMoE) {
    // Addressing of this CTA's first kItemCache items, written by the thread
    // of their slot (its planner reads are still in L1), so that an item
    // starts without a dependent global load.
    for (int sl = tid; sl < p.slots; sl += kBgmvThreads) {
      const int i0 = sm.prefix[sl], i1 = sm.prefix[sl + 1];
      if (i1 <= i0) continue;
      for (int k = 0; k < kItemCache; ++k) {
        const int item = item_of(true, k, (int)group, (int)ngroups);
        if (item < i0 || item >= i1 || item >= total) continue;
        const int p0 = p.slot_indptr[sl] + (item - i0) * p.tile;
        sm.sub_s[k] = sl;
        sm.sub_s[kItemCache + k] = p.ranks[sl];
        sm.sub_p[k] = p0;
        sm.sub_p[kItemCache + k] = kScaled ? __float_as_int(p.scalings[sl]) : 0;
        sm.sub_cnt[k] = max(0, min(p.tile, p.slot_indptr[sl + 1] - p0));
      }
    }
  }
  if (kClustered) {
    // Trip counts of loops holding a cluster barrier come from rank 0, so every
    // CTA of a cluster takes the same barriers.
    if (tid == 0) sm.ctrl[0] = total;
    cluster_sync();
    total = dsmem_ld_s32(dsmem_addr(&sm.ctrl[0], 0));
  } else {
    __syncthreads();
  }

  int hpar = 0;
  int iter = 0;
  for (int item = (int)group; item < total;
       ++iter, item = item_of(!kMoE, iter, (int)group, (int)ngroups)) {
    if (!kMoE) {
      // ---- linear / embedding item: (slot, tile of kTT positions) ----
      int s, p0, n, rank;
      float scal;
      if (iter < kItemCache) {
        s = sm.sub_s[iter];
        rank = sm.sub_s[kItemCache + iter];
        p0 = sm.sub_p[iter];
        scal = __int_as_float(sm.sub_p[kItemCache + iter]);
        n = sm.sub_cnt[iter];
      } else {
        s = find_segment(sm.prefix, p.slots, item);
        p0 = p.slot_indptr[s] + (item - sm.prefix[s]) * p.tile;
        n = max(0, min(p.tile, p.slot_indptr[s + 1] - p0));
        rank = p.ranks[s];
        scal = kScaled ? p.scalings[s] : 0.f;
      }
      const bool emb = (MODE == kModeEmbed || MODE == kModeGather);
      int t = -1;
      if (tid < n && p0 + tid >= 0 && p0 + tid < p.T)
        t = (p0 + tid < tokc_n) ? sm.sub_rows[p0 + tid] : p.token_order[p0 + tid];
      ShrinkGeom G = {};
      if (kClustered) {
        // the A rows do not depend on the tokens: start them while the reads land
        G = shrink_geom(p, rank, crank);
        if (G.nkb > 0) issue_stage(p, L, sm, G, s, rank, 0, 0, 0, kRowsA, sc);
      }
      if (MODE == kModeFused && iter == 0) grid_dep_wait();   // x and y from here on
      if (tid < kTT) {
        int id = -1;
        if (tid < n && p0 + tid >= 0 && p0 + tid < p.T) {
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
        const uint32_t tm = __ballot_sync(0xffffffffu, t >= 0);
        const uint32_t im = __ballot_sync(0xffffffffu, id >= 0);
        if (tid == 0) {
          sm.ctrl[4 + 2 * (iter & 1)] = tm;
          sm.ctrl[5 + 2 * (iter & 1)] = im;
        }
      }
      __syncthreads();
      const uint32_t tokmask = (uint32_t)sm.ctrl[4 + 2 * (iter & 1)];
      const uint32_t idmask = (uint32_t)sm.ctrl[5 + 2 * (iter & 1)];
      const uint32_t rowmask = emb ? (tokmask & idmask) : tokmask;
      if (staged && (tid >> 5) == 1) prefetch_expand(p, sm, s, n, rowmask, crank);
      if (kClustered) {
        float* hp = sm.hpart + (size_t)hpar * kTT * L.srp;
        shrink_partial(p, L, sm, G, s, rank, n, hp, sc);
        if (staged) stage_expand(p, sm, X, s, n, rowmask, crank, ebar);
        cluster_sync();
        produce_h<kFromCluster>(p, L, sm, hp, s, rank, n, rowmask, kExpands,
                                MODE == kModeShrink, crank);
        hpar ^= 1;
      } else if (MODE == kModeExpand) {
        produce_h<kFromGlobal>(p, L, sm, nullptr, s, rank, n, rowmask, true, false, crank);
      } else {
        produce_h<kFromGather>(p, L, sm, nullptr, s, rank, n, rowmask, kExpands,
                               MODE == kModeGather, crank);
      }
      __syncthreads();
      if (kExpands) {
        if (staged) {
          expand_after_stage(p, L, sm, X, ebar, ephase, rank, scal, n, rowmask, crank);
          ephase ^= 1u;
        } else {
          const int oc = bgmv_ochunk(p.out);
          const int j0 = min(p.out, (int)crank * oc);
          expand_mma(p, L, sm, s, rank, scal, n, rowmask, j0, min(p.out, j0 + oc));
        }
      }
      __syncthreads();
    } else {
      // ---- MoE item (one CTA): chunk of one expert's rows, split by slot ----
      const int E = p.num_experts;
      const int e = find_segment(sm.prefix, E, item);
      const int chunk = item - sm.prefix[e];
      const int start = p.expert_offsets[e] + chunk * kTT;
      const int m = max(0, min(kTT, p.expert_offsets[e + 1] - start));
      int* nsub_slot = &sm.ctrl[2 + (iter & 1)];
      if (tid < kTT) {
        // lane q classifies row start + q (the fold's skip rules) ...
        const int q = tid;
        uint32_t bad = 0;
        int rs = 0x7fffffff, rp = -1;
        const int rho = start + q;
        if (q < m && rho >= 0 && rho < p.T) {
          const int sl = p.row_slot[rho];
          if (sl < -1 || sl >= p.slots) {
            bad = LORA_FLAG_BAD_SLOT;
          } else if (sl != -1) {
            const int pi = p.pair_index[(size_t)sl * E + e];
            if (pi != -1) {
              if (pi < -1 || pi >= p.num_pairs) {
                bad = LORA_FLAG_BAD_PAIR;
              } else {
                const int r = p.ranks[sl];
                if (r < 0 || r > p.R) {
                  bad = LORA_FLAG_BAD_RANK;
                } else if (r != 0 && p.scalings[sl] != 0.0f) {
                  rs = sl;
                  rp = pi;
                }
              }
            }
          }
        }
        // ... and the warp forms the sub-batches: ascending slot order, rows in
        // row order
        const uint32_t lt = (1u << q) - 1u;
        int nsub = 0;
        for (int last = -1;;) {
          const int best = (int)__reduce_min_sync(0xffffffffu, (unsigned)(rs > last ? rs : 0x7fffffff));
          if (best == 0x7fffffff) break;
          const uint32_t mk = __ballot_sync(0xffffffffu, rs == best);
          if (rs == best) {
            sm.sub_rows[nsub * kTT + __popc(mk & lt)] = rho;
            if ((mk & lt) == 0u) {
              sm.sub_p[nsub] = rp;
              sm.sub_s[nsub] = best;
              sm.sub_cnt[nsub] = __popc(mk);
            }
          }
          ++nsub;
          last = best;
        }
        bad = __reduce_or_sync(0xffffffffu, bad);
        if (q == 0) {
          *nsub_slot = nsub;
          if (crank == 0) raise_flag(p.flags, bad);
        }
      }
      __syncthreads();
      const int nsub = *nsub_slot;
      for (int q = 0; q < nsub; ++q) {
        const int sl = sm.sub_s[q];
        const int w = sm.sub_p[q];
        const int n = sm.sub_cnt[q];
        const int rank = p.ranks[sl];
        const float scal = p.scalings[sl];
        const ShrinkGeom G = shrink_geom(p, rank, 0u);
        if (G.nkb > 0 && rank > 0) issue_stage(p, L, sm, G, w, rank, 0, 0, 0, kRowsA, sc);
        if (tid < kTT) sm.tok[tid] = (tid < n) ? sm.sub_rows[q * kTT + tid] : -1;
        __syncthreads();
        const uint32_t mask = (n >= 32) ? 0xffffffffu : ((1u << n) - 1u);
        float* hp = sm.hpart + (size_t)hpar * kTT * L.srp;
        shrink_partial(p, L, sm, G, w, rank, n, hp, sc);
        __syncthreads();
        produce_h<kFromLocal>(p, L, sm, hp, w, rank, n, mask, true, false, 0);
        hpar ^= 1;
        __syncthreads();
        if (p.ex_cw > 0)
          expand_chunked(p, L, sm, w, rank, scal, n, mask);
        else
          expand_mma(p, L, sm, w, rank, scal, n, mask, 0, p.out);
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

std::atomic<int> g_overlap{0};

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
cudaError_t launch_mode(const BgmvParams& p_in, int max_items, cudaStream_t stream,
                        const char** why) {
  BgmvParams p = p_in;
  p.tile = MODE == kModeFused ? kFusedTile : kTT;
  constexpr bool kClustered = (MODE == kModeFused || MODE == kModeShrink);
  constexpr bool kSolo = (MODE == kModeExpertSolo);
  p.kchunk = kSolo ? p.in : bgmv_kchunk(p.in);
  bgmv_pick_stages(p.kchunk, p.S, p.R, kSolo ? kSoloRingBudget : kRingBudget, &p.kb, &p.nst);
  const int npref = kSolo ? p.num_experts : p.slots;
  const BgmvLayout L0 = bgmv_layout(MODE, npref, p.S, p.R, p.kb, p.nst, 0);
  const int ex_bytes = bgmv_ex_stage_bytes(p.out, p.R);
  p.ex_stage = (MODE == kModeFused &&
                ex_bytes <= max(p.nst * L0.stage_bytes, kExStageMax))
                   ? 1
                   : 0;
  const BgmvLayout L = bgmv_layout(MODE, npref, p.S, p.R, p.kb, p.nst, p.ex_stage ? ex_bytes : 0);
  // MoE fold: widest column chunk (a multiple of 64, at most 512) whose B rows
  // and kTT y rows fit the ring, or 0 (expand straight from global memory)
  p.ex_cw = 0;
  if (kSolo) {
    const int ring = p.nst * L.stage_bytes;
    for (int cw = 512; cw >= 64 && p.ex_cw == 0; cw -= 64)
      if (round_up_i(cw * p.R * 2, 128) + kTT * (cw * 2 + 16) <= ring) p.ex_cw = cw;
  }
  // Wide stage rows (1 KB) go as one bulk copy each; narrower ones as 16-byte
  // cp.async copies, which land sooner for small rounds.
  p.bulk_stage = (p.kb >= 512 && (kClustered || kSolo)) ? 1 : 0;
  auto kern = bgmv_kernel<MODE>;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;

  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
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
  if (MODE == kModeFused && g_overlap.load(std::memory_order_relaxed) != 0) {
    attr[cfg.numAttrs].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[cfg.numAttrs].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs += 1;
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
      groups = kSolo ? per_sm * sms : max(1, per_sm * sms / kGroup);
    }
    std::lock_guard<std::mutex> lk(g_cache_mu);
    if (g_cache_n < 64) g_cache[g_cache_n++] = {dev, MODE, L.total, groups};
  }
  groups = max(1, min(groups, max_items));
  cfg.gridDim = dim3((unsigned)(kSolo ? groups : groups * kGroup), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

int bgmv_set_overlap(int enable) { return g_overlap.exchange(enable != 0 ? 1 : 0); }
bool launch_overlap_enabled() { return g_overlap.load(std::memory_order_relaxed) != 0; }

cudaError_t bgmv_launch(int mode, const BgmvParams& p, int max_items, cudaStream_t stream,
                        const char** why) {
  switch (mode) {
    case kModeFused: return launch_mode<kModeFused>(p, max_items, stream, why);
    case kModeShrink: return launch_mode<kModeShrink>(p, max_items, stream, why);
    case kModeExpand: return launch_mode<kModeExpand>(p, max_items, stream, why);
    case kModeEmbed: return launch_mode<kModeEmbed>(p, max_items, stream, why);
    case kModeGather: return launch_mode<kModeGather>(p, max_items, stream, why);
    case kModeExpertSolo: return launch_mode<kModeExpertSolo>(p, max_items, stream, why);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace lora
