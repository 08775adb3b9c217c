// SGMV regime of the LoRA delta path (many tokens per slot): tcgen05 MMAs
// with TMEM accumulators over 128-token tiles of one slot's segment.
//
// Shrink  D[128 tokens, S*K0] = X[128, in] A_s^T: x rows gathered by 16-byte
//         cp.async into 128-byte-swizzled K-major tiles, the slot's live A rows
//         by tensor TMA, both through a 4-stage ring; fp32 h to global (one
//         buffer per split of the input features).
// Expand  D[128 tokens, 128 columns] = H B_s^T with H = hi + lo in bf16 (two
//         MMAs, fp32 accumulate) built once per (tile, slice) in shared memory;
//         B tiles by tensor TMA; y rows prefetched by cp.async into shared
//         memory, updated with bf16_rne(y + scaling * D) and stored with
//         coalesced row writes.
// Both kernels are persistent (one CTA per SM over a contiguous run of work
// units) and warp-specialised: warp 1 issues MMAs (one thread); the shrink
// copies x with 4 warps (0 and 6-8, warp 0 also starts the A tiles) and
// drains TMEM with 4; the expand loads B with warp 0 and drains TMEM with 16
// (each 32 rows x 32 columns).  Every wait is bounded; on timeout the CTA raises
// LORA_FLAG_TIMEOUT, stops, frees its TMEM and exits.
//
// Sources: mstar.engine.resources.lora.backend (LoraBackend.shrink,
// expand_fused, apply_linear_, apply_ with embedding=True, gather_shrink).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "sgmv.h"
#include "tcgen05.cuh"

namespace lora {

namespace {

constexpr int kSgXWarps = 4;      // shrink: warps that copy x rows (warp 0 and warps 6..8)
constexpr int kSgThreads = 32 * (6 + kSgXWarps - 1);   // shrink: 9 warps
constexpr int kExEpiWarps = 16;   // expand epilogue: 4 TMEM lane quarters x 4 column groups
constexpr int kExThreads = 32 * (2 + kExEpiWarps);   // expand: producer, MMA, epilogue
constexpr int kNY = 3;            // y staging buffers (prefetch two units ahead)
constexpr int kTM = kSgmvTileM;   // 128 tokens per tile (MMA M)
constexpr int kBN = 128;          // output columns per expand unit (MMA N)
constexpr int kNB = 4;            // B ring stages (expand)
constexpr int kNS = 4;            // x/A ring stages (shrink)
constexpr int kKBLK = 64;         // input features per shrink stage (128 bytes)
constexpr int kYRow = kBN * 2 + 16;  // staged y row pitch in bytes

struct ExpandParams {
  void* y;
  const float* h;            // [ksplit][T][S*R] (linear) or nullptr (embedding)
  size_t h_split;            // elements between the ksplit partial buffers
  int ksplit;
  const int* ids;            // embedding ids [T]
  const void* a;             // embedding A [slots, S*R, vocab]
  const int* ranks;
  const float* scalings;
  const int* token_order;
  const int* slot_indptr;
  const int* seg_hi;         // grouped addressing: segment ends, or nullptr
  const int* slot_map;       // grouped addressing: a/b pair of each group, or nullptr
  uint32_t* flags;
  int T, vocab, slots, R, S, out;
  int span;                  // bytes per K-major row: 2*R (32, 64 or 128)
  int nchunk;                // sum over slices of ceil(out_i / kBN)
  int slice_off[LORA_MAX_SLICES + 1];
  int chunk_off[LORA_MAX_SLICES + 1];
};

struct ShrinkParams {
  const void* x;
  float* h;                  // [ksplit][T][S*R]
  size_t h_split;
  int ksplit;
  int kb_per_split;          // stages of kKBLK features per split
  const int* ranks;
  const float* scalings;     // nullptr: unscaled plan
  const int* token_order;
  const int* slot_indptr;
  const int* seg_hi;         // grouped addressing: segment ends, or nullptr
  const int* slot_map;       // grouped addressing: a/b pair of each group, or nullptr
  uint32_t* flags;
  int T, in, slots, R, S;
};

// Wait that also gives up when another role of the CTA aborted.
LORA_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                            uint32_t* flags) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      raise_flag(flags, LORA_FLAG_TIMEOUT);
      return false;
    }
  }
  return true;
}

// The same wait for a whole warp: lane 0 polls, every lane gets its verdict,
// so the warp never diverges around the .sync.aligned operations that follow.
LORA_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                        uint32_t* flags) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_or_abort(bar, parity, abort_flag, flags) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

LORA_DEV uint32_t align1024(uint32_t v) { return (v + 1023u) & ~1023u; }

// End of slot (or group) s's segment, and the a/b pair it uses.
LORA_DEV int seg_end(const int* indptr, const int* seg_hi, int s) {
  return seg_hi != nullptr ? seg_hi[s] : indptr[s + 1];
}
LORA_DEV int ab_of(const int* slot_map, int s) { return slot_map != nullptr ? slot_map[s] : s; }

// Walks consecutive expand units without divisions: the item (and its slot
// segment) is decoded only when the column chunks of an item run out.
struct UnitCursor {
  int item, cj, s, p0, n, slice, col0, width;

  LORA_DEV void set_item(const ExpandParams& p, const int* prefix, int it) {
    item = it;
    s = find_segment(prefix, p.slots, it);
    p0 = p.slot_indptr[s] + (it - prefix[s]) * kTM;
    n = max(0, min(kTM, seg_end(p.slot_indptr, p.seg_hi, s) - p0));
  }
  LORA_DEV void set_chunk(const ExpandParams& p) {
    while (slice + 1 < p.S && p.chunk_off[slice + 1] <= cj) ++slice;
    col0 = p.slice_off[slice] + (cj - p.chunk_off[slice]) * kBN;
    width = min(kBN, p.slice_off[slice + 1] - col0);
  }
  LORA_DEV void init(const ExpandParams& p, const int* prefix, long long u) {
    const int it = (int)(u / p.nchunk);
    cj = (int)(u - (long long)it * p.nchunk);
    slice = 0;
    set_item(p, prefix, it);
    set_chunk(p);
  }
  LORA_DEV void advance(const ExpandParams& p, const int* prefix) {
    if (++cj == p.nchunk) {
      cj = 0;
      slice = 0;
      set_item(p, prefix, item + 1);
    }
    set_chunk(p);
  }
};

}  // namespace

// ---------------------------------------------------------------------------
// Expand
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kExThreads, 1)
sgmv_expand_kernel(const __grid_constant__ CUtensorMap tmap_b, const ExpandParams p) {
  extern __shared__ uint8_t sg_smem_raw[];
  // Programmatic launch edge (when the caller opted in): let the next kernel
  // start as CTAs finish; only the epilogue, which reads y, h and ids and
  // writes y, waits for the preceding kernel.  No-ops otherwise.
  grid_dep_launch_dependents();
  const uint32_t raw = smem_u32(sg_smem_raw);
  uint8_t* base = sg_smem_raw + (align1024(raw) - raw);
  uint64_t* bfull = reinterpret_cast<uint64_t*>(base);
  uint64_t* bempty = bfull + kNB;
  uint64_t* accfull = bempty + kNB;
  uint64_t* accempty = accfull + 2;
  uint64_t* hready = accempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + 260);
  int* scratch = reinterpret_cast<int*>(base + 288);
  int* prefix = reinterpret_cast<int*>(base + 1024);
  const uint32_t pre_bytes = align1024((uint32_t)(p.slots + 1) * 4u);
  const uint32_t span = (uint32_t)p.span;
  const uint32_t tile_h = kTM * span;
  const uint32_t tile_b = kBN * span;
  uint8_t* hhi = base + 1024 + pre_bytes;
  uint8_t* hlo = hhi + tile_h;
  uint8_t* bring = hlo + tile_h;
  uint8_t* ystage = bring + kNB * tile_b;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&bfull[i], 1);
      mbar_init(&bempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], kExEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(hready, 32 * kExEpiWarps);   // one arrival per epilogue thread
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kBN);
    tmem_relinquish();
  }
  const int items = plan_linear<kExThreads>(p.slot_indptr, p.ranks, p.scalings, p.slots, p.T,
                                            p.R, kTM, prefix, scratch, p.flags,
                                            blockIdx.x == 0, p.seg_hi);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long units = (long long)items * p.nchunk;
  const long long u0 = units * blockIdx.x / gridDim.x;
  const long long u1 = units * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(u1 - u0);
  const uint32_t idesc = mma_idesc_bf16(kTM, kBN);

  if (warp == 0) {
    // ---------------- producer: B tiles by tensor TMA ----------------
    if (lane == 0) {
      UnitCursor U;
      if (nloc > 0) U.init(p, prefix, u0);
      for (int k = 0; k < nloc && !*abort_flag; ++k, U.advance(p, prefix)) {
        const int st = k % kNB;
        if (k >= kNB &&
            !wait_or_abort(&bempty[st], (uint32_t)((k / kNB - 1) & 1), abort_flag, p.flags))
          break;
        mbar_arrive_expect_tx(&bfull[st], tile_b);
        tma_load_2d(bring + st * tile_b, &tmap_b, 0, ab_of(p.slot_map, U.s) * p.out + U.col0,
                    &bfull[st]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int hcount = 0;
    int prev_item = -1, prev_slice = -1;
    UnitCursor U;
    if (nloc > 0) U.init(p, prefix, u0);
    for (int k = 0; k < nloc; ++k, U.advance(p, prefix)) {
      if (U.item != prev_item || U.slice != prev_slice) {
        if (!warp_wait(hready, (uint32_t)(hcount & 1), abort_flag, p.flags)) break;
        ++hcount;
        prev_item = U.item;
        prev_slice = U.slice;
      }
      const int st = k % kNB;
      if (!warp_wait(&bfull[st], (uint32_t)((k / kNB) & 1), abort_flag, p.flags)) break;
      const int as = k & 1;
      if (k >= 2 && !warp_wait(&accempty[as], (uint32_t)((k / 2 - 1) & 1), abort_flag, p.flags))
        break;
      tc_fence_after();
      const int rank = p.ranks[U.s];
      const int ksteps = ceil_div_i(rank, 16);
      uint8_t* btile = bring + st * tile_b;
      if (rank & 15) {
        // zero B columns [rank, 16*ksteps): they meet zero h columns, but NaN
        // or Inf there would still poison the product
        for (int row = lane; row < kBN; row += 32)
          for (int kk = rank; kk < ksteps * 16; ++kk)
            *reinterpret_cast<uint16_t*>(btile + kmajor_offset(row, kk, span)) = 0;
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (lane == 0) {
        const uint32_t d = tmem_base + (uint32_t)(as * kBN);
        const uint32_t hh = smem_u32(hhi), hl = smem_u32(hlo), bt = smem_u32(btile);
        for (int ks = 0; ks < ksteps; ++ks) {
          const uint64_t bdesc = smem_desc_kmajor(bt + ks * 32, span);
          mma_bf16_ss(d, smem_desc_kmajor(hh + ks * 32, span), bdesc, idesc, ks > 0 ? 1u : 0u);
          mma_bf16_ss(d, smem_desc_kmajor(hl + ks * 32, span), bdesc, idesc, 1u);
        }
        mma_commit(&bempty[st]);
        mma_commit(&accfull[as]);
      }
      __syncwarp();
    }
  } else {
    // ---------------- epilogue: warps 2..17 ----------------
    grid_dep_wait();
    // Warp w reads TMEM lanes 32*(w%4).. (one token row per thread) and owns
    // the 32 columns [32 cg, 32 cg + 32) of the unit, cg = (w - 2) / 4.
    const int quarter = warp & 3;
    const int cg = (warp - 2) >> 2;
    const int m = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const __nv_bfloat16* yb = reinterpret_cast<const __nv_bfloat16*>(p.y);
    uint8_t* ybytes = reinterpret_cast<uint8_t*>(p.y);
    int prev_item = -1, prev_slice = -1;

    auto row_token = [&](const UnitCursor& V) -> int {
      if (m >= V.n) return -1;
      const int t = p.token_order[V.p0 + m];
      return (t >= 0 && t < p.T) ? t : -1;
    };
    // The warp's 32 rows x 32 columns of y, as 16-byte copies: lane l takes
    // chunk l % 4 of row 8j + l / 4, so an instruction moves eight 64-byte row
    // segments.  `t` is this lane's own row token; rows read their token from
    // the lane that owns them.
    auto prefetch_y = [&](const UnitCursor& V, int t, int buf) {
      const int c = cg * 4 + (lane & 3);
      const bool cok = c < (V.width >> 3);
      const uint32_t base_s = smem_u32(ystage) + (uint32_t)(buf * kTM + quarter * 32) * kYRow;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = 8 * j + (lane >> 2);
        const int tr = __shfl_sync(0xffffffffu, t, r);
        if (tr >= 0 && cok)
          cp_async16(base_s + (uint32_t)r * kYRow + c * 16, yb + (size_t)tr * p.out + V.col0 + c * 8);
      }
      cp_async_commit();
    };

    // cursors of units k, k+1, k+2 (y of the last two is in flight)
    UnitCursor U, U1, U2;
    int tok = -1, t1 = -1, t2 = -1;
    if (nloc > 0) {
      U.init(p, prefix, u0);
      tok = row_token(U);
      prefetch_y(U, tok, 0);
      U1 = U;
      U1.advance(p, prefix);
    } else {
      cp_async_commit();
    }
    if (nloc > 1) {
      t1 = (U1.item == U.item) ? tok : row_token(U1);
      prefetch_y(U1, t1, 1);
      U2 = U1;
      U2.advance(p, prefix);
    } else {
      cp_async_commit();
    }
    // per item: the slot's rank and scaling, this row's validity and id
    int rank = 0;
    float scal = 0.f;
    bool row_ok = false;
    int id = -1;
    for (int k = 0; k < nloc; ++k) {
      // keep two units of y in flight
      if (k + 2 < nloc) {
        t2 = (U2.item == U1.item) ? t1 : row_token(U2);
        prefetch_y(U2, t2, (k + 2) % kNY);
      } else {
        cp_async_commit();
      }
      const bool new_item = U.item != prev_item;
      if (new_item) {
        if (cg == 0 && m < U.n && tok < 0 && U.col0 == 0) raise_flag(p.flags, LORA_FLAG_BAD_TOKEN);
        rank = p.ranks[U.s];
        scal = p.scalings[U.s];
        row_ok = tok >= 0;
        id = -1;
        if (p.h == nullptr && row_ok) {
          id = p.ids[tok];
          if (id < 0 || id >= p.vocab) row_ok = false;
        }
      }
      if (new_item || U.slice != prev_slice) {
        // Build H (hi and lo) for (tile, slice); the MMAs of the previous unit
        // are complete, since its epilogue waited for them.  The four warps of
        // a row split its 16-byte chunks.
        const int Kp = ceil_div_i(rank, 16) * 16;
        const int i = U.slice;
        for (int c8 = cg * 8; c8 < Kp; c8 += 32) {
          float v[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int r = c8 + q;
            float val = 0.f;
            if (row_ok && r < rank) {
              if (p.h != nullptr) {
                const float* hp = p.h + (size_t)tok * p.S * p.R + i * p.R + r;
                for (int ks = 0; ks < p.ksplit; ++ks) val += hp[(size_t)ks * p.h_split];
              } else {
                const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(p.a);
                val = __bfloat162float(
                    ab[((size_t)ab_of(p.slot_map, U.s) * p.S * p.R + i * p.R + r) * p.vocab + id]);
              }
            }
            v[q] = val;
          }
          uint32_t hi4[4], lo4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
            const float2 hf = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * q] - hf.x, v[2 * q + 1] - hf.y);
            hi4[q] = *reinterpret_cast<const uint32_t*>(&h2);
            lo4[q] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const uint32_t off = kmajor_offset(m, c8, span);
          *reinterpret_cast<uint4*>(hhi + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
          *reinterpret_cast<uint4*>(hlo + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(hready);
        prev_item = U.item;
        prev_slice = U.slice;
      }
      const int as = k & 1;
      if (!warp_wait(&accfull[as], (uint32_t)((k / 2) & 1), abort_flag, p.flags)) break;
      tc_fence_after();
      cp_async_wait<kNY - 1>();
      __syncwarp();   // the staged rows were copied by other lanes of this warp
      uint8_t* ybuf = ystage + (size_t)((k % kNY) * kTM) * kYRow;
      uint8_t* yrow = ybuf + (size_t)m * kYRow;
      const int c0 = cg * 32;                   // first column of this warp
      if (c0 < U.width) {                       // warp-uniform
        float acc[32];
        tmem_ld_32x32(tmem_base + lane_addr + (uint32_t)(as * kBN + c0), acc);
        if (row_ok) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (c0 + q * 8 < U.width) {
              const uint4 yv = *reinterpret_cast<const uint4*>(yrow + c0 * 2 + q * 16);
              uint32_t w[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = q * 8 + e * 2;
                w[e] = pack_bf16x2(fmaf(scal, acc[c], bf16_lo(w[e])),
                                   fmaf(scal, acc[c + 1], bf16_hi(w[e])));
              }
              *reinterpret_cast<uint4*>(yrow + c0 * 2 + q * 16) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[as]);
      // coalesced write-back of the warp's 32 rows x 32 columns
      {
        const int c = cg * 4 + (lane & 3);
        const bool cok = c < (U.width >> 3);
        const int tl = row_ok ? tok : -1;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = 8 * j + (lane >> 2);
          const int tr = __shfl_sync(0xffffffffu, tl, r);
          if (tr >= 0 && cok) {
            const uint4 v = *reinterpret_cast<const uint4*>(ybuf + (size_t)(quarter * 32 + r) * kYRow + c * 16);
            *reinterpret_cast<uint4*>(ybytes + ((size_t)tr * p.out + U.col0 + c * 8) * 2) = v;
          }
        }
      }
      U = U1;
      tok = t1;
      U1 = U2;
      t1 = t2;
      if (k + 3 < nloc) U2.advance(p, prefix);
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kBN);
  }
}

// ---------------------------------------------------------------------------
// Shrink
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kSgThreads, 1)
sgmv_shrink_kernel(const __grid_constant__ CUtensorMap tmap_a, const ShrinkParams p) {
  extern __shared__ uint8_t sg_smem_raw[];
  // Programmatic launch edge (when the caller opted in): the producers (x)
  // and the epilogue (writes h) wait for the preceding kernel.
  grid_dep_launch_dependents();
  const uint32_t raw = smem_u32(sg_smem_raw);
  uint8_t* base = sg_smem_raw + (align1024(raw) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(base);
  uint64_t* empty = full + kNS;
  uint64_t* accfull = empty + kNS;
  uint64_t* accempty = accfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + 256);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + 260);
  int* scratch = reinterpret_cast<int*>(base + 288);
  int* prefix = reinterpret_cast<int*>(base + 1024 + 512);
  const uint32_t pre_bytes = align1024((uint32_t)(p.slots + 1) * 4u + 512u);
  constexpr uint32_t kXTile = kTM * 128;            // 16 KB
  constexpr uint32_t kATile = 128 * 128;            // up to 128 rows of 128 bytes
  constexpr uint32_t kStage = kXTile + kATile;
  uint8_t* ring = base + 1024 + pre_bytes;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int SR = p.S * p.R;

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&full[i], 32 * kSgXWarps + 1);   // cp.async arrivals + 1 expect_tx arrival
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&accfull[i], 1);
      mbar_init(&accempty[i], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&tmap_a);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  const int items = plan_linear<kSgThreads>(p.slot_indptr, p.ranks, p.scalings, p.slots, p.T,
                                            p.R, kTM, prefix, scratch, p.flags,
                                            blockIdx.x == 0, p.seg_hi);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nkb_total = ceil_div_i(p.in, kKBLK);
  const long long units = (long long)items * p.ksplit;
  const long long u0 = units * blockIdx.x / gridDim.x;
  const long long u1 = units * (blockIdx.x + 1) / gridDim.x;
  const int nloc = (int)(u1 - u0);

  // unit -> (item, split)
  auto unit_geom = [&](long long u, int& s, int& p0, int& n, int& kb0, int& kb1, int& ks) {
    const int item = (int)(u / p.ksplit);
    ks = (int)(u - (long long)item * p.ksplit);
    s = find_segment(prefix, p.slots, item);
    p0 = p.slot_indptr[s] + (item - prefix[s]) * kTM;
    n = max(0, min(kTM, seg_end(p.slot_indptr, p.seg_hi, s) - p0));
    kb0 = min(nkb_total, ks * p.kb_per_split);
    kb1 = min(nkb_total, kb0 + p.kb_per_split);
  };

  if (warp == 0 || warp >= 6) {
    // ---------------- producers: x rows by cp.async (4 warps), A rows by tensor TMA (warp 0) ----
    grid_dep_wait();
    // Producer thread pt (0..127) copies 16-byte chunk c = pt % 8 of the tile
    // rows pt / 8 + 16 j (j < 8): eight lanes cover a 128-byte row segment,
    // and the chunk's swizzled position depends on the row only through
    // row % 8 = (pt / 8) % 8, fixed for the thread.
    const int pt = (warp == 0 ? 0 : warp - 5) * 32 + lane;
    const int c = pt & 7;
    const int r0 = pt >> 3;
    const uint32_t cswz = (uint32_t)(((c ^ (r0 & 7)) << 4));
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(p.x);
    int g = 0;  // stages issued
    for (int k = 0; k < nloc; ++k) {
      int s, p0, n, kb0, kb1, ks;
      unit_geom(u0 + k, s, p0, n, kb0, kb1, ks);
      const int rank = p.ranks[s];
      const int K0 = ceil_div_i(rank, 16) * 16;
      int trow[8];
#pragma unroll
      for (int j2 = 0; j2 < 8; ++j2) {
        const int mm = r0 + 16 * j2;
        int t = -1;
        if (mm < n) {
          t = p.token_order[p0 + mm];
          if (t < 0 || t >= p.T) {
            if (ks == 0 && c == 0) raise_flag(p.flags, LORA_FLAG_BAD_TOKEN);
            t = -1;
          }
        }
        trow[j2] = t;
      }
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int st = g % kNS;
        if (g >= kNS && !warp_wait(&empty[st], (uint32_t)((g / kNS - 1) & 1), abort_flag, p.flags)) {
          ok = false;
          break;
        }
        uint8_t* xt = ring + st * kStage;
        uint8_t* at = xt + kXTile;
        if (warp == 0 && lane == 0) {
          const int groups = ceil_div_i(rank, 16);
          mbar_arrive_expect_tx(&full[st], (uint32_t)(p.S * groups * 16 * 128));
          for (int i = 0; i < p.S; ++i)
            for (int q = 0; q < groups; ++q)
              tma_load_2d(at + (i * K0 + 16 * q) * 128, &tmap_a, kb * kKBLK,
                          ab_of(p.slot_map, s) * SR + i * p.R + 16 * q, &full[st]);
        }
        const int kcol = kb * kKBLK + c * 8;
        const bool cok = kcol < p.in;
        const uint32_t xbase = smem_u32(xt) + cswz;
#pragma unroll
        for (int j2 = 0; j2 < 8; ++j2) {
          const int t = trow[j2];
          const bool valid = t >= 0 && cok;
          cp_async16_zfill(xbase + (uint32_t)((r0 + 16 * j2) * 128),
                           valid ? xb + (size_t)t * p.in + kcol : xb, valid);
        }
        cp_async_arrive_noinc(&full[st]);
      }
      if (!ok) break;
    }
    cp_async_wait<0>();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int g = 0;
    for (int k = 0; k < nloc; ++k) {
      int s, p0, n, kb0, kb1, ks;
      unit_geom(u0 + k, s, p0, n, kb0, kb1, ks);
      const int rank = p.ranks[s];
      const int N = p.S * ceil_div_i(rank, 16) * 16;
      const uint32_t idesc = mma_idesc_bf16(kTM, N);
      const int as = k & 1;
      if (k >= 2 && !warp_wait(&accempty[as], (uint32_t)((k / 2 - 1) & 1), abort_flag, p.flags))
        break;
      tc_fence_after();
      const uint32_t d = tmem_base + (uint32_t)(as * 128);
      bool ok = true;
      bool first = true;
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int st = g % kNS;
        if (!warp_wait(&full[st], (uint32_t)((g / kNS) & 1), abort_flag, p.flags)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t xt = smem_u32(ring + st * kStage);
          const uint32_t at = xt + kXTile;
          for (int kk = 0; kk < kKBLK / 16; ++kk) {
            if (kb * kKBLK + kk * 16 >= p.in) break;
            mma_bf16_ss(d, smem_desc_kmajor(xt + kk * 32, 128), smem_desc_kmajor(at + kk * 32, 128),
                        idesc, first ? 0u : 1u);
            first = false;
          }
          mma_commit(&empty[st]);
        }
        __syncwarp();
      }
      if (!ok) break;
      // an empty input range accumulates nothing: its epilogue writes zeros
      if (lane == 0) mma_commit(&accfull[as]);
      __syncwarp();
    }
  } else {
    // ---------------- epilogue ----------------
    grid_dep_wait();
    const int quarter = warp & 3;
    const int m = quarter * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    for (int k = 0; k < nloc; ++k) {
      int s, p0, n, kb0, kb1, ks;
      unit_geom(u0 + k, s, p0, n, kb0, kb1, ks);
      const int rank = p.ranks[s];
      const int K0 = ceil_div_i(rank, 16) * 16;
      const int N = p.S * K0;
      const int as = k & 1;
      if (!warp_wait(&accfull[as], (uint32_t)((k / 2) & 1), abort_flag, p.flags)) break;
      tc_fence_after();
      int t = -1;
      if (m < n) {
        t = p.token_order[p0 + m];
        if (t < 0 || t >= p.T) t = -1;
      }
      float* hrow = (t >= 0) ? p.h + (size_t)ks * p.h_split + (size_t)t * SR : nullptr;
      const bool empty_range = kb1 <= kb0;
      for (int cg = 0; cg < N; cg += 32) {
        float acc[32];
        tmem_ld_32x32(tmem_base + lane_addr + (uint32_t)(as * 128 + cg), acc);
        if (hrow != nullptr) {
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            const int col = cg + q;
            const int i = col / K0;
            const int r = col - i * K0;
            if (col < N && r < rank) hrow[i * p.R + r] = empty_range ? 0.f : acc[q];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[as]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor map over `rows` rows of `cols` elements, box {box_cols, box_rows}.
cudaError_t make_map(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows,
                     uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz,
                     const char** why) {
  auto fn = encode_fn();
  if (fn == nullptr) {
    *why = "cuTensorMapEncodeTiled is not available";
    return cudaErrorNotSupported;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *why = "cuTensorMapEncodeTiled rejected the tensor";
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

struct DevInfo {
  int sms = 0;
  bool expand_attr = false, shrink_attr = false;
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

cudaError_t dev_info(DevInfo** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (d.sms == 0) {
    err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
  }
  *out = &d;
  return cudaSuccess;
}

// Launch with a programmatic stream-serialization edge when the process opted
// in (lora_set_launch_overlap), else as a plain launch.
template <typename P>
cudaError_t launch_overlapped(void (*kern)(const CUtensorMap, const P), int grid, int threads,
                              size_t smem, cudaStream_t stream, const CUtensorMap& map,
                              const P& p, bool allow_overlap = true) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3((unsigned)threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  if (allow_overlap && launch_overlap_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, map, p);
}

size_t expand_smem(int slots, int span) {
  const size_t pre = ((size_t)(slots + 1) * 4 + 1023) / 1024 * 1024;
  return 1024 + 1024 + pre + 2 * (size_t)kTM * span + (size_t)kNB * kBN * span +
         (size_t)kNY * kTM * kYRow;
}

size_t shrink_smem(int slots) {
  const size_t pre = ((size_t)(slots + 1) * 4 + 512 + 1023) / 1024 * 1024;
  return 1024 + 1024 + pre + (size_t)kNS * (kTM * 128 + 128 * 128);
}

int shrink_ksplit(int T, int slots, int in, int sms) {
  const int items = slots + ceil_div_i(T, kTM);
  const int nkb = ceil_div_i(in, kKBLK);
  int ks = ceil_div_i(sms, max(items, 1));
  ks = max(1, min(ks, 4));
  ks = min(ks, max(1, nkb / 8));
  return ks;
}

}  // namespace

bool sgmv_supported(int S, int R) {
  return (R == 16 || R == 32 || R == 64) && S * R <= 128;
}

size_t sgmv_workspace_bytes(int T, int R, int S) {
  // partial h buffers of the split shrink; the split factor is bounded by 4
  return (size_t)4 * T * R * S * sizeof(float);
}

cudaError_t sgmv_shrink_launch(const void* x, const void* a, float* h, const int* ranks,
                               const int* token_order, const int* slot_indptr, int T, int in,
                               int slots, int R, int S, uint32_t* flags, cudaStream_t stream,
                               const char** why, int ksplit_max, const float* scalings,
                               const SgmvGroups* groups) {
  if (in < kKBLK) {
    *why = "the SGMV shrink needs in_features >= 64";
    return cudaErrorNotSupported;
  }
  DevInfo* d = nullptr;
  cudaError_t err = dev_info(&d);
  if (err != cudaSuccess) return err;
  CUtensorMap map;
  const int ab_slots = groups != nullptr ? groups->ab_slots : slots;
  err = make_map(&map, a, (uint64_t)in, (uint64_t)ab_slots * S * R, kKBLK, 16,
                 CU_TENSOR_MAP_SWIZZLE_128B, why);
  if (err != cudaSuccess) return err;
  ShrinkParams p = {};
  p.x = x; p.h = h; p.ranks = ranks; p.scalings = scalings; p.token_order = token_order;
  p.slot_indptr = slot_indptr; p.flags = flags; p.T = T; p.in = in; p.slots = slots; p.R = R;
  p.S = S;
  if (groups != nullptr) {
    p.seg_hi = groups->seg_hi;
    p.slot_map = groups->slot_map;
  }
  p.ksplit = min(ksplit_max, shrink_ksplit(T, slots, in, d->sms));
  p.kb_per_split = ceil_div_i(ceil_div_i(in, kKBLK), p.ksplit);
  p.h_split = (size_t)T * S * R;
  const size_t smem = shrink_smem(slots);
  if (!d->shrink_attr) {
    err = cudaFuncSetAttribute(sgmv_shrink_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024);
    if (err != cudaSuccess) return err;
    d->shrink_attr = true;
  }
  const int units = (slots + ceil_div_i(T, kTM)) * p.ksplit;
  const int grid = max(1, min(d->sms, units));
  return launch_overlapped(sgmv_shrink_kernel, grid, kSgThreads, smem, stream, map, p,
                           groups == nullptr);
}

int sgmv_shrink_splits(int T, int slots, int in) {
  DevInfo* d = nullptr;
  if (dev_info(&d) != cudaSuccess) return 1;
  return shrink_ksplit(T, slots, in, d->sms);
}

cudaError_t sgmv_expand_launch(void* y, const float* h, int ksplit, const int* ids, const void* a,
                               const void* b, const int* ranks, const float* scalings,
                               const int* token_order, const int* slot_indptr, int T, int vocab,
                               int slots, int R, int S, const int* slice_off, int out,
                               uint32_t* flags, cudaStream_t stream, const char** why,
                               const SgmvGroups* groups) {
  DevInfo* d = nullptr;
  cudaError_t err = dev_info(&d);
  if (err != cudaSuccess) return err;
  CUtensorMap map;
  const CUtensorMapSwizzle swz = R == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : R == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                           : CU_TENSOR_MAP_SWIZZLE_32B;
  const int ab_slots = groups != nullptr ? groups->ab_slots : slots;
  err = make_map(&map, b, (uint64_t)R, (uint64_t)ab_slots * out, (uint32_t)R, kBN, swz, why);
  if (err != cudaSuccess) return err;
  ExpandParams p = {};
  p.y = y; p.h = h; p.ksplit = ksplit; p.h_split = (size_t)T * S * R; p.ids = ids; p.a = a;
  p.ranks = ranks; p.scalings = scalings; p.token_order = token_order;
  p.slot_indptr = slot_indptr; p.flags = flags; p.T = T; p.vocab = vocab; p.slots = slots;
  p.R = R; p.S = S; p.out = out; p.span = 2 * R;
  if (groups != nullptr) {
    p.seg_hi = groups->seg_hi;
    p.slot_map = groups->slot_map;
  }
  int nchunk = 0;
  for (int i = 0; i <= LORA_MAX_SLICES; ++i) p.slice_off[i] = slice_off[i];
  for (int i = 0; i < S; ++i) {
    p.chunk_off[i] = nchunk;
    nchunk += ceil_div_i(slice_off[i + 1] - slice_off[i], kBN);
  }
  for (int i = S; i <= LORA_MAX_SLICES; ++i) p.chunk_off[i] = nchunk;
  p.nchunk = nchunk;
  const size_t smem = expand_smem(slots, p.span);
  if (!d->expand_attr) {
    err = cudaFuncSetAttribute(sgmv_expand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               227 * 1024);
    if (err != cudaSuccess) return err;
    d->expand_attr = true;
  }
  const long long units = (long long)(slots + ceil_div_i(T, kTM)) * nchunk;
  const int grid = (int)max(1LL, min((long long)d->sms, units));
  return launch_overlapped(sgmv_expand_kernel, grid, kExThreads, smem, stream, map, p,
                           groups == nullptr);
}

}  // namespace lora
