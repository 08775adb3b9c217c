// BGMV regime (few tokens per slot), fused shrink + expand, split by bytes
// over every SM: the kernel lora_apply_linear runs when it is given a
// workspace.
//
// Work items are the planner's: up to kTT tokens of one slot.  A slot with
// more than kTT tokens is cut in token-id order (ties by position), so the
// item a token lands in -- and with it the order of every sum it takes part
// in -- does not depend on where the token sits in token_order.
//
// Shrink.  Item g reads its slot's S*rank live A rows and its tokens' x rows
// over all input features: (S*rank + n) rows x ceil(in/64) blocks of 64
// features.  The items' blocks are laid end to end and cut into gridDim.x
// contiguous ranges of equal rows x blocks, one per CTA; the part of an item a
// CTA owns is a piece.  A CTA stages all the rows of its pieces at once when
// they fit the staging ring (else in rounds): the A rows are copied before the
// launch-overlap wait (the preceding kernel may not write them), the x rows
// right after it (16-byte cp.async, rows padded for conflict-free ldmatrix).
// Each piece is reduced with m16n8k16 MMAs (A rows as M, tokens as N, fp32
// accumulate); its fp32 partial h goes to the workspace and is counted on the
// item's counter (release).
//
// Expand.  Item g writes n rows of y over all output columns, costing
// (2*rank + 4*n) bytes per column (B column, y read and write); those bytes
// are cut the same way.  The CTA stages the B columns and the y rows of its
// expand pieces' column ranges in the ring once its shrink is done (B and y
// were prefetched to L2 at the start), and for each piece waits (bounded) until the item's
// counter reaches the number of its shrink pieces (acquire), sums the partials
// in piece order into hi/lo bf16 h tiles, updates y with the staged m16n8k16
// expand of the cluster kernel and writes it back with 16-byte stores.  The
// last expand piece of an item to finish resets the item's counters, so the
// workspace is ready for the next call.
//
// Sources: mstar.engine.resources.lora.backend (LoraBackend.shrink,
// expand_fused, apply_linear_: a backend may fuse them; the token_order /
// slot_indptr addressing of shrink_reference and expand_reference_).
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "expand_tile.cuh"
#include "kernels.h"

namespace lora {

namespace {

constexpr int kSpThreads = kBgmvThreads;   // 256
constexpr int kSpWarps = kSpThreads / 32;

// ---------------------------------------------------------------------------
// Small device helpers
// ---------------------------------------------------------------------------

// Inclusive block scan of a u32 (blockDim.x == kSpThreads); the block total
// goes to *total.  scratch holds kSpWarps words.
LORA_DEV uint32_t block_scan_u32(uint32_t v, uint32_t* scratch, uint32_t* total) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kSpWarps; ++w) {
    const uint32_t s = scratch[w];
    if (w < warp) before += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return x + before;
}

// Largest g in [0, n) with cum[g] <= u (cum non-decreasing, cum[0] = 0).
LORA_DEV int seg_at(const uint32_t* cum, int n, uint32_t u) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cum[mid] <= u) lo = mid; else hi = mid;
  }
  return lo;
}

// v / d for d in 1..4 without a division instruction (0 <= v < 2^14).
LORA_DEV int div_small(int v, int d) {
  return d == 1 ? v : d == 2 ? (v >> 1) : d == 4 ? (v >> 2) : ((v * 21846) >> 16);
}

struct Item {
  int s, lo, ns, rank, tile, n;
};
LORA_DEV Item item_of(const int4* meta, int g) {
  const int4 m = meta[g];
  Item it;
  it.s = m.x;
  it.lo = m.y;
  it.ns = m.z;
  it.rank = m.w >> 16;
  it.tile = (m.w >> 8) & 0xff;
  it.n = m.w & 0xff;
  return it;
}
// Units per block of an item: for the shrink its rows (the bytes a block of
// features moves) plus 8 per (16-row, 8-token) MMA tile (the work a block
// takes once staged); for the expand the bytes per column.
LORA_DEV uint32_t units_per_block(const Item& it, int S, bool shrink) {
  return shrink ? (uint32_t)(S * it.rank + it.n + 8 * ceil_div_i(S * it.rank, 16) * ceil_div_i(it.n, 8))
                : (uint32_t)(2 * it.rank + 4 * it.n);
}

// Blocks [b0, b1) of item g inside the unit range [r0, r1).
LORA_DEV void piece_blocks(const uint32_t* cum, int g, uint32_t per, uint32_t r0, uint32_t r1,
                           int& b0, int& b1) {
  const uint32_t c0 = cum[g], c1 = cum[g + 1];
  const uint32_t lo = (r0 > c0 ? r0 : c0) - c0;
  const uint32_t hi = (r1 < c1 ? r1 : c1);
  b0 = (int)(lo / per);
  b1 = hi > c0 ? (int)((hi - c0) / per) : 0;
}

// Advances g to the first item at or after g with a non-empty piece in
// [r0, r1); false when there is none.
LORA_DEV bool find_piece(const int4* meta, const uint32_t* cum, int nitems, int S, bool shrink,
                         uint32_t r0, uint32_t r1, int& g, int& b0, int& b1) {
  for (; g < nitems && cum[g] < r1; ++g) {
    piece_blocks(cum, g, units_per_block(item_of(meta, g), S, shrink), r0, r1, b0, b1);
    if (b0 < b1) return true;
  }
  return false;
}

LORA_DEV float4 ld_cg_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
LORA_DEV void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Prefetches [src, src + bytes) into L2: 128-byte lines first, first + step, ...
LORA_DEV void prefetch_l2_span(const void* src, uint32_t bytes, int first, int step) {
  const char* c = static_cast<const char*>(src);
  for (uint32_t o = (uint32_t)first * 128u; o < bytes; o += (uint32_t)step * 128u)
    prefetch_l2_line(c + o);
}

// ---------------------------------------------------------------------------
// Shrink: rounds of pieces staged in the ring
// ---------------------------------------------------------------------------

// One staged part of a piece (blocks [b0, b1)): A rows at rows [0, S*rank),
// x rows right after them; row stride nb*128 + 16 bytes (odd in 16-byte units:
// conflict-free ldmatrix).  The rows span whole 16-row A tiles and 8-row x
// tiles (rows of a tile past its data hold other or stale values that only
// reach accumulator rows and columns that are never read).
struct Part {
  int g, b0, b1;
  uint32_t off;      // byte offset in the ring
  bool ends;         // last part of its piece
};
LORA_DEV int part_rows(const Item& it, int S) {
  const int nA = S * it.rank;
  return max(round_up_i(nA, 16), nA + round_up_i(it.n, 8));
}
LORA_DEV uint32_t part_stride(int nb) { return (uint32_t)(nb * 128 + 16); }

// Cursor over the CTA's shrink pieces: item g, blocks [b, bend) not yet staged.
struct ShrinkCursor {
  int g, b, bend;
  bool ok;
};

// Walks the parts of the next round from cursor `cur` (as many as fit `ring`
// bytes; the first always fits), calling f(part) for each; returns the cursor
// after the round.  Every thread walks the same parts.
template <class F>
LORA_DEV ShrinkCursor walk_round(ShrinkCursor cur, const int4* meta, const uint32_t* wcum,
                                 int nitems, int S, int ring, uint32_t r0, uint32_t r1, F&& f) {
  uint32_t off = 0;
  while (cur.ok) {
    const Item it = item_of(meta, cur.g);
    const int rows = part_rows(it, S);
    const int avail = ring - (int)off;
    const int nb_fit = (avail / rows - 16) / 128;
    if (nb_fit < 1) break;   // the round is full
    const int nb = min(cur.bend - cur.b, nb_fit);
    Part pt;
    pt.g = cur.g;
    pt.b0 = cur.b;
    pt.b1 = cur.b + nb;
    pt.off = off;
    pt.ends = pt.b1 == cur.bend;
    f(pt);
    off += (uint32_t)round_up_i(rows * (int)part_stride(nb), 128);
    cur.b = pt.b1;
    if (cur.b == cur.bend) {
      ++cur.g;
      cur.ok = find_piece(meta, wcum, nitems, S, true, r0, r1, cur.g, cur.b, cur.bend);
    }
  }
  return cur;
}

// The MMAs of one staged part, split along K over every warp: D[A rows,
// tokens] += A x^T.  Combo c is a (16-row, 8-token) tile; it is reduced by
// cpc chains, chain j taking k-steps j, j + cpc, ...  Chain q = c*cpc + j runs
// on warp q % 8 in accumulator slot q / 8, so a warp keeps up to 4 independent
// MMA chains in flight (the warp-level MMA has a long dependent latency on
// this GPU).  A part's chains are then summed per combo in chain order through
// the part's own shared memory (its rows have been read by then), and the
// result goes to `part_out` as fp32 partial h rows part[t][i*R + r].  A piece
// cut over two rounds adds its next part's sums to those rows (each thread
// re-reads only values it wrote itself).  Every thread must call it.
constexpr int kChainSlots = 4;

LORA_DEV void shrink_part(const Item& it, int S, int R, int in, const Part& pt, uint8_t* ring,
                          float* part_out, bool carry_in) {
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int fv = min(in, pt.b1 * kSpKQ) - pt.b0 * kSpKQ;
  const int nks = ceil_div_i(fv, 16);
  const bool half_last = (fv & 15) != 0;
  const uint32_t stride = part_stride(pt.b1 - pt.b0);
  uint8_t* base_p = ring + pt.off;
  const uint32_t base = smem_u32(base_p);
  const int nA = S * it.rank;
  const int NTt = ceil_div_i(it.n, 8);
  const int C = ceil_div_i(nA, 16) * NTt;
  const int qmax = min(kChainSlots * kSpWarps, part_rows(it, S) * (int)stride / 512);
  const int cpc = max(1, min(nks, qmax / C));
  const int Q = C * cpc;
  const int nsteps = ceil_div_i(nks, cpc);
  uint32_t a_addr[kChainSlots], x_addr[kChainSlots];
  int jj[kChainSlots];
#pragma unroll
  for (int sl = 0; sl < kChainSlots; ++sl) {
    const int q = min(sl * kSpWarps + warp, Q - 1);
    const int cb = q / cpc;
    jj[sl] = (sl * kSpWarps + warp < Q) ? q - cb * cpc : nks;   // nks: no k-steps
    const int mt = div_small(cb, NTt);
    const int nt = cb - mt * NTt;
    a_addr[sl] = base + (uint32_t)(mt * 16 + (lane & 15)) * stride + (lane >> 4) * 16;
    x_addr[sl] = base + (uint32_t)(nA + nt * 8 + (lane & 7)) * stride + ((lane >> 3) & 1) * 16;
  }
  float acc[kChainSlots][4];
#pragma unroll
  for (int sl = 0; sl < kChainSlots; ++sl)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[sl][e] = 0.f;
  for (int t = 0; t < nsteps; ++t) {
    uint32_t fa[kChainSlots][4], fb[kChainSlots][2];
#pragma unroll
    for (int sl = 0; sl < kChainSlots; ++sl) {
      const int ks = jj[sl] + t * cpc;
      if (ks < nks) {
        ldsm_x4(a_addr[sl] + ks * 32, fa[sl][0], fa[sl][1], fa[sl][2], fa[sl][3]);
        ldsm_x2(x_addr[sl] + ks * 32, fb[sl][0], fb[sl][1]);
        if (half_last && ks == nks - 1) {   // only 8 valid features in this step
          fa[sl][2] = 0u;
          fa[sl][3] = 0u;
          fb[sl][1] = 0u;
        }
      }
    }
#pragma unroll
    for (int sl = 0; sl < kChainSlots; ++sl)
      if (jj[sl] + t * cpc < nks)
        mma_bf16_16816(acc[sl], fa[sl][0], fa[sl][1], fa[sl][2], fa[sl][3], fb[sl][0], fb[sl][1]);
  }
  __syncthreads();   // every warp has read the part's rows
  float4* red = reinterpret_cast<float4*>(base_p);
#pragma unroll
  for (int sl = 0; sl < kChainSlots; ++sl) {
    const int q = sl * kSpWarps + warp;
    if (q < Q) red[q * 32 + lane] = make_float4(acc[sl][0], acc[sl][1], acc[sl][2], acc[sl][3]);
  }
  __syncthreads();
  const int SR = S * R;
  for (int pp = tid; pp < C * 32; pp += kSpThreads) {
    const int cb = pp >> 5;
    const int l = pp & 31;
    const int mt = div_small(cb, NTt);
    const int nt = cb - mt * NTt;
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < cpc; ++j) {
      const float4 f = red[(cb * cpc + j) * 32 + l];
      v[0] += f.x;
      v[1] += f.y;
      v[2] += f.z;
      v[3] += f.w;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = mt * 16 + (l >> 2) + 8 * h;
      if (row < nA) {
        const int i = row / it.rank;
        const int col = i * R + (row - i * it.rank);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = nt * 8 + 2 * (l & 3) + e;
          if (t < it.n) {
            float* dst = part_out + (size_t)t * SR + col;
            *dst = carry_in ? *dst + v[2 * h + e] : v[2 * h + e];
          }
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Expand: rounds of jobs (column chunks of pieces) staged in the ring
// ---------------------------------------------------------------------------

// A round holds up to kMaxJobs jobs of up to kMaxPieces pieces.  Thread 0
// plans it into two shared tables (all threads then read them):
//   job   [8 ints]: item, first column, end column, ring offset, piece, last job of its piece
//   piece [16 ints]: item, first slice, last slice, h offset (floats), shrink
//     candidates [cw0, cw1], expand candidates [cv0, cv1], shrink pieces (the
//     gate's target), expand pieces, non-empty mask of the shrink candidates
//     (two words; valid when cw1 - cw0 < 64), gate passed, live-token mask,
//     scaling bits, consumed count before this piece
constexpr int kMaxJobs = 8;
constexpr int kMaxPieces = 8;
constexpr int kJobInts = 8;
constexpr int kPieceInts = 16;
enum { kJG = 0, kJJ0, kJJ1, kJOff, kJPiece, kJLast };
enum { kPG = 0, kPIa, kPIb, kPHoff, kPCw0, kPCw1, kPCv0, kPCv1, kPTarget, kPNexp, kPMask0,
       kPMask1, kPOk, kPLive, kPScal, kPCons };

struct ExpandCursor {
  int g, cb, cbend, cb0;   // item, next block, end block, first block of the piece
  bool ok;
};

LORA_DEV uint32_t job_bytes(int cols, int n) { return (uint32_t)round_up_i(n * (cols * 2 + 16), 128); }

// Slices [ia, ib] that output columns [c0, c1) touch.
LORA_DEV void slice_span(const int* slice_off, int S, int c0, int c1, int& ia, int& ib) {
  ia = 0;
  while (ia + 1 < S && slice_off[ia + 1] <= c0) ++ia;
  ib = ia;
  while (ib + 1 < S && slice_off[ib + 1] < c1) ++ib;
}

// Every thread issues its share of the copies of a job: the y rows of its
// valid tokens over columns [j0, j1), a warp per row.
LORA_DEV void issue_job(const SplitParams& p, const int* ttok, int n, int j0, int j1,
                        uint32_t base) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int cols = j1 - j0;
  const uint32_t ystride = (uint32_t)(cols * 2 + 16);
  const int ych = cols / 8;
  for (int t = warp; t < n; t += kSpWarps) {
    const int tk = ttok[t];
    if (tk < 0 || tk >= p.T) continue;
    const __nv_bfloat16* ysrc =
        reinterpret_cast<const __nv_bfloat16*>(p.y) + (size_t)tk * p.out + j0;
    for (int q = lane; q < ych; q += 32)
      cp_async16(base + (uint32_t)t * ystride + (uint32_t)q * 16u, ysrc + q * 8);
  }
}

// The expand of one staged job on one slice, for a warp: 16-column tiles at
// ct0 = ls0 + 16*warp, ls0 + 16*(warp + 8), ...; for each tile its B fragment
// is loaded once and the MMAs of every 8-token tile follow (independent
// chains): D[16 columns, 8 tokens] = B H^T with H = hi + lo in bf16 (B read
// from global memory, where it was prefetched to L2), then
// y = bf16_rne(y + scal * D) on the live rows, in the staged copy.  Column
// 2g / 2g+1 of a tile is MMA row g / g + 8; rank 4c..4c+3 of a k-step is MMA
// k 2c, 2c+1, 2c+8, 2c+9 (one 8-byte load per operand, the same permutation
// in B and H).  hhi / hlo: the slice's h tiles, rows = tokens, row stride hst.
template <int NTT>
LORA_DEV void expand_slice(const uint16_t* __restrict__ bg, const uint16_t* __restrict__ hhi,
                           const uint16_t* __restrict__ hlo, int hst, uint8_t* __restrict__ ys,
                           int ystride, int R, int rank, int ls0, int ls1, uint32_t live,
                           float scal, int warp, int g, int c) {
  const int ksteps = ceil_div_i(rank, 16);
  // the h fragments of every token tile for k-step 0
  uint2 h0[NTT], l0[NTT];
  bool tv[NTT][2];
#pragma unroll
  for (int nt = 0; nt < NTT; ++nt) {
    const int o = (nt * 8 + g) * hst + 4 * c;
    h0[nt] = *reinterpret_cast<const uint2*>(hhi + o);
    l0[nt] = *reinterpret_cast<const uint2*>(hlo + o);
#pragma unroll
    for (int e = 0; e < 2; ++e) tv[nt][e] = (live >> (nt * 8 + 2 * c + e)) & 1u;
  }
  const uint2 m0 = rank_mask4(4 * c, rank);
  for (int ct0 = ls0 + 16 * warp; ct0 < ls1; ct0 += 16 * kSpWarps) {
    const int jl = ct0 + 2 * g;
    const bool ok = jl < ls1;
    float d[NTT][4];
    uint32_t yo[NTT][2];
#pragma unroll
    for (int nt = 0; nt < NTT; ++nt) {
#pragma unroll
      for (int k = 0; k < 4; ++k) d[nt][k] = 0.f;
#pragma unroll
      for (int e = 0; e < 2; ++e)
        yo[nt][e] = (ok && tv[nt][e])
                        ? *reinterpret_cast<const uint32_t*>(ys + (size_t)(nt * 8 + 2 * c + e) * ystride + jl * 2)
                        : 0u;
    }
    for (int ks = 0; ks < ksteps; ++ks) {
      const int k0 = ks * 16 + 4 * c;
      const uint2 mk = ks == 0 ? m0 : rank_mask4(k0, rank);
      uint2 b0 = make_uint2(0u, 0u), b1 = make_uint2(0u, 0u);
      if (ok && k0 < R) {
        b0 = __ldg(reinterpret_cast<const uint2*>(bg + (size_t)jl * R + k0));
        b1 = __ldg(reinterpret_cast<const uint2*>(bg + (size_t)(jl + 1) * R + k0));
      }
      b0 = make_uint2(b0.x & mk.x, b0.y & mk.y);
      b1 = make_uint2(b1.x & mk.x, b1.y & mk.y);
      uint2 hh[NTT], hl[NTT];
#pragma unroll
      for (int nt = 0; nt < NTT; ++nt) {
        if (ks == 0) {
          hh[nt] = h0[nt];
          hl[nt] = l0[nt];
        } else {
          const int o = (nt * 8 + g) * hst + k0;
          hh[nt] = *reinterpret_cast<const uint2*>(hhi + o);
          hl[nt] = *reinterpret_cast<const uint2*>(hlo + o);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NTT; ++nt)
        mma_bf16_16816(d[nt], b0.x, b1.x, b0.y, b1.y, hh[nt].x, hh[nt].y);
#pragma unroll
      for (int nt = 0; nt < NTT; ++nt)
        mma_bf16_16816(d[nt], b0.x, b1.x, b0.y, b1.y, hl[nt].x, hl[nt].y);
    }
#pragma unroll
    for (int nt = 0; nt < NTT; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e)
        if (ok && tv[nt][e])
          *reinterpret_cast<uint32_t*>(ys + (size_t)(nt * 8 + 2 * c + e) * ystride + jl * 2) =
              pack_bf16x2(fmaf(scal, d[nt][e], bf16_lo(yo[nt][e])),
                          fmaf(scal, d[nt][2 + e], bf16_hi(yo[nt][e])));
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(kSpThreads, 2) bgmv_split_kernel(const SplitParams p) {
  extern __shared__ __align__(128) uint8_t sp_smem[];
  // With a programmatic launch edge the next kernel may start its CTAs while
  // this one runs; x, y, the workspace and the flags are touched only after
  // grid_dep_wait().  Without one both are no-ops.
  grid_dep_launch_dependents();
  const SplitLayout L = split_layout(p.T, p.item_cap, p.ring);
  int* tok = reinterpret_cast<int*>(sp_smem + L.tok_off);
  int4* meta = reinterpret_cast<int4*>(sp_smem + L.meta_off);
  uint32_t* wcum = reinterpret_cast<uint32_t*>(sp_smem + L.wcum_off);
  uint32_t* vcum = reinterpret_cast<uint32_t*>(sp_smem + L.vcum_off);
  int* cand = reinterpret_cast<int*>(sp_smem + L.cand_off);
  uint32_t* wst = reinterpret_cast<uint32_t*>(sp_smem + L.wst_off);
  uint32_t* vst = reinterpret_cast<uint32_t*>(sp_smem + L.vst_off);
  int* ctrl = reinterpret_cast<int*>(sp_smem + L.ctrl_off);
  uint32_t* scan = reinterpret_cast<uint32_t*>(ctrl);        // [0, 16)
  uint8_t* ring = sp_smem + L.ring_off;
  int* prefix = reinterpret_cast<int*>(ring);   // planner prefix, in the ring until staging
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int G = (int)gridDim.x;
  const int c = (int)blockIdx.x;
  const int S = p.S;
  const int R = p.R;

  // ---- planning (addressing only: before the launch-overlap wait) ----------
  // Error bits found before the wait are collected here and raised after it
  // (the preceding kernel may be the one that clears the caller's flags).
  uint32_t* pre_flags = reinterpret_cast<uint32_t*>(ctrl + 32);
  if (tid == 0) *pre_flags = 0u;
  for (int i = tid; i < p.T; i += kSpThreads) tok[i] = p.token_order[i];
  const int planned = plan_linear<kSpThreads>(p.slot_indptr, p.ranks, p.scalings, p.slots, p.T,
                                              R, kTT, prefix, ctrl + 16, pre_flags, c == 0);
  const int nitems = min(planned, p.item_cap);
  if (planned > p.item_cap && c == 0 && tid == 0) atomicOr(pre_flags, LORA_FLAG_BAD_INDPTR);
  const int kblocks = ceil_div_i(p.in, kSpKQ);
  const int ncb = ceil_div_i(p.out, kSpCQ);
  uint32_t wcarry = 0, vcarry = 0, mcarry = 0;
  if (tid == 0) {
    wcum[0] = 0u;
    vcum[0] = 0u;
  }
  for (int base = 0; base < nitems; base += kSpThreads) {
    const int g = base + tid;
    uint32_t w = 0, v = 0, multi = 0;
    if (g < nitems) {
      const int s = find_segment(prefix, p.slots, g);
      const int k = g - prefix[s];
      const int lo = p.slot_indptr[s];
      const int ns = p.slot_indptr[s + 1] - lo;
      const int n = min(kTT, ns - k * kTT);
      const int r = p.ranks[s];
      meta[g] = make_int4(s, lo, ns, (r << 16) | (k << 8) | n);
      Item it;
      it.rank = r;
      it.n = n;
      w = units_per_block(it, S, true) * (uint32_t)kblocks;
      v = units_per_block(it, S, false) * (uint32_t)ncb;
      multi = (k == 1) ? 1u : 0u;   // the second item of a slot: the slot holds several
    }
    uint32_t tw, tv, tm;
    const uint32_t iw = block_scan_u32(w, scan, &tw);
    const uint32_t iv = block_scan_u32(v, scan + 8, &tv);
    const uint32_t im = block_scan_u32(multi, scan, &tm);
    if (g < nitems) {
      wcum[g + 1] = wcarry + iw;
      vcum[g + 1] = vcarry + iv;
      if (multi) cand[mcarry + im - 1] = g;   // at most nitems / 2 <= kSpMaxGrid entries
    }
    wcarry += tw;
    vcarry += tv;
    mcarry += tm;
  }
  const uint32_t Wt = wcarry, Vt = vcarry;
  // first unit of every CTA's shrink and expand range
  for (int c2 = tid; c2 <= G; c2 += kSpThreads) {
    wst[c2] = (uint32_t)(((unsigned long long)c2 * Wt) / (unsigned)G);
    vst[c2] = (uint32_t)(((unsigned long long)c2 * Vt) / (unsigned)G);
  }
  __syncthreads();
  // Slots with more than one item: order their tokens by (id, position), so the
  // item of a token does not depend on its position (the ring is free scratch).
  const int nmulti = (int)mcarry;
  for (int q = 0; q < nmulti; ++q) {
    const Item it = item_of(meta, cand[q]);
    int* scratch = reinterpret_cast<int*>(ring);
    for (int j = tid; j < it.ns; j += kSpThreads) scratch[j] = tok[it.lo + j];
    __syncthreads();
    for (int j = tid; j < it.ns; j += kSpThreads) {
      const int key = scratch[j];
      int rank = 0;
      for (int q2 = 0; q2 < it.ns; ++q2) {
        const int v = scratch[q2];
        rank += (v < key || (v == key && q2 < j)) ? 1 : 0;
      }
      tok[it.lo + rank] = key;
    }
    __syncthreads();
  }
  if (Wt == 0u) {   // no live item: only the flags to report
    grid_dep_wait();
    if (tid == 0) raise_flag(p.flags, *pre_flags);
    return;
  }
  const uint32_t w0 = wst[c], w1 = wst[c + 1];
  const uint32_t v0 = vst[c], v1 = vst[c + 1];

  // ---- B columns of this CTA's expand pieces into L2 (before the wait) -----
  {
    int g = seg_at(vcum, nitems, v0), b0, b1;
    while (find_piece(meta, vcum, nitems, S, false, v0, v1, g, b0, b1)) {
      const Item it = item_of(meta, g);
      const int j0 = b0 * kSpCQ, j1 = min(p.out, b1 * kSpCQ);
      prefetch_l2_span(reinterpret_cast<const __nv_bfloat16*>(p.b) + ((size_t)it.s * p.out + j0) * R,
                       (uint32_t)((j1 - j0) * R * 2), tid, kSpThreads);
      ++g;
    }
  }

  // ---- expand round tables -----------------------------------------------------
  // Thread 0 plans a round (jobs staged from the front of the ring, each
  // piece's h tiles from its back); then every thread fills in the pieces'
  // gate targets, expand piece counts and live tokens.  Round 0 is planned
  // here, before the wait: it needs only the addressing and the scalings.
  const int hst = split_hst(R) + 8;   // h tile row stride (bf16): padded against bank conflicts
  int* xtab = reinterpret_cast<int*>(sp_smem + L.xtab_off);
  int* jt = xtab;                                  // [kMaxJobs][kJobInts]
  int* pt = xtab + kMaxJobs * kJobInts;            // [kMaxPieces][kPieceInts]
  int* hdr = pt + kMaxPieces * kPieceInts;         // [0] jobs, [1] pieces
  // thread 0's expand cursor, kept in shared memory between rounds
  ExpandCursor* ecp = reinterpret_cast<ExpandCursor*>(hdr + 4);
  if (tid == 0) {
    ExpandCursor ec;
    ec.g = seg_at(vcum, nitems, v0);
    ec.ok = find_piece(meta, vcum, nitems, S, false, v0, v1, ec.g, ec.cb, ec.cbend);
    ec.cb0 = ec.cb;
    *ecp = ec;
  }
  auto expand_plan = [&](int) {
    if (tid == 0) {
      ExpandCursor ec = *ecp;
      int nj = 0, np = 0;
      uint32_t lo = 0, hi = (uint32_t)p.ring;
      while (ec.ok && nj < kMaxJobs) {
        const Item it = item_of(meta, ec.g);
        const bool new_piece = nj == 0 || jt[(nj - 1) * kJobInts + kJG] != ec.g;
        if (new_piece && np == kMaxPieces) break;
        int ia, ib;
        slice_span(p.slice_off, S, ec.cb0 * kSpCQ, min(p.out, ec.cbend * kSpCQ), ia, ib);
        const uint32_t hb =
            new_piece ? (uint32_t)round_up_i(2 * (ib - ia + 1) * round_up_i(it.n, 8) * hst * 2, 128)
                      : 0u;
        const int per_col = 2 * it.n;   // staged y bytes per column
        const int avail = (int)(hi - hb) - (int)lo - 256 - it.n * 16;
        const int nbk = avail > 0 ? min(ec.cbend - ec.cb, avail / (kSpCQ * per_col)) : 0;
        if (nbk < 1) break;   // the round is full
        if (new_piece) {
          int* P = pt + np * kPieceInts;
          hi -= hb;
          P[kPG] = ec.g;
          P[kPIa] = ia;
          P[kPIb] = ib;
          P[kPHoff] = (int)hi;
          P[kPCw0] = seg_at(wst, G, wcum[ec.g]);
          P[kPCw1] = seg_at(wst, G, wcum[ec.g + 1] - 1u);
          P[kPCv0] = seg_at(vst, G, vcum[ec.g]);
          P[kPCv1] = seg_at(vst, G, vcum[ec.g + 1] - 1u);
          P[kPTarget] = 0;
          P[kPNexp] = 0;
          P[kPMask0] = 0;
          P[kPMask1] = 0;
          P[kPScal] = __float_as_int(p.scalings[it.s]);
          ++np;
        }
        int* J = jt + nj * kJobInts;
        J[kJG] = ec.g;
        J[kJJ0] = ec.cb * kSpCQ;
        J[kJJ1] = min(p.out, (ec.cb + nbk) * kSpCQ);
        J[kJOff] = (int)lo;
        J[kJPiece] = np - 1;
        J[kJLast] = ec.cb + nbk == ec.cbend ? 1 : 0;
        lo += job_bytes(J[kJJ1] - J[kJJ0], it.n);
        ++nj;
        ec.cb += nbk;
        if (J[kJLast]) {
          ++ec.g;
          ec.ok = find_piece(meta, vcum, nitems, S, false, v0, v1, ec.g, ec.cb, ec.cbend);
          ec.cb0 = ec.cb;
        }
      }
      hdr[0] = nj;
      hdr[1] = np;
      *ecp = ec;
    }
    __syncthreads();
    const int np = hdr[1];
    // each piece's shrink pieces (non-empty candidates: the gate's target) and
    // expand pieces, and its live tokens
    for (int q = tid; q < np * 128; q += kSpThreads) {
      const int pi = q >> 7;
      const int j = q & 63;
      int* P = pt + pi * kPieceInts;
      const int g = P[kPG];
      const Item it = item_of(meta, g);
      if ((q & 64) == 0) {
        const int cw0 = P[kPCw0], cw1 = P[kPCw1];
        for (int j2 = j; j2 <= cw1 - cw0; j2 += 64) {
          int b0, b1;
          piece_blocks(wcum, g, units_per_block(it, S, true), wst[cw0 + j2], wst[cw0 + j2 + 1], b0,
                       b1);
          if (b0 < b1) {
            atomicAdd(&P[kPTarget], 1);
            if (j2 < 64) atomicOr(&P[kPMask0 + (j2 >> 5)], (int)(1u << (j2 & 31)));
          }
        }
      } else {
        const int cv0 = P[kPCv0], cv1 = P[kPCv1];
        for (int j2 = j; j2 <= cv1 - cv0; j2 += 64) {
          int b0, b1;
          piece_blocks(vcum, g, units_per_block(it, S, false), vst[cv0 + j2], vst[cv0 + j2 + 1],
                       b0, b1);
          if (b0 < b1) atomicAdd(&P[kPNexp], 1);
        }
      }
    }
    if (warp < np) {
      int* P = pt + warp * kPieceInts;
      const Item it = item_of(meta, P[kPG]);
      const int tk = lane < it.n ? tok[it.lo + it.tile * kTT + lane] : -1;
      const uint32_t live = __ballot_sync(0xffffffffu, lane < it.n && tk >= 0 && tk < p.T);
      if (lane == 0) {
        P[kPLive] = (int)live;
        if (live != (it.n >= 32 ? 0xffffffffu : ((1u << it.n) - 1u)))
          atomicOr(pre_flags, LORA_FLAG_BAD_TOKEN);
      }
    }
  };
  expand_plan(0);

  // ---- shrink ----------------------------------------------------------------
  const uint32_t ring_u32 = smem_u32(ring);
  const __nv_bfloat16* a_g = reinterpret_cast<const __nv_bfloat16*>(p.a);
  const __nv_bfloat16* x_g = reinterpret_cast<const __nv_bfloat16*>(p.x);
  // A rows of a part: warp w copies rows w, w + 8, ... (slice i and rank row r
  // carried without divisions), its lanes over the row's 16-byte chunks.
  auto issue_a = [&](const Part& pt) {
    const Item it = item_of(meta, pt.g);
    const int f0 = pt.b0 * kSpKQ;
    const int cpr = (min(p.in, pt.b1 * kSpKQ) - f0) >> 3;
    const uint32_t stride = part_stride(pt.b1 - pt.b0);
    const uint32_t base = ring_u32 + pt.off;
    const __nv_bfloat16* abase = a_g + (size_t)it.s * S * R * p.in + f0;
    const int nA = S * it.rank;
    int i = 0, r = warp;
    while (r >= it.rank) {
      r -= it.rank;
      ++i;
    }
    for (int row = warp; row < nA; row += kSpWarps) {
      const __nv_bfloat16* src = abase + (size_t)(i * R + r) * p.in;
      for (int ch = lane; ch < cpr; ch += 32)
        cp_async16(base + (uint32_t)row * stride + (uint32_t)ch * 16u, src + ch * 8);
      r += kSpWarps;
      while (r >= it.rank) {
        r -= it.rank;
        ++i;
      }
    }
  };
  // x rows of a part: warp w copies the rows of tokens w, w + 8, ...
  auto issue_x = [&](const Part& pt) {
    const Item it = item_of(meta, pt.g);
    const int f0 = pt.b0 * kSpKQ;
    const int cpr = (min(p.in, pt.b1 * kSpKQ) - f0) >> 3;
    const uint32_t stride = part_stride(pt.b1 - pt.b0);
    const uint32_t base = ring_u32 + pt.off + (uint32_t)(S * it.rank) * stride;
    const int* ttok = tok + it.lo + it.tile * kTT;
    for (int t = warp; t < it.n; t += kSpWarps) {
      const int tk = ttok[t];
      if (tk < 0 || tk >= p.T) continue;
      const __nv_bfloat16* src = x_g + (size_t)tk * p.in + f0;
      for (int ch = lane; ch < cpr; ch += 32)
        cp_async16(base + (uint32_t)t * stride + (uint32_t)ch * 16u, src + ch * 8);
    }
  };
  ShrinkCursor sc;
  sc.g = seg_at(wcum, nitems, w0);
  sc.ok = find_piece(meta, wcum, nitems, S, true, w0, w1, sc.g, sc.b, sc.bend);
  // the first round's A rows before the wait, its x rows after it
  if (sc.ok) walk_round(sc, meta, wcum, nitems, S, p.ring, w0, w1, issue_a);
  cp_async_commit();

  grid_dep_wait();   // x, y, the workspace and the flags from here on
  if (tid == 0) raise_flag(p.flags, *pre_flags);

  // y rows of this CTA's expand pieces into L2
  {
    int g = seg_at(vcum, nitems, v0), b0, b1;
    while (find_piece(meta, vcum, nitems, S, false, v0, v1, g, b0, b1)) {
      const Item it = item_of(meta, g);
      const int j0 = b0 * kSpCQ, j1 = min(p.out, b1 * kSpCQ);
      const int* ttok = tok + it.lo + it.tile * kTT;
      for (int t = warp; t < it.n; t += kSpWarps) {
        const int tk = ttok[t];
        if (tk >= 0 && tk < p.T)
          prefetch_l2_span(reinterpret_cast<const __nv_bfloat16*>(p.y) + (size_t)tk * p.out + j0,
                           (uint32_t)((j1 - j0) * 2), lane, 32);
      }
      ++g;
    }
  }

  const size_t piece_floats = (size_t)kTT * S * R;
  bool carry_in = false;   // the piece's earlier part left its sums in its partial rows
  bool first_round = true;
  while (sc.ok) {
    if (!first_round) {
      __syncthreads();   // the previous round's parts have been reduced
      walk_round(sc, meta, wcum, nitems, S, p.ring, w0, w1, issue_a);
    }
    walk_round(sc, meta, wcum, nitems, S, p.ring, w0, w1, issue_x);
    cp_async_commit();
    cp_async_wait<0>();
    __syncthreads();
    sc = walk_round(sc, meta, wcum, nitems, S, p.ring, w0, w1, [&](const Part& pt) {
      const Item it = item_of(meta, pt.g);
      shrink_part(it, S, R, p.in, pt, ring, p.part + (size_t)(pt.g + c) * piece_floats, carry_in);
      carry_in = !pt.ends;
      __syncthreads();
      if (pt.ends && tid == 0) {
        __threadfence();
        atomicAdd(&p.cnt[pt.g], 1u);
      }
    });
    first_round = false;
  }
  __syncthreads();   // the ring is free for the expand

  // ---- expand ---------------------------------------------------------------
  // Rounds of jobs, planned (round 0 before the wait) into the tables; then
  // every thread stages the round's jobs, the round's gates are polled
  // together, one sweep builds the pieces' h (hi / lo bf16 tiles), one sweep of
  // MMA units updates y in the staged rows and one writes them back.
  for (int xr = 0;; ++xr) {
    if (xr > 0) {
      expand_plan(xr);
      __syncthreads();
    }
    const int nj = hdr[0];
    const int np = hdr[1];
    if (nj == 0) break;
    // stage every job of the round
    for (int k = 0; k < nj; ++k) {
      const int* J = jt + k * kJobInts;
      const Item it = item_of(meta, J[kJG]);
      issue_job(p, tok + it.lo + it.tile * kTT, it.n, J[kJJ0], J[kJJ1], ring_u32 + J[kJOff]);
    }
    cp_async_commit();
    // the round's gates, polled together; a piece whose last job is in this
    // round then counts itself as consumed
    if (tid == 0) {
      uint32_t pending = (1u << np) - 1u;
      const uint64_t t0 = global_timer_ns();
      for (;;) {
        for (int pi = 0; pi < np; ++pi)
          if ((pending >> pi) & 1u) {
            const int* P = pt + pi * kPieceInts;
            if (ld_acquire_u32(p.cnt + P[kPG]) == (uint32_t)P[kPTarget]) pending &= ~(1u << pi);
          }
        if (pending == 0u || global_timer_ns() - t0 > p.wait_ns) break;
      }
      if (pending != 0u) raise_flag(p.flags, LORA_FLAG_TIMEOUT);
      for (int pi = 0; pi < np; ++pi) pt[pi * kPieceInts + kPOk] = ((pending >> pi) & 1u) ? 0 : 1;
      for (int k = 0; k < nj; ++k) {
        const int* J = jt + k * kJobInts;
        if (J[kJLast]) pt[J[kJPiece] * kPieceInts + kPCons] = (int)atomicAdd(p.cons + J[kJG], 1u);
      }
    }
    __syncthreads();
    // h of every piece: the sum of its shrink pieces' partials in CTA order,
    // split into hi / lo bf16 tiles [slice - ia][token][hst] (zero past the
    // rank and the tokens)
    for (int pi = 0; pi < np; ++pi) {
      const int* P = pt + pi * kPieceInts;
      if (!P[kPOk]) continue;
      const int g = P[kPG];
      const Item it = item_of(meta, g);
      const int ia = P[kPIa];
      const int n8 = round_up_i(it.n, 8);
      const int q4 = round_up_i(it.rank, 16) / 4;
      const int per_s = n8 * q4;
      const int total = (P[kPIb] - ia + 1) * per_s;
      const int cw0 = P[kPCw0];
      const int ncw = P[kPCw1] - cw0 + 1;
      const uint64_t mask = (uint32_t)P[kPMask0] | ((uint64_t)(uint32_t)P[kPMask1] << 32);
      const uint32_t per = units_per_block(it, S, true);
      const float* pbase = p.part + (size_t)g * piece_floats;
      uint16_t* hhi = reinterpret_cast<uint16_t*>(ring + P[kPHoff]);
      uint16_t* hlo = hhi + (size_t)(P[kPIb] - ia + 1) * n8 * hst;
      const int SR = S * R;
      for (int e = tid; e < total; e += kSpThreads) {
        const int iq = e / per_s;
        const int rem = e - iq * per_s;
        const int t = rem / q4;
        const int r0 = (rem - t * q4) * 4;
        float v[4] = {0.f, 0.f, 0.f, 0.f};
        if (t < it.n && r0 < it.rank) {
          const float* src = pbase + (size_t)t * SR + (ia + iq) * R + r0;
          for (int j = 0; j < ncw; j += 4) {
            float4 f[4];
            bool on[4];
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int jj2 = j + w;
              if (jj2 < 64) {
                on[w] = jj2 < ncw && ((mask >> jj2) & 1ull);
              } else {
                int b0 = 0, b1 = 0;
                if (jj2 < ncw)
                  piece_blocks(wcum, g, per, wst[cw0 + jj2], wst[cw0 + jj2 + 1], b0, b1);
                on[w] = b0 < b1;
              }
              f[w] = on[w] ? ld_cg_f4(src + (size_t)(cw0 + jj2) * piece_floats)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int w = 0; w < 4; ++w)
              if (on[w]) {
                v[0] += f[w].x;
                v[1] += f[w].y;
                v[2] += f[w].z;
                v[3] += f[w].w;
              }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (r0 + q >= it.rank) v[q] = 0.f;
        }
        uint32_t hi2[2], lo2[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * q], v[2 * q + 1]);
          const float2 hf = __bfloat1622float2(h2);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(v[2 * q] - hf.x, v[2 * q + 1] - hf.y);
          hi2[q] = *reinterpret_cast<const uint32_t*>(&h2);
          lo2[q] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        const size_t o = ((size_t)iq * n8 + t) * hst + r0;
        *reinterpret_cast<uint2*>(hhi + o) = make_uint2(hi2[0], hi2[1]);
        *reinterpret_cast<uint2*>(hlo + o) = make_uint2(lo2[0], lo2[1]);
      }
    }
    cp_async_wait<0>();
    __syncthreads();
    // y of every job: per slice, each warp takes 16-column tiles with all
    // their token tiles
    for (int k = 0; k < nj; ++k) {
      const int* J = jt + k * kJobInts;
      const int* P = pt + J[kJPiece] * kPieceInts;
      if (!P[kPOk]) continue;
      const Item it = item_of(meta, J[kJG]);
      const int j0 = J[kJJ0], j1 = J[kJJ1];
      const int cols = j1 - j0;
      const int ntt = ceil_div_i(it.n, 8);
      const int n8 = ntt * 8;
      const int pia = P[kPIa];
      int ia, ib;
      slice_span(p.slice_off, S, j0, j1, ia, ib);
      uint8_t* ys = ring + J[kJOff];
      const uint16_t* bs = reinterpret_cast<const uint16_t*>(p.b) + ((size_t)it.s * p.out + j0) * R;
      const uint16_t* hhi0 = reinterpret_cast<const uint16_t*>(ring + P[kPHoff]);
      const uint16_t* hlo0 = hhi0 + (size_t)(P[kPIb] - pia + 1) * n8 * hst;
      const uint32_t live = (uint32_t)P[kPLive];
      const float scal = __int_as_float(P[kPScal]);
      const int g4 = lane >> 2, c4 = lane & 3;
      for (int i = ia; i <= ib; ++i) {
        const int ls0 = max(j0, p.slice_off[i]) - j0, ls1 = min(j1, p.slice_off[i + 1]) - j0;
        const size_t ho = (size_t)(i - pia) * n8 * hst;
        const uint16_t* hhi = hhi0 + ho;
        const uint16_t* hlo = hlo0 + ho;
        switch (ntt) {
          case 1:
            expand_slice<1>(bs, hhi, hlo, hst, ys, cols * 2 + 16, R, it.rank, ls0, ls1, live, scal,
                            warp, g4, c4);
            break;
          case 2:
            expand_slice<2>(bs, hhi, hlo, hst, ys, cols * 2 + 16, R, it.rank, ls0, ls1, live, scal,
                            warp, g4, c4);
            break;
          case 3:
            expand_slice<3>(bs, hhi, hlo, hst, ys, cols * 2 + 16, R, it.rank, ls0, ls1, live, scal,
                            warp, g4, c4);
            break;
          default:
            expand_slice<4>(bs, hhi, hlo, hst, ys, cols * 2 + 16, R, it.rank, ls0, ls1, live, scal,
                            warp, g4, c4);
            break;
        }
      }
    }
    __syncthreads();
    // write the updated rows back: a warp per row, 16-byte stores
    int rows = 0;
    for (int k = 0; k < nj; ++k) rows += item_of(meta, jt[k * kJobInts + kJG]).n;
    for (int r = warp; r < rows; r += kSpWarps) {
      int k = 0, t = r;
      for (;;) {
        const int n = item_of(meta, jt[k * kJobInts + kJG]).n;
        if (t < n) break;
        t -= n;
        ++k;
      }
      const int* J = jt + k * kJobInts;
      const int* P = pt + J[kJPiece] * kPieceInts;
      if (!P[kPOk] || !(((uint32_t)P[kPLive] >> t) & 1u)) continue;
      const Item it = item_of(meta, J[kJG]);
      const int cols = J[kJJ1] - J[kJJ0];
      const uint4* src = reinterpret_cast<const uint4*>(ring + J[kJOff] + (size_t)t * (cols * 2 + 16));
      uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.y) +
                                            (size_t)tok[it.lo + it.tile * kTT + t] * p.out + J[kJJ0]);
      for (int q = lane; q < (cols >> 3); q += 32) dst[q] = src[q];
    }
    // the last expand piece of an item to finish resets its counters
    if (tid == 0) {
      for (int k = 0; k < nj; ++k) {
        const int* J = jt + k * kJobInts;
        const int* P = pt + J[kJPiece] * kPieceInts;
        if (J[kJLast] && P[kPCons] + 1 == P[kPNexp]) {
          p.cnt[J[kJG]] = 0u;
          p.cons[J[kJG]] = 0u;
        }
      }
    }
    __syncthreads();   // the round's staging and tables are free again
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------

namespace {

std::atomic<unsigned long long> g_wait_ns{0};

struct SplitCacheEntry {
  int dev, max_smem, sms, budget;
};
std::mutex g_split_mu;
SplitCacheEntry g_split_cache[64];
int g_split_n = 0;

}  // namespace

uint64_t set_wait_limit_ns(uint64_t ns) { return g_wait_ns.exchange(ns); }
uint64_t wait_limit_ns() {
  const unsigned long long v = g_wait_ns.load(std::memory_order_relaxed);
  return v == 0 ? kWaitLimitNs : v;
}

cudaError_t split_launch(const SplitParams& p_in, cudaStream_t stream, const char** why) {
  SplitParams p = p_in;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  SplitCacheEntry d = {-1, 0, 0, 0};
  {
    std::lock_guard<std::mutex> lk(g_split_mu);
    for (int i = 0; i < g_split_n; ++i)
      if (g_split_cache[i].dev == dev) d = g_split_cache[i];
  }
  if (d.dev < 0) {
    int per_sm = 0, reserved = 0;
    err = cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
    if (err == cudaSuccess)
      err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err == cudaSuccess)
      err = cudaFuncSetAttribute(bgmv_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 d.max_smem);
    if (err != cudaSuccess) return err;
    d.budget = per_sm / 2 - reserved;   // two CTAs per SM
    d.dev = dev;
    std::lock_guard<std::mutex> lk(g_split_mu);
    if (g_split_n < 64) g_split_cache[g_split_n++] = d;
  }
  p.ring = split_ring_bytes(p.T, p.item_cap, d.budget);
  p.wait_ns = wait_limit_ns();
  const SplitLayout L = split_layout(p.T, p.item_cap, p.ring);
  if (L.total > d.max_smem) {
    *why = "shared memory needed by the split kernel exceeds the device limit";
    return cudaErrorInvalidConfiguration;
  }
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)max(1, min(d.sms, kSpMaxGrid)), 1, 1);
  cfg.blockDim = dim3(kSpThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)L.total;
  cfg.stream = stream;
  if (launch_overlap_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, bgmv_split_kernel, p);
}

}  // namespace lora
