// Streamed expand in one launch over every SM: the embedding target (the
// kernel lora_apply_embedding runs in the STREAM regime) and the expand of a
// computed h (the grouped MoE fold's expand).
//
//   embedding  h[t, i*R + r] = a[slot, i*R + r, ids[t]]   (r < rank; 0 for an id outside [0, vocab))
//   computed   h[t, i*R + r] = sum over the partial buffers of h
//   expand     y[t, off_i + j] = bf16_rne(y + scaling[slot] * sum_r h[t, i*R + r] * b[slot, off_i + j, r])
//
// Sources: mstar.engine.resources.lora.backend, LoraBackend.gather_shrink (the
// one-hot shrink: a column of the slot's A per token id, nothing for an id
// outside the vocabulary), LoraBackend.expand_fused and apply_ with
// embedding=True (the expand over the slices of out_slices laid out in order
// as in mstar.model.components.linear, FusedColumnLinear);
// spark_model/lora/expert_apply.rs, apply_expert_lora_sorted (the MoE fold's
// expand over each (slot, expert) group of sorted rows).
//
// The work is the y read-modify-write: h is a few values per row and B of all
// slots stays in L2.  So the kernel is built around moving y at the HBM rate,
// with as few dependent memory round trips before the stream starts as the
// data allows:
//   * the positions of every slot (or group) that takes part are cut into
//     row groups of 16 (one MMA row tile) and the output columns into blocks
//     of W = 512 / ksteps columns within one slice; a unit is one (row group,
//     block) pair; the units, row group by row group, are split into equal
//     runs, one per CTA (one CTA per SM): the time a unit takes hardly depends
//     on how many of its 16 rows are live, so equal counts balance the CTAs,
//     and a row's h is read by one or two of them;
//   * a producer warp bulk-copies a B block (W x R bf16, contiguous) into a
//     ring of kStBBufs buffers whenever the (slot, block) changes; sixteen
//     consumer warps take a 32-column chunk of the block each and keep their
//     B fragments in registers while the block stays;
//   * each consumer thread owns 8 consecutive columns of two rows of a unit:
//     it loads them with one 16-byte load per row kStDepth units ahead (the y
//     stream stays in flight in registers: bulk copies of single rows are too
//     small to stream y at the HBM rate), runs m16n8k16 MMAs whose output
//     columns are permuted so that its accumulators land on exactly those
//     columns, and stores the 16 updated bytes of each row; a computed fp32 h
//     enters the MMAs as bf16 hi + lo (two MMAs, fp32 accumulate);
//   * the planning, the tokens and the first B block are read before the
//     wait on the preceding kernel (launch overlap); y, ids and h after it,
//     the first units' y in flight while h is gathered.
// Waits on the B buffers' mbarriers are bounded (LORA_FLAG_TIMEOUT).
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "expand_tile.cuh"
#include "kernels.h"

namespace lora {
namespace {

LORA_DEV void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kStConsumers * 32) : "memory");
}

// Waits for a phase with the kernel's limit; false if it ran out or the CTA
// has stopped (*abort set by another warp).
LORA_DEV bool ring_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns, const int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns || *(const volatile int*)abort) return false;
  }
  return true;
}

// Column block cb -> slice, first column (absolute) and width.
LORA_DEV void block_cols(const StreamParams& p, int cb, int& sl, int& c0, int& ncols) {
  int s = 0;
  while (s + 1 < p.S && cb >= p.block_off[s + 1]) ++s;
  const int j = cb - p.block_off[s];
  const int w = p.slice_off[s + 1] - p.slice_off[s];
  sl = s;
  c0 = p.slice_off[s] + j * p.W;
  ncols = (w - j * p.W) < p.W ? (w - j * p.W) : p.W;
}

// Sets the abort state after a wait that ran out (or after another warp's).
LORA_DEV bool ring_ok(bool ok, int lane, int* abort_ring, uint32_t* pre_flags) {
  ok = __all_sync(0xffffffffu, ok);
  if (!ok || *(volatile int*)abort_ring) {
    if (lane == 0) {
      atomicOr(pre_flags, LORA_FLAG_TIMEOUT);
      *(volatile int*)abort_ring = 1;
    }
    return false;
  }
  return true;
}

// kH: h is summed from partial buffers an earlier kernel wrote; otherwise it
// is gathered from a by token id.
template <int KS, bool kH>
__global__ void __launch_bounds__(kStThreads, 1)
    stream_kernel(const __grid_constant__ StreamParams p) {
  constexpr int Rp = KS * 16;
  constexpr int D = (KS >= 3 || (kH && KS >= 2)) ? 2 : kStDepth;   // wide h: fewer units in flight
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t pre_flags;
  __shared__ int abort_ring;

  uint64_t* bfull = reinterpret_cast<uint64_t*>(smem);
  uint64_t* bempty = bfull + kStBBufs;
  int* prefix = reinterpret_cast<int*>(smem + p.off_prefix);
  int4* segs = reinterpret_cast<int4*>(smem + p.off_segs);      // every slot's lo, hi, rank, scaling
  int* scratch = reinterpret_cast<int*>(smem + p.off_scratch);
  int* spec = reinterpret_cast<int*>(smem + p.off_spec);      // token_order read ahead
  int* ctok = reinterpret_cast<int*>(smem + p.off_ctok);      // tokens of the window
  int* cval = reinterpret_cast<int*>(smem + p.off_cval);      // token, or -1 (no h)
  int4* gmeta = reinterpret_cast<int4*>(smem + p.off_gmeta);  // slot, rank, scaling bits
  uint16_t* htab = reinterpret_cast<uint16_t*>(smem + p.off_htab);
  uint8_t* bbuf = smem + p.off_bbuf;
  const int SRp = p.S * Rp;
  uint16_t* hlo = htab + (size_t)p.gtab * kStRows * SRp;     // kH: the bf16 remainders

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    pre_flags = 0u;
    abort_ring = 0;
    for (int s = 0; s < kStBBufs; ++s) {
      mbar_init(bfull + s, 1);
      mbar_init(bempty + s, kStConsumers);
    }
    fence_mbar_init();
  }
  // token_order read ahead, next to the slot table: the positions this CTA
  // takes when every position is live (the common layout); others are read
  // when needed
  const long long spec_lo = (long long)p.T * blockIdx.x / gridDim.x;
  const long long spec_hi = (long long)p.T * (blockIdx.x + 1) / gridDim.x;
  const int nspec = (int)((spec_hi - spec_lo) < kStSpec ? (spec_hi - spec_lo) : kStSpec);
  constexpr int kSv = (kStSpec + kStThreads - 1) / kStThreads;
  int sv[kSv];
#pragma unroll
  for (int j = 0; j < kSv; ++j) {
    const int i = tid + j * kStThreads;
    sv[j] = i < nspec ? p.token_order[spec_lo + i] : -1;
  }
  // plan_linear synchronises the block before it reads or raises anything
  const int planned = plan_linear<kStThreads>(p.slot_indptr, p.ranks, p.scalings, p.slots, p.T,
                                              p.R, kStRows, prefix, scratch, &pre_flags,
                                              blockIdx.x == 0, p.seg_hi, segs);
#pragma unroll
  for (int j = 0; j < kSv; ++j) {
    const int i = tid + j * kStThreads;
    if (i < nspec) spec[i] = sv[j];
  }
  // Disjoint segments give at most ceil(T/16) + slots row groups; more means
  // that segments overlap (positions listed twice: the result is
  // unspecified), and the surplus is dropped so that every count below stays
  // in range.
  const long long gmax = ((long long)p.T + kStRows - 1) / kStRows + p.slots;
  const long long ng = (planned < 0 || planned > gmax) ? gmax : planned;
  // this CTA's run of units u = row_group * nblocks + block
  const long long nu_all = ng * p.nblocks;
  const long long u_lo = nu_all * blockIdx.x / gridDim.x;
  const long long u_hi = nu_all * (blockIdx.x + 1) / gridDim.x;
  grid_dep_launch_dependents();
  __syncthreads();

  uint8_t* Y = static_cast<uint8_t*>(p.y);
  const uint16_t* A = static_cast<const uint16_t*>(p.a);
  const uint8_t* B = static_cast<const uint8_t*>(p.b);
  const int SR = p.S * p.R;
  const int nb = p.nblocks;

  uint32_t bc = 0;                     // B blocks loaded (each role counts)
  int bkey_slot = -1, bkey_blk = -1;   // the B block in use (each role tracks it)
  bool waited = false;

  // consumer lanes: warp cw takes chunk cw (columns 32*cw ..) of every block
  const int cw = warp - 1;
  const int g8 = lane >> 2;
  const int q = lane & 3;
  const int cc = cw * 32 + 8 * q;       // this thread's 8 columns within a block
  // this lane's B row in the chunk for MMA n-tile jj is brow + 2*jj: output
  // column n of each MMA is chunk column 8*(n/2) + 2*jj + n%2, so the
  // accumulators of thread q land on its own columns 8q + 2*jj + {0, 1}
  const int brow = cw * 32 + 8 * (g8 >> 1) + (g8 & 1);
  uint2 bfr[4][KS];                    // B fragments of the block in use (consumers)

  const long long g_first = u_lo < u_hi ? u_lo / nb : 0;
  const long long g_end = u_lo < u_hi ? (u_hi - 1) / nb + 1 : 0;
  for (long long gw0 = g_first; gw0 < g_end; gw0 += p.gtab) {
    const int ngw = (int)((g_end - gw0) < p.gtab ? (g_end - gw0) : p.gtab);
    const int nrows = ngw * kStRows;
    // the window's units [wu0, wu1), row group by row group
    const long long wu0 = u_lo > gw0 * nb ? u_lo : gw0 * nb;
    const long long wu1 = u_hi < (gw0 + ngw) * nb ? u_hi : (gw0 + ngw) * nb;
    const int nu = (int)(wu1 - wu0);
    const int gi0 = (int)(wu0 / nb - gw0);
    const int cb0 = (int)(wu0 % nb);

    // --- the window's tokens (addressing only: before the preceding kernel ends)
    for (int e = tid; e < nrows; e += kStThreads) {
      const int g = (int)(gw0 + e / kStRows);
      const int i = e % kStRows;
      const int s = find_segment(prefix, p.slots, g);
      const int4 sg = segs[s];
      const long long lo = sg.x;
      const long long hi = sg.y;
      const long long pos = lo + (long long)(g - prefix[s]) * kStRows + i;
      int tok = -1;
      if (pos >= lo && pos < hi) {
        tok = (pos >= spec_lo && pos < spec_lo + nspec) ? spec[pos - spec_lo]
                                                        : p.token_order[pos];
        if (tok < 0 || tok >= p.T) {
          atomicOr(&pre_flags, LORA_FLAG_BAD_TOKEN);
          tok = -1;
        }
      }
      ctok[e] = tok;
      if (i == 0)
        gmeta[e / kStRows] = make_int4(s, sg.z, sg.w, 0);
    }
    __syncthreads();

    if (!waited) {
      // the first B block is an input: start it before the preceding kernel ends
      if (warp == 0) {
        const int slot0 = gmeta[gi0].x;
        if (lane == 0) {
          int sl, c0, ncols;
          block_cols(p, cb0, sl, c0, ncols);
          const uint32_t bb = (uint32_t)ncols * p.R * 2;
          const int pair = p.slot_map != nullptr ? p.slot_map[slot0] : slot0;
          mbar_arrive_expect_tx(bfull, bb);
          bulk_g2s(bbuf, B + ((size_t)pair * p.out + c0) * p.R * 2, bb, bfull);
        }
        bkey_slot = slot0;
        bkey_blk = cb0;
        bc = 1;
      }
      grid_dep_wait();
      waited = true;
    }

    if (warp == 0) {
      // ---------------------------------------------------------- producer
      int gi = gi0, cb = cb0;
      for (int u = 0; u < nu; ++u) {
        const int slot = gmeta[gi].x;
        if (slot != bkey_slot || cb != bkey_blk) {
          int sl, c0, ncols;
          block_cols(p, cb, sl, c0, ncols);
          // a new B block into the next buffer, once the consumers let it go
          const int nbuf = (int)(bc % kStBBufs);
          const uint32_t kb = bc / kStBBufs;
          const bool ok =
              kb > 0 ? ring_wait(bempty + nbuf, (kb - 1) & 1u, p.wait_ns, &abort_ring) : true;
          if (!ring_ok(ok, lane, &abort_ring, &pre_flags)) break;
          if (lane == 0) {
            const uint32_t bb = (uint32_t)ncols * p.R * 2;
            const int pair = p.slot_map != nullptr ? p.slot_map[slot] : slot;
            mbar_arrive_expect_tx(bfull + nbuf, bb);
            bulk_g2s(bbuf + (size_t)nbuf * p.bbytes, B + ((size_t)pair * p.out + c0) * p.R * 2,
                     bb, bfull + nbuf);
          }
          bkey_slot = slot;
          bkey_blk = cb;
          ++bc;
        }
        if (++cb == nb) {
          cb = 0;
          ++gi;
        }
      }
    } else {
      // ---------------------------------------------------------- consumers
      // units in order: row group by row group, the blocks inside each group.
      // y of unit u + D is requested while unit u is computed.
      uint4 ya[D], yb[D];
      int icb = cb0, igi = gi0, ireq = 0;  // next unit to request
      auto request = [&](uint4& ra, uint4& rb) {
        ra = rb = make_uint4(0u, 0u, 0u, 0u);
        if (ireq >= nu) return;
        ++ireq;
        int sl, c0, ncols;
        block_cols(p, icb, sl, c0, ncols);
        if (cc < ncols) {
          // a gathered h's rows are known once the ids are in (an id outside
          // the vocabulary leaves its row alone: it is not read)
          const int* rt = kH ? ctok : cval;
          const int tA = rt[igi * kStRows + g8];
          const int tB = rt[igi * kStRows + g8 + 8];
          if (tA >= 0) ra = *reinterpret_cast<const uint4*>(Y + ((size_t)tA * p.out + c0 + cc) * 2);
          if (tB >= 0) rb = *reinterpret_cast<const uint4*>(Y + ((size_t)tB * p.out + c0 + cc) * 2);
        }
        if (++icb == nb) {
          icb = 0;
          ++igi;
        }
      };
      // a computed h (L2-resident partials) is summed while the first units'
      // y is on its way; the ids and A columns of a gathered h go out first,
      // ahead of the y stream in the DRAM queues, and y follows them (the
      // two dependent loads took 3.8 us behind the y stream)
      if (kH) {
#pragma unroll
        for (int j = 0; j < D; ++j) request(ya[j], yb[j]);
      }

      const int ct = tid - 32;
      // h of the window's rows, every slice (zeros past the rank and for rows
      // without h)
      const int ncolh = SRp;
      const int nel = nrows * ncolh;
      if (kH) {
        // the sum of the partials in chunk order; two elements a thread and
        // up to eight partials each in flight at once
        constexpr int kStride = kStConsumers * 32;
        for (int e0 = ct; e0 < nel; e0 += 2 * kStride) {
          const float* hp[2];
          int hrow[2], hcol[2];
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int e = e0 + k * kStride;
            hp[k] = nullptr;
            hrow[k] = -1;
            hcol[k] = 0;
            if (e < nel) {
              const int row = e / ncolh;
              const int c = e - row * ncolh;
              const int sl = c / Rp;
              const int r = c % Rp;
              const int tok = ctok[row];
              hrow[k] = row;
              hcol[k] = sl * Rp + r;
              if (tok >= 0 && r < gmeta[row / kStRows].y)
                hp[k] = p.h + (size_t)tok * SR + sl * p.R + r;
              if (c == 0) cval[row] = tok;
            }
          }
          float v[2] = {0.0f, 0.0f};
          for (int k0 = 0; k0 < p.ksplit; k0 += 8) {
            float t[2][8];
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                t[k][j] = (hp[k] != nullptr && k0 + j < p.ksplit)
                              ? __ldcg(hp[k] + (size_t)(k0 + j) * p.h_split)
                              : 0.0f;
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
              for (int j = 0; j < 8; ++j)
                if (k0 + j < p.ksplit) v[k] += t[k][j];
          }
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            if (hrow[k] < 0) continue;
            const __nv_bfloat16 hi = __float2bfloat16_rn(v[k]);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v[k] - __bfloat162float(hi));
            htab[(size_t)hrow[k] * SRp + hcol[k]] = *reinterpret_cast<const uint16_t*>(&hi);
            hlo[(size_t)hrow[k] * SRp + hcol[k]] = *reinterpret_cast<const uint16_t*>(&lo);
          }
        }
      } else {
        for (int e = ct; e < nel; e += kStConsumers * 32) {
          const int row = e / ncolh;
          const int c = e - row * ncolh;
          const int sl = c / Rp;
          const int r = c % Rp;
          const int4 gm = gmeta[row / kStRows];
          const int tok = ctok[row];
          uint16_t v = 0;
          bool valid = false;
          if (tok >= 0) {
            const int id = p.ids[tok];
            valid = id >= 0 && id < p.vocab;
            if (valid && r < gm.y)
              v = A[((size_t)gm.x * p.S * p.R + (size_t)sl * p.R + r) * (size_t)p.vocab + id];
          }
          htab[(size_t)row * SRp + sl * Rp + r] = v;
          if (c == 0) cval[row] = valid ? tok : -1;
        }
      }
      consumer_sync();
      if (!kH) {
#pragma unroll
        for (int j = 0; j < D; ++j) request(ya[j], yb[j]);
      }

      int pcb = cb0, pgi = gi0;            // unit being computed
      bool stop = false;
      for (int u0 = 0; u0 < nu && !stop; u0 += D) {
#pragma unroll
        for (int j = 0; j < D; ++j) {
          if (u0 + j >= nu) break;
          int sl, c0, ncols;
          block_cols(p, pcb, sl, c0, ncols);
          const int4 gm = gmeta[pgi];
          if (gm.x != bkey_slot || pcb != bkey_blk) {
            // the next B block: its fragments into registers, then free the buffer
            const int nb = (int)(bc % kStBBufs);
            const uint32_t kb = bc / kStBBufs;
            if (!ring_ok(ring_wait(bfull + nb, kb & 1u, p.wait_ns, &abort_ring), lane, &abort_ring,
                         &pre_flags)) {
              stop = true;
              break;
            }
            const uint8_t* bs = bbuf + (size_t)nb * p.bbytes;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const int nc = brow + 2 * jj;
#pragma unroll
              for (int ks = 0; ks < KS; ++ks) {
                const int k0 = ks * 16 + 4 * q;
                uint2 v = make_uint2(0u, 0u);
                if (nc < ncols && k0 < p.R) {
                  v = *reinterpret_cast<const uint2*>(bs + ((size_t)nc * p.R + k0) * 2);
                  const uint2 m = rank_mask4(k0, gm.y);
                  v.x &= m.x;
                  v.y &= m.y;
                }
                bfr[jj][ks] = v;
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bempty + nb);
            bkey_slot = gm.x;
            bkey_blk = pcb;
            ++bc;
          }
          const bool cv = cc < ncols;
          const int rowA = pgi * kStRows + g8;
          const int tokA = cval[rowA];
          const int tokB = cval[rowA + 8];
          // the MMAs take every lane of the warp: skip only when no lane has columns
          if (__any_sync(0xffffffffu, cv)) {
            // h fragments; the k index is permuted (thread q holds k = 4q..4q+3
            // of each k-step) identically in h and B, which leaves the sum
            // unchanged
            uint2 hA[KS], hB[KS];
            const size_t hoff = (size_t)rowA * SRp + sl * Rp + 4 * q;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              hA[ks] = *reinterpret_cast<const uint2*>(htab + hoff + ks * 16);
              hB[ks] = *reinterpret_cast<const uint2*>(htab + hoff + 8 * SRp + ks * 16);
            }
            float d[4][4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
              for (int e = 0; e < 4; ++e) d[jj][e] = 0.f;
#pragma unroll
              for (int ks = 0; ks < KS; ++ks)
                mma_bf16_16816(d[jj], hA[ks].x, hB[ks].x, hA[ks].y, hB[ks].y, bfr[jj][ks].x,
                               bfr[jj][ks].y);
            }
            if (kH) {
#pragma unroll
              for (int ks = 0; ks < KS; ++ks) {
                hA[ks] = *reinterpret_cast<const uint2*>(hlo + hoff + ks * 16);
                hB[ks] = *reinterpret_cast<const uint2*>(hlo + hoff + 8 * SRp + ks * 16);
              }
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
                for (int ks = 0; ks < KS; ++ks)
                  mma_bf16_16816(d[jj], hA[ks].x, hB[ks].x, hA[ks].y, hB[ks].y, bfr[jj][ks].x,
                                 bfr[jj][ks].y);
              }
            }
            const float scal = __int_as_float(gm.z);
            const uint32_t yav[4] = {ya[j].x, ya[j].y, ya[j].z, ya[j].w};
            const uint32_t ybv[4] = {yb[j].x, yb[j].y, yb[j].z, yb[j].w};
            uint32_t oa[4], ob[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              oa[jj] = pack_bf16x2(fmaf(scal, d[jj][0], bf16_lo(yav[jj])),
                                   fmaf(scal, d[jj][1], bf16_hi(yav[jj])));
              ob[jj] = pack_bf16x2(fmaf(scal, d[jj][2], bf16_lo(ybv[jj])),
                                   fmaf(scal, d[jj][3], bf16_hi(ybv[jj])));
            }
            if (cv && tokA >= 0)
              *reinterpret_cast<uint4*>(Y + ((size_t)tokA * p.out + c0 + cc) * 2) =
                  make_uint4(oa[0], oa[1], oa[2], oa[3]);
            if (cv && tokB >= 0)
              *reinterpret_cast<uint4*>(Y + ((size_t)tokB * p.out + c0 + cc) * 2) =
                  make_uint4(ob[0], ob[1], ob[2], ob[3]);
          }
          if (++pcb == nb) {
            pcb = 0;
            ++pgi;
          }
          request(ya[j], yb[j]);     // unit u0 + j + D
        }
      }
    }
    __syncthreads();   // the window's units are done before its tables change
    if (*(volatile int*)&abort_ring) break;
  }
  if (!waited) grid_dep_wait();
  __syncthreads();
  if (tid == 0) raise_flag(p.flags, pre_flags);
}

struct StreamDev {
  int dev;
  int sms;
  int max_smem;
  unsigned attr_set;   // bit i: the shared-memory limit of kernel variant i is raised
};
std::mutex g_stream_mu;
StreamDev g_stream_dev[64];
int g_stream_n = 0;

template <int KS, bool kH>
cudaError_t launch_variant(const StreamParams& p, int grid, bool overlap, cudaStream_t stream,
                           bool raise_only, int smem_limit) {
  if (raise_only)
    return cudaFuncSetAttribute(stream_kernel<KS, kH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                smem_limit);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kStThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)p.smem;
  cfg.stream = stream;
  if (overlap) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, stream_kernel<KS, kH>, p);
}

// The kernel variant of (KS, kh): launched, or (raise_only) its shared-memory
// limit raised.
cudaError_t dispatch(int KS, bool kh, const StreamParams& p, int grid, bool overlap,
                     cudaStream_t stream, bool raise_only, int smem_limit) {
  switch (KS) {
    case 1: return kh ? launch_variant<1, true>(p, grid, overlap, stream, raise_only, smem_limit)
                      : launch_variant<1, false>(p, grid, overlap, stream, raise_only, smem_limit);
    case 2: return kh ? launch_variant<2, true>(p, grid, overlap, stream, raise_only, smem_limit)
                      : launch_variant<2, false>(p, grid, overlap, stream, raise_only, smem_limit);
    case 3: return kh ? launch_variant<3, true>(p, grid, overlap, stream, raise_only, smem_limit)
                      : launch_variant<3, false>(p, grid, overlap, stream, raise_only, smem_limit);
    default: return kh ? launch_variant<4, true>(p, grid, overlap, stream, raise_only, smem_limit)
                       : launch_variant<4, false>(p, grid, overlap, stream, raise_only, smem_limit);
  }
}

}  // namespace

cudaError_t stream_launch(StreamParams& p, cudaStream_t stream, bool allow_overlap,
                          const char** why) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int KS = round_up_i(p.R, 16) / 16;
  const bool kh = p.h != nullptr;
  const unsigned bit = 1u << ((KS - 1) * 2 + (kh ? 1 : 0));
  StreamDev d = {-1, 0, 0, 0u};
  int slot = -1;
  {
    std::lock_guard<std::mutex> lk(g_stream_mu);
    for (int i = 0; i < g_stream_n; ++i)
      if (g_stream_dev[i].dev == dev) {
        d = g_stream_dev[i];
        slot = i;
      }
  }
  if (d.dev < 0) {
    err = cudaDeviceGetAttribute(&d.max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    // the dynamic part: what the block may hold beyond the kernel's two static
    // variables (256 bytes kept for them)
    d.max_smem -= 256;
    d.dev = dev;
  }
  if (!(d.attr_set & bit)) {
    err = dispatch(KS, kh, p, 0, false, stream, true, d.max_smem);
    if (err != cudaSuccess) return err;
    d.attr_set |= bit;
    std::lock_guard<std::mutex> lk(g_stream_mu);
    if (slot >= 0) {
      g_stream_dev[slot] = d;
    } else if (g_stream_n < 64) {
      g_stream_dev[g_stream_n++] = d;
    }
  }

  const int Rp = KS * 16;
  p.W = KS == 1 ? 512 : KS == 2 ? 256 : 128;
  p.bbytes = round_up_i(p.W * p.R * 2, 128);
  p.block_off[0] = 0;
  for (int i = 0; i < p.S; ++i)
    p.block_off[i + 1] = p.block_off[i] + ceil_div_i(p.slice_off[i + 1] - p.slice_off[i], p.W);
  for (int i = p.S + 1; i <= LORA_MAX_SLICES; ++i) p.block_off[i] = p.block_off[p.S];
  p.nblocks = p.block_off[p.S];

  const int grid = d.sms;
  // row groups one CTA's run touches with disjoint segments: one window if
  // they fit
  const long long gmax = ((long long)p.T + kStRows - 1) / kStRows + p.slots;
  const long long per_cta = (gmax * p.nblocks + grid - 1) / grid / p.nblocks + 2;
  const long long share = ((long long)p.T + grid - 1) / grid;
  const int nspec = (int)(share < kStSpec ? share : kStSpec);

  // shared memory: barriers, the group prefix, scan scratch, the tokens read
  // ahead, tables (h twice when computed), B buffers
  int off = 2 * kStBBufs * 8;
  p.off_prefix = off;
  off += round_up_i((p.slots + 1) * 4, 16);
  p.off_segs = round_up_i(off, 16);
  off = p.off_segs + p.slots * 16;
  p.off_scratch = off;
  off += round_up_i(kStThreads / 32 * 4, 16);
  p.off_spec = off;
  off += round_up_i(nspec * 4, 16);
  // the tables take what is left beside the B buffers, at most kStMaxGroups
  const int per_group = kStRows * 4 * 2 + 16 + (kh ? 2 : 1) * kStRows * p.S * Rp * 2;
  const int room = d.max_smem - off - 64 - 128 - kStBBufs * p.bbytes;
  long long gt = per_cta < kStMaxGroups ? per_cta : kStMaxGroups;
  if (room / per_group < gt) gt = room / per_group;
  if (gt < 1) {
    *why = "shared memory of the streamed expand exceeds the device limit";
    return cudaErrorInvalidConfiguration;
  }
  p.gtab = (int)gt;
  p.off_ctok = off;
  off += p.gtab * kStRows * 4;
  p.off_cval = off;
  off += p.gtab * kStRows * 4;
  p.off_gmeta = round_up_i(off, 16);
  off = p.off_gmeta + p.gtab * 16;
  p.off_htab = round_up_i(off, 16);
  off = p.off_htab + (kh ? 2 : 1) * p.gtab * kStRows * p.S * Rp * 2;
  p.off_bbuf = round_up_i(off, 128);
  p.smem = p.off_bbuf + kStBBufs * p.bbytes;
  if (p.smem > d.max_smem) {
    *why = "shared memory of the streamed expand exceeds the device limit";
    return cudaErrorInvalidConfiguration;
  }
  p.wait_ns = wait_limit_ns();
  const bool overlap = allow_overlap && launch_overlap_enabled();

  return dispatch(KS, kh, p, grid, overlap, stream, false, 0);
}

}  // namespace lora
