// Embedding target (gather, then expand) in one launch over every SM: the
// kernel lora_apply_embedding runs in the STREAM regime.
//
//   h[t, i*R + r] = a[slot, i*R + r, ids[t]]        (r < rank; 0 for an id outside [0, vocab))
//   y[t, off_i + j] = bf16_rne(y + scaling[slot] * sum_r h[t, i*R + r] * b[slot, off_i + j, r])
//
// Sources: mstar.engine.resources.lora.backend, LoraBackend.gather_shrink (the
// one-hot shrink: a column of the slot's A per token id, nothing for an id
// outside the vocabulary) and LoraBackend.apply_ with embedding=True (the
// gathered h goes through the fused expand of expand_fused, over the slices
// of out_slices laid out in order as in mstar.model.components.linear,
// FusedColumnLinear).
//
// The work is the y read-modify-write: h is R bf16 values per token (exact:
// they are elements of A) and B of all slots stays in L2.  So the kernel is
// built around moving y at the HBM rate, with as few dependent memory round
// trips before the stream starts as the data allows:
//   * the output columns are cut into blocks of W = 512 / ksteps columns
//     within one slice and the token positions into equal shares; CTA c takes
//     block run c % bsplit and position share c / bsplit, so every CTA moves
//     the same number of y bytes and a token's h is gathered by bsplit CTAs;
//   * a CTA reads its share of token_order at once, next to the slot table,
//     clips every live slot's segment to the share and cuts it into groups of
//     16 positions (one MMA row tile); a unit is one (block, group) pair and
//     the CTA walks its units block by block;
//   * a producer warp bulk-copies a B block (W x R bf16, contiguous) into a
//     ring of kStBBufs buffers whenever the (slot, block) changes; sixteen
//     consumer warps take a 32-column chunk of the block each and keep their
//     B fragments in registers while the block stays;
//   * each consumer thread owns 8 consecutive columns of two rows of a unit:
//     it loads them with one 16-byte load per row kStDepth units ahead (the y
//     stream stays in flight in registers: bulk copies of single rows are too
//     small to stream y at the HBM rate), runs m16n8k16 MMAs whose output
//     columns are permuted so that its accumulators land on exactly those
//     columns, and stores the 16 updated bytes of each row;
//   * the planning, the tokens and the first B block are read before the
//     wait on the preceding kernel (launch overlap); y, ids and h after it,
//     the first units' y in flight while the ids and h are gathered.
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

// Waits for a phase with the kernel's limit; false if it ran out.
LORA_DEV bool ring_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
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

// The groups of one position share [plo, phi): slot s takes part when its
// segment is valid (0 <= lo <= hi <= T), its rank is in (0, R] and its scaling
// nonzero; its segment clipped to the share is cut into groups of kStRows.
// Writes prefix[0..slots] (exclusive prefix of group counts) to shared memory
// and returns the total.  Flags of bad segments and ranks are raised when
// `report` is set.
template <int NT>
LORA_DEV int plan_share(const int* __restrict__ slot_indptr, const int* __restrict__ ranks,
                        const float* __restrict__ scalings, int slots, int T, int R,
                        long long plo, long long phi, int* prefix, int* scratch,
                        uint32_t* flags, bool report) {
  uint32_t bad = 0;
  int carry = 0;
  if (threadIdx.x == 0) prefix[0] = 0;
  for (int base = 0; base < slots; base += NT) {
    const int s = base + threadIdx.x;
    int cnt = 0;
    if (s < slots) {
      const int lo = slot_indptr[s];
      const int hi = slot_indptr[s + 1];
      const int r = ranks[s];
      const bool seg_ok = lo >= 0 && lo <= hi && hi <= T;
      const bool rank_ok = r >= 0 && r <= R;
      if (!seg_ok) bad |= LORA_FLAG_BAD_INDPTR;
      if (!rank_ok) bad |= LORA_FLAG_BAD_RANK;
      if (seg_ok && rank_ok && r > 0 && scalings[s] != 0.0f) {
        const long long a = lo > plo ? lo : plo;
        const long long b = hi < phi ? hi : phi;
        if (b > a) cnt = (int)((b - a + kStRows - 1) / kStRows);
      }
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

template <int KS>
__global__ void __launch_bounds__(kStThreads, 1)
    stream_embed_kernel(const __grid_constant__ StreamParams p) {
  constexpr int Rp = KS * 16;
  constexpr int D = KS >= 3 ? 2 : kStDepth;   // wide ranks: fewer units in flight
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t pre_flags;
  __shared__ int abort_ring;

  uint64_t* bfull = reinterpret_cast<uint64_t*>(smem);
  uint64_t* bempty = bfull + kStBBufs;
  int* prefix = reinterpret_cast<int*>(smem + p.off_prefix);
  int* scratch = reinterpret_cast<int*>(smem + p.off_scratch);
  int* spec = reinterpret_cast<int*>(smem + p.off_spec);      // the share's token_order
  int* ctok = reinterpret_cast<int*>(smem + p.off_ctok);      // tokens of the window
  int* cval = reinterpret_cast<int*>(smem + p.off_cval);      // token, or -1 (id outside)
  int4* gmeta = reinterpret_cast<int4*>(smem + p.off_gmeta);  // slot, rank, scaling bits
  uint16_t* htab = reinterpret_cast<uint16_t*>(smem + p.off_htab);
  uint8_t* bbuf = smem + p.off_bbuf;
  const int SRp = p.S * Rp;

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
  // this CTA's rectangle: blocks [b0, b1) x positions [plo, phi)
  const int bsi = (int)(blockIdx.x % (unsigned)p.bsplit);
  const int gsi = (int)(blockIdx.x / (unsigned)p.bsplit);
  const int gsplit = (int)(gridDim.x / (unsigned)p.bsplit);
  const int b0 = p.nblocks * bsi / p.bsplit;
  const int b1 = p.nblocks * (bsi + 1) / p.bsplit;
  const long long plo = (long long)p.T * gsi / gsplit;
  const long long phi = (long long)p.T * (gsi + 1) / gsplit;
  const int nshare = (int)(phi - plo);
  const bool spec_ok = nshare <= kStSpec;
  // the share's token_order, read next to the slot table (both addressing)
  constexpr int kSv = (kStSpec + kStThreads - 1) / kStThreads;
  int sv[kSv];
#pragma unroll
  for (int j = 0; j < kSv; ++j) {
    const int i = tid + j * kStThreads;
    sv[j] = (spec_ok && i < nshare) ? p.token_order[plo + i] : -1;
  }
  // plan_share synchronises the block before it reads or raises anything
  const int planned = plan_share<kStThreads>(p.slot_indptr, p.ranks, p.scalings, p.slots, p.T,
                                             p.R, plo, phi, prefix, scratch, &pre_flags,
                                             blockIdx.x == 0);
#pragma unroll
  for (int j = 0; j < kSv; ++j) {
    const int i = tid + j * kStThreads;
    if (spec_ok && i < nshare) spec[i] = sv[j];
  }
  // Disjoint segments give at most ceil(share/16) + slots groups; more means
  // that segments overlap (tokens listed twice: the result is unspecified),
  // and the surplus is dropped so that every count below stays in range.
  const long long gcap = ((long long)nshare + kStRows - 1) / kStRows + p.slots;
  const long long ng = (planned < 0 || planned > gcap) ? gcap : planned;
  grid_dep_launch_dependents();
  __syncthreads();

  uint8_t* Y = static_cast<uint8_t*>(p.y);
  const uint16_t* A = static_cast<const uint16_t*>(p.a);
  const uint8_t* B = static_cast<const uint8_t*>(p.b);
  // slices the CTA's blocks fall in: its h is gathered for those only
  int sl_lo = 0, sl_hi = 0;
  if (b1 > b0) {
    while (sl_lo + 1 < p.S && b0 >= p.block_off[sl_lo + 1]) ++sl_lo;
    sl_hi = sl_lo;
    while (sl_hi + 1 < p.S && b1 - 1 >= p.block_off[sl_hi + 1]) ++sl_hi;
  }

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

  for (long long gw0 = 0; gw0 < ng && b1 > b0; gw0 += p.gtab) {
    const int ngw = (int)((ng - gw0) < p.gtab ? (ng - gw0) : p.gtab);
    const int nrows = ngw * kStRows;

    // --- the window's tokens (addressing only: before the preceding kernel ends)
    for (int e = tid; e < nrows; e += kStThreads) {
      const int g = (int)(gw0 + e / kStRows);
      const int i = e % kStRows;
      const int s = find_segment(prefix, p.slots, g);
      const int lo = p.slot_indptr[s];
      const int hi = p.slot_indptr[s + 1];
      const long long a = lo > plo ? lo : plo;
      const long long b = hi < phi ? hi : phi;
      const long long pos = a + (long long)(g - prefix[s]) * kStRows + i;
      int tok = -1;
      if (pos >= a && pos < b) {
        tok = spec_ok ? spec[pos - plo] : p.token_order[pos];
        if (tok < 0 || tok >= p.T) {
          atomicOr(&pre_flags, LORA_FLAG_BAD_TOKEN);
          tok = -1;
        }
      }
      ctok[e] = tok;
      if (i == 0)
        gmeta[e / kStRows] = make_int4(s, p.ranks[s], __float_as_int(p.scalings[s]), 0);
    }
    __syncthreads();

    if (!waited) {
      // the first B block is an input: start it before the preceding kernel ends
      if (warp == 0) {
        const int slot0 = gmeta[0].x;
        if (lane == 0) {
          int sl, c0, ncols;
          block_cols(p, b0, sl, c0, ncols);
          const uint32_t bb = (uint32_t)ncols * p.R * 2;
          mbar_arrive_expect_tx(bfull, bb);
          bulk_g2s(bbuf, B + ((size_t)slot0 * p.out + c0) * p.R * 2, bb, bfull);
        }
        bkey_slot = slot0;
        bkey_blk = b0;
        bc = 1;
      }
      grid_dep_wait();
      waited = true;
    }

    if (warp == 0) {
      // ---------------------------------------------------------- producer
      bool stop = false;
      for (int cb = b0; cb < b1 && !stop; ++cb) {
        int sl, c0, ncols;
        block_cols(p, cb, sl, c0, ncols);
        for (int gi = 0; gi < ngw; ++gi) {
          const int slot = gmeta[gi].x;
          if (slot == bkey_slot && cb == bkey_blk) continue;
          // a new B block into the next buffer, once the consumers let it go
          const int nb = (int)(bc % kStBBufs);
          const uint32_t kb = bc / kStBBufs;
          const bool ok = kb > 0 ? ring_wait(bempty + nb, (kb - 1) & 1u, p.wait_ns) : true;
          if (!ring_ok(ok, lane, &abort_ring, &pre_flags)) {
            stop = true;
            break;
          }
          if (lane == 0) {
            const uint32_t bb = (uint32_t)ncols * p.R * 2;
            mbar_arrive_expect_tx(bfull + nb, bb);
            bulk_g2s(bbuf + (size_t)nb * p.bbytes, B + ((size_t)slot * p.out + c0) * p.R * 2, bb,
                     bfull + nb);
          }
          bkey_slot = slot;
          bkey_blk = cb;
          ++bc;
        }
      }
    } else {
      // ---------------------------------------------------------- consumers
      // units in order: block by block, the window's groups inside each block.
      // y of unit u + D is requested while unit u is computed; the first D
      // units' y goes out before the ids are known (a row whose id turns out
      // to be outside the vocabulary is read and left alone).
      const int nu = (b1 - b0) * ngw;
      uint4 ya[D], yb[D];
      int icb = b0, igi = 0;               // next unit to request
      auto request = [&](uint4& ra, uint4& rb) {
        ra = rb = make_uint4(0u, 0u, 0u, 0u);
        if (icb >= b1) return;
        int sl, c0, ncols;
        block_cols(p, icb, sl, c0, ncols);
        if (cc < ncols) {
          const int tA = ctok[igi * kStRows + g8];
          const int tB = ctok[igi * kStRows + g8 + 8];
          if (tA >= 0) ra = *reinterpret_cast<const uint4*>(Y + ((size_t)tA * p.out + c0 + cc) * 2);
          if (tB >= 0) rb = *reinterpret_cast<const uint4*>(Y + ((size_t)tB * p.out + c0 + cc) * 2);
        }
        if (++igi == ngw) {
          igi = 0;
          ++icb;
        }
      };
#pragma unroll
      for (int j = 0; j < D; ++j) request(ya[j], yb[j]);

      const int ct = tid - 32;
      // the rows' ids, then h for the slices of the CTA's blocks (zeros past
      // the rank and for rows without a valid id)
      const int ncolh = (sl_hi - sl_lo + 1) * Rp;
      for (int e = ct; e < nrows * ncolh; e += kStConsumers * 32) {
        const int row = e / ncolh;
        const int c = e - row * ncolh;
        const int sl = sl_lo + c / Rp;
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
      consumer_sync();

      int pcb = b0, pgi = 0;               // unit being computed
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
            if (!ring_ok(ring_wait(bfull + nb, kb & 1u, p.wait_ns), lane, &abort_ring,
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
            const uint16_t* hrow = htab + (size_t)rowA * SRp + sl * Rp + 4 * q;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              hA[ks] = *reinterpret_cast<const uint2*>(hrow + ks * 16);
              hB[ks] = *reinterpret_cast<const uint2*>(hrow + 8 * SRp + ks * 16);
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
          if (++pgi == ngw) {
            pgi = 0;
            ++pcb;
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
  unsigned attr_set;   // bit KS-1: the kernel's shared-memory limit is raised
};
std::mutex g_stream_mu;
StreamDev g_stream_dev[64];
int g_stream_n = 0;

template <int KS>
cudaError_t launch_ks(const StreamParams& p, int grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kStThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)p.smem;
  cfg.stream = stream;
  if (launch_overlap_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, stream_embed_kernel<KS>, p);
}

template <int KS>
cudaError_t raise_smem_limit(int bytes) {
  return cudaFuncSetAttribute(stream_embed_kernel<KS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              bytes);
}

}  // namespace

cudaError_t stream_embed_launch(StreamParams& p, cudaStream_t stream, const char** why) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const int KS = round_up_i(p.R, 16) / 16;
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
  if (!(d.attr_set & (1u << (KS - 1)))) {
    switch (KS) {
      case 1: err = raise_smem_limit<1>(d.max_smem); break;
      case 2: err = raise_smem_limit<2>(d.max_smem); break;
      case 3: err = raise_smem_limit<3>(d.max_smem); break;
      default: err = raise_smem_limit<4>(d.max_smem); break;
    }
    if (err != cudaSuccess) return err;
    d.attr_set |= 1u << (KS - 1);
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
  // Two block runs when there are blocks enough and the grid is even (each
  // token's h is then gathered by two CTAs), else one.
  p.bsplit = (p.nblocks >= 4 && grid % 2 == 0) ? 2 : 1;
  const int gsplit = grid / p.bsplit;
  // groups of one share with disjoint segments: one window if they fit
  const long long share = ((long long)p.T + gsplit - 1) / gsplit;
  const long long per_cta = (share + kStRows - 1) / kStRows + p.slots;
  p.gtab = (int)(per_cta < kStMaxGroups ? per_cta : kStMaxGroups);
  const int nspec = (int)(share < kStSpec ? share : kStSpec);

  // shared memory: barriers, plan prefix and scan scratch, the share's
  // tokens, tables, B buffers
  int off = 2 * kStBBufs * 8;
  p.off_prefix = off;
  off += round_up_i((p.slots + 1) * 4, 16);
  p.off_scratch = off;
  off += round_up_i(kStThreads / 32 * 4, 16);
  p.off_spec = off;
  off += round_up_i(nspec * 4, 16);
  p.off_ctok = off;
  off += p.gtab * kStRows * 4;
  p.off_cval = off;
  off += p.gtab * kStRows * 4;
  p.off_gmeta = round_up_i(off, 16);
  off = p.off_gmeta + p.gtab * 16;
  p.off_htab = round_up_i(off, 16);
  off = p.off_htab + p.gtab * kStRows * p.S * Rp * 2;
  p.off_bbuf = round_up_i(off, 128);
  p.smem = p.off_bbuf + kStBBufs * p.bbytes;
  if (p.smem > d.max_smem) {
    *why = "shared memory of the streamed embedding exceeds the device limit";
    return cudaErrorInvalidConfiguration;
  }
  p.wait_ns = wait_limit_ns();

  switch (KS) {
    case 1: return launch_ks<1>(p, grid, stream);
    case 2: return launch_ks<2>(p, grid, stream);
    case 3: return launch_ks<3>(p, grid, stream);
    default: return launch_ks<4>(p, grid, stream);
  }
}

}  // namespace lora
