// Shrink over short segments: the (slot, expert) groups of the grouped MoE
// fold hold a few dozen rows each, and so do the slots of a mid-size batch,
// so the rows are taken 16 at a time (one m16n8k16 row tile) instead of in
// 128-row tensor-core tiles.
//
//   h[kc][t, i*R + r] = sum over the features k of chunk kc of x[t, k] * a[pair, i*R + r, k]
//
// Sources: mstar.engine.resources.lora.backend, LoraBackend.shrink (h = x A^T);
// spark_model/lora/expert_apply.rs, apply_expert_lora_sorted (the fold per
// (slot, expert) group of sorted rows, each with its pair's A).
//
// Every group's positions [seg_lo, seg_hi) (or, without seg_hi, CSR by slot:
// [seg_lo[s], seg_lo[s+1])) are cut into row groups of 16 and the input
// features into at most 8 chunks of 256 << k features; a unit is one (row
// group, chunk) pair and the units, row group by row group, are split into
// equal runs, one per CTA (one per SM).
//
// The 16 warps of a CTA form teams of TS warps (TS chosen per CTA from its
// unit count: the fewer the units, the larger the teams); a team takes every
// (16 / TS)-th unit of the run and its warps split the unit's 32-feature
// sub-steps round robin.  A warp streams its sub-steps without a break, unit
// after unit: thread q loads features 8q..8q+7 of the sub-step for its two x
// rows and its A rows with one 16-byte load each, the next sub-steps' loads in
// flight, and feeds 8q..8q+3 to one k-step MMA and 8q+4..8q+7 to the other
// (the same permutation of k in both operands leaves the sum unchanged).  At
// the end of a unit a one-warp team stores its fp32 tile straight to the
// chunk's partial buffer; a larger team sums its warps' tiles in warp order
// through shared memory first.  Columns past a group's rank are computed and
// never read.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace lora {
namespace {

constexpr int kGsWarps = 16;
constexpr int kGsThreads = 32 * kGsWarps;

struct GShrinkParams {
  const void* x;
  const void* a;
  float* h;                  // [nks][T][S*R]
  size_t h_split;
  const int* token_order;
  const int* seg_lo;
  const int* seg_hi;
  const int* slot_map;
  const int* ranks;
  const float* scalings;
  int T, in, slots, R, S, nks;
  int chunk;                 // features per chunk (256 << k)
  int off_segs, off_red;     // shared-memory offsets
};

// One sub-step's fragments of one thread: 8 features of rows g and g + 8 of
// x, and of A rows 8j + g.
template <int NT>
struct GsSet {
  uint4 xa, xb;
  uint4 af[NT];
};

LORA_DEV uint4 ldg16(const uint8_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

LORA_DEV void team_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Sub-steps in flight per warp (what the registers hold beside the tile).
template <int NT>
struct GsSets {
  static constexpr int value = NT <= 2 ? 4 : NT <= 4 ? 3 : NT <= 6 ? 2 : 1;
};

template <int NT>
__global__ void __launch_bounds__(kGsThreads, 1) group_shrink_kernel(const GShrinkParams p) {
  constexpr int SR = NT * 8;
  constexpr int SRP = SR + 8;     // padded tile row: conflict-free 8-byte stores
  constexpr int NSET = GsSets<NT>::value;
  extern __shared__ __align__(16) uint8_t smem[];
  int* prefix = reinterpret_cast<int*>(smem);                    // [slots + 1]
  int* scratch = prefix + p.slots + 1;                           // [kGsWarps]
  int4* segs = reinterpret_cast<int4*>(smem + p.off_segs);       // [slots]
  float* red = reinterpret_cast<float*>(smem + p.off_red);       // [kGsWarps][16][SRP]
  __shared__ int utok[kGsWarps][NSET][kStRows + 1];   // a unit's 16 row tokens and its chunk
  __shared__ int rtok[kGsWarps][kStRows];             // a team's 16 row tokens
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int g8 = lane >> 2;
  const int q = lane & 3;

  // the groups' row groups (flags of bad segments and ranks are raised by the
  // kernel that follows, which plans the same segments)
  const int planned = plan_linear<kGsThreads>(p.seg_lo, p.ranks, p.scalings, p.slots, p.T, p.R,
                                              kStRows, prefix, scratch, nullptr, false, p.seg_hi,
                                              segs);
  grid_dep_launch_dependents();
  const long long gmax = ((long long)p.T + kStRows - 1) / kStRows + p.slots;
  const long long ng = (planned < 0 || planned > gmax) ? gmax : planned;
  const long long nu = ng * p.nks;
  const long long u0 = nu * blockIdx.x / gridDim.x;
  const long long u1 = nu * (blockIdx.x + 1) / gridDim.x;
  const int cnt = (int)(u1 - u0);
  const int nsub = p.chunk / 32;

  // team size: the fewest sub-step times for this CTA's units, a team's
  // reduction counted as two (ties: the smaller team)
  int TS = 1;
  {
    long long best = -1;
    for (int ts = 1; ts <= kGsWarps && ts <= nsub; ts *= 2) {
      const int teams = kGsWarps / ts;
      const long long cost =
          (long long)((cnt + teams - 1) / teams) * (nsub / ts + (ts > 1 ? 2 : 0));
      if (best < 0 || cost < best) {
        best = cost;
        TS = ts;
      }
    }
  }
  const int nteams = kGsWarps / TS;
  const int tm = warp / TS;
  const int wt = warp - tm * TS;
  const int nun = cnt > tm ? (cnt - tm + nteams - 1) / nteams : 0;   // this team's units
  const int per = nsub / TS;                                          // sub-steps per unit and warp
  const int K = nun * per;

  const uint8_t* X = static_cast<const uint8_t*>(p.x);
  const uint8_t* A = static_cast<const uint8_t*>(p.a);

  // unit r of this team: its first position (row g8 of this lane), segment
  // end, pair and chunk
  auto unit_pos = [&](int r, int& pa, int& hi, int& pair, int& kc) {
    const long long u = u0 + tm + (long long)r * nteams;
    const int g = (int)(u / p.nks);
    kc = (int)(u - (long long)g * p.nks);
    const int s = find_segment(prefix, p.slots, g);
    const int4 sg = segs[s];
    pair = p.slot_map != nullptr ? p.slot_map[s] : s;
    pa = sg.x + (g - prefix[s]) * kStRows + g8;
    hi = sg.y;
  };
  // the unit the load cursor is in (its tokens, pair, feature range) and the
  // raw tokens of the next one, read while this one loads
  int lr = -1, l_ta = -1, l_tb = -1, l_pair = 0, l_k0 = 0, l_k1 = 0;
  int n_ta = -1, n_tb = -1;
  auto read_ahead = [&](int r) {
    n_ta = n_tb = -1;
    if (r < nun) {
      int pa, hi, pair, kc;
      unit_pos(r, pa, hi, pair, kc);
      if (pa < hi) n_ta = p.token_order[pa];
      if (pa + 8 < hi) n_tb = p.token_order[pa + 8];
    }
  };
  read_ahead(0);
  auto issue = [&](int k, GsSet<NT>& st) {
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    if (k >= K) {
      st.xa = st.xb = z;
#pragma unroll
      for (int j = 0; j < NT; ++j) st.af[j] = z;
      return;
    }
    const int r = k / per;
    if (r != lr) {
      // units are entered in order, so the read-ahead holds this one's tokens
      int pa, hi, pair, kc;
      unit_pos(r, pa, hi, pair, kc);
      lr = r;
      l_ta = (n_ta < 0 || n_ta >= p.T) ? -1 : n_ta;
      l_tb = (n_tb < 0 || n_tb >= p.T) ? -1 : n_tb;
      l_pair = pair;
      l_k0 = kc * p.chunk;
      l_k1 = min(p.in, l_k0 + p.chunk);
      if (q == 0) {
        utok[warp][r % NSET][g8] = l_ta;
        utok[warp][r % NSET][g8 + 8] = l_tb;
      }
      if (lane == 0) utok[warp][r % NSET][kStRows] = kc;
      read_ahead(r + 1);
    }
    const int j = wt + (k - r * per) * TS;
    const int k0 = l_k0 + 32 * j + 8 * q;
    const bool kin = k0 < l_k1;   // in is a multiple of 8: the 8 features are all in or all out
    st.xa = (kin && l_ta >= 0) ? ldg16(X + ((size_t)l_ta * p.in + k0) * 2) : z;
    st.xb = (kin && l_tb >= 0) ? ldg16(X + ((size_t)l_tb * p.in + k0) * 2) : z;
#pragma unroll
    for (int jj = 0; jj < NT; ++jj)
      st.af[jj] = kin ? ldg16(A + (((size_t)l_pair * SR + 8 * jj + g8) * p.in + k0) * 2) : z;
  };

  float d[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;
  // the end of unit r: its tile to the chunk's partial buffer
  auto finish = [&](int r) {
    __syncwarp();
    const int* ut = utok[warp][r % NSET];
    const int ra = ut[g8];
    const int rb = ut[g8 + 8];
    float* hk = p.h + (size_t)ut[kStRows] * p.h_split;
    if (TS == 1) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (ra >= 0)
          __stcg(reinterpret_cast<float2*>(hk + (size_t)ra * SR + 8 * j + 2 * q),
                 make_float2(d[j][0], d[j][1]));
        if (rb >= 0)
          __stcg(reinterpret_cast<float2*>(hk + (size_t)rb * SR + 8 * j + 2 * q),
                 make_float2(d[j][2], d[j][3]));
      }
    } else {
      float* rw = red + (size_t)warp * kStRows * SRP;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        *reinterpret_cast<float2*>(rw + g8 * SRP + 8 * j + 2 * q) = make_float2(d[j][0], d[j][1]);
        *reinterpret_cast<float2*>(rw + (g8 + 8) * SRP + 8 * j + 2 * q) =
            make_float2(d[j][2], d[j][3]);
      }
      if (wt == 0 && q == 0) {
        rtok[tm][g8] = ra;
        rtok[tm][g8 + 8] = rb;
      }
      team_sync(1 + tm, TS * 32);
      const float* rt = red + (size_t)tm * TS * kStRows * SRP;
      for (int idx = wt * 32 + lane; idx < kStRows * SR; idx += TS * 32) {
        const int row = idx / SR;
        const int col = idx - row * SR;
        const int t = rtok[tm][row];
        if (t < 0) continue;
        float v = 0.f;
        for (int w = 0; w < TS; ++w) v += rt[((size_t)w * kStRows + row) * SRP + col];
        __stcg(hk + (size_t)t * SR + col, v);
      }
      team_sync(1 + tm, TS * 32);
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;
  };

  grid_dep_wait();   // x (and the partial buffers) only after the preceding kernel
  GsSet<NT> set[NSET];
#pragma unroll
  for (int b = 0; b < NSET; ++b) issue(b, set[b]);
  for (int k = 0; k < K; k += NSET) {
#pragma unroll
    for (int b = 0; b < NSET; ++b) {
      const int kk = k + b;
      if (kk < K) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          mma_bf16_16816(d[j], set[b].xa.x, set[b].xb.x, set[b].xa.y, set[b].xb.y,
                         set[b].af[j].x, set[b].af[j].y);
          mma_bf16_16816(d[j], set[b].xa.z, set[b].xb.z, set[b].xa.w, set[b].xb.w,
                         set[b].af[j].z, set[b].af[j].w);
        }
        // a unit is finished before the load cursor may reuse its token slot
        if ((kk + 1) % per == 0) finish(kk / per);
        issue(kk + NSET, set[b]);
      }
    }
  }
}

template <int NT>
cudaError_t launch_nt(const cudaLaunchConfig_t& cfg, const GShrinkParams& p) {
  const cudaError_t err = cudaFuncSetAttribute(
      group_shrink_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
      (int)cfg.dynamicSmemBytes);
  if (err != cudaSuccess) return err;
  return cudaLaunchKernelEx(&cfg, group_shrink_kernel<NT>, p);
}

}  // namespace

int group_shrink_chunk(int in) {
  int c = 256;
  while ((long long)c * kGsMaxParts < in) c *= 2;
  return c;
}

int group_shrink_chunks(int in) { return ceil_div_i(in, group_shrink_chunk(in)); }

bool group_shrink_supported(int S, int R, int in) {
  const int SR = S * R;
  return (SR == 16 || SR == 32 || SR == 48 || SR == 64) && in >= 8 && in <= kGsMaxIn;
}

cudaError_t group_shrink_launch(const void* x, const void* a, float* h, const int* token_order,
                                const int* seg_lo, const int* seg_hi, const int* slot_map,
                                const int* ranks, const float* scalings, int T, int in,
                                int slots, int R, int S, int* ksplit_out, cudaStream_t stream,
                                bool allow_overlap) {
  int dev = 0, sms = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess) return err;
  GShrinkParams p = {};
  p.x = x; p.a = a; p.h = h; p.h_split = (size_t)T * S * R; p.token_order = token_order;
  p.seg_lo = seg_lo; p.seg_hi = seg_hi; p.slot_map = slot_map; p.ranks = ranks;
  p.scalings = scalings; p.T = T; p.in = in; p.slots = slots; p.R = R; p.S = S;
  p.chunk = group_shrink_chunk(in);
  p.nks = ceil_div_i(in, p.chunk);
  *ksplit_out = p.nks;
  const int SR = S * R;
  p.off_segs = round_up_i((slots + 1 + kGsWarps) * 4, 16);
  p.off_red = round_up_i(p.off_segs + slots * 16, 16);
  const size_t smem = (size_t)p.off_red + (size_t)kGsWarps * kStRows * (SR + 8) * 4;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3((unsigned)sms, 1, 1);
  cfg.blockDim = dim3(kGsThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  if (allow_overlap && launch_overlap_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  switch (SR / 8) {
    case 2: err = launch_nt<2>(cfg, p); break;
    case 4: err = launch_nt<4>(cfg, p); break;
    case 6: err = launch_nt<6>(cfg, p); break;
    default: err = launch_nt<8>(cfg, p); break;
  }
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace lora
