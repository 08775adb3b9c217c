// Shrink over short segments: the (slot, expert) groups of the grouped MoE
// fold hold a few dozen rows each, so the rows are taken 16 at a time (one
// m16n8k16 row tile) instead of in 128-row tensor-core tiles.
//
//   h[kc][t, i*R + r] = sum over the features k of chunk kc of x[t, k] * a[pair, i*R + r, k]
//
// Sources: mstar.engine.resources.lora.backend, LoraBackend.shrink (h = x A^T);
// spark_model/lora/expert_apply.rs, apply_expert_lora_sorted (the fold per
// (slot, expert) group of sorted rows, each with its pair's A).
//
// Every group's positions [seg_lo, seg_hi) (or, without seg_hi, CSR by slot:
// [seg_lo[s], seg_lo[s+1])) are cut into row groups of 16 and
// the input features into chunks of 512; a unit is one (row group, chunk)
// pair and the units, row group by row group, are split into equal runs, one
// per CTA (one per SM).  All 16 warps of a CTA work on one unit: warp w takes
// 32 of the chunk's features (two k-steps), loads its x and A fragments with
// 8-byte loads (the k index permuted identically in both, thread q holding
// k = 4q..4q+3 of each k-step, which leaves the sum unchanged) and runs the
// MMAs for all S*R columns; the 16 partial tiles are summed in a fixed order
// through shared memory and the chunk's fp32 h is written to its partial
// buffer.  Each thread keeps the loads of the next two units in flight.
// Columns past a group's rank are computed and never read.
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
  int off_red;               // shared-memory offset of the reduction tiles
};

// The fragments one thread loads for one unit.
template <int NT>
struct GsRegs {
  uint2 xa[2], xb[2];     // rows g and g + 8, k-steps 0 and 1
  uint2 af[NT][2];        // A rows 8j + g, k-steps 0 and 1
  int ta, tb;             // the two rows' tokens (-1: none)
};

template <int NT>
__global__ void __launch_bounds__(kGsThreads, 1) group_shrink_kernel(const GShrinkParams p) {
  constexpr int SR = NT * 8;
  extern __shared__ __align__(16) uint8_t smem[];
  int* prefix = reinterpret_cast<int*>(smem);     // [slots + 1]
  int* scratch = prefix + p.slots + 1;            // [kGsWarps]
  float* red = reinterpret_cast<float*>(smem + p.off_red);   // [kGsWarps][16][SR]
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int g8 = lane >> 2;
  const int q = lane & 3;

  // the groups' row groups (flags of bad segments and ranks are raised by the
  // kernel that follows, which plans the same segments)
  const int planned = plan_linear<kGsThreads>(p.seg_lo, p.ranks, p.scalings, p.slots, p.T, p.R,
                                              kStRows, prefix, scratch, nullptr, false, p.seg_hi);
  grid_dep_launch_dependents();
  const long long gmax = ((long long)p.T + kStRows - 1) / kStRows + p.slots;
  const long long ng = (planned < 0 || planned > gmax) ? gmax : planned;
  const long long nu = ng * p.nks;
  const long long u0 = nu * blockIdx.x / gridDim.x;
  const long long u1 = nu * (blockIdx.x + 1) / gridDim.x;
  const uint8_t* X = static_cast<const uint8_t*>(p.x);
  const uint8_t* A = static_cast<const uint8_t*>(p.a);

  // unit u: row group u / nks, feature chunk u % nks; this thread's loads
  auto load = [&](long long u, GsRegs<NT>& r) {
    const int g = (int)(u / p.nks);
    const int kc = (int)(u - (long long)g * p.nks);
    const int s = find_segment(prefix, p.slots, g);
    const int lo = p.seg_lo[s];
    const int hi = p.seg_hi != nullptr ? p.seg_hi[s] : p.seg_lo[s + 1];
    const int pair = p.slot_map != nullptr ? p.slot_map[s] : s;
    const int pa = lo + (g - prefix[s]) * kStRows + g8;
    const int pb = pa + 8;
    r.ta = pa < hi ? p.token_order[pa] : -1;
    r.tb = pb < hi ? p.token_order[pb] : -1;
    if (r.ta < 0 || r.ta >= p.T) r.ta = -1;
    if (r.tb < 0 || r.tb >= p.T) r.tb = -1;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const int k0 = kc * (32 * kGsWarps) + warp * 32 + ks * 16 + 4 * q;
      const bool kin = k0 < p.in;
      r.xa[ks] = (kin && r.ta >= 0)
                     ? *reinterpret_cast<const uint2*>(X + ((size_t)r.ta * p.in + k0) * 2)
                     : make_uint2(0u, 0u);
      r.xb[ks] = (kin && r.tb >= 0)
                     ? *reinterpret_cast<const uint2*>(X + ((size_t)r.tb * p.in + k0) * 2)
                     : make_uint2(0u, 0u);
#pragma unroll
      for (int j = 0; j < NT; ++j)
        r.af[j][ks] = kin ? *reinterpret_cast<const uint2*>(
                                A + (((size_t)pair * SR + 8 * j + g8) * p.in + k0) * 2)
                          : make_uint2(0u, 0u);
    }
  };
  // one unit: MMAs on r, the loads of unit un into rn (two units ahead), the
  // warp's partial tile and the rows' tokens into shared memory, then the sum
  // over the warps in a fixed order into the chunk's partial buffer
  int* rowtok = scratch;   // the plan is done: its scan scratch holds the 16 row tokens
  auto step = [&](long long u, GsRegs<NT>& r, long long un, GsRegs<NT>& rn) {
    float d[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) d[j][e] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma_bf16_16816(d[j], r.xa[ks].x, r.xb[ks].x, r.xa[ks].y, r.xb[ks].y, r.af[j][ks].x,
                       r.af[j][ks].y);
    }
    float* rw = red + (size_t)warp * kStRows * SR;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      rw[g8 * SR + 8 * j + 2 * q] = d[j][0];
      rw[g8 * SR + 8 * j + 2 * q + 1] = d[j][1];
      rw[(g8 + 8) * SR + 8 * j + 2 * q] = d[j][2];
      rw[(g8 + 8) * SR + 8 * j + 2 * q + 1] = d[j][3];
    }
    if (warp == 0 && q == 0) {
      rowtok[g8] = r.ta;
      rowtok[g8 + 8] = r.tb;
    }
    const int kc = (int)(u % p.nks);
    if (un < u1) load(un, rn);
    __syncthreads();
    for (int idx = tid; idx < kStRows * SR; idx += kGsThreads) {
      const int row = idx / SR;
      const int col = idx - row * SR;
      const int t = rowtok[row];
      if (t < 0) continue;
      float v = 0.f;
#pragma unroll 4
      for (int w = 0; w < kGsWarps; ++w) v += red[((size_t)w * kStRows + row) * SR + col];
      p.h[(size_t)kc * p.h_split + (size_t)t * SR + col] = v;
    }
    __syncthreads();
  };

  GsRegs<NT> r0, r1, r2;
  grid_dep_wait();   // x (and the partial buffers) only after the preceding kernel
  if (u0 < u1) load(u0, r0);
  if (u0 + 1 < u1) load(u0 + 1, r1);
  for (long long u = u0; u < u1; u += 3) {
    step(u, r0, u + 2, r2);
    if (u + 1 >= u1) break;
    step(u + 1, r1, u + 3, r0);
    if (u + 2 >= u1) break;
    step(u + 2, r2, u + 4, r1);
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

bool group_shrink_supported(int S, int R, int in) {
  const int SR = S * R;
  return (SR == 16 || SR == 32 || SR == 48 || SR == 64) && in <= kGsMaxIn;
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
  p.nks = group_shrink_chunks(in);
  static_assert(32 * kGsWarps == 512, "one chunk is 512 features");
  *ksplit_out = p.nks;
  p.off_red = round_up_i((slots + 1 + kGsWarps) * 4, 16);
  const int SR = S * R;
  const size_t smem = (size_t)p.off_red + (size_t)kGsWarps * kStRows * SR * 4;
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
