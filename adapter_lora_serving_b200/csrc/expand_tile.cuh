// The inner step of the staged expand shared by the few-tokens kernels: a
// warp's group of 16-column tiles of one slice against one 8-token tile,
// y = bf16_rne(y + scaling * (B H^T)) with H = hi + lo in bf16 (m16n8k16 MMAs,
// fp32 accumulate), B and y read from shared memory.
//
// Sources: mstar.engine.resources.lora.backend (LoraBackend.expand_fused:
// y[t, slice i] += scalings[slot] * h[t, slice i cols < rank] @ b[slot, slice i]^T).
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace lora {

// Zero masks of the bf16 B elements k0..k0+3 at or past the rank (as
// mask_rank4): .x covers (k0, k0+1), .y covers (k0+2, k0+3).
LORA_DEV uint2 rank_mask4(int k0, int rank) {
  return make_uint2((k0 < rank ? 0xffffu : 0u) | (k0 + 1 < rank ? 0xffff0000u : 0u),
                    (k0 + 2 < rank ? 0xffffu : 0u) | (k0 + 3 < rank ? 0xffff0000u : 0u));
}

constexpr int kExGroup = 4;   // 16-column tiles a warp expands per step

// One step of the staged expand: kExGroup 16-column tiles (columns jt + 128 q)
// of one slice and one 8-token tile.  All shared-memory loads of the step are
// issued before any MMA or store (the B copy, the h tiles and the y rows do
// not overlap), so the tiles' latencies overlap.  ks0 < ksteps k-steps of 16
// ranks; hh/hl are the h fragments of k-step 0 when kOneStep.
template <bool kOneStep>
LORA_DEV void expand_step(const uint16_t* __restrict__ bs, const uint16_t* __restrict__ hhi,
                          const uint16_t* __restrict__ hlo, uint8_t* __restrict__ yt, int ystride,
                          int R, int hrow, int ksteps, int rank, uint2 m0, uint2 hh, uint2 hl,
                          int jt, int ls1, int g, int c, uint32_t lv, float scal) {
  int jl[kExGroup];
  bool ok[kExGroup];
  float d[kExGroup][4];
  uint32_t yo[kExGroup][2];
#pragma unroll
  for (int q = 0; q < kExGroup; ++q) {
    jl[q] = jt + q * (kBgmvThreads / 2) + 2 * g;
    ok[q] = jl[q] < ls1;
#pragma unroll
    for (int k = 0; k < 4; ++k) d[q][k] = 0.f;
#pragma unroll
    for (int e = 0; e < 2; ++e)
      yo[q][e] = (ok[q] && ((lv >> e) & 1u))
                     ? *reinterpret_cast<const uint32_t*>(yt + e * ystride + jl[q] * 2)
                     : 0u;
  }
  if (kOneStep) {
    uint2 b0[kExGroup], b1[kExGroup];
#pragma unroll
    for (int q = 0; q < kExGroup; ++q) {
      b0[q] = b1[q] = make_uint2(0u, 0u);
      if (ok[q]) {
        b0[q] = *reinterpret_cast<const uint2*>(bs + (size_t)jl[q] * R + 4 * c);
        b1[q] = *reinterpret_cast<const uint2*>(bs + (size_t)(jl[q] + 1) * R + 4 * c);
      }
    }
#pragma unroll
    for (int q = 0; q < kExGroup; ++q) {
      const uint2 x0 = make_uint2(b0[q].x & m0.x, b0[q].y & m0.y);
      const uint2 x1 = make_uint2(b1[q].x & m0.x, b1[q].y & m0.y);
      mma_bf16_16816(d[q], x0.x, x1.x, x0.y, x1.y, hh.x, hh.y);
      mma_bf16_16816(d[q], x0.x, x1.x, x0.y, x1.y, hl.x, hl.y);
    }
  } else {
#pragma unroll 1
    for (int ks = 0; ks < ksteps; ++ks) {
      const int k0 = ks * 16 + 4 * c;
      const uint2 mk = rank_mask4(k0, rank);
      const uint2 h1 = *reinterpret_cast<const uint2*>(hhi + hrow + k0);
      const uint2 h2 = *reinterpret_cast<const uint2*>(hlo + hrow + k0);
#pragma unroll
      for (int q = 0; q < kExGroup; ++q) {
        uint2 x0 = make_uint2(0u, 0u), x1 = make_uint2(0u, 0u);
        if (ok[q] && k0 < R) {
          x0 = *reinterpret_cast<const uint2*>(bs + (size_t)jl[q] * R + k0);
          x1 = *reinterpret_cast<const uint2*>(bs + (size_t)(jl[q] + 1) * R + k0);
        }
        x0 = make_uint2(x0.x & mk.x, x0.y & mk.y);
        x1 = make_uint2(x1.x & mk.x, x1.y & mk.y);
        mma_bf16_16816(d[q], x0.x, x1.x, x0.y, x1.y, h1.x, h1.y);
        mma_bf16_16816(d[q], x0.x, x1.x, x0.y, x1.y, h2.x, h2.y);
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kExGroup; ++q) {
    if (!ok[q]) continue;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if ((lv >> e) & 1u)
        *reinterpret_cast<uint32_t*>(yt + e * ystride + jl[q] * 2) =
            pack_bf16x2(fmaf(scal, d[q][e], bf16_lo(yo[q][e])),
                        fmaf(scal, d[q][2 + e], bf16_hi(yo[q][e])));
    }
  }
}

}  // namespace lora
