// Stage 1: key mean-pool.
//
// MoBA cuts the keys into blocks and lets a parameter-less top-k gate pick,
// per query token, the most relevant blocks ("MoBA (Mixture of Block
// Attention)" project summary, "How It Works"). The gate score of block j for
// query row (t, h) is q[t][h] . mean_{u in blk j} k[u][g(h)]; this stage
// computes those block means (the gate itself is in gate_tc.cuh).
#pragma once

#include "common.cuh"

namespace moba {

// ------------------------------------------------------------------ pool
// grid (nb - 1, Hkv, splits), 256 threads. CTA (j, g, sp) sums rows
// [sp*B/splits, (sp+1)*B/splits) of block j: thread (rowgroup = tid / 16,
// chunk = tid % 16) adds 8 channels over every 16th row, then the 16
// row-group partials are added in a fixed order and scaled by 1/B. With one
// split that is the block mean; with several, the split kernel adds the
// splits in order. Only blocks that can be a past block (j <= nb - 2) are
// pooled; they are all full.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16* __restrict__ k, int Hkv, int B,
                                                            int nbp, int splits, int j0, float* __restrict__ out) {
  grid_dependency_sync();
  const int j = j0 + (int)blockIdx.x, g = blockIdx.y, sp = blockIdx.z;
  const int rows = B / splits;
  const int chunk = threadIdx.x & 15, rg = threadIdx.x >> 4;
  const int64_t row_stride = (int64_t)Hkv * kHeadDim;  // elements between consecutive tokens
  const __nv_bfloat16* base =
      k + ((int64_t)j * B + (int64_t)sp * rows) * row_stride + (int64_t)g * kHeadDim + chunk * 8;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  int r = rg;
  for (; r + 48 < rows; r += 64) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)(r + 16 * u) * row_stride));
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float2 f = __bfloat1622float2(p[c]);
        acc[2 * c] += f.x;
        acc[2 * c + 1] += f.y;
      }
    }
  }
  for (; r < rows; r += 16) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)r * row_stride));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float2 f = __bfloat1622float2(p[c]);
      acc[2 * c] += f.x;
      acc[2 * c + 1] += f.y;
    }
  }
  __shared__ float red[16][kHeadDim];
#pragma unroll
  for (int c = 0; c < 8; ++c) red[rg][chunk * 8 + c] = acc[c];
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) s += red[q][threadIdx.x];
    out[(((int64_t)g * nbp + j) * splits + sp) * kHeadDim + threadIdx.x] = s / (float)B;
  }
}

// Row splits per block so that small problems still fill the GPU: the
// smallest power of two giving at least `ctas` CTAs, at most B / 128.
inline int pool_splits(int nbp, int Hkv, int B, int ctas) {
  int sp = 1;
  while ((int64_t)nbp * Hkv * sp < ctas && sp * 2 <= B / 128 && (B / 128) % (sp * 2) == 0) sp *= 2;
  return sp;
}

}  // namespace moba
