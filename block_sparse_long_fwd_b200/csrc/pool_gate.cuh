// Stage 1: key mean-pool. Stage 2: gate scores + per-row top-k.
//
// MoBA cuts the keys into blocks and lets a parameter-less top-k gate pick,
// per query token, the most relevant blocks ("MoBA (Mixture of Block
// Attention)" project summary, "How It Works"). The gate score of block j for
// query row (t, h) is q[t][h] . mean_{u in blk j} k[u][g(h)]; a query may
// only pick past blocks (j < t/B), its own block is always picked and counts
// toward k ("MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
// "MoBAの技術的原則", causal design); ties go to the lower block index.
#pragma once

#include "common.cuh"

namespace moba {

// ------------------------------------------------------------------ pool
// grid (nb - 1, Hkv), 256 threads. Thread (rowgroup = tid / 16, chunk =
// tid % 16) sums 8 channels over rows rowgroup, rowgroup + 16, ... of block
// j, then the 16 row-group partials are added in a fixed order. Only blocks
// that can be a past block (j <= nb - 2) are pooled; they are all full.
constexpr int kPoolThreads = 256;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(const __nv_bfloat16* __restrict__ k, int Hkv, int B,
                                                            int nbp, float* __restrict__ kmean) {
  const int j = blockIdx.x, g = blockIdx.y;
  const int chunk = threadIdx.x & 15, rg = threadIdx.x >> 4;
  const int64_t row_stride = (int64_t)Hkv * kHeadDim;  // elements between consecutive tokens
  const __nv_bfloat16* base = k + ((int64_t)j * B) * row_stride + (int64_t)g * kHeadDim + chunk * 8;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.f;
  int r = rg;
  for (; r + 48 < B; r += 64) {
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
  for (; r < B; r += 16) {
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
    kmean[((int64_t)g * nbp + j) * kHeadDim + threadIdx.x] = s / (float)B;
  }
}

// ------------------------------------------------------------------ gate
// grid (ceil(S*G / 128), Hkv), 128 threads, one thread per group-row
// rr = t*G + hl (query t, head h = g*G + hl). The query row is held in
// registers as fp32; mean-pooled keys are staged in shared memory in chunks
// of kGateChunk blocks and read as broadcasts. Each score is one fp32 fma
// chain over the 128 channels in ascending order. A sorted list of the KP
// best (score, block) pairs is kept in registers; a later block enters only
// with a strictly larger score, so equal scores keep the lower index.
constexpr int kGateThreads = 128;
constexpr int kGateChunk = 32;

template <int KP>
__device__ __forceinline__ void topk_insert(float (&tv)[KP], int (&ti)[KP], float s, int j) {
#pragma unroll
  for (int i = KP - 1; i >= 0; --i) {
    const bool above = (i > 0) ? (s > tv[i - 1]) : false;
    const bool here = !above && (s > tv[i]);
    if (above) {
      tv[i] = tv[i - 1];
      ti[i] = ti[i - 1];
    } else if (here) {
      tv[i] = s;
      ti[i] = j;
    }
  }
}

template <int KP>
__global__ void __launch_bounds__(kGateThreads) gate_kernel(const __nv_bfloat16* __restrict__ q,
                                                            const float* __restrict__ kmean, int64_t S, int Hq,
                                                            int G, int B, int nbp, int k_eff,
                                                            int32_t* __restrict__ sel) {
  const int g = blockIdx.y;
  const int64_t rr = (int64_t)blockIdx.x * kGateThreads + threadIdx.x;
  const int64_t t = rr / G;
  const int h = g * G + (int)(rr % G);
  const bool valid = t < S;
  const int bt = valid ? (int)(t / B) : 0;
  const int P = k_eff - 1;  // past blocks picked by score
  const bool full = (k_eff == nbp + 1);  // every past block is picked

  // largest own-block index in this CTA (t grows with rr)
  int64_t t_last = ((int64_t)blockIdx.x * kGateThreads + kGateThreads - 1) / G;
  if (t_last > S - 1) t_last = S - 1;
  const int b_cta = full || P == 0 ? 0 : (int)(t_last / B);

  float tv[KP];
  int ti[KP];
#pragma unroll
  for (int i = 0; i < KP; ++i) {
    tv[i] = -INFINITY;
    ti[i] = -1;
  }

  if (b_cta > 0) {
    float qf[kHeadDim];
    if (valid && bt > 0) {
      const uint4* src = reinterpret_cast<const uint4*>(q + (t * Hq + h) * kHeadDim);
#pragma unroll
      for (int c = 0; c < kHeadDim / 8; ++c) {
        uint4 v = __ldg(src + c);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(p[e]);
          qf[c * 8 + 2 * e] = f.x;
          qf[c * 8 + 2 * e + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int c = 0; c < kHeadDim; ++c) qf[c] = 0.f;
    }
    __shared__ float4 sm[kGateChunk * kHeadDim / 4];
    const float4* km4 = reinterpret_cast<const float4*>(kmean + (int64_t)g * nbp * kHeadDim);
    for (int jc = 0; jc < b_cta; jc += kGateChunk) {
      const int nj = min(kGateChunk, b_cta - jc);
      __syncthreads();
      for (int i = threadIdx.x; i < nj * (kHeadDim / 4); i += kGateThreads)
        sm[i] = __ldg(km4 + (int64_t)jc * (kHeadDim / 4) + i);
      __syncthreads();
      const int jend = valid ? min(jc + nj, bt) : jc;
      int j = jc;
      for (; j + 4 <= jend; j += 4) {
        const float4* m0 = sm + (j - jc) * (kHeadDim / 4);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int c = 0; c < kHeadDim / 4; ++c) {
          const float4 x0 = m0[c], x1 = m0[c + 32], x2 = m0[c + 64], x3 = m0[c + 96];
          const float q0 = qf[4 * c], q1 = qf[4 * c + 1], q2 = qf[4 * c + 2], q3 = qf[4 * c + 3];
          a0 = fmaf(q0, x0.x, a0); a0 = fmaf(q1, x0.y, a0); a0 = fmaf(q2, x0.z, a0); a0 = fmaf(q3, x0.w, a0);
          a1 = fmaf(q0, x1.x, a1); a1 = fmaf(q1, x1.y, a1); a1 = fmaf(q2, x1.z, a1); a1 = fmaf(q3, x1.w, a1);
          a2 = fmaf(q0, x2.x, a2); a2 = fmaf(q1, x2.y, a2); a2 = fmaf(q2, x2.z, a2); a2 = fmaf(q3, x2.w, a2);
          a3 = fmaf(q0, x3.x, a3); a3 = fmaf(q1, x3.y, a3); a3 = fmaf(q2, x3.z, a3); a3 = fmaf(q3, x3.w, a3);
        }
        topk_insert<KP>(tv, ti, a0, j);
        topk_insert<KP>(tv, ti, a1, j + 1);
        topk_insert<KP>(tv, ti, a2, j + 2);
        topk_insert<KP>(tv, ti, a3, j + 3);
      }
      for (; j < jend; ++j) {
        const float4* m0 = sm + (j - jc) * (kHeadDim / 4);
        float a0 = 0.f;
#pragma unroll
        for (int c = 0; c < kHeadDim / 4; ++c) {
          const float4 x0 = m0[c];
          a0 = fmaf(qf[4 * c], x0.x, a0);
          a0 = fmaf(qf[4 * c + 1], x0.y, a0);
          a0 = fmaf(qf[4 * c + 2], x0.z, a0);
          a0 = fmaf(qf[4 * c + 3], x0.w, a0);
        }
        topk_insert<KP>(tv, ti, a0, j);
      }
    }
  }
  if (!valid) return;

  int32_t* out = sel + ((int64_t)h * S + t) * k_eff;
  if (full) {
    for (int i = 0; i < k_eff; ++i) out[i] = (i <= bt) ? i : -1;
    return;
  }
  const int npast = min(P, bt);
  // ascending order of the npast best indices (ti[0..npast) are the best)
  int key[KP];
#pragma unroll
  for (int i = 0; i < KP; ++i) key[i] = (i < npast) ? ti[i] : 0x7fffffff;
#pragma unroll
  for (int pass = 0; pass < KP; ++pass) {
#pragma unroll
    for (int i = (pass & 1); i + 1 < KP; i += 2) {
      const int a = key[i], b = key[i + 1];
      key[i] = min(a, b);
      key[i + 1] = max(a, b);
    }
  }
#pragma unroll
  for (int i = 0; i < KP; ++i)
    if (i < npast) out[i] = key[i];
  out[npast] = bt;
  for (int i = npast + 1; i < k_eff; ++i) out[i] = -1;
}

}  // namespace moba
