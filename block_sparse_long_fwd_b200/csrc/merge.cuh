// Stage 5: log-sum-exp merge of the partial outputs of one query row.
//
// A row attends its own block (own-tile partial) and up to k-1 past blocks
// (routed partials). Each partial i holds the normalised output O_i and
// lse_i = ln sum exp(scaled logits) over its keys, so the softmax over the
// union of the selected keys is
//   L = ln sum_i exp(lse_i),   O = sum_i exp(lse_i - L) O_i,
// added in a fixed order (ascending block index, own block last). A routed
// partial of past block j is found through the router's flag words: its
// list slot is wordbase[g][j][w] + popcount of the bits below the row.
#pragma once

#include "route.cuh"

namespace moba {

struct MergeParams {
  const int32_t* sel;
  const uint32_t* flags;
  const int32_t* wordbase;
  const __half* part_o;  // fp16 partial outputs
  const float* part_lse;
  const __half* own_o;
  const float* own_lse;
  __nv_bfloat16* out;  // [S - q0][Hq][128]: rows of the tokens with a query
  float* lse;          // [Hq][lse_ld]: row h, column t - q0
  int64_t lse_ld;      // S - q0, or the packed token count of a batch
  WindowGeom w;
};

// Four fp16 values (8 bytes) widened to fp32.
__device__ __forceinline__ float4 load_half4(const __half* p) {
  const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&r.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&r.y));
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Reductions over the 16 lanes of a half-warp (both halves at once).
__device__ __forceinline__ float half_max(float v) {
  for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float half_sum(float v) {
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Two fp16 values packed in a 32-bit word, widened to fp32.
__device__ __forceinline__ float2 half2_bits(uint32_t x) {
  __half2 h;
  memcpy(&h, &x, sizeof(h));
  return __half22float2(h);
}

// acc += w * (eight fp16 values in o)
__device__ __forceinline__ void fma_half8(float (&acc)[8], float w, uint4 o) {
  const uint32_t word[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = half2_bits(word[i]);
    acc[2 * i] = fmaf(w, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, f.y, acc[2 * i + 1]);
  }
}

// grid ceil(wlen * Hq / 16), 256 threads: one half-warp per (token, q head)
// row, lane l (of 16) owns channels 8l..8l+7 (16-byte loads and stores).
// Lane i of the half resolves routed partial i (its list slot from the
// router's flag words, and its lse); with NP > 0 and at most NP routed
// partials per row, every partial's O is requested as soon as its slot is
// known, together with its lse, so a row costs three dependent memory round
// trips (selection, flag words, partials). Rows with more partials take a
// three-pass path. The sums run in a fixed order either way: ascending
// block, own block last.
template <int NP>
__global__ void __launch_bounds__(256, NP > 0 && NP <= 12 ? 4 : 3) merge_kernel(MergeParams m) {
  grid_dependency_sync();
  const WindowGeom& w = m.w;
  const int l16 = threadIdx.x & 15;
  const int hbase = threadIdx.x & 16;  // first lane of this half-warp
  int64_t row = (int64_t)blockIdx.x * 16 + (threadIdx.x >> 4);
  const int64_t nrows = w.wlen * w.Hq;
  // both halves of a warp stay converged for the shuffles; a half past the
  // end (or a token before q0) runs on a harmless row and writes nothing
  bool live = row < nrows;
  if (!live) row = nrows - 1;
  // 32-bit divisions: a window's rows (wlen * Hq) and every token index fit
  // in 32 bits (the host bounds the window's list slots and seqlen by 2^31)
  const uint32_t tl32 = udiv32((uint32_t)row, (uint32_t)w.Hq);
  const int64_t tl = tl32;
  const int h = (int)((uint32_t)row - tl32 * (uint32_t)w.Hq);
  const int64_t t = w.w0 + tl;
  if (t < w.q0) live = false;
  const int64_t tq = max(t - w.q0, (int64_t)0), nq = w.S - w.q0;
  const int g = (int)udiv32((uint32_t)h, (uint32_t)w.G), hl = h - g * w.G;
  const int bt = (int)udiv32((uint32_t)t, (uint32_t)w.B);
  const int64_t rr = tl * w.G + hl;
  const int64_t word = rr >> 5;
  const uint32_t below = (1u << (rr & 31)) - 1u;
  const int32_t* srow = m.sel + ((int64_t)h * nq + tq) * w.k_eff;
  const int P = w.k_eff - 1;

  // routed partial i: list slot (or -1) and lse (-inf when absent)
  auto slot = [&](int i, float& li) -> int64_t {
    li = -INFINITY;
    if (i >= P) return -1;
    const int j = __ldg(srow + i);
    if (j < 0 || j >= bt) return -1;
    const int64_t f = ((int64_t)g * w.nbp + j) * w.wwords + word;
    const int64_t pos = (int64_t)__ldg(m.wordbase + f) + __popc(__ldg(m.flags + f) & below);
    if (!slot_ok(w, pos)) return -1;
    li = __ldg(m.part_lse + pos);
    return pos;
  };

  const float own_l = m.own_lse[tl * w.Hq + h];
  const uint4 own_v = __ldg(reinterpret_cast<const uint4*>(m.own_o + (tl * w.Hq + h) * kHeadDim + l16 * 8));
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  float L;
  if (NP > 0 && P <= NP) {
    float li;
    const int64_t pos = slot(l16, li);
    uint4 o[NP > 0 ? NP : 1];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const int64_t pk = __shfl_sync(0xffffffffu, pos, hbase + k);
      o[k] = make_uint4(0u, 0u, 0u, 0u);
      if (k < P && pk >= 0) o[k] = __ldg(reinterpret_cast<const uint4*>(m.part_o + pk * kHeadDim + l16 * 8));
    }
    const float mx = fmaxf(own_l, half_max(li));
    const float sum = half_sum(li == -INFINITY ? 0.f : expf(li - mx)) + expf(own_l - mx);
    L = mx + logf(sum);
    const float wl = li == -INFINITY ? 0.f : expf(li - L);  // lane i's weight (0 past P)
#pragma unroll
    for (int k = 0; k < NP; ++k) fma_half8(acc, __shfl_sync(0xffffffffu, wl, hbase + k), o[k]);
  } else {
    // any number of partials: maximum, sum, then the weighted partials, in
    // groups of 16 (each pass finds its slots again)
    float mx = own_l;
    for (int i0 = 0; i0 < P; i0 += 16) {
      float li;
      slot(i0 + l16, li);
      mx = fmaxf(mx, half_max(li));
    }
    float sum = 0.f;
    for (int i0 = 0; i0 < P; i0 += 16) {
      float li;
      slot(i0 + l16, li);
      sum += half_sum(li == -INFINITY ? 0.f : expf(li - mx));
    }
    sum += expf(own_l - mx);
    L = mx + logf(sum);
    for (int i0 = 0; i0 < P; i0 += 16) {
      float li;
      const int64_t pos = slot(i0 + l16, li);
      const float wl = li == -INFINITY ? 0.f : expf(li - L);
      for (int k0 = 0; k0 < 16; k0 += 4) {
        uint4 o[4];
        float wk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t pk = __shfl_sync(0xffffffffu, pos, hbase + k0 + u);
          wk[u] = __shfl_sync(0xffffffffu, wl, hbase + k0 + u);
          o[u] = make_uint4(0u, 0u, 0u, 0u);
          if (pk >= 0) o[u] = __ldg(reinterpret_cast<const uint4*>(m.part_o + pk * kHeadDim + l16 * 8));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) fma_half8(acc, wk[u], o[u]);
      }
    }
  }
  fma_half8(acc, expf(own_l - L), own_v);
  if (!live) return;
  uint4 packed;
  packed.x = pack_bf16x2(acc[0], acc[1]);
  packed.y = pack_bf16x2(acc[2], acc[3]);
  packed.z = pack_bf16x2(acc[4], acc[5]);
  packed.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(m.out + (tq * w.Hq + h) * kHeadDim + l16 * 8) = packed;
  if (l16 == 0) m.lse[(int64_t)h * m.lse_ld + tq] = L;
}

}  // namespace moba
