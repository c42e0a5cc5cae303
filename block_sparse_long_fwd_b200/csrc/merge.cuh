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

// grid ceil(wlen * Hq / 8), 256 threads: one warp per (token, q head) row,
// lane c owns channels 4c..4c+3. With NP > 0 and at most NP routed partials
// per row, every partial row is loaded as soon as its slot is known, before
// the weights (which wait for the partials' lse) are formed: the row then
// costs three dependent memory round trips (selection, flag words, partials)
// instead of four. It pays off for a few partials per row (small, latency
// bound problems); with many, the registers it holds cost more occupancy
// than it gains (measured: 1M workload merge 35 -> 39 ms with NP = 12), so
// the host uses it for up to 4. The sums run in the same order either way.
template <int NP>
__global__ void __launch_bounds__(256) merge_kernel(MergeParams m) {
  grid_dependency_sync();
  const WindowGeom& w = m.w;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= w.wlen * w.Hq) return;
  const int64_t tl = row / w.Hq;
  const int h = (int)(row % w.Hq);
  const int64_t t = w.w0 + tl;
  if (t < w.q0) return;  // no query at this token (padding of a window's first tile)
  const int64_t tq = t - w.q0, nq = w.S - w.q0;
  const int g = h / w.G, hl = h % w.G;
  const int bt = (int)(t / w.B);
  const int64_t rr = tl * w.G + hl;
  const int64_t word = rr >> 5;
  const uint32_t below = (1u << (rr & 31)) - 1u;
  const int32_t* srow = m.sel + ((int64_t)h * nq + tq) * w.k_eff;
  const int P = w.k_eff - 1;

  // lane i resolves routed partial i (slot and lse) once
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
  const __half* own_row = m.own_o + (tl * w.Hq + h) * kHeadDim + lane * 4;
  float4 own_v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (NP > 0) own_v = load_half4(own_row);  // early only where registers are cheap
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L;
  if (NP > 0 && P <= NP) {
    float li;
    const int64_t pos = slot(lane, li);
    float4 o[NP > 0 ? NP : 1];
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const int64_t pk = __shfl_sync(0xffffffffu, pos, k);
      o[k] = (k < P && pk >= 0) ? load_half4(m.part_o + pk * kHeadDim + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const float mx = fmaxf(own_l, warp_max(li));
    const float sum = warp_sum(li == -INFINITY ? 0.f : expf(li - mx)) + expf(own_l - mx);
    L = mx + logf(sum);
    const float wl = li == -INFINITY ? 0.f : expf(li - L);  // lane i's weight (0 past P)
#pragma unroll
    for (int k = 0; k < NP; ++k) {
      const float wk = __shfl_sync(0xffffffffu, wl, k);
      acc.x += wk * o[k].x;
      acc.y += wk * o[k].y;
      acc.z += wk * o[k].z;
      acc.w += wk * o[k].w;
    }
  } else if (P <= 32) {
    float li;
    const int64_t pos = slot(lane, li);
    const float mx = fmaxf(own_l, warp_max(li));
    const float sum = warp_sum(li == -INFINITY ? 0.f : expf(li - mx)) + expf(own_l - mx);
    L = mx + logf(sum);
    const float wl = li == -INFINITY ? 0.f : expf(li - L);  // lane i's weight
    // partials in ascending block order, four loads in flight
    const int n = min(P, 32);
    for (int k0 = 0; k0 < n; k0 += 4) {
      float4 o[4];
      float wk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + u;
        const int64_t pk = __shfl_sync(0xffffffffu, pos, k & 31);
        wk[u] = __shfl_sync(0xffffffffu, wl, k & 31);
        o[u] = (k < n && pk >= 0) ? load_half4(m.part_o + pk * kHeadDim + lane * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
        if (!(k < n && pk >= 0)) wk[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc.x += wk[u] * o[u].x;
        acc.y += wk[u] * o[u].y;
        acc.z += wk[u] * o[u].z;
        acc.w += wk[u] * o[u].w;
      }
    }
  } else {
    // every past block selected (topk >= number of blocks): chunks of 32
    float mx = own_l;
    for (int i0 = 0; i0 < P; i0 += 32) {
      float li;
      slot(i0 + lane, li);
      mx = fmaxf(mx, warp_max(li));
    }
    float sum = 0.f;
    for (int i0 = 0; i0 < P; i0 += 32) {
      float li;
      slot(i0 + lane, li);
      sum += warp_sum(li == -INFINITY ? 0.f : expf(li - mx));
    }
    sum += expf(own_l - mx);
    L = mx + logf(sum);
    for (int i0 = 0; i0 < P; i0 += 32) {
      float li;
      const int64_t pos = slot(i0 + lane, li);
      const int n = min(32, P - i0);
      for (int k = 0; k < n; ++k) {
        const int64_t pk = __shfl_sync(0xffffffffu, pos, k);
        const float lk = __shfl_sync(0xffffffffu, li, k);
        if (pk >= 0) {
          const float wk = expf(lk - L);
          const float4 o = load_half4(m.part_o + pk * kHeadDim + lane * 4);
          acc.x += wk * o.x;
          acc.y += wk * o.y;
          acc.z += wk * o.z;
          acc.w += wk * o.w;
        }
      }
    }
  }
  {
    if (NP == 0) own_v = load_half4(own_row);
    const float wk = expf(own_l - L);
    acc.x += wk * own_v.x;
    acc.y += wk * own_v.y;
    acc.z += wk * own_v.z;
    acc.w += wk * own_v.w;
  }
  uint2 packed = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  *reinterpret_cast<uint2*>(m.out + (tq * w.Hq + h) * kHeadDim + lane * 4) = packed;
  if (lane == 0) m.lse[(int64_t)h * m.lse_ld + tq] = L;
}

}  // namespace moba
