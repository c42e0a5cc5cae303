// Stage 3: the router. MoBA borrows the mixture-of-experts view: KV blocks
// play the experts and every query row is routed to the blocks its gate
// picked ("MoBA (Mixture of Block Attention)" project summary, "How It
// Works"; "MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
// high-performance implementation combining FlashAttention and MoE
// techniques). This stage turns the per-row choices into, for every
// (kv head g, past block j) bucket, the list of routed query rows, so the
// attention stage can stream each block's keys once per 128 routed rows.
//
// Rows are processed in query windows [w0, w0 + wlen). Within a window, a
// group-row is rr = (t - w0) * G + hl for query t and head h = g*G + hl.
// 1. flags: bit rr%32 of word flags[g][j][rr/32] is set when row rr routes
//    to block j (past blocks only; the own block goes to the diagonal pass);
//    the words are cleared first, and only the blocks picked are written.
// 2. count: popcount per bucket.
// 3. scan (one CTA): exclusive offsets of the lists and of their 128-row
//    tiles, plus the own-block tiles of the window, longest first.
// 4. fill: per bucket, prefix popcounts give each word's first list slot
//    (kept as wordbase for the merge) and the set bits expand, in (t, h)
//    order, into list entries rr. Every bucket's list is therefore sorted
//    and the whole router is deterministic.
#pragma once

#include "common.cuh"

namespace moba {

struct WindowGeom {
  int64_t S;
  int Hq, Hkv, G, B;
  int k_eff, nbp;   // blocks per row; number of poolable (past-able) blocks
  int64_t w0, wlen;  // window start token and length
  int64_t wwords;    // flag words per bucket: ceil(wlen * G / 32)
  int pair_tokens;   // own units pair consecutive 128-token tiles of one head
  int64_t q0;        // first token with a query (0 for a whole prefill); sel rows start there
  int64_t list_cap;  // routed list slots the scratch holds (every slot index is checked against it)
};

// A list slot outside [0, list_cap) means the router's tables are
// inconsistent: the kernel records MOBA_ERR_DEVICE_CHECK and skips the
// access instead of touching memory outside the scratch.
__device__ __forceinline__ bool slot_ok(const WindowGeom& w, int64_t pos, int64_t n = 1) {
  if (pos >= 0 && pos + n <= w.list_cap) return true;
  record_status(MOBA_ERR_DEVICE_CHECK);
  return false;
}

// First flag word of bucket j that can hold a set bit: rows with t >= (j+1)B.
__device__ __forceinline__ int64_t bucket_word_begin(const WindowGeom& w, int j) {
  int64_t t_first = (int64_t)(j + 1) * w.B - w.w0;
  if (t_first <= 0) return 0;
  int64_t wb = t_first * w.G / 32;
  return wb < w.wwords ? wb : w.wwords;
}

// 1. grid (ceil(wwords / 4), Hkv), 128 threads: one warp per flag word (32
// group-rows); dynamic shared memory 128 * (k_eff - 1) ints. The flag words
// start zeroed (the host clears them), so only the blocks some row of the
// word picked are visited: each step takes the smallest block still pending
// in any lane, and the lanes that picked it advance to their next entry (a
// row's past entries are ascending). Every lane first copies its row's
// entries into shared memory with all loads in flight, so the steps read
// them at shared-memory latency.
constexpr int kFlagsThreads = 128;
__global__ void __launch_bounds__(kFlagsThreads) route_flags_kernel(const int32_t* __restrict__ sel, WindowGeom w,
                                                                    uint32_t* __restrict__ flags) {
  grid_dependency_sync();
  extern __shared__ int32_t ent[];  // [P][kFlagsThreads]: entry i of this thread's row at ent[i * 128 + tid]
  const int g = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int64_t word = (int64_t)blockIdx.x * (kFlagsThreads / 32) + (threadIdx.x >> 5);
  if (word >= w.wwords) return;  // a whole warp: no block-wide barrier below
  const int64_t rr = word * 32 + lane;
  const int64_t tl = rr / w.G;
  const int64_t t = w.w0 + tl;
  const bool valid = tl < w.wlen && t >= w.q0;  // a token before q0 has no query: no bits
  const int h = g * w.G + (int)(rr % w.G);
  const int bt = valid ? (int)(t / w.B) : 0;
  const int P = w.k_eff - 1;
  const int32_t* srow = sel + ((int64_t)h * (w.S - w.q0) + (valid ? t - w.q0 : 0)) * w.k_eff;
  int32_t* mine = ent + threadIdx.x;
  for (int i = 0; i < P; ++i) {
    const int v = valid ? __ldg(srow + i) : -1;
    mine[i * kFlagsThreads] = (v >= 0 && v < bt) ? v : 0x7fffffff;
  }
  __syncwarp();
  int ptr = 0;
  int cur = P > 0 ? mine[0] : 0x7fffffff;
  uint32_t* dst = flags + (int64_t)g * w.nbp * w.wwords + word;
  for (;;) {
    const int j = __reduce_min_sync(0xffffffffu, cur);
    if (j == 0x7fffffff) break;
    const bool hit = (cur == j);
    if (hit) {
      ++ptr;
      cur = ptr < P ? mine[ptr * kFlagsThreads] : 0x7fffffff;
    }
    const uint32_t bits = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) dst[(int64_t)j * w.wwords] = bits;
  }
}

__device__ __forceinline__ int block_sum_256(int v, int* scratch) {
  // fixed-order reduction: warp shuffles, then warp 0 over the 8 partials
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) scratch[threadIdx.x >> 5] = v;
  __syncthreads();
  int r = 0;
  if (threadIdx.x < 32) {
    r = threadIdx.x < 8 ? scratch[threadIdx.x] : 0;
    for (int o = 16; o > 0; o >>= 1) r += __shfl_down_sync(0xffffffffu, r, o);
  }
  __syncthreads();
  return r;  // valid in thread 0
}

// 2. grid (nbp, Hkv), 256 threads.
__global__ void __launch_bounds__(256) route_count_kernel(const uint32_t* __restrict__ flags, WindowGeom w,
                                                          int32_t* __restrict__ cnt) {
  grid_dependency_sync();
  const int j = blockIdx.x, g = blockIdx.y;
  const uint32_t* f = flags + ((int64_t)g * w.nbp + j) * w.wwords;
  int c = 0;
  for (int64_t i = bucket_word_begin(w, j) + threadIdx.x; i < w.wwords; i += 256) c += __popc(__ldg(f + i));
  __shared__ int scratch[8];
  c = block_sum_256(c, scratch);
  if (threadIdx.x == 0) cnt[g * w.nbp + j] = c;
}

// Inclusive scan over 1024 threads (fixed order).
__device__ __forceinline__ int64_t block_incl_scan_1024(int64_t v, int64_t* scratch) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int o = 1; o < 32; o <<= 1) {
    int64_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) scratch[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int64_t s = scratch[lane];
    for (int o = 1; o < 32; o <<= 1) {
      int64_t n = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += n;
    }
    scratch[lane] = s;
  }
  __syncthreads();
  if (wid > 0) v += scratch[wid - 1];
  __syncthreads();
  return v;
}

// Work-unit descriptors for the attention stage (two 128-row query tiles
// that read the same keys):
//   routed {list_start, nrows (1..256), g, j >= 0}: 256 consecutive list
//          entries of bucket (g, j);
//   own    {t0, nrows (1..128), hA | hB << 16, -nsteps}: 128 tokens of two
//          q heads of one group (hB = 0xFFFF when the group has an odd
//          head left over); with one head per group (pair_tokens), tile A
//          is tokens [t0, t0 + 128) and tile B (hB = 0xFFFE) the next 128
//          tokens of the same head and block.
// hdr[0] = routed units, hdr[1] = all units, hdr[2] = list entries,
// hdr[3] = the attention kernel's next-unit counter (zeroed here).
constexpr int kUnitRowsRouted = 256;
// 3. one CTA of 1024 threads.
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ cnt, int nbuckets,
                                                          WindowGeom w, int32_t* __restrict__ list_off,
                                                          int32_t* __restrict__ tile_off, int4* __restrict__ units,
                                                          int32_t* __restrict__ hdr) {
  grid_dependency_sync();
  __shared__ int64_t scratch[32];
  __shared__ int64_t last[2];
  int64_t carry_l = 0, carry_t = 0;
  for (int base = 0; base < nbuckets; base += 1024) {
    const int b = base + threadIdx.x;
    const int64_t c = b < nbuckets ? cnt[b] : 0;
    const int64_t nt = (c + kUnitRowsRouted - 1) / kUnitRowsRouted;
    const int64_t il = block_incl_scan_1024(c, scratch);
    const int64_t it = block_incl_scan_1024(nt, scratch);
    if (b < nbuckets) {
      list_off[b] = (int32_t)(carry_l + il - c);
      tile_off[b] = (int32_t)(carry_t + it - nt);
    }
    if (threadIdx.x == 1023) {
      last[0] = il;
      last[1] = it;
    }
    __syncthreads();
    carry_l += last[0];
    carry_t += last[1];
    __syncthreads();
  }
  const int n_routed = (int)carry_t;
  // own-block units: 128-token tiles u of the window, one unit per pair of
  // q heads of a group; tile u of block-position p = ((w0/128 + u) mod
  // (B/128)) has p + 1 key steps. Units are ordered longest first.
  // With pair_tokens (one head per group, B/128 even, w0 a multiple of 256)
  // the same scheme runs over 256-token pairs of tiles: pair v of pair
  // position p has 2p + 2 key steps (2p + 1 when the window ends after its
  // first tile).
  const int period = w.pair_tokens ? w.B / (2 * kTile) : w.B / kTile;
  const int span = w.pair_tokens ? 2 * kTile : kTile;
  const int64_t nu = (w.wlen + span - 1) / span;
  const int64_t u_off = w.w0 / span;
  const int npairs = w.pair_tokens ? 1 : (w.G + 1) / 2;
  const int per_u = w.Hkv * npairs;
  // count tiles per position p (period <= 1024 checked on the host)
  __shared__ int cntp[1024];
  __shared__ int basep[1024];
  for (int p = threadIdx.x; p < period; p += 1024) {
    // u in [0, nu) with (u_off + u) % period == p
    const int64_t first = ((int64_t)p - u_off % period + period) % period;
    cntp[p] = first < nu ? (int)((nu - 1 - first) / period + 1) : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int p = period - 1; p >= 0; --p) {  // longest first
      basep[p] = acc;
      acc += cntp[p];
    }
  }
  __syncthreads();
  for (int64_t u = threadIdx.x; u < nu; u += 1024) {
    const int p = (int)((u_off + u) % period);
    const int64_t rank = basep[p] + u / period;  // u' < u with the same p: u / period of them
    const int64_t t0 = w.w0 + u * span;
    const int nrows = (int)min((int64_t)kTile, w.w0 + w.wlen - t0);
    if (w.pair_tokens) {
      const bool has_b = t0 + kTile < w.w0 + w.wlen;
      for (int g = 0; g < w.Hkv; ++g)
        units[n_routed + rank * per_u + g] =
            make_int4((int)t0, nrows, g | ((has_b ? 0xFFFE : 0xFFFF) << 16), -(2 * p + (has_b ? 2 : 1)));
      continue;
    }
    for (int g = 0; g < w.Hkv; ++g) {
      for (int q = 0; q < npairs; ++q) {
        const int hA = g * w.G + 2 * q;
        const int hB = (2 * q + 1 < w.G) ? hA + 1 : 0xFFFF;
        units[n_routed + rank * per_u + g * npairs + q] = make_int4((int)t0, nrows, hA | (hB << 16), -(p + 1));
      }
    }
  }
  if (threadIdx.x == 0) {
    hdr[0] = n_routed;
    hdr[1] = n_routed + (int)(nu * per_u);
    hdr[2] = (int)carry_l;
    hdr[3] = 0;
  }
}

// 4. grid (nbp, Hkv), 256 threads.
__global__ void __launch_bounds__(256) route_fill_kernel(const uint32_t* __restrict__ flags,
                                                         const int32_t* __restrict__ cnt,
                                                         const int32_t* __restrict__ list_off,
                                                         const int32_t* __restrict__ tile_off, WindowGeom w,
                                                         int32_t* __restrict__ wordbase, int32_t* __restrict__ list,
                                                         int4* __restrict__ tiles) {
  grid_dependency_sync();
  const int j = blockIdx.x, g = blockIdx.y;
  const int b = g * w.nbp + j;
  const int64_t foff = (int64_t)b * w.wwords;
  const int base = list_off[b];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  __shared__ int wsum[8];
  int running = 0;
  for (int64_t c0 = bucket_word_begin(w, j); c0 < w.wwords; c0 += 256) {
    const int64_t i = c0 + threadIdx.x;
    uint32_t word = i < w.wwords ? __ldg(flags + foff + i) : 0u;
    const int c = __popc(word);
    int incl = c;
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      before += (q < wid) ? wsum[q] : 0;
      total += wsum[q];
    }
    __syncthreads();
    if (i < w.wwords) {
      int pos = base + running + before + incl - c;
      wordbase[foff + i] = pos;
      if (!slot_ok(w, pos, c)) word = 0u;
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        list[pos++] = (int32_t)(i * 32 + bit);
      }
    }
    running += total;
  }
  const int n = cnt[b];
  const int nunits = (n + kUnitRowsRouted - 1) / kUnitRowsRouted;
  for (int k = threadIdx.x; k < nunits; k += 256)
    tiles[tile_off[b] + k] =
        make_int4(base + k * kUnitRowsRouted, min(kUnitRowsRouted, n - k * kUnitRowsRouted), g, j);
}

}  // namespace moba
