// Stage 4: block attention on the 5th-generation tensor cores.
//
// Each work tile is 128 query rows against the keys of one KV block:
//   routed tile: up to 128 rows routed to past block j of kv head g (from the
//     router's list), attending all B keys of block j, no mask (j < t/B);
//   own tile:    128 consecutive tokens of one q head attending their own
//     block from its start up to the tile, causal mask on the diagonal step
//     ("MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
//     "MoBAの技術的原則": a causal mask applies inside the current block).
// Both write a normalised partial output O_i (fp32) and its natural-log
// lse_i; the merge stage combines them. The FlashAttention-style online
// softmax ("MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
// high-performance implementation: FlashAttention plus MoE techniques) runs
// per 128-key step:
//   S = Q K^T             tcgen05.mma, A = Q and B = K from shared memory,
//                         fp32 accumulator in TMEM (two S buffers)
//   P = exp2(S*c - m)     softmax warps read S from TMEM, one row per thread
//   O += P V              tcgen05.mma, A = P from shared memory, B = V
//                         (MN-major) from shared memory, O in TMEM.
// The running max is only moved (and O, l rescaled) when it grows by more
// than 8 in log2 units, so most steps skip the O rescale.
//
// Warp roles (256 threads, one CTA per SM, persistent over the tile list):
//   warps 0-3  softmax + epilogue (thread = row = TMEM lane)
//   warp 4     TMA producer for K/V tiles (3-D tensor maps, 128B swizzle)
//   warp 5     TMEM owner and single-thread MMA issuer
//   warps 6-7  Q row gather (cp.async, 16 B per copy, swizzled by hand)
// Every mbarrier wait is bounded; a timeout sets an error status and the
// whole CTA winds down without trapping.
#pragma once

#include "common.cuh"

namespace moba {

constexpr int kAttnThreads = 256;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = kTile * kHeadDim * 2;  // 32 KB: 128 rows x 128 bf16
constexpr uint32_t kHalfBytes = kTileBytes / 2;        // one 64-column half
constexpr int kAttnSmemBytes = (2 + 2 * kStages + 1) * kTileBytes + 1024 + 256;

struct AttnParams {
  const __nv_bfloat16* q;   // [S][Hq][128]
  const int32_t* list;      // group-rows of the window, per bucket
  const int4* tiles;        // tile descriptors
  const int32_t* hdr;       // [1] = number of tiles
  float* part_o;            // [list entries][128]
  float* part_lse;          // [list entries]
  float* own_o;             // [wlen][Hq][128]
  float* own_lse;           // [wlen][Hq]
  int64_t S, w0;
  int Hq, G, B;
  float scale_log2;         // log2(e) / sqrt(128)
};

struct AttnShared {
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full, o_done, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct TileInfo {
  bool own;
  int nrows, nsteps;
  int g, h;        // kv head; q head (own tiles)
  int64_t key0;    // first key of step 0
  int list_start;  // routed
  int64_t t0;      // own
};

__device__ __forceinline__ TileInfo decode_tile(const AttnParams& p, int idx) {
  const int4 d = p.tiles[idx];
  TileInfo ti;
  ti.nrows = d.y;
  if (d.w < 0) {
    ti.own = true;
    ti.nsteps = -d.w;
    ti.t0 = d.x;
    ti.h = d.z;
    ti.g = d.z / p.G;
    ti.key0 = ti.t0 - (int64_t)(ti.nsteps - 1) * kTile;
    ti.list_start = 0;
  } else {
    ti.own = false;
    ti.list_start = d.x;
    ti.g = d.z;
    ti.h = 0;
    ti.key0 = (int64_t)d.w * p.B;
    ti.nsteps = p.B / kTile;
    ti.t0 = 0;
  }
  return ti;
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                              // 2 buffers
  uint8_t* sK = sQ + 2 * kTileBytes;               // kStages buffers
  uint8_t* sV = sK + kStages * kTileBytes;         // kStages buffers
  uint8_t* sP = sV + kStages * kTileBytes;         // 1 buffer
  AttnShared* sh = reinterpret_cast<AttnShared*>(sP + kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.hdr[1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh->q_full[i], 64);
      mbar_init(&sh->q_empty[i], 1);
      mbar_init(&sh->s_full[i], 1);
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh->kv_full[i], 1);
      mbar_init(&sh->kv_empty[i], 1);
    }
    mbar_init(&sh->p_full, 128);
    mbar_init(&sh->o_done, 1);
    mbar_init(&sh->o_free, 128);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t tS[2] = {tmem, tmem + 128};
  const uint32_t tO = tmem + 256;
  volatile int* abort_flag = &sh->abort_flag;

  if (warp < 4) {
    // ------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x;  // TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const TileInfo ti = decode_tile(p, tile);
      float m_run = -INFINITY, l_run = 0.f;
      for (int s = 0; s < ti.nsteps; ++s) {
        const uint32_t cur = it + s;
        const int sb = cur & 1;
        if (!mbar_wait(&sh->s_full[sb], (cur >> 1) & 1, abort_flag)) goto done;
        __syncwarp();
        tc_fence_after();
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tS[sb] + lane_off + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]) * p.scale_log2;
        }
        // causal mask on the diagonal step of an own tile: key > query
        const bool diag = ti.own && (s == ti.nsteps - 1);
        if (diag) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > row) x[e] = -INFINITY;
        }
        float mx = x[0];
#pragma unroll
        for (int e = 1; e < 128; ++e) mx = fmaxf(mx, x[e]);
        const float m_new = fmaxf(m_run, mx);
        float m_ref = m_run, factor = 1.f;
        bool rescale = false;
        if (s == 0) {
          m_ref = m_new;
        } else if (m_new > m_run + 8.f) {
          m_ref = m_new;
          factor = ex2_approx(m_run - m_new);
          rescale = true;
        }
        float sum = 0.f;
        uint32_t pk[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) {
          const float a = ex2_approx(x[2 * e] - m_ref);
          const float b = ex2_approx(x[2 * e + 1] - m_ref);
          sum += a + b;
          pk[e] = pack_bf16x2(a, b);
        }
        l_run = l_run * factor + sum;
        m_run = m_ref;
        // the previous P.V must be done before P is overwritten / O rescaled
        if (s > 0) {
          if (!mbar_wait(&sh->o_done, (cur - 1) & 1, abort_flag)) goto done;
          __syncwarp();
          tc_fence_after();
        }
        if (rescale) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(tO + lane_off + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * factor);
            tmem_st32(tO + lane_off + c * 32, r);
          }
          tmem_st_wait();
        }
        // P row -> shared memory, K-major, 128B swizzle (16-byte chunk c of
        // row r lands at chunk c ^ (r & 7))
#pragma unroll
        for (int c16 = 0; c16 < 16; ++c16) {
          const int half = c16 >> 3, c = c16 & 7;
          uint8_t* dst = sP + half * kHalfBytes + row * 128 + ((c ^ (row & 7)) << 4);
          *reinterpret_cast<uint4*>(dst) = make_uint4(pk[c16 * 4], pk[c16 * 4 + 1], pk[c16 * 4 + 2], pk[c16 * 4 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh->p_full);
      }
      {
        // epilogue: O / l and lse
        const uint32_t last = it + ti.nsteps - 1;
        if (!mbar_wait(&sh->o_done, last & 1, abort_flag)) goto done;
        __syncwarp();
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const float lse = (m_run + log2f(l_run)) * 0.69314718055994530942f;
        float* dst_o;
        float* dst_lse;
        if (ti.own) {
          const int64_t r = (ti.t0 + row - p.w0) * p.Hq + ti.h;
          dst_o = p.own_o + r * kHeadDim;
          dst_lse = p.own_lse + r;
        } else {
          const int64_t r = (int64_t)ti.list_start + row;
          dst_o = p.part_o + r * kHeadDim;
          dst_lse = p.part_lse + r;
        }
        const bool write = row < ti.nrows;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + c * 32, r);
          tmem_ld_wait();
          if (write) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst_o + c * 32 + e) =
                  make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                              __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
          }
        }
        if (write) *dst_lse = lse;
        tc_fence_before();
        mbar_arrive(&sh->o_free);
      }
      it += ti.nsteps;
    }
  } else if (warp == 4) {
    // ------------------------------------------------ K/V TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
        const TileInfo ti = decode_tile(p, tile);
        for (int s = 0; s < ti.nsteps; ++s, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&sh->kv_empty[st], ((it / kStages) & 1) ^ 1, abort_flag)) goto drain_kv;
          mbar_arrive_expect_tx(&sh->kv_full[st], 2 * kTileBytes);
          const int key = (int)(ti.key0 + (int64_t)s * kTile);
          uint8_t* k_dst = sK + st * kTileBytes;
          uint8_t* v_dst = sV + st * kTileBytes;
          tma_load_3d(k_dst, &tmap_k, &sh->kv_full[st], 0, ti.g, key);
          tma_load_3d(k_dst + kHalfBytes, &tmap_k, &sh->kv_full[st], 64, ti.g, key);
          tma_load_3d(v_dst, &tmap_v, &sh->kv_full[st], 0, ti.g, key);
          tma_load_3d(v_dst + kHalfBytes, &tmap_v, &sh->kv_full[st], 64, ti.g, key);
        }
      }
    drain_kv:
      // make sure no TMA write is still in flight when the CTA ends: the
      // last kStages loads are waited for (bounded) on their full barriers
      if (*abort_flag) {
        volatile int keep_waiting = 0;
        for (uint32_t k = (it > (uint32_t)kStages ? it - kStages : 0); k < it; ++k)
          mbar_wait(&sh->kv_full[k % kStages], (k / kStages) & 1, &keep_waiting, 100000000ull);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
      const uint32_t aQ0 = smem_u32(sQ), aK0 = smem_u32(sK), aV0 = smem_u32(sV), aP = smem_u32(sP);
      uint32_t it = 0, n = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++n) {
        const TileInfo ti = decode_tile(p, tile);
        const int qb = n & 1;
        if (!mbar_wait(&sh->q_full[qb], (n >> 1) & 1, abort_flag)) goto mma_done;
        tc_fence_after();
        const uint32_t aQ = aQ0 + qb * kTileBytes;
        // S_{step} = Q K_step^T into S buffer (step & 1)
        auto issue_s = [&](uint32_t step) -> bool {
          const int st = step % kStages;
          if (!mbar_wait(&sh->kv_full[st], (step / kStages) & 1, abort_flag)) return false;
          tc_fence_after();
          const uint32_t aK = aK0 + st * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_bf16_ss(tS[step & 1], sdesc_sw128(aQ + off, 16, 1024), sdesc_sw128(aK + off, 16, 1024), idesc_s,
                        kk > 0);
          }
          mma_commit(&sh->s_full[step & 1]);
          return true;
        };
        if (!issue_s(it)) goto mma_done;
        for (int s = 0; s < ti.nsteps; ++s) {
          const uint32_t cur = it + s;
          if (s + 1 < ti.nsteps && !issue_s(cur + 1)) goto mma_done;
          if (!mbar_wait(&sh->p_full, cur & 1, abort_flag)) goto mma_done;
          if (s == 0 && n > 0 && !mbar_wait(&sh->o_free, (n - 1) & 1, abort_flag)) goto mma_done;
          tc_fence_after();
          const int st = cur % kStages;
          const uint32_t aV = aV0 + st * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t offp = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_bf16_ss(tO, sdesc_sw128(aP + offp, 16, 1024), sdesc_sw128(aV + kk * 2048, kHalfBytes, 1024),
                        idesc_o, (s > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&sh->kv_empty[st]);
          mma_commit(&sh->o_done);
        }
        mma_commit(&sh->q_empty[qb]);
        it += ti.nsteps;
      }
    mma_done:
      // all issued MMAs must finish before TMEM is released
      mma_commit(&sh->drain);
      volatile int keep_waiting = 0;
      mbar_wait(&sh->drain, 0, &keep_waiting, 100000000ull);
    }
  } else {
    // ------------------------------------------------ Q gather (warps 6, 7)
    const int gt = threadIdx.x - 192;  // 0..63
    uint32_t n = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++n) {
      const TileInfo ti = decode_tile(p, tile);
      const int qb = n & 1;
      if (!mbar_wait(&sh->q_empty[qb], ((n >> 1) & 1) ^ 1, abort_flag)) break;
      const uint32_t dst0 = smem_u32(sQ + qb * kTileBytes);
#pragma unroll 4
      for (int i = 0; i < 32; ++i) {
        const int idx = gt + 64 * i;  // 2048 chunks of 16 B
        const int r = idx >> 4, c16 = idx & 15;
        const int half = c16 >> 3, c = c16 & 7;
        const __nv_bfloat16* src = p.q;
        uint32_t bytes = 0;
        if (r < ti.nrows) {
          int64_t t;
          int h;
          if (ti.own) {
            t = ti.t0 + r;
            h = ti.h;
          } else {
            const int rr = __ldg(p.list + ti.list_start + r);
            t = p.w0 + rr / p.G;
            h = ti.g * p.G + rr % p.G;
          }
          src = p.q + (t * p.Hq + h) * kHeadDim + c16 * 8;
          bytes = 16;
        }
        cp_async_16(dst0 + half * kHalfBytes + r * 128 + ((c ^ (r & 7)) << 4), src, bytes);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&sh->q_full[qb]);
    }
    cp_async_wait_all();
  }
done:
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace moba
