// Stage 2 on the tensor cores: gate scores Q . mean(K_block)^T with the
// causal block mask, and the per-row top-(k-1) with the own block forced
// ("MoBA (Mixture of Block Attention)" project summary, "How It Works": a
// parameter-less top-k gate per query token; "MoBA - Moonshot AIが提案した
// 新しいアテンションメカニズム", "MoBAの技術的原則": no future block). Ties go
// to the lower block index.
//
// The score matrix is a GEMM: 128 query rows (group-rows rr = t*G + hl of
// one kv head g) against 64 past blocks at a time. The block means are fp32;
// they are split into two bf16 parts, hi = bf16(m) and lo = bf16(m - hi),
// and S = Q.hi^T + Q.lo^T is accumulated in fp32 in TMEM. Q is exactly bf16,
// so the only rounding beyond fp32 accumulation is |m - hi - lo| <= 2^-18 |m|
// per channel. The 128 rows of a CTA read their scores from TMEM (thread =
// row = TMEM lane) and keep the KP best (score, block) pairs in registers; a
// block enters only with a strictly larger score, so equal scores keep the
// lower index. Chunks of block means come in by TMA into a two-stage ring,
// the Q rows by cp.async, and two TMEM score buffers let the MMA of the next
// chunk run while the current one is scanned.
#pragma once

#include "common.cuh"

namespace moba {

constexpr int kGateTcThreads = 128;
constexpr int kGateBlkChunk = 64;                              // blocks per MMA chunk
constexpr uint32_t kGateQBytes = 128 * kHeadDim * 2;          // 32 KB Q tile
constexpr uint32_t kGateSplitBytes = kGateBlkChunk * kHeadDim * 2;  // 16 KB: one part of a chunk
constexpr uint32_t kGateSplitHalf = kGateSplitBytes / 2;      // one 64-channel half
constexpr int kGateSmemBytes = kGateQBytes + 2 * 2 * kGateSplitBytes + 1024 + 256;

// Block-mean rows are padded to a multiple of the chunk so a chunk never
// crosses into the next kv head.
__host__ __device__ inline int gate_rows_padded(int nbp) {
  return (nbp + kGateBlkChunk - 1) / kGateBlkChunk * kGateBlkChunk;
}

// Block means -> hi, lo bf16 [Hkv][nbp_pad][128]; padding rows are zero.
// part holds `splits` partial means per block, [Hkv][nbp][splits][128],
// added in order (one split: part is the mean itself). grid (nbp_pad, Hkv),
// 128 threads.
__global__ void __launch_bounds__(128) kmean_split_kernel(const float* __restrict__ part, int splits, int nbp,
                                                          int nbp_pad, __nv_bfloat16* __restrict__ hi,
                                                          __nv_bfloat16* __restrict__ lo) {
  grid_dependency_sync();
  const int j = blockIdx.x, g = blockIdx.y, c = threadIdx.x;
  const int64_t o = ((int64_t)g * nbp_pad + j) * kHeadDim + c;
  if (j < nbp) {
    const float* src = part + ((int64_t)g * nbp + j) * splits * kHeadDim + c;
    float m = 0.f;
    for (int sp = 0; sp < splits; ++sp) m += src[(int64_t)sp * kHeadDim];
    const __nv_bfloat16 h = __float2bfloat16_rn(m);
    hi[o] = h;
    lo[o] = __float2bfloat16_rn(m - __bfloat162float(h));
  } else {
    hi[o] = __float2bfloat16_rn(0.f);
    lo[o] = __float2bfloat16_rn(0.f);
  }
}

struct GateParams {
  const __nv_bfloat16* q;  // [S - q0][Hq][128]: the tokens with a query
  int32_t* sel;            // [Hq][S - q0][k_eff]
  int64_t S, q0;           // q0: first token with a query
  int Hq, G, B, nbp_pad, k_eff;
};

template <int KP>
__device__ __forceinline__ void gate_insert(float (&tv)[KP], int (&ti)[KP], float s, int j) {
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

// Writes sel for one row: the npast best past blocks ascending, then the own
// block bt, then -1.
template <int KP>
__device__ __forceinline__ void gate_write_row(int32_t* out, const int (&ti)[KP], int npast, int bt, int k_eff) {
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

// grid (ceil((S - q0)*G / 128), Hkv), 128 threads; row = TMEM lane = group-row
// blockIdx.x*128 + threadIdx.x.
template <int KP>
__global__ void __launch_bounds__(kGateTcThreads)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                   GateParams p) {
  grid_dependency_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sM = smem + kGateQBytes;  // 2 stages x (hi, lo)
  __shared__ uint64_t full_bar[2], mma_bar[2], drain_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int row = threadIdx.x;
  const int64_t rr0 = p.q0 * p.G + (int64_t)blockIdx.x * 128;  // this CTA's first group-row
  const int64_t rr = rr0 + row;
  const int64_t t = rr / p.G;
  const int h = g * p.G + (int)(rr % p.G);
  const bool valid = t < p.S;
  const int bt = valid ? (int)(t / p.B) : 0;
  const int P = p.k_eff - 1;
  int64_t t_last = (rr0 + 127) / p.G;
  if (t_last > p.S - 1) t_last = p.S - 1;
  const int b_cta = (int)(t_last / p.B);  // past blocks of this CTA: j < b_cta
  const int nchunks = (b_cta + kGateBlkChunk - 1) / kGateBlkChunk;

  float tv[KP];
  int ti[KP];
#pragma unroll
  for (int i = 0; i < KP; ++i) {
    tv[i] = -INFINITY;
    ti[i] = -1;
  }

  if (nchunks > 0) {
    if (threadIdx.x == 0) {
      for (int i = 0; i < 2; ++i) {
        mbar_init(&full_bar[i], 1);
        mbar_init(&mma_bar[i], 1);
      }
      mbar_init(&drain_bar, 1);
      abort_flag = 0;
      fence_barrier_init();
    }
    if (warp == 0) {
      tmem_alloc(&tmem_base, 128);
      tmem_relinquish();
    }
    // gather the 128 Q rows (16-byte copies into the 128B-swizzled layout)
    {
      const uint32_t dst0 = smem_u32(sQ);
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int idx = threadIdx.x + 128 * i;  // 2048 chunks of 16 B
        const int r = idx >> 4, c16 = idx & 15;
        const int half = c16 >> 3, c = c16 & 7;
        const int64_t rr_r = rr0 + r;
        const int64_t t_r = rr_r / p.G;
        const __nv_bfloat16* src = p.q;
        uint32_t bytes = 0;
        if (t_r < p.S) {
          src = p.q + ((t_r - p.q0) * p.Hq + g * p.G + (int)(rr_r % p.G)) * kHeadDim + c16 * 8;
          bytes = 16;
        }
        cp_async_16(dst0 + half * (kGateQBytes / 2) + r * 128 + ((c ^ (r & 7)) << 4), src, bytes);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t idesc = idesc_bf16_f32(128, kGateBlkChunk, false);
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dM = sdesc_sw128(smem_u32(sM), 16, 1024);
    const int row0 = g * p.nbp_pad;  // first mean row of this kv head
    auto load_chunk = [&](int c) {   // thread 0 only
      const int st = c & 1;
      uint8_t* dst = sM + st * 2 * kGateSplitBytes;
      mbar_arrive_expect_tx(&full_bar[st], 2 * kGateSplitBytes);
      const int r0 = row0 + c * kGateBlkChunk;
      tma_load_2d(dst, &tm_hi, &full_bar[st], 0, r0);
      tma_load_2d(dst + kGateSplitHalf, &tm_hi, &full_bar[st], 64, r0);
      tma_load_2d(dst + kGateSplitBytes, &tm_lo, &full_bar[st], 0, r0);
      tma_load_2d(dst + kGateSplitBytes + kGateSplitHalf, &tm_lo, &full_bar[st], 64, r0);
    };
    volatile int* ab = &abort_flag;
    // scores of chunk c = Q.hi^T + Q.lo^T into TMEM columns [64*(c&1), +64)
    auto issue_mma = [&](int c) -> bool {  // warp 0
      const int st = c & 1;
      if (!mbar_wait(&full_bar[st], (c >> 1) & 1, ab)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t m0 = dM + ((st * 2 * kGateSplitBytes) >> 4);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t qoff = ((kk >> 2) * (kGateQBytes / 2) + (kk & 3) * 32) >> 4;
            const uint32_t moff = (part * kGateSplitBytes + (kk >> 2) * kGateSplitHalf + (kk & 3) * 32) >> 4;
            mma_bf16_ss(tmem + st * kGateBlkChunk, dQ + qoff, m0 + moff, idesc, (part > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&mma_bar[st]);
      }
      __syncwarp();
      return true;
    };
    int loaded = 0;  // chunks thread 0 has asked TMA for
    if (threadIdx.x == 0) {
      load_chunk(0);
      loaded = 1;
      if (nchunks > 1) {
        load_chunk(1);
        loaded = 2;
      }
    }
    bool ok = true;
    if (warp == 0) ok = issue_mma(0);
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    for (int c = 0; c < nchunks; ++c) {
      if (warp == 0 && ok && c + 1 < nchunks) ok = issue_mma(c + 1);
      if (ok && !*ab) ok = mbar_wait(&mma_bar[c & 1], (c >> 1) & 1, ab);
      __syncwarp();
      tc_fence_after();
      // This row's 64 scores of chunk c: TMEM -> registers -> ring stage c & 1
      // (free: MMA(c) has read it), swizzled so that a warp's 32 rows hit
      // distinct banks. Candidates are the columns that beat the current
      // k-th best; each lane then walks only its own candidates, so a warp
      // pays for the busiest lane instead of for every column some lane needs.
      const int j0 = c * kGateBlkChunk;
      const int jn = min(kGateBlkChunk, bt - j0);  // this row's past blocks in the chunk
      float* stage = reinterpret_cast<float*>(sM + (c & 1) * 2 * kGateSplitBytes) + row * kGateBlkChunk;
      const float thr = tv[KP - 1];
      uint64_t cand = 0;
#pragma unroll
      for (int h32 = 0; h32 < 2; ++h32) {
        uint32_t sc[32];
        tmem_ld32(tmem + (c & 1) * kGateBlkChunk + lane_off + h32 * 32, sc);
        tmem_ld_wait();
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4) {
          const int k16 = h32 * 8 + q4;  // 16-byte piece of the row
          *reinterpret_cast<uint4*>(stage + ((k16 ^ (row & 15)) << 2)) =
              make_uint4(sc[4 * q4], sc[4 * q4 + 1], sc[4 * q4 + 2], sc[4 * q4 + 3]);
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int i = h32 * 32 + e;
          if (i < jn && __uint_as_float(sc[e]) > thr) cand |= 1ull << i;
        }
      }
      if (KP >= 8 && KP <= 24 && c == 0 && jn > KP) {
        // First chunk, where every column beats an empty list (short lists
        // insert cheaply and skip this): split the
        // row's jn columns into KP strided groups; the smallest group
        // maximum tau0 is met by KP distinct columns, so a column strictly
        // below it cannot reach the top KP (a tie with it still can: ties go
        // to the lower block). Columns below tau0 leave the candidate set.
        float gm[KP > 24 ? 1 : KP];
#pragma unroll
        for (int g = 0; g < (KP > 24 ? 1 : KP); ++g) gm[g] = -INFINITY;
#pragma unroll
        for (int i = 0; i < kGateBlkChunk; ++i) {
          const float sv = i < jn ? stage[(((i >> 2) ^ (row & 15)) << 2) | (i & 3)] : -INFINITY;
          gm[i % (KP > 24 ? 1 : KP)] = fmaxf(gm[i % (KP > 24 ? 1 : KP)], sv);
        }
        float tau0 = gm[0];
#pragma unroll
        for (int g = 1; g < (KP > 24 ? 1 : KP); ++g) tau0 = fminf(tau0, gm[g]);
        uint64_t keep = 0;
#pragma unroll
        for (int i = 0; i < kGateBlkChunk; ++i)
          if (stage[(((i >> 2) ^ (row & 15)) << 2) | (i & 3)] >= tau0) keep |= 1ull << i;
        cand &= keep;
      }
      while (cand) {
        const int i = __ffsll((long long)cand) - 1;
        cand &= cand - 1;
        const float sv = stage[(((i >> 2) ^ (row & 15)) << 2) | (i & 3)];
        if (sv > tv[KP - 1]) gate_insert<KP>(tv, ti, sv, j0 + i);
      }
      // every thread is done with TMEM buffer c & 1 and ring stage c & 1;
      // order this thread's generic accesses to the stage before the TMA
      // write that refills it
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (*ab) break;
      if (threadIdx.x == 0 && c + 2 < nchunks) {
        load_chunk(c + 2);
        loaded = c + 3;
      }
    }
    if (*ab) {
      // after a timeout: let every issued copy and product land before the
      // shared memory and TMEM go away (bounded waits, flag ignored)
      volatile int keep_waiting = 0;
      if (threadIdx.x == 0)
        for (int c = 0; c < loaded; ++c) mbar_wait(&full_bar[c & 1], (c >> 1) & 1, &keep_waiting, (1ull << 28));
      if (warp == 0) {
        if (elect_one()) mma_commit(&drain_bar);
        __syncwarp();
        mbar_wait(&drain_bar, 0, &keep_waiting, (1ull << 28));
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, 128);
    }
  }
  if (!valid) return;
  const int npast = min(P, bt);
  gate_write_row<KP>(p.sel + ((int64_t)h * (p.S - p.q0) + (t - p.q0)) * p.k_eff, ti, npast, bt, p.k_eff);
}

// Rows that need no scores: topk = 1 (own block only) or topk >= nblocks
// (every past block), for the tokens [q0, S). grid ceil((S - q0)*Hq / 256),
// 256 threads.
__global__ void __launch_bounds__(256) sel_fill_kernel(int32_t* __restrict__ sel, int64_t S, int64_t q0, int Hq,
                                                        int B, int k_eff, int full) {
  grid_dependency_sync();
  const int64_t n = S - q0;
  const int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (i >= n * Hq) return;
  const int h = (int)(i / n);
  const int64_t t = q0 + i % n;
  const int bt = (int)(t / B);
  int32_t* out = sel + ((int64_t)h * n + (t - q0)) * k_eff;
  if (full) {
    for (int j = 0; j < k_eff; ++j) out[j] = (j <= bt) ? j : -1;
  } else {
    out[0] = bt;
    for (int j = 1; j < k_eff; ++j) out[j] = -1;
  }
}

}  // namespace moba
