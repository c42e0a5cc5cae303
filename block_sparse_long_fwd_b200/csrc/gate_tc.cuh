// Stage 2 on the tensor cores: gate scores Q . mean(K_block)^T with the
// causal block mask, and the per-row top-(k-1) with the own block forced
// ("MoBA (Mixture of Block Attention)" project summary, "How It Works": a
// parameter-less top-k gate per query token; "MoBA - Moonshot AIが提案した
// 新しいアテンションメカニズム", "MoBAの技術的原則": no future block). Ties go
// to the lower block index.
//
// The score matrix is a GEMM: 128 query rows (group-rows rr = t*G + hl of
// one kv head g) against 32 or 64 past blocks at a time (a chunk). The block means are fp32;
// they are split into two bf16 parts, hi = bf16(m) and lo = bf16(m - hi),
// and S = Q.hi^T + Q.lo^T is accumulated in fp32 in TMEM. Q is exactly bf16,
// so the only rounding beyond fp32 accumulation is |m - hi - lo| <= 2^-18 |m|
// per channel. The 128 rows of a CTA read their scores from TMEM (thread =
// row = TMEM lane) and keep the KP best (score, block) pairs in registers; a
// block enters only with a strictly larger score, so equal scores keep the
// lower index. Q comes in by TMA (or cp.async when a tile's rows are not
// whole tokens), chunks of block means by TMA into one shared-memory stage.
// A CTA holds one Q tile, one means stage and 128 TMEM columns, so three or
// four CTAs share an SM: the scan of one CTA's rows, which bounds the
// kernel, overlaps the copies and products of the others.
#pragma once

#include "common.cuh"

namespace moba {

constexpr int kGateTcThreads = 128;
constexpr int kGatePadRows = 64;   // block-mean rows per kv head are padded to a multiple of this
constexpr int kGateBoxRows = 32;   // block-mean rows of one TMA box
constexpr int kGateScCols = 128;   // TMEM columns of a super-chunk (the scores scanned at once)
constexpr int kGatePieces = kGateScCols / 32;          // 32-column pieces of a super-chunk
constexpr uint32_t kGateQBytes = 128 * kHeadDim * 2;  // 32 KB Q tile

// Shapes that depend on the list length KP.
template <int KP>
struct GateCfg {
  // lists of up to 16 entries: 32-block chunks (a 16 KB means stage) and four
  // CTAs per SM within 128 registers a thread; longer lists take more
  // registers: 64-block chunks, and as many CTAs as fit
  static constexpr int kChunk = KP <= 16 ? 32 : 64;
  static constexpr int kMinCtas = KP <= 16 ? 4 : (KP <= 48 ? 3 : 2);
  static constexpr int kScChunks = kGateScCols / kChunk;
  static constexpr uint32_t kSplitBytes = kChunk * kHeadDim * 2;  // one part (hi or lo) of a chunk
  static constexpr uint32_t kSplitHalf = kSplitBytes / 2;          // one 64-channel half
  static constexpr int kSmemBytes = kGateQBytes + 2 * kSplitBytes + 1024 + 256;  // Q tile, one means stage
  // the bound on a row's KP-th best score comes from the maxima of kGroups
  // disjoint column groups (about 3 KP of them, a power of two, at most 32);
  // lists of more than 32 entries go without it
  static constexpr bool kBound = KP <= 32;
  static constexpr int kGroups = KP <= 2 ? 8 : (KP <= 4 ? 16 : 32);
  // the means stage doubles as the per-row score staging area (128 rows x 128 B)
  static_assert(2 * kSplitBytes >= 128 * 128, "the staging area does not fit the means stage");
  static_assert(kChunk % kGateBoxRows == 0 && kGatePadRows % kChunk == 0, "chunk shape");
  static_assert(!kBound || kGroups >= KP, "the bound needs at least KP groups");
};

// Block-mean rows are padded to a multiple of kGatePadRows so a chunk never
// crosses into the next kv head.
__host__ __device__ inline int gate_rows_padded(int nbp) {
  return (nbp + kGatePadRows - 1) / kGatePadRows * kGatePadRows;
}

// Block means -> hi, lo bf16 [Hkv][nbp_pad][128]; padding rows are zero.
// part holds `splits` partial means per block, [Hkv][nbp][splits][128],
// added in order (one split: part is the mean itself). grid (rows, Hkv),
// 128 threads: rows j0 .. j0 + gridDim.x - 1.
__global__ void __launch_bounds__(128) kmean_split_kernel(const float* __restrict__ part, int splits, int nbp,
                                                          int nbp_pad, int j0, __nv_bfloat16* __restrict__ hi,
                                                          __nv_bfloat16* __restrict__ lo) {
  grid_dependency_sync();
  const int j = j0 + (int)blockIdx.x, g = blockIdx.y, c = threadIdx.x;
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
  int64_t t_begin, t_end;  // the rows of tokens [t_begin, t_end) (q0 <= t_begin < t_end <= S)
  int Hq, G, B, nbp_pad, k_eff;
  int q_tma;               // 1: G divides 128 and tm_q is valid (Q tiles by TMA)
  int one_pass;            // 1: the grid fits one wave, so latency beats issue: no separate pass 1
};

// Sorts N values (a power of two) in descending order: a bitonic network,
// every index a compile-time constant so the values stay in registers.
template <int N>
__device__ __forceinline__ void sort_desc(float (&a)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          const float x = a[i], y = a[l];
          if ((i & k) == 0) {
            a[i] = fmaxf(x, y);
            a[l] = fminf(x, y);
          } else {
            a[i] = fminf(x, y);
            a[l] = fmaxf(x, y);
          }
        }
      }
    }
  }
}

// The smallest float above x (x finite or -inf): v > x exactly when
// v >= float_above(x). Bit arithmetic, so it holds for subnormals too.
__device__ __forceinline__ float float_above(float x) {
  const uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) return __uint_as_float(1u);  // -0: the smallest positive subnormal
  return __uint_as_float((int32_t)u >= 0 ? u + 1u : u - 1u);
}

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

// grid (ceil((t_end - t_begin)*G / 128), Hkv), 128 threads; row = TMEM lane =
// group-row (t_begin - q0)*G + blockIdx.x*128 + threadIdx.x.
//
// The CTA's past blocks are scored in super-chunks of kGateScCols columns:
// warp 0 streams each chunk's hi/lo means through the one means stage and
// issues its products into the chunk's TMEM columns. Every row then selects
// in two passes over its scores:
//   1. tau = the KP-th largest of the maxima of kGroups disjoint column
//      groups (column c in group c mod kGroups) over all the row's past
//      blocks. KP columns reach tau, so a column strictly below it cannot be
//      among the row's best KP (an equal one still can: ties go to the lower
//      block);
//   2. the columns with score >= tau that also beat the row's current KP-th
//      best (strictly: the list's blocks are lower) are inserted in
//      ascending block order into the row's sorted list.
// With 32 groups, about 13 columns per row survive (in a warp, at most ~17),
// against ~30 (~55) for the smallest of KP group maxima over one
// super-chunk, and every candidate costs a sorted insertion. When a CTA's
// blocks fill one super-chunk, both passes read the same scores; with more,
// pass 1 runs over all super-chunks first and pass 2 issues their products
// again (the products are ~2 % of the kernel's time; TMEM for all scores
// would leave room for fewer CTAs). Lists of more than 32 entries skip pass 1.
template <int KP>
__global__ void __launch_bounds__(kGateTcThreads, GateCfg<KP>::kMinCtas)
    gate_tc_kernel(const __grid_constant__ CUtensorMap tm_hi, const __grid_constant__ CUtensorMap tm_lo,
                   const __grid_constant__ CUtensorMap tm_q, GateParams p) {
  using Cfg = GateCfg<KP>;
  constexpr int kChunk = Cfg::kChunk;
  constexpr int NG = Cfg::kGroups;
  grid_dependency_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sM = smem + kGateQBytes;  // the means stage (hi, lo); doubles as the score staging area
  __shared__ uint64_t full_bar, mma_bar, sc_bar, drain_bar, q_bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int g = blockIdx.y;
  const int warp = threadIdx.x >> 5;
  const int row = threadIdx.x;
  // group-row rr = t * G + hl; this CTA's rows start at rr0 = t_cta * G + rem0
  const uint32_t G = (uint32_t)p.G;
  const int64_t bxr = (p.t_begin - p.q0) * p.G + (int64_t)blockIdx.x * 128;
  const int64_t t_cta_off = bxr / p.G;  // the one 64-bit division of a thread
  const uint32_t rem0 = (uint32_t)(bxr - t_cta_off * p.G);
  const int64_t t_cta = p.q0 + t_cta_off;  // first token of this CTA's group-rows
  const uint32_t xr = rem0 + (uint32_t)row;
  const uint32_t tr = udiv32(xr, G);
  const int64_t t = t_cta + tr;
  const int h = g * p.G + (int)(xr - tr * G);
  const bool valid = t < p.t_end;
  const int bt = valid ? (int)udiv32((uint32_t)t, (uint32_t)p.B) : 0;
  const int P = p.k_eff - 1;
  int64_t t_last = t_cta + udiv32(rem0 + 127u, G);
  if (t_last > p.t_end - 1) t_last = p.t_end - 1;
  const int b_cta = (int)udiv32((uint32_t)t_last, (uint32_t)p.B);  // past blocks of this CTA: j < b_cta
  const int nchunks = (b_cta + kChunk - 1) / kChunk;

  float tv[KP];
  int ti[KP];
#pragma unroll
  for (int i = 0; i < KP; ++i) {
    tv[i] = -INFINITY;
    ti[i] = -1;
  }

  if (nchunks > 0) {
    uint32_t ncols = 32;  // a power of two >= 32 covering one super-chunk
    while ((int)ncols < min(nchunks, Cfg::kScChunks) * kChunk) ncols <<= 1;
    if (threadIdx.x == 0) {
      mbar_init(&full_bar, 1);
      mbar_init(&mma_bar, 1);
      mbar_init(&sc_bar, 1);
      mbar_init(&drain_bar, 1);
      mbar_init(&q_bar, 1);
      abort_flag = 0;
      fence_barrier_init();
    }
    const int row0 = g * p.nbp_pad;  // first mean row of this kv head
    // one lane of warp 0: the k-th chunk asked for completes phase k of
    // full_bar (chunks come in the order they are used)
    auto load_chunk = [&](int c) {
      mbar_arrive_expect_tx(&full_bar, 2 * Cfg::kSplitBytes);
      const int r0 = row0 + c * kChunk;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int bx = 0; bx < kChunk / kGateBoxRows; ++bx)
            tma_load_2d(sM + part * Cfg::kSplitBytes + half * Cfg::kSplitHalf + bx * kGateBoxRows * 128,
                        part ? &tm_lo : &tm_hi, &full_bar, half * 64, r0 + bx * kGateBoxRows);
        }
      }
    };
    // the first chunk of means does not depend on Q: its copy runs while the
    // Q rows come in (the thread that initialised the barriers issues it)
    if (threadIdx.x == 0) {
      if (p.q_tma) {
        // the CTA's 128 group-rows are 128 / G whole tokens x G heads: one
        // box (64 channels x G heads x 128/G tokens, 128B swizzle) per half
        // lands them in the layout the MMA reads (rows past S read zeros)
        mbar_arrive_expect_tx(&q_bar, kGateQBytes);
        const int tok = (int)(t_cta - p.q0);
        tma_load_3d(sQ, &tm_q, &q_bar, 0, g * p.G, tok);
        tma_load_3d(sQ + kGateQBytes / 2, &tm_q, &q_bar, 64, g * p.G, tok);
      }
      load_chunk(0);
    }
    if (warp == 0) {
      __syncwarp();
      tmem_alloc(&tmem_base, ncols);
      tmem_relinquish();
    }
    // gather the 128 Q rows (16-byte copies into the 128B-swizzled layout)
    if (!p.q_tma) {
      const uint32_t dst0 = smem_u32(sQ);
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int idx = threadIdx.x + 128 * i;  // 2048 chunks of 16 B
        const int r = idx >> 4, c16 = idx & 15;
        const int half = c16 >> 3, c = c16 & 7;
        const uint32_t x = rem0 + (uint32_t)r;
        const uint32_t dt = udiv32(x, G);
        const int64_t t_r = t_cta + dt;
        const __nv_bfloat16* src = p.q;
        uint32_t bytes = 0;
        if (t_r < p.t_end) {
          src = p.q + ((t_r - p.q0) * p.Hq + g * p.G + (int)(x - dt * G)) * kHeadDim + c16 * 8;
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
    if (p.q_tma && warp == 0) {
      // the products read Q: warp 0 (the issuer) waits for its copy (a
      // timeout sets the abort flag, and nothing is issued)
      mbar_wait(&q_bar, 0, &abort_flag);
      __syncwarp();
    }
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t idesc = idesc_bf16_f32(128, kChunk, false);
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dM = sdesc_sw128(smem_u32(sM), 16, 1024);
    volatile int* ab = &abort_flag;
    int loaded = 1;          // chunks asked of TMA so far
    int seq = 0;             // chunks whose products were issued (warp 0): phases of full_bar, mma_bar
    bool prefetched = false;  // warp 0: the next phase's first chunk is already on its way
    // staging of one 32-column piece of scores per row (for the insertions,
    // which index columns per lane): 128 B per row in the means stage, 16-byte
    // pieces swizzled by row so that 8 consecutive rows hit distinct banks
    float* stg = reinterpret_cast<float*>(sM) + row * 32;
    const int nsc = (nchunks + Cfg::kScChunks - 1) / Cfg::kScChunks;
    // phases: pass 1 over the super-chunks, then pass 2 over them again; one
    // super-chunk (or no bound, or a grid of one wave, where each CTA's chain
    // of copies and products is the kernel's time): the passes share each
    // phase's scores. Then the bound grows phase by phase: the maxima are
    // sorted in place and later columns fold into the sorted slots, so the
    // NG slots still hold NG distinct columns and their KP-th largest is
    // still a lower bound on the row's KP-th best.
    const bool two_pass = Cfg::kBound && nsc > 1 && !p.one_pass;
    const int nphase = two_pass ? 2 * nsc : nsc;
    float gm[NG];
#pragma unroll
    for (int i = 0; i < NG; ++i) gm[i] = -INFINITY;
    float tau = -INFINITY;
    for (int ph = 0; ph < nphase; ++ph) {
      if (*ab) break;
      const int sc = ph < nsc ? ph : ph - nsc;
      const bool pass1_only = two_pass && ph < nsc;           // group maxima, no insertions
      const bool maxima = Cfg::kBound && (pass1_only || !two_pass);
      const int c_lo = Cfg::kScChunks * sc;
      const int nc = min(Cfg::kScChunks, nchunks - c_lo);
      if (warp == 0) {
        // scores of this super-chunk: chunk c_lo + c into TMEM columns
        // c * kChunk (the first phase's first chunk is already on its way)
        if (ph > 0 && !prefetched) {
          if (elect_one()) load_chunk(c_lo);
          __syncwarp();
          ++loaded;
        }
        prefetched = false;
        for (int c = 0; c < nc; ++c, ++seq) {
          if (!mbar_wait(&full_bar, seq & 1, ab)) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int part = 0; part < 2; ++part) {
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t qoff = ((kk >> 2) * (kGateQBytes / 2) + (kk & 3) * 32) >> 4;
                const uint32_t moff = (part * Cfg::kSplitBytes + (kk >> 2) * Cfg::kSplitHalf + (kk & 3) * 32) >> 4;
                mma_bf16_ss(tmem + c * kChunk, dQ + qoff, dM + moff, idesc, (part > 0 || kk > 0) ? 1u : 0u);
              }
            }
            mma_commit(&mma_bar);
          }
          __syncwarp();
          const bool more = c + 1 < nc;
          // a pass-1 phase stages no scores: the next phase's first chunk can
          // come in while the rows take their maxima
          const bool ahead = !more && pass1_only;
          if (more || ahead) {
            // the stage is free once this chunk's products have read it
            if (!mbar_wait(&mma_bar, seq & 1, ab)) break;
            const int next = more ? c_lo + c + 1 : (ph + 1 < nsc ? c_lo + nc : 0);
            if (elect_one()) load_chunk(next);
            __syncwarp();
            ++loaded;
            prefetched = ahead;
          }
        }
        if (elect_one()) mma_commit(&sc_bar);
        __syncwarp();
      }
      if (*ab || !mbar_wait(&sc_bar, ph & 1, ab)) break;
      __syncwarp();
      tc_fence_after();
      // ---- selection over this super-chunk's columns [0, nc * kChunk)
      const int jb = sc * kGateScCols;                   // block of column 0
      const int jn = max(0, min(nc * kChunk, bt - jb));  // this row's past blocks here
      if (maxima) {
        // pass 1: group maxima (column c of a super-chunk is in group c mod NG)
#pragma unroll
        for (int pc = 0; pc < kGatePieces; ++pc) {
          if (pc * 32 < nc * kChunk) {
            uint32_t r[32];
            tmem_ld32(tmem + pc * 32 + lane_off, r);
            tmem_ld_wait();
            const int rem = jn - pc * 32;  // columns of this piece that are the row's past blocks
            if (rem >= 32) {
#pragma unroll
              for (int e = 0; e < 32; ++e) gm[e % NG] = fmaxf(gm[e % NG], __uint_as_float(r[e]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) gm[e % NG] = fmaxf(gm[e % NG], e < rem ? __uint_as_float(r[e]) : -INFINITY);
            }
          }
        }
        if (!two_pass || ph == nsc - 1) {
          // the maxima so far are in: tau = the KP-th largest (-inf while
          // fewer than KP slots hold a past block)
          sort_desc<NG>(gm);
          tau = gm[KP - 1];
        }
      }
      if (!pass1_only) {
        // pass 2: the candidates of this super-chunk into the row's list
#pragma unroll
        for (int pc = 0; pc < kGatePieces; ++pc) {
          if (pc * 32 < nc * kChunk) {
            uint32_t r[32];
            tmem_ld32(tmem + pc * 32 + lane_off, r);
            tmem_ld_wait();
            // a column is a candidate when it is one of the row's past blocks,
            // reaches tau and beats the row's KP-th best; the last two tests
            // are one: v >= max(tau, the float just above the KP-th best)
            const float lo = fmaxf(tau, float_above(tv[KP - 1]));
            uint32_t cand = 0;
#pragma unroll
            for (int e = 0; e < 32; ++e) cand |= (__uint_as_float(r[e]) >= lo) ? (1u << e) : 0u;
            const int rem = jn - pc * 32;
            cand &= rem >= 32 ? 0xffffffffu : (rem > 0 ? (1u << rem) - 1u : 0u);
            if (__any_sync(0xffffffffu, cand != 0u)) {
#pragma unroll
              for (int k4 = 0; k4 < 8; ++k4)
                *reinterpret_cast<uint4*>(stg + ((k4 ^ (row & 7)) << 2)) =
                    make_uint4(r[4 * k4], r[4 * k4 + 1], r[4 * k4 + 2], r[4 * k4 + 3]);
              __syncwarp();
              while (cand) {
                const int e = __ffs(cand) - 1;
                cand &= cand - 1;
                const float sv = stg[(((e >> 2) ^ (row & 7)) << 2) | (e & 3)];
                if (sv > tv[KP - 1]) gate_insert<KP>(tv, ti, sv, jb + pc * 32 + e);
              }
              __syncwarp();
            }
          }
        }
      }
      // every thread is done with TMEM and the staging area; order the
      // staging writes before the TMA writes that refill the stage
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    }
    if (*ab) {
      // after a timeout: let every issued copy and product land before the
      // shared memory and TMEM go away (bounded waits, flag ignored)
      volatile int keep_waiting = 0;
      if (warp == 0) {
        if (elect_one()) {
          // one stage: at most one copy of means is in flight, the last one
          // asked for, and only if its products were never issued
          if (seq < loaded) mbar_wait(&full_bar, (loaded - 1) & 1, &keep_waiting, (1ull << 28));
          if (p.q_tma) mbar_wait(&q_bar, 0, &keep_waiting, (1ull << 28));
        }
        __syncwarp();
        if (elect_one()) mma_commit(&drain_bar);
        __syncwarp();
        mbar_wait(&drain_bar, 0, &keep_waiting, (1ull << 28));
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, ncols);
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
