// Stage 4: block attention on the 5th-generation tensor cores.
//
// A work unit is a pair of 128-row query tiles (A and B) that read the same
// keys, so one K/V stream feeds M = 256 rows:
//   routed unit: up to 256 rows routed to past block j of kv head g (rows
//     [0,128) form tile A, [128,256) tile B), attending all B keys of block
//     j without a mask (j < t/B);
//   own unit:    128 consecutive tokens of two q heads of one GQA group
//     (tile B absent when the group has no second head left), attending
//     their own block from its start up to the tile, causal mask on the
//     diagonal step ("MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
//     "MoBAの技術的原則": a causal mask applies inside the current block).
// Every tile writes a normalised partial output O_i (fp16: a convex
// combination of bf16 values, so |O_i| <= max |v|, at 2^-11 relative
// rounding, four times finer than the bf16 output) and its
// natural-log lse_i; the merge stage combines them. The online softmax
// (FlashAttention-style; the same page credits MoBA's speed to FlashAttention
// plus MoE techniques) runs per 128-key step, per tile X in {A, B}:
//   S_X = Q_X K^T      tcgen05.mma (M = N = 128), Q and K from shared memory
//                      (128B swizzle), fp32 accumulator in TMEM
//   P_X = 2^(S_X*c-m)  the tile's softmax warpgroup reads S_X from TMEM
//                      (thread = row = TMEM lane) into registers and writes
//                      bf16 P_X to its own TMEM columns
//   O_X += P_X V       tcgen05.mma with A = P_X from TMEM, B = V (MN-major)
//                      from shared memory, O_X in TMEM.
// One S buffer serves both tiles: S_A(s), S_B(s), S_A(s+1), ... each issued
// as soon as the previous S has been read into the registers of its
// softmax warpgroup. Because P has columns of its own, the next S never
// waits for a P.V product, and both tiles' softmaxes run concurrently while
// the tensor core works through S_A(s+1), PV_A(s), S_B(s+1), PV_B(s).
// The running max moves (and O, l are rescaled) only when it grows by more
// than 8 in log2 units. Every exponential is one MUFU ex2: with the tensor
// core this busy the SM runs at its power limit, and moving a share of them
// to a polynomial on the FMA pipe cost more (issue slots, energy) than it
// saved on the MUFU unit (measured at 1M tokens: 1,124 against 1,186 TFLOP/s).
//
// TMEM (512 columns): S 0..127, P_A 128..191, P_B 192..255 (bf16 pairs),
// O_A 256..383, O_B 384..511.
// Warp roles (384 threads, one CTA per SM, persistent over the unit list):
//   warps 0-3  softmax + epilogue of tile A     warps 4-7  same for tile B
//   warp 8     TMA producer for K/V (3-D tensor maps, 128B swizzle)
//   warp 9     TMEM owner; issues the S = Q K^T products
//   warp 10    Q row gather (cp.async, 16 B per copy, swizzled by hand)
//   warp 11    issues the O += P V products
// Two issuers keep the tensor core fed: an MMA issue returns at about the
// rate the tensor core executes, so one issuer's barrier waits and fences
// between its product groups would leave the pipe idle; with S and P.V
// issued by different warps, one issuer's MMAs run while the other waits.
// Every mbarrier wait is bounded; a timeout sets an error status and the
// whole CTA winds down without trapping.
#pragma once

#include "common.cuh"

namespace moba {

constexpr int kAttnThreads = 384;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = kTile * kHeadDim * 2;  // 32 KB: 128 rows x 128 bf16
constexpr uint32_t kHalfBytes = kTileBytes / 2;        // one 64-column half
constexpr int kUnitRows = 2 * kTile;                   // rows of a routed unit
constexpr int kAttnSmemBytes = (2 + 2 * kStages) * kTileBytes + 1024 + 512;
constexpr uint32_t kNoHead = 0xFFFFu;
constexpr uint32_t kNextTile = 0xFFFEu;  // own tile B: the next 128 tokens of tile A's head

// TMEM columns
constexpr uint32_t kTmemS = 0;
constexpr uint32_t kTmemP = 128;  // + 64 * X
constexpr uint32_t kTmemO = 256;  // + 128 * X

struct AttnParams {
  const __nv_bfloat16* q;   // [S - q0][Hq][128]: the tokens with a query
  const int32_t* list;      // group-rows of the window, per bucket
  const int4* units;        // unit descriptors
  int32_t* hdr;             // [1] = number of units, [3] = next-unit counter (starts at 0)
  __half* part_o;           // [list entries][128], fp16
  float* part_lse;          // [list entries]
  __half* own_o;            // [wlen][Hq][128], fp16
  float* own_lse;           // [wlen][Hq]
  int64_t S, w0, q0;        // q0: first token with a query
  int64_t wlen;             // tokens of the window
  int Hq, G, B;
  float scale_log2;         // log2(e) / sqrt(128)
};

constexpr int kRing = 8;                               // unit indices in flight per CTA
constexpr uint32_t kRingReaders = 1 + 32 + 32 + 256 + 32;  // producer lane, two issuer warps, softmax, gather

struct AttnShared {
  uint64_t ring_full[kRing], ring_empty[kRing];
  int ring[kRing];
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[kStages], k_empty[kStages], v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free, p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Unit descriptor: routed {list_start, nrows (1..256), g, j >= 0};
//                  own    {t0, nrows (1..128), hA | hB << 16, -nsteps}.
struct UnitInfo {
  bool own, has_b;
  int nsteps;
  int g;
  int64_t key0;    // first key of step 0
  int rows[2];     // valid rows of tile A, B
  int h[2];        // own: q heads of tile A, B
  int list0[2];    // routed: first list slot of tile A, B
  int64_t tq[2];   // own: first token of tile A, B
  int diag[2];     // own: the step whose keys start at tile X's first token
};

__device__ __forceinline__ UnitInfo decode_unit(const AttnParams& p, int idx) {
  const int4 d = p.units[idx];
  UnitInfo u;
  if (d.w < 0) {
    u.own = true;
    u.nsteps = -d.w;
    u.tq[0] = d.x;
    u.h[0] = d.z & 0xFFFF;
    const uint32_t hb = (uint32_t)d.z >> 16;
    u.g = u.h[0] / p.G;
    u.rows[0] = d.y;
    u.list0[0] = u.list0[1] = 0;
    if (hb == kNextTile) {
      // the same head's next 128 tokens: one more key step than tile A
      u.has_b = true;
      u.h[1] = u.h[0];
      u.tq[1] = u.tq[0] + kTile;
      u.rows[1] = (int)min((int64_t)kTile, p.S - u.tq[1]);
      u.diag[0] = u.nsteps - 2;
      u.diag[1] = u.nsteps - 1;
    } else {
      u.has_b = hb != kNoHead;
      u.h[1] = (int)hb;
      u.tq[1] = u.tq[0];
      u.rows[1] = u.has_b ? d.y : 0;
      u.diag[0] = u.diag[1] = u.nsteps - 1;
    }
    u.key0 = u.tq[0] - (int64_t)u.diag[0] * kTile;
  } else {
    u.own = false;
    u.nsteps = p.B / kTile;
    u.g = d.z;
    u.key0 = (int64_t)d.w * p.B;
    u.rows[0] = min(d.y, kTile);
    u.rows[1] = max(d.y - kTile, 0);
    u.has_b = u.rows[1] > 0;
    u.list0[0] = d.x;
    u.list0[1] = d.x + kTile;
    u.h[0] = u.h[1] = 0;
    u.tq[0] = u.tq[1] = 0;
    u.diag[0] = u.diag[1] = u.nsteps;
  }
  return u;
}

// P = 2^(s*c - m) for one 128-column row of S held as raw fp32 bits in r,
// on column pairs with packed fp32 arithmetic, into 64 registers of bf16
// pairs (pk[i] = columns 2i, 2i+1). Row sums accumulate into sum2 (four
// packed pairs).
__device__ __forceinline__ void exp_row(const uint32_t (&r)[128], uint64_t c2, uint64_t nm2, uint64_t (&sum2)[4],
                                        uint32_t (&pk)[64]) {
#pragma unroll
  for (int e = 0; e < 128; e += 2) {
    const uint64_t x2 = f2_fma((uint64_t)r[e] | ((uint64_t)r[e + 1] << 32), c2, nm2);
    const float a = ex2_approx(f2_lo(x2));
    const float b = ex2_approx(f2_hi(x2));
    sum2[(e >> 1) & 3] = f2_add(sum2[(e >> 1) & 3], f2_pack(a, b));
    pk[e >> 1] = pack_bf16x2(a, b);
  }
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                AttnParams p) {
  grid_dependency_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                         // tile A, tile B
  uint8_t* sK = sQ + 2 * kTileBytes;          // kStages buffers
  uint8_t* sV = sK + kStages * kTileBytes;    // kStages buffers
  AttnShared* sh = reinterpret_cast<AttnShared*>(sV + kStages * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sh->q_full[x], 32);  // the gather warp's lanes
      mbar_init(&sh->q_empty[x], 1);
      mbar_init(&sh->s_full[x], 1);
      mbar_init(&sh->p_full[x], 128);
      mbar_init(&sh->pv_done[x], 1);
    }
    mbar_init(&sh->s_free, 4);  // one lane of each warp of the consuming warpgroup
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh->k_full[i], 1);
      mbar_init(&sh->k_empty[i], 1);
      mbar_init(&sh->v_full[i], 1);
      mbar_init(&sh->v_empty[i], 1);
    }
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&sh->ring_full[i], 1);
      mbar_init(&sh->ring_empty[i], kRingReaders);
    }
    mbar_init(&sh->drain, 2);  // one commit from each issuer
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort_flag = &sh->abort_flag;
  // Work units are handed out dynamically: a gather thread takes the next
  // index from the global counter and publishes it in the CTA's ring; every
  // role reads the same sequence from the ring (-1 ends it). Returns false
  // on a timeout.
  auto next_unit = [&](uint32_t n, int& ui) -> bool {
    const int slot = n % kRing;
    if (!mbar_wait(&sh->ring_full[slot], (n / kRing) & 1, abort_flag)) return false;
    ui = *reinterpret_cast<volatile int*>(&sh->ring[slot]);
    mbar_arrive(&sh->ring_empty[slot]);
    return true;
  };

  // register split: the two softmax warpgroups take 192 per thread, the
  // producer/MMA/gather warpgroup 120 (256*192 + 128*120 = 64512, exactly
  // the 384*168 registers the block is launched with)
  if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;\n" ::: "memory");
  }

  if (warp < 8) {
    // -------------------------------------------- softmax + epilogue of tile X
    const int X = warp >> 2;
    const int row = threadIdx.x & 127;  // TMEM lane
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + kTmemS + lane_off;
    const uint32_t tP = tmem + kTmemP + X * 64 + lane_off;
    const uint32_t tO = tmem + kTmemO + X * 128 + lane_off;
    uint32_t sx = 0;  // steps done by tile X
    for (uint32_t un = 0;; ++un) {
      int ui;
      if (!next_unit(un, ui)) goto done;
      if (ui < 0) break;
      const UnitInfo u = decode_unit(p, ui);
      if (X == 1 && !u.has_b) continue;
      // own unit: from step dstep on, tile X's keys reach its first token
      const int dstep = u.own ? (X ? u.diag[1] : u.diag[0]) : u.nsteps;
      float m_run = -INFINITY, l_run = 0.f;
      for (int s = 0; s < u.nsteps; ++s, ++sx) {
        if (!mbar_wait(&sh->s_full[X], sx & 1, abort_flag)) goto done;
        __syncwarp();
        tc_fence_after();
        uint32_t r[128];
        {
          uint32_t (&r0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[0]);
          uint32_t (&r1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[32]);
          uint32_t (&r2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[64]);
          uint32_t (&r3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&r[96]);
          tmem_ld32(tS, r0);
          tmem_ld32(tS + 32, r1);
          tmem_ld32(tS + 64, r2);
          tmem_ld32(tS + 96, r3);
          tmem_ld_wait();
        }
        // the S buffer is free for the next tile's product
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->s_free);
        // causal mask in an own unit from the step whose keys start at the
        // tile's first token: key > query (a later step is fully masked)
        const bool diag = s >= dstep;
        if (diag) {
          const int lim = row - (s - dstep) * kTile;  // keys e > lim are masked
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e > lim) r[e] = __float_as_uint(-INFINITY);
        }
        // row max: eight independent chains of 3-input max over columns
        // c, c+8, ..., c+120
        float mx8[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float m = fmax3(__uint_as_float(r[c]), __uint_as_float(r[c + 8]), __uint_as_float(r[c + 16]));
#pragma unroll
          for (int e = 24; e < 120; e += 16) m = fmax3(m, __uint_as_float(r[e + c]), __uint_as_float(r[e + 8 + c]));
          mx8[c] = fmaxf(m, __uint_as_float(r[120 + c]));
        }
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]));
        const float m_new = fmaxf(m_run, mx * p.scale_log2);
        float m_ref = m_run, factor = 1.f;
        bool rescale = false;
        if (s == 0) {
          m_ref = m_new;
        } else if (m_new > m_run + 8.f) {
          m_ref = m_new;
          factor = ex2_approx(m_run - m_new);
          rescale = true;
        }
        // p = 2^(s*c - m), held in registers as bf16 pairs
        uint32_t pk[64];
        {
          const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
          const uint64_t nm2 = f2_pack(-m_ref, -m_ref);
          uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
          exp_row(r, c2, nm2, sum2, pk);
          const uint64_t s01 = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
          l_run = l_run * factor + (f2_lo(s01) + f2_hi(s01));
          m_run = m_ref;
        }
        // PV_X(s-1) has completed: P_X's columns are free again and O_X is
        // settled for a rescale. (This wait also keeps every thread's arrival
        // on p_full for step s behind the completion of step s-1.)
        if (s > 0) {
          if (!mbar_wait(&sh->pv_done[X], (sx - 1) & 1, abort_flag)) goto done;
          __syncwarp();
          tc_fence_after();
        }
        // O rescale. The decision is per row, but tcgen05.ld/st are
        // warp-collective: the whole warp takes the branch when any of its
        // rows moves its reference (the others multiply by factor 1).
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(tO + c * 32, o);
          }
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_st16(tP + ch * 16, pk + ch * 16);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh->p_full[X]);
      }
      {
        // epilogue: O / l and lse for this tile's rows (the next unit's
        // first P.V product waits for this tile's p_full, which comes after)
        if (!mbar_wait(&sh->pv_done[X], (sx - 1) & 1, abort_flag)) goto done;
        __syncwarp();
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const float lse = (m_run + log2f(l_run)) * 0.69314718055994530942f;
        const bool write = row < (X ? u.rows[1] : u.rows[0]) && (!u.own || (X ? u.tq[1] : u.tq[0]) + row >= p.q0);
        __half* dst_o;
        float* dst_lse;
        if (u.own) {
          const int64_t rr = ((X ? u.tq[1] : u.tq[0]) + row - p.w0) * p.Hq + (X ? u.h[1] : u.h[0]);
          dst_o = p.own_o + rr * kHeadDim;
          dst_lse = p.own_lse + rr;
        } else {
          const int64_t rr = (int64_t)(X ? u.list0[1] : u.list0[0]) + row;
          dst_o = p.part_o + rr * kHeadDim;
          dst_lse = p.part_lse + rr;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
          if (write) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 hv;
              hv.x = pack_half2(__uint_as_float(o[e]) * inv_l, __uint_as_float(o[e + 1]) * inv_l);
              hv.y = pack_half2(__uint_as_float(o[e + 2]) * inv_l, __uint_as_float(o[e + 3]) * inv_l);
              hv.z = pack_half2(__uint_as_float(o[e + 4]) * inv_l, __uint_as_float(o[e + 5]) * inv_l);
              hv.w = pack_half2(__uint_as_float(o[e + 6]) * inv_l, __uint_as_float(o[e + 7]) * inv_l);
              *reinterpret_cast<uint4*>(dst_o + c * 32 + e) = hv;
            }
          }
        }
        if (write) *dst_lse = lse;
        tc_fence_before();
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------ K/V TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      for (uint32_t un = 0;; ++un) {
        int ui;
        if (!next_unit(un, ui)) goto drain_kv;
        if (ui < 0) break;
        const UnitInfo u = decode_unit(p, ui);
        for (int s = 0; s < u.nsteps; ++s, ++it) {
          const int st = it % kStages;
          const uint32_t ph = ((it / kStages) & 1) ^ 1;
          const int key = (int)(u.key0 + (int64_t)s * kTile);
          if (!mbar_wait(&sh->k_empty[st], ph, abort_flag)) goto drain_kv;
          mbar_arrive_expect_tx(&sh->k_full[st], kTileBytes);
          tma_load_3d(sK + st * kTileBytes, &tmap_k, &sh->k_full[st], 0, u.g, key);
          tma_load_3d(sK + st * kTileBytes + kHalfBytes, &tmap_k, &sh->k_full[st], 64, u.g, key);
          if (!mbar_wait(&sh->v_empty[st], ph, abort_flag)) goto drain_kv;
          mbar_arrive_expect_tx(&sh->v_full[st], kTileBytes);
          tma_load_3d(sV + st * kTileBytes, &tmap_v, &sh->v_full[st], 0, u.g, key);
          tma_load_3d(sV + st * kTileBytes + kHalfBytes, &tmap_v, &sh->v_full[st], 64, u.g, key);
        }
      }
    drain_kv:
      // no TMA write may still be in flight when the CTA ends
      if (*abort_flag) {
        volatile int keep_waiting = 0;
        for (uint32_t k = (it > (uint32_t)kStages ? it - kStages : 0); k <= it; ++k) {
          mbar_wait(&sh->k_full[k % kStages], (k / kStages) & 1, &keep_waiting, (1ull << 28));
          mbar_wait(&sh->v_full[k % kStages], (k / kStages) & 1, &keep_waiting, (1ull << 28));
        }
      }
    }
  } else if (warp == 9 || warp == 11) {
    // ------------------------------------------------ MMA issuers
    // warp 9, per unit: S_A(0), S_B(0), S_A(1), S_B(1), ...; each S waits
    //   until the softmax warpgroup of the previous S has read it (s_free)
    // warp 11, per unit: PV_A(0), PV_B(0), PV_A(1), ...; each waits for its
    //   tile's P (p_full)
    // Each whole warp runs its loop (descriptors stay warp-uniform); one
    // elected lane issues every MMA and commit.
    const bool s_issuer = warp == 9;
    const uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
    // Descriptors are built once; moving the start address by b bytes adds
    // b >> 4 to the descriptor (the 14-bit start field cannot carry inside
    // the 228 KB of shared memory).
    const uint64_t dQ = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(sV), kHalfBytes, 1024);
    uint32_t it = 0;          // K/V steps
    uint32_t ns = 0;          // products issued into the S buffer
    uint32_t npv[2] = {0, 0};  // P.V products per tile
    uint32_t ux[2] = {0, 0};  // units per tile
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) mma_commit(bar);
      __syncwarp();
    };
    // S_X = Q_X K^T for the 128 keys of K stage st, once the S buffer's
    // previous product has been read; closes tile X's Q buffer when this is
    // the unit's last product of that tile
    auto issue_s = [&](int x, int st, bool last_of_unit) -> bool {
      if (ns > 0 && !mbar_wait(&sh->s_free, (ns - 1) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint64_t q0 = dQ + ((x * kTileBytes) >> 4);
      const uint64_t k0 = dK + ((st * kTileBytes) >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_bf16_ss(tmem + kTmemS, q0 + off, k0 + off, idesc_s, kk > 0);
        }
        mma_commit(&sh->s_full[x]);
        if (last_of_unit) mma_commit(&sh->q_empty[x]);
      }
      __syncwarp();
      ++ns;
      return true;
    };
    // O_X (+)= P_X V for V stage st
    auto issue_pv = [&](int x, int st, bool accumulate) -> bool {
      if (!mbar_wait(&sh->p_full[x], npv[x] & 1, abort_flag)) return false;
      tc_fence_after();
      const uint64_t v0 = dV + ((st * kTileBytes) >> 4);
      const uint32_t tPx = tmem + kTmemP + x * 64;
      const uint32_t tOx = tmem + kTmemO + x * 128;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tOx, tPx + kk * 8, v0 + ((kk * 2048) >> 4), idesc_o, (accumulate || kk > 0) ? 1u : 0u);
        mma_commit(&sh->pv_done[x]);
      }
      __syncwarp();
      ++npv[x];
      return true;
    };
    for (uint32_t un = 0;; ++un) {
      int ui;
      if (!next_unit(un, ui)) goto mma_done;
      if (ui < 0) break;
      const UnitInfo u = decode_unit(p, ui);
      const int nx = u.has_b ? 2 : 1;
      const int n = u.nsteps;
      for (int s = 0; s < n; ++s) {
        const uint32_t cur = it + s;
        const int st = cur % kStages;
        if (s_issuer) {
          if (!mbar_wait(&sh->k_full[st], (cur / kStages) & 1, abort_flag)) goto mma_done;
          for (int x = 0; x < nx; ++x) {
            if (s == 0 && !mbar_wait(&sh->q_full[x], ux[x] & 1, abort_flag)) goto mma_done;
            if (!issue_s(x, st, s + 1 == n)) goto mma_done;
          }
          commit(&sh->k_empty[st]);
        } else {
          if (!mbar_wait(&sh->v_full[st], (cur / kStages) & 1, abort_flag)) goto mma_done;
          for (int x = 0; x < nx; ++x)
            if (!issue_pv(x, st, s > 0)) goto mma_done;
          commit(&sh->v_empty[st]);
        }
      }
      it += n;
      ux[0] += 1;
      ux[1] += (nx > 1) ? 1 : 0;
    }
  mma_done:
    // every issued MMA must finish before TMEM is released (each issuer
    // commits once to the drain barrier; both wait for both)
    __syncwarp();
    if (elect_one()) mma_commit(&sh->drain);
    __syncwarp();
    {
      volatile int keep_waiting = 0;
      mbar_wait(&sh->drain, 0, &keep_waiting, (1ull << 28));
    }
  } else {
    // ------------------------------------------------ Q gather (warp 10)
    const int gt = threadIdx.x - 320;  // 0..31
    uint32_t ux[2] = {0, 0};
    const int n_units = p.hdr[1];
    const int64_t group_rows = p.wlen * p.G;  // group-rows of the window
    for (uint32_t un = 0;; ++un) {
      if (gt == 0) {
        // publish the next unit index (slot reuse waits for every reader)
        const int slot = un % kRing;
        if (!mbar_wait(&sh->ring_empty[slot], ((un / kRing) & 1) ^ 1, abort_flag)) goto gather_done;
        int nxt = atomicAdd(p.hdr + 3, 1);
        sh->ring[slot] = nxt < n_units ? nxt : -1;
        mbar_arrive(&sh->ring_full[slot]);
      }
      int ui;
      if (!next_unit(un, ui)) goto gather_done;
      if (ui < 0) break;
      const UnitInfo u = decode_unit(p, ui);
      const int nx = u.has_b ? 2 : 1;
      // Thread gt copies whole rows gt, gt + 32, gt + 64, gt + 96 of each
      // tile (16 chunks of 16 B each). Their element offsets in q are found
      // first (a routed tile reads its row list), before waiting for the
      // tiles' buffers, so the list reads overlap the previous unit's last
      // step; then both tiles' copies are in flight together and complete
      // with one wait.
      int64_t off[2][4];
#pragma unroll
      for (int x = 0; x < 2; ++x) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = gt + 32 * k;
          off[x][k] = -1;
          if (x < nx && r < u.rows[x]) {
            int64_t t;
            int h;
            if (u.own) {
              t = u.tq[x] + r;
              h = u.h[x];
            } else {
              const int rr = __ldg(p.list + u.list0[x] + r);
              if (rr < 0 || rr >= group_rows) {
                // an inconsistent router list: record it, gather nothing
                record_status(MOBA_ERR_DEVICE_CHECK);
                continue;
              }
              t = p.w0 + rr / p.G;
              h = u.g * p.G + rr % p.G;
            }
            // a token before q0 has no query: its row stays zero and is not written
            if (t >= p.q0) off[x][k] = ((t - p.q0) * p.Hq + h) * kHeadDim;
          }
        }
      }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (x >= nx) break;
        if (!mbar_wait(&sh->q_empty[x], (ux[x] & 1) ^ 1, abort_flag)) goto gather_done;
        const uint32_t dst0 = smem_u32(sQ + x * kTileBytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = gt + 32 * k;
          const bool valid = off[x][k] >= 0;
          const __nv_bfloat16* src = valid ? p.q + off[x][k] : p.q;
#pragma unroll
          for (int c16 = 0; c16 < 16; ++c16) {
            const int half = c16 >> 3, c = c16 & 7;
            cp_async_16(dst0 + half * kHalfBytes + r * 128 + ((c ^ (r & 7)) << 4), src + (valid ? c16 * 8 : 0),
                        valid ? 16u : 0u);
          }
        }
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (x >= nx) break;
        mbar_arrive(&sh->q_full[x]);
        ++ux[x];
      }
    }
  gather_done:
    cp_async_wait_all();
  }
done:
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace moba
