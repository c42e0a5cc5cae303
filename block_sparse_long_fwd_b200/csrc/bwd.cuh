// The backward pass: dQ, dK, dV of the MoBA forward with the gate's choice
// held fixed (the top-k choice is piecewise constant, so the block means get
// no gradient). MoBA is meant to be trained further from a full-attention
// model ("MoBA (Mixture of Block Attention)" project summary, "Key Features";
// "Efficient Long-Context Attention with MoBA", "How MoBA Works"), which
// needs this gradient. Per q head h of kv head g, with c = 1/sqrt(128), the
// row's attended keys (its selected past blocks and the causal part of its
// own block), P = softmax(c Q K^T) there, D = rowsum(dO * O):
//   dV = sum over the group's heads of P^T dO
//   dS = P * (dO V^T - D)
//   dQ = c dS K,   dK = sum over the group's heads of c dS^T Q.
// P is rebuilt from the forward's lse: P = 2^(S c log2(e) - lse log2(e)).
//
// The work follows the forward's routing (pool, gate and router run again,
// so the selection is the forward's):
//   bwd_dq_kernel    per forward work unit and tile of 128 query rows:
//                    S = Q K^T and dP = dO V^T on the tensor cores for each
//                    128-key step of the unit's block (the next step's
//                    issued while this step's element-wise work runs), dS to
//                    TMEM as bf16, dQ += dS K accumulated in TMEM; the unit's
//                    c*dQ goes out as an fp16 partial into the slot the
//                    forward uses for its partial output.
//   bwd_dq_reduce    dQ = sum of a row's partials in a fixed order (its
//                    selected past blocks ascending, its own block last).
//   bwd_dkdv_kernel  per (kv head, block, 128-key tile): the transposed
//                    products S^T = K Q^T and dP^T = V dO^T for every
//                    64-row slice of the rows that attend the block (its
//                    router list, then its own causal rows), P^T and dS^T
//                    written back as bf16, dV += P^T dO and dK += dS^T Q
//                    accumulated in TMEM over all of them (two slice
//                    buffers, so one slice's element-wise step overlaps the
//                    other's products); one fp32 read-add-write per key row
//                    and query window.
// Both tensor-core kernels take K, V, Q and dO tiles in the 128-byte-swizzled
// layout, read K-major for S / dP and MN-major for the dQ / dK / dV products.
// Every mbarrier wait is bounded and sets the device status on a timeout.
#pragma once

#include "attn.cuh"
#include "merge.cuh"
#include "route.cuh"

namespace moba {

// dK / dV kernel: K, V, four 64-row Q and dO slices, its shared state
constexpr int kBwdSmemBytes = 6 * kTileBytes + 1024 + 4096;

struct BwdParams {
  const __nv_bfloat16* q;     // [S][Hq][128]
  const __nv_bfloat16* dout;  // [S][Hq][128]
  const float* lse2;          // [Hq][S]: the forward's lse times log2(e)
  const float* dd;            // [Hq][S]: rowsum(dO * O)
  int64_t S, w0, wlen;
  int Hq, Hkv, G, B, nbp;
  float scale_log2;  // log2(e) / sqrt(128)
  float scale;       // 1 / sqrt(128)
};

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float bwd_warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Row (t, h) of q / dO into row r of a 128-row tile in the 128-byte-swizzled
// layout (two 64-column halves); a missing row (off < 0) is zero-filled.
__device__ __forceinline__ void gather_row(uint32_t dst0, const __nv_bfloat16* base, int64_t off, int r) {
  const bool valid = off >= 0;
  const __nv_bfloat16* src = valid ? base + off : base;
#pragma unroll
  for (int c16 = 0; c16 < 16; ++c16) {
    const int half = c16 >> 3, c = c16 & 7;
    cp_async_16(dst0 + half * kHalfBytes + r * 128 + ((c ^ (r & 7)) << 4), src + (valid ? c16 * 8 : 0),
                valid ? 16u : 0u);
  }
}

// D = rowsum(dO * O) and lse * log2(e) per row. grid ceil(S*Hq/8), 256
// threads: one warp per row (t, h); fixed-order shuffle sums.
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse, int64_t S, int Hq,
                                                       float* __restrict__ lse2, float* __restrict__ dd) {
  grid_dependency_sync();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= S * Hq) return;
  const int64_t t = row / Hq;
  const int h = (int)(row % Hq);
  const uint2 a = __ldg(reinterpret_cast<const uint2*>(o + row * kHeadDim + lane * 4));
  const uint2 b = __ldg(reinterpret_cast<const uint2*>(dout + row * kHeadDim + lane * 4));
  const float2 a0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.x));
  const float2 a1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a.y));
  const float2 b0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.x));
  const float2 b1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b.y));
  float s = a0.x * b0.x;
  s = fmaf(a0.y, b0.y, s);
  s = fmaf(a1.x, b1.x, s);
  s = fmaf(a1.y, b1.y, s);
  s = bwd_warp_sum(s);
  if (lane == 0) {
    dd[(int64_t)h * S + t] = s;
    lse2[(int64_t)h * S + t] = lse[(int64_t)h * S + t] * 1.4426950408889634f;
  }
}

// n float4 zeros (the dK / dV accumulators before the first window).
__global__ void __launch_bounds__(256) bwd_zero_kernel(float4* __restrict__ p, int64_t n) {
  grid_dependency_sync();
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256)
    p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// fp32 accumulators to bf16 outputs (n groups of four values).
__global__ void __launch_bounds__(256) bwd_cast_kernel(const float4* __restrict__ a, __nv_bfloat16* __restrict__ out,
                                                       int64_t n) {
  grid_dependency_sync();
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const float4 v = a[i];
    *reinterpret_cast<uint2*>(out + i * 4) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

constexpr int kDqThreads = 256;  // two warps per TMEM lane quadrant
constexpr int kDqKStages = 3;    // K is read by S(s) and dQ(s): three stages in flight
constexpr int kDqSmemBytes = (2 + kDqKStages + 2) * kTileBytes + 1024 + 512;

struct BwdShared {
  uint64_t k_full[kDqKStages], v_full[2];
  uint64_t s_done, x_done, drain;
  uint32_t tmem_base;
  int abort_flag;
};

// grid = number of SMs, 256 threads: two warps per TMEM lane quadrant (lane =
// query row), each taking 64 of a step's 128 key columns and 64 of dQ's
// columns; threads 0..127 gather Q rows, 128..255 dO rows. Items (unit,
// tile) are taken with a fixed stride. Per 128-key step s:
//   S(s) = Q K^T, dP(s) = dO V^T   (SS MMAs into TMEM 0..127, 128..255)
//   every warp loads its S / dP columns, then S(s+1), dP(s+1) are issued
//   into the same columns while the warps compute dS(s) = P (dP - D)
//   dS(s) goes to TMEM 384..447 (bf16) once dQ(s-1) has read the previous
//   one, and dQ += dS(s) K (TS MMA, K as an MN-major B operand) into
//   256..383.
// K sits in a 3-stage ring (read by S(s) and by dQ(s)), V in 2 stages; the
// loads for step s+2 go out once dQ(s-1) is done.
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                  AttnParams ap, BwdParams p) {
  grid_dependency_sync();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + kTileBytes;
  uint8_t* sK = sdO + kTileBytes;             // kDqKStages stages
  uint8_t* sV = sK + kDqKStages * kTileBytes;  // 2 stages
  BwdShared* sh = reinterpret_cast<BwdShared*>(sV + 2 * kTileBytes);
  const int warp = threadIdx.x >> 5;
  const int row = threadIdx.x & (kTile - 1);  // query row (TMEM lane) and gathered row
  const int hf = warp >> 2;                   // this warp's half of the columns
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDqKStages; ++i) mbar_init(&sh->k_full[i], 1);
    mbar_init(&sh->v_full[0], 1);
    mbar_init(&sh->v_full[1], 1);
    mbar_init(&sh->s_done, 1);
    mbar_init(&sh->x_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  if (warp == 0) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  volatile int* ab = &sh->abort_flag;
  const uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
  const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
  const uint64_t dQd = sdesc_sw128(smem_u32(sQ), 16, 1024);
  const uint64_t ddOd = sdesc_sw128(smem_u32(sdO), 16, 1024);
  const uint64_t dK = sdesc_sw128(smem_u32(sK), 16, 1024);
  const uint64_t dV = sdesc_sw128(smem_u32(sV), 16, 1024);
  const uint64_t dKmn = sdesc_sw128(smem_u32(sK), kHalfBytes, 1024);
  const float c2 = p.scale_log2;
  const int n_units = ap.hdr[1];
  uint32_t L0 = 0;      // global index of this item's first step
  uint32_t loaded = 0;  // K/V step loads issued (thread 0)
  uint32_t waited = 0;  // K/V step loads waited for (thread 0)
  auto load_kv = [&](uint32_t L, const UnitInfo& u, int s) {  // thread 0
    const int ks = L % kDqKStages, vs = L & 1;
    const int key = (int)(u.key0 + (int64_t)s * kTile);
    mbar_arrive_expect_tx(&sh->k_full[ks], kTileBytes);
    tma_load_3d(sK + ks * kTileBytes, &tmap_k, &sh->k_full[ks], 0, u.g, key);
    tma_load_3d(sK + ks * kTileBytes + kHalfBytes, &tmap_k, &sh->k_full[ks], 64, u.g, key);
    mbar_arrive_expect_tx(&sh->v_full[vs], kTileBytes);
    tma_load_3d(sV + vs * kTileBytes, &tmap_v, &sh->v_full[vs], 0, u.g, key);
    tma_load_3d(sV + vs * kTileBytes + kHalfBytes, &tmap_v, &sh->v_full[vs], 64, u.g, key);
    loaded = L + 1;
  };
  // S(L) and dP(L) (thread 0's warp; K / V of step L must have landed)
  auto issue_s = [&](uint32_t L) -> bool {
    if (threadIdx.x == 0) {
      if (!mbar_wait(&sh->k_full[L % kDqKStages], (L / kDqKStages) & 1, ab)) return false;
      if (!mbar_wait(&sh->v_full[L & 1], (L >> 1) & 1, ab)) return false;
      waited = L + 1;
    }
    __syncwarp();
    tc_fence_after();
    if (elect_one()) {
      const uint64_t k0 = dK + (((L % kDqKStages) * kTileBytes) >> 4), v0 = dV + (((L & 1) * kTileBytes) >> 4);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t o = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
        mma_bf16_ss(tmem, dQd + o, k0 + o, idesc_s, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t o = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
        mma_bf16_ss(tmem + 128, ddOd + o, v0 + o, idesc_s, kk > 0 ? 1u : 0u);
      }
      mma_commit(&sh->s_done);
    }
    __syncwarp();
    return !*ab;
  };
  for (int item = blockIdx.x; item < 2 * n_units; item += gridDim.x) {
    const UnitInfo u = decode_unit(ap, item >> 1);
    const int x = item & 1;
    if (x == 1 && !u.has_b) continue;
    // this thread's query row
    int64_t t = -1;
    int h = 0;
    if (row < u.rows[x]) {
      if (u.own) {
        t = u.tq[x] + row;
        h = u.h[x];
      } else {
        const int rr = __ldg(ap.list + u.list0[x] + row);
        t = p.w0 + rr / p.G;
        h = u.g * p.G + rr % p.G;
      }
    }
    const int64_t off = t >= 0 ? (t * p.Hq + h) * kHeadDim : -1;
    if (threadIdx.x < kTile)
      gather_row(smem_u32(sQ), p.q, off, row);
    else
      gather_row(smem_u32(sdO), p.dout, off, row);
    float lse2_r = INFINITY, dd_r = 0.f;  // a missing row gets P = 0
    if (t >= 0) {
      lse2_r = __ldg(p.lse2 + (int64_t)h * p.S + t);
      dd_r = __ldg(p.dd + (int64_t)h * p.S + t);
    }
    if (threadIdx.x == 0) {
      // the previous item's products are all done: every stage is free
      load_kv(L0, u, 0);
      if (u.nsteps > 1) load_kv(L0 + 1, u, 1);
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const int dstep = u.own ? u.diag[x] : u.nsteps;
    if (warp == 0 && !issue_s(L0)) goto done;
    for (int s = 0; s < u.nsteps; ++s) {
      const uint32_t L = L0 + s;
      if (!mbar_wait(&sh->s_done, L & 1, ab)) goto done;
      __syncwarp();
      tc_fence_after();
      uint32_t sr[64], pr[64];
      tmem_ld32(tmem + lane_off + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tmem + lane_off + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tmem + lane_off + 128 + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld32(tmem + lane_off + 128 + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncthreads();  // every warp holds its S(s) / dP(s) columns
      tc_fence_after();
      if (warp == 0 && s + 1 < u.nsteps && !issue_s(L + 1)) goto done;
      // dS(s), keys e > lim masked on and after the diagonal step
      uint32_t dk[32];
      {
        const int lim = s >= dstep ? row - (s - dstep) * kTile : kTile;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float dv[2];
#pragma unroll
          for (int v2 = 0; v2 < 2; ++v2) {
            float pe = ex2_approx(fmaf(__uint_as_float(sr[e + v2]), c2, -lse2_r));
            if (hf * 64 + e + v2 > lim) pe = 0.f;
            dv[v2] = pe * (__uint_as_float(pr[e + v2]) - dd_r);
          }
          dk[e >> 1] = pack_bf16x2(dv[0], dv[1]);
        }
      }
      // dQ(s-1) has read the previous dS; its K stage is then free, and V's
      // stage was freed by dP(s): load step s+2
      if (s > 0 && !mbar_wait(&sh->x_done, (L - 1) & 1, ab)) goto done;
      if (threadIdx.x == 0 && s + 2 < u.nsteps) load_kv(L + 2, u, s + 2);
      tc_fence_after();
      tmem_st16(tmem + lane_off + 384 + hf * 32, dk);
      tmem_st16(tmem + lane_off + 384 + hf * 32 + 16, dk + 16);
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (warp == 0) {
        if (elect_one()) {
          const uint64_t k0 = dKmn + (((L % kDqKStages) * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ts(tmem + 256, tmem + 384 + kk * 8, k0 + ((kk * 2048) >> 4), idesc_o,
                        (s > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sh->x_done);
        }
        __syncwarp();
      }
    }
    L0 += u.nsteps;
    // the item's last dQ product, then c * dQ as an fp16 partial
    if (!mbar_wait(&sh->x_done, (L0 - 1) & 1, ab)) goto done;
    __syncwarp();
    tc_fence_after();
    {
      __half* dst = nullptr;
      if (t >= 0)
        dst = u.own ? ap.own_o + ((t - p.w0) * p.Hq + h) * kHeadDim
                    : ap.part_o + ((int64_t)u.list0[x] + row) * kHeadDim;
#pragma unroll
      for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + 256 + c * 32, o);
        tmem_ld_wait();
        if (dst) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 hv;
            hv.x = pack_half2(__uint_as_float(o[e]) * p.scale, __uint_as_float(o[e + 1]) * p.scale);
            hv.y = pack_half2(__uint_as_float(o[e + 2]) * p.scale, __uint_as_float(o[e + 3]) * p.scale);
            hv.z = pack_half2(__uint_as_float(o[e + 4]) * p.scale, __uint_as_float(o[e + 5]) * p.scale);
            hv.w = pack_half2(__uint_as_float(o[e + 6]) * p.scale, __uint_as_float(o[e + 7]) * p.scale);
            *reinterpret_cast<uint4*>(dst + c * 32 + e) = hv;
          }
        }
      }
      // the next item's gather and products overwrite shared memory and TMEM
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
    }
  }
done:
  if (*ab) {
    // after a timeout: let issued copies and products land first (bounded)
    volatile int keep = 0;
    if (threadIdx.x == 0)
      for (uint32_t L = waited; L < loaded; ++L) {
        mbar_wait(&sh->k_full[L % kDqKStages], (L / kDqKStages) & 1, &keep, (1ull << 28));
        mbar_wait(&sh->v_full[L & 1], (L >> 1) & 1, &keep, (1ull << 28));
      }
    if (warp == 0) {
      if (elect_one()) mma_commit(&sh->drain);
      __syncwarp();
      mbar_wait(&sh->drain, 0, &keep, (1ull << 28));
    }
  }
  cp_async_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dQ of the window's rows: the sum of each row's fp16 partials in a fixed
// order (selected past blocks ascending, own block last), already scaled by
// c. grid ceil(wlen*Hq/8), 256 threads: one warp per row (t, h).
__global__ void __launch_bounds__(256) bwd_dq_reduce_kernel(const int32_t* __restrict__ sel,
                                                            const uint32_t* __restrict__ flags,
                                                            const int32_t* __restrict__ wordbase,
                                                            const __half* __restrict__ part_o,
                                                            const __half* __restrict__ own_o, WindowGeom w,
                                                            __nv_bfloat16* __restrict__ dq) {
  grid_dependency_sync();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= w.wlen * w.Hq) return;
  const int64_t tl = row / w.Hq;
  const int h = (int)(row % w.Hq);
  const int64_t t = w.w0 + tl;
  const int g = h / w.G, hl = h % w.G;
  const int bt = (int)(t / w.B);
  const int64_t rr = tl * w.G + hl;
  const int64_t word = rr >> 5;
  const uint32_t below = (1u << (rr & 31)) - 1u;
  const int32_t* srow = sel + ((int64_t)h * w.S + t) * w.k_eff;
  const int P = w.k_eff - 1;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < P; ++i) {
    const int j = __ldg(srow + i);
    if (j < 0 || j >= bt) continue;
    const int64_t f = ((int64_t)g * w.nbp + j) * w.wwords + word;
    const int64_t pos = (int64_t)__ldg(wordbase + f) + __popc(__ldg(flags + f) & below);
    if (!slot_ok(w, pos)) continue;
    const float4 o = load_half4(part_o + pos * kHeadDim + lane * 4);
    acc.x += o.x;
    acc.y += o.y;
    acc.z += o.z;
    acc.w += o.w;
  }
  const float4 o = load_half4(own_o + (tl * w.Hq + h) * kHeadDim + lane * 4);
  acc.x += o.x;
  acc.y += o.y;
  acc.z += o.z;
  acc.w += o.w;
  *reinterpret_cast<uint2*>(dq + (t * w.Hq + h) * kHeadDim + lane * 4) =
      make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
}

struct DkdvParams {
  const int32_t* list;    // the window's router lists (group-rows)
  const int32_t* cnt;     // [Hkv][nbp] routed rows per bucket (valid when routed)
  const int32_t* loff;    // [Hkv][nbp] first list slot per bucket
  float* dk_acc;          // [S][Hkv][128] fp32
  float* dv_acc;          // [S][Hkv][128] fp32
  int routed;             // the window has router lists
};

// dK / dV pipeline: query rows come in 64-row slices through a 4-stage
// shared-memory ring; TMEM holds two slice buffers (S^T and dP^T, 64
// columns each) beside the dV and dK accumulators, so the products of one
// slice run while the element-wise step of the other is under way.
constexpr int kSlice = 64;
constexpr uint32_t kSliceHalf = kSlice * 128;    // one 64-channel half of a slice: 8 KB
constexpr uint32_t kSliceBytes = 2 * kSliceHalf;  // 16 KB
constexpr int kDkdvStages = 4;
constexpr int kDkdvThreads = 352;  // warps 0-7 element-wise, 8 MMA + TMA, 9-10 gather

struct DkdvShared {
  uint64_t kv_full, drain, all_done;
  uint64_t q_full[kDkdvStages], q_empty[kDkdvStages];
  uint64_t s_full[2], p_full[2], x_done[2];
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float lse2[kDkdvStages][kSlice];
  alignas(16) float dd[kDkdvStages][kSlice];
  alignas(16) int tok[kDkdvStages][kSlice];
};

// The 32 rows rbase .. rbase+31 of a 64-row slice (two 8 KB halves, 128-byte
// swizzle), one warp: lane l holds the element offset of row rbase + l
// (-1: a missing row, zero-filled). Each copy instruction moves two whole
// rows, 16 lanes per 256-byte row, so a warp instruction touches 4 cache
// lines instead of one line in each of 32 rows.
__device__ __forceinline__ void gather_slice_rows(uint32_t dst0, const __nv_bfloat16* base, int64_t off_mine,
                                                  int rbase, int lane) {
  const int c16 = lane & 15, half = c16 >> 3, c = c16 & 7;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int rl = 2 * i + (lane >> 4);
    const int64_t off = __shfl_sync(0xffffffffu, off_mine, rl);
    const int r = rbase + rl;
    const bool valid = off >= 0;
    cp_async_16(dst0 + half * kSliceHalf + r * 128 + ((c ^ (r & 7)) << 4), valid ? base + off + c16 * 8 : base,
                valid ? 16u : 0u);
  }
}

// grid (B/128 * nblocks * Hkv), key tile fastest, so the CTAs of one block
// (which gather the same query rows) run together and share them in L2.
// One CTA owns 128 keys (TMEM lane = key) and loops over 64-row slices of
// the rows that attend them in this window: the bucket's router list, then
// the own block's rows from the tile's first key on (causal). Per slice m
// (TMEM buffer b = m & 1, ring stage m % 4):
//   warp 8      S^T = K Q^T and dP^T = V dO^T (N = 64) into buffer b; once
//               the slice's P^T and dS^T are back, dV += P^T dO and
//               dK += dS^T Q (TS MMAs, dO and Q as MN-major B operands),
//               which also free the ring stage and the buffer
//   warps 0-3 / 4-7 (even / odd slices): P^T = 2^(S^T c - lse2) (0 where
//               masked), dS^T = P^T (dP^T - D), both back as bf16 over the
//               first half of S^T and of dP^T
//   warps 9-10  gather the slice's Q and dO rows (cp.async) and per-row
//               values, two slices in flight.
// TMEM: buffer b at 128b (S^T 0..63, dP^T 64..127), dV 256..383, dK 384..511.
__global__ void __launch_bounds__(kDkdvThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                    BwdParams p, DkdvParams d) {
  grid_dependency_sync();
  const int ntb = p.B / kTile;
  const int kt = (int)(blockIdx.x % ntb);
  const int j = (int)((blockIdx.x / ntb) % (p.nbp + 1));
  const int g = (int)(blockIdx.x / ((int64_t)ntb * (p.nbp + 1)));
  const int64_t kstart = (int64_t)j * p.B + (int64_t)kt * kTile;
  if (kstart >= p.S) return;
  const int nr = (d.routed && j < p.nbp) ? __ldg(d.cnt + g * p.nbp + j) : 0;
  const int lbase = (d.routed && j < p.nbp) ? __ldg(d.loff + g * p.nbp + j) : 0;
  const int64_t t_lo = max(kstart, p.w0);
  const int64_t t_hi = min(min((int64_t)(j + 1) * p.B, p.S), p.w0 + p.wlen);
  const int64_t n_own = t_hi > t_lo ? (t_hi - t_lo) * p.G : 0;
  const int64_t own_rr0 = (t_lo - p.w0) * p.G;
  const int n_rs = (nr + kSlice - 1) / kSlice;
  const int ns = n_rs + (int)((n_own + kSlice - 1) / kSlice);
  if (ns == 0) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = sK + kTileBytes;
  uint8_t* sQ = sV + kTileBytes;                      // kDkdvStages slices
  uint8_t* sdO = sQ + kDkdvStages * kSliceBytes;      // kDkdvStages slices
  DkdvShared* sh = reinterpret_cast<DkdvShared*>(sdO + kDkdvStages * kSliceBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&sh->kv_full, 1);
    mbar_init(&sh->drain, 1);
    mbar_init(&sh->all_done, 1);
    for (int i = 0; i < kDkdvStages; ++i) {
      mbar_init(&sh->q_full[i], 64);
      mbar_init(&sh->q_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->s_full[b], 1);
      mbar_init(&sh->p_full[b], 128);
      mbar_init(&sh->x_done[b], 1);
    }
    sh->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* ab = &sh->abort_flag;

  if (warp < 8) {
    // ------------------------------------------------ element-wise, then the epilogue
    const int X = warp >> 2;  // slices m with m % 2 == X, TMEM buffer X
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tb = tmem + lane_off + 128 * X;
    const int key = (int)kstart + (warp & 3) * 32 + lane;
    const float c2 = p.scale_log2;
    for (int m = X; m < ns; m += 2) {
      const int st = m % kDkdvStages;
      if (!mbar_wait(&sh->s_full[X], (m >> 1) & 1, ab)) goto ew_done;
      if (!mbar_wait(&sh->q_full[st], (m / kDkdvStages) & 1, ab)) goto ew_done;  // per-row values
      __syncwarp();
      tc_fence_after();
      uint32_t sr[64], pr[64];
      tmem_ld32(tb, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tb + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tb + 64, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
      tmem_ld32(tb + 96, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        // columns 32*ch.. (slice rows); their bf16 pairs go to columns 16*ch..,
        // which this thread has already read
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const int col = ch * 32 + e4;
          const float4 a = *reinterpret_cast<const float4*>(&sh->lse2[st][col]);
          const float4 bq = *reinterpret_cast<const float4*>(&sh->dd[st][col]);
          const int4 c = *reinterpret_cast<const int4*>(&sh->tok[st][col]);
          const float l2[4] = {a.x, a.y, a.z, a.w}, dd4[4] = {bq.x, bq.y, bq.z, bq.w};
          const int tk[4] = {c.x, c.y, c.z, c.w};
          float pv[4], dv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float pe = ex2_approx(fmaf(__uint_as_float(sr[col + u]), c2, -l2[u]));
            if (key > tk[u]) pe = 0.f;
            pv[u] = pe;
            dv[u] = pe * (__uint_as_float(pr[col + u]) - dd4[u]);
          }
          pk[e4 >> 1] = pack_bf16x2(pv[0], pv[1]);
          pk[(e4 >> 1) + 1] = pack_bf16x2(pv[2], pv[3]);
          dk[e4 >> 1] = pack_bf16x2(dv[0], dv[1]);
          dk[(e4 >> 1) + 1] = pack_bf16x2(dv[2], dv[3]);
        }
        tmem_st16(tb + ch * 16, pk);
        tmem_st16(tb + 64 + ch * 16, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh->p_full[X]);
    }
    {
      // all_done is committed once, after the last slice's dV / dK (a
      // parity wait on x_done could match an older phase for the warpgroup
      // that did not take the last slice); warps 0-3 add dV, warps 4-7
      // c * dK to the window's accumulators
      if (!mbar_wait(&sh->all_done, 0, ab)) goto ew_done;
      __syncwarp();
      tc_fence_after();
      const bool valid = key < p.S;
      float* dst = (X ? d.dk_acc : d.dv_acc) + ((int64_t)key * p.Hkv + g) * kHeadDim;
      const float mul = X ? p.scale : 1.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + 256 + X * 128 + c * 32, a);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 x = *reinterpret_cast<float4*>(dst + c * 32 + e);
            x.x = fmaf(__uint_as_float(a[e]), mul, x.x);
            x.y = fmaf(__uint_as_float(a[e + 1]), mul, x.y);
            x.z = fmaf(__uint_as_float(a[e + 2]), mul, x.z);
            x.w = fmaf(__uint_as_float(a[e + 3]), mul, x.w);
            *reinterpret_cast<float4*>(dst + c * 32 + e) = x;
          }
        }
      }
    }
  ew_done:;
  } else if (warp == 8) {
    // ------------------------------------------------ K/V load and MMA issue
    const uint32_t idesc_s = idesc_bf16_f32(128, kSlice, false);
    const uint32_t idesc_o = idesc_bf16_f32(128, 128, true);
    const uint64_t dKd = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t dVd = sdesc_sw128(smem_u32(sV), 16, 1024);
    const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024);
    const uint64_t ddOk = sdesc_sw128(smem_u32(sdO), 16, 1024);
    const uint64_t dQm = sdesc_sw128(smem_u32(sQ), kSliceHalf, 1024);
    const uint64_t ddOm = sdesc_sw128(smem_u32(sdO), kSliceHalf, 1024);
    if (lane == 0) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_v);
      mbar_arrive_expect_tx(&sh->kv_full, 2 * kTileBytes);
      tma_load_3d(sK, &tmap_k, &sh->kv_full, 0, g, (int)kstart);
      tma_load_3d(sK + kHalfBytes, &tmap_k, &sh->kv_full, 64, g, (int)kstart);
      tma_load_3d(sV, &tmap_v, &sh->kv_full, 0, g, (int)kstart);
      tma_load_3d(sV + kHalfBytes, &tmap_v, &sh->kv_full, 64, g, (int)kstart);
    }
    __syncwarp();
    // S^T and dP^T of slice m into buffer m & 1
    auto issue_s = [&](int m) -> bool {
      const int st = m % kDkdvStages, b = m & 1;
      if (!mbar_wait(&sh->q_full[st], (m / kDkdvStages) & 1, ab)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t so = (st * kSliceBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          const uint32_t bo = ((kk >> 2) * kSliceHalf + (kk & 3) * 32) >> 4;
          mma_bf16_ss(tmem + 128 * b, dKd + ao, dQk + so + bo, idesc_s, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = ((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          const uint32_t bo = ((kk >> 2) * kSliceHalf + (kk & 3) * 32) >> 4;
          mma_bf16_ss(tmem + 128 * b + 64, dVd + ao, ddOk + so + bo, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sh->s_full[b]);
      }
      __syncwarp();
      return true;
    };
    if (!mbar_wait(&sh->kv_full, 0, ab)) goto mma_done;
    tc_fence_after();
    if (!issue_s(0)) goto mma_done;
    if (ns > 1 && !issue_s(1)) goto mma_done;
    for (int m = 0; m < ns; ++m) {
      const int st = m % kDkdvStages, b = m & 1;
      if (!mbar_wait(&sh->p_full[b], (m >> 1) & 1, ab)) goto mma_done;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t so = (st * kSliceBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < kSlice / 16; ++kk)
          mma_bf16_ts(tmem + 256, tmem + 128 * b + kk * 8, ddOm + so + ((kk * 2048) >> 4), idesc_o,
                      (m > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kSlice / 16; ++kk)
          mma_bf16_ts(tmem + 384, tmem + 128 * b + 64 + kk * 8, dQm + so + ((kk * 2048) >> 4), idesc_o,
                      (m > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&sh->q_empty[st]);
        mma_commit(&sh->x_done[b]);
        if (m == ns - 1) mma_commit(&sh->all_done);
      }
      __syncwarp();
      if (m + 2 < ns) {
        // buffer b is rewritten only after this slice's products have read it
        if (!mbar_wait(&sh->x_done[b], (m >> 1) & 1, ab)) goto mma_done;
        tc_fence_after();
        if (!issue_s(m + 2)) goto mma_done;
      }
    }
  mma_done:
    __syncwarp();
    if (*ab) {
      // after a timeout: let the K/V load and every issued product land
      volatile int keep = 0;
      if (lane == 0) mbar_wait(&sh->kv_full, 0, &keep, (1ull << 28));
      if (elect_one()) mma_commit(&sh->drain);
      __syncwarp();
      mbar_wait(&sh->drain, 0, &keep, (1ull << 28));
    }
  } else {
    // ------------------------------------------------ row gather (64 threads)
    // slice m+1's row and per-row values are loaded while slice m's copies
    // go out, and slice m+2's list entry one step earlier still, so a step
    // does not wait on a global load before it can hand its slice over
    const int r = threadIdx.x - 9 * 32;  // row of the slice
    auto list_entry = [&](int m) -> int {
      return (m < n_rs && m * kSlice + r < nr) ? __ldg(d.list + lbase + m * kSlice + r) : -1;
    };
    // (t, h) of this thread's row in slice m (t = -1: no row)
    auto row_of = [&](int m, int lst, int64_t& t, int& h) {
      t = -1;
      h = 0;
      if (m >= ns) return;
      if (m < n_rs) {
        if (lst >= 0) {
          t = p.w0 + lst / p.G;
          h = g * p.G + lst % p.G;
        }
      } else {
        const int64_t k = (int64_t)(m - n_rs) * kSlice + r;
        if (k < n_own) {
          const int64_t rr = own_rr0 + k;
          t = p.w0 + rr / p.G;
          h = g * p.G + (int)(rr % p.G);
        }
      }
    };
    int64_t t_cur;
    int h_cur;
    row_of(0, list_entry(0), t_cur, h_cur);
    float l2_cur = t_cur >= 0 ? __ldg(p.lse2 + (int64_t)h_cur * p.S + t_cur) : INFINITY;
    float dd_cur = t_cur >= 0 ? __ldg(p.dd + (int64_t)h_cur * p.S + t_cur) : 0.f;
    int lst_next = list_entry(1);
    for (int m = 0; m < ns; ++m) {
      const int st = m % kDkdvStages;
      int64_t t_nx;
      int h_nx;
      row_of(m + 1, lst_next, t_nx, h_nx);
      const float l2_nx = t_nx >= 0 ? __ldg(p.lse2 + (int64_t)h_nx * p.S + t_nx) : INFINITY;
      const float dd_nx = t_nx >= 0 ? __ldg(p.dd + (int64_t)h_nx * p.S + t_nx) : 0.f;
      lst_next = list_entry(m + 2);
      // the copies below are warp-collective: a timeout sends the whole warp out
      const bool ok = mbar_wait(&sh->q_empty[st], ((m / kDkdvStages) & 1) ^ 1, ab);
      if (__any_sync(0xffffffffu, !ok)) goto gather_done;
      const int64_t off = t_cur >= 0 ? (t_cur * p.Hq + h_cur) * kHeadDim : -1;
      gather_slice_rows(smem_u32(sQ + st * kSliceBytes), p.q, off, r & ~31, r & 31);
      gather_slice_rows(smem_u32(sdO + st * kSliceBytes), p.dout, off, r & ~31, r & 31);
      cp_async_commit();
      sh->lse2[st][r] = l2_cur;
      sh->dd[st][r] = dd_cur;
      // routed rows lie past the block: no key of it is masked for them
      sh->tok[st][r] = (t_cur < 0 || m < n_rs) ? 0x7fffffff : (int)t_cur;
      if (m > 0) {
        // the previous slice's copies have landed
        cp_async_wait_group<1>();
        fence_proxy_async_smem();
        mbar_arrive(&sh->q_full[(m - 1) % kDkdvStages]);
      }
      t_cur = t_nx;
      h_cur = h_nx;
      l2_cur = l2_nx;
      dd_cur = dd_nx;
    }
    cp_async_wait_group<0>();
    fence_proxy_async_smem();
    mbar_arrive(&sh->q_full[(ns - 1) % kDkdvStages]);
  gather_done:
    cp_async_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace moba
