// Host side of the C ABI declared in include/moba.h: argument checks,
// scratch layout, query windows and the launch sequence
//   pool -> gate -> for each window: route (flags, count, scan, fill)
//                                    -> attention -> merge.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <string>
#include <vector>

#include "attn.cuh"
#include "bwd.cuh"
#include "common.cuh"
#include "gate_tc.cuh"
#include "merge.cuh"
#include "pool.cuh"
#include "route.cuh"

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define MOBA_CUDA(call)                                                                                  \
  do {                                                                                                   \
    cudaError_t e_ = (call);                                                                             \
    if (e_ != cudaSuccess) return fail(MOBA_ERR_CUDA, "%s failed: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

struct DeviceInfo {
  bool ready = false;
  bool sm100 = false;
  int sms = 0;
  int* status_host = nullptr;  // host-mapped copy of the device status word
};

std::mutex g_dev_mu;
DeviceInfo g_dev[64];

// The gate kernel for lists of KP entries takes GateCfg<KP>::kSmemBytes of
// dynamic shared memory.
template <int KP>
cudaError_t set_gate_smem() {
  return cudaFuncSetAttribute(moba::gate_tc_kernel<KP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              moba::GateCfg<KP>::kSmemBytes);
}
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

int device_info(DeviceInfo* out) {
  int dev = 0;
  MOBA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOBA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    int major = 0, minor = 0;
    MOBA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    MOBA_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
    MOBA_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    d.sm100 = (major == 10 && minor == 0);
    if (d.sm100) {
      MOBA_CUDA(cudaFuncSetAttribute(moba::attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     moba::kAttnSmemBytes));
      MOBA_CUDA(cudaFuncSetAttribute(moba::bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     moba::kDqSmemBytes));
      MOBA_CUDA(cudaFuncSetAttribute(moba::bwd_dkdv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     moba::kBwdSmemBytes));
      MOBA_CUDA(set_gate_smem<2>());
      MOBA_CUDA(set_gate_smem<4>());
      MOBA_CUDA(set_gate_smem<8>());
      MOBA_CUDA(set_gate_smem<11>());
      MOBA_CUDA(set_gate_smem<12>());
      MOBA_CUDA(set_gate_smem<16>());
      MOBA_CUDA(set_gate_smem<24>());
      MOBA_CUDA(set_gate_smem<32>());
      MOBA_CUDA(set_gate_smem<48>());
      MOBA_CUDA(set_gate_smem<64>());
      // host-mapped copy of the status word (kernels store an error code
      // there too, so a later call sees it without a device read)
      int* h = nullptr;
      MOBA_CUDA(cudaHostAlloc(reinterpret_cast<void**>(&h), sizeof(int), cudaHostAllocMapped | cudaHostAllocPortable));
      *h = 0;
      int* hd = nullptr;
      MOBA_CUDA(cudaHostGetDevicePointer(reinterpret_cast<void**>(&hd), h, 0));
      MOBA_CUDA(cudaMemcpyToSymbol(moba::g_status_mirror, &hd, sizeof(hd)));
      d.status_host = h;
    }
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      MOBA_CUDA(cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q));
      if (q != cudaDriverEntryPointSuccess || !fn)
        return fail(MOBA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    d.ready = true;
  }
  *out = d;
  if (!d.sm100) return fail(MOBA_ERR_UNSUPPORTED, "device %d is not sm_100 (B200); this library is sm_100a only", dev);
  return MOBA_OK;
}

// [S][H][128] bf16 viewed as 3-D (channel, head, token); box 64 x 1 x 128,
// 128-byte swizzle (one 64-channel half of a 128-token tile per load).
int make_kv_map(CUtensorMap* map, const void* base, int64_t S, int H) {
  cuuint64_t dims[3] = {(cuuint64_t)moba::kHeadDim, (cuuint64_t)H, (cuuint64_t)S};
  cuuint64_t strides[2] = {(cuuint64_t)moba::kHeadDim * 2, (cuuint64_t)H * moba::kHeadDim * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)moba::kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOBA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MOBA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// An error code a kernel of an earlier call left in the host-mapped status
// word: this call reports it (once) instead of launching, and clears it and
// the device word, so the call after starts clean.
int take_pending_status(const DeviceInfo& dev, cudaStream_t st) {
  if (!dev.status_host) return MOBA_OK;
  volatile int* h = dev.status_host;
  const int s = *h;
  if (!s) return MOBA_OK;
  *h = 0;
  static const int zero = 0;
  cudaMemcpyToSymbolAsync(moba::g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
  return fail(s, "a kernel of an earlier call on this device reported status %d (a bounded wait ran out or a "
              "check failed); its results are not valid", s);
}

// MOBA_SYNC=1: every call synchronises its stream and returns the kernels'
// status itself.
bool sync_mode() {
  const char* e = getenv("MOBA_SYNC");
  return e && e[0] == '1';
}

// A call's result: under MOBA_SYNC=1 a successful launch waits for its stream
// and returns the kernels' status.
int finish_call(int rc, cudaStream_t st) {
  if (rc == MOBA_OK && sync_mode()) return moba_device_status(st);
  return rc;
}

int check_shape(int64_t S, int Hq, int Hkv, int d, int B, int topk) {
  if (S < 1) return fail(MOBA_ERR_INVALID_ARG, "seqlen must be >= 1 (got %lld)", (long long)S);
  if (Hkv < 1 || Hq < 1) return fail(MOBA_ERR_INVALID_ARG, "heads must be >= 1 (q %d, kv %d)", Hq, Hkv);
  if (Hq % Hkv) return fail(MOBA_ERR_INVALID_ARG, "heads_q (%d) must be a multiple of heads_kv (%d)", Hq, Hkv);
  if (d != MOBA_HEAD_DIM) return fail(MOBA_ERR_INVALID_ARG, "head_dim must be %d (got %d)", MOBA_HEAD_DIM, d);
  if (B < 128 || B % 128) return fail(MOBA_ERR_INVALID_ARG, "block_size must be a positive multiple of 128 (got %d)", B);
  if (B > 128 * 1024) return fail(MOBA_ERR_UNSUPPORTED, "block_size above %d is not supported", 128 * 1024);
  if (topk < 1) return fail(MOBA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", topk);
  if (S > (int64_t)INT32_MAX - 2 * B) return fail(MOBA_ERR_UNSUPPORTED, "seqlen too large");
  const int64_t nb = (S + B - 1) / B;
  const int64_t k_eff = std::min<int64_t>(topk, nb);
  if (k_eff < nb && k_eff - 1 > MOBA_MAX_TOPK)
    return fail(MOBA_ERR_UNSUPPORTED, "topk %d above %d + 1 with fewer than all blocks is not supported", topk,
                MOBA_MAX_TOPK);
  if ((int64_t)Hq * S * k_eff > ((int64_t)1 << 40)) return fail(MOBA_ERR_UNSUPPORTED, "selection table too large");
  return MOBA_OK;
}

struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  }
};

struct Plan {
  int64_t S;
  int64_t q0 = 0;     // first token with a query (0: a whole prefill)
  const float* means = nullptr;  // caller's block means [Hkv][nbp][128] (then no pooling)
  int64_t wbase = 0;  // first window start: q0 rounded down to 256 tokens
  int64_t lse_ld = 0;  // lse row stride: S - q0, or a packed batch's tokens
  int Hq, Hkv, G, B, topk, k_eff, P, nb, nbp;
  int splits = 1;  // pool row splits per block
  int64_t W;       // window tokens (multiple of 128)
  int64_t wwords;  // flag words per bucket for a full window
  int64_t list_cap, tile_cap;
  size_t o_kmean, o_khi, o_klo, o_sel, o_flags, o_wordbase, o_cnt, o_loff, o_toff, o_list, o_tiles, o_hdr, o_part_o,
      o_part_lse, o_own_o, o_own_lse, total;
};

// Scratch budget for one query window: min(8 GiB, a third of the memory
// free when the device was first used). Measured once per device, since
// cudaMemGetInfo costs tens of microseconds per call.
size_t window_budget() {
  static std::mutex mu;
  static size_t budget[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (size_t)1 << 30;
  std::lock_guard<std::mutex> lk(mu);
  if (!budget[dev]) {
    size_t free_b = 0, total_b = 0;
    if (cudaMemGetInfo(&free_b, &total_b) != cudaSuccess) free_b = (size_t)16 << 30;
    budget[dev] = std::max<size_t>((size_t)64 << 20, std::min<size_t>((size_t)8 << 30, free_b / 3));
  }
  return budget[dev];
}

size_t window_bytes(const Plan& p, int64_t W) {
  const int64_t nbk = (int64_t)p.Hkv * p.nbp;
  const int64_t wwords = (W * p.G + 31) / 32;
  const int64_t list = W * p.Hq * p.P;
  const int64_t tiles = list / moba::kUnitRowsRouted + nbk + (W / moba::kTile + 1) * p.Hkv * ((p.G + 1) / 2);
  return (size_t)(nbk * wwords * 8 + list * (4 + 4 + 2 * moba::kHeadDim) + tiles * 16 +
                  W * p.Hq * (4 + 2 * moba::kHeadDim));
}

// Own-block work units pair two consecutive 128-token tiles of one head when
// a group has a single q head (else they pair two heads of a group); pairs
// stay inside a block, so B / 128 must be even, and inside a window, so
// windows then start at multiples of 256 tokens.
bool pair_tokens(const Plan& p) { return p.G == 1 && (p.B / moba::kTile) % 2 == 0; }

// Scratch layout for a query window of W tokens.
void layout_for_window(Plan& p, int64_t W) {
  if (pair_tokens(p) && W < (p.S - p.wbase + 127) / 128 * 128) W = std::max<int64_t>(256, W / 256 * 256);
  p.W = W;
  p.wwords = (W * p.G + 31) / 32;
  const int64_t nbk = (int64_t)p.Hkv * p.nbp;
  p.list_cap = W * p.Hq * p.P;
  p.tile_cap = p.list_cap / moba::kUnitRowsRouted + nbk + (W / moba::kTile + 1) * p.Hkv * ((p.G + 1) / 2);
  Carve c;
  p.splits = moba::pool_splits(std::max(p.nbp, 1), p.Hkv, p.B, 296);
  p.o_kmean = c.take((size_t)nbk * p.splits * moba::kHeadDim * 4);
  const size_t nbk_pad = (size_t)p.Hkv * moba::gate_rows_padded(std::max(p.nbp, 1));
  p.o_khi = c.take(nbk_pad * moba::kHeadDim * 2);
  p.o_klo = c.take(nbk_pad * moba::kHeadDim * 2);
  p.o_sel = c.take((size_t)p.Hq * (p.S - p.q0) * p.k_eff * 4);
  p.o_flags = c.take((size_t)nbk * p.wwords * 4);
  p.o_wordbase = c.take((size_t)nbk * p.wwords * 4);
  p.o_cnt = c.take((size_t)(nbk + 1) * 4);
  p.o_loff = c.take((size_t)(nbk + 1) * 4);
  p.o_toff = c.take((size_t)(nbk + 1) * 4);
  p.o_list = c.take((size_t)std::max<int64_t>(p.list_cap, 1) * 4);
  p.o_tiles = c.take((size_t)p.tile_cap * 16);
  p.o_hdr = c.take(16);
  p.o_part_o = c.take((size_t)std::max<int64_t>(p.list_cap, 1) * moba::kHeadDim * 2);
  p.o_part_lse = c.take((size_t)std::max<int64_t>(p.list_cap, 1) * 4);
  p.o_own_o = c.take((size_t)W * p.Hq * moba::kHeadDim * 2);
  p.o_own_lse = c.take((size_t)W * p.Hq * 4);
  p.total = c.off;
}

// Full causal attention (topk >= the number of blocks) does not depend on the
// block size: every row attends all keys up to itself. It then runs with the
// largest block the kernels take (a single block when the sequence fits in
// one), so the work is own-block units (a causal FlashAttention-style pass):
// no gate scores, no routing, one partial per row.
void dense_blocks(Plan& p) {
  if (p.nb <= 1 || p.k_eff < p.nb) return;
  const int64_t S256 = (p.S + 255) / 256 * 256;
  p.B = (int)std::min<int64_t>(S256, 128 * 1024);
  p.nb = (int)((p.S + p.B - 1) / p.B);
  p.nbp = p.nb - 1;
  p.k_eff = p.nb;
  p.P = p.k_eff - 1;
}

// The problem's shape; the scratch layout comes after.
void plan_shape(Plan& p, int64_t S, int64_t q0, int Hq, int Hkv, int B, int topk) {
  p.S = S;
  p.q0 = q0;
  p.wbase = q0 / 256 * 256;
  p.lse_ld = S - q0;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.B = B;
  p.topk = topk;
  p.nb = (int)((S + B - 1) / B);
  p.nbp = p.nb - 1;
  p.k_eff = std::min(topk, p.nb);
  p.P = p.k_eff - 1;
  dense_blocks(p);
}

// `share` > 1: the problem runs beside share - 1 others, each with its own
// scratch, so its windows take a 1/share part of the budget.
int make_plan(Plan* pl, int64_t S, int64_t q0, int Hq, int Hkv, int B, int topk, int share = 1) {
  Plan& p = *pl;
  plan_shape(p, S, q0, Hq, Hkv, B, topk);
  const int64_t S128 = (S - p.wbase + 127) / 128 * 128;  // tokens the windows cover
  int64_t W = 0;
  if (const char* env = getenv("MOBA_WINDOW")) {
    W = atoll(env);
    W = std::max<int64_t>(128, (W + 127) / 128 * 128);
  } else {
    const size_t budget = std::max<size_t>((size_t)64 << 20, window_budget() / std::max(share, 1));
    const size_t per = window_bytes(p, 128);
    W = std::max<int64_t>(1, (int64_t)(budget / std::max<size_t>(per, 1))) * 128;
    if (W > 1024 && W % 1024) W = W / 1024 * 1024;
  }
  W = std::min(W, S128);
  // list slots, positions and a window's rows (token x head) are 32-bit
  const int64_t per_tok = (int64_t)Hq * std::max(p.P, 1);
  while (W > 128 && W * per_tok >= ((int64_t)1 << 31) - 1) W = std::max<int64_t>(128, W / 2 / 128 * 128);
  if (W * per_tok >= ((int64_t)1 << 31) - 1) return fail(MOBA_ERR_UNSUPPORTED, "window too large");
  layout_for_window(p, W);
  return MOBA_OK;
}

// Block-mean rows as a 2-D tensor [Hkv * nbp_pad][128] bf16; box 64 x 32,
// 128-byte swizzle (one 64-channel half of 32 blocks per load).
int make_mean_map(CUtensorMap* map, const void* base, int64_t rows) {
  cuuint64_t dims[2] = {(cuuint64_t)moba::kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)moba::kHeadDim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)moba::kGateBoxRows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOBA_ERR_CUDA, "cuTensorMapEncodeTiled (block means) failed (%d)", (int)r);
  return MOBA_OK;
}

// Launches a pipeline kernel with programmatic stream serialization: it may
// be scheduled while the previous kernel on the stream is still running; the
// kernel itself waits for that kernel's completion before reading anything
// (grid_dependency_sync in common.cuh).
template <typename... KArgs, typename... Args>
void launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int KP>
void launch_gate_tc(const Plan& p, const CUtensorMap& mhi, const CUtensorMap& mlo, const CUtensorMap& mq,
                    moba::GateParams gp, int sms, cudaStream_t st) {
  dim3 grid((unsigned)(((gp.t_end - gp.t_begin) * p.G + 127) / 128), p.Hkv);
  // a grid that fits one wave (four CTAs per SM) takes the single pass
  gp.one_pass = (int64_t)grid.x * grid.y <= 4 * (int64_t)sms ? 1 : 0;
  launch_chained(moba::gate_tc_kernel<KP>, grid, dim3(moba::kGateTcThreads), moba::GateCfg<KP>::kSmemBytes, st, mhi,
                 mlo, mq, gp);
}

// q [S - q0][Hq][128] bf16 as 3-D (channel, head, token) for the gate's Q
// tiles: box 64 x G x 128/G (one 64-channel half of 128 group-rows), 128-byte
// swizzle. Only when G divides 128.
int make_gate_q_map(CUtensorMap* map, const void* q, int64_t ntok, int Hq, int G) {
  cuuint64_t dims[3] = {(cuuint64_t)moba::kHeadDim, (cuuint64_t)Hq, (cuuint64_t)ntok};
  cuuint64_t strides[2] = {(cuuint64_t)moba::kHeadDim * 2, (cuuint64_t)Hq * moba::kHeadDim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)(128 / G)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MOBA_ERR_CUDA, "cuTensorMapEncodeTiled (gate q) failed (%d)", (int)r);
  return MOBA_OK;
}

// Rows that need no scores (topk 1, or every past block): sel written
// directly, no inputs read.
bool gate_free(const Plan& p) { return p.P == 0 || p.k_eff == p.nb || p.nbp <= 0; }

void launch_sel_fill(const Plan& p, int32_t* sel, cudaStream_t st) {
  const int64_t n = (p.S - p.q0) * p.Hq;
  launch_chained(moba::sel_fill_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, sel, p.S, p.q0, p.Hq, p.B,
                 p.k_eff, p.k_eff == p.nb ? 1 : 0);
}

// Block means [j0, j1) (fp32, `splits` partial sums each) into the padded
// bf16 hi/lo rows the gate reads; the range ending at nbp also writes the
// zero padding rows up to the chunk multiple.
void launch_mean_split(const Plan& p, const float* kmean, int splits, __nv_bfloat16* khi, __nv_bfloat16* klo, int j0,
                       int j1, cudaStream_t st) {
  const int nbp_pad = moba::gate_rows_padded(p.nbp);
  if (j1 >= p.nbp) j1 = nbp_pad;
  if (j1 <= j0) return;
  launch_chained(moba::kmean_split_kernel, dim3(j1 - j0, p.Hkv), dim3(128), 0, st, kmean, splits, p.nbp, nbp_pad, j0,
                 khi, klo);
}

// The gate's scores and top-k for the rows of tokens [t_begin, t_end), from
// the hi/lo block means. Returns -status on failure, else 0.
int launch_gate_rows(const Plan& p, const void* q, const __nv_bfloat16* khi, const __nv_bfloat16* klo, int32_t* sel,
                     int64_t t_begin, int64_t t_end, cudaStream_t st) {
  const int nbp_pad = moba::gate_rows_padded(p.nbp);
  CUtensorMap mhi, mlo;
  int rc = make_mean_map(&mhi, khi, (int64_t)p.Hkv * nbp_pad);
  if (rc) return -rc;
  rc = make_mean_map(&mlo, klo, (int64_t)p.Hkv * nbp_pad);
  if (rc) return -rc;
  // Q tiles by TMA when a CTA's 128 group-rows are whole tokens (G | 128)
  CUtensorMap mq;
  memset(&mq, 0, sizeof(mq));
  const bool q_tma = p.G <= 128 && 128 % p.G == 0;
  if (q_tma) {
    rc = make_gate_q_map(&mq, q, p.S - p.q0, p.Hq, p.G);
    if (rc) return -rc;
  }
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return -rc;
  const int sms = dev.sms;
  moba::GateParams gp;
  gp.q_tma = q_tma ? 1 : 0;
  gp.one_pass = 0;
  gp.q = static_cast<const __nv_bfloat16*>(q);
  gp.sel = sel;
  gp.S = p.S;
  gp.q0 = p.q0;
  gp.t_begin = t_begin;
  gp.t_end = t_end;
  gp.Hq = p.Hq;
  gp.G = p.G;
  gp.B = p.B;
  gp.nbp_pad = nbp_pad;
  gp.k_eff = p.k_eff;
  if (p.P <= 2) launch_gate_tc<2>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 4) launch_gate_tc<4>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 8) launch_gate_tc<8>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P == 11) launch_gate_tc<11>(p, mhi, mlo, mq, gp, sms, st);  // top-12: a list of exactly k - 1
  else if (p.P <= 12) launch_gate_tc<12>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 16) launch_gate_tc<16>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 24) launch_gate_tc<24>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 32) launch_gate_tc<32>(p, mhi, mlo, mq, gp, sms, st);
  else if (p.P <= 48) launch_gate_tc<48>(p, mhi, mlo, mq, gp, sms, st);
  else launch_gate_tc<64>(p, mhi, mlo, mq, gp, sms, st);
  return 0;
}

// Gate + top-k into sel for every row. kmean (fp32) is split into khi/klo
// (bf16, padded rows) first. Returns the number of kernels launched, or
// -status.
int launch_gate(const Plan& p, const void* q, const float* kmean, int splits, __nv_bfloat16* khi,
                __nv_bfloat16* klo, int32_t* sel, cudaStream_t st) {
  if (gate_free(p)) {
    launch_sel_fill(p, sel, st);
    return 1;
  }
  launch_mean_split(p, kmean, splits, khi, klo, 0, p.nbp, st);
  const int rc = launch_gate_rows(p, q, khi, klo, sel, p.q0, p.S, st);
  return rc < 0 ? rc : 2;
}

// Means of the complete blocks [j0, j1) (every one by default).
void launch_pool(const Plan& p, const void* k, float* kmean, int splits, cudaStream_t st, int j0 = 0, int j1 = -1) {
  if (j1 < 0 || j1 > p.nbp) j1 = p.nbp;
  if (j1 <= j0) return;
  dim3 grid(j1 - j0, p.Hkv, splits);
  launch_chained(moba::pool_kernel, grid, dim3(moba::kPoolThreads), 0, st, static_cast<const __nv_bfloat16*>(k), p.Hkv,
                 p.B, p.nbp, splits, j0, kmean);
}

// Optional per-stage device timing: an event after every stage, tagged with
// the stage it closes (-1 opens a call); elapsed times between consecutive
// events are summed per stage when the profile ends.
enum Stage {
  kPool = 0,
  kGate = 1,
  kRoute = 2,
  kAttn = 3,
  kMerge = 4,
  kBwdPrep = 5,
  kBwdDq = 6,
  kBwdDkdv = 7,
  kNumStages = 8
};

struct StageTimer {
  bool on = false;
  cudaStream_t st = nullptr;
  int launches = 0;
  int calls = 0;
  struct Mark {
    int stage;
    cudaEvent_t ev;
  };
  std::vector<Mark> marks;
  void mark(int stage) {
    if (!on) return;
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    cudaEventRecord(e, st);
    marks.push_back({stage, e});
  }
  void count(int n) {
    if (on) launches += n;
  }
  int finish(float* ms) {
    for (int i = 0; i < kNumStages; ++i) ms[i] = 0.f;
    cudaError_t err = cudaSuccess;
    if (!marks.empty()) err = cudaEventSynchronize(marks.back().ev);
    for (size_t i = 1; i < marks.size() && err == cudaSuccess; ++i) {
      float d = 0.f;
      if (marks[i].stage >= 0 && cudaEventElapsedTime(&d, marks[i - 1].ev, marks[i].ev) == cudaSuccess)
        ms[marks[i].stage] += d;
    }
    for (auto& m : marks) cudaEventDestroy(m.ev);
    marks.clear();
    on = false;
    if (err != cudaSuccess) return fail(MOBA_ERR_CUDA, "event synchronise failed: %s", cudaGetErrorString(err));
    return MOBA_OK;
  }
};

thread_local StageTimer g_timer;

moba::WindowGeom window_geom(const Plan& p, int64_t w0) {
  moba::WindowGeom wg;
  wg.S = p.S;
  wg.Hq = p.Hq;
  wg.Hkv = p.Hkv;
  wg.G = p.G;
  wg.B = p.B;
  wg.k_eff = p.k_eff;
  wg.nbp = p.nbp;
  wg.w0 = w0;
  wg.wlen = std::min(p.W, p.S - w0);
  wg.q0 = p.q0;
  wg.wwords = (wg.wlen * p.G + 31) / 32;
  wg.pair_tokens = pair_tokens(p) ? 1 : 0;
  wg.list_cap = std::max<int64_t>(p.list_cap, 1);
  return wg;
}

// Some row of the window can have a past block.
bool window_routed(const Plan& p, const moba::WindowGeom& wg) {
  return p.P > 0 && p.nbp > 0 && (wg.w0 + wg.wlen) > p.B;
}

// The router for one query window (flags, counts, scan, fill); returns the
// number of kernels launched, or -status.
int launch_route(const Plan& p, const moba::WindowGeom& wg, bool routed, uint8_t* ws, cudaStream_t st) {
  const int32_t* sel = reinterpret_cast<const int32_t*>(ws + p.o_sel);
  uint32_t* flags = reinterpret_cast<uint32_t*>(ws + p.o_flags);
  int32_t* wordbase = reinterpret_cast<int32_t*>(ws + p.o_wordbase);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + p.o_cnt);
  int32_t* loff = reinterpret_cast<int32_t*>(ws + p.o_loff);
  int32_t* toff = reinterpret_cast<int32_t*>(ws + p.o_toff);
  int32_t* list = reinterpret_cast<int32_t*>(ws + p.o_list);
  int4* tiles = reinterpret_cast<int4*>(ws + p.o_tiles);
  int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.o_hdr);
  const int nbk = p.Hkv * p.nbp;
  int n = 0;
  if (routed) {
    dim3 gf((unsigned)((wg.wwords + 3) / 4), p.Hkv);
    // the flags kernel writes only the words of picked blocks
    if (cudaMemsetAsync(flags, 0, (size_t)nbk * (size_t)wg.wwords * sizeof(uint32_t), st) != cudaSuccess)
      return -fail(MOBA_ERR_CUDA, "cudaMemsetAsync (route flags) failed");
    launch_chained(moba::route_flags_kernel, gf, dim3(moba::kFlagsThreads),
                   (size_t)moba::kFlagsThreads * std::max(p.P, 1) * sizeof(int32_t), st, sel, wg, flags);
    dim3 gb(p.nbp, p.Hkv);
    launch_chained(moba::route_count_kernel, gb, dim3(256), 0, st, static_cast<const uint32_t*>(flags), wg, cnt);
    n += 2;
  }
  launch_chained(moba::route_scan_kernel, dim3(1), dim3(1024), 0, st, static_cast<const int32_t*>(cnt),
                 routed ? nbk : 0, wg, loff, toff, tiles, hdr);
  ++n;
  if (routed) {
    dim3 gb(p.nbp, p.Hkv);
    launch_chained(moba::route_fill_kernel, gb, dim3(256), 0, st, static_cast<const uint32_t*>(flags),
                   static_cast<const int32_t*>(cnt), static_cast<const int32_t*>(loff),
                   static_cast<const int32_t*>(toff), wg, wordbase, list, tiles);
    ++n;
  }
  return n;
}

// Callbacks around each query window [w0, w0 + wlen) of run_forward, for
// the pipelined copies of moba_fwd_host: `inputs` before the window's first
// kernel (which may read q, k, v rows [0, w0 + wlen) and nothing beyond),
// `done` after its merge (out rows and lse columns of the window are final).
// With hooks, the pool, mean split and gate run window by window too.
struct WindowHooks {
  std::function<int(int64_t w0, int64_t wlen)> inputs, done;
};

int run_forward(const Plan& p, const DeviceInfo& dev, const void* q, const void* k, const void* v, void* out,
                float* lse, uint8_t* ws, cudaStream_t st, const WindowHooks* hooks = nullptr) {
  StageTimer* tm = &g_timer;
  tm->st = st;
  if (tm->on) tm->calls++;
  float* kmean = p.means ? const_cast<float*>(p.means) : reinterpret_cast<float*>(ws + p.o_kmean);
  const int mean_splits = p.means ? 1 : p.splits;
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.o_sel);
  uint32_t* flags = reinterpret_cast<uint32_t*>(ws + p.o_flags);
  int32_t* wordbase = reinterpret_cast<int32_t*>(ws + p.o_wordbase);
  int32_t* list = reinterpret_cast<int32_t*>(ws + p.o_list);
  int4* tiles = reinterpret_cast<int4*>(ws + p.o_tiles);
  int32_t* hdr = reinterpret_cast<int32_t*>(ws + p.o_hdr);
  __half* part_o = reinterpret_cast<__half*>(ws + p.o_part_o);
  float* part_lse = reinterpret_cast<float*>(ws + p.o_part_lse);
  __half* own_o = reinterpret_cast<__half*>(ws + p.o_own_o);
  float* own_lse = reinterpret_cast<float*>(ws + p.o_own_lse);

  CUtensorMap tmk, tmv;
  int rc = make_kv_map(&tmk, k, p.S, p.Hkv);
  if (rc) return rc;
  rc = make_kv_map(&tmv, v, p.S, p.Hkv);
  if (rc) return rc;

  tm->mark(-1);
  const bool pooled = p.P > 0 && p.k_eff < p.nb && p.nbp > 0 && !p.means;
  __nv_bfloat16* khi = reinterpret_cast<__nv_bfloat16*>(ws + p.o_khi);
  __nv_bfloat16* klo = reinterpret_cast<__nv_bfloat16*>(ws + p.o_klo);
  if (!hooks) {
    if (pooled) {
      launch_pool(p, k, kmean, p.splits, st);
      tm->count(1);
      tm->mark(kPool);
    }
    const int n = launch_gate(p, q, kmean, mean_splits, khi, klo, sel, st);
    if (n < 0) return -n;
    tm->count(n);
    tm->mark(kGate);
  } else if (gate_free(p)) {
    launch_sel_fill(p, sel, st);  // reads no input
  }
  int j_done = 0;  // windowed: blocks pooled and split so far

  moba::AttnParams ap;
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.list = list;
  ap.units = tiles;
  ap.hdr = hdr;
  ap.part_o = part_o;
  ap.part_lse = part_lse;
  ap.own_o = own_o;
  ap.own_lse = own_lse;
  ap.S = p.S;
  ap.q0 = p.q0;
  ap.Hq = p.Hq;
  ap.G = p.G;
  ap.B = p.B;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)moba::kHeadDim));

  for (int64_t w0 = p.wbase; w0 < p.S; w0 += p.W) {
    const moba::WindowGeom wg = window_geom(p, w0);
    if (hooks) {
      int hr = hooks->inputs(w0, wg.wlen);
      if (hr) return hr;
      if (!gate_free(p)) {
        // the blocks this window completes, then the gate of its rows (their
        // past blocks all end at or before the window's end)
        const int j_new = (int)std::min<int64_t>(p.nbp, (w0 + wg.wlen) / p.B);
        if (j_new > j_done) {
          if (pooled) launch_pool(p, k, kmean, p.splits, st, j_done, j_new);
          launch_mean_split(p, kmean, mean_splits, khi, klo, j_done, j_new, st);
          j_done = j_new;
        }
        hr = launch_gate_rows(p, q, khi, klo, sel, std::max(w0, p.q0), w0 + wg.wlen, st);
        if (hr < 0) return -hr;
      }
    }
    const bool routed = window_routed(p, wg);
    const int nr = launch_route(p, wg, routed, ws, st);
    if (nr < 0) return -nr;
    tm->count(nr);
    tm->mark(kRoute);
    ap.w0 = w0;
    ap.wlen = wg.wlen;
    launch_chained(moba::attn_kernel, dim3(dev.sms), dim3(moba::kAttnThreads), moba::kAttnSmemBytes, st, tmk, tmv, ap);
    tm->count(1);
    tm->mark(kAttn);
    moba::MergeParams mp;
    mp.sel = sel;
    mp.flags = flags;
    mp.wordbase = wordbase;
    mp.part_o = part_o;
    mp.part_lse = part_lse;
    mp.own_o = own_o;
    mp.own_lse = own_lse;
    mp.out = static_cast<__nv_bfloat16*>(out);
    mp.lse = lse;
    mp.lse_ld = p.lse_ld;
    mp.w = wg;
    const int64_t rows = wg.wlen * p.Hq;
    const dim3 mg((unsigned)((rows + 15) / 16));
    if (p.P <= 2) launch_chained(moba::merge_kernel<2>, mg, dim3(256), 0, st, mp);
    else if (p.P <= 4) launch_chained(moba::merge_kernel<4>, mg, dim3(256), 0, st, mp);
    else if (p.P <= 8) launch_chained(moba::merge_kernel<8>, mg, dim3(256), 0, st, mp);
    else if (p.P <= 12) launch_chained(moba::merge_kernel<12>, mg, dim3(256), 0, st, mp);
    else if (p.P <= 16) launch_chained(moba::merge_kernel<16>, mg, dim3(256), 0, st, mp);
    else launch_chained(moba::merge_kernel<0>, mg, dim3(256), 0, st, mp);
    tm->count(1);
    tm->mark(kMerge);
    if (hooks) {
      const int hr = hooks->done(w0, wg.wlen);
      if (hr) return hr;
    }
  }
  MOBA_CUDA(cudaGetLastError());
  return MOBA_OK;
}

// Scratch of the backward pass beyond the forward's layout: lse * log2(e)
// and D = rowsum(dO * O) per row, and fp32 dK / dV accumulators.
struct BwdLayout {
  size_t o_lse2, o_dd, o_dk, o_dv, total;
};

BwdLayout bwd_layout(const Plan& p) {
  BwdLayout b;
  Carve c;
  c.off = p.total;
  b.o_lse2 = c.take((size_t)p.Hq * p.S * 4);
  b.o_dd = c.take((size_t)p.Hq * p.S * 4);
  b.o_dk = c.take((size_t)p.S * p.Hkv * moba::kHeadDim * 4);
  b.o_dv = c.take((size_t)p.S * p.Hkv * moba::kHeadDim * 4);
  b.total = c.off;
  return b;
}

// The backward launch sequence: the forward's pool, gate and router (so the
// selection is the forward's), then per query window the dQ partials, their
// reduction and the window's dK / dV contributions; the fp32 accumulators are
// cast to bf16 at the end.
int run_backward(const Plan& p, const BwdLayout& bl, const DeviceInfo& dev, const void* q, const void* k,
                 const void* v, const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                 uint8_t* ws, cudaStream_t st) {
  StageTimer* tm = &g_timer;
  tm->st = st;
  if (tm->on) tm->calls++;
  float* kmean = reinterpret_cast<float*>(ws + p.o_kmean);
  int32_t* sel = reinterpret_cast<int32_t*>(ws + p.o_sel);
  float* lse2 = reinterpret_cast<float*>(ws + bl.o_lse2);
  float* dd = reinterpret_cast<float*>(ws + bl.o_dd);
  float* dk_acc = reinterpret_cast<float*>(ws + bl.o_dk);
  float* dv_acc = reinterpret_cast<float*>(ws + bl.o_dv);
  CUtensorMap tmk, tmv;
  int rc = make_kv_map(&tmk, k, p.S, p.Hkv);
  if (rc) return rc;
  rc = make_kv_map(&tmv, v, p.S, p.Hkv);
  if (rc) return rc;

  tm->mark(-1);
  if (p.P > 0 && p.k_eff < p.nb && p.nbp > 0) {
    launch_pool(p, k, kmean, p.splits, st);
    tm->count(1);
    tm->mark(kPool);
  }
  {
    const int n = launch_gate(p, q, kmean, p.splits, reinterpret_cast<__nv_bfloat16*>(ws + p.o_khi),
                              reinterpret_cast<__nv_bfloat16*>(ws + p.o_klo), sel, st);
    if (n < 0) return -n;
    tm->count(n);
  }
  tm->mark(kGate);
  {
    const int64_t rows = p.S * p.Hq;
    launch_chained(moba::bwd_prep_kernel, dim3((unsigned)((rows + 7) / 8)), dim3(256), 0, st,
                   static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, p.S, p.Hq,
                   lse2, dd);
    const int64_t n4 = 2 * p.S * p.Hkv * moba::kHeadDim / 4;  // dK then dV accumulators, contiguous
    launch_chained(moba::bwd_zero_kernel, dim3((unsigned)std::min<int64_t>((n4 + 255) / 256, dev.sms * 16)),
                   dim3(256), 0, st, reinterpret_cast<float4*>(dk_acc), n4);
    tm->count(2);
  }
  tm->mark(kBwdPrep);

  moba::AttnParams ap;
  ap.q = static_cast<const __nv_bfloat16*>(q);
  ap.list = reinterpret_cast<const int32_t*>(ws + p.o_list);
  ap.units = reinterpret_cast<const int4*>(ws + p.o_tiles);
  ap.hdr = reinterpret_cast<int32_t*>(ws + p.o_hdr);
  ap.part_o = reinterpret_cast<__half*>(ws + p.o_part_o);
  ap.part_lse = reinterpret_cast<float*>(ws + p.o_part_lse);
  ap.own_o = reinterpret_cast<__half*>(ws + p.o_own_o);
  ap.own_lse = reinterpret_cast<float*>(ws + p.o_own_lse);
  ap.S = p.S;
  ap.q0 = 0;
  ap.Hq = p.Hq;
  ap.G = p.G;
  ap.B = p.B;
  ap.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)moba::kHeadDim));
  moba::BwdParams bp;
  bp.q = static_cast<const __nv_bfloat16*>(q);
  bp.dout = static_cast<const __nv_bfloat16*>(dout);
  bp.lse2 = lse2;
  bp.dd = dd;
  bp.S = p.S;
  bp.Hq = p.Hq;
  bp.Hkv = p.Hkv;
  bp.G = p.G;
  bp.B = p.B;
  bp.nbp = p.nbp;
  bp.scale_log2 = ap.scale_log2;
  bp.scale = (float)(1.0 / std::sqrt((double)moba::kHeadDim));
  moba::DkdvParams dp;
  dp.list = ap.list;
  dp.cnt = reinterpret_cast<const int32_t*>(ws + p.o_cnt);
  dp.loff = reinterpret_cast<const int32_t*>(ws + p.o_loff);
  dp.dk_acc = dk_acc;
  dp.dv_acc = dv_acc;

  for (int64_t w0 = 0; w0 < p.S; w0 += p.W) {
    const moba::WindowGeom wg = window_geom(p, w0);
    const bool routed = window_routed(p, wg);
    const int nr = launch_route(p, wg, routed, ws, st);
    if (nr < 0) return -nr;
    tm->count(nr);
    tm->mark(kRoute);
    ap.w0 = w0;
    ap.wlen = wg.wlen;
    bp.w0 = w0;
    bp.wlen = wg.wlen;
    launch_chained(moba::bwd_dq_kernel, dim3(dev.sms), dim3(moba::kDqThreads), moba::kDqSmemBytes, st, tmk, tmv,
                   ap, bp);
    launch_chained(moba::bwd_dq_reduce_kernel, dim3((unsigned)((wg.wlen * p.Hq + 7) / 8)), dim3(256), 0, st,
                   static_cast<const int32_t*>(sel), reinterpret_cast<const uint32_t*>(ws + p.o_flags),
                   reinterpret_cast<const int32_t*>(ws + p.o_wordbase), static_cast<const __half*>(ap.part_o),
                   static_cast<const __half*>(ap.own_o), wg, static_cast<__nv_bfloat16*>(dq));
    tm->count(2);
    tm->mark(kBwdDq);
    dp.routed = routed ? 1 : 0;
    launch_chained(moba::bwd_dkdv_kernel, dim3((unsigned)((int64_t)(p.B / moba::kTile) * p.nb * p.Hkv)),
                   dim3(moba::kDkdvThreads), moba::kBwdSmemBytes, st, tmk, tmv, bp, dp);
    tm->count(1);
    tm->mark(kBwdDkdv);
  }
  {
    const int64_t n4 = p.S * p.Hkv * moba::kHeadDim / 4;
    const dim3 gc((unsigned)std::min<int64_t>((n4 + 255) / 256, dev.sms * 16));
    launch_chained(moba::bwd_cast_kernel, gc, dim3(256), 0, st, reinterpret_cast<const float4*>(dk_acc),
                   static_cast<__nv_bfloat16*>(dk), n4);
    launch_chained(moba::bwd_cast_kernel, gc, dim3(256), 0, st, reinterpret_cast<const float4*>(dv_acc),
                   static_cast<__nv_bfloat16*>(dv), n4);
    tm->count(2);
    tm->mark(kBwdDkdv);
  }
  MOBA_CUDA(cudaGetLastError());
  return MOBA_OK;
}

}  // namespace

extern "C" const char* moba_last_error(void) { return g_err.c_str(); }

namespace {

// A launch sequence over one scratch buffer of `total` bytes.
using Runner = std::function<int(uint8_t* ws, cudaStream_t st)>;

bool g_pool_kept[64] = {};

// The entry points that take stream-ordered scratch raise the release
// threshold of the device's default pool once, so scratch freed at the end
// of a call stays reserved for the next one. (moba_fwd_noalloc never gets
// here: it leaves the caller's allocator alone.)
void keep_freed_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return;
  }
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_pool_kept[dev]) return;
  cudaMemPool_t pool;
  if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
    uint64_t thr = UINT64_MAX;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
  }
  cudaGetLastError();
  g_pool_kept[dev] = true;
}

// Bytes to request for `total` bytes of scratch. MOBA_TEST_SCRATCH_PAD=<n>
// adds n bytes to every request: a test hook that makes the stream-ordered
// allocation fail on purpose, so the MOBA_ERR_OOM path can be exercised.
size_t scratch_request(size_t total) {
  const char* e = getenv("MOBA_TEST_SCRATCH_PAD");
  return e ? total + (size_t)strtoull(e, nullptr, 10) : total;
}

// The launch sequence with stream-ordered scratch, issued on `stream`.
int direct_run(size_t total, const Runner& run, cudaStream_t stream) {
  keep_freed_scratch();
  void* ws = nullptr;
  total = scratch_request(total);
  cudaError_t e = cudaMallocAsync(&ws, total, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOBA_ERR_OOM, "scratch allocation of %zu bytes failed: %s", total, cudaGetErrorString(e));
  }
  int rc = run(static_cast<uint8_t*>(ws), stream);
  cudaError_t ef = cudaFreeAsync(ws, stream);
  if (rc) return rc;
  if (ef != cudaSuccess) return fail(MOBA_ERR_CUDA, "cudaFreeAsync failed: %s", cudaGetErrorString(ef));
  return MOBA_OK;
}

// Repeated calls with the same buffers and shape replay a CUDA graph of the
// whole launch sequence (scratch allocation and release included as graph
// memory nodes), so the host enqueues one graph launch instead of about ten
// kernels per sequence. Graphs are captured on an internal stream, launched
// on the caller's, and kept for the last kGraphCache argument sets; a set is
// only captured the second time it is seen. MOBA_GRAPH=0 turns this off.
struct GraphKey {
  int dev;
  const void *q, *k, *v;
  void* out;
  float* lse;
  const float* means;
  int64_t S, q0, W, lse_ld;
  int Hq, Hkv, B, topk;
  std::vector<int64_t> cu;  // a packed batch's sequence offsets (empty: one sequence)
  bool operator==(const GraphKey& o) const {
    return dev == o.dev && q == o.q && k == o.k && v == o.v && out == o.out && lse == o.lse && means == o.means &&
           S == o.S && q0 == o.q0 && W == o.W && lse_ld == o.lse_ld && Hq == o.Hq && Hkv == o.Hkv && B == o.B &&
           topk == o.topk && cu == o.cu;
  }
};

struct GraphEntry {
  GraphKey key;
  cudaGraphExec_t exec;  // set once captured
  int state;             // 0 seen once, 1 captured, 2 capture failed
};

constexpr size_t kGraphCache = 16;
std::mutex g_graph_mu;
std::vector<GraphEntry> g_graphs;
cudaStream_t g_capture_stream[64] = {};

bool graphs_enabled() {
  const char* e = getenv("MOBA_GRAPH");
  return !(e && e[0] == '0');
}

// MOBA_OK / error after launching a graph; -1 when the caller should launch
// directly. key.dev is filled in here.
int graph_run(GraphKey key, size_t total, const Runner& run, cudaStream_t stream) {
  if (!graphs_enabled() || getenv("MOBA_TEST_SCRATCH_PAD")) return -1;
  keep_freed_scratch();
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return -1;
  key.dev = d;
  std::lock_guard<std::mutex> lk(g_graph_mu);
  GraphEntry* hit = nullptr;
  for (GraphEntry& en : g_graphs)
    if (en.key == key) hit = &en;
  if (hit && hit->state == 1) {
    cudaError_t e = cudaGraphLaunch(hit->exec, stream);
    if (e != cudaSuccess) return fail(MOBA_ERR_CUDA, "cudaGraphLaunch failed: %s", cudaGetErrorString(e));
    return MOBA_OK;
  }
  if (hit && hit->state == 2) return -1;
  if (!hit) {
    // first sighting: launch directly; capture only when the same buffers
    // and shape come back
    if (g_graphs.size() >= kGraphCache) {
      if (g_graphs.front().state == 1) cudaGraphExecDestroy(g_graphs.front().exec);
      g_graphs.erase(g_graphs.begin());
    }
    g_graphs.push_back({std::move(key), nullptr, 0});
    return -1;
  }
  if (!g_capture_stream[d] && cudaStreamCreateWithFlags(&g_capture_stream[d], cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    g_capture_stream[d] = nullptr;
    return -1;
  }
  cudaStream_t cs = g_capture_stream[d];
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  bool ok = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
  if (ok) {
    void* ws = nullptr;
    ok = cudaMallocAsync(&ws, total, cs) == cudaSuccess;
    if (ok) {
      ok = run(static_cast<uint8_t*>(ws), cs) == MOBA_OK;
      ok = (cudaFreeAsync(ws, cs) == cudaSuccess) && ok;
    }
    ok = (cudaStreamEndCapture(cs, &graph) == cudaSuccess) && ok;
    ok = ok && graph && cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess;
  }
  if (graph) cudaGraphDestroy(graph);
  if (!ok) {
    cudaGetLastError();
    if (exec) cudaGraphExecDestroy(exec);
    exec = nullptr;
    g_err.clear();
  }
  hit->exec = exec;
  hit->state = exec ? 1 : 2;
  if (!exec) return -1;
  cudaError_t e = cudaGraphLaunch(exec, stream);
  if (e != cudaSuccess) return fail(MOBA_ERR_CUDA, "cudaGraphLaunch failed: %s", cudaGetErrorString(e));
  return MOBA_OK;
}

int fwd_impl(const void* q, const void* k, const void* v, int64_t seqlen, int64_t q_start, int heads_q, int heads_kv,
             int head_dim, int block_size, int topk, void* out, float* lse, cudaStream_t stream, bool use_graph,
             const float* means = nullptr) {
  g_err.clear();
  if (!q || !k || !v || !out || !lse) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_q, heads_kv, head_dim, block_size, topk);
  if (rc) return rc;
  if (q_start < 0 || q_start >= seqlen)
    return fail(MOBA_ERR_INVALID_ARG, "q_start must be in [0, seqlen) (got %lld, seqlen %lld)", (long long)q_start,
                (long long)seqlen);
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  Plan p;
  rc = make_plan(&p, seqlen, q_start, heads_q, heads_kv, block_size, topk);
  if (rc) return rc;
  if (means && !aligned16(means)) return fail(MOBA_ERR_INVALID_ARG, "kmean must be 16-byte aligned");
  p.means = means;
  const Runner run = [&](uint8_t* ws, cudaStream_t st) { return run_forward(p, dev, q, k, v, out, lse, ws, st); };
  if (use_graph && !g_timer.on) {
    GraphKey key{0, q, k, v, out, lse, p.means, p.S, p.q0, p.W, p.lse_ld, p.Hq, p.Hkv, p.B, p.topk, {}};
    const int g = graph_run(std::move(key), p.total, run, stream);
    if (g >= 0) return finish_call(g, stream);  // negative: no graph for this call, launch directly
  }
  return finish_call(direct_run(p.total, run, stream), stream);
}

constexpr int kVarlenLanes = 4;
cudaStream_t g_lane_streams[64][kVarlenLanes] = {};

// The internal streams a packed batch's sequences run on (created once per
// device).
int lane_streams(cudaStream_t** out) {
  int dev = 0;
  MOBA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOBA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  for (int l = 0; l < kVarlenLanes; ++l)
    if (!g_lane_streams[dev][l]) MOBA_CUDA(cudaStreamCreateWithFlags(&g_lane_streams[dev][l], cudaStreamNonBlocking));
  *out = g_lane_streams[dev];
  return MOBA_OK;
}

// A packed batch of independent sequences: sequence b holds tokens
// cu[b] .. cu[b+1]-1 of q, k, v and out, and columns cu[b] .. of lse. The
// sequences are dealt, longest first, onto up to four lanes (the least
// loaded lane takes the next one); each lane has its own part of the scratch
// and its own stream, forked from and joined back to the caller's stream, so
// the small kernels of short sequences overlap and one sequence's attention
// tail is filled by the next one's. Within a lane the sequences run one
// after another. Replayed as one graph when the same batch comes back.
// (Under moba_profile_begin the sequences run one after another on the
// caller's stream, so that the per-stage times stay meaningful.)
int varlen_impl(const void* q, const void* k, const void* v, const int64_t* cu, int batch, int heads_q, int heads_kv,
                int head_dim, int block_size, int topk, void* out, float* lse, cudaStream_t stream) {
  g_err.clear();
  if (!q || !k || !v || !out || !lse || !cu) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  if (batch < 1) return fail(MOBA_ERR_INVALID_ARG, "batch must be >= 1 (got %d)", batch);
  if (cu[0] != 0) return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens[0] must be 0 (got %lld)", (long long)cu[0]);
  for (int b = 0; b < batch; ++b)
    if (cu[b + 1] < cu[b])
      return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing (cu_seqlens[%d] = %lld < %lld)", b + 1,
                  (long long)cu[b + 1], (long long)cu[b]);
  const int64_t T = cu[batch];
  if (T < 1) return fail(MOBA_ERR_INVALID_ARG, "the batch holds no tokens");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
    return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(lse) & 3) return fail(MOBA_ERR_INVALID_ARG, "lse must be 4-byte aligned");
  std::vector<int> seqs;  // non-empty sequences, longest first
  for (int b = 0; b < batch; ++b) {
    const int64_t L = cu[b + 1] - cu[b];
    if (!L) continue;  // an empty sequence has nothing to compute
    int rc = check_shape(L, heads_q, heads_kv, head_dim, block_size, topk);
    if (rc) return rc;
    seqs.push_back(b);
  }
  std::stable_sort(seqs.begin(), seqs.end(),
                   [&](int a, int b) { return cu[a + 1] - cu[a] > cu[b + 1] - cu[b]; });
  const bool serial = g_timer.on;
  const int nlanes = serial ? 1 : std::min<int>(kVarlenLanes, (int)seqs.size());
  std::vector<Plan> plans;
  std::vector<int64_t> starts;
  std::vector<int> lane_of;
  std::vector<int64_t> lane_tokens(nlanes, 0);
  std::vector<size_t> lane_bytes(nlanes, 0);
  for (int b : seqs) {
    const int64_t L = cu[b + 1] - cu[b];
    Plan p;
    int rc = make_plan(&p, L, 0, heads_q, heads_kv, block_size, topk, nlanes);
    if (rc) return rc;
    p.lse_ld = T;
    int l = 0;
    for (int i = 1; i < nlanes; ++i)
      if (lane_tokens[i] < lane_tokens[l]) l = i;
    lane_tokens[l] += L;
    lane_bytes[l] = std::max(lane_bytes[l], p.total);
    plans.push_back(p);
    starts.push_back(cu[b]);
    lane_of.push_back(l);
  }
  std::vector<size_t> lane_off(nlanes, 0);
  size_t total = 0;
  for (int l = 0; l < nlanes; ++l) {
    lane_off[l] = total;
    total += (lane_bytes[l] + 255) & ~size_t(255);
  }
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  cudaStream_t* lanes = nullptr;
  if (nlanes > 1) {
    rc = lane_streams(&lanes);
    if (rc) return rc;
  }
  const size_t qrow = (size_t)heads_q * head_dim * 2, kvrow = (size_t)heads_kv * head_dim * 2;
  const Runner run = [&](uint8_t* ws, cudaStream_t st) {
    auto seq = [&](size_t i, cudaStream_t s) {
      const size_t t0 = (size_t)starts[i];
      return run_forward(plans[i], dev, static_cast<const uint8_t*>(q) + t0 * qrow,
                         static_cast<const uint8_t*>(k) + t0 * kvrow, static_cast<const uint8_t*>(v) + t0 * kvrow,
                         static_cast<uint8_t*>(out) + t0 * qrow, lse + t0, ws + lane_off[lane_of[i]], s);
    };
    if (nlanes == 1) {
      for (size_t i = 0; i < plans.size(); ++i) {
        const int r = seq(i, st);
        if (r) return r;
      }
      return (int)MOBA_OK;
    }
    // fork the lanes from the caller's stream and join them back
    cudaEvent_t fork = nullptr, join[kVarlenLanes] = {};
    MOBA_CUDA(cudaEventCreateWithFlags(&fork, cudaEventDisableTiming));
    MOBA_CUDA(cudaEventRecord(fork, st));
    int r = MOBA_OK;
    for (int l = 0; l < nlanes && !r; ++l) {
      if (cudaStreamWaitEvent(lanes[l], fork, 0) != cudaSuccess) r = fail(MOBA_ERR_CUDA, "cudaStreamWaitEvent failed");
      for (size_t i = 0; i < plans.size() && !r; ++i)
        if (lane_of[i] == l) r = seq(i, lanes[l]);
      if (!r && (cudaEventCreateWithFlags(&join[l], cudaEventDisableTiming) != cudaSuccess ||
                 cudaEventRecord(join[l], lanes[l]) != cudaSuccess || cudaStreamWaitEvent(st, join[l], 0) != cudaSuccess))
        r = fail(MOBA_ERR_CUDA, "joining the lane streams failed");
    }
    cudaEventDestroy(fork);
    for (int l = 0; l < nlanes; ++l)
      if (join[l]) cudaEventDestroy(join[l]);
    return r;
  };
  if (!g_timer.on) {
    GraphKey key{0, q, k, v, out, lse, nullptr, T, 0, 0, T, heads_q, heads_kv, block_size, topk,
                 std::vector<int64_t>(cu, cu + batch + 1)};
    const int g = graph_run(std::move(key), total, run, stream);
    if (g >= 0) return finish_call(g, stream);
  }
  return finish_call(direct_run(total, run, stream), stream);
}

cudaStream_t g_copy_streams[64][2] = {};

// The internal copy streams of moba_fwd_host (host to device, device to
// host), created once per device.
int copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  int dev = 0;
  MOBA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOBA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  for (int i = 0; i < 2; ++i)
    if (!g_copy_streams[dev][i]) MOBA_CUDA(cudaStreamCreateWithFlags(&g_copy_streams[dev][i], cudaStreamNonBlocking));
  *h2d = g_copy_streams[dev][0];
  *d2h = g_copy_streams[dev][1];
  return MOBA_OK;
}

// moba_fwd on host buffers, pipelined by query window: the q, k, v rows a
// window needs go up on one copy stream ahead of its kernels (pool, gate,
// router, attention and merge all run window by window), and its out rows
// and lse columns come back on another while the next window computes. So
// only the first window's inputs and the last window's outputs are not
// hidden behind kernels.
int host_impl(const void* q_host, const void* k_host, const void* v_host, int64_t seqlen, int heads_q, int heads_kv,
              int head_dim, int block_size, int topk, void* out_host, float* lse_host, cudaStream_t stream) {
  g_err.clear();
  if (!q_host || !k_host || !v_host || !out_host || !lse_host) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_q, heads_kv, head_dim, block_size, topk);
  if (rc) return rc;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  Plan p;
  rc = make_plan(&p, seqlen, 0, heads_q, heads_kv, block_size, topk);
  if (rc) return rc;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  rc = copy_streams(&h2d, &d2h);
  if (rc) return rc;
  const size_t qrow = (size_t)heads_q * head_dim * 2, kvrow = (size_t)heads_kv * head_dim * 2;
  const size_t qb = (size_t)seqlen * qrow, kb = (size_t)seqlen * kvrow, lb = (size_t)seqlen * heads_q * 4;
  Carve c;
  const size_t oq = c.take(qb), ok = c.take(kb), ov = c.take(kb), oo = c.take(qb), ol = c.take(lb);
  keep_freed_scratch();
  void* buf = nullptr;
  cudaError_t e = cudaMallocAsync(&buf, c.off, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOBA_ERR_OOM, "device buffers of %zu bytes: %s", c.off, cudaGetErrorString(e));
  }
  void* ws = nullptr;
  const size_t total = scratch_request(p.total);
  e = cudaMallocAsync(&ws, total, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaFreeAsync(buf, stream);
    cudaStreamSynchronize(stream);
    return fail(MOBA_ERR_OOM, "scratch allocation of %zu bytes failed: %s", total, cudaGetErrorString(e));
  }
  uint8_t* b = static_cast<uint8_t*>(buf);
  const uint8_t* qh = static_cast<const uint8_t*>(q_host);
  const uint8_t* kh = static_cast<const uint8_t*>(k_host);
  const uint8_t* vh = static_cast<const uint8_t*>(v_host);

  // one event per window each way, plus the fork from and the joins back to
  // the caller's stream
  const int64_t nwin = (p.S - p.wbase + p.W - 1) / p.W;
  std::vector<cudaEvent_t> ev(2 * (size_t)nwin + 3, nullptr);
  for (auto& x : ev)
    if (!rc && cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess)
      rc = fail(MOBA_ERR_CUDA, "cudaEventCreate failed");
  cudaEvent_t ev_alloc = ev[2 * nwin], ev_h2d_end = ev[2 * nwin + 1], ev_d2h_end = ev[2 * nwin + 2];
  auto ev_in = [&](int64_t i) { return ev[2 * i]; };
  auto ev_out = [&](int64_t i) { return ev[2 * i + 1]; };
  bool h2d_forked = false, d2h_forked = false;
  if (!rc) {
    // the copy streams start once the buffers exist
    if (cudaEventRecord(ev_alloc, stream) != cudaSuccess || cudaStreamWaitEvent(h2d, ev_alloc, 0) != cudaSuccess ||
        cudaStreamWaitEvent(d2h, ev_alloc, 0) != cudaSuccess)
      rc = fail(MOBA_ERR_CUDA, "forking the copy streams failed");
    else
      h2d_forked = d2h_forked = true;
  }
  // inputs, window by window: rows [done, w0 + wlen) of k (pool), q (gate),
  // v (attention)
  int64_t done = 0;
  for (int64_t i = 0; i < nwin && !rc; ++i) {
    const int64_t w0 = p.wbase + i * p.W, hi = std::min(p.S, w0 + p.W);
    const int64_t n = hi - done;
    if (cudaMemcpyAsync(b + ok + done * kvrow, kh + done * kvrow, n * kvrow, cudaMemcpyHostToDevice, h2d) !=
            cudaSuccess ||
        cudaMemcpyAsync(b + oq + done * qrow, qh + done * qrow, n * qrow, cudaMemcpyHostToDevice, h2d) != cudaSuccess ||
        cudaMemcpyAsync(b + ov + done * kvrow, vh + done * kvrow, n * kvrow, cudaMemcpyHostToDevice, h2d) !=
            cudaSuccess ||
        cudaEventRecord(ev_in(i), h2d) != cudaSuccess)
      rc = fail(MOBA_ERR_CUDA, "host to device copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    done = hi;
  }
  WindowHooks hooks;
  hooks.inputs = [&](int64_t w0, int64_t) -> int {
    if (cudaStreamWaitEvent(stream, ev_in((w0 - p.wbase) / p.W), 0) != cudaSuccess)
      return fail(MOBA_ERR_CUDA, "waiting for the input copies failed");
    return MOBA_OK;
  };
  hooks.done = [&](int64_t w0, int64_t wlen) -> int {
    cudaEvent_t x = ev_out((w0 - p.wbase) / p.W);
    if (cudaEventRecord(x, stream) != cudaSuccess || cudaStreamWaitEvent(d2h, x, 0) != cudaSuccess ||
        cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + w0 * qrow, b + oo + w0 * qrow, wlen * qrow,
                        cudaMemcpyDeviceToHost, d2h) != cudaSuccess ||
        cudaMemcpy2DAsync(lse_host + w0, (size_t)seqlen * 4, b + ol + w0 * 4, (size_t)seqlen * 4, wlen * 4,
                          heads_q, cudaMemcpyDeviceToHost, d2h) != cudaSuccess)
      return fail(MOBA_ERR_CUDA, "device to host copy failed: %s", cudaGetErrorString(cudaGetLastError()));
    return MOBA_OK;
  };
  if (!rc)
    rc = run_forward(p, dev, b + oq, b + ok, b + ov, b + oo, reinterpret_cast<float*>(b + ol),
                     static_cast<uint8_t*>(ws), stream, &hooks);
  // join both copy streams back before the buffers go
  if (h2d_forked && (cudaEventRecord(ev_h2d_end, h2d) != cudaSuccess ||
                     cudaStreamWaitEvent(stream, ev_h2d_end, 0) != cudaSuccess) && !rc)
    rc = fail(MOBA_ERR_CUDA, "joining the copy streams failed");
  if (d2h_forked && (cudaEventRecord(ev_d2h_end, d2h) != cudaSuccess ||
                     cudaStreamWaitEvent(stream, ev_d2h_end, 0) != cudaSuccess) && !rc)
    rc = fail(MOBA_ERR_CUDA, "joining the copy streams failed");
  cudaFreeAsync(ws, stream);
  cudaFreeAsync(buf, stream);
  const cudaError_t es = cudaStreamSynchronize(stream);
  for (auto& x : ev)
    if (x) cudaEventDestroy(x);
  if (!rc && es != cudaSuccess) rc = fail(MOBA_ERR_CUDA, "stream synchronise failed: %s", cudaGetErrorString(es));
  return finish_call(rc, stream);
}

}  // namespace

extern "C" {

int moba_fwd(const void* q, const void* k, const void* v, int64_t seqlen, int heads_q, int heads_kv, int head_dim,
             int block_size, int topk, void* out, float* lse, cudaStream_t stream) {
  return fwd_impl(q, k, v, seqlen, 0, heads_q, heads_kv, head_dim, block_size, topk, out, lse, stream, true);
}

int moba_fwd_chunk(const void* q, const void* k, const void* v, int64_t seqlen, int64_t q_start, int heads_q,
                   int heads_kv, int head_dim, int block_size, int topk, void* out, float* lse, cudaStream_t stream) {
  return fwd_impl(q, k, v, seqlen, q_start, heads_q, heads_kv, head_dim, block_size, topk, out, lse, stream, true);
}

int moba_fwd_chunk_means(const void* q, const void* k, const void* v, const float* kmean, int64_t seqlen,
                         int64_t q_start, int heads_q, int heads_kv, int head_dim, int block_size, int topk, void* out,
                         float* lse, cudaStream_t stream) {
  if (!kmean) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument (kmean)");
  return fwd_impl(q, k, v, seqlen, q_start, heads_q, heads_kv, head_dim, block_size, topk, out, lse, stream, true,
                  kmean);
}

int moba_fwd_varlen(const void* q, const void* k, const void* v, const int64_t* cu_seqlens, int batch, int heads_q,
                    int heads_kv, int head_dim, int block_size, int topk, void* out, float* lse,
                    cudaStream_t stream) {
  return varlen_impl(q, k, v, cu_seqlens, batch, heads_q, heads_kv, head_dim, block_size, topk, out, lse, stream);
}

int moba_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse, const void* dout,
             int64_t seqlen, int heads_q, int heads_kv, int head_dim, int block_size, int topk, void* dq, void* dk,
             void* dv, cudaStream_t stream) {
  g_err.clear();
  if (!q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv)
    return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_q, heads_kv, head_dim, block_size, topk);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  Plan p;
  rc = make_plan(&p, seqlen, 0, heads_q, heads_kv, block_size, topk);
  if (rc) return rc;
  const BwdLayout bl = bwd_layout(p);
  const Runner run = [&](uint8_t* ws, cudaStream_t st) {
    return run_backward(p, bl, dev, q, k, v, out, lse, dout, dq, dk, dv, ws, st);
  };
  return finish_call(direct_run(bl.total, run, stream), stream);
}

int moba_profile_begin(void) {
  g_err.clear();
  for (auto& m : g_timer.marks) cudaEventDestroy(m.ev);
  g_timer.marks.clear();
  g_timer.launches = 0;
  g_timer.calls = 0;
  g_timer.on = true;
  return MOBA_OK;
}

int moba_profile_end(float* stage_ms, int* launches, int* calls) {
  g_err.clear();
  if (!stage_ms || !launches || !calls) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = g_timer.finish(stage_ms);
  *launches = g_timer.launches;
  *calls = g_timer.calls;
  return rc;
}

int moba_fwd_host(const void* q_host, const void* k_host, const void* v_host, int64_t seqlen, int heads_q,
                  int heads_kv, int head_dim, int block_size, int topk, void* out_host, float* lse_host,
                  cudaStream_t stream) {
  return host_impl(q_host, k_host, v_host, seqlen, heads_q, heads_kv, head_dim, block_size, topk, out_host, lse_host,
                   stream);
}

int moba_pool(const void* k, int64_t seqlen, int heads_kv, int head_dim, int block_size, float* kmean,
              cudaStream_t stream) {
  g_err.clear();
  if (!k || !kmean) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_kv, heads_kv, head_dim, block_size, 1);
  if (rc) return rc;
  if (!aligned16(k) || !aligned16(kmean)) return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  Plan p;
  p.S = seqlen;
  p.Hkv = heads_kv;
  p.B = block_size;
  p.nb = (int)((seqlen + block_size - 1) / block_size);
  p.nbp = p.nb - 1;
  launch_pool(p, k, kmean, 1, stream);
  MOBA_CUDA(cudaGetLastError());
  return finish_call(MOBA_OK, stream);
}

int moba_gate(const void* q, const float* kmean, int64_t seqlen, int heads_q, int heads_kv, int head_dim,
              int block_size, int topk, int32_t* sel, cudaStream_t stream) {
  g_err.clear();
  if (!q || !sel) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_q, heads_kv, head_dim, block_size, topk);
  if (rc) return rc;
  const int nb = (int)((seqlen + block_size - 1) / block_size);
  if (std::min(topk, nb) > 1 && std::min(topk, nb) < nb && !kmean)
    return fail(MOBA_ERR_INVALID_ARG, "kmean is required when the gate chooses");
  if (!aligned16(q)) return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  Plan p;
  p.S = seqlen;
  p.Hq = heads_q;
  p.Hkv = heads_kv;
  p.G = heads_q / heads_kv;
  p.B = block_size;
  p.nb = nb;
  p.nbp = nb - 1;
  p.k_eff = std::min(topk, nb);
  p.P = p.k_eff - 1;
  // bf16 hi/lo parts of the means: stream-ordered scratch for this call
  const size_t part = (size_t)heads_kv * moba::gate_rows_padded(std::max(p.nbp, 1)) * moba::kHeadDim * 2;
  keep_freed_scratch();
  void* parts = nullptr;
  cudaError_t e = cudaMallocAsync(&parts, 2 * part, stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(MOBA_ERR_OOM, "scratch allocation of %zu bytes failed: %s", 2 * part, cudaGetErrorString(e));
  }
  __nv_bfloat16* khi = static_cast<__nv_bfloat16*>(parts);
  const int n = launch_gate(p, q, kmean, 1, khi, khi + part / 2, sel, stream);
  cudaError_t ef = cudaFreeAsync(parts, stream);
  if (n < 0) return -n;
  MOBA_CUDA(cudaGetLastError());
  if (ef != cudaSuccess) return fail(MOBA_ERR_CUDA, "cudaFreeAsync failed: %s", cudaGetErrorString(ef));
  return finish_call(MOBA_OK, stream);
}

int moba_device_status(cudaStream_t stream) {
  g_err.clear();
  MOBA_CUDA(cudaStreamSynchronize(stream));
  int s = 0;
  MOBA_CUDA(cudaMemcpyFromSymbol(&s, moba::g_status, sizeof(int)));
  const int zero = 0;
  MOBA_CUDA(cudaMemcpyToSymbol(moba::g_status, &zero, sizeof(int)));
  DeviceInfo dev;
  if (device_info(&dev) == MOBA_OK && dev.status_host) *reinterpret_cast<volatile int*>(dev.status_host) = 0;
  g_err.clear();
  if (s) fail(s, "a kernel reported device status %d", s);
  return s;
}

}  // extern "C"

namespace moba {

// One thread waits on an mbarrier that nothing ever arrives on.
__global__ void selftest_wait_kernel(uint64_t timeout_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, timeout_cycles);
}

}  // namespace moba

extern "C" int moba_selftest_bounded_wait(int timeout_us, cudaStream_t stream) {
  g_err.clear();
  if (timeout_us < 1 || timeout_us > 2000000) return fail(MOBA_ERR_INVALID_ARG, "timeout_us must be in [1, 2e6]");
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  rc = moba_device_status(stream);  // clear earlier state
  // the bound counts SM cycles; 2000 per microsecond is about the B200 clock
  moba::selftest_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)timeout_us * 2000ull);
  MOBA_CUDA(cudaGetLastError());
  return moba_device_status(stream);
}

// A tiny merge whose router tables are inconsistent on purpose: rows
// 128..255 of a 256-token, 2-block problem route to past block 0, but the
// flag words' list slots start at 2^20 while the list holds one entry. The
// merge kernel must record MOBA_ERR_DEVICE_CHECK and skip those reads (it
// never touches memory outside the buffers allocated here).
extern "C" int moba_selftest_device_check(cudaStream_t stream) {
  g_err.clear();
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  rc = moba_device_status(stream);  // clear earlier state
  if (rc) return rc;
  constexpr int S = 256, K = 2, WW = 8;
  std::vector<int32_t> sel(S * K), wordbase(WW, 1 << 20);
  std::vector<uint32_t> flags(WW, 0u);
  for (int t = 0; t < S; ++t) {  // t < 128: own block 0 only; else past block 0, own block 1
    sel[t * K] = 0;
    sel[t * K + 1] = t < 128 ? -1 : 1;
  }
  for (int w = 4; w < WW; ++w) flags[w] = 0xFFFFFFFFu;
  Carve c;
  const size_t o_sel = c.take(sel.size() * 4), o_flags = c.take(WW * 4), o_wb = c.take(WW * 4),
               o_po = c.take(moba::kHeadDim * 2), o_pl = c.take(4), o_oo = c.take((size_t)S * moba::kHeadDim * 2),
               o_ol = c.take(S * 4), o_out = c.take((size_t)S * moba::kHeadDim * 2), o_lse = c.take(S * 4);
  uint8_t* b = nullptr;
  MOBA_CUDA(cudaMalloc(reinterpret_cast<void**>(&b), c.off));
  rc = MOBA_OK;
  if (cudaMemsetAsync(b, 0, c.off, stream) != cudaSuccess ||
      cudaMemcpyAsync(b + o_sel, sel.data(), sel.size() * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(b + o_flags, flags.data(), WW * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
      cudaMemcpyAsync(b + o_wb, wordbase.data(), WW * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    rc = fail(MOBA_ERR_CUDA, "self-test set-up failed: %s", cudaGetErrorString(cudaGetLastError()));
  if (!rc) {
    moba::MergeParams mp;
    mp.sel = reinterpret_cast<const int32_t*>(b + o_sel);
    mp.flags = reinterpret_cast<const uint32_t*>(b + o_flags);
    mp.wordbase = reinterpret_cast<const int32_t*>(b + o_wb);
    mp.part_o = reinterpret_cast<const __half*>(b + o_po);
    mp.part_lse = reinterpret_cast<const float*>(b + o_pl);
    mp.own_o = reinterpret_cast<const __half*>(b + o_oo);
    mp.own_lse = reinterpret_cast<const float*>(b + o_ol);
    mp.out = reinterpret_cast<__nv_bfloat16*>(b + o_out);
    mp.lse = reinterpret_cast<float*>(b + o_lse);
    mp.lse_ld = S;
    moba::WindowGeom& w = mp.w;
    w.S = S;
    w.Hq = w.Hkv = w.G = 1;
    w.B = 128;
    w.k_eff = K;
    w.nbp = 1;
    w.w0 = 0;
    w.wlen = S;
    w.wwords = WW;
    w.pair_tokens = 0;
    w.q0 = 0;
    w.list_cap = 1;
    moba::merge_kernel<0><<<S / 16, 256, 0, stream>>>(mp);
    if (cudaGetLastError() != cudaSuccess) rc = fail(MOBA_ERR_CUDA, "self-test launch failed");
  }
  const int st = moba_device_status(stream);
  cudaFree(b);
  if (rc) return rc;
  if (st) fail(st, "the merge kernel reported device status %d", st);
  return st;
}

extern "C" int moba_selftest_bounded_wait_async(int timeout_us, cudaStream_t stream) {
  g_err.clear();
  if (timeout_us < 1 || timeout_us > 2000000) return fail(MOBA_ERR_INVALID_ARG, "timeout_us must be in [1, 2e6]");
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  moba::selftest_wait_kernel<<<1, 32, 0, stream>>>((uint64_t)timeout_us * 2000ull);
  MOBA_CUDA(cudaGetLastError());
  return finish_call(MOBA_OK, stream);
}

// ------------------------------------------------------------ no allocation
// moba_fwd_noalloc: the forward pass for callers that may not allocate
// device memory once they are running -- for example a serving process that
// reserves its whole memory budget at start-up, or a plug-in that lives under
// an allocator it does not own. Its scratch is this fixed array, which every
// GPU that loads the library holds until the process exits.

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)64 << 20;  // 64 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (in host code the array's name is only a host-side stand-in).
int noalloc_scratch(void** out) {
  int dev = 0;
  MOBA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(MOBA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(MOBA_ERR_CUDA, "cudaGetSymbolAddress of the no-allocation scratch failed: %s",
                  cudaGetErrorString(e));
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MOBA_OK;
}

// The largest query window (a multiple of 128 tokens) whose scratch fits in
// `cap` bytes; fails when not even a 128-token window fits.
int plan_within(Plan* pl, int64_t S, int Hq, int Hkv, int B, int topk, size_t cap) {
  Plan& p = *pl;
  plan_shape(p, S, 0, Hq, Hkv, B, topk);
  int64_t W = (S + 127) / 128 * 128;
  while (true) {
    if (W * Hq * (int64_t)std::max(p.P, 1) < ((int64_t)1 << 31) - 1) {
      layout_for_window(p, W);
      if (p.total <= cap) return MOBA_OK;
    }
    if (W == 128) break;
    W = std::max<int64_t>(128, W / 2 / 128 * 128);
  }
  return fail(MOBA_ERR_UNSUPPORTED,
              "problem too large for moba_fwd_noalloc: its scratch needs more than the fixed %zu bytes "
              "(seqlen %lld, heads_q %d, heads_kv %d, block_size %d, topk %d); use moba_fwd",
              cap, (long long)S, Hq, Hkv, B, topk);
}

}  // namespace

extern "C" int moba_fwd_noalloc(const void* q, const void* k, const void* v, int64_t seqlen, int heads_q,
                                int heads_kv, int head_dim, int block_size, int topk, void* out, float* lse,
                                cudaStream_t stream) {
  g_err.clear();
  if (!q || !k || !v || !out || !lse) return fail(MOBA_ERR_INVALID_ARG, "null pointer argument");
  int rc = check_shape(seqlen, heads_q, heads_kv, head_dim, block_size, topk);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(MOBA_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  Plan p;
  rc = plan_within(&p, seqlen, heads_q, heads_kv, block_size, topk, kNoAllocScratchBytes);
  if (rc) return rc;
  DeviceInfo dev;
  rc = device_info(&dev);
  if (rc) return rc;
  void* scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  rc = take_pending_status(dev, stream);
  if (rc) return rc;
  return finish_call(run_forward(p, dev, q, k, v, out, lse, static_cast<uint8_t*>(scratch), stream), stream);
}
