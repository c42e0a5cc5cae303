/*
 * moba.h - C ABI of the B200 (sm_100a) MoBA causal prefill forward pass.
 *
 * MoBA (Mixture of Block Attention; "MoBA: Mixture of Block Attention for
 * Long-Context LLMs", abstract) cuts the context into blocks of block_size
 * tokens, lets a parameter-less top-k gate pick for every query token the
 * key/value blocks most relevant to it, and runs attention over the picked
 * blocks only ("MoBA (Mixture of Block Attention)" project summary, section
 * "How It Works"). Causality: a query never picks a future block, its own
 * block is always picked, and a causal mask applies inside the own block
 * ("MoBA - Moonshot AIが提案した新しいアテンションメカニズム", section
 * "MoBAの技術的原則").
 *
 * Conventions of this library (the pages leave them open):
 *   - gate score of block j for query row (t, h): q[t][h] . mean_{u in blk j}
 *     k[u][g(h)], unscaled; ties go to the lower block index;
 *   - the own block counts toward topk: a row attends min(topk, t/B + 1)
 *     blocks; topk >= number of blocks gives full causal attention;
 *   - GQA: q head h reads kv head h / (heads_q / heads_kv);
 *   - softmax scale 1/sqrt(head_dim); lse is the natural log of the sum of
 *     exp(scaled logits) over the attended keys.
 *
 * All tensors are batch 1, dense, row-major:
 *   q, out : [seqlen][heads_q][head_dim]   bf16
 *   k, v   : [seqlen][heads_kv][head_dim]  bf16
 *   lse    : [heads_q][seqlen]             fp32
 *   kmean  : [heads_kv][nblocks - 1][head_dim] fp32 (only blocks that can be
 *            a past block are pooled; nblocks = ceil(seqlen / block_size))
 *   sel    : [heads_q][seqlen][min(topk, nblocks)] int32, ascending block
 *            indices (the own block is last), padded with -1
 *
 * Ownership and ordering: the caller owns every buffer. Device pointers must
 * be 16-byte aligned. Outputs must not alias inputs. Calls are asynchronous
 * on `stream`; the library keeps no pointer after a call returns. Scratch
 * memory is taken from the stream-ordered allocator (cudaMallocAsync) and
 * returned (cudaFreeAsync) on the same stream inside each call.
 *
 * Errors: argument checks run before any launch and return a nonzero
 * moba_status; moba_last_error() then gives a message (thread-local). Device
 * side faults that the kernels detect are recorded in a per-device status
 * word that moba_device_status() reads after synchronising the stream: a
 * bounded wait that ran out (MOBA_ERR_DEVICE_TIMEOUT), or a router list slot
 * outside the scratch's list (MOBA_ERR_DEVICE_CHECK; the kernel skips that
 * access). The kernels also store the code in a host-mapped copy, so the next
 * call on the device (any entry point that launches) returns it before
 * launching anything, once, and clears it. With the environment variable
 * MOBA_SYNC=1, every call synchronises its stream and returns that status
 * itself. A failed scratch allocation returns MOBA_ERR_OOM; the environment
 * variable MOBA_TEST_SCRATCH_PAD=<bytes> (a test hook) adds that many bytes
 * to every scratch request so that this path can be exercised.
 *
 * Value range: routed and own-block partial outputs are kept in fp16 between
 * the attention and merge stages, so v must hold finite values of magnitude
 * below 65504 (each partial output is a convex combination of v rows).
 */
#ifndef MOBA_B200_H
#define MOBA_B200_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOBA_OK = 0,
    MOBA_ERR_INVALID_ARG = 1,    /* null pointer, bad shape, misaligned    */
    MOBA_ERR_UNSUPPORTED = 2,    /* device is not sm_100, or a shape limit */
    MOBA_ERR_OOM = 3,            /* scratch allocation failed              */
    MOBA_ERR_CUDA = 4,           /* a CUDA runtime call failed             */
    MOBA_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out        */
    MOBA_ERR_DEVICE_CHECK = 6    /* a kernel found a list slot out of range */
} moba_status;

/* Limits checked before launch. */
#define MOBA_HEAD_DIM 128      /* head_dim must equal this                  */
#define MOBA_MAX_TOPK 64       /* topk - 1 past blocks at most, unless topk >= nblocks */

/*
 * moba_fwd - the whole forward pass: key mean-pool, gate + top-k, router,
 * block attention and log-sum-exp merge, all on the GPU.
 *
 * q, k, v    device bf16 inputs (layouts above).
 * seqlen     number of tokens, >= 1.
 * heads_q    query heads, a positive multiple of heads_kv.
 * heads_kv   key/value heads, >= 1.
 * head_dim   must be 128.
 * block_size tokens per block: a positive multiple of 128. seqlen need not
 *            be a multiple of it (the last block is then partial).
 * topk       blocks per query including its own block, >= 1. Values above
 *            the number of blocks are clamped (full causal attention). When
 *            topk < nblocks, topk - 1 must not exceed MOBA_MAX_TOPK.
 * out        device bf16 output [seqlen][heads_q][head_dim].
 * lse        device fp32 output [heads_q][seqlen].
 * stream     CUDA stream for every launch and the scratch memory.
 *
 * Returns MOBA_OK once all work is queued. Scratch size grows with seqlen;
 * long sequences are processed in query windows whose size the library
 * picks (environment MOBA_WINDOW=<tokens> overrides it, rounded to 128).
 */
int moba_fwd(const void* q, const void* k, const void* v, int64_t seqlen,
             int heads_q, int heads_kv, int head_dim, int block_size, int topk,
             void* out, float* lse, cudaStream_t stream);

/*
 * moba_fwd_chunk - the forward pass for the queries of the last
 * seqlen - q_start tokens only, against keys and values of all seqlen
 * tokens: a chunk of prefill (or, with q_start = seqlen - 1, one decode step)
 * appended to a cache. By causality the result equals rows q_start..seqlen-1
 * of moba_fwd on the whole sequence (the queries of earlier tokens never
 * enter them); the pages' causal gate and own-block mask ("MoBA - Moonshot
 * AIが提案した新しいアテンションメカニズム", "MoBAの技術的原則") are applied
 * at the tokens' absolute positions. The pages describe no such entry point;
 * it serves the serving use they mention (Kimi's long-context requests).
 *
 * q          device bf16 [seqlen - q_start][heads_q][head_dim]: the queries
 *            of tokens q_start .. seqlen - 1.
 * k, v       device bf16 [seqlen][heads_kv][head_dim]: every token's keys and
 *            values (the cache followed by the chunk's own).
 * q_start    first token with a query, 0 <= q_start < seqlen (0 is moba_fwd).
 * out        device bf16 [seqlen - q_start][heads_q][head_dim].
 * lse        device fp32 [heads_q][seqlen - q_start].
 * Other arguments, ownership and errors as moba_fwd; a q_start outside
 * [0, seqlen) returns MOBA_ERR_INVALID_ARG. Each call pools the means of all
 * complete blocks again: the library keeps nothing between calls.
 */
int moba_fwd_chunk(const void* q, const void* k, const void* v, int64_t seqlen,
                   int64_t q_start, int heads_q, int heads_kv, int head_dim,
                   int block_size, int topk, void* out, float* lse,
                   cudaStream_t stream);

/*
 * moba_fwd_chunk_means - moba_fwd_chunk with the block means supplied by the
 * caller instead of pooled from k on every call: a decode loop computes them
 * once with moba_pool and pools again only when the cache completes a block.
 *
 * kmean      device fp32 [heads_kv][nblocks - 1][head_dim], exactly what
 *            moba_pool writes for these k and block_size (nblocks =
 *            ceil(seqlen / block_size)); means of blocks that cannot be past
 *            blocks of any token are not read. The caller keeps it matching k;
 *            a stale kmean silently changes the gate's choices. NULL returns
 *            MOBA_ERR_INVALID_ARG.
 * Other arguments, ownership and errors as moba_fwd_chunk.
 */
int moba_fwd_chunk_means(const void* q, const void* k, const void* v,
                         const float* kmean, int64_t seqlen, int64_t q_start,
                         int heads_q, int heads_kv, int head_dim,
                         int block_size, int topk, void* out, float* lse,
                         cudaStream_t stream);

/*
 * moba_fwd_varlen - moba_fwd over a packed batch of independent sequences
 * (serving several long-context requests in one call: "MoBA (Mixture of
 * Block Attention)" project summary, "Deployment"; "MoBA: Mixture of Block
 * Attention for Long-Context LLMs" abstract). Sequence b is tokens
 * cu_seqlens[b] .. cu_seqlens[b+1]-1 of the packed buffers. Each sequence is
 * its own causal problem: its blocks start at its first token, and no query
 * attends across a sequence boundary, so sequence b's rows equal moba_fwd
 * called on its tokens alone.
 *
 * q, k, v    device bf16 [T][heads][head_dim], T = cu_seqlens[batch].
 * cu_seqlens HOST int64 [batch + 1]: 0 = cu_seqlens[0] <= cu_seqlens[1] <=
 *            ...; a zero-length sequence is skipped. Read during the call
 *            only.
 * batch      number of sequences, >= 1.
 * out        device bf16 output [T][heads_q][head_dim].
 * lse        device fp32 output [heads_q][T] (column = packed token index),
 *            4-byte aligned.
 * Shape rules per sequence, stream, graph replay, ownership and errors as
 * moba_fwd; cu_seqlens that are not 0-based and non-decreasing, or hold no
 * token, return MOBA_ERR_INVALID_ARG before any launch.
 */
int moba_fwd_varlen(const void* q, const void* k, const void* v,
                    const int64_t* cu_seqlens, int batch, int heads_q,
                    int heads_kv, int head_dim, int block_size, int topk,
                    void* out, float* lse, cudaStream_t stream);

/*
 * moba_bwd - the gradient of moba_fwd: dq, dk, dv from the upstream gradient
 * dout, with the gate's choice held fixed (the top-k choice is piecewise
 * constant; the block means receive no gradient). Needed to train MoBA on
 * from a full-attention model ("MoBA (Mixture of Block Attention)" project
 * summary, "Key Features"; "Efficient Long-Context Attention with MoBA", "How
 * MoBA Works"). Per q head h of kv head g, with P the forward's attention
 * weights over the row's attended keys and c = 1/sqrt(head_dim):
 *   dv = sum over g's q heads of P^T dout, dS = P * (dout v^T - rowsum(dout * out)),
 *   dq = c dS k, dk = sum over g's q heads of c dS^T q.
 * The pool, gate and router run again, so the selection is the forward's.
 *
 * q, k, v    device bf16, as passed to moba_fwd.
 * out, lse   device, moba_fwd's outputs for them (bf16 [S][heads_q][128],
 *            fp32 [heads_q][S]); P is rebuilt from lse.
 * dout       device bf16 [S][heads_q][head_dim].
 * dq         device bf16 output [S][heads_q][head_dim].
 * dk, dv     device bf16 outputs [S][heads_kv][head_dim].
 * Shapes and checks as moba_fwd; every pointer 16-byte aligned. Scratch is
 * stream-ordered, as for moba_fwd (dK / dV accumulate in fp32 scratch).
 * The result is deterministic: every sum runs in a fixed order.
 */
int moba_bwd(const void* q, const void* k, const void* v, const void* out,
             const float* lse, const void* dout, int64_t seqlen, int heads_q,
             int heads_kv, int head_dim, int block_size, int topk, void* dq,
             void* dk, void* dv, cudaStream_t stream);

/*
 * moba_fwd_host - moba_fwd on HOST buffers (same layouts and results):
 * copies q, k, v to the device, runs the forward pass and copies out and lse
 * back, and synchronises `stream` before returning. The work is pipelined
 * by query window: the rows of q, k and v a window needs go up on a
 * library-internal copy stream ahead of that window's kernels (pool, gate,
 * router, attention and merge run window by window, on `stream`), and the
 * window's out rows and lse columns come back on a second internal stream
 * while the next window computes; both copy streams are forked from and
 * joined back to `stream`. Host buffers that are page-locked (cudaHostAlloc /
 * pinned) overlap; pageable ones are copied correctly but without overlap.
 * Device buffers come from the stream-ordered allocator and are released
 * before returning. out_host and lse_host must not alias the inputs.
 */
int moba_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                  int64_t seqlen, int heads_q, int heads_kv, int head_dim,
                  int block_size, int topk, void* out_host, float* lse_host,
                  cudaStream_t stream);

/*
 * moba_pool - the first stage alone: kmean[g][j][:] = mean of k[t][g][:]
 * over the tokens t of block j, for j < nblocks - 1 (fp32 accumulation, fixed
 * order). The blocks are the method's partition of the context into
 * block_size consecutive tokens ("MoBA (Mixture of Block Attention)" project
 * summary, "How It Works"); the mean is what the gate scores a query
 * against (the pages call the gate parameter-less without printing its
 * score; this library takes the inner product with the block's mean key).
 * kmean is a device fp32 buffer [heads_kv][nblocks-1][head_dim]. Does
 * nothing when nblocks == 1. Errors as moba_fwd.
 */
int moba_pool(const void* k, int64_t seqlen, int heads_kv, int head_dim,
              int block_size, float* kmean, cudaStream_t stream);

/*
 * moba_gate - the second stage alone: gate scores q . kmean over past blocks
 * and the per-row top-(k-1) with the own block forced, written as `sel`
 * (layout above): the parameter-less top-k gate of "MoBA (Mixture of Block
 * Attention)" project summary, "How It Works", with the causal rules of
 * "MoBA - Moonshot AIが提案した新しいアテンションメカニズム",
 * "MoBAの技術的原則" (no future block; the own block always chosen). Ties go
 * to the lower block index. kmean as produced by moba_pool (it may be NULL
 * when no row chooses: topk 1, or topk >= nblocks). sel is a device int32
 * buffer the caller owns. Errors as moba_fwd.
 */
int moba_gate(const void* q, const float* kmean, int64_t seqlen, int heads_q,
              int heads_kv, int head_dim, int block_size, int topk,
              int32_t* sel, cudaStream_t stream);

/*
 * Per-stage device timing of the forward passes issued from this host
 * thread. After moba_profile_begin(), every moba_fwd call also records CUDA
 * events on its stream between its stages (no extra synchronisation).
 * moba_profile_end() waits for the last recorded event, writes the summed
 * milliseconds per stage to stage_ms[0..7] = {pool, gate, route, attention,
 * merge, bwd_prep, bwd_dq, bwd_dkdv} (the last three for moba_bwd calls),
 * the number of kernels launched to *launches and the number of forward and
 * backward calls to *calls, then turns the timing off. Returns a
 * moba_status.
 */
int moba_profile_begin(void);
int moba_profile_end(float* stage_ms, int* launches, int* calls);

/*
 * moba_fwd_noalloc - moba_fwd for callers that may not allocate device
 * memory while they run (a serving process that reserves its memory budget
 * at start-up, a plug-in under an allocator it does not own). The pages have
 * no counterpart: this is a property of this library, not of the method.
 *
 * Same arguments, layouts and results as moba_fwd. Instead of the
 * stream-ordered allocator it uses one fixed 64 MiB device array that the
 * library defines; every GPU that loads the library holds that array until
 * the process exits. The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine. Problems whose scratch would not fit in the
 * array (the selection table and at least a 128-token query window) are
 * rejected with MOBA_ERR_UNSUPPORTED before any launch; moba_fwd handles
 * them. The first call on a device (of this or any other entry point) does
 * the library's one-time set-up for that device: it reads device attributes,
 * sets the kernels' shared-memory limits, pins one 4-byte host word
 * (cudaHostAlloc, mapped) that mirrors the device status, loads the module
 * (which maps the 64 MiB array) and looks up the array's device address
 * (cudaGetSymbolAddress) with that device current. A caller that must not
 * allocate at all at run time makes that first call during its own set-up,
 * and before any stream capture. This entry point never changes the
 * stream-ordered allocator's settings. Every call shares the one array:
 * calls that overlap on the GPU (different streams, or threads) race on it
 * and must be serialised by the caller. Nothing in the array needs to start
 * at zero; every call writes each part before reading it.
 */
int moba_fwd_noalloc(const void* q, const void* k, const void* v,
                     int64_t seqlen, int heads_q, int heads_kv, int head_dim,
                     int block_size, int topk, void* out, float* lse,
                     cudaStream_t stream);

/* Message of the last failed call on this host thread ("" if none). */
const char* moba_last_error(void);

/*
 * Synchronises `stream`, then returns and clears the status word that the
 * kernels on the current device write when a bounded wait runs out
 * (MOBA_ERR_DEVICE_TIMEOUT) or a list slot check fails (MOBA_ERR_DEVICE_CHECK);
 * MOBA_OK when neither happened. The word is shared by every call on the
 * device since the last read.
 */
int moba_device_status(cudaStream_t stream);

/*
 * Launches one tiny kernel whose single wait can never be satisfied, bounded
 * at `timeout_us` microseconds, and returns the status it leaves
 * (MOBA_ERR_DEVICE_TIMEOUT when the bound works). It exercises the same
 * bounded-wait helper the attention kernel uses, without faulting the GPU.
 */
int moba_selftest_bounded_wait(int timeout_us, cudaStream_t stream);

/*
 * Runs the merge kernel once on a tiny problem whose router tables point a
 * routed partial outside the list (the scratch of this call is its own
 * small cudaMalloc'd buffer), and returns the status it leaves:
 * MOBA_ERR_DEVICE_CHECK when the kernel's slot check caught it and skipped
 * the read. No access leaves the allocated buffers.
 */
int moba_selftest_device_check(cudaStream_t stream);

/*
 * The same kernel, launched without reading the status afterwards: the next
 * call on the device reports MOBA_ERR_DEVICE_TIMEOUT (or this call does, with
 * MOBA_SYNC=1). Exercises the error reporting of the other entry points.
 */
int moba_selftest_bounded_wait_async(int timeout_us, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_B200_H */
