/*
 * Seeded synthetic inputs for the MoBA causal prefill forward pass.
 *
 * This file draws random numbers and rounds them to bf16. It holds none of
 * the attention method's arithmetic: no pooling, no gate, no softmax. Both
 * the fp64 oracle and the CUDA path receive the bytes it writes.
 *
 * Generator (counter-based, so any slice can be regenerated on its own):
 *   - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the i-th output of a stream started at state
 *     s0 is mix64(s0 + (i + 1) * GAMMA).
 *   - Stream state: s0(seed, stream) = mix64(seed + GAMMA * (stream + 1)).
 *   - Element i of a stream uses outputs 2i and 2i+1: u1 = (a + 1) / 2^53 in
 *     (0, 1], u2 = b / 2^53 in [0, 1), with a, b the top 53 bits.
 *   - Normal deviate by Box and Muller (1958): sqrt(-2 ln u1) cos(2 pi u2).
 *   - bf16 rounding: round-to-nearest-even directly from the fp64 value.
 *
 * Workload recipe (keys): K[t][g][c] = bf16(N_K(t,g,c) + mu[g][t / B][c]) with
 * mu[g][j] = 0.5 * sqrt(d) * u / |u|, u ~ N(0, I_d) drawn from its own stream,
 * so that each block's keys share a random offset and gate scores separate.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_stream_state(uint64_t seed, uint64_t stream) {
    return mix64(seed + GAMMA * (stream + 1));
}

/* i-th raw SplitMix64 output of the stream started at s0. */
uint64_t synth_splitmix_output(uint64_t s0, uint64_t i) {
    return mix64(s0 + (i + 1) * GAMMA);
}

static inline double normal_at(uint64_t s0, uint64_t i) {
    const double two_m53 = 1.0 / 9007199254740992.0; /* 2^-53 */
    uint64_t a = synth_splitmix_output(s0, 2 * i) >> 11;
    uint64_t b = synth_splitmix_output(s0, 2 * i + 1) >> 11;
    double u1 = (double)(a + 1) * two_m53;
    double u2 = (double)b * two_m53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

double synth_normal(uint64_t seed, uint64_t stream, uint64_t i) {
    return normal_at(synth_stream_state(seed, stream), i);
}

/* Round an fp64 value to bf16 bits, nearest-even, in one step (no double
 * rounding through fp32). Values whose magnitude is below the smallest
 * normal bf16 flush to signed zero; values past the largest finite bf16
 * become infinity. Neither occurs for the workloads drawn here. */
uint16_t synth_f64_to_bf16(double x) {
    uint64_t u;
    memcpy(&u, &x, 8);
    uint64_t sign = u >> 63;
    int64_t e = (int64_t)((u >> 52) & 0x7FF);
    uint64_t m = u & 0xFFFFFFFFFFFFFULL;
    if (e == 0x7FF) return (uint16_t)((sign << 15) | 0x7F80 | (m ? 0x40 : 0));
    if (e == 0) return (uint16_t)(sign << 15);
    /* keep 7 mantissa bits: drop 45 */
    uint64_t keep = m >> 45;
    uint64_t rem = m & ((1ULL << 45) - 1);
    uint64_t half = 1ULL << 44;
    int64_t eb = e - 1023 + 127;
    if (rem > half || (rem == half && (keep & 1))) {
        keep += 1;
        if (keep == 0x80) { keep = 0; eb += 1; }
    }
    if (eb <= 0) return (uint16_t)(sign << 15);
    if (eb >= 0xFF) return (uint16_t)((sign << 15) | 0x7F80);
    return (uint16_t)((sign << 15) | ((uint64_t)eb << 7) | keep);
}

/* ---- threaded fills ---------------------------------------------------- */

typedef struct {
    uint16_t* out;
    int64_t begin, end;
    uint64_t s0;
    int64_t offset;
    /* key-offset mode */
    const double* mu; /* [Hkv][nb][d] or NULL */
    int64_t Hkv, d, B, nb;
} fill_job;

static void* fill_worker(void* arg) {
    fill_job* j = (fill_job*)arg;
    for (int64_t i = j->begin; i < j->end; ++i) {
        double x = normal_at(j->s0, (uint64_t)(j->offset + i));
        if (j->mu) {
            int64_t gi = j->offset + i;
            int64_t c = gi % j->d;
            int64_t g = (gi / j->d) % j->Hkv;
            int64_t t = gi / (j->d * j->Hkv);
            x += j->mu[(g * j->nb + t / j->B) * j->d + c];
        }
        j->out[i] = synth_f64_to_bf16(x);
    }
    return NULL;
}

static void run_fill(uint16_t* out, int64_t n, uint64_t s0, int64_t offset,
                     const double* mu, int64_t Hkv, int64_t d, int64_t B,
                     int64_t nb, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if (n < 65536) nthreads = 1;
    fill_job jobs[1024];
    pthread_t th[1024];
    int64_t per = (n + nthreads - 1) / nthreads;
    int started = 0;
    for (int k = 0; k < nthreads; ++k) {
        int64_t b = (int64_t)k * per, e = b + per;
        if (b >= n) break;
        if (e > n) e = n;
        fill_job jb = {out + b, 0, e - b, s0, offset + b, mu, Hkv, d, B, nb};
        jobs[k] = jb;
        if (nthreads == 1) { fill_worker(&jobs[k]); continue; }
        pthread_create(&th[k], NULL, fill_worker, &jobs[k]);
        started = k + 1;
    }
    for (int k = 0; k < started; ++k) pthread_join(th[k], NULL);
}

/* out[i] = bf16(N(seed, stream, offset + i)) for i in [0, n). */
void synth_fill_normal_bf16(uint16_t* out, int64_t n, uint64_t seed,
                            uint64_t stream, int64_t offset, int nthreads) {
    run_fill(out, n, synth_stream_state(seed, stream), offset, NULL, 0, 1, 1, 1,
             nthreads);
}

/* Per-(kv head, block) key offsets mu[g][j][c] (fp64), norm 0.5*sqrt(d). */
void synth_key_offsets(double* mu, int64_t Hkv, int64_t nb, int64_t d,
                       uint64_t seed, uint64_t stream) {
    uint64_t s0 = synth_stream_state(seed, stream);
    for (int64_t r = 0; r < Hkv * nb; ++r) {
        double n2 = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            double u = normal_at(s0, (uint64_t)(r * d + c));
            mu[r * d + c] = u;
            n2 += u * u;
        }
        double s = 0.5 * sqrt((double)d) / sqrt(n2);
        for (int64_t c = 0; c < d; ++c) mu[r * d + c] *= s;
    }
}

/* Keys [rows t0 .. t0+nrows) of a [S][Hkv][d] tensor: normal draws plus the
 * block offsets mu (from synth_key_offsets). Flat index of (t, g, c) is
 * (t * Hkv + g) * d + c in the key stream. */
void synth_fill_keys_bf16(uint16_t* out, int64_t t0, int64_t nrows,
                          int64_t Hkv, int64_t d, int64_t B, int64_t nb,
                          const double* mu, uint64_t seed, uint64_t stream,
                          int nthreads) {
    run_fill(out, nrows * Hkv * d, synth_stream_state(seed, stream),
             t0 * Hkv * d, mu, Hkv, d, B, nb, nthreads);
}
