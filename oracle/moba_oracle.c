/*
 * fp64 CPU oracle for the MoBA (Mixture of Block Attention) causal prefill
 * forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path calls, links or
 * loads this file: only the tests, the smoke check and the benchmark's CPU
 * baseline do. It shares no code with the CUDA library.
 *
 * What the method computes, and where the pages say so:
 *   - The context is cut into blocks of B consecutive tokens ("MoBA (Mixture
 *     of Block Attention)" project summary, section "How It Works"; "MoBA -
 *     Moonshot AIが提案した新しいアテンションメカニズム", section
 *     "MoBAの主な機能", block sparse attention).
 *   - A parameter-less top-k gate picks, for every query token, the KV blocks
 *     most relevant to it (same sections; "MoBA: Mixture of Block Attention
 *     for Long-Context LLMs", abstract). The pages do not print the score:
 *     this oracle takes q . mean(K_block), the inner product of the query
 *     with the mean of the block's keys.
 *   - Causality: a query never attends a future block, and a causal mask
 *     applies inside its own block ("MoBA - Moonshot AIが提案した新しい
 *     アテンションメカニズム", section "MoBAの技術的原則", causal design).
 *     The own block is always chosen and counts toward k.
 *   - Ties in the gate go to the lower block index.
 *   - Attention then runs over the selected blocks only. The mask-based
 *     ("naive") form ("MoBA (Mixture of Block Attention)" project summary,
 *     section "Limitations & Caveats") is what is written out here: a dense
 *     0/1 mask row over all keys, then softmax of the masked, scaled logits,
 *     scale 1/sqrt(d), and the natural-log log-sum-exp of those logits.
 *
 * Speed without changing a result: every row is computed on its own, its
 * sums in the order written; four independent inner products may be formed
 * side by side (separate accumulators), bf16 rows are widened to fp64 into a
 * small buffer before use, and threads take interleaved rows. None of this
 * changes any rounding (the results are bit-identical to one key at a time).
 *
 * Parity unpinned: the choice of q . mean(K_block) as the gate score, the
 * softmax scale 1/sqrt(d) and the LSE convention are not stated on the pages;
 * the tests pin the arithmetic of each step, not these choices.
 *
 * Layouts (batch 1, bf16 stored as uint16 bit patterns):
 *   q [S][Hq][d], k and v [S][Hkv][d]; q head h reads kv head h / (Hq/Hkv).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_f64(uint16_t x) {
    uint32_t u = (uint32_t)x << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static int64_t nblocks_of(int64_t S, int B) { return (S + B - 1) / B; }

/* One bf16 row of d values widened (exactly) to fp64. */
static void row_to_f64(const uint16_t* x, int d, double* out) {
    for (int c = 0; c < d; ++c) out[c] = bf16_to_f64(x[c]);
}

/* Step 1: block partition and key mean-pool.
 * m[g][j][c] = (1/|blk j|) * sum over t in block j of K[t][g][c], summed in
 * ascending t. The last block may be partial: the mean is over the keys it
 * holds. */
void oracle_kmean(const uint16_t* k, int64_t S, int Hkv, int d, int B,
                  double* m) {
    int64_t nb = nblocks_of(S, B);
    for (int g = 0; g < Hkv; ++g) {
        for (int64_t j = 0; j < nb; ++j) {
            int64_t t0 = j * B, t1 = t0 + B < S ? t0 + B : S;
            double* mj = m + ((int64_t)g * nb + j) * d;
            for (int c = 0; c < d; ++c) mj[c] = 0.0;
            for (int64_t t = t0; t < t1; ++t)
                for (int c = 0; c < d; ++c)
                    mj[c] += bf16_to_f64(k[(t * Hkv + g) * d + c]);
            for (int c = 0; c < d; ++c) mj[c] /= (double)(t1 - t0);
        }
    }
}

/* Step 2: gate scores of query row (t, h) against every past block.
 * s[j] = sum_c Q[t][h][c] * m[g(h)][j][c] for j < t / B (unscaled), each
 * sum taken over c in ascending order. Four blocks' sums are formed side by
 * side (four separate accumulators, the same order of additions in each), so
 * the results are those of one block at a time. */
void oracle_gate_scores(const uint16_t* q, const double* m, int64_t S, int Hq,
                        int Hkv, int d, int B, int64_t t, int h, double* s) {
    int64_t nb = nblocks_of(S, B);
    int g = h / (Hq / Hkv);
    int64_t b = t / B;
    const uint16_t* qr = q + (t * Hq + h) * d;
    const double* mg = m + (int64_t)g * nb * d;
    int64_t j = 0;
    for (; j + 4 <= b; j += 4) {
        const double *m0 = mg + j * d, *m1 = m0 + d, *m2 = m1 + d, *m3 = m2 + d;
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int c = 0; c < d; ++c) {
            double qc = bf16_to_f64(qr[c]);
            a0 += qc * m0[c];
            a1 += qc * m1[c];
            a2 += qc * m2[c];
            a3 += qc * m3[c];
        }
        s[j] = a0;
        s[j + 1] = a1;
        s[j + 2] = a2;
        s[j + 3] = a3;
    }
    for (; j < b; ++j) {
        const double* mj = mg + j * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += bf16_to_f64(qr[c]) * mj[c];
        s[j] = acc;
    }
}

typedef struct {
    double s;
    int64_t j;
} scored;

/* higher score first; equal scores: lower block index first */
static int by_score_then_index(const void* a, const void* b) {
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* Step 3: top-k selection for one row.
 * Sel = {b(t)} U (the first min(k-1, b(t)) past blocks ordered by score
 * descending, ties to the lower index). Written ascending into sel[0..k_eff),
 * padded with -1, k_eff = min(topk, nb).
 * info[0] = relative gap between the last selected and the first unselected
 *           past score, (s_a - s_b) / max_j |s_j|, relative to the largest
 *           score magnitude of the row's past blocks (a two-score
 *           denominator max(|s_a|, |s_b|) vanishes as both approach zero,
 *           where the gap says nothing about how well the ranking is
 *           determined); +inf when nothing was left out or nothing was
 *           chosen by score;
 * info[1] = s_a (the cut), info[2] = s_b, info[3] = max_j |s_j|. */
static void select_row(const uint16_t* q, const double* m, int64_t S, int Hq,
                       int Hkv, int d, int B, int topk, int64_t t, int h,
                       int32_t* sel, double* info, scored* work,
                       double* sbuf) {
    int64_t nb = nblocks_of(S, B);
    int64_t k_eff = topk < nb ? topk : nb;
    int64_t b = t / B;
    int64_t npast = (k_eff - 1) < b ? (k_eff - 1) : b;
    oracle_gate_scores(q, m, S, Hq, Hkv, d, B, t, h, sbuf);
    for (int64_t j = 0; j < b; ++j) {
        work[j].s = sbuf[j];
        work[j].j = j;
    }
    qsort(work, (size_t)b, sizeof(scored), by_score_then_index);
    for (int64_t i = 0; i < k_eff; ++i) sel[i] = -1;
    for (int64_t i = 0; i < npast; ++i) sel[i] = (int32_t)work[i].j;
    qsort(sel, (size_t)npast, sizeof(int32_t), cmp_i32);
    sel[npast] = (int32_t)b;
    double scale = 0.0;
    for (int64_t j = 0; j < b; ++j) scale = fmax(scale, fabs(sbuf[j]));
    info[0] = INFINITY;
    info[1] = NAN;
    info[2] = NAN;
    info[3] = scale;
    if (npast >= 1 && npast < b) {
        double sa = work[npast - 1].s, sb = work[npast].s;
        info[0] = scale > 0 ? (sa - sb) / scale : 0.0;
        info[1] = sa;
        info[2] = sb;
    }
}

/* Step 4: attention of row (t, h) under the block mask of Sel.
 * Mask row M[u] = [block(u) in Sel and u <= t] over all keys u in [0, S).
 * z_u = Q[t][h] . K[u][g] / sqrt(d) where M[u] = 1;
 * O = sum_u softmax(z)_u V[u][g];  LSE = ln sum_u exp(z_u). */
static void attend_row(const uint16_t* q, const uint16_t* k,
                       const uint16_t* v, int64_t S, int Hq, int Hkv, int d,
                       int B, int64_t t, int h, const int32_t* sel,
                       int64_t k_eff, double* out, double* lse,
                       unsigned char* blk_in, double* z, int64_t* zu,
                       double* qd, double* kd) {
    int64_t nb = nblocks_of(S, B);
    int g = h / (Hq / Hkv);
    const double scale = 1.0 / sqrt((double)d);
    memset(blk_in, 0, (size_t)nb);
    for (int64_t i = 0; i < k_eff; ++i)
        if (sel[i] >= 0) blk_in[sel[i]] = 1;
    for (int c = 0; c < d; ++c) qd[c] = bf16_to_f64(q[(t * Hq + h) * d + c]);
    /* the mask row: the keys u in [0, S) with M[u] = 1, ascending (bu and
     * ru walk u / B and u % B) */
    int64_t n = 0;
    for (int64_t u = 0, bu = 0, ru = 0; u < S; ++u) {
        int on = blk_in[bu] && (u <= t);
        if (on) zu[n++] = u;
        if (++ru == B) {
            ru = 0;
            ++bu;
        }
    }
    /* logits of those keys, each inner product summed over c in ascending
     * order; four keys side by side (four separate accumulators, the same
     * order of additions in each) */
    int64_t i = 0;
    for (; i + 4 <= n; i += 4) {
        double* k0 = kd;
        double *k1 = k0 + d, *k2 = k1 + d, *k3 = k2 + d;
        row_to_f64(k + (zu[i] * Hkv + g) * d, d, k0);
        row_to_f64(k + (zu[i + 1] * Hkv + g) * d, d, k1);
        row_to_f64(k + (zu[i + 2] * Hkv + g) * d, d, k2);
        row_to_f64(k + (zu[i + 3] * Hkv + g) * d, d, k3);
        double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
        for (int c = 0; c < d; ++c) {
            a0 += qd[c] * k0[c];
            a1 += qd[c] * k1[c];
            a2 += qd[c] * k2[c];
            a3 += qd[c] * k3[c];
        }
        z[i] = a0 * scale;
        z[i + 1] = a1 * scale;
        z[i + 2] = a2 * scale;
        z[i + 3] = a3 * scale;
    }
    for (; i < n; ++i) {
        row_to_f64(k + (zu[i] * Hkv + g) * d, d, kd);
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qd[c] * kd[c];
        z[i] = acc * scale;
    }
    double mx = -INFINITY;
    for (i = 0; i < n; ++i)
        if (z[i] > mx) mx = z[i];
    double l = 0.0;
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (i = 0; i < n; ++i) {
        double p = exp(z[i] - mx);
        l += p;
        row_to_f64(v + (zu[i] * Hkv + g) * d, d, kd);
        for (int c = 0; c < d; ++c) out[c] += p * kd[c];
    }
    for (int c = 0; c < d; ++c) out[c] /= l;
    *lse = mx + log(l);
}

/* ---- row-parallel drivers ---------------------------------------------- */

typedef struct {
    const uint16_t *q, *k, *v;
    const double* m;
    int64_t S;
    int Hq, Hkv, d, B, topk;
    const int64_t* rows_t;
    const int32_t* rows_h;
    int64_t r0, r1, rstep; /* rows r0, r0 + rstep, ... below r1 */
    const int32_t* sel_in; /* [nrows][k_eff] or NULL */
    int32_t* sel_out;      /* [nrows][k_eff] or NULL */
    double* info_out;      /* [nrows][4] or NULL */
    double* out;           /* [nrows][d] or NULL */
    double* lse;           /* [nrows] or NULL */
} row_job;

static void* row_worker(void* arg) {
    row_job* J = (row_job*)arg;
    int64_t nb = nblocks_of(J->S, J->B);
    int64_t k_eff = J->topk < nb ? J->topk : nb;
    int64_t kmax = k_eff * (int64_t)J->B;
    scored* work = (scored*)malloc(sizeof(scored) * (size_t)(nb + 1));
    double* sbuf = (double*)malloc(sizeof(double) * (size_t)(nb + 1));
    unsigned char* blk_in = (unsigned char*)malloc((size_t)nb + 1);
    double* z = (double*)malloc(sizeof(double) * (size_t)kmax);
    int64_t* zu = (int64_t*)malloc(sizeof(int64_t) * (size_t)kmax);
    double* qd = (double*)malloc(sizeof(double) * (size_t)J->d);
    double* kd = (double*)malloc(sizeof(double) * 4 * (size_t)J->d);
    int32_t* selr = (int32_t*)malloc(sizeof(int32_t) * (size_t)k_eff);
    double info[4];
    for (int64_t r = J->r0; r < J->r1; r += J->rstep) {
        int64_t t = J->rows_t[r];
        int h = J->rows_h[r];
        const int32_t* sel;
        if (J->sel_in) {
            sel = J->sel_in + r * k_eff;
        } else {
            select_row(J->q, J->m, J->S, J->Hq, J->Hkv, J->d, J->B, J->topk,
                       t, h, selr, info, work, sbuf);
            sel = selr;
            if (J->sel_out) memcpy(J->sel_out + r * k_eff, selr, sizeof(int32_t) * (size_t)k_eff);
            if (J->info_out) memcpy(J->info_out + r * 4, info, sizeof(info));
        }
        if (J->out)
            attend_row(J->q, J->k, J->v, J->S, J->Hq, J->Hkv, J->d, J->B, t,
                       h, sel, k_eff, J->out + r * J->d, J->lse + r, blk_in,
                       z, zu, qd, kd);
    }
    free(work); free(sbuf); free(blk_in); free(z); free(zu); free(qd); free(kd); free(selr);
    return NULL;
}

/* Thread i takes rows i, i + nthreads, i + 2 nthreads, ...: rows next to
 * each other in the caller's order run at the same time, so when they read
 * the same keys those stay in the shared cache. Every row is computed on its
 * own; the order only affects speed. */
static void run_rows(row_job base, int64_t nrows, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    if (nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
    row_job jobs[1024];
    pthread_t th[1024];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].r0 = i;
        jobs[i].r1 = nrows;
        jobs[i].rstep = nthreads;
        if (jobs[i].r0 >= jobs[i].r1) break;
        if (nthreads == 1) { row_worker(&jobs[i]); continue; }
        pthread_create(&th[i], NULL, row_worker, &jobs[i]);
        started = i + 1;
    }
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
}

/* Selection only, for rows (rows_t[r], rows_h[r]); m from oracle_kmean. */
void oracle_select(const uint16_t* q, const double* m, int64_t S, int Hq,
                   int Hkv, int d, int B, int topk, const int64_t* rows_t,
                   const int32_t* rows_h, int64_t nrows, int32_t* sel,
                   double* info, int nthreads) {
    row_job J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.m = m; J.S = S; J.Hq = Hq; J.Hkv = Hkv; J.d = d; J.B = B;
    J.topk = topk; J.rows_t = rows_t; J.rows_h = rows_h;
    J.sel_out = sel; J.info_out = info;
    run_rows(J, nrows, nthreads);
}

/* Full forward for rows: gate (unless sel_in is given) then masked softmax.
 * m may be NULL when sel_in is given. out [nrows][d], lse [nrows]. */
void oracle_attend(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const double* m, int64_t S, int Hq, int Hkv, int d, int B,
                   int topk, const int64_t* rows_t, const int32_t* rows_h,
                   int64_t nrows, const int32_t* sel_in, int32_t* sel_out,
                   double* out, double* lse, int nthreads) {
    row_job J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.m = m; J.S = S; J.Hq = Hq; J.Hkv = Hkv;
    J.d = d; J.B = B; J.topk = topk; J.rows_t = rows_t; J.rows_h = rows_h;
    J.sel_in = sel_in; J.sel_out = sel_out; J.out = out; J.lse = lse;
    run_rows(J, nrows, nthreads);
}
