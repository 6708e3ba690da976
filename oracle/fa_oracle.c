/*
 * fa_oracle.c -- plain fp64 CPU statement of exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA library is compared
 * against.  Only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg load it; the library itself never links, loads or calls it, and it
 * shares no code, header or table with the CUDA path.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "AI infra. 一层全看懂(五)Flash Attention:AI编译优化的集大成者"
 *        (AI infra explained, part 5: Flash Attention), sections 三 (the three
 *        passes of standard attention), 四 (safe softmax).
 *   [P2] "FlashAttention：为什么少搬数据，反而算得更快"
 *        (FlashAttention: why moving less data computes faster), sections
 *        02 (the S = QK^T, P = softmax(S), O = PV table; scale and causal mask are
 *        present in real computation), 04 (the online-softmax worked example and
 *        the m / l / U recurrence), 05 (training backward by recomputation).
 *   [P3] "FlashAttention技术原理详解：通过内存优化加速注意力计算"
 *        (FlashAttention explained) -- MHA / MQA / GQA support.
 *
 * What is computed, for every batch b, query head h and query row i, with the
 * key/value head kv = floor(h / G), G = Hq / Hkv (contiguous grouping of query
 * heads onto kv heads; the pages only say GQA is supported, [P3]):
 *
 *   s_j   = scale * sum_k q_ik k_jk                ([P2] §02, row of S = QK^T)
 *   s_j   = -inf  if causal and j > i + (Nk - Nq)  (bottom-right causal mask)
 *   m     = max_j s_j                              ([P1] §四 safe softmax)
 *   l     = sum_j exp(s_j - m)
 *   P_j   = exp(s_j - m) / l                       ([P2] §02, row of P)
 *   O_i   = sum_j P_j v_j                          ([P2] §02, O = PV)
 *   LSE_i = m + ln l                               (the per-row statistic kept
 *                                                   for the backward, [P2] §05)
 *   A row whose keys are all masked has O_i = 0 and LSE_i = -inf ([P2] §04 says
 *   fully masked rows must be handled; this is the reading taken).
 *
 * Backward of the scalar L = sum(dO * O) (standard softmax Jacobian; the pages
 * say only that P is recomputed from the saved statistics, [P2] §05):
 *   dP_j = dO_i . v_j ;  D_i = sum_j P_j dP_j ;  dS_j = P_j (dP_j - D_i)
 *   dQ_i = scale sum_j dS_j k_j ;  dK_j += scale dS_j q_i ;  dV_j += P_j dO_i
 * with dK/dV summed over all rows of all query heads of the kv group.
 *
 * The whole S and P row is materialised for each query row; there is no tiling
 * and no online softmax on this path.  The online recurrence of [P2] §04 is
 * provided separately (oracle_online_row_*) only to check the oracle against the
 * worked example and the "blocked equals full" invariant.
 *
 * All arithmetic is IEEE double, compiled without fast-math.  Inputs are read
 * either as bf16 bit patterns (exactly representable in double) or as doubles.
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_BF16 0
#define ORACLE_F64 1

/* ---------------------------------------------------------------------------
 * element access
 * ------------------------------------------------------------------------- */
static inline double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static inline double ld(const void* p, int dtype, int64_t idx)
{
    if (dtype == ORACLE_BF16)
        return bf16_bits_to_double(((const uint16_t*)p)[idx]);
    return ((const double*)p)[idx];
}

/* copy one d-vector into doubles */
static void load_vec(const void* p, int dtype, int64_t off, int64_t n, double* out)
{
    for (int64_t t = 0; t < n; ++t)
        out[t] = ld(p, dtype, off + t);
}

typedef struct {
    const void *q, *k, *v, *dout;
    int dtype;
    int64_t B, Hq, Hkv, Nq, Nk, d;
    double scale;
    int causal;
} problem_t;

static int64_t q_off(const problem_t* pb, int64_t b, int64_t h, int64_t i)
{
    return ((b * pb->Hq + h) * pb->Nq + i) * pb->d;
}

static int64_t kv_off(const problem_t* pb, int64_t b, int64_t g, int64_t j)
{
    return ((b * pb->Hkv + g) * pb->Nk + j) * pb->d;
}

/* Key j is visible to query i under the bottom-right causal mask. */
static int visible(const problem_t* pb, int64_t i, int64_t j)
{
    if (!pb->causal)
        return 1;
    return j <= i + (pb->Nk - pb->Nq);
}

/* ---------------------------------------------------------------------------
 * one query row, forward.  s and p are caller scratch of length Nk.
 * Returns the number of visible keys.
 * ------------------------------------------------------------------------- */
static int64_t row_forward(const problem_t* pb, int64_t b, int64_t h, int64_t i,
                           const double* qi, double* s, double* p,
                           double* o_row, double* lse_out, double* kvec)
{
    const int64_t d = pb->d, Nk = pb->Nk;
    const int64_t g = h / (pb->Hq / pb->Hkv);
    int64_t nvis = 0;

    /* row of S = scale * q_i K^T, masked */
    for (int64_t j = 0; j < Nk; ++j) {
        if (!visible(pb, i, j)) {
            s[j] = -INFINITY;
            continue;
        }
        load_vec(pb->k, pb->dtype, kv_off(pb, b, g, j), d, kvec);
        double acc = 0.0;
        for (int64_t t = 0; t < d; ++t)
            acc += qi[t] * kvec[t];
        s[j] = pb->scale * acc;
        ++nvis;
    }

    for (int64_t t = 0; t < d; ++t)
        o_row[t] = 0.0;
    if (nvis == 0) {
        for (int64_t j = 0; j < Nk; ++j)
            p[j] = 0.0;
        *lse_out = -INFINITY;
        return 0;
    }

    /* safe softmax over the whole row */
    double m = -INFINITY;
    for (int64_t j = 0; j < Nk; ++j)
        if (s[j] > m)
            m = s[j];
    double l = 0.0;
    for (int64_t j = 0; j < Nk; ++j)
        l += exp(s[j] - m);
    for (int64_t j = 0; j < Nk; ++j)
        p[j] = exp(s[j] - m) / l;

    /* O_i = P row times V */
    for (int64_t j = 0; j < Nk; ++j) {
        if (p[j] == 0.0)
            continue;
        load_vec(pb->v, pb->dtype, kv_off(pb, b, g, j), d, kvec);
        for (int64_t t = 0; t < d; ++t)
            o_row[t] += p[j] * kvec[t];
    }
    *lse_out = m + log(l);
    return nvis;
}

/* ---------------------------------------------------------------------------
 * thread pool helper: static partition of [0, n) over nthreads
 * ------------------------------------------------------------------------- */
typedef void (*range_fn)(void* ctx, int64_t begin, int64_t end, int tid);

typedef struct {
    range_fn fn;
    void* ctx;
    int64_t begin, end;
    int tid;
} range_job_t;

static void* range_trampoline(void* arg)
{
    range_job_t* j = (range_job_t*)arg;
    j->fn(j->ctx, j->begin, j->end, j->tid);
    return NULL;
}

static int resolve_threads(int nthreads)
{
    if (nthreads > 0)
        return nthreads;
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void parallel_for(int64_t n, int nthreads, range_fn fn, void* ctx)
{
    nthreads = resolve_threads(nthreads);
    if (nthreads > n)
        nthreads = (int)(n > 0 ? n : 1);
    if (nthreads <= 1) {
        fn(ctx, 0, n, 0);
        return;
    }
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    range_job_t* jobs = (range_job_t*)malloc(sizeof(range_job_t) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].fn = fn;
        jobs[t].ctx = ctx;
        jobs[t].begin = n * t / nthreads;
        jobs[t].end = n * (t + 1) / nthreads;
        jobs[t].tid = t;
        pthread_create(&th[t], NULL, range_trampoline, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
}

/* ---------------------------------------------------------------------------
 * forward over a list of flattened rows  r = (b * Hq + h) * Nq + i
 * ------------------------------------------------------------------------- */
typedef struct {
    const problem_t* pb;
    const int64_t* rows; /* NULL = all rows in order */
    double* o;           /* [nrows, d] */
    double* lse;         /* [nrows] */
} fwd_ctx_t;

static void fwd_range(void* vctx, int64_t begin, int64_t end, int tid)
{
    (void)tid;
    fwd_ctx_t* c = (fwd_ctx_t*)vctx;
    const problem_t* pb = c->pb;
    double* s = (double*)malloc(sizeof(double) * pb->Nk);
    double* p = (double*)malloc(sizeof(double) * pb->Nk);
    double* qi = (double*)malloc(sizeof(double) * pb->d);
    double* kvec = (double*)malloc(sizeof(double) * pb->d);
    for (int64_t r = begin; r < end; ++r) {
        int64_t flat = c->rows ? c->rows[r] : r;
        int64_t i = flat % pb->Nq;
        int64_t h = (flat / pb->Nq) % pb->Hq;
        int64_t b = flat / (pb->Nq * pb->Hq);
        load_vec(pb->q, pb->dtype, q_off(pb, b, h, i), pb->d, qi);
        row_forward(pb, b, h, i, qi, s, p, c->o + r * pb->d, c->lse + r, kvec);
    }
    free(s);
    free(p);
    free(qi);
    free(kvec);
}

static int check_dims(int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d)
{
    if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || d < 1)
        return 1;
    if (Hq % Hkv != 0)
        return 1;
    return 0;
}

/* Forward for all rows (rows == NULL, nrows ignored) or for the listed flattened
 * rows.  o: [nrows, d] doubles, lse: [nrows] doubles.  Returns 0 on success. */
int oracle_fwd(const void* q, const void* k, const void* v, int dtype,
               int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
               double scale, int causal, const int64_t* rows, int64_t nrows,
               double* o, double* lse, int nthreads)
{
    if (check_dims(B, Hq, Hkv, Nq, Nk, d))
        return 1;
    problem_t pb = {q, k, v, NULL, dtype, B, Hq, Hkv, Nq, Nk, d, scale, causal};
    fwd_ctx_t c = {&pb, rows, o, lse};
    int64_t n = rows ? nrows : B * Hq * Nq;
    parallel_for(n, nthreads, fwd_range, &c);
    return 0;
}

/* ---------------------------------------------------------------------------
 * backward.  Work unit = (b, kv head g, chunk of the group's rows).  Each unit
 * writes dQ rows directly (rows are disjoint) and accumulates dK/dV of its kv
 * head into a private buffer; buffers are summed in chunk order afterwards, so
 * the result does not depend on the thread count.
 * ------------------------------------------------------------------------- */
typedef struct {
    const problem_t* pb;
    int64_t chunks;        /* row chunks per (b, g) */
    double* dq;            /* [B, Hq, Nq, d] */
    double* dk_part;       /* [B*Hkv*chunks, Nk, d] */
    double* dv_part;
} bwd_ctx_t;

static void bwd_range(void* vctx, int64_t begin, int64_t end, int tid)
{
    (void)tid;
    bwd_ctx_t* c = (bwd_ctx_t*)vctx;
    const problem_t* pb = c->pb;
    const int64_t d = pb->d, Nk = pb->Nk, Nq = pb->Nq;
    const int64_t G = pb->Hq / pb->Hkv;
    const int64_t rows_per_group = G * Nq;
    double* s = (double*)malloc(sizeof(double) * Nk);
    double* p = (double*)malloc(sizeof(double) * Nk);
    double* dp = (double*)malloc(sizeof(double) * Nk);
    double* qi = (double*)malloc(sizeof(double) * d);
    double* doi = (double*)malloc(sizeof(double) * d);
    double* oi = (double*)malloc(sizeof(double) * d);
    double* kvec = (double*)malloc(sizeof(double) * d);

    for (int64_t u = begin; u < end; ++u) {
        int64_t chunk = u % c->chunks;
        int64_t bg = u / c->chunks;
        int64_t g = bg % pb->Hkv;
        int64_t b = bg / pb->Hkv;
        double* dk = c->dk_part + u * Nk * d;
        double* dv = c->dv_part + u * Nk * d;
        memset(dk, 0, sizeof(double) * Nk * d);
        memset(dv, 0, sizeof(double) * Nk * d);
        int64_t r0 = rows_per_group * chunk / c->chunks;
        int64_t r1 = rows_per_group * (chunk + 1) / c->chunks;
        for (int64_t r = r0; r < r1; ++r) {
            int64_t h = g * G + r / Nq;
            int64_t i = r % Nq;
            double* dqi = c->dq + q_off(pb, b, h, i);
            load_vec(pb->q, pb->dtype, q_off(pb, b, h, i), d, qi);
            load_vec(pb->dout, pb->dtype, q_off(pb, b, h, i), d, doi);
            double lse;
            int64_t nvis = row_forward(pb, b, h, i, qi, s, p, oi, &lse, kvec);
            for (int64_t t = 0; t < d; ++t)
                dqi[t] = 0.0;
            if (nvis == 0)
                continue;
            /* dP row = dO_i V^T and D_i = sum_j P_ij dP_ij */
            double D = 0.0;
            for (int64_t j = 0; j < Nk; ++j) {
                dp[j] = 0.0;
                if (p[j] == 0.0 && s[j] == -INFINITY)
                    continue;
                load_vec(pb->v, pb->dtype, kv_off(pb, b, g, j), d, kvec);
                double acc = 0.0;
                for (int64_t t = 0; t < d; ++t)
                    acc += doi[t] * kvec[t];
                dp[j] = acc;
                D += p[j] * acc;
            }
            for (int64_t j = 0; j < Nk; ++j) {
                if (s[j] == -INFINITY)
                    continue;
                double ds = p[j] * (dp[j] - D);
                load_vec(pb->k, pb->dtype, kv_off(pb, b, g, j), d, kvec);
                double* dkj = dk + j * d;
                double* dvj = dv + j * d;
                for (int64_t t = 0; t < d; ++t) {
                    dqi[t] += pb->scale * ds * kvec[t];
                    dkj[t] += pb->scale * ds * qi[t];
                    dvj[t] += p[j] * doi[t];
                }
            }
        }
    }
    free(s);
    free(p);
    free(dp);
    free(qi);
    free(doi);
    free(oi);
    free(kvec);
}

/* Full backward.  dq: [B,Hq,Nq,d]; dk, dv: [B,Hkv,Nk,d] (doubles).
 * Returns 0 on success, 2 if scratch could not be allocated. */
int oracle_bwd(const void* q, const void* k, const void* v, const void* dout, int dtype,
               int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
               double scale, int causal, double* dq, double* dk, double* dv, int nthreads)
{
    if (check_dims(B, Hq, Hkv, Nq, Nk, d))
        return 1;
    problem_t pb = {q, k, v, dout, dtype, B, Hq, Hkv, Nq, Nk, d, scale, causal};
    nthreads = resolve_threads(nthreads);
    int64_t groups = B * Hkv;
    /* a fixed number of row chunks per kv group, so the order in which partial
     * dK/dV sums are added does not depend on the thread count */
    int64_t chunks = 16;
    int64_t rows_per_group = (Hq / Hkv) * Nq;
    if (chunks > rows_per_group)
        chunks = rows_per_group;
    if (chunks < 1)
        chunks = 1;
    size_t part = (size_t)(groups * chunks) * (size_t)(Nk * d);
    double* dk_part = (double*)malloc(sizeof(double) * part);
    double* dv_part = (double*)malloc(sizeof(double) * part);
    if (!dk_part || !dv_part) {
        free(dk_part);
        free(dv_part);
        return 2;
    }
    bwd_ctx_t c = {&pb, chunks, dq, dk_part, dv_part};
    parallel_for(groups * chunks, nthreads, bwd_range, &c);
    for (int64_t bg = 0; bg < groups; ++bg) {
        double* dkg = dk + bg * Nk * d;
        double* dvg = dv + bg * Nk * d;
        memset(dkg, 0, sizeof(double) * Nk * d);
        memset(dvg, 0, sizeof(double) * Nk * d);
        for (int64_t ch = 0; ch < chunks; ++ch) {
            const double* pk = dk_part + (bg * chunks + ch) * Nk * d;
            const double* pv = dv_part + (bg * chunks + ch) * Nk * d;
            for (int64_t t = 0; t < Nk * d; ++t) {
                dkg[t] += pk[t];
                dvg[t] += pv[t];
            }
        }
    }
    free(dk_part);
    free(dv_part);
    return 0;
}

/* dQ for a list of flattened query rows only (each dQ row depends on its own
 * P and dP rows alone).  dq: [nrows, d]. */
typedef struct {
    const problem_t* pb;
    const int64_t* rows;
    double* dq;
} dqrow_ctx_t;

static void dqrow_range(void* vctx, int64_t begin, int64_t end, int tid)
{
    (void)tid;
    dqrow_ctx_t* c = (dqrow_ctx_t*)vctx;
    const problem_t* pb = c->pb;
    const int64_t d = pb->d, Nk = pb->Nk;
    const int64_t G = pb->Hq / pb->Hkv;
    double* s = (double*)malloc(sizeof(double) * Nk);
    double* p = (double*)malloc(sizeof(double) * Nk);
    double* qi = (double*)malloc(sizeof(double) * d);
    double* doi = (double*)malloc(sizeof(double) * d);
    double* oi = (double*)malloc(sizeof(double) * d);
    double* kvec = (double*)malloc(sizeof(double) * d);
    double* dp = (double*)malloc(sizeof(double) * Nk);
    for (int64_t r = begin; r < end; ++r) {
        int64_t flat = c->rows[r];
        int64_t i = flat % pb->Nq;
        int64_t h = (flat / pb->Nq) % pb->Hq;
        int64_t b = flat / (pb->Nq * pb->Hq);
        int64_t g = h / G;
        double* dqi = c->dq + r * d;
        load_vec(pb->q, pb->dtype, q_off(pb, b, h, i), d, qi);
        load_vec(pb->dout, pb->dtype, q_off(pb, b, h, i), d, doi);
        double lse;
        int64_t nvis = row_forward(pb, b, h, i, qi, s, p, oi, &lse, kvec);
        for (int64_t t = 0; t < d; ++t)
            dqi[t] = 0.0;
        if (nvis == 0)
            continue;
        double D = 0.0;
        for (int64_t j = 0; j < Nk; ++j) {
            dp[j] = 0.0;
            if (s[j] == -INFINITY)
                continue;
            load_vec(pb->v, pb->dtype, kv_off(pb, b, g, j), d, kvec);
            double acc = 0.0;
            for (int64_t t = 0; t < d; ++t)
                acc += doi[t] * kvec[t];
            dp[j] = acc;
            D += p[j] * acc;
        }
        for (int64_t j = 0; j < Nk; ++j) {
            if (s[j] == -INFINITY)
                continue;
            double ds = p[j] * (dp[j] - D);
            load_vec(pb->k, pb->dtype, kv_off(pb, b, g, j), d, kvec);
            for (int64_t t = 0; t < d; ++t)
                dqi[t] += pb->scale * ds * kvec[t];
        }
    }
    free(s);
    free(p);
    free(qi);
    free(doi);
    free(oi);
    free(kvec);
    free(dp);
}

int oracle_bwd_dq_rows(const void* q, const void* k, const void* v, const void* dout, int dtype,
                       int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
                       double scale, int causal, const int64_t* rows, int64_t nrows,
                       double* dq, int nthreads)
{
    if (check_dims(B, Hq, Hkv, Nq, Nk, d))
        return 1;
    problem_t pb = {q, k, v, dout, dtype, B, Hq, Hkv, Nq, Nk, d, scale, causal};
    dqrow_ctx_t c = {&pb, rows, dq};
    parallel_for(nrows, nthreads, dqrow_range, &c);
    return 0;
}

/* dK and dV for a list of keys (b, g, j) given as flattened key rows
 * kr = (b * Hkv + g) * Nk + j.  Every query row of the group that sees key j
 * contributes, and each such row needs its own full P and dP rows for D_i.
 * dk, dv: [nkeys, d].
 *
 * The work unit is (kv group, chunk of the group's query rows): each row's P
 * and dP are computed once and then added into every requested key of that
 * group the row sees.  For each key the rows are still added in the same order
 * (row order inside a chunk, then the chunks in order), so the result does not
 * depend on which other keys are requested with it. */
typedef struct {
    const problem_t* pb;
    const int64_t* keys;
    int64_t nkeys;
    const int64_t* groups;   /* distinct b * Hkv + g among the keys */
    int64_t ngroups;
    double* dk_part; /* [nchunks, nkeys, d] */
    double* dv_part;
    int64_t nchunks;
} dkrow_ctx_t;

static void dkrow_range(void* vctx, int64_t begin, int64_t end, int tid)
{
    (void)tid;
    dkrow_ctx_t* c = (dkrow_ctx_t*)vctx;
    const problem_t* pb = c->pb;
    const int64_t d = pb->d, Nk = pb->Nk, Nq = pb->Nq;
    const int64_t G = pb->Hq / pb->Hkv;
    double* s = (double*)malloc(sizeof(double) * Nk);
    double* p = (double*)malloc(sizeof(double) * Nk);
    double* qi = (double*)malloc(sizeof(double) * d);
    double* doi = (double*)malloc(sizeof(double) * d);
    double* oi = (double*)malloc(sizeof(double) * d);
    double* kvec = (double*)malloc(sizeof(double) * d);
    double* dp = (double*)malloc(sizeof(double) * Nk);
    /* unit = (group, chunk) */
    for (int64_t u = begin; u < end; ++u) {
        const int64_t gi = u / c->nchunks;
        const int64_t chunk = u % c->nchunks;
        const int64_t grp = c->groups[gi];
        const int64_t g = grp % pb->Hkv, b = grp / pb->Hkv;
        int64_t jmin = Nk;   /* smallest requested key of the group: rows that miss it miss all */
        for (int64_t kk = 0; kk < c->nkeys; ++kk) {
            if (c->keys[kk] / Nk != grp)
                continue;
            const int64_t j = c->keys[kk] % Nk;
            if (j < jmin)
                jmin = j;
            double* dkj = c->dk_part + (chunk * c->nkeys + kk) * d;
            double* dvj = c->dv_part + (chunk * c->nkeys + kk) * d;
            for (int64_t t = 0; t < d; ++t) {
                dkj[t] = 0.0;
                dvj[t] = 0.0;
            }
        }
        int64_t rows = G * Nq;
        int64_t r0 = rows * chunk / c->nchunks, r1 = rows * (chunk + 1) / c->nchunks;
        for (int64_t r = r0; r < r1; ++r) {
            int64_t h = g * G + r / Nq;
            int64_t i = r % Nq;
            if (!visible(pb, i, jmin))
                continue;
            load_vec(pb->q, pb->dtype, q_off(pb, b, h, i), d, qi);
            load_vec(pb->dout, pb->dtype, q_off(pb, b, h, i), d, doi);
            double lse;
            row_forward(pb, b, h, i, qi, s, p, oi, &lse, kvec);
            double D = 0.0;
            for (int64_t jj = 0; jj < Nk; ++jj) {
                dp[jj] = 0.0;
                if (s[jj] == -INFINITY)
                    continue;
                load_vec(pb->v, pb->dtype, kv_off(pb, b, g, jj), d, kvec);
                double acc = 0.0;
                for (int64_t t = 0; t < d; ++t)
                    acc += doi[t] * kvec[t];
                dp[jj] = acc;
                D += p[jj] * acc;
            }
            for (int64_t kk = 0; kk < c->nkeys; ++kk) {
                if (c->keys[kk] / Nk != grp)
                    continue;
                const int64_t j = c->keys[kk] % Nk;
                if (!visible(pb, i, j))
                    continue;
                double* dkj = c->dk_part + (chunk * c->nkeys + kk) * d;
                double* dvj = c->dv_part + (chunk * c->nkeys + kk) * d;
                double ds = p[j] * (dp[j] - D);
                for (int64_t t = 0; t < d; ++t) {
                    dkj[t] += pb->scale * ds * qi[t];
                    dvj[t] += p[j] * doi[t];
                }
            }
        }
    }
    free(s);
    free(p);
    free(qi);
    free(doi);
    free(oi);
    free(kvec);
    free(dp);
}

int oracle_bwd_dkv_rows(const void* q, const void* k, const void* v, const void* dout, int dtype,
                        int64_t B, int64_t Hq, int64_t Hkv, int64_t Nq, int64_t Nk, int64_t d,
                        double scale, int causal, const int64_t* keys, int64_t nkeys,
                        double* dk, double* dv, int nthreads)
{
    if (check_dims(B, Hq, Hkv, Nq, Nk, d))
        return 1;
    problem_t pb = {q, k, v, dout, dtype, B, Hq, Hkv, Nq, Nk, d, scale, causal};
    nthreads = resolve_threads(nthreads);
    /* fixed chunking of the group's rows: results do not depend on nthreads */
    int64_t nchunks = 16;
    if (nchunks > (Hq / Hkv) * Nq)
        nchunks = (Hq / Hkv) * Nq;
    double* dk_part = (double*)malloc(sizeof(double) * nchunks * nkeys * d);
    double* dv_part = (double*)malloc(sizeof(double) * nchunks * nkeys * d);
    if (!dk_part || !dv_part) {
        free(dk_part);
        free(dv_part);
        return 2;
    }
    int64_t* groups = (int64_t*)malloc(sizeof(int64_t) * (nkeys > 0 ? nkeys : 1));
    if (!groups) {
        free(dk_part);
        free(dv_part);
        return 2;
    }
    int64_t ngroups = 0;
    for (int64_t kk = 0; kk < nkeys; ++kk) {
        const int64_t grp = keys[kk] / Nk;
        int64_t seen = 0;
        for (int64_t x = 0; x < ngroups; ++x)
            seen |= (groups[x] == grp);
        if (!seen)
            groups[ngroups++] = grp;
    }
    dkrow_ctx_t c = {&pb, keys, nkeys, groups, ngroups, dk_part, dv_part, nchunks};
    parallel_for(ngroups * nchunks, nthreads, dkrow_range, &c);
    free(groups);
    for (int64_t kk = 0; kk < nkeys; ++kk) {
        for (int64_t t = 0; t < d; ++t) {
            double a = 0.0, bsum = 0.0;
            for (int64_t ch = 0; ch < nchunks; ++ch) {
                a += dk_part[(ch * nkeys + kk) * d + t];
                bsum += dv_part[(ch * nkeys + kk) * d + t];
            }
            dk[kk * d + t] = a;
            dv[kk * d + t] = bsum;
        }
    }
    free(dk_part);
    free(dv_part);
    return 0;
}

/* ---------------------------------------------------------------------------
 * The online-softmax recurrence of [P2] §04, over one row of scores s[0..n)
 * and value rows v[0..n) of width dv, processed in consecutive blocks of size
 * `block`.  State per row: m (max of scores seen), l (rescaled exp-sum) and U
 * (unnormalised output), initialised to m = -inf, l = 0, U = 0.  Per block:
 *     m_new = max(m_old, max(scores_block))
 *     a     = exp(m_old - m_new)
 *     p     = exp(scores_block - m_new)
 *     l     = a * l + sum(p)
 *     U     = a * U + p @ V_block
 * and at the end O = U / l.  Masked entries are -inf scores.  A block whose
 * running max is still -inf leaves the state at its initial value.
 *
 * trace (optional, may be NULL): for every block, four records are appended:
 *   [m_after, l_before_rescale*a (= l after rescale), U after rescale (dv values),
 *    l after adding the block, U after adding the block (dv values)]
 * laid out as (2 + 2*dv + 1) doubles per block:
 *   m_new, l_rescaled, U_rescaled[dv], l_new, U_new[dv]
 * The fp64 and fp32 versions differ only in the arithmetic type.
 * Returns the number of blocks processed.
 * ------------------------------------------------------------------------- */
#define DEFINE_ONLINE_ROW(NAME, T, EXP)                                                      \
    int64_t NAME(const double* s, const double* v, int64_t n, int64_t dv, int64_t block,    \
                 double* o, double* m_out, double* l_out, double* trace)                    \
    {                                                                                        \
        T m = (T)-INFINITY, l = (T)0;                                                        \
        T* U = (T*)calloc((size_t)(dv > 0 ? dv : 1), sizeof(T));                             \
        int64_t nb = 0;                                                                      \
        for (int64_t j0 = 0; j0 < n; j0 += block, ++nb) {                                    \
            int64_t j1 = j0 + block < n ? j0 + block : n;                                    \
            T bmax = (T)-INFINITY;                                                           \
            for (int64_t j = j0; j < j1; ++j)                                                \
                if ((T)s[j] > bmax)                                                          \
                    bmax = (T)s[j];                                                          \
            T m_new = m > bmax ? m : bmax;                                                   \
            T a = (m_new == (T)-INFINITY) ? (T)1 : EXP(m - m_new);                           \
            l = a * l;                                                                       \
            for (int64_t t = 0; t < dv; ++t)                                                 \
                U[t] = a * U[t];                                                             \
            double* tr = trace ? trace + nb * (3 + 2 * dv) : NULL;                           \
            if (tr) {                                                                        \
                tr[0] = (double)m_new;                                                       \
                tr[1] = (double)l;                                                           \
                for (int64_t t = 0; t < dv; ++t)                                             \
                    tr[2 + t] = (double)U[t];                                                \
            }                                                                                \
            if (m_new != (T)-INFINITY) {                                                     \
                for (int64_t j = j0; j < j1; ++j) {                                          \
                    T p = EXP((T)s[j] - m_new);                                              \
                    l += p;                                                                  \
                    for (int64_t t = 0; t < dv; ++t)                                         \
                        U[t] += p * (T)v[j * dv + t];                                        \
                }                                                                            \
            }                                                                                \
            m = m_new;                                                                       \
            if (tr) {                                                                        \
                tr[2 + dv] = (double)l;                                                      \
                for (int64_t t = 0; t < dv; ++t)                                             \
                    tr[3 + dv + t] = (double)U[t];                                           \
            }                                                                                \
        }                                                                                    \
        for (int64_t t = 0; t < dv; ++t)                                                     \
            o[t] = (l > (T)0) ? (double)(U[t] / l) : 0.0;                                    \
        *m_out = (double)m;                                                                  \
        *l_out = (double)l;                                                                  \
        free(U);                                                                             \
        return nb;                                                                           \
    }

DEFINE_ONLINE_ROW(oracle_online_row_f64, double, exp)
DEFINE_ONLINE_ROW(oracle_online_row_f32, float, expf)

/* The same row, softmax over the whole row at once (no blocking), in fp32:
 * m = max s, l = sum exp(s - m), O = sum exp(s - m) v / l.  Used beside the
 * fp32 blocked recurrence for the two-block check. */
void oracle_full_row_f32(const double* s, const double* v, int64_t n, int64_t dv,
                         double* o, double* m_out, double* l_out)
{
    float m = -INFINITY, l = 0.0f;
    for (int64_t j = 0; j < n; ++j)
        if ((float)s[j] > m)
            m = (float)s[j];
    float* U = (float*)calloc((size_t)(dv > 0 ? dv : 1), sizeof(float));
    if (m != -INFINITY) {
        for (int64_t j = 0; j < n; ++j) {
            float p = expf((float)s[j] - m);
            l += p;
            for (int64_t t = 0; t < dv; ++t)
                U[t] += p * (float)v[j * dv + t];
        }
    }
    for (int64_t t = 0; t < dv; ++t)
        o[t] = l > 0.0f ? (double)(U[t] / l) : 0.0;
    *m_out = (double)m;
    *l_out = (double)l;
    free(U);
}

/* ---------------------------------------------------------------------------
 * Merge of partial results over disjoint key ranges, in log-sum-exp form.
 * Each part s holds lse_s = m_s + ln l_s and O_s = U_s / l_s for its own keys;
 * the rule of [P2] §04 (rescale old numerator and denominator together, then
 * add) gives  lse = ln sum_s exp(lse_s)  and  O = sum_s exp(lse_s - lse) O_s.
 * Parts with lse_s = -inf (no visible key) contribute nothing.
 * o_parts: [nparts, d], lse_parts: [nparts]; writes o[d], *lse.
 * ------------------------------------------------------------------------- */
void oracle_lse_merge(const double* o_parts, const double* lse_parts, int64_t nparts,
                      int64_t d, double* o, double* lse)
{
    double mx = -INFINITY;
    for (int64_t s = 0; s < nparts; ++s)
        if (lse_parts[s] > mx)
            mx = lse_parts[s];
    for (int64_t t = 0; t < d; ++t)
        o[t] = 0.0;
    if (mx == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double sum = 0.0;
    for (int64_t s = 0; s < nparts; ++s)
        sum += exp(lse_parts[s] - mx);
    double L = mx + log(sum);
    for (int64_t s = 0; s < nparts; ++s) {
        double w = exp(lse_parts[s] - L);
        for (int64_t t = 0; t < d; ++t)
            o[t] += w * o_parts[s * d + t];
    }
    *lse = L;
}

/*
 * e4m3 code -> double, from the definition of the OCP 8-bit floating point
 * format E4M3 (the variant without infinities used for FP8 attention inputs):
 *   bit 7 sign, bits 6..3 exponent e (bias 7), bits 2..0 mantissa m;
 *   e = 0:            (-1)^sign * m * 2^-9          (subnormal; m = 0 is zero)
 *   e = 15, m = 7:    NaN
 *   otherwise:        (-1)^sign * (1 + m / 8) * 2^(e - 7)
 * so the largest finite magnitude is 0x7E = 1.75 * 2^8 = 448.
 */
void oracle_e4m3_to_f64(const uint8_t* codes, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i) {
        const unsigned c = codes[i];
        const int sign = (c >> 7) & 1;
        const int e = (c >> 3) & 15;
        const int m = c & 7;
        double mag;
        if (e == 15 && m == 7)
            mag = NAN;
        else if (e == 0)
            mag = ldexp((double)m, -9);
        else
            mag = ldexp(1.0 + m / 8.0, e - 7);
        out[i] = sign ? -mag : mag;
    }
}

int oracle_abi_version(void) { return 1; }
