/*
 * Plain CPU oracle for tile-sparse softmax attention (forward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header or table with the CUDA library.
 *
 * What it computes follows "FG-Attn: Leveraging Fine-Grained Sparse Attention
 * in Video Diffusion Models", Abstract: score computations are skipped for
 * whole M x N tiles (M queries x N keys, M >= 16, N >= 1); a skipped score is
 * taken as -inf, i.e. it contributes nothing to the softmax.  Everything else
 * is the textbook definition of softmax attention, evaluated in double
 * precision with plain loops and no blocking, fusion or reordering:
 *
 *   s_ij  = scale * sum_t q_it k_jt              if tile (i / M, j / N) is kept
 *         = -inf                                 otherwise
 *   m_i   = max_j s_ij
 *   l_i   = sum_j exp(s_ij - m_i)
 *   out_i = sum_j exp(s_ij - m_i) v_j / l_i
 *   lse_i = m_i + ln l_i                         (natural logarithm)
 *
 * Readings where the page is silent (the CUDA library takes the same ones,
 * written separately):
 *   - mask layout: uint32 words, tile (qb, g) is bit (g % 32) of word g / 32 of
 *     row (b, h, qb); W = ceil(G / 32) words per row; bits >= G are ignored;
 *   - the "diagonal" tiles a query block always keeps are the tiles that hold
 *     each of its rows' own key index: groups floor(qb*M/N) ..
 *     floor((min(qb*M+M, L) - 1) / N);
 *   - keys >= L do not exist; the last group holds L - (G-1)*N keys;
 *     query rows >= L are neither computed nor written.
 *
 * The backward pass (oracle_attention_backward, at the end of this file) is the
 * plain gradient of the same definition, also in double precision.
 *
 * Build with any C99 compiler:  cc -O2 -shared -fPIC -pthread fgattn_oracle.c
 * (no -ffast-math: the sums must be evaluated in program order).
 *
 * ORACLE_MUTANT (compile-time, default 0) plants one deliberate mistake so the
 * test suite can show that its pins catch it; it is never set for real use.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* bf16 bit pattern -> double (exact: bf16 is the top half of an IEEE binary32). */
static double bf16_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Is tile (row, g) kept?  Reads the packed mask bit, then the diagonal rule. */
static int tile_kept(const uint32_t* mask_row, int64_t qb, int64_t g, int64_t L, int64_t M, int64_t N) {
#if ORACLE_MUTANT == 6 /* planted: bits read most-significant first */
    int bit = (int)((mask_row[g / 32] >> (31 - (g % 32))) & 1u);
#else
    int bit = (int)((mask_row[g / 32] >> (g % 32)) & 1u);
#endif
    if (bit) return 1;
#if ORACLE_MUTANT == 3 /* planted: no diagonal forcing */
    return 0;
#else
    int64_t row_lo = qb * M;
    int64_t row_hi = (qb * M + M < L ? qb * M + M : L) - 1;
    return g >= row_lo / N && g <= row_hi / N;
#endif
}

/*
 * Mask compaction: for every row (b, h, qb) list the kept key indices in
 * ascending order, kept_idx[row * cap + n], and their number kept_cnt[row].
 * Returns 0, or -1 if a list would not fit in cap.
 */
int oracle_compact(const uint32_t* mask, int64_t B, int64_t H, int64_t L, int64_t M, int64_t N,
                   int32_t* kept_idx, int32_t* kept_cnt, int64_t cap) {
    const int64_t QB = (L + M - 1) / M;
    const int64_t G = (L + N - 1) / N;
    const int64_t W = (G + 31) / 32;
    for (int64_t row = 0; row < B * H * QB; ++row) {
        const uint32_t* mrow = mask + row * W;
        const int64_t qb = row % QB;
        int64_t n = 0;
        for (int64_t g = 0; g < G; ++g) {
            if (!tile_kept(mrow, qb, g, L, M, N)) continue;
            int64_t start = g * N;
#if ORACLE_MUTANT == 4 /* planted: the ragged last group is given N keys */
            int64_t stop = start + N;
#else
            int64_t stop = start + N < L ? start + N : L;
#endif
            for (int64_t j = start; j < stop; ++j) {
                if (n >= cap) return -1;
                kept_idx[row * cap + n++] = (int32_t)j;
            }
        }
        kept_cnt[row] = (int32_t)n;
    }
    return 0;
}

typedef struct {
    const uint16_t *q, *k, *v;
    const uint32_t* mask;
    int64_t B, H, L, d, M, N;
    double scale;
    const int64_t* blocks;
    int64_t nblocks;
    double *out, *lse;
    int64_t first, last; /* this worker's share of blocks */
    int status;
} job_t;

/* One query block (b, h, qb): rows qb*M .. min(qb*M+M, L)-1. */
static int attention_block(const job_t* J, int64_t bi) {
    const int64_t L = J->L, d = J->d, M = J->M, N = J->N;
    const int64_t QB = (L + M - 1) / M;
    const int64_t G = (L + N - 1) / N;
    const int64_t W = (G + 31) / 32;
    const int64_t blk = J->blocks[bi];
    if (blk < 0 || blk >= J->B * J->H * QB) return -1;
    const int64_t bh = blk / QB, qb = blk % QB;
    const uint32_t* mrow = J->mask + blk * W;
    const uint16_t* Q = J->q + bh * L * d;
    const uint16_t* K = J->k + bh * L * d;
    const uint16_t* V = J->v + bh * L * d;
    double* out = J->out + bi * M * d;
    double* lse = J->lse + bi * M;

    double* s = (double*)malloc((size_t)L * sizeof(double));
    char* kept = (char*)malloc((size_t)G);
    if (!s || !kept) { free(s); free(kept); return -2; }
    for (int64_t g = 0; g < G; ++g) kept[g] = (char)tile_kept(mrow, qb, g, L, M, N);

    for (int64_t r = 0; r < M; ++r) {
        const int64_t i = qb * M + r;
        if (i >= L) { /* rows past the sequence end are not computed */
            for (int64_t t = 0; t < d; ++t) out[r * d + t] = NAN;
            lse[r] = NAN;
            continue;
        }
        /* pass 1: scores, -inf where the tile is skipped */
        for (int64_t j = 0; j < L; ++j) {
#if ORACLE_MUTANT == 8 /* planted: the mask is ignored */
            if (0) {
#else
            if (!kept[j / N]) {
#endif
                s[j] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int64_t t = 0; t < d; ++t) {
#if ORACLE_MUTANT == 2 /* planted: query and key swapped */
                acc += bf16_to_double(Q[j * d + t]) * bf16_to_double(K[i * d + t]);
#else
                acc += bf16_to_double(Q[i * d + t]) * bf16_to_double(K[j * d + t]);
#endif
            }
#if ORACLE_MUTANT == 1 /* planted: scale dropped */
            s[j] = acc;
#else
            s[j] = J->scale * acc;
#endif
        }
        /* pass 2: max, normaliser, weighted sum of values */
        double m = -INFINITY;
        for (int64_t j = 0; j < L; ++j) if (s[j] > m) m = s[j];
        double l = 0.0;
        for (int64_t j = 0; j < L; ++j) l += exp(s[j] - m);
        for (int64_t t = 0; t < d; ++t) out[r * d + t] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (s[j] == -INFINITY) continue; /* exp(-inf) = 0: the term is exactly zero */
            const double p = exp(s[j] - m);
            for (int64_t t = 0; t < d; ++t) out[r * d + t] += p * bf16_to_double(V[j * d + t]);
        }
#if ORACLE_MUTANT == 7 /* planted: no division by the normaliser */
        (void)0;
#else
        for (int64_t t = 0; t < d; ++t) out[r * d + t] /= l;
#endif
#if ORACLE_MUTANT == 5 /* planted: base-2 logarithm */
        lse[r] = m + log2(l);
#else
        lse[r] = m + log(l);
#endif
    }
    free(s);
    free(kept);
    return 0;
}

static void* worker(void* arg) {
    job_t* J = (job_t*)arg;
    for (int64_t bi = J->first; bi < J->last; ++bi) {
        int st = attention_block(J, bi);
        if (st) { J->status = st; break; }
    }
    return NULL;
}

/*
 * Attention for a list of query blocks.  q, k, v: bf16 bit patterns,
 * [B][H][L][d] contiguous.  blocks[i] = (b*H + h)*QB + qb.  Writes
 * out[i][r][t] and lse[i][r] for r < M (NaN for rows >= L).  nthreads <= 0
 * means one thread.  Returns 0 on success.
 */
int oracle_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint32_t* mask,
                     int64_t B, int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, double scale,
                     const int64_t* blocks, int64_t nblocks, double* out, double* lse, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nblocks) nthreads = (int)(nblocks > 0 ? nblocks : 1);
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return -2; }
    for (int w = 0; w < nthreads; ++w) {
        job_t* J = &jobs[w];
        J->q = q; J->k = k; J->v = v; J->mask = mask;
        J->B = B; J->H = H; J->L = L; J->d = d; J->M = M; J->N = N;
        J->scale = scale; J->blocks = blocks; J->nblocks = nblocks;
        J->out = out; J->lse = lse;
        J->first = nblocks * w / nthreads;
        J->last = nblocks * (w + 1) / nthreads;
        J->status = 0;
    }
    int status = 0;
    if (nthreads == 1) {
        worker(&jobs[0]);
        status = jobs[0].status;
    } else {
        int started = 0;
        for (int w = 0; w < nthreads; ++w) {
            if (pthread_create(&tid[w], NULL, worker, &jobs[w]) != 0) { status = -3; break; }
            ++started;
        }
        for (int w = 0; w < started; ++w) pthread_join(tid[w], NULL);
        for (int w = 0; w < nthreads && !status; ++w) status = jobs[w].status;
    }
    free(jobs);
    free(tid);
    return status;
}

/*
 * Backward pass (gradients of the forward above), evaluated in double precision
 * by the definition, per (b, h) head: with p_ij = exp(s_ij - m_i) / l_i for the
 * kept scores (0 for skipped ones) and the upstream gradient dO of out,
 *
 *   dP_ij = dO_i . v_j                 D_i   = sum_j p_ij dP_ij  (= dO_i . out_i)
 *   dS_ij = p_ij (dP_ij - D_i)
 *   dq_i  = scale * sum_j dS_ij k_j    dk_j  = scale * sum_i dS_ij q_i
 *   dv_j  = sum_i p_ij dO_i
 *
 * (the chain rule through s = scale * q . k, the softmax and out = P v; a
 * skipped score has p = 0 and contributes to no gradient).  q, k, v, dout:
 * bf16 bit patterns [B][H][L][d]; dq, dk, dv: double [B][H][L][d].
 */
typedef struct {
    const uint16_t *q, *k, *v, *dout;
    const uint32_t* mask;
    int64_t B, H, L, d, M, N;
    double scale;
    int64_t bh;                /* the head */
    int64_t row_first, row_last; /* this worker's query rows */
    double *dq;                /* dq of the head (rows are disjoint between workers) */
    double *dk, *dv;           /* this worker's partial sums over its rows, [L][d] */
    int status;
} bjob_t;

/* Rows row_first .. row_last-1 of one head: dq of those rows, and their terms
 * of dk and dv added into the worker's own partial sums. */
static int backward_rows(const bjob_t* J) {
    const int64_t L = J->L, d = J->d, M = J->M, N = J->N, bh = J->bh;
    const int64_t QB = (L + M - 1) / M;
    const int64_t G = (L + N - 1) / N;
    const int64_t W = (G + 31) / 32;
    const uint16_t* Q = J->q + bh * L * d;
    const uint16_t* K = J->k + bh * L * d;
    const uint16_t* V = J->v + bh * L * d;
    const uint16_t* DO = J->dout + bh * L * d;
    double* dq = J->dq;
    double* dk = J->dk;
    double* dv = J->dv;
    double* s = (double*)malloc((size_t)L * sizeof(double));
    double* dp = (double*)malloc((size_t)L * sizeof(double));
    char* kept = (char*)malloc((size_t)G);
    if (!s || !dp || !kept) { free(s); free(dp); free(kept); return -2; }
    for (int64_t x = 0; x < L * d; ++x) { dk[x] = 0.0; dv[x] = 0.0; }
    for (int64_t i = J->row_first; i < J->row_last; ++i) {
        const int64_t qb = i / M;
        const uint32_t* mrow = J->mask + (bh * QB + qb) * W;
        for (int64_t g = 0; g < G; ++g) kept[g] = (char)tile_kept(mrow, qb, g, L, M, N);
        /* probabilities of row i */
        double m = -INFINITY;
        for (int64_t j = 0; j < L; ++j) {
            if (!kept[j / N]) { s[j] = -INFINITY; continue; }
            double acc = 0.0;
            for (int64_t t = 0; t < d; ++t) acc += bf16_to_double(Q[i * d + t]) * bf16_to_double(K[j * d + t]);
            s[j] = J->scale * acc;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < L; ++j) l += exp(s[j] - m);
        /* dP_ij and D_i */
        double D = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (s[j] == -INFINITY) { dp[j] = 0.0; continue; }
            double acc = 0.0;
            for (int64_t t = 0; t < d; ++t) acc += bf16_to_double(DO[i * d + t]) * bf16_to_double(V[j * d + t]);
            dp[j] = acc;
#if ORACLE_MUTANT == 11 /* planted: dv from unnormalised probabilities (no division by l) */
            const double p = exp(s[j] - m);
#else
            const double p = exp(s[j] - m) / l;
#endif
            D += p * acc;
        }
        for (int64_t t = 0; t < d; ++t) dq[i * d + t] = 0.0;
        for (int64_t j = 0; j < L; ++j) {
            if (s[j] == -INFINITY) continue;
#if ORACLE_MUTANT == 11
            const double p = exp(s[j] - m);
#else
            const double p = exp(s[j] - m) / l;
#endif
#if ORACLE_MUTANT == 9 /* planted: the -D_i term dropped */
            const double ds = p * dp[j];
#else
            const double ds = p * (dp[j] - D);
#endif
            for (int64_t t = 0; t < d; ++t) {
#if ORACLE_MUTANT == 12 /* planted: dq accumulates the query instead of the key */
                dq[i * d + t] += J->scale * ds * bf16_to_double(Q[i * d + t]);
#else
                dq[i * d + t] += J->scale * ds * bf16_to_double(K[j * d + t]);
#endif
#if ORACLE_MUTANT == 10 /* planted: dk without the scale */
                dk[j * d + t] += ds * bf16_to_double(Q[i * d + t]);
#else
                dk[j * d + t] += J->scale * ds * bf16_to_double(Q[i * d + t]);
#endif
                dv[j * d + t] += p * bf16_to_double(DO[i * d + t]);
            }
        }
    }
    free(s);
    free(dp);
    free(kept);
    return 0;
}

static void* bworker(void* arg) {
    bjob_t* J = (bjob_t*)arg;
    J->status = backward_rows(J);
    return NULL;
}

/* Gradients dq, dk, dv of every head (see above).  Returns 0 on success.
 * Heads one after the other; the rows of a head split between up to nthreads
 * workers, each summing its rows' terms of dk and dv on its own; the head's dk
 * and dv are then those partial sums added in worker order. */
int oracle_attention_backward(const uint16_t* q, const uint16_t* k, const uint16_t* v, const uint16_t* dout,
                              const uint32_t* mask, int64_t B, int64_t H, int64_t L, int64_t d, int64_t M,
                              int64_t N, double scale, double* dq, double* dk, double* dv, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > L) nthreads = (int)L;
    /* partial sums take 2 * L * d doubles per worker: at most about 1 GiB of them */
    const int64_t per = 2 * L * d * (int64_t)sizeof(double);
    const int64_t cap = per > 0 ? (((int64_t)1 << 30) / per) : 1;
    if (cap < nthreads) nthreads = cap < 1 ? 1 : (int)cap;
    bjob_t* jobs = (bjob_t*)calloc((size_t)nthreads, sizeof(bjob_t));
    pthread_t* tid = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    double* part = (double*)malloc((size_t)nthreads * (size_t)per);
    if (!jobs || !tid || !part) { free(jobs); free(tid); free(part); return -2; }
    int status = 0;
    for (int64_t bh = 0; bh < B * H && !status; ++bh) {
        for (int w = 0; w < nthreads; ++w) {
            bjob_t* J = &jobs[w];
            J->q = q; J->k = k; J->v = v; J->dout = dout; J->mask = mask;
            J->B = B; J->H = H; J->L = L; J->d = d; J->M = M; J->N = N; J->scale = scale;
            J->bh = bh;
            J->row_first = L * w / nthreads;
            J->row_last = L * (w + 1) / nthreads;
            J->dq = dq + bh * L * d;
            J->dk = part + (size_t)w * 2 * (size_t)(L * d);
            J->dv = J->dk + L * d;
            J->status = 0;
        }
        if (nthreads == 1) {
            bworker(&jobs[0]);
        } else {
            int started = 0;
            for (int w = 0; w < nthreads; ++w) {
                if (pthread_create(&tid[w], NULL, bworker, &jobs[w]) != 0) { status = -3; break; }
                ++started;
            }
            for (int w = 0; w < started; ++w) pthread_join(tid[w], NULL);
        }
        for (int w = 0; w < nthreads && !status; ++w) status = jobs[w].status;
        if (status) break;
        double* hk = dk + bh * L * d;
        double* hv = dv + bh * L * d;
        for (int64_t x = 0; x < L * d; ++x) { hk[x] = 0.0; hv[x] = 0.0; }
        for (int w = 0; w < nthreads; ++w)
            for (int64_t x = 0; x < L * d; ++x) { hk[x] += jobs[w].dk[x]; hv[x] += jobs[w].dv[x]; }
    }
    free(part);
    free(jobs);
    free(tid);
    return status;
}
