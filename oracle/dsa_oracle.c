/*
 * CPU oracle for the DSA hot path.  TEST INFRASTRUCTURE: only the tests, the
 * smoke check and the benchmark's CPU-baseline leg may load this library.
 * It shares no code with the CUDA path.
 *
 * What it computes (Kwai Keye-VL-2.0 technical-report summary, section 1
 * "why long video is hard": a light MQA-style "Lightning Indexer" scores every
 * visible position, each query keeps its 2048 best positions, attention runs
 * over those only; the base model is GQA; section 8: the same selection at
 * decode).  The pages do not print the indexer formula; the DeepSeek Sparse
 * Attention indexer that they name is read as
 *
 *     I[t,s] = sum_j w[t,j] * max(0, sum_c qI[t,j,c] * kI[s,c]),   s <= t
 *
 * (one shared key vector per token, per-head ReLU, weighted head sum, no
 * scale, no position encoding).  Selection keeps the min(k, t+1) largest
 * scores under the total order (higher score first, then lower index) and
 * lists them in ascending index order, padded with -1.  Attention:
 *
 *     O[t,h] = sum_{s in idx[t]} softmax_s(scale * Q[t,h] . K[s,g]) V[s,g],
 *     g = h / (Hq / Hkv)
 *
 * one index set per query token, shared by every KV group and query head.
 *
 * Arithmetic: fp64.  Each e4m3 value is m * 2^e with a 4-bit m, so every
 * product of two of them is a multiple of 2^-18 below 2^18 and any dot
 * product of up to 2^17 terms is exact in fp64; with integer-valued weights
 * the scores are exact integers.  Softmax uses exp() in fp64 after
 * subtracting the row maximum.  A row with no valid index gives O = 0.
 *
 * Pins (tests marked "not gpu"): brute-force full sort of every (score, s)
 * on tiny inputs, a hand-derived worked example, closed forms (all-zero
 * scores select 0..k-1; equal keys give the mean of V; constant V), head
 * permutation / weight scaling invariance, softmax weights summing to one,
 * equality with the separate dense causal routine below when k >= t+1, and
 * decode equal to the last prefill row on the same data.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------ decoding */

/* FP8 e4m3 (OCP FP8 spec): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities, S.1111.111 is NaN; exponent field 0 is subnormal. */
double oracle_e4m3(uint8_t b) {
    int s = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);              /* m/8 * 2^-6 */
    else v = ldexp(8.0 + m, e - 10);                   /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* bf16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double E4M3[256];
static pthread_once_t e4m3_once = PTHREAD_ONCE_INIT;
static void e4m3_init(void) {
    for (int i = 0; i < 256; ++i) E4M3[i] = oracle_e4m3((uint8_t)i);
}

/* ------------------------------------------------------------ threads */

typedef void (*row_fn)(void* ctx, int64_t r, void* scratch);
typedef struct {
    row_fn fn;
    void* ctx;
    int64_t nrows;
    size_t scratch_bytes;
    int64_t next;
    pthread_mutex_t mu;
    int failed;
} pool_t;

static void* pool_worker(void* p) {
    pool_t* P = (pool_t*)p;
    void* scratch = P->scratch_bytes ? malloc(P->scratch_bytes) : NULL;
    if (P->scratch_bytes && !scratch) {
        pthread_mutex_lock(&P->mu);
        P->failed = 1;
        pthread_mutex_unlock(&P->mu);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&P->mu);
        int64_t r = P->next++;
        pthread_mutex_unlock(&P->mu);
        if (r >= P->nrows) break;
        P->fn(P->ctx, r, scratch);
    }
    free(scratch);
    return NULL;
}

/* Runs fn(ctx, r, scratch) for r in [0, nrows) on nthreads threads (0: all
 * online cores).  Returns 0, or -1 if a scratch buffer could not be had. */
static int run_rows(row_fn fn, void* ctx, int64_t nrows, size_t scratch_bytes, int nthreads) {
    pthread_once(&e4m3_once, e4m3_init);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    if (nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
    pool_t P = {fn, ctx, nrows, scratch_bytes, 0, PTHREAD_MUTEX_INITIALIZER, 0};
    pthread_t th[512];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, pool_worker, &P) != 0) break;
        started++;
    }
    if (started == 0) pool_worker(&P);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    return P.failed ? -1 : 0;
}

/* ------------------------------------------------------------ indexer */

/* scores[s] for s in [0, n): sum_j w[j] * max(0, q[j,:] . kI[s,:]). */
static void score_row(const uint8_t* q, const float* w, const uint8_t* kI, int64_t n, int H,
                      int d, double* qd, double* scores) {
    for (int j = 0; j < H; ++j)
        for (int c = 0; c < d; ++c) qd[(int64_t)j * d + c] = E4M3[q[(int64_t)j * d + c]];
    for (int64_t s = 0; s < n; ++s) {
        const uint8_t* kr = kI + s * d;
        double score = 0.0;
        for (int j = 0; j < H; ++j) {
            const double* qj = qd + (int64_t)j * d;
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += qj[c] * E4M3[kr[c]];
            score += (double)w[j] * (dot > 0.0 ? dot : 0.0);
        }
        scores[s] = score;
    }
}

typedef struct { double score; int64_t s; } cand_t;

/* Total order: higher score first, then lower index. */
static int cand_cmp(const void* a_, const void* b_) {
    const cand_t* a = (const cand_t*)a_;
    const cand_t* b = (const cand_t*)b_;
    if (a->score != b->score) return a->score > b->score ? -1 : 1;
    return (a->s > b->s) - (a->s < b->s);
}

static int i32_cmp(const void* a_, const void* b_) {
    int32_t a = *(const int32_t*)a_, b = *(const int32_t*)b_;
    return (a > b) - (a < b);
}

/* Keeps the min(k, n) best of scores[0..n) and writes them ascending,
 * padded with -1 up to k. */
static void select_row(const double* scores, int64_t n, int k, cand_t* cand, int32_t* out) {
    for (int64_t s = 0; s < n; ++s) { cand[s].score = scores[s]; cand[s].s = s; }
    qsort(cand, (size_t)n, sizeof(cand_t), cand_cmp);
    int64_t m = n < k ? n : k;
    for (int64_t i = 0; i < m; ++i) out[i] = (int32_t)cand[i].s;
    qsort(out, (size_t)m, sizeof(int32_t), i32_cmp);
    for (int64_t i = m; i < k; ++i) out[i] = -1;
}

typedef struct {
    const uint8_t* qI; const uint8_t* kI; const float* w;
    int64_t L; int H, d, k;
    const int64_t* rows;
    int32_t* idx;
    double* scores_out;
} index_ctx;

static size_t index_scratch(int64_t L, int H, int d) {
    return (size_t)L * sizeof(double) + (size_t)L * sizeof(cand_t) +
           (size_t)H * d * sizeof(double);
}

static void index_row(void* c_, int64_t r, void* scratch) {
    index_ctx* c = (index_ctx*)c_;
    int64_t t = c->rows[r];
    double* scores = (double*)scratch;
    cand_t* cand = (cand_t*)(scores + c->L);
    double* qd = (double*)(cand + c->L);
    int64_t n = t + 1;
    score_row(c->qI + t * c->H * c->d, c->w + t * c->H, c->kI, n, c->H, c->d, qd, scores);
    if (c->idx) select_row(scores, n, c->k, cand, c->idx + r * (int64_t)c->k);
    if (c->scores_out) {
        double* o = c->scores_out + r * c->L;
        for (int64_t s = 0; s < c->L; ++s) o[s] = s < n ? scores[s] : -INFINITY;
    }
}

/* Prefill selection for query rows rows[0..nrows): idx_out[r][0..k) holds the
 * selected keys of token rows[r], ascending, -1 padded.  q_I [L][H][d] e4m3,
 * k_I [L][d] e4m3, w [L][H] fp32.  Returns 0, or -1 on allocation failure. */
int oracle_index_topk(const uint8_t* qI, const uint8_t* kI, const float* w, int64_t L, int H,
                      int d, int k, const int64_t* rows, int64_t nrows, int32_t* idx_out,
                      int nthreads) {
    index_ctx c = {qI, kI, w, L, H, d, k, rows, idx_out, NULL};
    return run_rows(index_row, &c, nrows, index_scratch(L, H, d), nthreads);
}

/* Dense causal indexer scores for rows[0..nrows): scores_out[r][s] = I[t,s]
 * for s <= t, -inf for s > t ([nrows][L], fp64). */
int oracle_index_scores(const uint8_t* qI, const uint8_t* kI, const float* w, int64_t L, int H,
                        int d, const int64_t* rows, int64_t nrows, double* scores_out,
                        int nthreads) {
    index_ctx c = {qI, kI, w, L, H, d, 0, rows, NULL, scores_out};
    return run_rows(index_row, &c, nrows, index_scratch(L, H, d), nthreads);
}

/* ------------------------------------------------------------ attention */

/* Softmax weights of one (query, head) over the listed rows.  K [n][Hkv][d]
 * bf16 bits; q points at Q[t,h] (d bf16 bits); rows outside [0, n) are not
 * valid and get weight 0.  Returns the number of valid rows; p[i] is the
 * weight of idx[i]. */
static int64_t softmax_weights(const uint16_t* q, const uint16_t* K, int64_t n, int Hkv, int d,
                               int g, const int32_t* idx, int64_t m, double scale, double* x,
                               double* p) {
    int64_t valid = 0;
    double mx = -INFINITY;
    for (int64_t i = 0; i < m; ++i) {
        int64_t s = idx[i];
        if (s < 0 || s >= n) { x[i] = -INFINITY; continue; }
        const uint16_t* kr = K + (s * Hkv + g) * (int64_t)d;
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += oracle_bf16(q[c]) * oracle_bf16(kr[c]);
        x[i] = scale * dot;
        if (x[i] > mx) mx = x[i];
        valid++;
    }
    double z = 0.0;
    for (int64_t i = 0; i < m; ++i) {
        p[i] = (x[i] == -INFINITY) ? 0.0 : exp(x[i] - mx);
        z += p[i];
    }
    for (int64_t i = 0; i < m; ++i) p[i] = valid ? p[i] / z : 0.0;
    return valid;
}

typedef struct {
    const uint16_t *Q, *K, *V;
    int64_t n;              /* rows of K/V */
    const int32_t* idx;     /* [rows of Q][k], or [nrows][k] when idx_by_r */
    int idx_by_r;
    int k, Hq, Hkv, d;
    double scale;
    const int64_t* rows;
    double* out;            /* [nrows][Hq][d] */
} attn_ctx;

static void attn_row(void* c_, int64_t r, void* scratch) {
    attn_ctx* c = (attn_ctx*)c_;
    int64_t t = c->rows[r];
    double* x = (double*)scratch;
    double* p = x + c->k;
    int G = c->Hq / c->Hkv;
    const int32_t* idx = c->idx + (c->idx_by_r ? r : t) * (int64_t)c->k;
    for (int h = 0; h < c->Hq; ++h) {
        int g = h / G;
        const uint16_t* q = c->Q + (t * c->Hq + h) * (int64_t)c->d;
        softmax_weights(q, c->K, c->n, c->Hkv, c->d, g, idx, c->k, c->scale, x, p);
        double* o = c->out + (r * c->Hq + h) * (int64_t)c->d;
        for (int e = 0; e < c->d; ++e) o[e] = 0.0;
        for (int i = 0; i < c->k; ++i) {
            if (p[i] == 0.0) continue;
            const uint16_t* vr = c->V + ((int64_t)idx[i] * c->Hkv + g) * c->d;
            for (int e = 0; e < c->d; ++e) o[e] += p[i] * oracle_bf16(vr[e]);
        }
    }
}

/* Sparse GQA attention for query rows rows[0..nrows) of Q [*][Hq][d] over
 * K, V [n][Hkv][d] (bf16 bits) at the positions idx[t][0..k) (or idx[r][..]
 * for the r-th listed row when idx_by_r is set); entries outside [0, n) are
 * skipped.  out [nrows][Hq][d] fp64. */
int oracle_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t n,
                       const int32_t* idx, int idx_by_r, int k, int Hq, int Hkv, int d,
                       double scale, const int64_t* rows, int64_t nrows, double* out,
                       int nthreads) {
    attn_ctx c = {Q, K, V, n, idx, idx_by_r, k, Hq, Hkv, d, scale, rows, out};
    return run_rows(attn_row, &c, nrows, 2 * (size_t)k * sizeof(double), nthreads);
}

/* Softmax weights for one (t, h): p_out[i] is the weight of idx[t][i]. */
int64_t oracle_attn_weights(const uint16_t* Q, const uint16_t* K, int64_t n, const int32_t* idx,
                            int k, int Hq, int Hkv, int d, double scale, int64_t t, int h,
                            double* p_out) {
    double* x = (double*)malloc((size_t)k * sizeof(double));
    if (!x) return -1;
    int G = Hq / Hkv;
    int64_t v = softmax_weights(Q + (t * Hq + h) * (int64_t)d, K, n, Hkv, d, h / G,
                                idx + t * (int64_t)k, k, scale, x, p_out);
    free(x);
    return v;
}

/* Dense causal softmax attention, written on its own (no selection, no
 * shared helper): O[t,h] = sum_{s<=t} softmax(scale Q.K) V. */
typedef struct {
    const uint16_t *Q, *K, *V;
    int Hq, Hkv, d;
    double scale;
    const int64_t* rows;
    double* out;
} dense_ctx;

static void dense_row(void* c_, int64_t r, void* scratch) {
    dense_ctx* c = (dense_ctx*)c_;
    int64_t t = c->rows[r];
    double* x = (double*)scratch;
    int G = c->Hq / c->Hkv;
    for (int h = 0; h < c->Hq; ++h) {
        int g = h / G;
        const uint16_t* q = c->Q + (t * c->Hq + h) * (int64_t)c->d;
        double mx = -INFINITY;
        for (int64_t s = 0; s <= t; ++s) {
            const uint16_t* kr = c->K + (s * c->Hkv + g) * (int64_t)c->d;
            double dot = 0.0;
            for (int e = 0; e < c->d; ++e) dot += oracle_bf16(q[e]) * oracle_bf16(kr[e]);
            x[s] = c->scale * dot;
            if (x[s] > mx) mx = x[s];
        }
        double z = 0.0;
        for (int64_t s = 0; s <= t; ++s) z += exp(x[s] - mx);
        double* o = c->out + (r * c->Hq + h) * (int64_t)c->d;
        for (int e = 0; e < c->d; ++e) {
            double acc = 0.0;
            for (int64_t s = 0; s <= t; ++s)
                acc += exp(x[s] - mx) / z * oracle_bf16(c->V[(s * c->Hkv + g) * (int64_t)c->d + e]);
            o[e] = acc;
        }
    }
}

int oracle_dense_causal_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t L,
                             int Hq, int Hkv, int d, double scale, const int64_t* rows,
                             int64_t nrows, double* out, int nthreads) {
    dense_ctx c = {Q, K, V, Hq, Hkv, d, scale, rows, out};
    return run_rows(dense_row, &c, nrows, (size_t)L * sizeof(double), nthreads);
}

/* ------------------------------------------------------------ decode */

/* One new token per sequence; its row is the last row of the sequence's
 * cache (n_b includes it), so decode equals the prefill row t = n_b - 1 of
 * that sequence.  Caches are packed: sequence b owns rows
 * [cache_off[b], cache_off[b+1]).  For the sequences seqs[0..nseq):
 * idx_out [nseq][k] (sequence-local positions, ascending, -1 padded) and
 * out [nseq][Hq][d]. */
typedef struct {
    const uint8_t* qI; const float* w; const uint16_t* Q;
    const uint8_t* kI; const uint16_t *K, *V;
    const int64_t* off;
    int H, dI, Hq, Hkv, d, k;
    double scale;
    const int64_t* seqs;
    int32_t* idx;
    double* out;
    int64_t max_n;
} decode_ctx;

static void decode_row(void* c_, int64_t r, void* scratch) {
    decode_ctx* c = (decode_ctx*)c_;
    int64_t b = c->seqs[r];
    int64_t base = c->off[b], n = c->off[b + 1] - c->off[b];
    double* scores = (double*)scratch;
    cand_t* cand = (cand_t*)(scores + c->max_n);
    double* qd = (double*)(cand + c->max_n);
    double* x = qd + (int64_t)c->H * c->dI;
    double* p = x + c->k;
    int32_t* idx = c->idx + r * (int64_t)c->k;
    score_row(c->qI + b * c->H * c->dI, c->w + b * c->H, c->kI + base * c->dI, n, c->H, c->dI,
              qd, scores);
    select_row(scores, n, c->k, cand, idx);
    const uint16_t* K = c->K + base * c->Hkv * c->d;
    const uint16_t* V = c->V + base * c->Hkv * c->d;
    int G = c->Hq / c->Hkv;
    for (int h = 0; h < c->Hq; ++h) {
        int g = h / G;
        softmax_weights(c->Q + (b * c->Hq + h) * (int64_t)c->d, K, n, c->Hkv, c->d, g, idx, c->k,
                        c->scale, x, p);
        double* o = c->out + (r * c->Hq + h) * (int64_t)c->d;
        for (int e = 0; e < c->d; ++e) o[e] = 0.0;
        for (int i = 0; i < c->k; ++i) {
            if (p[i] == 0.0) continue;
            const uint16_t* vr = V + ((int64_t)idx[i] * c->Hkv + g) * c->d;
            for (int e = 0; e < c->d; ++e) o[e] += p[i] * oracle_bf16(vr[e]);
        }
    }
}

int oracle_decode(const uint8_t* qI, const float* w, const uint16_t* Q, const uint8_t* kI_cache,
                  const uint16_t* K_cache, const uint16_t* V_cache, const int64_t* cache_off,
                  int H, int dI, int Hq, int Hkv, int d, int k, double scale,
                  const int64_t* seqs, int64_t nseq, int32_t* idx_out, double* out,
                  int nthreads) {
    int64_t max_n = 0;
    for (int64_t r = 0; r < nseq; ++r) {
        int64_t b = seqs[r], n = cache_off[b + 1] - cache_off[b];
        if (n > max_n) max_n = n;
    }
    decode_ctx c = {qI, w, Q, kI_cache, K_cache, V_cache, cache_off, H, dI, Hq, Hkv, d, k,
                    scale, seqs, idx_out, out, max_n};
    size_t scratch = (size_t)max_n * (sizeof(double) + sizeof(cand_t)) +
                     (size_t)H * dI * sizeof(double) + 2 * (size_t)k * sizeof(double);
    return run_rows(decode_row, &c, nseq, scratch, nthreads);
}
