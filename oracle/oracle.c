/*
 * oracle.c -- plain, slow fp64 CPU definition of top-k context-sparse decode
 * attention.  TEST INFRASTRUCTURE: only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table
 * or helper with the CUDA library, and neither includes nor links the other.
 *
 * What it computes (citations are to the pages the method comes from):
 *  - score: for kv-head group G, s_j = max_{h in G} scale * <q_h, k_j>
 *    ("inference-time context sparsity: illusion or opportunity?", sec. 2,
 *    oracle top-k picks the k highest-importance tokens exactly; the group
 *    reduction by max is the reading this library takes for GQA, since the
 *    pages only say sparsity may be head-wise);
 *  - top-k: the k_b = min(k_req, n_b) largest scores, ties to the lower index,
 *    returned in ascending index order (same page, sec. 2 "oracle Top-K");
 *  - attention: exact softmax attention of every query head of the group over
 *    only the selected rows (HyLRA sec. 2.3 "attention restricted to the
 *    subset"; "Flash Attention vs Sparse Attention", DSA stage 2), written as
 *    the textbook two-pass softmax (max, then exp-sum), in double;
 *  - block mode: 128-token block means scored like keys, top blocks expanded
 *    to their valid tokens (HyLRA sec. 2.4, block-level sparsity).
 *
 * Every input is bf16 bit patterns (uint16) decoded here exactly to double.
 * Units are (b, kv-head) pairs, u = b * Hkv + kvh; an optional list restricts
 * the work to some units (used to sample large workloads).
 *
 * Parallelism: OpenMP over units only; no blocking or reordering of any sum
 * beyond the definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* dot product of a double query row with a double key row */
static double dot_d(const double* a, const double* b, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += a[c] * b[c];
    return s;
}

static void decode_row(const uint16_t* src, double* dst, int d) {
    for (int c = 0; c < d; ++c) dst[c] = bf16_bits_to_double(src[c]);
}

static int unit_at(const int32_t* units, int i) { return units ? units[i] : i; }

/* Token-mode scores.  S is [B, Hkv, Ncap]; entries j >= len_b are left as is. */
int oracle_scores(const uint16_t* Q, const uint16_t* K, const int32_t* lens, int B, int Hq,
                  int Hkv, int Ncap, int d, double scale, const int32_t* units, int n_units,
                  double* S) {
    if (Hkv <= 0 || Hq % Hkv != 0) return 1;
    const int g = Hq / Hkv;
    const int nu = units ? n_units : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nu; ++i) {
        const int u = unit_at(units, i);
        const int b = u / Hkv, kvh = u % Hkv;
        double* q = (double*)malloc(sizeof(double) * (size_t)g * d);
        double* k = (double*)malloc(sizeof(double) * (size_t)d);
        for (int h = 0; h < g; ++h)
            decode_row(Q + ((size_t)b * Hq + (size_t)kvh * g + h) * d, q + (size_t)h * d, d);
        const uint16_t* Kb = K + ((size_t)b * Hkv + kvh) * (size_t)Ncap * d;
        double* Su = S + ((size_t)b * Hkv + kvh) * (size_t)Ncap;
        for (int j = 0; j < lens[b]; ++j) {
            decode_row(Kb + (size_t)j * d, k, d);
            double best = -INFINITY;
            for (int h = 0; h < g; ++h) {
                double z = scale * dot_d(q + (size_t)h * d, k, d);
                if (z > best) best = z;
            }
            Su[j] = best;
        }
        free(q);
        free(k);
    }
    return 0;
}

/* Block means: M[b,kvh,beta,:] = mean of the valid K rows of block beta
 * (rows [beta*block, min(beta*block+block, len_b))).  M is [B,Hkv,NB,d],
 * NB = ceil(Ncap/block); blocks with no valid row are left as is. */
int oracle_block_means(const uint16_t* K, const int32_t* lens, int B, int Hkv, int Ncap, int d,
                       int block, const int32_t* units, int n_units, double* M) {
    if (block <= 0) return 1;
    const int NB = (Ncap + block - 1) / block;
    const int nu = units ? n_units : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nu; ++i) {
        const int u = unit_at(units, i);
        const int b = u / Hkv, kvh = u % Hkv;
        const uint16_t* Kb = K + ((size_t)b * Hkv + kvh) * (size_t)Ncap * d;
        double* Mu = M + ((size_t)b * Hkv + kvh) * (size_t)NB * d;
        const int nblk = (lens[b] + block - 1) / block;
        for (int beta = 0; beta < nblk; ++beta) {
            const int t0 = beta * block;
            int t1 = t0 + block;
            if (t1 > lens[b]) t1 = lens[b];
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int t = t0; t < t1; ++t) s += bf16_bits_to_double(Kb[(size_t)t * d + c]);
                Mu[(size_t)beta * d + c] = s / (double)(t1 - t0);
            }
        }
    }
    return 0;
}

/* Block-mode scores: the same group max of scaled logits, against the block
 * means.  S is [B, Hkv, NB]; nrows[b] = number of valid blocks of sequence b. */
int oracle_block_scores(const uint16_t* Q, const double* M, const int32_t* nrows, int B, int Hq,
                        int Hkv, int NB, int d, double scale, const int32_t* units, int n_units,
                        double* S) {
    if (Hkv <= 0 || Hq % Hkv != 0) return 1;
    const int g = Hq / Hkv;
    const int nu = units ? n_units : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nu; ++i) {
        const int u = unit_at(units, i);
        const int b = u / Hkv, kvh = u % Hkv;
        double* q = (double*)malloc(sizeof(double) * (size_t)g * d);
        for (int h = 0; h < g; ++h)
            decode_row(Q + ((size_t)b * Hq + (size_t)kvh * g + h) * d, q + (size_t)h * d, d);
        const double* Mu = M + ((size_t)b * Hkv + kvh) * (size_t)NB * d;
        double* Su = S + ((size_t)b * Hkv + kvh) * (size_t)NB;
        for (int j = 0; j < nrows[b]; ++j) {
            double best = -INFINITY;
            for (int h = 0; h < g; ++h) {
                double z = scale * dot_d(q + (size_t)h * d, Mu + (size_t)j * d, d);
                if (z > best) best = z;
            }
            Su[j] = best;
        }
        free(q);
    }
    return 0;
}

typedef struct {
    double s;
    int32_t j;
} scored_t;

/* order: higher score first; equal scores -> lower index first */
static int by_score_then_index(const void* pa, const void* pb) {
    const scored_t* a = (const scored_t*)pa;
    const scored_t* b = (const scored_t*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_int(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/* Exact top-k per unit by a full sort.  S is [B,Hkv,rows_cap]; sequence b has
 * nrows[b] valid rows and wants kreq[b] of them; idx is [B,Hkv,k_max],
 * ascending, padded with -1.  Returns 2 if some k_b exceeds k_max. */
int oracle_topk(const double* S, const int32_t* nrows, const int32_t* kreq, int B, int Hkv,
                int rows_cap, int k_max, const int32_t* units, int n_units, int32_t* idx) {
    for (int b = 0; b < B; ++b) {
        int kb = kreq[b] < nrows[b] ? kreq[b] : nrows[b];
        if (kb > k_max) return 2;
    }
    const int nu = units ? n_units : B * Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nu; ++i) {
        const int u = unit_at(units, i);
        const int b = u / Hkv;
        const int n = nrows[b];
        int kb = kreq[b] < n ? kreq[b] : n;
        if (kb < 0) kb = 0;
        const double* Su = S + (size_t)u * rows_cap;
        scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
        for (int j = 0; j < n; ++j) {
            all[j].s = Su[j];
            all[j].j = j;
        }
        qsort(all, (size_t)n, sizeof(scored_t), by_score_then_index);
        int32_t* out = idx + (size_t)u * k_max;
        for (int t = 0; t < kb; ++t) out[t] = all[t].j;
        qsort(out, (size_t)kb, sizeof(int32_t), by_int);
        for (int t = kb; t < k_max; ++t) out[t] = -1;
        free(all);
    }
    return 0;
}

/* Exact softmax attention of each query head over a set of cache rows.
 *  idx == NULL: the set is every valid row [0, len_b) (a full-attention layer);
 *  block == 1 : the set is idx[u, 0:k_b), k_b = min(kreq[b], len_b), entries < 0 skipped;
 *  block  > 1 : idx holds block numbers, k_b = min(kreq[b], ceil(len_b/block)), and
 *               each block contributes its valid rows [beta*block, min(+block, len_b)).
 * O is [B, Hq, d]; a head whose set is empty gets O = 0.  Returns 3 if an index is
 * out of range. */
int oracle_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* lens,
                const int32_t* idx, const int32_t* kreq, int k_max, int block, int B, int Hq,
                int Hkv, int Ncap, int d, double scale, const int32_t* units, int n_units,
                double* O) {
    if (Hkv <= 0 || Hq % Hkv != 0 || block <= 0) return 1;
    const int g = Hq / Hkv;
    const int nu = units ? n_units : B * Hkv;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < nu; ++i) {
        const int u = unit_at(units, i);
        const int b = u / Hkv, kvh = u % Hkv;
        const int len = lens[b];
        /* 1. the attended rows */
        int cap = idx ? k_max * block : len;
        int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(cap > 0 ? cap : 1));
        int nr = 0;
        if (!idx) {
            for (int j = 0; j < len; ++j) rows[nr++] = j;
        } else {
            int units_valid = block == 1 ? len : (len + block - 1) / block;
            int kb = kreq[b] < units_valid ? kreq[b] : units_valid;
            if (kb > k_max) kb = k_max;
            const int32_t* iu = idx + (size_t)u * k_max;
            for (int t = 0; t < kb; ++t) {
                int e = iu[t];
                if (e < 0) continue;
                if (e >= units_valid) {
#pragma omp atomic write
                    err = 3;
                    continue;
                }
                int t0 = e * block, t1 = e * block + block;
                if (t1 > len) t1 = len;
                for (int j = t0; j < t1; ++j) rows[nr++] = j;
            }
        }
        if (nr == 0) { /* nothing to attend (len_b = 0 or k_b = 0): output 0 by definition */
            for (int hh = 0; hh < g; ++hh)
                memset(O + ((size_t)b * Hq + (size_t)kvh * g + hh) * d, 0, sizeof(double) * d);
            free(rows);
            continue;
        }
        const uint16_t* Kb = K + ((size_t)b * Hkv + kvh) * (size_t)Ncap * d;
        const uint16_t* Vb = V + ((size_t)b * Hkv + kvh) * (size_t)Ncap * d;
        double* q = (double*)malloc(sizeof(double) * (size_t)d);
        double* kv = (double*)malloc(sizeof(double) * (size_t)d);
        double* z = (double*)malloc(sizeof(double) * (size_t)nr);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        for (int hh = 0; hh < g; ++hh) {
            const int h = kvh * g + hh;
            decode_row(Q + ((size_t)b * Hq + h) * d, q, d);
            /* 2. logits and their maximum */
            double m = -INFINITY;
            for (int t = 0; t < nr; ++t) {
                decode_row(Kb + (size_t)rows[t] * d, kv, d);
                z[t] = scale * dot_d(q, kv, d);
                if (z[t] > m) m = z[t];
            }
            /* 3. weights, their sum, and the weighted sum of V rows */
            double den = 0.0;
            for (int c = 0; c < d; ++c) acc[c] = 0.0;
            for (int t = 0; t < nr; ++t) {
                double w = exp(z[t] - m);
                den += w;
                decode_row(Vb + (size_t)rows[t] * d, kv, d);
                for (int c = 0; c < d; ++c) acc[c] += w * kv[c];
            }
            double* Oh = O + ((size_t)b * Hq + h) * d;
            for (int c = 0; c < d; ++c) Oh[c] = acc[c] / den;
        }
        free(q);
        free(kv);
        free(z);
        free(acc);
        free(rows);
    }
    return err;
}
