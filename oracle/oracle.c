/*
 * Plain, slow fp64 CPU oracle for the CSA lightning-indexer top-k step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes follows "StreamIndex: Memory-Bounded Compressed Sparse
 * Attention via Streaming Top-k", Abstract: a lightning indexer scores the
 * compressed keys each query can see, and the top-k keys are kept per query.
 * The abstract prints no formula; this oracle uses the plainest reading that
 * the rest of the text supports:
 *
 *   score(b,t,j) = sum_h w[b,t,h] * max(0, sum_d q[b,t,h,d] * kc[b,j,d])
 *   key j is visible to query t  iff  (j+1)*m - 1 <= t,
 *     i.e. query t sees V_t = min(T, floor((t+1)/m)) keys, T = S/m
 *   keep the min(k, V_t) best keys, ordered by score descending then index
 *   ascending (-0 and +0 are equal scores); pad the rest with index -1 and
 *   score -inf.
 *
 * Every product and sum is taken in fp64 in ascending h and d order.  bf16 and
 * fp32 inputs convert to fp64 exactly.  The sort is the C library's qsort.
 * No blocking, no fusion, no streaming: each row is scored in full, then sorted.
 *
 * FP8 variant: rows are quantised to OCP FP8 E4M3 with a per-row scale
 * (FP8 Formats for Deep Learning, cited in the abstract's reference list):
 *   scale = amax(|x_row|) / 448   (fp32 division; 1 for an all-zero row)
 *   code  = E4M3 round-to-nearest-even, saturating at 448, of x / scale (fp32)
 * and scored as
 *   score = sum_h w[t,h] * max(0, s_q[t,h]*s_k[j]*sum_d q8[t,h,d]*k8[j,d])
 * with the codes decoded exactly to fp64.  The MX block-scaled variant (one
 * power-of-two scale per 32 elements) has its own section below.
 */
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    double s;
    int32_t j;
} pair_t;

typedef struct {
    float s;
    int32_t j;
} pairf_t;

/* score descending, then index ascending.  IEEE comparison treats -0 == +0. */
static int cmp_pair(const void* a, const void* b) {
    const pair_t* x = (const pair_t*)a;
    const pair_t* y = (const pair_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int cmp_pairf(const void* a, const void* b) {
    const pairf_t* x = (const pairf_t*)a;
    const pairf_t* y = (const pairf_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static double bf16_to_f64(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Threads the oracle's parallel loops use (1 without OpenMP). */
int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Number of compressed keys query t can see: all j with (j+1)*m - 1 <= t. */
int oracle_visible(int t, int T, int m) {
    int v = 0;
    while (v < T && (v + 1) * m - 1 <= t) v++;
    return v;
}

/* Score of key j for one query, given that query's own rows:
 *   qr [H,D] bf16 bits, wr [H] fp32, kcb [T,D] bf16 bits (the query's batch). */
double oracle_score_row(const uint16_t* qr, const float* wr, const uint16_t* kcb, int H, int D,
                        int j) {
    const uint16_t* kr = kcb + (int64_t)j * D;
    double s = 0.0;
    for (int h = 0; h < H; h++) {
        double dot = 0.0;
        for (int d = 0; d < D; d++) dot += bf16_to_f64(qr[h * D + d]) * bf16_to_f64(kr[d]);
        double r = dot > 0.0 ? dot : 0.0;
        s += (double)wr[h] * r;
    }
    return s;
}

/* Top-k for one query at position t: score every visible key, sort, keep k.
 * out_idx [k] int32, out_score [k] fp64. */
void oracle_topk_row(const uint16_t* qr, const float* wr, const uint16_t* kcb, int T, int H, int D,
                     int m, int t, int k, int32_t* out_idx, double* out_score) {
    int V = oracle_visible(t, T, m);
    pair_t* p = (pair_t*)malloc(sizeof(pair_t) * (size_t)(V > 0 ? V : 1));
    for (int j = 0; j < V; j++) {
        p[j].s = oracle_score_row(qr, wr, kcb, H, D, j);
        p[j].j = j;
    }
    qsort(p, (size_t)V, sizeof(pair_t), cmp_pair);
    for (int r = 0; r < k; r++) {
        out_idx[r] = r < V ? p[r].j : -1;
        out_score[r] = r < V ? p[r].s : -INFINITY;
    }
    free(p);
}

/*
 * Top-k of the visible keys for listed queries, each given by its own rows.
 *   q_rows [n,H,D] bf16 bits, w_rows [n,H] fp32, kc [B,T,D] bf16 bits,
 *   rows[n]: flat positions b*S + t of those queries.
 *   out_idx [n,k] int32, out_score [n,k] fp64.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_indexer_topk_rows(const uint16_t* q_rows, const float* w_rows, const uint16_t* kc,
                             int B, int S, int H, int D, int m, int k, const int64_t* rows, int n,
                             int32_t* out_idx, double* out_score) {
    if (B < 1 || S < 1 || H < 1 || D < 1 || m < 1 || k < 1 || S % m != 0) return -1;
    int T = S / m;
    for (int i = 0; i < n; i++)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * S) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int t = (int)(rows[i] % S);
        oracle_topk_row(q_rows + (int64_t)i * H * D, w_rows + (int64_t)i * H,
                        kc + b * T * (int64_t)D, T, H, D, m, t, k, out_idx + (int64_t)i * k,
                        out_score + (int64_t)i * k);
    }
    return 0;
}

/* As oracle_indexer_topk_rows, also returning each row's largest |score|
 * over its visible keys (out_absmax [n]); one scoring pass per row. */
int oracle_indexer_topk_rows_absmax(const uint16_t* q_rows, const float* w_rows,
                                    const uint16_t* kc, int B, int S, int H, int D, int m, int k,
                                    const int64_t* rows, int n, int32_t* out_idx,
                                    double* out_score, double* out_absmax) {
    if (B < 1 || S < 1 || H < 1 || D < 1 || m < 1 || k < 1 || S % m != 0) return -1;
    int T = S / m;
    for (int i = 0; i < n; i++)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * S) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int t = (int)(rows[i] % S);
        int V = oracle_visible(t, T, m);
        const uint16_t* qr = q_rows + (int64_t)i * H * D;
        const float* wr = w_rows + (int64_t)i * H;
        const uint16_t* kcb = kc + b * T * (int64_t)D;
        pair_t* p = (pair_t*)malloc(sizeof(pair_t) * (size_t)(V > 0 ? V : 1));
        for (int j = 0; j < V; j++) {
            p[j].s = oracle_score_row(qr, wr, kcb, H, D, j);
            p[j].j = j;
        }
        /* the scale of the tolerance rule: largest |score| over the visible keys */
        double mx = 0.0;
        for (int j = 0; j < V; j++)
            if (fabs(p[j].s) > mx) mx = fabs(p[j].s);
        qsort(p, (size_t)V, sizeof(pair_t), cmp_pair);
        for (int r = 0; r < k; r++) {
            out_idx[(int64_t)i * k + r] = r < V ? p[r].j : -1;
            out_score[(int64_t)i * k + r] = r < V ? p[r].s : -INFINITY;
        }
        out_absmax[i] = mx;
        free(p);
    }
    return 0;
}

/* Full tensors: q [B,S,H,D], w [B,S,H]; rows as above. */
int oracle_indexer_topk(const uint16_t* q, const float* w, const uint16_t* kc, int B, int S, int H,
                        int D, int m, int k, const int64_t* rows, int n, int32_t* out_idx,
                        double* out_score) {
    if (B < 1 || S < 1 || H < 1 || D < 1 || m < 1 || k < 1 || S % m != 0) return -1;
    int T = S / m;
    for (int i = 0; i < n; i++)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * S) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t row = rows[i];
        int64_t b = row / S;
        int t = (int)(row % S);
        oracle_topk_row(q + row * H * (int64_t)D, w + row * (int64_t)H, kc + b * T * (int64_t)D, T,
                        H, D, m, t, k, out_idx + (int64_t)i * k, out_score + (int64_t)i * k);
    }
    return 0;
}

/* fp64 scores of keys js[i, 0..kk) for listed queries given by their own
 * rows; used to judge keys outside the oracle's own top-k.  A key the query
 * cannot see (j < 0 or j >= V_t) has no score: its entry is left untouched, so
 * the caller's fill value (NaN) marks it, and no key past the batch's T is
 * ever read. */
void oracle_score_keys_rows(const uint16_t* q_rows, const float* w_rows, const uint16_t* kc, int S,
                            int H, int D, int m, const int64_t* rows, int n, const int32_t* js,
                            int kk, double* out) {
    int T = S / m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int V = oracle_visible((int)(rows[i] % S), T, m);
        for (int r = 0; r < kk; r++) {
            int j = js[(int64_t)i * kk + r];
            if (j < 0 || j >= V) continue;
            out[(int64_t)i * kk + r] = oracle_score_row(q_rows + (int64_t)i * H * D,
                                                        w_rows + (int64_t)i * H,
                                                        kc + b * T * (int64_t)D, H, D, j);
        }
    }
}

/* Largest |score| over each listed query's visible keys (the scale used by
 * the end-to-end tolerance rule). */
void oracle_row_absmax_rows(const uint16_t* q_rows, const float* w_rows, const uint16_t* kc, int S,
                            int H, int D, int m, const int64_t* rows, int n, double* out) {
    int T = S / m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int t = (int)(rows[i] % S);
        int V = oracle_visible(t, T, m);
        double mx = 0.0;
        for (int j = 0; j < V; j++) {
            double s = fabs(oracle_score_row(q_rows + (int64_t)i * H * D, w_rows + (int64_t)i * H,
                                             kc + b * T * (int64_t)D, H, D, j));
            if (s > mx) mx = s;
        }
        out[i] = mx;
    }
}

/*
 * Selection alone, on given fp32 scores X [B,S,T]: the same visibility rule
 * and order, applied to the fp32 values as given.  The selected scores are
 * returned with their exact input bit patterns.
 */
int oracle_topk_scores(const float* X, int B, int S, int T, int m, int k, const int64_t* rows, int n,
                       int32_t* out_idx, float* out_score) {
    if (B < 1 || S < 1 || T < 1 || m < 1 || k < 1) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t row = rows[i];
        int t = (int)(row % S);
        int V = oracle_visible(t, T, m);
        const float* xr = X + row * (int64_t)T;
        pairf_t* p = (pairf_t*)malloc(sizeof(pairf_t) * (size_t)(V > 0 ? V : 1));
        for (int j = 0; j < V; j++) {
            p[j].s = xr[j];
            p[j].j = j;
        }
        qsort(p, (size_t)V, sizeof(pairf_t), cmp_pairf);
        for (int r = 0; r < k; r++) {
            if (r < V) {
                out_idx[(int64_t)i * k + r] = p[r].j;
                out_score[(int64_t)i * k + r] = p[r].s;
            } else {
                out_idx[(int64_t)i * k + r] = -1;
                out_score[(int64_t)i * k + r] = -INFINITY;
            }
        }
        free(p);
    }
    return 0;
}

/* ----------------------------------------------------------------- FP8 E4M3 */

/* Exact value of an E4M3 code: 1 sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits; exponent field 0 is subnormal (2^-6 * m/8); code S.1111.111
 * is NaN (never produced here). */
double oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, mnt = c & 7;
    double v;
    if (e == 15 && mnt == 7) return NAN;
    if (e == 0)
        v = ldexp((double)mnt / 8.0, -6);
    else
        v = ldexp(1.0 + (double)mnt / 8.0, e - 7);
    return s ? -v : v;
}

/* Round half to even of a non-negative value to an integer. */
static double rne(double x) {
    double f = floor(x);
    double r = x - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return fmod(f, 2.0) == 0.0 ? f : f + 1.0;
}

/* fp32 -> E4M3, round to nearest even, saturating to +-448 (the largest finite
 * E4M3 value).  The sign of zero is kept. */
uint8_t oracle_e4m3_encode(float y) {
    uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) { /* subnormal grid: multiples of 2^-9 */
        double n = rne(a / ldexp(1.0, -9));
        return sign | (uint8_t)n; /* n == 8 is exactly the smallest normal, code 0x08 */
    }
    int E;
    (void)frexp(a, &E); /* a = f * 2^E with f in [0.5, 1) */
    int ex = E - 1;     /* so a = (2f) * 2^ex with 2f in [1, 2) */
    double n = rne((ldexp(a, -ex) - 1.0) * 8.0);
    if (n == 8.0) {
        n = 0.0;
        ex += 1;
    }
    int field = ex + 7;
    if (field > 15 || (field == 15 && n == 7.0)) return sign | 0x7E;
    return sign | (uint8_t)((field << 3) | (int)n);
}

/* Per-row quantisation of a bf16 matrix [rows, cols] to E4M3 codes plus one
 * fp32 scale per row. */
void oracle_quantize_e4m3_rows(const uint16_t* x, int64_t rows, int cols, uint8_t* codes,
                               float* scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        const uint16_t* xr = x + r * cols;
        float amax = 0.0f;
        for (int c = 0; c < cols; c++) {
            float v = fabsf((float)bf16_to_f64(xr[c]));
            if (v > amax) amax = v;
        }
        volatile float s = amax / 448.0f; /* volatile: keep one fp32 rounding */
        if (amax == 0.0f) s = 1.0f;
        scale[r] = s;
        for (int c = 0; c < cols; c++) {
            volatile float y = (float)bf16_to_f64(xr[c]) / s;
            codes[r * cols + c] = oracle_e4m3_encode(y);
        }
    }
}

/* FP8 score of key j for one query given its own rows: q8r [H,D] codes,
 * sqr [H] scales, wr [H]; k8b [T,D] codes and skb [T] scales of its batch. */
double oracle_score_row_fp8(const uint8_t* q8r, const float* sqr, const float* wr,
                            const uint8_t* k8b, const float* skb, int H, int D, int j) {
    const uint8_t* kr = k8b + (int64_t)j * D;
    double skj = (double)skb[j];
    double s = 0.0;
    for (int h = 0; h < H; h++) {
        double dot = 0.0;
        for (int d = 0; d < D; d++)
            dot += oracle_e4m3_decode(q8r[h * D + d]) * oracle_e4m3_decode(kr[d]);
        double x = (double)sqr[h] * skj * dot;
        s += (double)wr[h] * (x > 0.0 ? x : 0.0);
    }
    return s;
}

/* Top-k of the FP8 score for listed queries given by their own rows:
 * q8_rows [n,H,D] codes, sq_rows [n,H], w_rows [n,H]; k8 [B,T,D] codes,
 * sk [B,T].  Same order and padding as oracle_indexer_topk_rows. */
int oracle_indexer_topk_fp8_rows(const uint8_t* q8_rows, const float* sq_rows,
                                 const float* w_rows, const uint8_t* k8, const float* sk, int B,
                                 int S, int H, int D, int m, int k, const int64_t* rows, int n,
                                 int32_t* out_idx, double* out_score) {
    if (B < 1 || S < 1 || H < 1 || D < 1 || m < 1 || k < 1 || S % m != 0) return -1;
    int T = S / m;
    for (int i = 0; i < n; i++)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * S) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int t = (int)(rows[i] % S);
        int V = oracle_visible(t, T, m);
        pair_t* p = (pair_t*)malloc(sizeof(pair_t) * (size_t)(V > 0 ? V : 1));
        for (int j = 0; j < V; j++) {
            p[j].s = oracle_score_row_fp8(q8_rows + (int64_t)i * H * D, sq_rows + (int64_t)i * H,
                                          w_rows + (int64_t)i * H, k8 + b * T * (int64_t)D,
                                          sk + b * T, H, D, j);
            p[j].j = j;
        }
        qsort(p, (size_t)V, sizeof(pair_t), cmp_pair);
        for (int r = 0; r < k; r++) {
            out_idx[(int64_t)i * k + r] = r < V ? p[r].j : -1;
            out_score[(int64_t)i * k + r] = r < V ? p[r].s : -INFINITY;
        }
        free(p);
    }
    return 0;
}

/* FP8 scores of keys js[i, 0..kk) for listed queries given by their own rows;
 * keys the query cannot see are left untouched, as in oracle_score_keys_rows. */
void oracle_score_keys_fp8_rows(const uint8_t* q8_rows, const float* sq_rows, const float* w_rows,
                                const uint8_t* k8, const float* sk, int S, int H, int D, int m,
                                const int64_t* rows, int n, const int32_t* js, int kk,
                                double* out) {
    int T = S / m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int V = oracle_visible((int)(rows[i] % S), T, m);
        for (int r = 0; r < kk; r++) {
            int j = js[(int64_t)i * kk + r];
            if (j < 0 || j >= V) continue;
            out[(int64_t)i * kk + r] = oracle_score_row_fp8(
                q8_rows + (int64_t)i * H * D, sq_rows + (int64_t)i * H, w_rows + (int64_t)i * H,
                k8 + b * T * (int64_t)D, sk + b * T, H, D, j);
        }
    }
}

/* --------------------------------------------------------------- MX block FP8
 * Block-scaled E4M3 (MXFP8), from "Microscaling Data Formats for Deep
 * Learning" (cited in the abstract's reference list) and the OCP MX v1.0
 * rule it describes: every block of 32 consecutive elements of a row shares
 * one power-of-two scale X = 2^e, stored as an E8M0 byte e + 127, with
 *
 *   e = floor(log2(amax_block)) - 8        (8: the exponent of E4M3's largest
 *                                           normal value, 448 = 1.75 * 2^8)
 *
 * clamped to [-127, 127] (a block of zeros takes -127), and every element
 * becomes the E4M3 code (round to nearest even, saturating at 448) of x / X.
 * The scaled block maximum then lies in [256, 512) before rounding.  The
 * pages give no parameters; the block of 32 and the E4M3 element type are
 * the MXFP8 format of that specification.  The score is the definition with
 * every element decoded exactly:
 *
 *   score = sum_h w[t,h] * max(0, sum_d q8[t,h,d]*2^eq[t,h,d/32] * k8[j,d]*2^ek[j,d/32])
 */
#define MX_BLOCK 32

/* E8M0 byte of a block whose largest magnitude is amax. */
uint8_t oracle_mx_scale_byte(double amax) {
    if (!(amax > 0.0)) return 0; /* zeros: e = -127 */
    int E;
    (void)frexp(amax, &E); /* amax = f * 2^E, f in [0.5, 1): floor(log2 amax) = E - 1 */
    int e = (E - 1) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* x [rows, cols] bf16 bits, cols a multiple of 32 -> codes [rows, cols] and
 * scale bytes [rows, cols/32].  Returns -1 on bad sizes. */
int oracle_quantize_mxfp8_rows(const uint16_t* x, int64_t rows, int cols, uint8_t* codes,
                               uint8_t* scales) {
    if (rows < 0 || cols < MX_BLOCK || cols % MX_BLOCK != 0) return -1;
    int nb = cols / MX_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; r++) {
        for (int blk = 0; blk < nb; blk++) {
            const uint16_t* xb = x + r * cols + blk * MX_BLOCK;
            double amax = 0.0;
            for (int i = 0; i < MX_BLOCK; i++) {
                double v = fabs(bf16_to_f64(xb[i]));
                if (v > amax) amax = v;
            }
            uint8_t sb = oracle_mx_scale_byte(amax);
            scales[r * nb + blk] = sb;
            for (int i = 0; i < MX_BLOCK; i++) {
                /* x / 2^e is exact in fp64 and in fp32 (8 significant bits,
                 * far from fp32's range limits at the magnitudes E4M3 keeps) */
                double y = ldexp(bf16_to_f64(xb[i]), -((int)sb - 127));
                codes[r * cols + blk * MX_BLOCK + i] = oracle_e4m3_encode((float)y);
            }
        }
    }
    return 0;
}

/* MXFP8 score of key j for one query: q8r [H,D] codes, qsr [H,D/32] scale
 * bytes, wr [H]; k8b [T,D] codes and ksb [T,D/32] scale bytes of its batch. */
double oracle_score_row_mxfp8(const uint8_t* q8r, const uint8_t* qsr, const float* wr,
                              const uint8_t* k8b, const uint8_t* ksb, int H, int D, int j) {
    int nb = D / MX_BLOCK;
    const uint8_t* kr = k8b + (int64_t)j * D;
    const uint8_t* ks = ksb + (int64_t)j * nb;
    double s = 0.0;
    for (int h = 0; h < H; h++) {
        double dot = 0.0;
        for (int d = 0; d < D; d++) {
            double qv = ldexp(oracle_e4m3_decode(q8r[h * D + d]), (int)qsr[h * nb + d / MX_BLOCK] - 127);
            double kv = ldexp(oracle_e4m3_decode(kr[d]), (int)ks[d / MX_BLOCK] - 127);
            dot += qv * kv;
        }
        s += (double)wr[h] * (dot > 0.0 ? dot : 0.0);
    }
    return s;
}

/* Top-k of the MXFP8 score for listed queries given by their own rows:
 * q8_rows [n,H,D], qs_rows [n,H,D/32], w_rows [n,H]; k8 [B,T,D], ks [B,T,D/32].
 * Same order and padding as oracle_indexer_topk_rows. */
int oracle_indexer_topk_mxfp8_rows(const uint8_t* q8_rows, const uint8_t* qs_rows,
                                   const float* w_rows, const uint8_t* k8, const uint8_t* ks,
                                   int B, int S, int H, int D, int m, int k, const int64_t* rows,
                                   int n, int32_t* out_idx, double* out_score) {
    if (B < 1 || S < 1 || H < 1 || D < MX_BLOCK || D % MX_BLOCK != 0 || m < 1 || k < 1 ||
        S % m != 0)
        return -1;
    int T = S / m, nb = D / MX_BLOCK;
    for (int i = 0; i < n; i++)
        if (rows[i] < 0 || rows[i] >= (int64_t)B * S) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        int64_t b = rows[i] / S;
        int t = (int)(rows[i] % S);
        int V = oracle_visible(t, T, m);
        pair_t* p = (pair_t*)malloc(sizeof(pair_t) * (size_t)(V > 0 ? V : 1));
        for (int j = 0; j < V; j++) {
            p[j].s = oracle_score_row_mxfp8(q8_rows + (int64_t)i * H * D,
                                            qs_rows + (int64_t)i * H * nb, w_rows + (int64_t)i * H,
                                            k8 + b * T * (int64_t)D, ks + b * T * (int64_t)nb, H,
                                            D, j);
            p[j].j = j;
        }
        qsort(p, (size_t)V, sizeof(pair_t), cmp_pair);
        for (int r = 0; r < k; r++) {
            out_idx[(int64_t)i * k + r] = r < V ? p[r].j : -1;
            out_score[(int64_t)i * k + r] = r < V ? p[r].s : -INFINITY;
        }
        free(p);
    }
    return 0;
}

/* ------------------------------------------------------------ sparse attention
 * The consumer of the indexer's rows ("StreamIndex: Memory-Bounded Compressed
 * Sparse Attention via Streaming Top-k", Abstract: the top-k keys are kept per
 * query and a sparse attention kernel reads only those).  The abstract gives
 * no formula; the reading used here is multi-query attention over the listed
 * compressed entries, every query head sharing one key row and one value row
 * per entry:
 *
 *   J = the listed entries idx[r], 0 <= r < k, with 0 <= idx[r] < T
 *       (padding -1 and out-of-range entries skipped; entries count as listed)
 *   l_j(h) = scale * sum_d qa[h,d] * ka[j,d]
 *   o[h,:] = sum_{j in J} exp(l_j(h) - M) * va[j,:] / sum_{j in J} exp(l_j(h) - M),
 *            M = max_{j in J} l_j(h)                (o = 0 when J is empty)
 *
 * and, for the tolerance of a lower-precision result, the probability-
 * weighted magnitude a[h,d] = sum_j p_j(h) * |va[j,d]|.  fp64 throughout, sums
 * in ascending d and in list order.
 *
 * qa_rows [n,H,D] bf16 (row i belongs to batch batch[i]); ka, va [B,T,D]
 * bf16; idx_rows [n,k]; out, absw [n,H,D].  Returns -1 on bad sizes.
 */
int oracle_sparse_attention_rows(const uint16_t* qa_rows, const uint16_t* ka, const uint16_t* va,
                                 const int32_t* idx_rows, const int64_t* batch, int n, int B,
                                 int T, int H, int D, int k, double scale, double* out,
                                 double* absw) {
    if (n < 0 || B < 1 || T < 1 || H < 1 || D < 1 || k < 1) return -1;
    for (int i = 0; i < n; i++)
        if (batch[i] < 0 || batch[i] >= B) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n; i++) {
        const int32_t* ir = idx_rows + (int64_t)i * k;
        const uint16_t* kb = ka + batch[i] * (int64_t)T * D;
        const uint16_t* vb = va + batch[i] * (int64_t)T * D;
        double* l = (double*)malloc(sizeof(double) * (size_t)k);
        for (int h = 0; h < H; h++) {
            const uint16_t* qh = qa_rows + ((int64_t)i * H + h) * D;
            double* oh = out + ((int64_t)i * H + h) * D;
            double* ah = absw + ((int64_t)i * H + h) * D;
            for (int d = 0; d < D; d++) oh[d] = ah[d] = 0.0;
            double M = -INFINITY;
            int any = 0;
            for (int r = 0; r < k; r++) {
                const int j = ir[r];
                if (j < 0 || j >= T) continue;
                double s = 0.0;
                for (int d = 0; d < D; d++)
                    s += bf16_to_f64(qh[d]) * bf16_to_f64(kb[(int64_t)j * D + d]);
                l[r] = scale * s;
                if (!any || l[r] > M) M = l[r];
                any = 1;
            }
            if (!any) continue;
            double Z = 0.0;
            for (int r = 0; r < k; r++) {
                const int j = ir[r];
                if (j < 0 || j >= T) continue;
                Z += exp(l[r] - M);
            }
            for (int r = 0; r < k; r++) {
                const int j = ir[r];
                if (j < 0 || j >= T) continue;
                const double p = exp(l[r] - M) / Z;
                for (int d = 0; d < D; d++) {
                    const double v = bf16_to_f64(vb[(int64_t)j * D + d]);
                    oh[d] += p * v;
                    ah[d] += p * fabs(v);
                }
            }
        }
        free(l);
    }
    return 0;
}
