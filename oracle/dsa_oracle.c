/*
 * Float64 CPU oracle for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The CUDA library never
 * links, loads or calls it, and this file includes nothing from the CUDA
 * sources: it has its own e4m3 and bf16 decoders and its own loops.
 *
 * Everything is the plain definition, evaluated in double precision, one query
 * row at a time (OpenMP over rows only; no blocking, no fusion, no reordering
 * of a sum beyond its natural index order):
 *
 *   1. Dequantise ("Lightning Indexer 的计算过程", step 2 <2>, FP8 量化, on
 *      adg.csdn.net/695234...): q[t,j,i] = e4m3(q8[t,j,i]) * q_scale[t],
 *      k[s,i] = e4m3(k8[s,i]) * k_scale[s].
 *   2. Index score (same page, step 3 <1>-<2>: dot product, ReLU, head-weighted
 *      sum; "DeepSeek-V3.2-Exp解析", dtcms.com, section 一.1):
 *      I[t,s] = sum_j w[t,j] * max(0, sum_i q[t,j,i] * k[s,i]),  s <= t.
 *      No 1/sqrt(d) factor.
 *   3. Selection (same page, step 4 <1>; deepseek.csdn.net section 2.2 细粒度
 *      词元选择): the first min(k, t+1) elements of {0..t} ordered by
 *      (I descending, s ascending); the rest of the row is -1.
 *   4. Sparse MQA over the MLA latent (deepseek.csdn.net section 2.2; the
 *      576-value latent row, yudonglee.me "DeepSeek-V3.2 explained" section 2.4):
 *      z_s = scale * sum_{i<576} Q[t,h,i] * C[s,i] for the selected s,
 *      p_s = exp(z_s - max z) / sum exp(.), u[t,h,:] = sum_s p_s * C[s, 0:512].
 *
 * The causal bound is s <= t (a token scores itself), and rows with fewer than
 * k candidates select all of them.
 *
 * For quantising newly appended tokens on the device ("Lightning Indexer 的计算
 * 过程", step 2 <2>, FP8 量化): per row, scale = absmax/448 in fp32 (1 for an
 * all-zero row) and codes = E4M3(x/scale) by round-to-nearest-even with
 * saturation to +-448 (oracle_double_to_e4m3, oracle_quantize_e4m3).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* OCP 8-bit floating point, E4M3 ("fn" flavour: no infinities, S.1111.111 is
 * NaN). Exponent bias 7, 3 mantissa bits, subnormals below exponent field 1. */
double oracle_e4m3_to_double(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Step 1 and 2 for a list of queries.
 *   q8      [nrows, H, D] e4m3      q_scale [nrows]
 *   w       [nrows, H] f32
 *   k8      [S, D] e4m3             k_scale [S]
 *   rows    [nrows] causal position t of each query (each < S)
 *   out     [nrows, S] f64: I[t,s] for s <= t, -INFINITY for s > t.
 */
/* E4M3 encoding of a finite value by the plain definition: round to the
 * nearest representable value, ties to the even code, saturating to +-448.
 * The representable magnitudes are m * 2^-9 (m = 0..7, subnormal) and
 * (1 + m/8) * 2^e (e = -6..8, m = 0..7, at most 448 = 1.75 * 2^8). NaN maps to
 * the NaN code 0x7F (sign kept). */
uint8_t oracle_double_to_e4m3(double x) {
    uint8_t sign = (x < 0.0 || (x == 0.0 && signbit(x))) ? 0x80 : 0x00;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    double a = fabs(x);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    /* candidates on the grid of the binade of a (or the subnormal grid) */
    double step;
    if (a < ldexp(1.0, -6)) {
        step = ldexp(1.0, -9);
    } else {
        int e;
        frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): binade [2^(e-1), 2^e) */
        step = ldexp(1.0, e - 1 - 3);
    }
    double q = a / step; /* exact: step is a power of two */
    double lo = floor(q);
    double frac = q - lo;
    double n = lo;
    if (frac > 0.5 || (frac == 0.5 && fmod(lo, 2.0) != 0.0)) n = lo + 1.0;
    double v = n * step; /* the rounded magnitude (may be the next binade's first value) */
    if (v > 448.0) v = 448.0;
    /* encode v exactly */
    if (v < ldexp(1.0, -6)) return (uint8_t)(sign | (uint8_t)(v / ldexp(1.0, -9)));
    int e;
    double f = frexp(v, &e); /* v = f * 2^e, f in [0.5, 1) */
    int m = (int)((f * 2.0 - 1.0) * 8.0);
    int ef = e - 1 + 7;
    return (uint8_t)(sign | (uint8_t)(ef << 3) | (uint8_t)m);
}

/* Per-row FP8 quantiser for newly appended keys / queries: scale = absmax/448
 * (1 for an all-zero row) in fp32, codes = e4m3(fp32(x / scale)) clamped to
 * +-448. The division is the float32 one the quantised caches are defined
 * with; the encoding is oracle_double_to_e4m3. */
void oracle_quantize_e4m3(const float *x, int64_t n, int64_t d, uint8_t *codes, float *scale) {
    for (int64_t r = 0; r < n; ++r) {
        float amax = 0.0f;
        for (int64_t i = 0; i < d; ++i) {
            float v = fabsf(x[r * d + i]);
            if (v > amax) amax = v;
        }
        float sc = (amax > 0.0f) ? amax / 448.0f : 1.0f;
        scale[r] = sc;
        for (int64_t i = 0; i < d; ++i) {
            float y = x[r * d + i] / sc;
            if (y > 448.0f) y = 448.0f;
            if (y < -448.0f) y = -448.0f;
            codes[r * d + i] = oracle_double_to_e4m3((double)y);
        }
    }
}

void oracle_index_scores(const uint8_t *q8, const float *q_scale, const float *w,
                         const uint8_t *k8, const float *k_scale, int64_t S, int H, int D,
                         const int64_t *rows, int64_t nrows, double *out) {
    double *k = (double *)malloc(sizeof(double) * (size_t)S * (size_t)D);
    for (int64_t s = 0; s < S; ++s)
        for (int i = 0; i < D; ++i)
            k[s * D + i] = oracle_e4m3_to_double(k8[s * D + i]) * (double)k_scale[s];

#pragma omp parallel
    {
        double *q = (double *)malloc(sizeof(double) * (size_t)H * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = rows[r];
            double *o = out + r * S;
            for (int j = 0; j < H; ++j)
                for (int i = 0; i < D; ++i)
                    q[j * D + i] = oracle_e4m3_to_double(q8[(r * H + j) * D + i]) * (double)q_scale[r];
            for (int64_t s = 0; s < S; ++s) {
                if (s > t) { o[s] = -INFINITY; continue; }
                double I = 0.0;
                for (int j = 0; j < H; ++j) {
                    double dot = 0.0;
                    for (int i = 0; i < D; ++i) dot += q[j * D + i] * k[s * D + i];
                    I += (double)w[r * H + j] * (dot > 0.0 ? dot : 0.0);
                }
                o[s] = I;
            }
        }
        free(q);
    }
    free(k);
}

/* Ordering of step 3: a before b when I_a > I_b, or I_a == I_b and s_a < s_b. */
typedef struct { double v; int64_t s; } oracle_scored;

static int oracle_rank_cmp(const void *pa, const void *pb) {
    const oracle_scored *a = (const oracle_scored *)pa, *b = (const oracle_scored *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->s < b->s) ? -1 : (a->s > b->s) ? 1 : 0;
}

/*
 * Step 3 for rows whose scores are given (any source: the oracle's own, or a
 * caller's fp32 scores widened to f64).
 *   scores [nrows, S] f64 (only entries s <= rows[r] are read)
 *   idx    [nrows, k] int32, ranked order, -1 beyond min(k, t+1).
 */
void oracle_topk(const double *scores, int64_t S, const int64_t *rows, int64_t nrows, int k,
                 int32_t *idx) {
#pragma omp parallel
    {
        oracle_scored *buf = (oracle_scored *)malloc(sizeof(oracle_scored) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t t = rows[r];
            int64_t n = t + 1;
            for (int64_t s = 0; s < n; ++s) { buf[s].v = scores[r * S + s]; buf[s].s = s; }
            qsort(buf, (size_t)n, sizeof(oracle_scored), oracle_rank_cmp);
            for (int i = 0; i < k; ++i) idx[r * k + i] = (i < n) ? (int32_t)buf[i].s : -1;
        }
        free(buf);
    }
}

/*
 * Step 4 for a list of queries and their selections.
 *   q    [nrows, Hq, Dqk] bf16 bits     kv [S, Dqk] bf16 bits
 *   idx  [nrows, k] int32 rows of kv (entries < 0 are skipped)
 *   out  [nrows, Hq, Dv] f64; lse [nrows, Hq] f64 (natural log of sum exp(z)),
 *   lse may be NULL. A row with no valid entry yields zeros and lse = -inf.
 */
void oracle_sparse_mla(const uint16_t *q, const uint16_t *kv, const int32_t *idx, int k,
                       int64_t nrows, int Hq, int Dqk, int Dv, double scale,
                       double *out, double *lse) {
#pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        double *qh = (double *)malloc(sizeof(double) * (size_t)Dqk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int32_t *sel = idx + r * k;
            for (int h = 0; h < Hq; ++h) {
                double *u = out + (r * Hq + h) * Dv;
                for (int i = 0; i < Dqk; ++i) qh[i] = oracle_bf16_to_double(q[(r * Hq + h) * Dqk + i]);
                double zmax = -INFINITY;
                for (int e = 0; e < k; ++e) {
                    if (sel[e] < 0) continue;
                    const uint16_t *c = kv + (int64_t)sel[e] * Dqk;
                    double dot = 0.0;
                    for (int i = 0; i < Dqk; ++i) dot += qh[i] * oracle_bf16_to_double(c[i]);
                    z[e] = scale * dot;
                    if (z[e] > zmax) zmax = z[e];
                }
                for (int d = 0; d < Dv; ++d) u[d] = 0.0;
                double denom = 0.0;
                for (int e = 0; e < k; ++e) {
                    if (sel[e] < 0) continue;
                    double p = exp(z[e] - zmax);
                    denom += p;
                    const uint16_t *c = kv + (int64_t)sel[e] * Dqk;
                    for (int d = 0; d < Dv; ++d) u[d] += p * oracle_bf16_to_double(c[d]);
                }
                if (denom > 0.0)
                    for (int d = 0; d < Dv; ++d) u[d] /= denom;
                if (lse) lse[r * Hq + h] = (denom > 0.0) ? zmax + log(denom) : -INFINITY;
            }
        }
        free(z);
        free(qh);
    }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
