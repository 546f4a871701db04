/*
 * CPU oracle for the LLM.int8() mixed-precision decomposed matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * It is plain and slow on purpose: every step is the definition written out,
 * in the order the pages give it, with no blocking, fusion or reordering
 * beyond a loop order over independent output elements.  Rows are spread
 * over host threads with OpenMP where they are independent.
 *
 * Sources (web pages about "LLM.int8(): 8-bit Matrix Multiplication for
 * Transformers at Scale", Dettmers et al., 2022):
 *  [estelledc] "LLM.int8() — 大模型激活值里藏着几个超大异常通道",
 *              sections 方法1 (vector-wise quantization) and 方法2
 *              (mixed-precision decomposition), 案例1 (worked example).
 *  [aliyun]    "AI 十大核心论文解读: LLM.int8()", §2.2 and the Fig. 2 caption.
 *  [gartu]     "LLM.int8()" (brain.gartu.xyz), sections "La solution",
 *              "Seuil de détection α" and "Vector-wise INT8 Quantization".
 *
 * Readings where the pages leave a detail open (each is also a test):
 *  - outlier test is strict: column j is an outlier iff max_i |X[i,j]| > α
 *    ([estelledc] 方法2; [gartu] "Seuil de détection α").
 *  - scale c = 127 / absmax as an IEEE fp32 division, codes are
 *    clamp(rne(x * c), -127, 127) with the product rounded to fp32 first and
 *    ties going to even; an all-zero vector gets c = 0 and all codes 0.
 *  - a row of X is scaled over its non-outlier columns only (the Fig. 2
 *    caption of [aliyun] splits first, then scales); outlier columns get code 0.
 *  - a column of W is scaled over all K rows: W is prepared once, before the
 *    outlier set of any input is known.  Its outlier rows multiply code 0.
 *  - dequantisation is acc / (c_x[i] * c_w[j]) ([estelledc] 方法1), here in
 *    double; the fp16 outlier product is accumulated in double in ascending
 *    column order; the sum is rounded once to fp16, ties to even.
 *  - memory-saving weight: the fp16 rows of W are kept for a fixed set of
 *    input dimensions only ([estelledc]: the outliers sit in a few fixed
 *    feature dimensions; 方法2: only those go through fp16).  The pages leave
 *    open what an outlier column outside the set uses: here its row is
 *    rebuilt from the codes, w = q * (1/c_w) in fp32, rounded to fp16.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * Floating point is IEEE binary32/binary64 with SSE arithmetic (no x87
 * excess precision, no contraction into FMA).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#if defined(_OPENMP)
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16, written out from the format definition:                */
/* 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.                 */

double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);              /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);  /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a double to the nearest binary16, ties to even; overflow to +-inf. */
uint16_t orc_double_to_half(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00);
    /* 65504 is the largest finite value; 65520 is the midpoint to 2^16,
     * which ties to the even neighbour, i.e. to infinity. */
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00);
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: integer multiple of 2^-24.  A result of 1024
         * is the smallest normal number, whose encoding is also 1024. */
        double m = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)m);
    }
    int E;
    frexp(a, &E);               /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;              /* a in [2^e, 2^(e+1)) */
    double m = nearbyint(ldexp(a, 10 - e));   /* in [1024, 2048] */
    if (m == 2048.0) { m = 1024.0; e += 1; }
    /* a < 65520 keeps e <= 15 here */
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)m - 1024));
}

void orc_half_to_double_array(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_half_to_double(h[i]);
}

void orc_double_to_half_array(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_double_to_half(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Vector-wise quantisation of one value with scale c ([estelledc] 方法1).   */

float orc_scale_from_absmax(float absmax)
{
    if (absmax == 0.0f) return 0.0f;      /* all-zero vector: no 0/0 */
    return 127.0f / absmax;               /* IEEE fp32 division */
}

int8_t orc_quantize_value(float x, float c)
{
    float p = x * c;                      /* fp32 product, rounded once */
    float r = nearbyintf(p);              /* ties to even (default mode) */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* ------------------------------------------------------------------------ */
/* Step 1 — outlier feature detection ([estelledc] 方法2; [gartu] Seuil α):  */
/* column j of X is an outlier iff max_i |X[i,j]| > alpha.                   */
/* Writes colmax[K] (fp32, exact) and the ascending outlier list idx.       */
/* Returns |O|.                                                              */
int64_t orc_outlier_columns(const uint16_t *X, int64_t M, int64_t K, float alpha,
                            float *colmax, int32_t *idx)
{
    for (int64_t j = 0; j < K; ++j) colmax[j] = 0.0f;
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < K; ++j) {
            float a = (float)fabs(orc_half_to_double(X[i * K + j]));
            if (a > colmax[j]) colmax[j] = a;
        }
    int64_t n = 0;
    for (int64_t j = 0; j < K; ++j)
        if (colmax[j] > alpha) idx[n++] = (int32_t)j;
    return n;
}

/* Step 2a — quantise each row of X over its non-outlier columns            */
/* ([estelledc] 方法1: one constant c_x[i] per row; [aliyun] Fig. 2: the     */
/* outlier columns are split off before scaling).  Outlier columns get 0.   */
void orc_quantize_rows(const uint16_t *X, int64_t M, int64_t K,
                       const int32_t *idx, int64_t n_out,
                       int8_t *q, float *c)
{
    unsigned char *is_out = (unsigned char *)calloc((size_t)K, 1);
    for (int64_t o = 0; o < n_out; ++o) is_out[idx[o]] = 1;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        float amax = 0.0f;
        for (int64_t j = 0; j < K; ++j) {
            if (is_out[j]) continue;
            float a = (float)fabs(orc_half_to_double(X[i * K + j]));
            if (a > amax) amax = a;
        }
        float ci = orc_scale_from_absmax(amax);
        c[i] = ci;
        for (int64_t j = 0; j < K; ++j) {
            float x = (float)orc_half_to_double(X[i * K + j]);
            q[i * K + j] = is_out[j] ? 0 : orc_quantize_value(x, ci);
        }
    }
    free(is_out);
}

/* Step 2b — quantise each column of W over all K rows ([estelledc] 方法1:   */
/* one constant c_w[j] per column).  q has W's layout, [K, N].              */
void orc_quantize_cols(const uint16_t *W, int64_t K, int64_t N, int8_t *q, float *c)
{
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = (float)fabs(orc_half_to_double(W[k * N + j]));
            if (a > amax) amax = a;
        }
        c[j] = orc_scale_from_absmax(amax);
    }
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j) {
            float w = (float)orc_half_to_double(W[k * N + j]);
            q[k * N + j] = orc_quantize_value(w, c[j]);
        }
}

/* Memory-saving weight, rows outside the stored set: the weight row rebuilt */
/* from its codes (the reading in the header: the pages leave it open).     */
/* out[k,j] = binary16(rne(float(q[k,j]) * (1/c_w[j]))), the reciprocal an */
/* fp32 division rounded once, 0 for an all-zero column (c_w = 0).          */
void orc_rebuild_weight_rows(const int8_t *q, const float *c, int64_t K, int64_t N, uint16_t *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k) {
        for (int64_t j = 0; j < N; ++j) {
            float inv = (c[j] == 0.0f) ? 0.0f : 1.0f / c[j];
            float w = (float)q[k * N + j] * inv;
            out[k * N + j] = orc_double_to_half((double)w);
        }
    }
}

/* Step 3 — int8 x int8 -> int32 contraction ([aliyun] Fig. 2: Out_i32).    */
/* acc[i,j] = sum_k qx[i,k] * qw[k,j], summed in int64 and checked to fit   */
/* int32.  Returns 0, or -1 if some sum does not fit.                       */
int orc_int8_matmul(const int8_t *qx, const int8_t *qw, int64_t M, int64_t K, int64_t N,
                    int32_t *acc)
{
    int bad = 0;
    #pragma omp parallel
    {
        int64_t *row = (int64_t *)malloc((size_t)N * sizeof(int64_t));
        #pragma omp for schedule(dynamic, 1) reduction(|:bad)
        for (int64_t i = 0; i < M; ++i) {
            for (int64_t j = 0; j < N; ++j) row[j] = 0;
            for (int64_t k = 0; k < K; ++k) {
                int64_t a = qx[i * K + k];
                const int8_t *wk = qw + k * N;
                for (int64_t j = 0; j < N; ++j) row[j] += a * (int64_t)wk[j];
            }
            for (int64_t j = 0; j < N; ++j) {
                if (row[j] > INT32_MAX || row[j] < INT32_MIN) bad = 1;
                acc[i * N + j] = (int32_t)row[j];
            }
        }
        free(row);
    }
    return bad ? -1 : 0;
}

/* Steps 4 and 5 — dequantise by the outer product of the scales and add   */
/* the fp16 outlier product ([estelledc] 方法1/方法2; [gartu] La solution):  */
/*   y[i,j] = acc[i,j] / (c_x[i] * c_w[j]) + sum_{k in O} X[i,k] * W[k,j]    */
/* in double, rounded once to fp16.  A zero scale means a zero int8 term.   */
/* bias (optional, fp16 [N]) is the layer's bias b[j] ([gartu] Exemple      */
/* pratique: the int8 layer that replaces nn.Linear keeps bias=True), added */
/* to the double sum before the rounding.                                   */
/* Y_exact (optional) receives the unrounded double.                         */
void orc_dequant_add_outliers(const int32_t *acc, const float *cx, const float *cw,
                              const uint16_t *X, const uint16_t *W,
                              int64_t M, int64_t K, int64_t N,
                              const int32_t *idx, int64_t n_out,
                              const uint16_t *bias,
                              uint16_t *Y, double *Y_exact)
{
    #pragma omp parallel
    {
        double *row = (double *)malloc((size_t)N * sizeof(double));
        #pragma omp for schedule(static)
        for (int64_t i = 0; i < M; ++i) {
            for (int64_t j = 0; j < N; ++j) {
                double s = (double)cx[i] * (double)cw[j];
                row[j] = (s == 0.0) ? 0.0 : (double)acc[i * N + j] / s;
            }
            for (int64_t o = 0; o < n_out; ++o) {
                int64_t k = idx[o];
                double x = orc_half_to_double(X[i * K + k]);
                for (int64_t j = 0; j < N; ++j)
                    row[j] += x * orc_half_to_double(W[k * N + j]);
            }
            if (bias)  /* the layer's bias, added before the one rounding */
                for (int64_t j = 0; j < N; ++j) row[j] += orc_half_to_double(bias[j]);
            for (int64_t j = 0; j < N; ++j) {
                Y[i * N + j] = orc_double_to_half(row[j]);
                if (Y_exact) Y_exact[i * N + j] = row[j];
            }
        }
        free(row);
    }
}

/* ------------------------------------------------------------------------ */
/* Comparators.                                                              */

/* Exact-as-double matmul of the fp16 inputs: y[i,j] = sum_k x[i,k] w[k,j]. */
void orc_matmul_f64(const uint16_t *X, const uint16_t *W, int64_t M, int64_t K, int64_t N,
                    double *Y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double *y = Y + i * N;
        for (int64_t j = 0; j < N; ++j) y[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double x = orc_half_to_double(X[i * K + k]);
            for (int64_t j = 0; j < N; ++j)
                y[j] += x * orc_half_to_double(W[k * N + j]);
        }
    }
}

/* Tensor-wise absmax int8 ([estelledc] 案例1 and 案例2's "8-bit absmax"):   */
/* one scale 127/max|X| for all of X, one 127/max|W| for all of W, no       */
/* decomposition.  Writes the codes, both scales and the fp16 result.       */
int orc_tensorwise_absmax(const uint16_t *X, const uint16_t *W,
                          int64_t M, int64_t K, int64_t N,
                          int8_t *qx, int8_t *qw, float *c_x, float *c_w, uint16_t *Y)
{
    float ax = 0.0f, aw = 0.0f;
    for (int64_t t = 0; t < M * K; ++t) {
        float a = (float)fabs(orc_half_to_double(X[t]));
        if (a > ax) ax = a;
    }
    for (int64_t t = 0; t < K * N; ++t) {
        float a = (float)fabs(orc_half_to_double(W[t]));
        if (a > aw) aw = a;
    }
    float cxs = orc_scale_from_absmax(ax), cws = orc_scale_from_absmax(aw);
    *c_x = cxs;
    *c_w = cws;
    for (int64_t t = 0; t < M * K; ++t) qx[t] = orc_quantize_value((float)orc_half_to_double(X[t]), cxs);
    for (int64_t t = 0; t < K * N; ++t) qw[t] = orc_quantize_value((float)orc_half_to_double(W[t]), cws);
    int32_t *acc = (int32_t *)malloc((size_t)(M * N) * sizeof(int32_t));
    int rc = orc_int8_matmul(qx, qw, M, K, N, acc);
    double s = (double)cxs * (double)cws;
    for (int64_t t = 0; t < M * N; ++t)
        Y[t] = orc_double_to_half(s == 0.0 ? 0.0 : (double)acc[t] / s);
    free(acc);
    return rc;
}

int orc_num_threads(void)
{
#if defined(_OPENMP)
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n)
{
#if defined(_OPENMP)
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
