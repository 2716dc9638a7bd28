/*
 * llmint8_oracle.c -- plain CPU definition of the LLM.int8() mixed-precision
 * decomposition matmul  Y = X . W.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing here is on the product path: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load this file's
 * library.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (page title, section):
 *  [P1] "LLM.int8(): 8-bit Matrix Multiplication for Transformers at Scale",
 *       arXiv abstract: vector-wise quantization with a separate normalization
 *       constant per inner product; outlier feature dimensions isolated into a
 *       16-bit matmul while >99.9 % of values are multiplied in 8-bit.
 *  [P2] "8-bit Matrix Multiplication for Large Language Models", Summary &
 *       Methodology Analysis: the int8 result is dequantized by the outer
 *       product of row and column normalization constants and both parts are
 *       accumulated into 16-bit floating-point outputs.
 *  [P3] "Compress your LLMs", bullet "Vector-wise quantization": one constant
 *       per row of the input matrix X, one per column of the weight matrix W;
 *       bullet "Mixed-precision decomposition": 16-bit matmul for the outlier
 *       feature dimensions, 8-bit for the rest.
 *  [P4] "What is 8-bit LLM quantization?", How does INT8 quantization work?:
 *       a value is mapped to round(value / step) and recovered as q * step.
 *
 * Readings where the pages leave a step open (all stated in the design notes):
 *  - outlier column k: some |X[i,k]| >= tau over all rows of the call;
 *  - scale s = absmax of the vector (fp16 value held exactly in a float),
 *    step = s/127, q = round-half-away-from-zero(127 x / s) in [-127,127];
 *  - the row absmax excludes outlier columns; outlier columns of Xq are zero;
 *  - the weight column absmax runs over all K rows;
 *  - Y = fp16_RNE(acc * rs * cs / 127^2 + sum over outliers of x*w), in double.
 *
 * Arithmetic notes.  The quantizer takes its decision in binary32: 127*x is
 * exact (11-bit x 7-bit significands) and the division is one correctly
 * rounded IEEE operation; roundf() rounds halves away from zero.  Build with
 * -fno-fast-math -ffp-contract=off on a target without excess precision.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* IEEE binary16 codec, written from the format's definition.          */
/* ------------------------------------------------------------------ */

/* Exact value of an fp16 bit pattern: (-1)^s * 2^(e-15) * 1.m, or
 * 2^-14 * 0.m for e == 0; e == 31 encodes Inf/NaN. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24);
    } else if (e == 31) {
        v = (m == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + m), e - 25);
    }
    return sign ? -v : v;
}

/* Round a double to the nearest fp16, ties to the even significand. */
uint16_t oracle_double_to_half(double v)
{
    if (isnan(v))
        return 0x7e00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    /* 65504 is the largest finite fp16 and 65536 the next power of two; the
     * midpoint 65520 and anything above rounds to infinity. */
    if (a >= 65520.0)
        return sign | 0x7c00;
    int exp2;
    if (a < ldexp(1.0, -14)) {
        exp2 = -24; /* subnormal range: units of 2^-24 */
    } else {
        int e;
        frexp(a, &e);        /* a = f * 2^e, f in [0.5, 1) */
        exp2 = (e - 1) - 10; /* 11 significant bits: units of 2^(E-10) */
    }
    double scaled = ldexp(a, -exp2); /* exact: power-of-two scaling */
    double r = floor(scaled);
    double frac = scaled - r;        /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    /* r * 2^exp2 is the rounded magnitude; re-encode it. */
    uint32_t n = (uint32_t)r;
    if (exp2 == -24) {
        /* n in [0, 1024]; 1024 is exactly the smallest normal 0x0400 */
        return sign | (uint16_t)n;
    }
    int E = exp2 + 10; /* unbiased exponent of the leading bit */
    if (n == 2048) {   /* rounding carried into the next binade */
        n = 1024;
        E += 1;
    }
    if (E > 15)
        return sign | 0x7c00;
    return sign | (uint16_t)(((E + 15) << 10) | (n - 1024));
}

void oracle_half_to_double_array(const uint16_t* h, int64_t n, double* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_half_to_double(h[i]);
}

void oracle_double_to_half_array(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_double_to_half(v[i]);
}

static float half_to_float(uint16_t h) { return (float)oracle_half_to_double(h); }

/* ------------------------------------------------------------------ */
/* Scalar absmax quantizer [P4], scale convention of [P1]/[P3].        */
/* ------------------------------------------------------------------ */

/* q = round-half-away-from-zero(127 * x / s), with s the vector's absmax.
 * s == 0 means the whole vector is zero: q = 0 and no division happens. */
int8_t oracle_quantize_value(float x, float s)
{
    if (s == 0.0f || isnan(x))
        return 0;
    float r = (127.0f * x) / s;
    float q = roundf(r);
    if (q > 127.0f)
        q = 127.0f; /* unreachable for |x| <= s; kept as a guard */
    if (q < -127.0f)
        q = -127.0f;
    return (int8_t)q;
}

/* ------------------------------------------------------------------ */
/* a1: outlier feature dimensions [P1], [P2], [P3].                    */
/* ------------------------------------------------------------------ */

/* O = ascending list of columns k with |X[i,k]| >= tau for some row i.
 * X is fp16 [M, K] with row stride ldx.  Returns n_o. */
int64_t oracle_outlier_columns(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, float tau,
                               int32_t* O)
{
    int64_t n_o = 0;
    for (int64_t k = 0; k < K; ++k) {
        int is_outlier = 0;
        for (int64_t i = 0; i < M; ++i) {
            double a = fabs(oracle_half_to_double(X[i * ldx + k]));
            if (a >= (double)tau) {
                is_outlier = 1;
                break;
            }
        }
        if (is_outlier)
            O[n_o++] = (int32_t)k;
    }
    return n_o;
}

static unsigned char* outlier_mask(int64_t K, const int32_t* O, int64_t n_o)
{
    unsigned char* mask = (unsigned char*)calloc((size_t)(K > 0 ? K : 1), 1);
    for (int64_t t = 0; t < n_o; ++t)
        mask[O[t]] = 1;
    return mask;
}

/* ------------------------------------------------------------------ */
/* a2: row scales of X over the non-outlier columns [P3].              */
/* ------------------------------------------------------------------ */

void oracle_row_scales(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, const int32_t* O,
                       int64_t n_o, float* rs)
{
    unsigned char* mask = outlier_mask(K, O, n_o);
    for (int64_t i = 0; i < M; ++i) {
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            if (mask[k])
                continue;
            float a = fabsf(half_to_float(X[i * ldx + k]));
            if (a > m)
                m = a;
        }
        rs[i] = m;
    }
    free(mask);
}

/* ------------------------------------------------------------------ */
/* a3: row-wise int8 quantization of X; outlier columns are zero.      */
/* ------------------------------------------------------------------ */

void oracle_quantize_rows(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, const int32_t* O,
                          int64_t n_o, const float* rs, int8_t* Xq)
{
    unsigned char* mask = outlier_mask(K, O, n_o);
    for (int64_t i = 0; i < M; ++i)
        for (int64_t k = 0; k < K; ++k)
            Xq[i * K + k] = mask[k] ? 0 : oracle_quantize_value(half_to_float(X[i * ldx + k]), rs[i]);
    free(mask);
}

/* ------------------------------------------------------------------ */
/* a0: column-wise int8 quantization of W [P3] (all K rows).           */
/* ------------------------------------------------------------------ */

void oracle_col_scales(const uint16_t* W, int64_t K, int64_t N, float* cs)
{
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        float m = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(half_to_float(W[k * N + j]));
            if (a > m)
                m = a;
        }
        cs[j] = m;
    }
}

/* Wq has W's layout: [K, N] row-major. */
void oracle_quantize_cols(const uint16_t* W, int64_t K, int64_t N, const float* cs, int8_t* Wq)
{
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j)
            Wq[k * N + j] = oracle_quantize_value(half_to_float(W[k * N + j]), cs[j]);
}

/* ------------------------------------------------------------------ */
/* a4: gather of the outlier columns of X and outlier rows of W.       */
/* ------------------------------------------------------------------ */

void oracle_gather_outliers(const uint16_t* X, int64_t M, int64_t ldx, const int32_t* O, int64_t n_o,
                            uint16_t* Xo /* [M, n_o] */, const uint16_t* W, int64_t N,
                            uint16_t* Wo /* [n_o, N], may be NULL */)
{
    for (int64_t i = 0; i < M; ++i)
        for (int64_t t = 0; t < n_o; ++t)
            Xo[i * n_o + t] = X[i * ldx + O[t]];
    if (Wo)
        for (int64_t t = 0; t < n_o; ++t)
            memcpy(Wo + t * N, W + (int64_t)O[t] * N, (size_t)N * sizeof(uint16_t));
}

/* ------------------------------------------------------------------ */
/* a5: int8 x int8 -> integer matmul, accumulated in int64.            */
/* ------------------------------------------------------------------ */

/* acc[r, j] = sum_k Xq[rows[r], k] * Wq[k, j] for r < n_rows.
 * rows == NULL means rows 0..n_rows-1.  Integer sums are exact, so the
 * loop order does not change the result. */
void oracle_int8_matmul(const int8_t* Xq, const int8_t* Wq, int64_t N, int64_t K, const int64_t* rows,
                        int64_t n_rows, int64_t* acc)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        int64_t* out = acc + r * N;
        for (int64_t j = 0; j < N; ++j)
            out[j] = 0;
        for (int64_t k = 0; k < K; ++k) {
            int64_t a = Xq[i * K + k];
            const int8_t* w = Wq + k * N;
            for (int64_t j = 0; j < N; ++j)
                out[j] += a * (int64_t)w[j];
        }
    }
}

/* ------------------------------------------------------------------ */
/* a6 + a7: dequantize by the outer product of scales [P2], add the     */
/* 16-bit product of the outlier dimensions [P1], round to fp16.       */
/* ------------------------------------------------------------------ */

/* For each selected row i = rows[r]:
 *   Yd[r,j] = acc[r,j] * rs[i] * cs[j] / 127^2 + sum_t X[i,O[t]] * W[O[t],j] (+ b[j])
 *   Y[r,j]  = fp16_RNE(Yd[r,j])
 * evaluated in double, outlier terms added in ascending column order.  The
 * optional bias b (fp16 [N], NULL for none) is the linear layer's: a layer's
 * output is X W + b ("LLM.int8()" arXiv abstract: the method replaces the
 * feed-forward and attention projection layers), added last. */
void oracle_mixed_output(const int64_t* acc, const float* rs, const float* cs, const uint16_t* X,
                         int64_t ldx, const uint16_t* W, int64_t N, const int32_t* O, int64_t n_o,
                         const uint16_t* bias, const int64_t* rows, int64_t n_rows, double* Yd, uint16_t* Y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t i = rows ? rows[r] : r;
        double* yd = Yd + r * N;
        for (int64_t j = 0; j < N; ++j)
            yd[j] = (double)acc[r * N + j] * (double)rs[i] * (double)cs[j] / 16129.0;
        for (int64_t t = 0; t < n_o; ++t) {
            double x = oracle_half_to_double(X[i * ldx + O[t]]);
            const uint16_t* w = W + (int64_t)O[t] * N;
            for (int64_t j = 0; j < N; ++j)
                yd[j] += x * oracle_half_to_double(w[j]);
        }
        if (bias)
            for (int64_t j = 0; j < N; ++j)
                yd[j] += oracle_half_to_double(bias[j]);
        for (int64_t j = 0; j < N; ++j)
            Y[r * N + j] = oracle_double_to_half(yd[j]);
    }
}

/* ------------------------------------------------------------------ */
/* Outlier statistics of an activation: how many values reach the         */
/* threshold, in how many feature dimensions (columns) and in how many    */
/* rows -- the quantities the pages report ("8-bit Matrix Multiplication  */
/* for Large Language Models", Summary & Methodology Analysis: at 6.7B,   */
/* 150,000 outliers per sequence, in 6 feature dimensions).               */
/* ------------------------------------------------------------------ */

/* out[0] = #{(i,k) : |X[i,k]| >= tau}, out[1] = #{k : some |X[i,k]| >= tau},
 * out[2] = #{i : some |X[i,k]| >= tau}; NaN never counts. */
void oracle_outlier_stats(const uint16_t* X, int64_t M, int64_t K, int64_t ldx, float tau, int64_t* out)
{
    unsigned char* col = (unsigned char*)calloc((size_t)(K > 0 ? K : 1), 1);
    int64_t values = 0, rows = 0, cols = 0;
    for (int64_t i = 0; i < M; ++i) {
        int any = 0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs(oracle_half_to_double(X[i * ldx + k]));
            if ((double)tau <= a) {  /* false for NaN */
                ++values;
                any = 1;
                col[k] = 1;
            }
        }
        rows += any;
    }
    for (int64_t k = 0; k < K; ++k)
        cols += col[k];
    free(col);
    out[0] = values;
    out[1] = cols;
    out[2] = rows;
}

/* ------------------------------------------------------------------ */
/* The 16-bit weight rows recovered from the int8 weight, for callers     */
/* that keep only the int8 form: the point of the method is halving the   */
/* weight memory ("LLM.int8()" arXiv abstract: inference memory cut by    */
/* half; "What is 8-bit LLM quantization?", How much memory can it save:  */
/* 14 GB of fp16 weights become 7 GB of int8).  Each value is the         */
/* column's dequantized code, Wq * cs / 127, rounded once to fp16.        */
/* ------------------------------------------------------------------ */

/* Wd[k,j] = fp16_RNE(Wq[k,j] * cs[j] / 127), evaluated in double. */
void oracle_dequantize_weight(const int8_t* Wq, int64_t K, int64_t N, const float* cs, uint16_t* Wd)
{
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j)
            Wd[k * N + j] = oracle_double_to_half((double)Wq[k * N + j] * (double)cs[j] / 127.0);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
