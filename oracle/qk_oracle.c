/*
 * qk_oracle.c -- plain CPU oracle for the W8A8 / W4A8 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct statement
 * of what the quantized linear computes.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load it.  It shares no code,
 * header, table or helper with the CUDA library: the library never links it and
 * it never includes anything from the library.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fopenmp -fPIC -shared
 * (x86-64 SSE arithmetic, so every float operation below is one IEEE binary32
 * operation in round-to-nearest-even, and no multiply-add is fused).
 *
 * Threads: the outer loop over independent rows (tokens, or output channels
 * for the weight quantization) may be split over OpenMP threads.  Each output
 * is still computed by one thread in the order written here, so the results
 * are the same bits at any thread count.  oracle_set_threads picks the count
 * (the Python loader sets 1 unless asked otherwise).
 *
 * Sources (by page and section):
 *   [qlip] "qlip-mlx" README, intro bullet "w8a8_linear / W8A8Linear":
 *          per-token activation quantization, INT8 x INT8 -> INT32 matmul,
 *          dequant + bias fused; weights quantized offline.
 *   [qlip-py] same page, "Quick start" -> "Use it from Python":
 *          quantize_weight_int8 maps an [N, K] weight to int8 codes plus fp32
 *          per-output-channel scales; w8a8_linear(x, w_i8, sw, bias).
 *   [qlip-w4] same page, intro bullet "w4a8_linear / W4A8Linear": weights as
 *          packed int4, the same INT8 compute, a GEMV for M <= 16.
 *   [mlx4722] "MLX PR #4722" (int8-staged quantized matmul), "Selector rules":
 *          affine-quantized weights, group size 64, K % 64 == 0; the
 *          "SIMD fix" bullet: x is quantized to int8 by its own kernel.
 *   [kquant89] "mlx-kquant PR #89", commit list: a quantized matmul with a
 *          gated residual epilogue, each element held within 2 ulp.
 *   [qlip-sage] "qlip-mlx" README, intro bullet "sage_attention" and the
 *          "Exact where it matters" bullet: INT8 Q K^T inside a flash-attention
 *          structure, exact online softmax, per-token / per-block scales, and
 *          softmax and P V kept in floating point; head dim 128, no mask.
 *
 * Readings taken where the pages are silent (each is stated where it is used):
 *   R1  codes are rne(x * r) with r = 127 / absmax (one fp32 division per row,
 *       one fp32 multiply per element); the scale is absmax / 127.
 *   R2  the clamp is symmetric, [-127, 127].
 *   R3  an all-zero row gets scale 1.0 and all-zero codes.
 *   R4  weights (W8) use the activation formula, per output channel.
 *   R5  W4: affine per group of 64 along K, offset = group min, scale =
 *       (max - min) / 15, both stored as fp16; codes from the fp16 values,
 *       clamp [0, 15]; a zero scale gives all-zero codes.
 *   R6  packing: code k = 2j in the low nibble of byte j, k = 2j + 1 in the high.
 *   R7  W4A8 keeps an exact int32 partial sum per group of 64 and folds the
 *       groups with the scale/offset afterwards.
 *   R13 the gated residual epilogue is out = r + g[n] * (linear output before
 *       rounding), r a bf16 [M, N] residual, g one fp32 gate per output channel
 *       (one sample's adaLN gate of a DiT block).
 *   R14 INT8 attention: q and k rows (tokens) are quantized per token by the
 *       activation rule (R1-R3); scores s[i, j] = (q_i . k_j exact) * sq[i] *
 *       sk[j] * scale; softmax over all keys (no mask); o_i = sum_j p_ij v_j
 *       (v bf16); the exact result is rounded once to bf16.  No smoothing of k.
 *   dequant is evaluated in fp64 and rounded once to bf16 (nearest, ties even).
 */
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of threads the row loops below may use; returns the count in effect
 * (1 when the library is built without OpenMP). */
int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* ---------------------------------------------------------------- encodings */

/* A bf16 is the upper 16 bits of an IEEE binary32: widening is exact. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> fp16, IEEE round-to-nearest-even (the C compiler's _Float16 cast). */
uint16_t oracle_f32_to_f16(float f)
{
    _Float16 h = (_Float16)f;
    uint16_t u;
    memcpy(&u, &h, sizeof u);
    return u;
}

float oracle_f16_to_f32(uint16_t u)
{
    _Float16 h;
    memcpy(&h, &u, sizeof h);
    return (float)h;
}

/*
 * fp64 -> bf16, round to nearest, ties to even, in one step (no intermediate
 * fp32 rounding, which could round twice).  bf16 keeps 8 significant bits and
 * the binary32 exponent range; below 2^-126 its spacing is 2^-133.  The two
 * bf16 neighbours of |v| are found in double arithmetic, where every step here
 * is exact (scaling by a power of two, floor, and differences smaller than the
 * spacing).
 */
uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80);

    int e;
    (void)frexp(a, &e);                 /* a = f * 2^e, f in [0.5, 1) */
    int qexp = (e < -125 ? -125 : e) - 8;
    double quantum = ldexp(1.0, qexp);  /* spacing of bf16 values around a */
    double units = floor(a / quantum);  /* exact: a / quantum is a power-of-two scaling */
    double lo = units * quantum;
    double hi = lo + quantum;
    double dlo = a - lo, dhi = hi - a;
    double r;
    if (dlo < dhi)
        r = lo;
    else if (dhi < dlo)
        r = hi;
    else
        r = (fmod(units, 2.0) == 0.0) ? lo : hi;   /* tie: even last bit */

    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80);           /* past the largest bf16 */
    float rf = (float)r;                            /* exact: r is a bf16 value */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}

/* ------------------------------------------------- symmetric per-row int8 */

/*
 * One row of the per-token (or per-output-channel) symmetric quantization
 * [qlip]: absmax over the row, scale = absmax / 127, codes = round-half-even
 * of x * (127 / absmax) clamped to [-127, 127] (R1, R2); a zero row gets
 * scale 1 and zero codes (R3).
 */
static void quant_row_sym(const float *v, int64_t K, int8_t *q, float *scale)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float m = fabsf(v[k]);
        if (m > amax)
            amax = m;
    }
    if (amax == 0.0f) {
        for (int64_t k = 0; k < K; ++k)
            q[k] = 0;
        *scale = 1.0f;
        return;
    }
    float s = amax / 127.0f;
    float r = 127.0f / amax;
    for (int64_t k = 0; k < K; ++k) {
        float t = v[k] * r;
        float n = nearbyintf(t);      /* current mode is round-to-nearest-even */
        if (n > 127.0f)
            n = 127.0f;
        if (n < -127.0f)
            n = -127.0f;
        q[k] = (int8_t)n;
    }
    *scale = s;
}

/* Activation quantization: x bf16 [M, K] -> xq int8 [M, K], sx fp32 [M]. */
void oracle_quant_act_bf16(const uint16_t *x, int64_t M, int64_t K,
                           int8_t *xq, float *sx)
{
#pragma omp parallel
    {
        float *row = (float *)malloc((size_t)K * sizeof(float));
#pragma omp for schedule(static)
        for (int64_t m = 0; m < M; ++m) {
            if (!row)
                continue;
            for (int64_t k = 0; k < K; ++k)
                row[k] = oracle_bf16_to_f32(x[m * K + k]);
            quant_row_sym(row, K, xq + m * K, sx + m);
        }
        free(row);
    }
}

/* W8 weight quantization (R4): W fp32 [N, K] -> Wq int8 [N, K], sw fp32 [N]. */
void oracle_quant_w8(const float *W, int64_t N, int64_t K, int8_t *Wq, float *sw)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        quant_row_sym(W + n * K, K, Wq + n * K, sw + n);
}

/* Per-group-of-64 sums of the activation codes: xsum[m, g] = sum_{k in g} xq. */
void oracle_group_sums(const int8_t *xq, int64_t M, int64_t K, int32_t *xsum)
{
    int64_t G = K / 64;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t g = 0; g < G; ++g) {
            int32_t s = 0;
            for (int64_t k = 64 * g; k < 64 * g + 64; ++k)
                s += xq[m * K + k];
            xsum[m * G + g] = s;
        }
}

/* ------------------------------------------------------ affine W4, g = 64 */

/*
 * W4 affine group-64 quantization (R5) [qlip-w4], [mlx4722]: per (n, g) the
 * group min lo and max hi; scale s = fp16((hi - lo) / 15), offset o = fp16(lo);
 * codes rne((w - o) * (1 / s)) clamped to [0, 15], from the fp16 values; s == 0
 * gives zero codes.  Packed two codes per byte, even k low nibble (R6).
 * Wp is [N, K/2] bytes, s16 and o16 are [N, K/64] fp16 bit patterns.
 */
void oracle_quant_w4(const float *W, int64_t N, int64_t K,
                     uint8_t *Wp, uint16_t *s16, uint16_t *o16)
{
    int64_t G = K / 64;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + n * K + 64 * g;
            float lo = w[0], hi = w[0];
            for (int i = 1; i < 64; ++i) {
                if (w[i] < lo)
                    lo = w[i];
                if (w[i] > hi)
                    hi = w[i];
            }
            uint16_t sb = oracle_f32_to_f16((hi - lo) / 15.0f);
            uint16_t ob = oracle_f32_to_f16(lo);
            s16[n * G + g] = sb;
            o16[n * G + g] = ob;
            float s = oracle_f16_to_f32(sb);
            float o = oracle_f16_to_f32(ob);
            uint8_t codes[64];
            if (s == 0.0f) {
                memset(codes, 0, sizeof codes);
            } else {
                float r = 1.0f / s;
                for (int i = 0; i < 64; ++i) {
                    float t = (w[i] - o) * r;
                    float c = nearbyintf(t);
                    if (c < 0.0f)
                        c = 0.0f;
                    if (c > 15.0f)
                        c = 15.0f;
                    codes[i] = (uint8_t)c;
                }
            }
            uint8_t *dst = Wp + n * (K / 2) + 32 * g;
            for (int j = 0; j < 32; ++j)
                dst[j] = (uint8_t)(codes[2 * j] | (codes[2 * j + 1] << 4));
        }
}

/* Code k of row n of a packed [N, K/2] W4 matrix (R6). */
static int w4_code(const uint8_t *Wp, int64_t K, int64_t n, int64_t k)
{
    uint8_t b = Wp[n * (K / 2) + k / 2];
    return (k & 1) ? (b >> 4) : (b & 0x0F);
}

/* ------------------------------------------------------------ accumulate */

/* acc[m, n] = sum_k xq[m, k] * Wq[n, k], exact (int64) [qlip]. */
void oracle_w8a8_acc(const int8_t *xq, int64_t M, int64_t K,
                     const int8_t *Wq, int64_t N, int64_t *acc)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k)
                s += (int64_t)xq[m * K + k] * (int64_t)Wq[n * K + k];
            acc[m * N + n] = s;
        }
}

/*
 * acc[m, n, g] = sum_{k in group g} xq[m, k] * q[n, k] on the raw codes 0..15
 * (R7), exact (int64).  acc is [M, N, G].
 */
void oracle_w4a8_group_acc(const int8_t *xq, int64_t M, int64_t K,
                           const uint8_t *Wp, int64_t N, int64_t *acc)
{
    int64_t G = K / 64;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            for (int64_t g = 0; g < G; ++g) {
                int64_t s = 0;
                for (int64_t k = 64 * g; k < 64 * g + 64; ++k)
                    s += (int64_t)xq[m * K + k] * (int64_t)w4_code(Wp, K, n, k);
                acc[(m * N + n) * G + g] = s;
            }
}

/* --------------------------------------------------------------- dequant */

/*
 * W8A8 dequant + bias [qlip]: v = acc * sx[m] * sw[n] + bias[n] in fp64 (no
 * fused multiply-add).  bias may be NULL (no bias term).  v is [M, N].
 */
void oracle_w8a8_dequant_f64(const int64_t *acc, int64_t M, int64_t N,
                             const float *sx, const float *sw, const float *bias,
                             double *v)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double t = ((double)acc[m * N + n] * (double)sx[m]) * (double)sw[n];
            if (bias)
                t = t + (double)bias[n];
            v[m * N + n] = t;
        }
}

/* The same, rounded once to bf16 (nearest, ties to even): y bf16 [M, N]. */
void oracle_w8a8_dequant(const int64_t *acc, int64_t M, int64_t N,
                         const float *sx, const float *sw, const float *bias,
                         uint16_t *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double v;
        for (int64_t n = 0; n < N; ++n) {
            oracle_w8a8_dequant_f64(acc + m * N + n, 1, 1, sx + m, sw + n,
                                    bias ? bias + n : NULL, &v);
            y[m * N + n] = oracle_f64_to_bf16(v);
        }
    }
}

/*
 * W8A8 with the gated residual epilogue [kquant89], (R13):
 *   out = r[m,n] + g[n] * (acc * sx[m] * sw[n] + bias[n])
 * in fp64 with no fused multiply-add (the bracket exactly as
 * oracle_w8a8_dequant_f64 evaluates it), rounded once to bf16.
 * r bf16 [M, N], g fp32 [N], bias may be NULL; out bf16 [M, N].
 */
void oracle_w8a8_gated(const int64_t *acc, int64_t M, int64_t N,
                       const float *sx, const float *sw, const float *bias,
                       const float *gate, const uint16_t *r, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v;
            oracle_w8a8_dequant_f64(acc + m * N + n, 1, 1, sx + m, sw + n,
                                    bias ? bias + n : NULL, &v);
            double t = (double)gate[n] * v;
            t = t + (double)oracle_bf16_to_f32(r[m * N + n]);
            out[m * N + n] = oracle_f64_to_bf16(t);
        }
}

/*
 * W4A8 dequant [qlip-w4], (R7): the weight is q * s + o per group and the
 * activation xq * sx, so
 *   v = sx[m] * sum_g ( s[n,g] * acc[m,n,g] + o[n,g] * xsum[m,g] ) + bias[n]
 * in fp64 with no fused multiply-add.  bias may be NULL.  v is [M, N].
 */
void oracle_w4a8_dequant_f64(const int64_t *acc, const int32_t *xsum,
                             int64_t M, int64_t N, int64_t G,
                             const float *sx, const uint16_t *s16, const uint16_t *o16,
                             const float *bias, double *v)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double f = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                double s = (double)oracle_f16_to_f32(s16[n * G + g]);
                double o = (double)oracle_f16_to_f32(o16[n * G + g]);
                double t = s * (double)acc[(m * N + n) * G + g];
                double u = o * (double)xsum[m * G + g];
                f = f + (t + u);
            }
            double r = (double)sx[m] * f;
            if (bias)
                r = r + (double)bias[n];
            v[m * N + n] = r;
        }
}

/* The same, rounded once to bf16: y bf16 [M, N]. */
void oracle_w4a8_dequant(const int64_t *acc, const int32_t *xsum,
                         int64_t M, int64_t N, int64_t G,
                         const float *sx, const uint16_t *s16, const uint16_t *o16,
                         const float *bias, uint16_t *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v;
            oracle_w4a8_dequant_f64(acc + (m * N + n) * G, xsum + m * G, 1, 1, G,
                                    sx + m, s16 + n * G, o16 + n * G,
                                    bias ? bias + n : NULL, &v);
            y[m * N + n] = oracle_f64_to_bf16(v);
        }
}

/*
 * INT8 attention of one head [qlip-sage], (R14), for the query rows `rows`
 * (nrows of them) against all L keys, head dim D: q and k are given as their
 * per-token codes and scales (from oracle_quant_act_bf16), v as bf16 bits
 * [L, D].  Everything after the integer dot products is fp64:
 * s = dot * sq[i] * sk[j] * scale, p = exp(s - max_j s),
 * o = (sum_j p v_j) / (sum_j p).  out_f64 (nullable, [nrows, D]) receives o
 * before the rounding; out ([nrows, D]) receives it rounded to bf16.
 */
void oracle_sage_attention_rows(const int8_t *qc, const float *sq, const int8_t *kc,
                                const float *sk, const uint16_t *v, int64_t L, int64_t D,
                                double scale, const int64_t *rows, int64_t nrows,
                                double *out_f64, uint16_t *out)
{
#pragma omp parallel
    {
        double *s = (double *)malloc((size_t)L * sizeof(double));
        double *o = (double *)malloc((size_t)D * sizeof(double));
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows[r];
            double mx = -INFINITY;
            for (int64_t j = 0; j < L; ++j) {
                int64_t dot = 0;
                for (int64_t d = 0; d < D; ++d)
                    dot += (int64_t)qc[i * D + d] * (int64_t)kc[j * D + d];
                s[j] = (double)dot * (double)sq[i] * (double)sk[j] * scale;
                if (s[j] > mx)
                    mx = s[j];
            }
            double l = 0.0;
            for (int64_t d = 0; d < D; ++d)
                o[d] = 0.0;
            for (int64_t j = 0; j < L; ++j) {
                double p = exp(s[j] - mx);
                l += p;
                for (int64_t d = 0; d < D; ++d)
                    o[d] += p * (double)oracle_bf16_to_f32(v[j * D + d]);
            }
            for (int64_t d = 0; d < D; ++d) {
                double res = o[d] / l;
                if (out_f64)
                    out_f64[r * D + d] = res;
                out[r * D + d] = oracle_f64_to_bf16(res);
            }
        }
        free(s);
        free(o);
    }
}

/* The same for every query row 0 .. L - 1 (outputs [L, D]). */
void oracle_sage_attention(const int8_t *qc, const float *sq, const int8_t *kc,
                           const float *sk, const uint16_t *v, int64_t L, int64_t D,
                           double scale, double *out_f64, uint16_t *out)
{
    int64_t *rows = (int64_t *)malloc((size_t)L * sizeof(int64_t));
    for (int64_t i = 0; i < L; ++i)
        rows[i] = i;
    oracle_sage_attention_rows(qc, sq, kc, sk, v, L, D, scale, rows, L, out_f64, out);
    free(rows);
}
