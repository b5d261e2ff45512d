/*
 * CPU oracle for the block-scaled FP8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: it exists so that the tests, the smoke check and the CPU
 * baseline leg of the benchmark can compare the CUDA kernels against a plain,
 * slow, obviously correct restatement of what the method computes.  It shares
 * no code, header, table or constant with the CUDA library.
 *
 * What it restates (sources are the five web pages about the Puro-2B report):
 *   - "FP8 块级混合精度训练" (background section of the paper.rainbus.top
 *     summary): E4M3 has 4 exponent and 3 mantissa bits; activations are cut
 *     into groups of 128 values along the GEMM reduction dimension, weights
 *     into 128x128 blocks; every block gets one power-of-two scale computed
 *     online.
 *   - "方法步骤详情" step (3) of the same page: fprop, dgrad and wgrad of the
 *     linear layers all run in E4M3.
 *   - §3.2 of the ta-paperlens explainer: activations AND gradients carry one
 *     scale per 128 elements along the reduction direction, weights one per
 *     128x128 block.
 *   - Appendix C "FP8 implementation pipeline" of the paperlayer.ai summary:
 *     the three GEMMs (forward, data-gradient, weight-gradient) use blockwise
 *     E4M3; hidden flow stays BF16.
 *
 * Readings where the pages are silent:
 *   - E4M3 is the OCP "FN" variant: bias 7, max finite 448, NaN 0x7F/0xFF,
 *     no infinities, subnormals 2^-6 * m/8.
 *   - The scale 2^e of a group is the smallest power of two with
 *     amax <= 448 * 2^e, so no element saturates; e is clamped to
 *     [-127, 127] and stored as the byte e + 127 (UE8M0).  amax == 0 gives e=0.
 *   - Elements are encoded with round-to-nearest-even and saturation to the
 *     largest finite value.
 *   - GEMMs multiply the dequantized operands and sum in FP64.
 *
 * Every function below is written from those definitions, with plain loops and
 * no blocking or reordering beyond what the definition states.  Parallelism is
 * only over independent output rows (OpenMP), which does not change any sum.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

/* ---- BF16 and E4M3 formats ------------------------------------------------ */

/* BF16 is the upper half of an IEEE binary32: widening is a 16-bit shift. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP E4M3 ("FN") decode: sign, 4-bit exponent (bias 7), 3-bit mantissa.
 * Normal:    (-1)^s * 2^(E-7) * (1 + m/8)
 * Subnormal: (-1)^s * 2^-6 * (m/8)
 * 0x7F / 0xFF are NaN; there is no infinity. */
double oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7;
    int E = (c >> 3) & 0xF;
    int m = c & 0x7;
    double v;
    if (E == 15 && m == 7)
        return NAN;
    if (E == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, E - 7);
    return s ? -v : v;
}

/* OCP E4M3 encode with round-to-nearest-even and saturation to +-448.
 * The representable magnitudes form, binade by binade, an evenly spaced grid:
 * below 2^-6 the spacing is 2^-9 (subnormals), in [2^E, 2^(E+1)) it is
 * 2^(E-3).  Rounding to the grid is done with nearbyint() in the default
 * rounding mode, i.e. ties to even; the grid index of an even mantissa is even,
 * so "even integer" and "even code" coincide. */
uint8_t oracle_e4m3_encode(double v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    int e2, E, code;
    double q;

    if (isnan(v))
        return (uint8_t)(sign | 0x7F);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7E);          /* satfinite */
    if (a < ldexp(1.0, -6)) {
        q = nearbyint(ldexp(a, 9));             /* multiples of 2^-9 */
        return (uint8_t)(sign | (int)q);        /* q == 8 is 2^-6 = code 0x08 */
    }
    frexp(a, &e2);                              /* a in [2^(e2-1), 2^e2) */
    E = e2 - 1;
    q = nearbyint(ldexp(a, 3 - E));             /* grid index in [8, 16] */
    if (q == 16.0) {                            /* rounded up into next binade */
        E += 1;
        q = 8.0;
    }
    code = ((E + 7) << 3) | ((int)q - 8);
    if (code > 0x7E)
        code = 0x7E;                            /* satfinite */
    return (uint8_t)(sign | code);
}

/* ---- the scale rule ----------------------------------------------------- */

/* Smallest integer e with amax <= 448 * 2^e, clamped to [-127, 127];
 * amax == 0 gives 0.  Written as the definition: walk e until it holds. */
int oracle_scale_exponent(double amax)
{
    int e = 0;
    if (amax == 0.0)
        return 0;
    while (e < 127 && amax > ldexp(448.0, e))
        e++;
    while (e > -127 && amax <= ldexp(448.0, e - 1))
        e--;
    return e;
}

/* Quantize one group of n values held as doubles: writes the codes and returns
 * the scale exponent. */
static int quant_group(const double *v, int64_t n, int64_t stride, uint8_t *codes,
                       int64_t code_stride)
{
    double amax = 0.0;
    int64_t i;
    int e;
    for (i = 0; i < n; i++) {
        double a = fabs(v[i * stride]);
        if (a > amax)
            amax = a;
    }
    e = oracle_scale_exponent(amax);
    for (i = 0; i < n; i++)
        codes[i * code_stride] = oracle_e4m3_encode(ldexp(v[i * stride], -e));
    return e;
}

/* ---- quantizers ---------------------------------------------------------- */

/* 1x128 groups along the columns of X [rows, cols] (row stride ld_x elements).
 * q: [rows][cols] dense codes; s: [rows][cols/128] dense UE8M0 bytes. */
void oracle_quant_rowwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *q, uint8_t *s)
{
    int64_t groups = cols / 128;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        double v[128];
        int64_t g, i;
        for (g = 0; g < groups; g++) {
            for (i = 0; i < 128; i++)
                v[i] = oracle_bf16_to_double(x[r * ld_x + g * 128 + i]);
            s[r * groups + g] =
                (uint8_t)(quant_group(v, 128, 1, q + r * cols + g * 128, 1) + 127);
        }
    }
}

/* 1x128 groups along the ROWS of X [rows, cols]: column c, group g holds rows
 * 128g .. min(128g+127, rows-1) (the last group may be short; only its valid
 * rows enter the amax).  Output is transposed:
 * qt: [cols][rows] dense codes; st: [cols][ceil(rows/128)] dense bytes. */
void oracle_quant_colwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *qt, uint8_t *st)
{
    int64_t groups = (rows + 127) / 128;
    int64_t c;
#pragma omp parallel for schedule(static)
    for (c = 0; c < cols; c++) {
        double v[128];
        int64_t g, i;
        for (g = 0; g < groups; g++) {
            int64_t r0 = g * 128;
            int64_t n = rows - r0 < 128 ? rows - r0 : 128;
            for (i = 0; i < n; i++)
                v[i] = oracle_bf16_to_double(x[(r0 + i) * ld_x + c]);
            st[c * groups + g] =
                (uint8_t)(quant_group(v, n, 1, qt + c * rows + r0, 1) + 127);
        }
    }
}

/* 128x128 blocks of W [n, k]: one scale per block.
 * q: [n][k] dense codes; s: [n/128][k/128] dense bytes. */
void oracle_quant_weight(const uint16_t *w, int64_t n, int64_t k, int64_t ld_w,
                         uint8_t *q, uint8_t *s)
{
    int64_t bn_count = n / 128, bk_count = k / 128;
    int64_t blk;
#pragma omp parallel for schedule(static)
    for (blk = 0; blk < bn_count * bk_count; blk++) {
        int64_t bn = blk / bk_count, bk = blk % bk_count;
        double *v = (double *)malloc(sizeof(double) * 128 * 128);
        uint8_t codes[128 * 128];
        int64_t i, j;
        int e;
        for (i = 0; i < 128; i++)
            for (j = 0; j < 128; j++)
                v[i * 128 + j] = oracle_bf16_to_double(w[(bn * 128 + i) * ld_w + bk * 128 + j]);
        e = quant_group(v, 128 * 128, 1, codes, 1);
        for (i = 0; i < 128; i++)
            for (j = 0; j < 128; j++)
                q[(bn * 128 + i) * k + bk * 128 + j] = codes[i * 128 + j];
        s[bn * bk_count + bk] = (uint8_t)(e + 127);
        free(v);
    }
}

/* ---- dequantization ------------------------------------------------------ */

/* d = decode(q) * 2^(s - 127), exact in FP64.
 * Activation-style operand: q [rows][cols], one scale per (row, 128-col group),
 * s [rows][ceil(cols/128)] dense. */
void oracle_dequant_groups(const uint8_t *q, int64_t rows, int64_t cols, const uint8_t *s,
                           double *out)
{
    int64_t groups = (cols + 127) / 128;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < rows; r++) {
        int64_t c;
        for (c = 0; c < cols; c++)
            out[r * cols + c] =
                ldexp(oracle_e4m3_decode(q[r * cols + c]), (int)s[r * groups + c / 128] - 127);
    }
}

/* Weight operand: q [n][k], one scale per 128x128 block, s [n/128][k/128]. */
void oracle_dequant_blocks(const uint8_t *q, int64_t n, int64_t k, const uint8_t *s,
                           double *out)
{
    int64_t bk_count = k / 128;
    int64_t r;
#pragma omp parallel for schedule(static)
    for (r = 0; r < n; r++) {
        int64_t c;
        for (c = 0; c < k; c++)
            out[r * k + c] = ldexp(oracle_e4m3_decode(q[r * k + c]),
                                   (int)s[(r / 128) * bk_count + c / 128] - 127);
    }
}

/* ---- the three GEMMs, FP64, on dequantized operands ------------------------
 * Each computes only the output rows listed in `rows_sel` (n_sel of them), so
 * a test can sample a large problem; out is [n_sel][cols of the output]. */

/* fprop: Y[m][n] = sum_k X[m][k] * W[n][k];  x [M][K], w [N][K]. */
void oracle_gemm_fprop(const double *x, const double *w, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *y)
{
    int64_t t;
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < n_sel; t++) {
        int64_t m = rows_sel[t], n, k;
        for (n = 0; n < N; n++) {
            double acc = 0.0;
            for (k = 0; k < K; k++)
                acc += x[m * K + k] * w[n * K + k];
            y[t * N + n] = acc;
        }
    }
}

/* dgrad: dX[m][k] = sum_n dY[m][n] * W[n][k];  dy [M][N], w [N][K]. */
void oracle_gemm_dgrad(const double *dy, const double *w, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *dx)
{
    int64_t t;
    (void)M;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < n_sel; t++) {
        int64_t m = rows_sel[t], n, k;
        for (k = 0; k < K; k++) {
            double acc = 0.0;
            for (n = 0; n < N; n++)
                acc += dy[m * N + n] * w[n * K + k];
            dx[t * K + k] = acc;
        }
    }
}

/* wgrad: dW[n][k] = sum_m dY[m][n] * X[m][k], given the transposed operands
 * dyt [N][M] (dY^T) and xt [K][M] (X^T), as the method quantizes them along M. */
void oracle_gemm_wgrad(const double *dyt, const double *xt, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *dw)
{
    int64_t t;
    (void)N;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < n_sel; t++) {
        int64_t n = rows_sel[t], k, m;
        for (k = 0; k < K; k++) {
            double acc = 0.0;
            for (m = 0; m < M; m++)
                acc += dyt[n * M + m] * xt[k * M + m];
            dw[t * K + k] = acc;
        }
    }
}

/* ---- BF16 output rounding (round to nearest even), for reporting ---------- */

/* Round a double to the nearest BF16 (ties to even) and return its bits.
 * Done in two exact steps: to binary32 would double-round, so the rounding is
 * made directly on the double's value: find the BF16 grid spacing of |v| and
 * round v / spacing to an integer with nearbyint (ties to even). */
uint16_t oracle_double_to_bf16(double v)
{
    double a = fabs(v), q, r;
    int e2, E;
    uint32_t u;
    float f;
    if (isnan(v))
        return 0x7FC0;
    if (a == 0.0)
        return signbit(v) ? 0x8000 : 0x0000;
    frexp(a, &e2);
    E = e2 - 1;                                  /* a in [2^E, 2^(E+1)) */
    if (E < -126)
        E = -126;                                /* subnormal spacing 2^-133 */
    q = nearbyint(ldexp(a, 7 - E));              /* 8 significant bits */
    r = ldexp(q, E - 7);
    if (r > ldexp(255.0 / 128.0, 127))           /* beyond the largest BF16 */
        r = INFINITY;
    f = (float)(signbit(v) ? -r : r);            /* exact: r has <= 8 bits */
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void oracle_round_bf16_array(const double *v, int64_t n, uint16_t *out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; i++)
        out[i] = oracle_double_to_bf16(v[i]);
}
