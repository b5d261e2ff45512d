/*
 * abi_consumer.c -- a plain C99 program that uses libpuro_fp8 through
 * include/puro_fp8.h alone: no Python, no torch.  Test infrastructure.
 *
 * Host mode (default build): argument checks, no-op shapes, the layout and
 * status helpers.  Nothing here touches the GPU: every call below fails or
 * returns before the library's first CUDA call.
 *
 * GPU mode (-DABI_CONSUMER_GPU, linked with the CUDA runtime and the oracle
 * library): one linear layer through the C ABI on device buffers this program
 * allocates -- the 1x128 quantization of X and dY in both layouts, the 128x128
 * quantization of W with its transposed codes, and the fprop, dgrad and wgrad
 * GEMMs (separately and as one dgrad+wgrad launch) -- compared with the CPU
 * oracle: codes and scale bytes exactly, GEMM results within the tolerance the
 * parity tests use (relative Frobenius error <= 1e-3 against the oracle's
 * FP64 result rounded once to BF16, and every element within
 * 4e-3 * rms + 1 BF16 ulp of the FP64 result).
 *
 * Method: the Puro-2B block-scaled FP8 linear layer (paper.rainbus.top
 * summary, "方法步骤详情" step (3); ta-paperlens explainer §3.2; paperlayer.ai
 * summary, Appendix C "FP8 implementation pipeline").
 *
 * Exit status 0 and a last line "abi_consumer: <mode> ok" on success.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "puro_fp8.h"

static int g_fail = 0;

#define CHECK(cond, ...)                                       \
    do {                                                       \
        if (!(cond)) {                                         \
            fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
            fprintf(stderr, __VA_ARGS__);                      \
            fprintf(stderr, "\n");                             \
            g_fail = 1;                                        \
        }                                                      \
    } while (0)

/* ------------------------------------------------------------------ host mode */

static void host_checks(void)
{
    /* a 16-byte-aligned address that no call below dereferences */
    void *A = (void *)(uintptr_t)(1u << 20);
    char *Ab = (char *)A;
    int code;

    CHECK(puro_fp8_blocked_scale_bytes(0, 4) == 0, "blocked bytes of 0 rows");
    CHECK(puro_fp8_blocked_scale_bytes(1, 1) == 512, "blocked bytes of 1 x 1");
    CHECK(puro_fp8_blocked_scale_bytes(129, 4) == 1024, "blocked bytes of 129 x 4");
    CHECK(puro_fp8_blocked_scale_bytes(8000, 63) == 63 * 16 * 512, "blocked bytes of 8000 x 63");

    for (code = 0; code >= -7; --code) {
        const char *s = puro_fp8_status_string(code);
        CHECK(s != NULL && strncmp(s, "PURO_", 5) == 0, "status string of %d", code);
    }

    /* quant_act: errors, then the empty no-ops */
    CHECK(puro_fp8_quant_act(A, 16, 128, 128, 7, A, 128, A, NULL, 0, NULL, NULL, NULL) ==
              PURO_ERR_LAYOUT, "quant_act bad layout");
    CHECK(puro_fp8_quant_act(A, 16, 100, 128, PURO_ROWWISE, A, 128, A, NULL, 0, NULL, NULL,
                             NULL) == PURO_ERR_SHAPE, "quant_act cols %% 128");
    CHECK(puro_fp8_quant_act(NULL, 16, 128, 128, PURO_ROWWISE, A, 128, A, NULL, 0, NULL, NULL,
                             NULL) == PURO_ERR_NULL, "quant_act null input");
    CHECK(puro_fp8_quant_act(Ab + 2, 16, 128, 128, PURO_ROWWISE, A, 128, A, NULL, 0, NULL, NULL,
                             NULL) == PURO_ERR_ALIGN, "quant_act misaligned input");
    CHECK(puro_fp8_quant_act(A, 16, 128, 128, PURO_COLWISE, NULL, 0, NULL, A, 16, NULL, NULL,
                             NULL) == PURO_ERR_NULL, "quant_act colwise without st");
    CHECK(puro_fp8_quant_act(A, 16, 128, 128, PURO_ROWWISE, A, 128, A, NULL, 0, NULL,
                             (uint32_t *)(Ab + 4), NULL) == PURO_ERR_ALIGN,
          "quant_act misaligned tile counter");
    CHECK(puro_fp8_quant_act(NULL, 0, 128, 128, PURO_BOTH, NULL, 0, NULL, NULL, 0, NULL, NULL,
                             NULL) == PURO_OK, "quant_act 0 rows");
    CHECK(puro_fp8_quant_act_static_scratch(A, 16, 128, 128, 7, A, 128, A, A, 16, A, NULL) ==
              PURO_ERR_LAYOUT, "static scratch bad layout");
    CHECK(puro_fp8_quant_act_static_scratch(A, 32768, (1ll << 31) - 128, (1ll << 31) - 128,
                                            PURO_BOTH, A, (1ll << 31) - 128, A, A, 32768, A,
                                            NULL) == PURO_ERR_SHAPE,
          "static scratch beyond 2^31 tiles");

    /* quant_weight */
    CHECK(puro_fp8_quant_weight(A, 100, 128, 128, A, 128, A, NULL, 0, A, NULL, NULL) ==
              PURO_ERR_SHAPE, "quant_weight n %% 128");
    CHECK(puro_fp8_quant_weight(A, 128, 128, 128, NULL, 128, A, NULL, 0, A, NULL, NULL) ==
              PURO_ERR_NULL, "quant_weight null q");
    CHECK(puro_fp8_quant_weight(A, 128, 128, 128, A, 128, A, NULL, 0, Ab + 4, NULL, NULL) ==
              PURO_ERR_ALIGN, "quant_weight misaligned s_fwd");

    /* the GEMMs */
    CHECK(puro_fp8_gemm_fprop(A, 256, A, A, 256, A, A, 320, 64, 320, 256, NULL) ==
              PURO_ERR_SHAPE, "fprop n %% 128");
    CHECK(puro_fp8_gemm_fprop(A, 256, A, A, 256, NULL, A, 256, 64, 256, 256, NULL) ==
              PURO_ERR_NULL, "fprop null weight scales");
    CHECK(puro_fp8_gemm_dgrad(A, 128, A, A, 256, A, A, 256, 64, 256, 256, NULL) ==
              PURO_ERR_SHAPE, "dgrad ld_qdy < n");
    CHECK(puro_fp8_gemm_wgrad(A, 48, A, A, 64, A, A, 256, 64, 256, 256, NULL) ==
              PURO_ERR_SHAPE, "wgrad ld_qdyt < m");
    CHECK(puro_fp8_gemm_wgrad_f32(A, 64, A, A, 64, A, A, 256, 64, 256, 256, 2, NULL) ==
              PURO_ERR_LAYOUT, "wgrad_f32 accumulate flag");
    CHECK(puro_fp8_gemm_dgrad_wgrad(A, 256, A, A, 256, A, A, 256, A, 64, A, A, 64, A, A, 256,
                                    64, 256, 256, 3, NULL) == PURO_ERR_LAYOUT,
          "dgrad_wgrad dW kind");
    CHECK(puro_fp8_gemm_fprop(NULL, 0, NULL, NULL, 0, NULL, NULL, 0, 0, 256, 256, NULL) ==
              PURO_OK, "fprop m = 0");
    CHECK(puro_fp8_gemm_wgrad(NULL, 0, NULL, NULL, 0, NULL, NULL, 0, 64, 0, 256, NULL) ==
              PURO_OK, "wgrad n = 0");
}

#ifdef ABI_CONSUMER_GPU
/* ------------------------------------------------------------------- GPU mode */
#include <cuda_runtime_api.h>

/* the oracle (oracle/puro_oracle.c, test infrastructure) */
double oracle_bf16_to_double(uint16_t b);
uint16_t oracle_double_to_bf16(double v);
void oracle_quant_rowwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *q, uint8_t *s);
void oracle_quant_colwise(const uint16_t *x, int64_t rows, int64_t cols, int64_t ld_x,
                          uint8_t *qt, uint8_t *st);
void oracle_quant_weight(const uint16_t *w, int64_t n, int64_t k, int64_t ld_w, uint8_t *q,
                         uint8_t *s);
void oracle_dequant_groups(const uint8_t *q, int64_t rows, int64_t cols, const uint8_t *s,
                           double *out);
void oracle_dequant_blocks(const uint8_t *q, int64_t n, int64_t k, const uint8_t *s,
                           double *out);
void oracle_gemm_fprop(const double *x, const double *w, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *y);
void oracle_gemm_dgrad(const double *dy, const double *w, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *dx);
void oracle_gemm_wgrad(const double *dyt, const double *xt, int64_t M, int64_t N, int64_t K,
                       const int64_t *rows_sel, int64_t n_sel, double *dw);

/* Seeded BF16 inputs (splitmix64 bits): random sign and mantissa, exponent
 * field in [118, 131], so magnitudes between 2^-9 and 2^5; no NaN or Inf. */
static uint64_t g_rng = 0x243F6A8885A308D3ull;
static uint64_t splitmix64(void)
{
    uint64_t z = (g_rng += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
static void fill_bf16(uint16_t *v, int64_t n)
{
    int64_t i;
    for (i = 0; i < n; i++) {
        uint64_t r = splitmix64();
        uint16_t sign = (uint16_t)((r >> 63) << 15);
        uint16_t expo = (uint16_t)(118 + (r >> 32) % 14);
        uint16_t mant = (uint16_t)(r & 0x7F);
        v[i] = (uint16_t)(sign | (expo << 7) | mant);
    }
}

/* byte offset of (row r, group g) in a blocked scale array of `groups` groups
 * (the layout include/puro_fp8.h specifies) */
static int64_t blocked(int64_t r, int64_t g, int64_t groups)
{
    int64_t g4 = (groups + 3) / 4;
    return ((r / 128) * g4 + g / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + g % 4;
}

#define CUDA_OK(call)                                                                   \
    do {                                                                                \
        cudaError_t e_ = (call);                                                        \
        if (e_ != cudaSuccess) {                                                        \
            fprintf(stderr, "FAIL %s:%d: %s: %s\n", __FILE__, __LINE__, #call,          \
                    cudaGetErrorString(e_));                                            \
            exit(2);                                                                    \
        }                                                                               \
    } while (0)

static void *dev_alloc(size_t bytes)
{
    void *p = NULL;
    CUDA_OK(cudaMalloc(&p, bytes ? bytes : 16));
    CUDA_OK(cudaMemset(p, 0, bytes ? bytes : 16));
    return p;
}
static void *host_get(const void *d, size_t bytes)
{
    void *h = malloc(bytes ? bytes : 1);
    CUDA_OK(cudaMemcpy(h, d, bytes, cudaMemcpyDeviceToHost));
    return h;
}

/* ulp of a BF16 number of magnitude |v| (8 significant bits) */
static double bf16_ulp(double v)
{
    int e;
    double a = fabs(v) > ldexp(1.0, -126) ? fabs(v) : ldexp(1.0, -126);
    frexp(a, &e);
    return ldexp(1.0, e - 1 - 7);
}

/* got: BF16 [rows, cols] with row stride ld; ref: FP64 [rows, cols] dense */
static void check_gemm(const char *what, const uint16_t *got, int64_t ld, const double *ref,
                       int64_t rows, int64_t cols)
{
    double ss_ref = 0.0, ss_den = 0.0, ss_err = 0.0, rms, worst = -1.0;
    int64_t i, j;
    for (i = 0; i < rows * cols; i++) ss_ref += ref[i] * ref[i];
    rms = rows * cols > 0 ? sqrt(ss_ref / (double)(rows * cols)) : 0.0;
    for (i = 0; i < rows; i++)
        for (j = 0; j < cols; j++) {
            double g = oracle_bf16_to_double(got[i * ld + j]);
            double r = ref[i * cols + j];
            double rb = oracle_bf16_to_double(oracle_double_to_bf16(r));
            double excess = fabs(g - r) - (4e-3 * rms + bf16_ulp(r));
            ss_den += rb * rb;
            ss_err += (g - rb) * (g - rb);
            if (excess > worst) worst = excess;
        }
    CHECK(ss_den > 0.0 && sqrt(ss_err / ss_den) <= 1e-3, "%s: relative Frobenius error %.3g",
          what, ss_den > 0.0 ? sqrt(ss_err / ss_den) : -1.0);
    CHECK(worst <= 0.0, "%s: an element exceeds 4e-3*rms + 1 ulp by %.3g", what, worst);
}

static void gpu_checks(void)
{
    /* one linear layer: X [M, K], W [N, K], dY [M, N]; M ragged (3 token
     * groups, the last short), several tiles along every dimension */
    const int64_t M = 300, K = 384, N = 256;
    const int64_t GK = K / 128, GN = N / 128, GM = (M + 127) / 128;
    const int64_t LDT = (M + 15) / 16 * 16; /* leading dim of the transposed codes */
    int64_t i, j, r, g;
    int rc;

    uint16_t *x = malloc(sizeof(uint16_t) * M * K), *w = malloc(sizeof(uint16_t) * N * K);
    uint16_t *dy = malloc(sizeof(uint16_t) * M * N);
    fill_bf16(x, M * K);
    fill_bf16(w, N * K);
    fill_bf16(dy, M * N);
    for (j = 128; j < 256; j++) x[7 * K + j] = (uint16_t)(j & 1 ? 0x8000 : 0x0000); /* zero row group */
    for (r = 128; r < 256; r++) x[r * K + 5] = 0;                                   /* zero column group */

    /* device buffers */
    void *d_x = dev_alloc(sizeof(uint16_t) * M * K), *d_w = dev_alloc(sizeof(uint16_t) * N * K);
    void *d_dy = dev_alloc(sizeof(uint16_t) * M * N);
    CUDA_OK(cudaMemcpy(d_x, x, sizeof(uint16_t) * M * K, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(d_w, w, sizeof(uint16_t) * N * K, cudaMemcpyHostToDevice));
    CUDA_OK(cudaMemcpy(d_dy, dy, sizeof(uint16_t) * M * N, cudaMemcpyHostToDevice));
    const int64_t sx_b = puro_fp8_blocked_scale_bytes(M, GK), sxt_b = puro_fp8_blocked_scale_bytes(K, GM);
    const int64_t sdy_b = puro_fp8_blocked_scale_bytes(M, GN), sdyt_b = puro_fp8_blocked_scale_bytes(N, GM);
    const int64_t sfw_b = puro_fp8_blocked_scale_bytes(N, GK), sbw_b = puro_fp8_blocked_scale_bytes(K, GN);
    void *d_qx = dev_alloc(M * K), *d_sx = dev_alloc(sx_b), *d_qxt = dev_alloc(K * LDT),
         *d_sxt = dev_alloc(sxt_b);
    void *d_qdy = dev_alloc(M * N), *d_sdy = dev_alloc(sdy_b), *d_qdyt = dev_alloc(N * LDT),
         *d_sdyt = dev_alloc(sdyt_b);
    void *d_qw = dev_alloc(N * K), *d_sw = dev_alloc(GN * GK), *d_qwt = dev_alloc(K * N),
         *d_sfw = dev_alloc(sfw_b), *d_sbw = dev_alloc(sbw_b);
    void *d_y = dev_alloc(sizeof(uint16_t) * M * N), *d_dx = dev_alloc(sizeof(uint16_t) * M * K),
         *d_dw = dev_alloc(sizeof(uint16_t) * N * K);
    void *d_dx2 = dev_alloc(sizeof(uint16_t) * M * K), *d_dw2 = dev_alloc(sizeof(uint16_t) * N * K);
    void *d_ctr = dev_alloc(8);
    void *d_q2 = dev_alloc(M * K), *d_s2 = dev_alloc(sx_b), *d_qt2 = dev_alloc(K * LDT),
         *d_st2 = dev_alloc(sxt_b);

    /* the layer through the C ABI, on the legacy default stream */
    rc = puro_fp8_quant_act(d_x, M, K, K, PURO_BOTH, d_qx, K, d_sx, d_qxt, LDT, d_sxt,
                            (uint32_t *)d_ctr, NULL);
    CHECK(rc == PURO_OK, "quant_act X: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_quant_act(d_dy, M, N, N, PURO_BOTH, d_qdy, N, d_sdy, d_qdyt, LDT, d_sdyt,
                            (uint32_t *)d_ctr, NULL);
    CHECK(rc == PURO_OK, "quant_act dY: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_quant_act_static_scratch(d_x, M, K, K, PURO_BOTH, d_q2, K, d_s2, d_qt2, LDT,
                                           d_st2, NULL);
    CHECK(rc == PURO_OK, "quant_act_static_scratch X: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_quant_weight(d_w, N, K, K, d_qw, K, d_sw, d_qwt, N, d_sfw, d_sbw, NULL);
    CHECK(rc == PURO_OK, "quant_weight: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_gemm_fprop(d_qx, K, d_sx, d_qw, K, d_sfw, d_y, N, M, N, K, NULL);
    CHECK(rc == PURO_OK, "fprop: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_gemm_dgrad(d_qdy, N, d_sdy, d_qwt, N, d_sbw, d_dx, K, M, N, K, NULL);
    CHECK(rc == PURO_OK, "dgrad: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_gemm_wgrad(d_qdyt, LDT, d_sdyt, d_qxt, LDT, d_sxt, d_dw, K, M, N, K, NULL);
    CHECK(rc == PURO_OK, "wgrad: %s", puro_fp8_status_string(rc));
    rc = puro_fp8_gemm_dgrad_wgrad(d_qdy, N, d_sdy, d_qwt, N, d_sbw, d_dx2, K, d_qdyt, LDT,
                                   d_sdyt, d_qxt, LDT, d_sxt, d_dw2, K, M, N, K, PURO_DW_BF16,
                                   NULL);
    CHECK(rc == PURO_OK, "dgrad_wgrad: %s", puro_fp8_status_string(rc));
    CUDA_OK(cudaDeviceSynchronize());
    rc = puro_fp8_device_status(NULL);
    CHECK(rc == PURO_OK, "device status: %s", puro_fp8_status_string(rc));

    /* the oracle */
    uint8_t *q_ref = malloc(M * K), *s_ref = malloc(M * GK), *qt_ref = malloc(K * M),
            *st_ref = malloc(K * GM);
    uint8_t *qdy_ref = malloc(M * N), *sdy_ref = malloc(M * GN), *qdyt_ref = malloc(N * M),
            *sdyt_ref = malloc(N * GM);
    uint8_t *qw_ref = malloc(N * K), *sw_ref = malloc(GN * GK);
    oracle_quant_rowwise(x, M, K, K, q_ref, s_ref);
    oracle_quant_colwise(x, M, K, K, qt_ref, st_ref);
    oracle_quant_rowwise(dy, M, N, N, qdy_ref, sdy_ref);
    oracle_quant_colwise(dy, M, N, N, qdyt_ref, sdyt_ref);
    oracle_quant_weight(w, N, K, K, qw_ref, sw_ref);

    /* codes and scales, byte for byte */
    {
        uint8_t *qx = host_get(d_qx, M * K), *sx = host_get(d_sx, sx_b);
        uint8_t *qxt = host_get(d_qxt, K * LDT), *sxt = host_get(d_sxt, sxt_b);
        uint8_t *qdy = host_get(d_qdy, M * N), *sdy = host_get(d_sdy, sdy_b);
        uint8_t *qdyt = host_get(d_qdyt, N * LDT), *sdyt = host_get(d_sdyt, sdyt_b);
        uint8_t *qw = host_get(d_qw, N * K), *sw = host_get(d_sw, GN * GK);
        uint8_t *qwt = host_get(d_qwt, K * N), *sfw = host_get(d_sfw, sfw_b),
                *sbw = host_get(d_sbw, sbw_b);
        uint8_t *q2 = host_get(d_q2, M * K), *s2 = host_get(d_s2, sx_b);
        uint8_t *qt2 = host_get(d_qt2, K * LDT), *st2 = host_get(d_st2, sxt_b);
        int64_t bad = 0;
        for (i = 0; i < M * K; i++) bad += qx[i] != q_ref[i];
        for (r = 0; r < M; r++)
            for (g = 0; g < GK; g++) bad += sx[blocked(r, g, GK)] != s_ref[r * GK + g];
        for (i = 0; i < K; i++)
            for (j = 0; j < LDT; j++) bad += qxt[i * LDT + j] != (j < M ? qt_ref[i * M + j] : 0);
        for (r = 0; r < K; r++)
            for (g = 0; g < GM; g++) bad += sxt[blocked(r, g, GM)] != st_ref[r * GM + g];
        CHECK(bad == 0, "quant_act X: %lld bytes differ from the oracle", (long long)bad);
        CHECK(s_ref[7 * GK + 1] == 127 && st_ref[5 * GM + 1] == 127,
              "the zero groups of the input carry the scale byte 127");
        bad = 0;
        for (i = 0; i < M * N; i++) bad += qdy[i] != qdy_ref[i];
        for (r = 0; r < M; r++)
            for (g = 0; g < GN; g++) bad += sdy[blocked(r, g, GN)] != sdy_ref[r * GN + g];
        for (i = 0; i < N; i++)
            for (j = 0; j < M; j++) bad += qdyt[i * LDT + j] != qdyt_ref[i * M + j];
        for (r = 0; r < N; r++)
            for (g = 0; g < GM; g++) bad += sdyt[blocked(r, g, GM)] != sdyt_ref[r * GM + g];
        CHECK(bad == 0, "quant_act dY: %lld bytes differ from the oracle", (long long)bad);
        bad = 0;
        for (i = 0; i < N * K; i++) bad += qw[i] != qw_ref[i];
        for (i = 0; i < GN * GK; i++) bad += sw[i] != sw_ref[i];
        for (i = 0; i < K; i++)
            for (j = 0; j < N; j++) bad += qwt[i * N + j] != qw_ref[j * K + i];
        for (r = 0; r < N; r++)
            for (g = 0; g < GK; g++) bad += sfw[blocked(r, g, GK)] != sw_ref[(r / 128) * GK + g];
        for (r = 0; r < K; r++)
            for (g = 0; g < GN; g++) bad += sbw[blocked(r, g, GN)] != sw_ref[g * GK + r / 128];
        CHECK(bad == 0, "quant_weight: %lld bytes differ from the oracle", (long long)bad);
        bad = 0;
        for (i = 0; i < M * K; i++) bad += q2[i] != qx[i];
        for (r = 0; r < M; r++)
            for (g = 0; g < GK; g++) bad += s2[blocked(r, g, GK)] != sx[blocked(r, g, GK)];
        for (i = 0; i < K * LDT; i++) bad += qt2[i] != qxt[i];
        for (r = 0; r < K; r++)
            for (g = 0; g < GM; g++) bad += st2[blocked(r, g, GM)] != sxt[blocked(r, g, GM)];
        CHECK(bad == 0, "quant_act_static_scratch: %lld bytes differ from quant_act",
              (long long)bad);
        {
            uint32_t ctr[2];
            CUDA_OK(cudaMemcpy(ctr, d_ctr, 8, cudaMemcpyDeviceToHost));
            CHECK(ctr[0] == 0 && ctr[1] == 0, "the tile counter is left zero");
        }
        free(qx); free(sx); free(qxt); free(sxt); free(qdy); free(sdy); free(qdyt); free(sdyt);
        free(qw); free(sw); free(qwt); free(sfw); free(sbw); free(q2); free(s2); free(qt2);
        free(st2);
    }

    /* the GEMMs against the FP64 products of the oracle's dequantized operands */
    {
        double *xd = malloc(sizeof(double) * M * K), *wd = malloc(sizeof(double) * N * K);
        double *dyd = malloc(sizeof(double) * M * N), *dytd = malloc(sizeof(double) * N * M);
        double *xtd = malloc(sizeof(double) * K * M);
        double *y_ref = malloc(sizeof(double) * M * N), *dx_ref = malloc(sizeof(double) * M * K);
        double *dw_ref = malloc(sizeof(double) * N * K);
        int64_t *rows = malloc(sizeof(int64_t) * (M > N ? M : N));
        uint16_t *y = host_get(d_y, sizeof(uint16_t) * M * N);
        uint16_t *dx = host_get(d_dx, sizeof(uint16_t) * M * K);
        uint16_t *dw = host_get(d_dw, sizeof(uint16_t) * N * K);
        uint16_t *dx2 = host_get(d_dx2, sizeof(uint16_t) * M * K);
        uint16_t *dw2 = host_get(d_dw2, sizeof(uint16_t) * N * K);
        for (i = 0; i < (M > N ? M : N); i++) rows[i] = i;
        oracle_dequant_groups(q_ref, M, K, s_ref, xd);
        oracle_dequant_groups(qdy_ref, M, N, sdy_ref, dyd);
        oracle_dequant_groups(qdyt_ref, N, M, sdyt_ref, dytd);
        oracle_dequant_groups(qt_ref, K, M, st_ref, xtd);
        oracle_dequant_blocks(qw_ref, N, K, sw_ref, wd);
        oracle_gemm_fprop(xd, wd, M, N, K, rows, M, y_ref);
        oracle_gemm_dgrad(dyd, wd, M, N, K, rows, M, dx_ref);
        oracle_gemm_wgrad(dytd, xtd, M, N, K, rows, N, dw_ref);
        check_gemm("fprop", y, N, y_ref, M, N);
        check_gemm("dgrad", dx, K, dx_ref, M, K);
        check_gemm("wgrad", dw, K, dw_ref, N, K);
        CHECK(memcmp(dx, dx2, sizeof(uint16_t) * M * K) == 0,
              "the one-launch dgrad differs from the separate call");
        CHECK(memcmp(dw, dw2, sizeof(uint16_t) * N * K) == 0,
              "the one-launch wgrad differs from the separate call");
        free(xd); free(wd); free(dyd); free(dytd); free(xtd); free(y_ref); free(dx_ref);
        free(dw_ref); free(rows); free(y); free(dx); free(dw); free(dx2); free(dw2);
    }

    free(x); free(w); free(dy); free(q_ref); free(s_ref); free(qt_ref); free(st_ref);
    free(qdy_ref); free(sdy_ref); free(qdyt_ref); free(sdyt_ref); free(qw_ref); free(sw_ref);
    CUDA_OK(cudaDeviceSynchronize());
}
#endif /* ABI_CONSUMER_GPU */

int main(void)
{
    host_checks();
#ifdef ABI_CONSUMER_GPU
    gpu_checks();
#endif
    if (g_fail) return 1;
#ifdef ABI_CONSUMER_GPU
    printf("abi_consumer: gpu ok\n");
#else
    printf("abi_consumer: host ok\n");
#endif
    return 0;
}
