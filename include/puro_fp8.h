/*
 * puro_fp8.h -- C ABI of the block-scaled FP8 linear layer for NVIDIA B200
 * (sm_100a).
 *
 * The method (Puro-2B report; paper.rainbus.top summary, background
 * "FP8 块级混合精度训练" and "方法步骤详情" step (3); ta-paperlens explainer
 * §3.2; paperlayer.ai summary, Appendix C "FP8 implementation pipeline"):
 * the fprop, dgrad and wgrad GEMMs of every transformer linear layer run in
 * E4M3 FP8.  Activations and gradients carry one power-of-two scale per 128
 * consecutive values along the GEMM reduction dimension, weights one per
 * 128x128 block; scales are computed online from the BF16 tensor.  This
 * library implements that hot path: the quantizers and the three GEMMs
 * (FP32 accumulation, BF16 output).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer is a DEVICE pointer owned by the caller.  The library never
 *    allocates or frees memory on a call.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream).  Nothing synchronizes the host except
 *    puro_fp8_device_status().
 *  - Errors are returned as puro_status codes; nothing throws or aborts.  An
 *    argument error is detected on the host and returns before any launch.
 *  - Calls work on the calling thread's current CUDA device.  Several host
 *    threads may call the library at once (each with its own stream): the
 *    per-device state (device checks, kernel attributes, launch limits) is
 *    set up once behind a mutex or atomics, and launch parameters are
 *    per-thread.
 *  - Element formats:
 *      BF16   : IEEE binary32 upper half (torch.bfloat16).
 *      E4M3   : OCP FP8 "FN" (torch.float8_e4m3fn): bias 7, max 448, NaN 0x7F
 *               and 0xFF, no infinity.  Round to nearest even, saturating.
 *      UE8M0  : one byte b per scale, scale = 2^(b - 127).  b = e + 127 where e
 *               is the smallest integer with amax <= 448 * 2^e over the group,
 *               clamped to [-127, 127]; an all-zero group has e = 0 (b = 127).
 *               0xFF is never produced.
 *  - Matrices are row-major; every leading dimension (`ld_*`) is in ELEMENTS
 *    of the array it describes (bytes for FP8 arrays) and must make each row
 *    start on a 16-byte boundary.  Every pointer must be 16-byte aligned.
 *  - Scale arrays a GEMM reads are stored in the BLOCKED layout that the
 *    tensor core's block-scaled MMA consumes (the MX scale-factor layout):
 *    for an operand with `rows` rows and `groups` 128-wide groups along its
 *    reduction dimension, the scale of (row r, group g) is the byte at
 *        ((r / 128) * G4 + g / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + g % 4
 *    with G4 = ceil(groups / 4); the array holds ceil(rows / 128) * G4 * 512
 *    bytes (puro_fp8_blocked_scale_bytes).  Every 512-byte chunk covers 128
 *    rows x 4 groups, so a GEMM tile loads its scales as whole chunks.
 *    Bytes of groups >= `groups` are never written; bytes of rows >= `rows`
 *    in the last chunk are written as 127 by the activation quantizer.
 *  - The canonical weight scale array is compact row-major [n/128, k/128];
 *    the weight quantizer can also write it expanded to one byte per row in
 *    the blocked layout, once per GEMM that reads the weight.
 */
#ifndef PURO_FP8_H
#define PURO_FP8_H

#include <stdint.h>

#if defined(__GNUC__)
#define PURO_API __attribute__((visibility("default")))
#else
#define PURO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PURO_OK = 0,
    PURO_ERR_NULL = -1,               /* a required pointer is NULL               */
    PURO_ERR_ALIGN = -2,              /* pointer or leading dim not 16-B aligned   */
    PURO_ERR_SHAPE = -3,              /* a size or leading dim is out of range     */
    PURO_ERR_LAYOUT = -4,             /* unknown layout flag                       */
    PURO_ERR_CUDA = -5,               /* a CUDA runtime/driver call failed         */
    PURO_ERR_UNSUPPORTED_DEVICE = -6, /* current device is not sm_100              */
    PURO_ERR_DEVICE_TIMEOUT = -7      /* a bounded on-device wait expired          */
} puro_status;

/* Layout flags of puro_fp8_quant_act. */
enum {
    PURO_ROWWISE = 1,  /* groups of 128 along cols, codes kept in place          */
    PURO_COLWISE = 2,  /* groups of 128 along rows, codes written transposed     */
    PURO_BOTH = 3      /* both outputs from one read of x                         */
};

/* Bytes of a blocked scale array for `rows` rows and `groups` groups
 * (ceil(rows/128) * ceil(groups/4) * 512); 0 if either is <= 0.  A support
 * call of this library's storage layout; the pages have no counterpart. */
PURO_API int64_t puro_fp8_blocked_scale_bytes(int64_t rows, int64_t groups);

/*
 * puro_fp8_quant_act -- online 1x128 quantization of an activation or
 * gradient: one scale for every 128 consecutive values along the GEMM
 * reduction dimension, for activations and for gradients alike (ta-paperlens
 * explainer §3.2; the 1-D groups of paper.rainbus.top, "方法步骤详情" step (3)).
 *
 * x      : BF16 [rows, cols], row stride ld_x elements (ld_x >= cols).
 * layout : PURO_ROWWISE, PURO_COLWISE or PURO_BOTH.  cols % 128 == 0.
 *
 * ROWWISE output (the fprop/dgrad operand: the reduction dim is cols):
 *   q  : E4M3 [rows, cols], row stride ld_q bytes (ld_q >= cols).
 *   s  : blocked scales, `rows` rows x cols/128 groups; group (r, g) is
 *        x[r, 128g .. 128g+127].
 * COLWISE output (the wgrad operand: the reduction dim is rows = tokens):
 *   qt : E4M3 [cols, ld_qt], ld_qt >= rows rounded up to 16; qt[c*ld_qt + r]
 *        is the code of x[r, c].  Bytes [rows, round_up(rows,16)) of each row
 *        are written as 0; bytes beyond are not touched.
 *   st : blocked scales, `cols` rows x ceil(rows/128) groups; group (c, g) is
 *        x[128g .. min(128g+127, rows-1), c] -- the last group may be short
 *        and only its valid rows enter the amax.
 * Unused outputs may be NULL.  rows == 0 or cols == 0 is a no-op.
 *
 * tile_counter : NULL, or two 32-bit words of device memory, 8-byte aligned,
 *   owned by the caller and zero before the first call that gets them.  On
 *   long inputs (more than about 16 tiles of 128 x 128 per SM) the call then
 *   hands the tiles out by ticket from this counter, which keeps every SM
 *   busy to the end; NULL, or a shorter input, takes a static tile schedule.
 *   The results are the same either way.  Every call that completes leaves
 *   the words zero (the CTA that draws the last ticket clears the counter), so
 *   one counter serves any number of calls in stream order (CUDA graph
 *   replays included); after a call that reported PURO_ERR_DEVICE_TIMEOUT,
 *   clear it before using it again.  Calls that may run at the same time on
 *   the GPU need distinct counters -- one per output set is natural, since
 *   such calls need distinct outputs anyway.
 * Limits: rows, cols < 2^31.
 */
PURO_API int puro_fp8_quant_act(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                int layout, void* q, int64_t ld_q, void* s,
                                void* qt, int64_t ld_qt, void* st, uint32_t* tile_counter,
                                void* stream);

/*
 * puro_fp8_quant_act_static_scratch -- puro_fp8_quant_act for callers that
 * cannot provide the tile counter's eight bytes of device memory.  (A support
 * call of this library; the paper has no counterpart.)
 *
 * Who needs it: a caller that owns no device memory besides its inputs and
 * outputs -- an engine that hands the GPU's memory to its own pool at
 * start-up, so that a cudaMalloc would fail or stall the device, or a C
 * caller that was only given the buffers it works on.  Passing a NULL
 * tile_counter to puro_fp8_quant_act also allocates nothing, but then long
 * inputs run on the static tile schedule, which waits for the slowest SM.
 *
 * Arguments, layouts, results and errors are those of puro_fp8_quant_act.
 * The counter lives in a 256-byte array in this library's device memory
 * (one counter pair is used; every GPU that loads the library holds the
 * array until the process exits).  Nothing is allocated: no cudaMalloc,
 * cudaFree or allocating library call.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - Every call clears the counter on `stream` before its kernel.  All calls
 *   share the one array, so calls whose kernels may overlap on the GPU
 *   (other streams) race on it and must not be made; stream-ordered calls are
 *   safe.
 * - Limit: fewer than 2^31 tiles of 128 x 128 (the counter hands out 32-bit
 *   tickets), as for puro_fp8_quant_act; larger inputs return PURO_ERR_SHAPE.
 */
PURO_API int puro_fp8_quant_act_static_scratch(const void* x, int64_t rows, int64_t cols,
                                               int64_t ld_x, int layout, void* q, int64_t ld_q,
                                               void* s, void* qt, int64_t ld_qt, void* st,
                                               void* stream);

/*
 * puro_fp8_quant_weight -- 128x128 block quantization of a weight: one
 * power-of-two scale, computed online, for each 128x128 block
 * (paper.rainbus.top summary, background "FP8 块级混合精度训练" and
 * "方法步骤详情" step (3)).
 *
 * w     : BF16 [n, k], row stride ld_w elements; n % 128 == 0, k % 128 == 0.
 * q     : E4M3 [n, k], row stride ld_q bytes.
 * s     : UE8M0 [n/128, k/128] compact row-major; s[bn*(k/128) + bk].
 * qt    : optional (NULL to skip) E4M3 [k, n], row stride ld_qt bytes, the byte
 *         transpose of q -- the K-contiguous weight operand of dgrad.  The
 *         blocks are square, so block (bk, bn) of qt has the scale
 *         s[bn*(k/128) + bk].
 * s_fwd : optional blocked scales of q as the fprop B operand: n rows x k/128
 *         groups, row j of group kb holding s[(j/128)*(k/128) + kb].
 * s_bwd : optional blocked scales of qt as the dgrad B operand: k rows x n/128
 *         groups, row j of group nb holding s[nb*(k/128) + j/128].
 */
PURO_API int puro_fp8_quant_weight(const void* w, int64_t n, int64_t k, int64_t ld_w,
                                   void* q, int64_t ld_q, void* s,
                                   void* qt, int64_t ld_qt, void* s_fwd, void* s_bwd,
                                   void* stream);

/*
 * puro_fp8_gemm_fprop -- Y = X W^T (forward GEMM of paperlayer.ai Appendix C).
 *   Y[i,j] = sum_kb 2^(ex[i,kb] + ew[j/128,kb]) * sum_{k in kb} qx[i,k] qw[j,k]
 * accumulated in FP32 on the tensor cores, rounded once to BF16 (RNE).
 * qx : E4M3 [m, k] (ld_qx),  sx    : blocked, m rows x k/128 groups (quant_act ROWWISE of X)
 * qw : E4M3 [n, k] (ld_qw),  sw_fwd: blocked, n rows x k/128 groups (quant_weight s_fwd)
 * y  : BF16 [m, n], row stride ld_y elements.
 * k % 128 == 0, n % 128 == 0; any m >= 0 (rows >= m are neither read nor written).
 */
PURO_API int puro_fp8_gemm_fprop(const void* qx, int64_t ld_qx, const void* sx,
                                 const void* qw, int64_t ld_qw, const void* sw_fwd,
                                 void* y, int64_t ld_y, int64_t m, int64_t n, int64_t k,
                                 void* stream);

/*
 * puro_fp8_gemm_dgrad -- dX = dY W, the data-gradient GEMM (paperlayer.ai
 * summary, Appendix C "FP8 implementation pipeline": the forward,
 * data-gradient and weight-gradient GEMMs all run in blockwise E4M3;
 * paper.rainbus.top summary, "方法步骤详情" step (3): Dgrad in E4M3).  Its
 * reduction runs over n, so dY carries its 1x128 row-wise groups along n and
 * the weight its 128x128 blocks, read through the transposed codes.
 * qdy : E4M3 [m, n] (ld_qdy), sdy   : blocked, m rows x n/128 groups (quant_act ROWWISE of dY)
 * qwt : E4M3 [k, n] (ld_qwt), sw_bwd: blocked, k rows x n/128 groups (quant_weight qt, s_bwd)
 * dx  : BF16 [m, k], row stride ld_dx elements.
 * k % 128 == 0, n % 128 == 0; any m >= 0.
 */
PURO_API int puro_fp8_gemm_dgrad(const void* qdy, int64_t ld_qdy, const void* sdy,
                                 const void* qwt, int64_t ld_qwt, const void* sw_bwd,
                                 void* dx, int64_t ld_dx, int64_t m, int64_t n, int64_t k,
                                 void* stream);

/*
 * puro_fp8_gemm_wgrad -- dW = dY^T X (weight-gradient GEMM, reduction over the
 * m tokens, both operands quantized along m as ta-paperlens §3.2 prescribes
 * for gradients and activations).
 * qdyt : E4M3 [n, ld_qdyt], sdyt : blocked, n rows x ceil(m/128) groups (COLWISE of dY)
 * qxt  : E4M3 [k, ld_qxt],  sxt  : blocked, k rows x ceil(m/128) groups (COLWISE of X)
 * dw   : BF16 [n, k], row stride ld_dw elements.
 * n % 128 == 0, k % 128 == 0; any m >= 0 (a short last token group is read
 * with zero padding; m == 0 writes dW = 0).
 */
PURO_API int puro_fp8_gemm_wgrad(const void* qdyt, int64_t ld_qdyt, const void* sdyt,
                                 const void* qxt, int64_t ld_qxt, const void* sxt,
                                 void* dw, int64_t ld_dw, int64_t m, int64_t n, int64_t k,
                                 void* stream);

/*
 * puro_fp8_gemm_wgrad_f32 -- the weight-gradient GEMM with an FP32 result:
 *   accumulate == 0 : dW  = dY^T X
 *   accumulate == 1 : dW += dY^T X   (accumulation into an FP32 gradient
 *                                     buffer across micro-batches)
 * The pages keep gradients in FP32 while the three linear-layer GEMMs run in
 * E4M3 (paperlayer.ai Appendix C, "Production Training Details", the FP8
 * implementation pipeline; micro-batch size 2 under a 1,536-sequence global
 * batch in the same appendix, hence the accumulation).
 * Operands as puro_fp8_gemm_wgrad.  dw : FP32 [n, k], row stride ld_dw
 * elements (ld_dw * 4 a multiple of 16 bytes), caller-owned, 16-byte aligned.
 * Each element receives exactly one FP32 store or one FP32 add per call (the
 * add is done by the memory system, as a TMA reduce-add), so repeated calls
 * give the same result for the same inputs.  m == 0: dW = 0, or unchanged
 * when accumulating.  accumulate other than 0/1 -> PURO_ERR_LAYOUT.
 */
PURO_API int puro_fp8_gemm_wgrad_f32(const void* qdyt, int64_t ld_qdyt, const void* sdyt,
                                     const void* qxt, int64_t ld_qxt, const void* sxt,
                                     void* dw, int64_t ld_dw, int64_t m, int64_t n, int64_t k,
                                     int accumulate, void* stream);

/* Output kinds of the weight gradient in puro_fp8_gemm_dgrad_wgrad. */
enum {
  PURO_DW_BF16 = 0,            /* dW = dY^T X, BF16 (as puro_fp8_gemm_wgrad)               */
  PURO_DW_F32 = 1,             /* dW = dY^T X, FP32 (as puro_fp8_gemm_wgrad_f32, acc. 0)   */
  PURO_DW_F32_ACCUMULATE = 2   /* dW += dY^T X, FP32 (as puro_fp8_gemm_wgrad_f32, acc. 1)  */
};

/*
 * puro_fp8_gemm_dgrad_wgrad -- the two backward GEMMs of one linear layer
 * (the data- and weight-gradient GEMMs of paperlayer.ai Appendix C) in one
 * launch: dX = dY W (arguments and result exactly as puro_fp8_gemm_dgrad)
 * and dW = dY^T X (as puro_fp8_gemm_wgrad, or the FP32 forms, by dw_kind).
 * The two are independent given the quantized dY, X and W.  Sharing the launch
 * only changes which SM computes which output tile: the tiles of both are
 * assigned to the clusters longest-first (by K blocks) to the least-loaded
 * cluster, so that neither GEMM leaves most of the GPU idle in a last,
 * partly-filled wave of tiles.  Every output element is computed exactly as in
 * the separate calls (bit-identical results).
 * m, n, k: tokens, layer outputs, layer inputs (dY [m, n], X [m, k], W [n, k]).
 * Errors as the separate calls; dw_kind outside PURO_DW_* -> PURO_ERR_LAYOUT.
 * If either product is empty the other one runs on its own.
 */
PURO_API int puro_fp8_gemm_dgrad_wgrad(const void* qdy, int64_t ld_qdy, const void* sdy,
                                       const void* qwt, int64_t ld_qwt, const void* sw_bwd,
                                       void* dx, int64_t ld_dx,
                                       const void* qdyt, int64_t ld_qdyt, const void* sdyt,
                                       const void* qxt, int64_t ld_qxt, const void* sxt,
                                       void* dw, int64_t ld_dw,
                                       int64_t m, int64_t n, int64_t k, int dw_kind,
                                       void* stream);

/*
 * Support calls (error reporting and self-tests of this library; the pages
 * have no counterpart).
 *
 * puro_fp8_device_status -- synchronizes `stream`, then returns and clears the
 * library's device error word for the current device: PURO_OK, or
 * PURO_ERR_DEVICE_TIMEOUT if a kernel gave up a bounded wait since the last
 * call (that kernel's output is then undefined), or PURO_ERR_CUDA if the
 * synchronization itself failed.
 */
PURO_API int puro_fp8_device_status(void* stream);

/* Human-readable name of a puro_status code (static storage). */
PURO_API const char* puro_fp8_status_string(int status);

/*
 * puro_fp8_test_bounded_wait -- self-test of the bounded-wait machinery: launches
 * one block that waits on a shared-memory barrier nothing will ever arrive on,
 * with a limit of `limit_ns` nanoseconds (clamped to [1e3, 5e9]).  The wait
 * must give up, record PURO_ERR_DEVICE_TIMEOUT in the device error word and
 * return; puro_fp8_device_status() then reports it.  Nothing faults or traps.
 */
PURO_API int puro_fp8_test_bounded_wait(int64_t limit_ns, void* stream);

/*
 * puro_fp8_test_schedule -- host-only view of how a two-problem GEMM launch
 * (puro_fp8_gemm_dgrad_wgrad) spreads its work units over the launch's
 * clusters.  Problem 0 has `units0` units of `kblocks0` K blocks each, problem
 * 1 `units1` units of `kblocks1`; units [0, units0) are problem 0's.  The
 * units are taken longest first (cost = K blocks + 2, ties in unit order) and
 * each goes to the least-loaded cluster so far (ties: lowest cluster index).
 * On return cluster c runs units[offsets[c] .. offsets[c + 1]) in that order.
 *   offsets : host array of clusters + 1 entries (written)
 *   units   : host array of units0 + units1 entries (written)
 * No device work.  PURO_ERR_NULL for a null array; PURO_ERR_SHAPE unless
 * 1 <= clusters <= 128, units0, units1, kblocks0, kblocks1 >= 0 and
 * units0 + units1 <= 2048 (the launch schedules at most that many units and
 * falls back to round robin beyond).
 */
PURO_API int puro_fp8_test_schedule(int32_t units0, int32_t kblocks0, int32_t units1,
                                    int32_t kblocks1, int32_t clusters, int32_t* offsets,
                                    int32_t* units);

#ifdef __cplusplus
}
#endif

#endif /* PURO_FP8_H */
