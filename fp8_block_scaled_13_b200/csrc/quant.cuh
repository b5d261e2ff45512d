// Online BF16 -> E4M3 quantizers with power-of-two (UE8M0) scales.
//
// Method: Puro-2B report -- paper.rainbus.top summary, background
// "FP8 块级混合精度训练" and "方法步骤详情" step (3); ta-paperlens explainer §3.2.
// Activations and gradients get one scale per 128 values along the GEMM
// reduction dimension, weights one per 128x128 block; the scale 2^e is the
// smallest power of two with amax <= 448 * 2^e (so nothing saturates),
// e clamped to [-127, 127], and every element is encoded round-to-nearest-even
// with saturation.
//
// One persistent kernel serves every layout.  Each CTA (256 threads; two or
// three per SM, so as many tiles are processed side by side) walks a list of
// 128x128 tiles of the BF16 input; a TMA ring of STAGES 32 KB tile buffers
// keeps the next tiles in flight while the current one is processed, and a
// stage is handed back to the TMA as soon as every thread has copied its part
// into registers.  Long tile streams run one stage and three CTAs per SM (the
// next tile's load still has a whole tile's processing time to land, and the
// third CTA hides more latency: 2-3% faster on 4096+ tiles), the tiles after
// each CTA's first handed out by ticket; short streams keep two stages, two
// CTAs per SM and a static list (the first tiles are also prefetched into L2
// before the kernel waits on its predecessor).  Thread (i, j) = (tid/16,
// tid%16) holds rows 8i..8i+7 and columns 8j..8j+7.  From those registers:
//   ROW   : row amax by a 16-lane shuffle reduction; codes stored in place.
//   COL   : column amax by a shuffle + shared-memory reduction over the 8
//           warps; codes transposed through a swizzled 16 KB shared tile
//           (conflict-free 8-byte writes) that one TMA tensor store writes
//           out (a 3-D view of the transposed matrix whose swizzle matches
//           the staging layout).  The transposed tile is double-buffered and
//           stored at the start of the next tile, after the barrier every
//           tile starts with anyway.
//   BLOCK : one amax over the whole tile (128x128 weight block); codes written
//           in place and, optionally, transposed.
// Per tile the block meets at three barriers: stage consumed (which also
// publishes the previous tile's transposed codes), column partial maxima
// published, column scales published.  The column scales are reduced by 64
// threads while the others already encode their rows.
// The amax is taken with the max-of-absolute-values instruction on BF16
// pairs and then compared as integer magnitude bits (|x| is itself a BF16,
// and the order of non-negative floats equals the order of their bits), and
// the scale exponent comes from the exponent/mantissa fields alone, two
// groups per 32-bit word: with amax = 1.f * 2^E, e = E - 8 if 1.f <= 1.75
// (mantissa bits <= 0x60), else E - 7.  Scaling by 2^-e is an exact
// BF16 x BF16 -> FP32 fused multiply-add (no flush to zero: this file must
// not be built with fast-math), followed by one hardware round-to-nearest-even,
// saturating conversion to E4M3 per value.
#pragma once

#include "common.cuh"

namespace puro {

// 256 threads: 16 threads cover a 128-column row chunk (8 columns each) and
// 16 row groups of 8 rows cover the 128-row tile.  (4 rows per thread with 512
// threads and 64 registers was measured slower for the BOTH layout.)
constexpr int kQThreads = 256;
constexpr uint32_t kQTileBytes = 128 * 128 * 2;
constexpr uint32_t kQtTileBytes = 128 * 128;  // one transposed code tile

struct QuantParams {
  int64_t rows, cols;
  uint8_t* q;   // codes, same orientation as x (ROW / BLOCK)
  int64_t ld_q;
  uint8_t* s;   // ROW: blocked scales, rows x cols/128 groups
  int64_t s_g4;  // ceil(groups / 4) of s
  uint8_t* qt;  // transposed codes [cols][ld_qt] (COL / BLOCK with transpose)
  int64_t ld_qt;
  uint8_t* st;  // COL: blocked scales, cols x ceil(rows/128) groups
  int64_t st_g4;
  uint8_t* sw;  // BLOCK: compact scales [rows/128][cols/128]
  uint8_t* sw_fwd;  // BLOCK: optional blocked, rows x cols/128 groups
  int64_t fwd_g4;
  uint8_t* sw_bwd;  // BLOCK: optional blocked, cols x rows/128 groups
  int64_t bwd_g4;
  int32_t tiles_c, tiles;
  // Row tile of tile t without a division: t / tiles_c == umulhi(t,
  // tc_magic) >> tc_shift for every t < 2^31 when tiles_c > 1 (set by the
  // launcher: l = ceil(log2(tiles_c)), tc_magic = ceil(2^(31+l) / tiles_c),
  // tc_shift = l - 1; the product's error stays below 1 / tiles_c).  The
  // producer thread decodes every tile it loads, and the rest of the block
  // waits for it at the stage barrier: a 32-bit division there cost ~2 us per
  // 4096-tile launch.
  uint32_t tc_magic;
  int32_t tc_shift;
  // Optional tile counter (a zeroed 32-bit word; null: static schedule),
  // used with one stage only.  Each CTA takes its first tile statically and
  // the rest by ticket, so SMs that stream faster take more tiles.  Tickets
  // 0 .. tiles-1 go out in order (the valid ones map to tiles gridDim.x ..
  // tiles-1, and each CTA stops at its first invalid one), so the CTA that
  // draws ticket tiles-1 knows every other CTA has drawn its last, and sets
  // the counter back to zero.
  uint32_t* ctr;
};

// Scale exponents of two groups at once.  a2 holds two amax magnitudes (BF16
// bits, sign cleared) in its 16-bit halves; each half of the result is
// k = 127 - e, the FP32 exponent field of 2^-e: with t the biased exponent
// field and c = (mantissa > 0x60), e = t - 135 + c, clamped to e >= -127
// (k <= 254; a subnormal amax always clamps).  The largest finite BF16 gives
// k = 7, so no upper clamp is needed.  A zero amax also comes out as
// k = 254; its codes are zero for any scale, and its scale byte is fixed up
// by scale_bytes2.
__device__ __forceinline__ uint32_t scale_k2(uint32_t a2) {
  const uint32_t t2 = (a2 >> 7) & 0x00FF00FFu;
  const uint32_t c2 = (((a2 & 0x007F007Fu) + 0x001F001Fu) >> 7) & 0x00010001u;
  return __vminu2(0x01060106u - t2 - c2, 0x00FE00FEu);
}

// UE8M0 scale bytes e + 127 = 254 - k of the two groups of scale_k2, with the
// zero-amax rule (e = 0, byte 127) applied; one byte in each 16-bit half.
__device__ __forceinline__ uint32_t scale_bytes2(uint32_t a2, uint32_t k2) {
  const uint32_t z2 = __vcmpeq2(a2, 0u);
  return ((0x00FE00FEu - k2) & ~z2) | (0x007F007Fu & z2);
}

// 2^-e of the low / high group of scale_k2 as an FP32.
__device__ __forceinline__ float scale_lo(uint32_t k2) { return __uint_as_float(k2 << 23); }
__device__ __forceinline__ float scale_hi(uint32_t k2) { return __uint_as_float((k2 << 7) & 0x7F800000u); }

// 2^-e as BF16 bits, from its FP32 form (exact: a power of two with e in
// [-127, 120] is a normal BF16).
__device__ __forceinline__ uint16_t bf16_bits(float f) {
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

// Encoding x * 2^-e to E4M3: fma.rn.f32.bf16 forms the product of the BF16
// value and the BF16 scale exactly in FP32 (two 8-bit significands fit in
// FP32's 24; subnormals kept) and adds -0.0, which leaves every value and the
// sign of zero unchanged; then one round-to-nearest-even, saturating
// conversion per value.  Taking the BF16 operand straight from a half of the
// loaded word saves the separate widening to FP32 (measured: one instruction
// per element less than widening and a packed FP32 multiply); the codes are
// the same for every BF16 value and every scale (checked exhaustively).
// The two 16-bit results are joined by a register move.

// Four codes of the BF16 pairs w01 = (x0, x1) and w23 = (x2, x3), x0 in the
// low byte.
__device__ __forceinline__ uint32_t encode4_pairs(uint32_t w01, uint32_t w23, uint16_t s) {
  uint32_t r;
  asm("{\n\t.reg .b16 a0, a1, b0, b1, lo, hi;\n\t.reg .f32 f0, f1, f2, f3;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.bf16 f0, a0, %3, 0f80000000;\n\t"
      "fma.rn.f32.bf16 f1, a1, %3, 0f80000000;\n\t"
      "fma.rn.f32.bf16 f2, b0, %3, 0f80000000;\n\t"
      "fma.rn.f32.bf16 f3, b1, %3, 0f80000000;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, f1, f0;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, f3, f2;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "r"(w01), "r"(w23), "h"(s));
  return r;
}

// Four codes of one half (H = 0: low, 1: high) of the words w0..w3 -- one
// column of four consecutive rows -- w0's in the low byte.
template <int H>
__device__ __forceinline__ uint32_t encode4_col(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3,
                                                uint16_t s) {
  uint32_t r;
  if (H == 0)
    asm("{\n\t.reg .b16 x0, x1, x2, x3, y0, y1, y2, y3, lo, hi;\n\t.reg .f32 f0, f1, f2, f3;\n\t"
        "mov.b32 {x0, y0}, %1;\n\t"
        "mov.b32 {x1, y1}, %2;\n\t"
        "mov.b32 {x2, y2}, %3;\n\t"
        "mov.b32 {x3, y3}, %4;\n\t"
        "fma.rn.f32.bf16 f0, x0, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f1, x1, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f2, x2, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f3, x3, %5, 0f80000000;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, f1, f0;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, f3, f2;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "h"(s));
  else
    asm("{\n\t.reg .b16 x0, x1, x2, x3, y0, y1, y2, y3, lo, hi;\n\t.reg .f32 f0, f1, f2, f3;\n\t"
        "mov.b32 {y0, x0}, %1;\n\t"
        "mov.b32 {y1, x1}, %2;\n\t"
        "mov.b32 {y2, x2}, %3;\n\t"
        "mov.b32 {y3, x3}, %4;\n\t"
        "fma.rn.f32.bf16 f0, x0, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f1, x1, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f2, x2, %5, 0f80000000;\n\t"
        "fma.rn.f32.bf16 f3, x3, %5, 0f80000000;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, f1, f0;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, f3, f2;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "r"(w0), "r"(w1), "r"(w2), "r"(w3), "h"(s));
  return r;
}

__device__ __forceinline__ uint32_t word(const uint4& v, int idx) {
  return idx == 0 ? v.x : idx == 1 ? v.y : idx == 2 ? v.z : v.w;
}

// Eight codes of one 8-element row chunk, all scaled by 2^-e (BF16 bits s).
__device__ __forceinline__ uint2 encode_row8(const uint4& v, uint16_t s) {
  uint2 o;
  o.x = encode4_pairs(v.x, v.y, s);
  o.y = encode4_pairs(v.z, v.w, s);
  return o;
}

// Eight codes of column l of the thread's 8x8 block (rows 0..7), scaled by s.
template <int L>
__device__ __forceinline__ uint2 encode_col8(const uint4 (&v)[8], uint16_t s) {
  uint2 o;
  o.x = encode4_col<L & 1>(word(v[0], L >> 1), word(v[1], L >> 1), word(v[2], L >> 1), word(v[3], L >> 1), s);
  o.y = encode4_col<L & 1>(word(v[4], L >> 1), word(v[5], L >> 1), word(v[6], L >> 1), word(v[7], L >> 1), s);
  return o;
}

// Magnitude maximum of two BF16 pairs, half by half, with the float
// max-of-absolute-values instruction on the raw words: the result's halves
// hold the larger |.| (its sign bits are the xor of the inputs' and are
// cleared once at the end).  Measured 0.36 fewer instructions per element
// than masking every word and taking integer maxima (the order of
// non-negative BF16 values is the order of their bits, so both give the same
// amax; NaN inputs are outside the contract).
__device__ __forceinline__ uint32_t amax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Larger of the two 16-bit halves.
__device__ __forceinline__ uint32_t hmax(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ uint4 lds_v4(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ int32_t tile_row(const QuantParams& p, int32_t t) {
  return p.tiles_c == 1 ? t : (int32_t)(__umulhi((uint32_t)t, p.tc_magic) >> p.tc_shift);
}

// Byte offset, inside one 512-byte chunk of a blocked scale array, of the
// chunk's row r (0..127).
__device__ __forceinline__ uint32_t blocked_in_chunk(int r) {
  return static_cast<uint32_t>((r & 31) * 16 + ((r >> 5) & 3) * 4);
}

// RSHFL marks the row-scale form of activation launches (ROW without BLOCK):
// the 16 lanes of a row group reduce-scatter the row maxima, one lane per row
// derives the exponent and the others read 2^-e with shuffles.  (An earlier
// form had every lane derive its own 8 rows' exponents after a butterfly:
// faster at two CTAs per SM on long streams, 7% more instructions, and slower
// at three CTAs per SM.)  Weight blocks take one scale for the whole tile.
//
// Addressing is kept out of the per-element work: every output pointer is
// formed once per tile from per-thread constants and advanced by its stride,
// and the ragged-edge tests are one 32-bit compare against a per-tile count.
template <bool ROW, bool COL, bool BLOCK, bool RSHFL, int STAGES>
__global__ void __launch_bounds__(kQThreads, STAGES == 1 ? 3 : 2)
    quant_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_qt,
                 const QuantParams p) {
  static_assert(!ROW || BLOCK || RSHFL, "activation row scales are shared by shuffles");
  constexpr int kWarps = kQThreads / 32;
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;                                    // STAGES x 32 KB
  uint8_t* qt_buf = smem + STAGES * kQTileBytes;            // 2 x 16 KB transposed codes
  uint32_t* col_part = reinterpret_cast<uint32_t*>(qt_buf + 2 * kQtTileBytes);  // [8 warps][16][4]
  float* col_scale = reinterpret_cast<float*>(col_part + kWarps * 64);  // [128] 2^-e per column
  uint32_t* blk_part = reinterpret_cast<uint32_t*>(col_scale + 128);    // [8]
  uint64_t* full = reinterpret_cast<uint64_t*>(blk_part + kWarps);
  int2* tile_rc = reinterpret_cast<int2*>(full + STAGES);  // [STAGES] (row, col) tile of the stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tile_rc + STAGES);

  const int tid = threadIdx.x;
  const int i = tid >> 4, j = tid & 15, warp = tid >> 5;
  // Tile t is (row tile t / tiles_c, col tile t % tiles_c).  Load k of this
  // CTA fetches tile blockIdx.x + k * gridDim.x; with a tile counter, loads
  // from STAGES on fetch tile STAGES * gridDim.x + ticket instead.  The tile
  // of each load is published in tile_rc (-1: no more tiles).
  const bool dyn = STAGES == 1 && p.ctr != nullptr;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_x);
    if (COL) prefetch_tmap(&tm_qt);
  }
  __syncthreads();
  if (tid == 0) {
    // Warm L2 with this CTA's first tiles while the kernel before this one is
    // still finishing.  A prefetch only moves data into L2, the point of
    // coherence, and the loads that fill shared memory still follow the
    // dependency wait below, so a producer's later writes are what they read.
    for (int32_t k = 0; k < STAGES; ++k) {
      const int32_t t = (int32_t)blockIdx.x + k * (int32_t)gridDim.x;
      if (t >= p.tiles) break;
      const int32_t r = tile_row(p, t);
      tma_prefetch_l2_2d(&tm_x, (t - r * p.tiles_c) * 128, r * 128);
    }
  }
  // the input may come from the kernel just before this one on the stream
  pdl_wait();
  pdl_trigger();
  // producer state (thread 0 only): loads issued, whether the end marker
  // went out, and the ticket for the next load (taken one load ahead, so its
  // round trip overlaps a tile of work)
  int32_t p_it = 0;
  bool p_end = false;
  uint32_t ticket = 0;
  auto issue_next = [&]() {
    if (p_end) return;
    const int s = p_it % STAGES;
    const bool by_ticket = dyn && p_it >= STAGES;
    const int32_t t = by_ticket ? STAGES * (int32_t)gridDim.x + (int32_t)ticket
                                : (int32_t)blockIdx.x + p_it * (int32_t)gridDim.x;
    if (by_ticket && ticket == (uint32_t)(p.tiles - 1)) atomicExch(p.ctr, 0u);
    ++p_it;
    if (t < p.tiles) {
      const int32_t r = tile_row(p, t), c = t - r * p.tiles_c;
      tile_rc[s] = make_int2(r, c);
      mbar_arrive_expect_tx(&full[s], kQTileBytes);
      tma_load_2d<1>(tiles + s * kQTileBytes, &tm_x, c * 128, r * 128, smem_u32(&full[s]));
      if (dyn && p_it >= STAGES) ticket = atomicAdd(p.ctr, 1u);
    } else {
      tile_rc[s] = make_int2(-1, -1);
      mbar_arrive(&full[s]);
      p_end = true;
    }
  };
  if (tid == 0)
    for (int k = 0; k < STAGES; ++k) issue_next();

  // per-thread constants of the output addressing
  const uint32_t s_half_chunk = blocked_in_chunk(8 * i + (j >> 1));  // the same, row j >> 1
  const uint32_t st_in_chunk = blocked_in_chunk(2 * (tid & 63));     // column scale bytes (tid < 64)

  int32_t prev_r0 = 0, prev_c0 = 0;  // the tile whose transposed codes wait in qt_buf
  int32_t it = 0;
  for (;; ++it) {
    const int s = it % STAGES;
    const bool ok = mbar_wait(&full[s], (uint32_t)((it / STAGES) & 1), abort_flag);
    const int2 rc = ok ? tile_rc[s] : make_int2(-1, -1);
    const int32_t tr = rc.x, tc = rc.y;
    const int32_t r0 = tr * 128, c0 = tc * 128;
    // this thread's 8 rows x 8 columns; rows past the end were filled with 0
    uint4 v[8];
    const uint8_t* tile = tiles + s * kQTileBytes + (8 * i) * 256 + 16 * j;
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (ok && tr >= 0) ? lds_v4(tile + k * 256) : make_uint4(0, 0, 0, 0);
    // every thread holds its part: stage s is free again, and every thread
    // has finished the previous tile, its transposed codes included (and if
    // any wait gave up, the whole block stops here together; every thread
    // read the same end marker)
    if (__syncthreads_or(!ok) || tr < 0) break;
    if (tid == 0) issue_next();
    if (COL && it > 0 && tid == 0) {
      // the previous tile's transposed codes (their writers fenced them for
      // the async proxy before the barrier above) out by one tensor store;
      // then make sure the store before it has finished reading the buffer
      // this tile's codes go to
      tma_store_3d(&tm_qt, qt_buf + ((it - 1) & 1) * kQtTileBytes, prev_r0, prev_c0 >> 3, 0);
      bulk_commit_group();
      bulk_wait_group_read<1>();
    }

    // ---- magnitudes: per-row amax of this thread's 8 columns (two rows per
    // word) and per-column-pair amax of its 8 rows
    uint32_t rowmax[4];
    uint32_t cm[4];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t a0 = v[k].x, a1 = v[k].y, a2 = v[k].z, a3 = v[k].w;
      if (ROW || BLOCK) {
        const uint32_t t = amax2(amax2(a0, a1), amax2(a2, a3));
        // rows k-1, k side by side: low halves in one word, high halves in another
        if (k & 1) {
          const uint32_t e = rowmax[k >> 1];
          rowmax[k >> 1] = amax2(__byte_perm(e, t, 0x5410), __byte_perm(e, t, 0x7632));
        } else {
          rowmax[k >> 1] = t;
        }
      }
      if (COL && !BLOCK) {
        if (k == 0) {
          cm[0] = a0; cm[1] = a1; cm[2] = a2; cm[3] = a3;
        } else {
          cm[0] = amax2(cm[0], a0);
          cm[1] = amax2(cm[1], a1);
          cm[2] = amax2(cm[2], a2);
          cm[3] = amax2(cm[3], a3);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      rowmax[q] &= 0x7FFF7FFFu;
      if (COL && !BLOCK) cm[q] &= 0x7FFF7FFFu;
    }

    // ---- partial maxima for the block-wide reductions, then one barrier
    if (COL && !BLOCK) {
#pragma unroll
      for (int pp = 0; pp < 4; ++pp)
        cm[pp] = __vmaxu2(cm[pp], __shfl_xor_sync(0xFFFFFFFFu, cm[pp], 16));
      if ((tid & 16) == 0)
        *reinterpret_cast<uint4*>(&col_part[(warp * 16 + j) * 4]) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
    }
    if (BLOCK) {
      uint32_t m = __vmaxu2(__vmaxu2(rowmax[0], rowmax[1]), __vmaxu2(rowmax[2], rowmax[3]));
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = __vmaxu2(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      if ((tid & 31) == 0) blk_part[warp] = hmax(m);
    }
    if ((COL && !BLOCK) || BLOCK) __syncthreads();

    // ---- column scales: threads 0..63 reduce columns 2t, 2t+1 over the 8
    // warps, store the two scale bytes and 2^-e for the encoders (published
    // by the next barrier; meanwhile the other warps encode their rows)
    if (COL && !BLOCK && tid < 64) {
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) m = __vmaxu2(m, col_part[(w * 16 + (tid >> 2)) * 4 + (tid & 3)]);
      const uint32_t k2 = scale_k2(m);
      const uint32_t b2 = scale_bytes2(m, k2);
      uint8_t* scol = p.st + ((int64_t)tc * p.st_g4 + (tr >> 2)) * 512 + (tr & 3) + st_in_chunk;
      scol[0] = static_cast<uint8_t>(b2);
      scol[16] = static_cast<uint8_t>(b2 >> 16);
      *reinterpret_cast<float2*>(&col_scale[2 * tid]) = make_float2(scale_lo(k2), scale_hi(k2));
    }

    int e_blk = 0;
    if (BLOCK) {
      uint32_t bm = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) bm = max(bm, blk_part[w]);
      const uint32_t k = scale_k2(bm) & 0xFFFFu;
      e_blk = 127 - (int)k;
      if (bm == 0) e_blk = 0;
      if (tid == 0) p.sw[tr * p.tiles_c + tc] = static_cast<uint8_t>(e_blk + 127);
    }

    // ---- in-place codes (ROW, BLOCK) and the row scale bytes
    if (ROW || BLOCK) {
      uint8_t* qrow = p.q + (int64_t)(r0 + 8 * i) * p.ld_q + (c0 + 8 * j);
      const int32_t nrow = (int32_t)(p.rows - r0) - 8 * i;  // rows of the block that exist
      constexpr bool kRowScatter = ROW && !BLOCK && RSHFL;
      if (kRowScatter) {
        // Reduce-scatter of the four row-pair words over the 16 lanes (lane
        // bits b3 b2 b1 b0 = j): at distance 8 a lane keeps the pair of words
        // for rows 4*b3.. and sends the other pair, at distance 4 it keeps the
        // word for rows 4*b3 + 2*b2 + {0, 1}, then distances 2 and 1 finish
        // that word.  Lane j then holds row j >> 1 in half b1 and derives its
        // exponent; even lanes store the scale byte, and row k's 2^-e is read
        // from lane 2k.
        const bool b3 = (j >> 3) & 1, b2 = (j >> 2) & 1, b1 = (j >> 1) & 1;
        uint32_t k0 = b3 ? rowmax[2] : rowmax[0], k1 = b3 ? rowmax[3] : rowmax[1];
        const uint32_t s0 = b3 ? rowmax[0] : rowmax[2], s1 = b3 ? rowmax[1] : rowmax[3];
        k0 = __vmaxu2(k0, __shfl_xor_sync(0xFFFFFFFFu, s0, 8));
        k1 = __vmaxu2(k1, __shfl_xor_sync(0xFFFFFFFFu, s1, 8));
        uint32_t w = b2 ? k1 : k0;
        w = __vmaxu2(w, __shfl_xor_sync(0xFFFFFFFFu, b2 ? k0 : k1, 4));
        w = __vmaxu2(w, __shfl_xor_sync(0xFFFFFFFFu, w, 2));
        w = __vmaxu2(w, __shfl_xor_sync(0xFFFFFFFFu, w, 1));
        const uint32_t k2 = scale_k2(w);
        const uint32_t bytes = scale_bytes2(w, k2);
        if ((j & 1) == 0)
          p.s[((int64_t)tr * p.s_g4 + (tc >> 2)) * 512 + (tc & 3) + s_half_chunk] =
              static_cast<uint8_t>(b1 ? (bytes >> 16) : bytes);
        const float s_mine = b1 ? scale_hi(k2) : scale_lo(k2);
        const int lane16 = tid & 16;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float sk = __shfl_sync(0xFFFFFFFFu, s_mine, lane16 + 2 * k);
          const uint2 o = encode_row8(v[k], bf16_bits(sk));
          if (k < nrow) *reinterpret_cast<uint2*>(qrow) = o;
          qrow += p.ld_q;
        }
      } else {
        // a weight block: one scale for every row
        const uint16_t sb = bf16_bits(__uint_as_float(static_cast<uint32_t>(127 - e_blk) << 23));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint2 o = encode_row8(v[k], sb);
          if (k < nrow) *reinterpret_cast<uint2*>(qrow) = o;
          qrow += p.ld_q;
        }
      }
    }

    // ---- transposed codes (COL, BLOCK with a transposed copy)
    if (COL) {
      if (!BLOCK) __syncthreads();   // column scales published
      float cs[8];
      if (BLOCK) {
        const float f = __uint_as_float(static_cast<uint32_t>(127 - e_blk) << 23);
#pragma unroll
        for (int l = 0; l < 8; ++l) cs[l] = f;
      } else {
        const float4 a = *reinterpret_cast<const float4*>(&col_scale[8 * j]);
        const float4 b = *reinterpret_cast<const float4*>(&col_scale[8 * j + 4]);
        cs[0] = a.x; cs[1] = a.y; cs[2] = a.z; cs[3] = a.w;
        cs[4] = b.x; cs[5] = b.y; cs[6] = b.z; cs[7] = b.w;
      }
      uint8_t* qt_s = qt_buf + (it & 1) * kQtTileBytes;
      // Transposed row c = 8j + l of the tile sits at staging row 16l + j,
      // and this thread's 8 codes of it (rows 8i..8i+7) in 8-byte chunk
      // i ^ 2(j & 7), i.e. 16-byte unit (i/2) ^ (j & 7): the 32 stores of a
      // warp fill 16 distinct chunk positions twice (two wavefronts, the
      // minimum for 256 bytes).  This is the layout the tensor store reads:
      // its map views the transposed codes as {rows, cols/8 (stride 8 rows),
      // 8 (stride 1 row)}, so staging row 16l + j is transposed row 8j + l,
      // and its 128-byte swizzle XORs unit u with staging row & 7 = j & 7.
      uint8_t* dst = qt_s + j * 128 + ((i ^ (2 * (j & 7))) << 3);
      *reinterpret_cast<uint2*>(dst + 0 * 2048) = encode_col8<0>(v, bf16_bits(cs[0]));
      *reinterpret_cast<uint2*>(dst + 1 * 2048) = encode_col8<1>(v, bf16_bits(cs[1]));
      *reinterpret_cast<uint2*>(dst + 2 * 2048) = encode_col8<2>(v, bf16_bits(cs[2]));
      *reinterpret_cast<uint2*>(dst + 3 * 2048) = encode_col8<3>(v, bf16_bits(cs[3]));
      *reinterpret_cast<uint2*>(dst + 4 * 2048) = encode_col8<4>(v, bf16_bits(cs[4]));
      *reinterpret_cast<uint2*>(dst + 5 * 2048) = encode_col8<5>(v, bf16_bits(cs[5]));
      *reinterpret_cast<uint2*>(dst + 6 * 2048) = encode_col8<6>(v, bf16_bits(cs[6]));
      *reinterpret_cast<uint2*>(dst + 7 * 2048) = encode_col8<7>(v, bf16_bits(cs[7]));
      fence_proxy_async_smem();  // visible to the tensor store after the next barrier
      prev_r0 = r0;
      prev_c0 = c0;
    }

    if (BLOCK && tid < 128) {
      const uint8_t b = static_cast<uint8_t>(e_blk + 127);
      const uint32_t in_chunk = blocked_in_chunk(tid);
      if (p.sw_fwd) p.sw_fwd[((int64_t)tr * p.fwd_g4 + (tc >> 2)) * 512 + (tc & 3) + in_chunk] = b;
      if (p.sw_bwd) p.sw_bwd[((int64_t)tc * p.bwd_g4 + (tr >> 2)) * 512 + (tr & 3) + in_chunk] = b;
    }
    // No barrier here: the shared tiles (col_part, col_scale, blk_part, the
    // other transposed buffer) are next written after the barrier at the top
    // of the next iteration, which no thread passes before every thread has
    // finished this tile.
  }
  // the last tile's transposed codes (if every wait succeeded), and every
  // tensor store complete before the block exits
  if (COL && it > 0) {
    if (!__syncthreads_or(*abort_flag != 0) && tid == 0) {
      tma_store_3d(&tm_qt, qt_buf + ((it - 1) & 1) * kQtTileBytes, prev_r0, prev_c0 >> 3, 0);
      bulk_commit_group();
    }
  }
  if (COL && tid == 0) bulk_wait_group<0>();
  // Copies are only issued for tiles this CTA processes, and each one was
  // waited for above, unless a wait gave up; then let the outstanding ones
  // land (bounded) before the block exits.
  if (tid == 0 && *abort_flag) {
    for (int s = 0; s < STAGES; ++s) {
      volatile int no_abort = 0;
      mbar_wait(&full[s], 0, &no_abort, 100000000ull);
      mbar_wait(&full[s], 1, &no_abort, 100000000ull);
    }
  }
}

// Shared memory the quantizer needs (plus alignment slack).
template <int STAGES>
constexpr uint32_t quant_smem_bytes() {
  return STAGES * kQTileBytes + 2 * kQtTileBytes + (kQThreads / 32) * 64 * 4 + 128 * 4 +
         (kQThreads / 32) * 4 + STAGES * 8 + STAGES * 8 + 16 + 1024;
}

}  // namespace puro
