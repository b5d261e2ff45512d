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
// One kernel serves every layout.  A CTA of 256 threads owns a 128x128 tile of
// the BF16 input; thread (i, j) = (tid/16, tid%16) holds rows 8i..8i+7 and
// columns 8j..8j+7 in registers (eight 16-byte loads, one per row; a warp
// instruction reads two full 256-byte tile rows).  From those registers:
//   ROW   : row amax by a 16-lane shuffle reduction; codes stored in place.
//   COL   : column amax by a shuffle + shared-memory reduction across the 8
//           warps; codes transposed through an XOR-swizzled 16 KB shared tile
//           (conflict-free 8-byte writes, 16-byte reads) and written out as
//           full 128-byte rows of the transposed matrix.
//   BLOCK : one amax over the whole tile (128x128 weight block); codes written
//           in place and, optionally, transposed.
// The amax is taken on the integer BF16 magnitude bits (|x| is itself a BF16,
// and the order of non-negative floats equals the order of their bits), and
// the scale exponent comes from the exponent/mantissa fields alone: with
// amax = 1.f * 2^E, e = E - 8 if 1.f <= 1.75 (mantissa bits <= 0x60), else
// E - 7.  Scaling by 2^-e is an exact FP32 multiply (no flush to zero: this
// file must not be built with fast-math), followed by one hardware
// round-to-nearest-even, saturating conversion to E4M3.
#pragma once

#include "common.cuh"

namespace puro {

struct QuantParams {
  const uint16_t* x;  // BF16 bits [rows, cols], row stride ld_x
  int64_t rows, cols, ld_x;
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
  int64_t tiles_c, tiles;
};

// Byte offset of (row r, group g) in a blocked scale array whose rows hold
// g4 = ceil(groups / 4) chunks of 512 bytes per 128-row block.
__device__ __forceinline__ int64_t blocked_offset(int64_t r, int64_t g, int64_t g4) {
  return ((r >> 7) * g4 + (g >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (g & 3);
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Scale exponent from the BF16 bits of a group's amax (sign already cleared).
__device__ __forceinline__ int scale_exponent_from_bits(uint32_t a) {
  if (a == 0) return 0;
  const int ef = static_cast<int>(a >> 7);  // biased exponent field
  if (ef == 0) return -127;                 // subnormal amax: always clamps
  const int e = ef - 127 - 8 + ((a & 0x7Fu) > 0x60u ? 1 : 0);
  return e < -127 ? -127 : e;
}

// 2^-e as an FP32 (e in [-127, 120], so the result is a normal number).
__device__ __forceinline__ float pow2_neg(int e) {
  return __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// Two FP32 values -> two E4M3 codes (RNE, satfinite); `lo` in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t word(const uint4& v, int idx) {
  return idx == 0 ? v.x : idx == 1 ? v.y : idx == 2 ? v.z : v.w;
}

// Element l (0..7) of an 8-BF16 row chunk, widened to FP32.
__device__ __forceinline__ float elem(const uint4& v, int l) {
  const uint32_t w = word(v, l >> 1);
  return (l & 1) ? bf16_hi(w) : bf16_lo(w);
}

// Eight codes of one 8-element row chunk, all scaled by `inv`.
__device__ __forceinline__ uint2 encode_row8(const uint4& v, float inv) {
  uint2 o;
  o.x = e4m3x2(bf16_lo(v.x) * inv, bf16_hi(v.x) * inv) |
        (e4m3x2(bf16_lo(v.y) * inv, bf16_hi(v.y) * inv) << 16);
  o.y = e4m3x2(bf16_lo(v.z) * inv, bf16_hi(v.z) * inv) |
        (e4m3x2(bf16_lo(v.w) * inv, bf16_hi(v.w) * inv) << 16);
  return o;
}

template <bool ROW, bool COL, bool BLOCK>
__global__ void __launch_bounds__(256) quant_tile_kernel(const QuantParams p) {
  constexpr uint32_t kMag = 0x7FFF7FFFu;
  __shared__ uint32_t col_part[8][16][4];
  __shared__ uint32_t col_final[64];
  __shared__ uint32_t blk_part[8];
  __shared__ __align__(16) uint8_t qt_s[COL ? 128 * 128 : 16];

  const int tid = threadIdx.x;
  const int i = tid >> 4, j = tid & 15, warp = tid >> 5;

  for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x) {
    const int64_t r0 = (t / p.tiles_c) * 128;
    const int64_t c0 = (t % p.tiles_c) * 128;

    uint4 v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t r = r0 + 8 * i + k;
      v[k] = (r < p.rows) ? ld_stream_v4(p.x + r * p.ld_x + c0 + 8 * j) : make_uint4(0, 0, 0, 0);
    }

    // ---- row amax (reduced over the 16 lanes sharing i), packed two rows per word
    uint32_t rowmax[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t m2[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4& a = v[2 * q + h];
        const uint32_t m = __vmaxu2(__vmaxu2(a.x & kMag, a.y & kMag), __vmaxu2(a.z & kMag, a.w & kMag));
        m2[h] = max(m & 0xFFFFu, m >> 16);
      }
      rowmax[q] = m2[0] | (m2[1] << 16);
    }
    if (ROW || BLOCK) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
          rowmax[q] = __vmaxu2(rowmax[q], __shfl_xor_sync(0xFFFFFFFFu, rowmax[q], off));
      }
    }

    int e_row[8];
    int e_col[8];
    if (BLOCK) {
      // one exponent for the whole 128x128 block
      uint32_t m = __vmaxu2(__vmaxu2(rowmax[0], rowmax[1]), __vmaxu2(rowmax[2], rowmax[3]));
      m = __vmaxu2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
      if ((tid & 31) == 0) blk_part[warp] = max(m & 0xFFFFu, m >> 16);
      __syncthreads();
      uint32_t bm = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) bm = max(bm, blk_part[w]);
      const int e = scale_exponent_from_bits(bm);
#pragma unroll
      for (int k = 0; k < 8; ++k) e_row[k] = e_col[k] = e;
      if (tid == 0) p.sw[(r0 / 128) * p.tiles_c + c0 / 128] = static_cast<uint8_t>(e + 127);
    } else {
      if (ROW) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          e_row[2 * q] = scale_exponent_from_bits(rowmax[q] & 0xFFFFu);
          e_row[2 * q + 1] = scale_exponent_from_bits(rowmax[q] >> 16);
        }
      }
      if (COL) {
        uint32_t cm[4];
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          uint32_t m = 0;
#pragma unroll
          for (int k = 0; k < 8; ++k) m = __vmaxu2(m, word(v[k], pp) & kMag);
          m = __vmaxu2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
          cm[pp] = m;
        }
        if ((tid & 16) == 0) {
#pragma unroll
          for (int pp = 0; pp < 4; ++pp) col_part[warp][j][pp] = cm[pp];
        }
        __syncthreads();
        if (tid < 64) {
          uint32_t m = 0;
#pragma unroll
          for (int w = 0; w < 8; ++w) m = __vmaxu2(m, col_part[w][tid >> 2][tid & 3]);
          col_final[tid] = m;
        }
        __syncthreads();
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const uint32_t m = col_final[j * 4 + pp];
          e_col[2 * pp] = scale_exponent_from_bits(m & 0xFFFFu);
          e_col[2 * pp + 1] = scale_exponent_from_bits(m >> 16);
        }
      }
    }

    // ---- in-place codes (ROW, BLOCK)
    if (ROW || BLOCK) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int64_t r = r0 + 8 * i + k;
        const uint2 o = encode_row8(v[k], pow2_neg(e_row[k]));
        if (r < p.rows) *reinterpret_cast<uint2*>(p.q + r * p.ld_q + c0 + 8 * j) = o;
      }
    }

    // ---- transposed codes (COL, BLOCK with a transposed copy)
    if (COL) {
      if (BLOCK && p.qt == nullptr) {
        // nothing to transpose
      } else {
#pragma unroll
        for (int l = 0; l < 8; ++l) {
          const float inv = pow2_neg(e_col[l]);
          uint2 o;
          o.x = e4m3x2(elem(v[0], l) * inv, elem(v[1], l) * inv) |
                (e4m3x2(elem(v[2], l) * inv, elem(v[3], l) * inv) << 16);
          o.y = e4m3x2(elem(v[4], l) * inv, elem(v[5], l) * inv) |
                (e4m3x2(elem(v[6], l) * inv, elem(v[7], l) * inv) << 16);
          // row (8j+l) of the transposed tile, 8-byte chunk i, XOR-swizzled by j
          *reinterpret_cast<uint2*>(qt_s + (8 * j + l) * 128 + ((i ^ j) << 3)) = o;
        }
        __syncthreads();
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int idx = pass * 256 + tid;
          const int c = idx >> 3, part = idx & 7;
          const int jj = (c >> 3) & 15;
          const uint4 w = *reinterpret_cast<const uint4*>(qt_s + c * 128 + ((part ^ (jj >> 1)) << 4));
          const uint4 o = (jj & 1) ? make_uint4(w.z, w.w, w.x, w.y) : w;
          const int64_t rr = r0 + 16 * part;
          if (rr < p.rows) *reinterpret_cast<uint4*>(p.qt + (c0 + c) * p.ld_qt + rr) = o;
        }
      }
    }

    // ---- scales (blocked layout); rows past the end hold zeros, so their
    // scale byte is 127
    if (ROW && !BLOCK && j == 0) {
      const int64_t g = c0 / 128;
#pragma unroll
      for (int k = 0; k < 8; ++k)
        p.s[blocked_offset(r0 + 8 * i + k, g, p.s_g4)] = static_cast<uint8_t>(e_row[k] + 127);
    }
    if (COL && !BLOCK && i == 0) {
      const int64_t g = r0 / 128;
#pragma unroll
      for (int l = 0; l < 8; ++l)
        p.st[blocked_offset(c0 + 8 * j + l, g, p.st_g4)] = static_cast<uint8_t>(e_col[l] + 127);
    }
    if (BLOCK && tid < 128) {
      const uint8_t b = static_cast<uint8_t>(e_row[0] + 127);
      if (p.sw_fwd) p.sw_fwd[blocked_offset(r0 + tid, c0 / 128, p.fwd_g4)] = b;
      if (p.sw_bwd) p.sw_bwd[blocked_offset(c0 + tid, r0 / 128, p.bwd_g4)] = b;
    }
    if (COL || BLOCK) __syncthreads();  // shared tiles are reused by the next tile
  }
}

}  // namespace puro
