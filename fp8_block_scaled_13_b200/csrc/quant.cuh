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
// One persistent kernel serves every layout.  Each CTA (256 threads, two per
// SM, so two tiles are processed side by side) walks a strided list of
// 128x128 tiles of the BF16 input; a TMA ring of kQStages 32 KB tile buffers
// keeps the next tiles in flight while the current one is processed, and a
// stage is handed back to the TMA as soon as every thread has copied its part
// into registers (the first tiles are also prefetched into L2 before the
// kernel waits on its predecessor).  Thread (i, j) = (tid/16, tid%16) holds
// rows 8i..8i+7 and columns 8j..8j+7.  From those registers:
//   ROW   : row amax by a 16-lane shuffle reduction; codes stored in place.
//   COL   : column amax by a shuffle + shared-memory reduction over the 8
//           warps; codes transposed through an XOR-swizzled 16 KB shared tile
//           (conflict-free 8-byte writes, 16-byte reads) and written out as
//           128-byte rows of the transposed matrix.
//   BLOCK : one amax over the whole tile (128x128 weight block); codes written
//           in place and, optionally, transposed.
// The amax is taken on the integer BF16 magnitude bits (|x| is itself a BF16,
// and the order of non-negative floats equals the order of their bits), and
// the scale exponent comes from the exponent/mantissa fields alone: with
// amax = 1.f * 2^E, e = E - 8 if 1.f <= 1.75 (mantissa bits <= 0x60), else
// E - 7.  Scaling by 2^-e is an exact packed FP32 multiply (no flush to zero:
// this file must not be built with fast-math), followed by one hardware
// round-to-nearest-even, saturating conversion to E4M3 per value.
#pragma once

#include "common.cuh"

namespace puro {

#ifndef PURO_QUANT_RPT
#define PURO_QUANT_RPT 8
#endif
// rows of the 128x128 tile per thread (each thread holds RPT rows x 8 columns;
// 16 threads cover a row, 128/RPT row groups cover the tile).  8 (256 threads,
// two CTAs per SM) was measured faster than 4 (512 threads, 64 registers) for
// the BOTH layout at every size tried (8192x3072: 20.9 vs 22.8 us; 16384x12288:
// 147 vs 162 us) and equal within a few % for the single layouts.
constexpr int kQRpt = PURO_QUANT_RPT;
static_assert(kQRpt == 4 || kQRpt == 8, "4 or 8 rows per thread");
constexpr int kQThreads = 16 * 128 / kQRpt;
constexpr int kQStages = 2;
constexpr uint32_t kQTileBytes = 128 * 128 * 2;

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
};

// Scale exponent from the BF16 bits of a group's amax (sign already cleared).
__device__ __forceinline__ int scale_exponent_from_bits(uint32_t a) {
  if (a == 0) return 0;
  const int ef = static_cast<int>(a >> 7);  // biased exponent field
  if (ef == 0) return -127;                 // subnormal amax: always clamps
  const int e = ef - 127 - 8 + ((a & 0x7Fu) > 0x60u ? 1 : 0);
  return e < -127 ? -127 : e;
}

// 2^-e as an FP32 (e in [-127, 120], so the result is a normal number), in
// both lanes of a float2.
__device__ __forceinline__ float2 pow2_neg_x2(int e) {
  const float f = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
  return make_float2(f, f);
}

// Four values (pairs a, b) times 2^-e (s2) -> four E4M3 codes in one word,
// a.x in the low byte.  The packed multiply is exact (a power of two,
// subnormals kept), then one RNE saturating conversion per value; the two
// 16-bit results are joined by a register move rather than shift-and-or
// (measured: 8 fewer ALU instructions per 32 values on sm_100a).
__device__ __forceinline__ uint32_t encode4(float2 a, float2 b, float2 s2) {
  const float2 x = __fmul2_rn(a, s2), y = __fmul2_rn(b, s2);
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(x.x), "f"(x.y), "f"(y.x), "f"(y.y));
  return r;
}

// The two BF16 of a packed word widened to FP32 (exact).
__device__ __forceinline__ float2 bf16x2_f32(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint32_t word(const uint4& v, int idx) {
  return idx == 0 ? v.x : idx == 1 ? v.y : idx == 2 ? v.z : v.w;
}

// Element l (0..7) of an 8-BF16 row chunk, widened to FP32.
__device__ __forceinline__ float elem_f32(const uint4& v, int l) {
  const uint32_t w = word(v, l >> 1);
  return __uint_as_float((l & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// Eight codes of one 8-element row chunk, all scaled by s2.
__device__ __forceinline__ uint2 encode_row8(const uint4& v, float2 s2) {
  uint2 o;
  o.x = encode4(bf16x2_f32(v.x), bf16x2_f32(v.y), s2);
  o.y = encode4(bf16x2_f32(v.z), bf16x2_f32(v.w), s2);
  return o;
}

// Four codes of column l of rows 0..3 of the thread's block, scaled by s2.
__device__ __forceinline__ uint32_t encode_col4(const uint4 (&v)[4], int l, float2 s2) {
  return encode4(make_float2(elem_f32(v[0], l), elem_f32(v[1], l)),
                 make_float2(elem_f32(v[2], l), elem_f32(v[3], l)), s2);
}

// Eight codes of column l of the thread's 8x8 block (rows 0..7), scaled by s2.
__device__ __forceinline__ uint2 encode_col8(const uint4 (&v)[8], int l, float2 s2) {
  uint2 o;
  o.x = encode4(make_float2(elem_f32(v[0], l), elem_f32(v[1], l)),
                make_float2(elem_f32(v[2], l), elem_f32(v[3], l)), s2);
  o.y = encode4(make_float2(elem_f32(v[4], l), elem_f32(v[5], l)),
                make_float2(elem_f32(v[6], l), elem_f32(v[7], l)), s2);
  return o;
}

// Column l of the thread's block as codes into its transposed-tile row `row`.
// 8 rows per thread: 8 codes at 8-byte chunk i ^ 2(j & 7), so that a 16-byte
// unit holds two consecutive chunks in order (one plain 16-byte load per 16
// rows on the way out) while the 32 stores of a warp still fill 16 distinct
// chunk positions twice (two wavefronts, the minimum for 256 bytes).
// 4 rows per thread: 4 codes at 4-byte slot i ^ 2j (conflict-free; the
// readout swaps the 8-byte halves of odd column groups).
__device__ __forceinline__ void put_col_codes(uint8_t* row, const uint4 (&v)[8], int l, float2 s2,
                                              int i, int j) {
  *reinterpret_cast<uint2*>(row + ((i ^ (2 * (j & 7))) << 3)) = encode_col8(v, l, s2);
}

__device__ __forceinline__ void put_col_codes(uint8_t* row, const uint4 (&v)[4], int l, float2 s2,
                                              int i, int j) {
  *reinterpret_cast<uint32_t*>(row + ((i ^ (2 * j)) << 2)) = encode_col4(v, l, s2);
}

// Larger of the two 16-bit halves.
__device__ __forceinline__ uint32_t hmax(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

__device__ __forceinline__ uint4 lds_v4(const uint8_t* p) {
  return *reinterpret_cast<const uint4*>(p);
}

// Row k's amax (BF16 bits) out of the row-pair words of row_amax, for a
// lane-dependent k: byte permutes pick the half-word (a plain or selected
// array index would be lowered to a local-memory round trip).
template <int NQ>
__device__ __forceinline__ uint32_t pick_row_amax(const uint32_t (&rm)[NQ], int k) {
  static_assert(NQ == 2 || NQ == 4, "2 or 4 row-pair words");
  const uint32_t b = 2u * static_cast<uint32_t>(k & 3);  // byte of the half within a word pair
  const uint32_t sel = b | ((b + 1u) << 4);
  uint32_t w = __byte_perm(rm[0], rm[1], sel);
  if constexpr (NQ == 4) w = (k & 4) ? __byte_perm(rm[2], rm[3], sel) : w;
  return w & 0xFFFFu;
}

// Byte offset, inside one 512-byte chunk of a blocked scale array, of the
// chunk's row r (0..127).
__device__ __forceinline__ uint32_t blocked_in_chunk(int r) {
  return static_cast<uint32_t>((r & 31) * 16 + ((r >> 5) & 3) * 4);
}

// RSHFL selects how the row scales reach the threads (ROW without BLOCK):
// one thread per row derives the exponent and the 16 threads of the row read
// it with shuffles (fewer ALU instructions: faster when each CTA has only a
// few tiles), or all 16 derive it themselves (no cross-lane latency on the
// encode path: faster on long tile streams).  Both give identical results.
//
// Addressing is kept out of the per-element work: every output pointer is
// formed once per tile from per-thread constants and advanced by its stride,
// and the ragged-edge tests are one 32-bit compare against a per-tile count.
template <bool ROW, bool COL, bool BLOCK, bool RSHFL>
__global__ void __launch_bounds__(kQThreads, 2)
    quant_kernel(const __grid_constant__ CUtensorMap tm_x, const QuantParams p) {
  constexpr uint32_t kMag = 0x7FFF7FFFu;
  constexpr int kWarps = kQThreads / 32;
  constexpr int RPT = kQRpt;
  constexpr int kColsPerPass = kQThreads / 8;  // transposed rows copied out per pass
  extern __shared__ uint8_t qsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(qsmem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* tiles = smem;                                    // kQStages x 32 KB
  uint8_t* qt_s = smem + kQStages * kQTileBytes;            // 16 KB transposed codes
  uint32_t* col_part = reinterpret_cast<uint32_t*>(qt_s + 128 * 128);  // [8 warps][16][4]
  float* col_scale = reinterpret_cast<float*>(col_part + kWarps * 64);  // [128] 2^-e per column
  uint32_t* blk_part = reinterpret_cast<uint32_t*>(col_scale + 128);    // [8]
  uint64_t* full = reinterpret_cast<uint64_t*>(blk_part + kWarps);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + kQStages);

  const int tid = threadIdx.x;
  const int i = tid >> 4, j = tid & 15, warp = tid >> 5;
  // tiles t = blockIdx.x + it * gridDim.x, walked as (row tile, col tile)
  const int32_t tc_step = (int32_t)(gridDim.x % p.tiles_c), tr_step = (int32_t)(gridDim.x / p.tiles_c);
  const int32_t my_tiles =
      (int32_t)blockIdx.x < p.tiles ? (p.tiles - (int32_t)blockIdx.x + (int32_t)gridDim.x - 1) / (int32_t)gridDim.x : 0;

  if (tid == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_x);
  }
  __syncthreads();
  if (tid == 0) {
    // Warm L2 with this CTA's first tiles while the kernel before this one is
    // still finishing.  A prefetch only moves data into L2, the point of
    // coherence, and the loads that fill shared memory still follow the
    // dependency wait below, so a producer's later writes are what they read.
    int32_t r = (int32_t)blockIdx.x / p.tiles_c, c = (int32_t)blockIdx.x % p.tiles_c;
    for (int32_t t = 0; t < kQStages && t < my_tiles; ++t) {
      tma_prefetch_l2_2d(&tm_x, c * 128, r * 128);
      c += tc_step;
      r += tr_step;
      if (c >= p.tiles_c) { c -= p.tiles_c; ++r; }
    }
  }
  // the input may come from the kernel just before this one on the stream
  pdl_wait();
  pdl_trigger();
  // producer-side tile cursor (thread 0 only)
  int32_t ptr_r = (int32_t)blockIdx.x / p.tiles_c, ptr_c = (int32_t)blockIdx.x % p.tiles_c;
  int32_t p_it = 0;
  auto issue_next = [&]() {
    const int s = p_it % kQStages;
    mbar_arrive_expect_tx(&full[s], kQTileBytes);
    tma_load_2d<1>(tiles + s * kQTileBytes, &tm_x, ptr_c * 128, ptr_r * 128, smem_u32(&full[s]));
    ++p_it;
    ptr_c += tc_step;
    ptr_r += tr_step;
    if (ptr_c >= p.tiles_c) { ptr_c -= p.tiles_c; ++ptr_r; }
  };
  if (tid == 0)
    while (p_it < my_tiles && p_it < kQStages) issue_next();

  // per-thread constants of the output addressing
  const uint32_t s_in_chunk = blocked_in_chunk(RPT * i + (j & (RPT - 1)));  // row scale byte (j < RPT)
  const uint32_t s_half_chunk = blocked_in_chunk(RPT * i + (j >> 1));      // the same, row j >> 1
  const uint32_t st_in_chunk = blocked_in_chunk(2 * (tid & 63));            // column scale bytes (tid < 64)
  const int c_base = tid >> 3, part = tid & 7;                               // transposed readout
  const int64_t qt_pass_stride = (int64_t)kColsPerPass * p.ld_qt;
  // 4 rows per thread: the readout's 16-byte unit has its 8-byte halves
  // swapped for odd column groups, the same parity in every pass
  // (kColsPerPass is a multiple of 16)
  const bool swap_halves = RPT == 4 && ((c_base >> 3) & 1);

  int32_t tr = (int32_t)blockIdx.x / p.tiles_c, tc = (int32_t)blockIdx.x % p.tiles_c;
  for (int32_t it = 0; it < my_tiles; ++it) {
    const int32_t r0 = tr * 128, c0 = tc * 128;
    const int s = it % kQStages;
    const bool ok = mbar_wait(&full[s], (uint32_t)((it / kQStages) & 1), abort_flag);
    // this thread's RPT rows x 8 columns; rows past the end were filled with 0
    uint4 v[RPT];
    const uint8_t* tile = tiles + s * kQTileBytes + (RPT * i) * 256 + 16 * j;
#pragma unroll
    for (int k = 0; k < RPT; ++k) v[k] = ok ? lds_v4(tile + k * 256) : make_uint4(0, 0, 0, 0);
    // every thread holds its part: stage s is free again (and if any wait gave
    // up, the whole block stops here together)
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && p_it < my_tiles) issue_next();

    // ---- magnitudes: per-row amax of this thread's 8 columns (two rows per
    // word) and per-column-pair amax of its 8 rows, from the same masked words
    uint32_t rowmax[RPT / 2];
#pragma unroll
    for (int q = 0; q < RPT / 2; ++q) rowmax[q] = 0u;
    uint32_t cm[4] = {0u, 0u, 0u, 0u};
    uint32_t even_row = 0u;  // (even, odd)-column maxima of the last even row
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const uint32_t a0 = v[k].x & kMag, a1 = v[k].y & kMag, a2 = v[k].z & kMag,
                     a3 = v[k].w & kMag;
      if (ROW || BLOCK) {
        // two rows per word: the low halves of rows k-1, k side by side, the
        // high halves side by side, and one packed max of the two
        const uint32_t t = __vmaxu2(__vmaxu2(a0, a1), __vmaxu2(a2, a3));
        if (k & 1)
          rowmax[k >> 1] = __vmaxu2(__byte_perm(even_row, t, 0x5410), __byte_perm(even_row, t, 0x7632));
        else
          even_row = t;
      }
      if (COL && !BLOCK) {
        cm[0] = __vmaxu2(cm[0], a0);
        cm[1] = __vmaxu2(cm[1], a1);
        cm[2] = __vmaxu2(cm[2], a2);
        cm[3] = __vmaxu2(cm[3], a3);
      }
    }
    // Row reductions over the 16 lanes of a row group.  On the shared-scale
    // path with 8 rows per thread this is a reduce-scatter (rs_row below);
    // elsewhere every lane needs every row's amax: a full butterfly.
    constexpr bool kRowScatter = ROW && !BLOCK && RSHFL && RPT == 8;
    if ((ROW || BLOCK) && !kRowScatter) {
#pragma unroll
      for (int q = 0; q < RPT / 2; ++q) {
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
          rowmax[q] = __vmaxu2(rowmax[q], __shfl_xor_sync(0xFFFFFFFFu, rowmax[q], off));
      }
    }

    int e_blk = 0;
    if (BLOCK) {
      // one exponent for the whole 128x128 block
      uint32_t m = rowmax[0];
#pragma unroll
      for (int q = 1; q < RPT / 2; ++q) m = __vmaxu2(m, rowmax[q]);
      m = __vmaxu2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
      if ((tid & 31) == 0) blk_part[warp] = hmax(m);
      __syncthreads();
      uint32_t bm = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) bm = max(bm, blk_part[w]);
      e_blk = scale_exponent_from_bits(bm);
      if (tid == 0) p.sw[tr * p.tiles_c + tc] = static_cast<uint8_t>(e_blk + 127);
    }

    // ---- in-place codes (ROW, BLOCK) and the row scale bytes; thread j < RPT
    // owns the scale byte of row RPT*i + j
    if (ROW || BLOCK) {
      uint8_t* qrow = p.q + (int64_t)(r0 + RPT * i) * p.ld_q + (c0 + 8 * j);
      const int32_t nrow = (int32_t)(p.rows - r0) - RPT * i;  // rows of the block that exist
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
        const int e_mine = scale_exponent_from_bits(b1 ? (w >> 16) : (w & 0xFFFFu));
        if ((j & 1) == 0)
          p.s[((int64_t)tr * p.s_g4 + (tc >> 2)) * 512 + (tc & 3) + s_half_chunk] = static_cast<uint8_t>(e_mine + 127);
        const float s_mine = pow2_neg_x2(e_mine).x;
        const int lane16 = tid & 16;
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
          const float sk = __shfl_sync(0xFFFFFFFFu, s_mine, lane16 + 2 * k);
          const uint2 o = encode_row8(v[k], make_float2(sk, sk));
          if (k < nrow) *reinterpret_cast<uint2*>(qrow) = o;
          qrow += p.ld_q;
        }
      } else if (RSHFL && !BLOCK) {
        // thread j derives row RPT*i + j's exponent; the 16 threads of the
        // rows read 2^-e of row k from thread k
        const int e_mine = scale_exponent_from_bits(pick_row_amax(rowmax, j & (RPT - 1)));
        if (j < RPT)
          p.s[((int64_t)tr * p.s_g4 + (tc >> 2)) * 512 + (tc & 3) + s_in_chunk] = static_cast<uint8_t>(e_mine + 127);
        const float s_mine = pow2_neg_x2(e_mine).x;
        const int lane16 = tid & 16;
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
          const float sk = __shfl_sync(0xFFFFFFFFu, s_mine, lane16 + k);
          const uint2 o = encode_row8(v[k], make_float2(sk, sk));
          if (k < nrow) *reinterpret_cast<uint2*>(qrow) = o;
          qrow += p.ld_q;
        }
      } else {
        // every thread derives the exponents of its rows itself (the scale
        // byte is stored inside the loop, its address formed there: deriving
        // the byte ahead of the encodes, or keeping its pointer live across
        // the loop, was measured 10 % slower on long tile streams)
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
          const uint32_t m = (k & 1) ? (rowmax[k >> 1] >> 16) : (rowmax[k >> 1] & 0xFFFFu);
          const int e = BLOCK ? e_blk : scale_exponent_from_bits(m);
          const uint2 o = encode_row8(v[k], pow2_neg_x2(e));
          if (!BLOCK && j == k)
            p.s[((int64_t)tr * p.s_g4 + (tc >> 2)) * 512 + (tc & 3) + s_in_chunk] = static_cast<uint8_t>(e + 127);
          if (k < nrow) *reinterpret_cast<uint2*>(qrow) = o;
          qrow += p.ld_q;
        }
      }
    }

    // ---- transposed codes (COL, BLOCK with a transposed copy)
    if (COL) {
      if (!BLOCK) {
#pragma unroll
        for (int pp = 0; pp < 4; ++pp)
          cm[pp] = __vmaxu2(cm[pp], __shfl_xor_sync(0xFFFFFFFFu, cm[pp], 16));
        if ((tid & 16) == 0)
          *reinterpret_cast<uint4*>(&col_part[(warp * 16 + j) * 4]) = make_uint4(cm[0], cm[1], cm[2], cm[3]);
        __syncthreads();
        if (tid < 64) {
          // columns 2*tid and 2*tid+1: amax over the 8 warps, then the exponent,
          // its scale byte and 2^-e for every thread's encode
          uint32_t m = 0;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) m = __vmaxu2(m, col_part[(w * 16 + (tid >> 2)) * 4 + (tid & 3)]);
          const int e0 = scale_exponent_from_bits(m & 0xFFFFu);
          const int e1 = scale_exponent_from_bits(m >> 16);
          uint8_t* scol = p.st + ((int64_t)tc * p.st_g4 + (tr >> 2)) * 512 + (tr & 3) + st_in_chunk;
          scol[0] = static_cast<uint8_t>(e0 + 127);
          scol[16] = static_cast<uint8_t>(e1 + 127);
          *reinterpret_cast<float2*>(&col_scale[2 * tid]) = make_float2(pow2_neg_x2(e0).x, pow2_neg_x2(e1).x);
        }
        __syncthreads();
      }
      float cs[8];
      if (!BLOCK) {
        const float4 a = *reinterpret_cast<const float4*>(&col_scale[8 * j]);
        const float4 b = *reinterpret_cast<const float4*>(&col_scale[8 * j + 4]);
        cs[0] = a.x; cs[1] = a.y; cs[2] = a.z; cs[3] = a.w;
        cs[4] = b.x; cs[5] = b.y; cs[6] = b.z; cs[7] = b.w;
      }
#pragma unroll
      for (int l = 0; l < 8; ++l) {
        const float2 s2 = BLOCK ? pow2_neg_x2(e_blk) : make_float2(cs[l], cs[l]);
        // row (8j+l) of the transposed tile: this thread's RPT codes go to an
        // XOR-swizzled chunk (put_col_codes) that the readout below undoes
        put_col_codes(qt_s + (8 * j + l) * 128, v, l, s2, i, j);
      }
      __syncthreads();
      // transposed row c = pass * kColsPerPass + c_base, rows 16*part.. of the
      // tile: with jj = c / 8 its 16 codes sit in 16-byte unit part ^ (jj & 7)
      // (8 rows per thread) or part ^ (jj >> 1) (4 rows per thread)
      if (r0 + 16 * part < p.rows) {
        uint8_t* dst = p.qt + (int64_t)(c0 + c_base) * p.ld_qt + (r0 + 16 * part);
#pragma unroll
        for (int pass = 0; pass < 128 / kColsPerPass; ++pass) {
          const int c = pass * kColsPerPass + c_base;
          const int unit = part ^ (RPT == 8 ? ((c >> 3) & 7) : ((c >> 4) & 7));
          uint4 w = lds_v4(qt_s + c * 128 + (unit << 4));
          if (swap_halves) w = make_uint4(w.z, w.w, w.x, w.y);
          *reinterpret_cast<uint4*>(dst) = w;
          dst += qt_pass_stride;
        }
      }
    }

    if (BLOCK && tid < 128) {
      const uint8_t b = static_cast<uint8_t>(e_blk + 127);
      const uint32_t in_chunk = blocked_in_chunk(tid);
      if (p.sw_fwd) p.sw_fwd[((int64_t)tr * p.fwd_g4 + (tc >> 2)) * 512 + (tc & 3) + in_chunk] = b;
      if (p.sw_bwd) p.sw_bwd[((int64_t)tc * p.bwd_g4 + (tr >> 2)) * 512 + (tr & 3) + in_chunk] = b;
    }
    // No barrier here: the shared tiles (qt_s, col_part, blk_part) are next
    // written after the __syncthreads_or at the top of the next iteration,
    // which no thread passes before every thread has finished this tile.
    tc += tc_step;
    tr += tr_step;
    if (tc >= p.tiles_c) { tc -= p.tiles_c; ++tr; }
  }
  // Copies are only issued for tiles this CTA processes, and each one was
  // waited for above, unless a wait gave up; then let the outstanding ones
  // land (bounded) before the block exits.
  if (tid == 0 && *abort_flag) {
    for (int s = 0; s < kQStages; ++s) {
      volatile int no_abort = 0;
      mbar_wait(&full[s], 0, &no_abort, 100000000ull);
      mbar_wait(&full[s], 1, &no_abort, 100000000ull);
    }
  }
}

// Shared memory the quantizer needs (plus alignment slack).
constexpr uint32_t quant_smem_bytes() {
  return kQStages * kQTileBytes + 128 * 128 + (kQThreads / 32) * 64 * 4 + 128 * 4 +
         (kQThreads / 32) * 4 + kQStages * 8 + 16 + 1024;
}

}  // namespace puro
