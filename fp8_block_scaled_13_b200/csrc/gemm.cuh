// Block-scaled FP8 GEMM on the sm_100a tensor cores (tcgen05, TMEM, TMA).
//
//   D[i, j] = sum_kb 2^(ea[i,kb] + eb[j,kb]) * sum_{r in kb} A[i, r] * B[j, r]
//
// A [rows_a, K] and B [rows_b, K] are E4M3 and K-contiguous; kb runs over the
// 128-wide groups of the reduction dimension (Puro-2B report: 1x128 groups
// along the reduction dimension for activations and gradients, 128x128 blocks
// for weights -- paper.rainbus.top "方法步骤详情" step (3), ta-paperlens §3.2).
// fprop, dgrad and wgrad are all this one contraction with different operands
// (see the host entry points).  FP32 accumulation in TMEM, BF16 output (RNE).
//
// The pages' "Blackwell MXFP8 path" maps onto tcgen05.mma kind::mxf8f6f4 with
// block scaling: the MMA multiplies each 32-element K slice by one UE8M0 scale
// per row of A and per row of B.  A 128-group scale is the same for its four
// 32-element slices, so every slice of a 128-deep K block uses the same scale
// byte (it is replicated into all four bytes of its TMEM word).
//
// CTA organisation (one CTA per SM, persistent over output tiles of
// 128 x BN):
//   warp 0   : TMA producer -- per 128-deep K block loads the A tile
//              (128 x 128 B), the B tile (BN x 128 B), the 128 A scales and,
//              for per-row B scales, the BN B scales into a STAGES-deep ring.
//              For 128x128-block B scales it stages the tile's scale panel.
//   warp 1   : MMA issuer and TMEM owner -- rearranges the stage's scales into
//              the 32-lane x 4-column TMEM scale layout (tcgen05.cp source),
//              copies them to TMEM, issues four K=32 block-scaled MMAs and
//              releases the stage with tcgen05.commit.
//   warps 2-5: epilogue -- tcgen05.ld of the FP32 accumulator (warp w reads
//              TMEM lanes 32*(w%4)..+31, i.e. tile rows), BF16 conversion,
//              16-byte stores; masks rows >= rows_a and columns >= rows_b.
// With NACC = 2 the epilogue of one tile overlaps the MMAs of the next.
//
// Every wait is bounded (common.cuh): on expiry the kernel records
// PURO_ERR_DEVICE_TIMEOUT, stops issuing work, lets its own copies and MMAs
// drain (bounded again), frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace puro {

struct GemmParams {
  int32_t rows_a;   // output rows (M of the tile grid)
  int32_t rows_b;   // output cols
  int32_t kblocks;  // ceil(K / 128)
  int32_t tiles_m, tiles_n;
  // 128x128-block scales of B: scale(j, kb) = bsf[(j/128) * bsf_row + kb * bsf_col]
  const uint8_t* bsf;
  int32_t bsf_row, bsf_col;
  __nv_bfloat16* d;  // BF16 [rows_a, rows_b], row stride ldd
  int64_t ldd;
};

template <int BN>
struct GemmCfg {
  static constexpr int kStages = (BN == 256) ? 4 : 5;
  static constexpr int kNacc = (BN <= 224) ? 2 : 1;
  static constexpr int kAccStride = 256;          // TMEM columns between accumulators
  static constexpr int kSfaCol = 480;             // TMEM columns of the A scales (4)
  static constexpr int kSfbCol = 484;             // TMEM columns of the B scales (8)
  static constexpr int kNB = (BN + 127) / 128;    // 128-row blocks of B per tile
  static constexpr int kPanel = kNB * 256;        // block-scale panel bytes (K <= 32768)
  static constexpr int kPanels = kStages + 1;
  static constexpr uint32_t kABytes = 128 * 128;
  static constexpr uint32_t kBBytes = BN * 128;
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
  static constexpr uint32_t kOffSfaRaw = kOffB + kStages * kBBytes;
  static constexpr uint32_t kOffSfbRaw = kOffSfaRaw + kStages * 128;
  static constexpr uint32_t kOffSfaIl = kOffSfbRaw + kStages * (kNB * 128);
  static constexpr uint32_t kOffSfbIl = kOffSfaIl + kStages * 512;
  static constexpr uint32_t kOffPanel = kOffSfbIl + kStages * kNB * 512;
  static constexpr uint32_t kOffBar = (kOffPanel + kPanels * kPanel + 15) & ~15u;
  static constexpr uint32_t kNumBars = 2 * kStages + 2 * kNacc + 1;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  // instruction descriptor: E4M3 x E4M3, UE8M0 scales, K-major A and B,
  // N = BN, M = 128, scale-factor byte 0 for A and B, dense, K = 32.
  static constexpr uint32_t kIdesc =
      (0u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (0u << 16) |
      ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(128 >> 4) << 24);
};

template <int BN, bool B_PER_ROW>
__global__ void __launch_bounds__(192, 1)
    gemm_block_scaled_kernel(const __grid_constant__ CUtensorMap tm_a,
                             const __grid_constant__ CUtensorMap tm_b,
                             const __grid_constant__ CUtensorMap tm_sfa,
                             const __grid_constant__ CUtensorMap tm_sfb, const GemmParams p) {
  using C = GemmCfg<BN>;
  constexpr int S = C::kStages;
  constexpr int NA = C::kNacc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* accf = bars + 2 * S;
  uint64_t* acce = bars + 2 * S + NA;
  uint64_t* drain = bars + 2 * S + 2 * NA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    if (B_PER_ROW) prefetch_tmap(&tm_sfb);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_phase = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      uint8_t* panel = smem + C::kOffPanel + (it % C::kPanels) * C::kPanel;
      for (int kb = 0; kb < p.kblocks; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
        if (!B_PER_ROW && kb == 0) {
          // scale panel of this tile's B rows: panel[h * kblocks + kb]
          const int n = C::kNB * p.kblocks;
          for (int idx = lane; idx < n; idx += 32) {
            const int h = idx / p.kblocks, k = idx - h * p.kblocks;
            const int jb = tn * (BN / 128) + h;
            uint8_t v = 127;
            if (jb * 128 < p.rows_b) v = __ldg(p.bsf + (int64_t)jb * p.bsf_row + (int64_t)k * p.bsf_col);
            panel[idx] = v;
          }
          __syncwarp();
        }
        if (lane == 0) {
          const uint32_t bytes = C::kABytes + C::kBBytes + 128 + (B_PER_ROW ? BN : 0);
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d(smem + C::kOffA + stage * C::kABytes, &tm_a, kb * 128, tm * 128, &full[stage]);
          tma_load_2d(smem + C::kOffB + stage * C::kBBytes, &tm_b, kb * 128, tn * BN, &full[stage]);
          tma_load_2d(smem + C::kOffSfaRaw + stage * 128, &tm_sfa, tm * 128, kb, &full[stage]);
          if (B_PER_ROW)
            tma_load_2d(smem + C::kOffSfbRaw + stage * (C::kNB * 128), &tm_sfb, tn * BN, kb,
                        &full[stage]);
        }
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
    // let every load this warp issued land before the block can exit
    if (lane == 0) {
      for (int s = 0; s < S; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full[s], (issued_phase >> s) & 1u, &no_abort, 100000000ull);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    const uint32_t t_sfa = tmem + C::kSfaCol;
    const uint32_t t_sfb = tmem + C::kSfbCol;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
      const int acc = it % NA;
      const uint32_t acc_phase = (it / NA) & 1;
      const uint8_t* panel = smem + C::kOffPanel + (it % C::kPanels) * C::kPanel;
      if (!mbar_wait(&acce[acc], acc_phase ^ 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_acc = tmem + acc * C::kAccStride;
      for (int kb = 0; kb < p.kblocks; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        // scales -> tcgen05.cp source layout: 16-byte row `lane` holds the
        // words of tile rows lane, lane+32, lane+64, lane+96 (byte replicated)
        {
          const uint8_t* raw = smem + C::kOffSfaRaw + stage * 128;
          uint4 w;
          w.x = raw[lane] * 0x01010101u;
          w.y = raw[lane + 32] * 0x01010101u;
          w.z = raw[lane + 64] * 0x01010101u;
          w.w = raw[lane + 96] * 0x01010101u;
          *reinterpret_cast<uint4*>(smem + C::kOffSfaIl + stage * 512 + lane * 16) = w;
        }
#pragma unroll
        for (int h = 0; h < C::kNB; ++h) {
          uint4 w;
          if (B_PER_ROW) {
            const uint8_t* raw = smem + C::kOffSfbRaw + stage * (C::kNB * 128) + h * 128;
            const int base = h * 128 + lane;
            w.x = (base < BN ? raw[lane] : 0u) * 0x01010101u;
            w.y = (base + 32 < BN ? raw[lane + 32] : 0u) * 0x01010101u;
            w.z = (base + 64 < BN ? raw[lane + 64] : 0u) * 0x01010101u;
            w.w = (base + 96 < BN ? raw[lane + 96] : 0u) * 0x01010101u;
          } else {
            const uint32_t v = panel[h * p.kblocks + kb] * 0x01010101u;
            w = make_uint4(v, v, v, v);
          }
          *reinterpret_cast<uint4*>(smem + C::kOffSfbIl + (stage * C::kNB + h) * 512 + lane * 16) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc_cp_32x128b_warpx4(t_sfa, desc_dense_rows16(smem_u32(smem + C::kOffSfaIl + stage * 512)));
#pragma unroll
          for (int h = 0; h < C::kNB; ++h)
            tc_cp_32x128b_warpx4(t_sfb + 4 * h, desc_dense_rows16(smem_u32(
                                                     smem + C::kOffSfbIl + (stage * C::kNB + h) * 512)));
          const uint64_t adesc = desc_sw128_kmajor(smem_u32(smem + C::kOffA + stage * C::kABytes));
          const uint64_t bdesc = desc_sw128_kmajor(smem_u32(smem + C::kOffB + stage * C::kBBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_mxf8(t_acc, adesc + 2 * k, bdesc + 2 * k, C::kIdesc, t_sfa, t_sfb,
                        (kb | k) != 0 ? 1u : 0u);
          tc_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&accf[acc]);
      __syncwarp();
    }
    // wait until every MMA and copy this warp issued has completed
    if (lane == 0) {
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int sp = warp & 3;  // TMEM sub-partition this warp may access
    const int row_in_tile = sp * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int acc = it % NA;
      const uint32_t acc_phase = (it / NA) & 1;
      if (!mbar_wait(&accf[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const int grow = tm * 128 + row_in_tile;
      const uint32_t t_row = tmem + ((uint32_t)(sp * 32) << 16) + acc * C::kAccStride;
      __nv_bfloat16* drow = p.d + (int64_t)grow * p.ldd + tn * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(t_row + c * 32, r);
        tmem_ld_wait();
        if (grow < p.rows_a && tn * BN + c * 32 < p.rows_b) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * e]),
                                                     __uint_as_float(r[2 * e + 1]));
            pk[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          uint4* dst = reinterpret_cast<uint4*>(drow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace puro
