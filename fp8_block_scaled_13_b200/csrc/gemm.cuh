// Block-scaled FP8 GEMM on the sm_100a tensor cores (tcgen05, TMEM, TMA).
//
//   D[i, j] = sum_kb 2^(ea[i,kb] + eb[j,kb]) * sum_{r in kb} A[i, r] * B[j, r]
//
// A [rows_a, K] and B [rows_b, K] are E4M3 and K-contiguous; kb runs over the
// 128-wide groups of the reduction dimension (Puro-2B report: 1x128 groups
// along the reduction dimension for activations and gradients, 128x128 blocks
// for weights -- paper.rainbus.top "方法步骤详情" step (3), ta-paperlens §3.2).
// fprop, dgrad and wgrad are all this one contraction with different operands
// (see the host entry points).  FP32 accumulation in TMEM; BF16 (RNE) or FP32
// output.  A launch computes one GEMM, or two independent ones (a layer's
// data and weight gradients), over one list of output-tile work units that
// the clusters take round robin or from a host-made schedule (GemmParams).
//
// The pages' "Blackwell MXFP8 path" maps onto tcgen05.mma kind::mxf8f6f4 with
// block scaling: the MMA multiplies each 32-element K slice by one UE8M0 scale
// per row of A and per row of B, read from TMEM.  A 128-group scale holds for
// all four 32-element slices of its K block.  The scale arrays come in the
// blocked layout (include/puro_fp8.h): one 512-byte chunk holds the scales of
// 128 rows x 4 K blocks exactly as tcgen05.cp expects them in shared memory
// (16-byte row i = the words of rows i, i+32, i+64, i+96; byte g of a word =
// K block g), so a chunk goes from global memory to shared memory with one
// TMA copy and to TMEM with one tcgen05.cp, once per four K blocks; each MMA
// then selects its byte with the scale-factor id of the instruction
// descriptor.
//
// Tiles are (128*CG) x BN.  With CG = 2 a cluster of two CTAs on two SMs
// computes one tile with cta_group::2 MMAs: each CTA holds 128 rows of A and
// BN/2 rows of B in its shared memory (so each SM loads half of B), the
// leader CTA issues the MMAs for both, and each CTA's TMEM holds its 128 rows
// of the accumulator.  Scales: each CTA loads the A scales of its own rows
// and the B scales of all BN rows.  There is no TMA multicast; every CTA
// loads its own tiles.
//
// Warp roles (per CTA, persistent over the tiles of its cluster):
//   warp 0    : TMA producer -- A, B and (every 4th K block) scale chunks into
//               a STAGES-deep ring; both CTAs' copies complete on the leader's
//               full barrier.
//   warp 1    : TMEM owner; in the leader, MMA issuer -- tcgen05.cp of the
//               scale chunks, four K=32 MMAs per K block, tcgen05.commit to
//               release the stage in both CTAs and to publish the tile.
//   warps 2-9 : epilogue -- warp w reads TMEM lanes 32*(w%4)..+31 (tile rows)
//               and one half of the columns, releases the accumulator as soon
//               as its loads completed, then writes the rows through shared
//               memory with TMA tensor stores, 64-byte row segments at a time
//               (32 BF16 or 16 FP32 columns; one thread per row storing
//               straight to global memory touched 32 lines per instruction and
//               was the throughput limit of the kernel).  Output kinds: BF16
//               (RNE), FP32, or FP32 added into the existing output by TMA
//               reduce-add (accumulation into an FP32 gradient buffer).
//
// TMEM (512 columns) holds two accumulators, so the MMAs of the next tile
// overlap the epilogue of the previous one.  With BN = 256 the two 256-column
// accumulators fill TMEM, and the scale factors of a tile (two 16-column
// slots) live in the last 32 columns of the OTHER accumulator: the epilogue
// drains those 32 columns first and hands them over (barrier `sft`), so the
// next tile can start after a 32-column drain instead of a 256-column one.
// The next-but-one tile, which accumulates into those columns again, starts
// only after this tile's MMAs completed (its own `sft` wait follows this
// tile's accumulator commit), so scales are never overwritten while in use.
//
// Every wait is bounded (common.cuh): on expiry the kernel records
// PURO_ERR_DEVICE_TIMEOUT, stops issuing work, lets its own copies and MMAs
// drain (bounded again), frees TMEM and returns.
#pragma once

#include "common.cuh"

namespace puro {

// One GEMM of a launch: D [rows_a, rows_b] (through its tm_d tensor map).
// Its work units are its output tiles, except that tiles from split_from on
// are each split into two half-width tiles (two units: left and right 128
// columns), so that a last, partly-filled wave of tiles takes half as long.
struct GemmProblem {
  int32_t rows_a;      // output rows
  int32_t rows_b;      // output cols
  int32_t kblocks;     // ceil(K / BK)
  int32_t tiles_m, tiles_n;
  int32_t n_fastest;   // tile t -> (t / tiles_n, t % tiles_n) instead of (t % tiles_m, t / tiles_m)
  int32_t split_from;  // first split tile (== tiles_m * tiles_n: none)
  int32_t units;       // split_from + 2 * (tiles - split_from)
};

// Row and column tile of tile index t.  Consecutive tiles run at the same
// time on consecutive clusters, so the operand whose tiles are shared by
// consecutive indices is the one L2 keeps: with n_fastest they share A's rows
// (the host sets it when A is the larger operand, e.g. the activations of a
// forward or data-gradient GEMM with many tokens); otherwise they share B's.
__device__ __forceinline__ void tile_coords(const GemmProblem& P, int t, int& tm, int& tn) {
  if (P.n_fastest) {
    tm = t / P.tiles_n;
    tn = t - tm * P.tiles_n;
  } else {
    tn = t / P.tiles_m;
    tm = t - tn * P.tiles_m;
  }
}

// Tile and half (-1: whole tile, 0/1: left/right half) of a problem's unit.
__device__ __forceinline__ void decode_unit(const GemmProblem& P, int lu, int& tile, int& h) {
  if (lu < P.split_from) {
    tile = lu;
    h = -1;
  } else {
    const int d = lu - P.split_from;
    tile = P.split_from + (d >> 1);
    h = d & 1;
  }
}

constexpr int kMaxSchedClusters = 128;
constexpr int kMaxSchedUnits = 2048;

// A launch computes one or two independent GEMMs (the data and weight
// gradients of one layer share a launch).  Units [0, tiles0) are problem 0's,
// the rest problem 1's.  Clusters take
// units either round robin (unit u -> cluster u % clusters) or from a host-made
// schedule: cluster c runs sched_unit[sched_off[c] .. sched_off[c+1]) in order.
struct GemmParams {
  GemmProblem prob[2];
  int32_t nprob;
  int32_t tiles0;
  int32_t units;
  int32_t sched;
  uint16_t sched_off[kMaxSchedClusters + 1];
  uint16_t sched_unit[kMaxSchedUnits];
};

__device__ __forceinline__ int unit_count(const GemmParams& p, int cluster, int nclusters) {
  if (p.sched) return (int)p.sched_off[cluster + 1] - (int)p.sched_off[cluster];
  return cluster < p.units ? (p.units - cluster + nclusters - 1) / nclusters : 0;
}

__device__ __forceinline__ int unit_at(const GemmParams& p, int cluster, int nclusters, int i) {
  return p.sched ? (int)p.sched_unit[p.sched_off[cluster] + i] : cluster + i * nclusters;
}

#ifndef PURO_GEMM_BK
#define PURO_GEMM_BK 128
#endif
#ifndef PURO_GEMM_EPI_BUFS
#define PURO_GEMM_EPI_BUFS 1
#endif

// Output of the GEMM: D = AB^T as BF16, as FP32, or D += AB^T in FP32.
enum GemmOut : int { kOutBf16 = 0, kOutF32 = 1, kOutF32Add = 2 };

template <int CG, int BN, int BK>
struct GemmCfg {
  static_assert(CG == 1 || CG == 2, "CTA group of 1 or 2");
  static_assert(BN == 128 || BN == 256, "tile width 128 or 256");
  static_assert(BK == 64 || BK == 128, "stage depth 64 or 128");
  static constexpr int kBM = 128 * CG;            // tile rows
  static constexpr int kBNC = BN / CG;            // rows of B in each CTA
  static constexpr int kNB = BN / 128;            // 128-row scale chunks of B
  static constexpr int kSub = 128 / BK;           // stages per 128-deep scale group
  static constexpr int kStagesPerSf = 4 * kSub;   // stages per scale chunk (4 groups)
  static constexpr uint32_t kABytes = 128 * BK;
  static constexpr uint32_t kBBytes = kBNC * BK;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr int kSfSlots = 3;              // shared-memory ring of scale chunks
  static constexpr uint32_t kSfaBytes = 512;
  static constexpr uint32_t kSfbBytes = 512 * kNB;
  static constexpr uint32_t kSfSlotBytes = kSfaBytes + kSfbBytes;
  static constexpr int kEpiWarps = 8;
  // epilogue staging: per warp kEpiBufs buffers of 32 rows x 32 BF16 columns
  static constexpr int kEpiBufs = PURO_GEMM_EPI_BUFS;
  static constexpr uint32_t kEpiChunkBytes = 32 * 32 * 2;
  static constexpr uint32_t kEpiBytes = kEpiWarps * kEpiBufs * kEpiChunkBytes;
  static constexpr int kStages0 =
      (int)((221 * 1024 - kSfSlots * kSfSlotBytes - kEpiBytes - 1024) / kStageBytes);
  static constexpr int kStages = kStages0 > 16 ? 16 : kStages0;
  static constexpr int kNacc = 2;                 // accumulators in TMEM
  static constexpr bool kSfInTail = (BN == 256);  // scales in the other accumulator's tail
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kEpiCols = BN / 2;         // columns per epilogue warp
  static constexpr int kSfCol = 256;              // BN = 128: 2 slots of 16 columns after both accumulators
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr uint32_t kOffA = 0;
  static constexpr uint32_t kOffB = kOffA + kStages * kABytes;
  static constexpr uint32_t kOffSf = kOffB + kStages * kBBytes;
  static constexpr uint32_t kOffEpi = (kOffSf + kSfSlots * kSfSlotBytes + 1023) / 1024 * 1024;
  static constexpr uint32_t kOffBar = kOffEpi + kEpiBytes;
  static constexpr uint32_t kNumBars = 2 * kStages + kSfSlots + 4 * kNacc + 1;
  static constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
  static constexpr uint32_t kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert(kStages >= 4, "pipeline depth");
  // instruction descriptor: E4M3 x E4M3 (formats 0), UE8M0 scales (bit 23),
  // K-major A and B, N = BN (bits 17-22, N >> 3), M = 128*CG (bits 24-28,
  // M >> 4), dense, K = 32; the scale-factor ids (bits 29-30 for A, 4-5 for
  // B) are or-ed in per MMA.
  static constexpr uint32_t kIdesc =
      ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(kBM >> 4) << 24);
  static constexpr uint32_t kTxPerStage = CG * (kABytes + kBBytes);
  // half-width tiles (BN/2 output columns: N = BN/2 MMAs, half the B rows)
  static constexpr uint32_t kIdescHalf =
      ((uint32_t)((BN / 2) >> 3) << 17) | (1u << 23) | ((uint32_t)(kBM >> 4) << 24);
  static constexpr uint32_t kTxPerStageHalf = CG * (kABytes + kBBytes / 2);
  static constexpr uint32_t kTxPerSf = CG * kSfSlotBytes;
};

// Shared-memory matrix descriptor of a K-major operand tile whose rows are BK
// bytes: 128-byte swizzle (8-row groups 1024 B apart) for BK = 128, 64-byte
// swizzle (8-row groups 512 B apart) for BK = 64.
template <int BK>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  if (BK == 128) return desc_sw128_kmajor(saddr);
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | (1ull << 16) | ((uint64_t)(512u >> 4) << 32) |
         (1ull << 46) | (4ull << 61);
}

// Epilogue of one warp for one tile: its 32 accumulator rows x kEpiCols
// columns (in r) go through the warp's staging buffers, 64 bytes per row per
// chunk (32 BF16 or 16 FP32 columns), one TMA store or reduce-add per chunk.
template <class C, int OUT>
__device__ __forceinline__ void epilogue_store(const uint32_t (&r)[C::kEpiCols], const CUtensorMap* tmd,
                                               uint8_t* ebuf, int& ebufc, int lane, int row0, int gcol,
                                               int rows_a, int rows_b) {
  constexpr int kCC = (OUT == kOutBf16) ? 32 : 16;  // columns per chunk
  if (row0 >= rows_a) return;
#pragma unroll
  for (int c = 0; c < C::kEpiCols / kCC; ++c) {
    if (gcol + c * kCC < rows_b) {
      uint8_t* buf = ebuf + (ebufc % C::kEpiBufs) * C::kEpiChunkBytes;
      if (lane == 0) bulk_wait_group_read<C::kEpiBufs - 1>();
      __syncwarp();
      uint32_t pk[16];
      if (OUT == kOutBf16) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[c * 32 + 2 * e]),
                                                   __uint_as_float(r[c * 32 + 2 * e + 1]));
          pk[e] = *reinterpret_cast<uint32_t*>(&h);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) pk[e] = r[c * 16 + e];
      }
      uint4* dst = reinterpret_cast<uint4*>(buf + lane * 64);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (OUT == kOutF32Add)
          tma_reduce_add_2d(tmd, buf, gcol + c * kCC, row0);
        else
          tma_store_2d(tmd, buf, gcol + c * kCC, row0);
        bulk_commit_group();
      }
      ++ebufc;
    }
  }
}

template <int CG, int BN, int BK, int OUT0, int OUT1>
__global__ void __launch_bounds__(GemmCfg<CG, BN, BK>::kThreads, 1)
    gemm_block_scaled_kernel(const __grid_constant__ CUtensorMap tm_a0,
                             const __grid_constant__ CUtensorMap tm_b0,
                             const __grid_constant__ CUtensorMap tm_sfa0,
                             const __grid_constant__ CUtensorMap tm_sfb0,
                             const __grid_constant__ CUtensorMap tm_d0,
                             const __grid_constant__ CUtensorMap tm_a1,
                             const __grid_constant__ CUtensorMap tm_b1,
                             const __grid_constant__ CUtensorMap tm_sfa1,
                             const __grid_constant__ CUtensorMap tm_sfb1,
                             const __grid_constant__ CUtensorMap tm_d1,
                             const __grid_constant__ CUtensorMap tm_bh0,
                             const __grid_constant__ CUtensorMap tm_bh1,
                             const __grid_constant__ GemmParams p) {
  using C = GemmCfg<CG, BN, BK>;
  constexpr int S = C::kStages;
  constexpr int NA = C::kNacc;
  constexpr int R = C::kSfSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + S;
  uint64_t* sfe = bars + 2 * S;                 // scale ring slots free again
  uint64_t* accf = bars + 2 * S + R;
  uint64_t* acce = bars + 2 * S + R + NA;
  uint64_t* drain = bars + 2 * S + R + 2 * NA;
  uint64_t* sft = bars + 2 * S + R + 2 * NA + 1;  // accumulator tail (scale area) drained
  uint64_t* tld = sft + NA;                        // this CTA's tail loads done (local)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = (CG == 2) ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  const int cluster_id = blockIdx.x / CG;
  const int num_clusters = gridDim.x / CG;
  const int nunits = unit_count(p, cluster_id, num_clusters);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int r = 0; r < R; ++r) mbar_init(&sfe[r], 1);
    for (int a = 0; a < NA; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], C::kEpiWarps * CG);
      mbar_init(&sft[a], (C::kEpiWarps / 2) * CG);
      mbar_init(&tld[a], C::kEpiWarps / 2);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_a0);
    prefetch_tmap(&tm_b0);
    prefetch_tmap(&tm_sfa0);
    prefetch_tmap(&tm_sfb0);
    prefetch_tmap(&tm_d0);
    prefetch_tmap(&tm_bh0);
    if (p.nprob > 1) {
      prefetch_tmap(&tm_a1);
      prefetch_tmap(&tm_b1);
      prefetch_tmap(&tm_sfa1);
      prefetch_tmap(&tm_sfb1);
      prefetch_tmap(&tm_d1);
    }
  }
  if (warp == 1) {
    tmem_alloc<CG>(tmem_slot, 512);
    tmem_relinquish<CG>();
  }
  tc_fence_before();
  cluster_or_block_sync<CG>();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // operands may come from the kernel just before this one on the stream
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int sfc = 0;  // scale chunks loaded so far (ring position)
    uint32_t issued_mask = 0, issued_phase = 0;
    bool ok = true;
    for (int ui = 0; ui < nunits && ok; ++ui) {
      const int u = unit_at(p, cluster_id, num_clusters, ui);
      const int pr = u >= p.tiles0 ? 1 : 0;
      const GemmProblem& P = p.prob[pr];
      int tile, h;
      decode_unit(P, u - (pr ? p.tiles0 : 0), tile, h);
      const bool halft = h >= 0;
      const CUtensorMap* tm_a = pr ? &tm_a1 : &tm_a0;
      const CUtensorMap* tm_b = halft ? (pr ? &tm_bh1 : &tm_bh0) : (pr ? &tm_b1 : &tm_b0);
      const CUtensorMap* tm_sfa = pr ? &tm_sfa1 : &tm_sfa0;
      const CUtensorMap* tm_sfb = pr ? &tm_sfb1 : &tm_sfb0;
      int tm, tn;
      tile_coords(P, tile, tm, tn);
      const int a_row = tm * C::kBM + 128 * (int)rank;
      const int b_col0 = tn * BN + (halft ? (BN / 2) * h : 0);   // first output column
      const int b_row = b_col0 + (halft ? C::kBNC / 2 : C::kBNC) * (int)rank;
      const uint32_t tx = halft ? C::kTxPerStageHalf : C::kTxPerStage;
      for (int kb = 0; kb < P.kblocks; ++kb) {
        if (!mbar_wait_warp(&empty[stage], phase ^ 1, abort_flag)) { ok = false; break; }
        const bool sf = (kb % C::kStagesPerSf) == 0;
        const int slot = sfc % R;
        if (sf && !mbar_wait_warp(&sfe[slot], ((sfc / R) & 1) ^ 1, abort_flag)) { ok = false; break; }
        if (elect_one()) {
          if (leader)
            mbar_arrive_expect_tx(&full[stage], tx + (sf ? C::kTxPerSf : 0u));
          const uint32_t bar = leader_addr<CG>(&full[stage]);
          tma_load_2d<CG>(smem + C::kOffA + stage * C::kABytes, tm_a, kb * BK, a_row, bar);
          tma_load_2d<CG>(smem + C::kOffB + stage * C::kBBytes, tm_b, kb * BK, b_row, bar);
          if (sf) {
            uint8_t* sfbuf = smem + C::kOffSf + slot * C::kSfSlotBytes;
            const int chunk = kb / C::kStagesPerSf;
            tma_load_3d<CG>(sfbuf, tm_sfa, 0, chunk, a_row >> 7, bar);
            tma_load_3d<CG>(sfbuf + C::kSfaBytes, tm_sfb, 0, chunk, b_col0 >> 7, bar);
          }
        }
        if (sf) ++sfc;
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1; }
      }
    }
    // in the leader, let every load of this cluster land before the block can exit
    if (lane == 0 && leader) {
      for (int s = 0; s < S; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(&full[s], (issued_phase >> s) & 1u, &no_abort, 100000000ull);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      int sfc = 0;  // scale chunks copied to TMEM so far
      const uint64_t adesc0 = desc_kmajor<BK>(smem_u32(smem + C::kOffA));
      const uint64_t bdesc0 = desc_kmajor<BK>(smem_u32(smem + C::kOffB));
      for (int ui = 0; ui < nunits && ok; ++ui, ++it) {
        const int u = unit_at(p, cluster_id, num_clusters, ui);
        const int pr = u >= p.tiles0 ? 1 : 0;
        const int kblocks = p.prob[pr].kblocks;
        int tile_unused, h;
        decode_unit(p.prob[pr], u - (pr ? p.tiles0 : 0), tile_unused, h);
        const uint32_t idesc_base = h >= 0 ? C::kIdescHalf : C::kIdesc;
        const int acc = it % NA;
        const uint32_t acc_phase = (it / NA) & 1;
        if (!mbar_wait_warp(&acce[acc], acc_phase ^ 1, abort_flag)) break;
        // scale slots of this tile: the tail of the other accumulator, free once
        // the previous tile's epilogue has read it
        if (C::kSfInTail && it > 0 &&
            !mbar_wait_warp(&sft[acc ^ 1], ((it - 1) / NA) & 1, abort_flag))
          break;
        tc_fence_after();
        const uint32_t t_acc = tmem + acc * BN;
        const uint32_t t_sfreg = tmem + (C::kSfInTail ? (uint32_t)((acc ^ 1) * BN + BN - 32) : C::kSfCol);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          if ((kb % C::kStagesPerSf) == 0) {
            // a new chunk of scales (4 groups of 128 along K) -> TMEM slot sfc & 1;
            // its shared-memory slot is released once the copy has completed
            if (elect_one()) {
              const uint32_t t_new = t_sfreg + 16 * (sfc & 1);
              const uint8_t* sfbuf = smem + C::kOffSf + (sfc % R) * C::kSfSlotBytes;
              tc_cp_32x128b_warpx4<CG>(t_new, desc_dense_rows16(smem_u32(sfbuf)));
#pragma unroll
              for (int h = 0; h < C::kNB; ++h)
                tc_cp_32x128b_warpx4<CG>(t_new + 4 + 4 * h,
                                         desc_dense_rows16(smem_u32(sfbuf + C::kSfaBytes + 512 * h)));
              tc_commit_all<CG>(&sfe[sfc % R]);
            }
            ++sfc;
          }
          if (elect_one()) {
            const uint32_t t_sf = t_sfreg + 16 * ((sfc - 1) & 1);
            const uint32_t j = (uint32_t)((kb / C::kSub) & 3);  // 128-group within the chunk
            const uint32_t idesc = idesc_base | (j << 29) | (j << 4);
            // start-address field (16-byte units) of the stage's descriptors
            const uint64_t adesc = adesc0 + (uint64_t)(stage * (C::kABytes >> 4));
            const uint64_t bdesc = bdesc0 + (uint64_t)(stage * (C::kBBytes >> 4));
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              tc_mma_mxf8<CG>(t_acc, adesc + 2 * k, bdesc + 2 * k, idesc, t_sf, t_sf + 4,
                              (kb | k) != 0 ? 1u : 0u);
            tc_commit_all<CG>(&empty[stage]);
          }
          if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_all<CG>(&accf[acc]);
      }
      // wait until every MMA and copy this warp issued has completed
      if (elect_one()) tc_commit_local<CG>(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, 100000000ull);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int sp = warp & 3;                 // TMEM sub-partition this warp may access
    const int half = (warp - 2) >> 2;        // which half of the columns
    uint8_t* ebuf = smem + C::kOffEpi + (warp - 2) * C::kEpiBufs * C::kEpiChunkBytes;
    int ebufc = 0;  // chunks staged so far (staging buffer ring position)
    int it = 0;
    for (int ui = 0; ui < nunits; ++ui, ++it) {
      const int u = unit_at(p, cluster_id, num_clusters, ui);
      const int pr = u >= p.tiles0 ? 1 : 0;
      const GemmProblem& P = p.prob[pr];
      int tile, h;
      decode_unit(P, u - (pr ? p.tiles0 : 0), tile, h);
      int tm, tn;
      tile_coords(P, tile, tm, tn);
      const int acc = it % NA;
      const uint32_t acc_phase = (it / NA) & 1;
      if (!mbar_wait(&accf[acc], acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t t_base =
          tmem + ((uint32_t)(sp * 32) << 16) + acc * BN + half * C::kEpiCols;
      uint32_t r[C::kEpiCols];
      constexpr int NC = C::kEpiCols / 32;
      if (C::kSfInTail && half == 1) {
        // the last 32 columns first: the next tile's scales go there.  The
        // other warp of this sub-partition holds its own loads back until
        // these have completed (barrier tld), so the hand-over is not queued
        // behind 128 columns of its loads.
        tmem_ld_32x32b_x32(t_base + (NC - 1) * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[(NC - 1) * 32]));
        tmem_ld_wait();
        regs_after_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[(NC - 1) * 32]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive_leader<CG>(&sft[acc]);
          mbar_arrive(&tld[acc]);
        }
#pragma unroll
        for (int c = 0; c < NC - 1; ++c)
          tmem_ld_32x32b_x32(t_base + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < NC - 1; ++c) regs_after_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
      } else {
        // (per-accumulator barrier: its phase cannot run two tiles ahead of
        // this wait, since that tile's MMAs need this warp's release below)
        if (C::kSfInTail && !mbar_wait(&tld[acc], acc_phase, abort_flag)) break;
#pragma unroll
        for (int c = 0; c < NC; ++c)
          tmem_ld_32x32b_x32(t_base + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < NC; ++c) regs_after_wait(*reinterpret_cast<uint32_t(*)[32]>(&r[c * 32]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader<CG>(&acce[acc]);
      const int row0 = tm * C::kBM + 128 * (int)rank + sp * 32;
      // a half-width unit has BN/2 valid accumulator columns (the MMA wrote only
      // those; the rest were loaded above for the tail hand-over and are dropped)
      const int gcol = tn * BN + (h >= 0 ? (BN / 2) * h : 0) + half * C::kEpiCols;
      if (h < 0 || half * C::kEpiCols < BN / 2) {
        if (pr == 0)
          epilogue_store<C, OUT0>(r, &tm_d0, ebuf, ebufc, lane, row0, gcol, P.rows_a, P.rows_b);
        else
          epilogue_store<C, OUT1>(r, &tm_d1, ebuf, ebufc, lane, row0, gcol, P.rows_a, P.rows_b);
      }
    }
    // the staging buffers must stay valid until the stores have read them
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }

  tc_fence_before();
  cluster_or_block_sync<CG>();
  tc_fence_after();
  if (warp == 1) tmem_dealloc<CG>(tmem, 512);
}

}  // namespace puro
