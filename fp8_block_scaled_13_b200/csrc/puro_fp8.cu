// C ABI of the block-scaled FP8 linear layer (declared in include/puro_fp8.h).
//
// Host side: argument validation (before any CUDA call), device check
// (sm_100 only), TMA tensor-map encoding through the driver entry point
// (no link against libcuda), and kernel launches on the caller's stream.
// All kernels live in this one translation unit so that they share the
// device error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <functional>
#include <mutex>
#include <queue>
#include <vector>

#include "../../include/puro_fp8.h"
#include "common.cuh"
#include "gemm.cuh"
#include "quant.cuh"

namespace {

constexpr int kMaxDevices = 64;

#ifndef PURO_GEMM_BN
#define PURO_GEMM_BN 256
#endif
#ifndef PURO_GEMM_CG
#define PURO_GEMM_CG 2
#endif

struct DeviceInfo {
  bool checked = false;
  bool supported = false;
  int index = 0;  // CUDA device ordinal (index into the per-device caches)
  int sms = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device: must be compute capability 10.0 (B200, sm_100a).
int current_device(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PURO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return PURO_ERR_CUDA;
    d.supported = (major == 10 && minor == 0);
    d.index = dev;
    d.sms = sms;
    d.checked = true;
  }
  if (!d.supported) return PURO_ERR_UNSUPPORTED_DEVICE;
  *out = &d;
  return PURO_OK;
}

int get_encoder() {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_encode) return PURO_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return PURO_ERR_CUDA;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return PURO_OK;
}

// 2-D byte tensor [outer, inner] with row stride `ld` bytes; box {box_inner,
// box_outer} stored with the given shared-memory swizzle; out-of-range reads
// return zero.
int make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld,
                uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {ld};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PURO_OK : PURO_ERR_CUDA;
}

// Blocked scale array of `rows` rows x `groups` groups seen as a 3-D tensor
// of 32-bit words {128 words per chunk, ceil(groups/4) chunks, ceil(rows/128)
// row blocks}; a box of {128, 1, nblk} loads nblk consecutive row blocks of
// one group quadruple.
int make_map_scales(CUtensorMap* m, const void* base, int64_t rows, int64_t groups, uint32_t nblk) {
  const uint64_t g4 = (uint64_t)((groups + 3) / 4), rb = (uint64_t)((rows + 127) / 128);
  cuuint64_t dims[3] = {128, g4, rb};
  cuuint64_t strides[2] = {512, g4 * 512};
  cuuint32_t box[3] = {128, 1, nblk};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? PURO_OK : PURO_ERR_CUDA;
}

int64_t g4_of(int64_t groups) { return (groups + 3) / 4; }

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? PURO_OK : PURO_ERR_CUDA;
}

// ------------------------------------------------------------------ quant

template <bool ROW, bool COL, bool BLOCK, bool RSHFL, int STAGES>
int launch_quant_cfg(const void* x, int64_t ld_x, const puro::QuantParams& p, const DeviceInfo& dev,
                     cudaStream_t stream) {
  int st = get_encoder();
  if (st != PURO_OK) return st;
  // BF16 input as a 2-D tensor of 16-bit elements {cols, rows}, 128 x 128 boxes
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)p.cols, (cuuint64_t)p.rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld_x * 2};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  if (g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void*>(x), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return PURO_ERR_CUDA;
  // The transposed codes qt [cols][ld_qt] as a 3-D tensor {qt_cols, cols/8,
  // 8} with strides {1, 8 ld_qt, ld_qt} bytes and 128-byte swizzle: a 128 x
  // 16 x 8 box is one tile, its transposed row 8 c_hi + c_lo at staging row
  // 16 c_lo + c_hi, which is how the kernel stages it.  qt_cols: the bytes of
  // a transposed row that are written (rows rounded up to 16 for
  // activations, whose padding codes are 0; n for weights).
  CUtensorMap mqt = m;
  if (COL) {
    const int64_t qt_cols = BLOCK ? p.rows : (p.rows + 15) / 16 * 16;
    cuuint64_t qdims[3] = {(cuuint64_t)qt_cols, (cuuint64_t)(p.cols / 8), 8};
    cuuint64_t qstrides[2] = {(cuuint64_t)p.ld_qt * 8, (cuuint64_t)p.ld_qt};
    cuuint32_t qbox[3] = {128, 16, 8};
    cuuint32_t qestr[3] = {1, 1, 1};
    if (g_encode(&mqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, p.qt, qdims, qstrides, qbox, qestr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return PURO_ERR_CUDA;
  }
  auto kern = puro::quant_kernel<ROW, COL, BLOCK, RSHFL, STAGES>;
  constexpr uint32_t smem = puro::quant_smem_bytes<STAGES>();
  // per device, once (threads racing on the first call both set the same value)
  static std::atomic<bool> attr_done[kMaxDevices] = {};
  if (!attr_done[dev.index].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return PURO_ERR_CUDA;
    attr_done[dev.index].store(true, std::memory_order_release);
  }
  constexpr int64_t kPerSm = STAGES == 1 ? 3 : 2;  // resident CTAs per SM (shared memory)
  const int64_t grid = p.tiles < kPerSm * dev.sms ? p.tiles : kPerSm * dev.sms;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(puro::kQThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, m, mqt, p) != cudaSuccess) return PURO_ERR_CUDA;
  return launch_status();
}

// Short tile streams (up to about 8 tiles per CTA at two CTAs per SM): two
// stages, two CTAs per SM, a static tile schedule.  Longer streams: one
// stage, three CTAs per SM, and the tiles after each CTA's first handed out
// by ticket when the caller gave a tile counter (SMs stream at different
// rates, up to ~35% apart on a B200; with a static split the launch lasts as
// long as its slowest SM: 32768 x 12288 BOTH took 298 us static and 255 us by
// ticket).  Activations share their row scales by shuffles in both forms
// (7% fewer instructions than every lane deriving its own; with three CTAs
// per SM there are warps enough to hide the shuffles' latency).  Weights (at
// most a few thousand tiles) take two stages and the static schedule.  Each
// form was measured faster in its own range.
template <bool ROW, bool COL, bool BLOCK>
int launch_quant(const void* x, int64_t ld_x, const puro::QuantParams& p, const DeviceInfo& dev,
                 cudaStream_t stream) {
  const bool short_stream = p.tiles <= 8 * 2 * (int64_t)dev.sms;
  puro::QuantParams ps = p;
  if (BLOCK || short_stream) ps.ctr = nullptr;
  // the kernel's division-free tile decode (tiles_c >= 1 here; < 2^24)
  ps.tc_magic = 0;
  ps.tc_shift = 0;
  if (ps.tiles_c > 1) {
    int l = 0;
    while ((int64_t(1) << l) < ps.tiles_c) ++l;
    ps.tc_magic = (uint32_t)(((uint64_t(1) << (31 + l)) + (uint64_t)ps.tiles_c - 1) / (uint64_t)ps.tiles_c);
    ps.tc_shift = l - 1;
  }
  if constexpr (BLOCK) {
    return launch_quant_cfg<ROW, COL, BLOCK, false, 2>(x, ld_x, ps, dev, stream);
  } else {
    if (short_stream) return launch_quant_cfg<ROW, COL, BLOCK, ROW, 2>(x, ld_x, ps, dev, stream);
    return launch_quant_cfg<ROW, COL, BLOCK, ROW, 1>(x, ld_x, ps, dev, stream);
  }
}

// ------------------------------------------------------------------ gemm

struct GemmArgs {
  const void* a;    int64_t lda;   // E4M3 [rows_a, K]
  const void* sfa;                 // blocked, rows_a x ceil(K/128) groups
  const void* b;    int64_t ldb;   // E4M3 [rows_b, K]
  const void* sfb;                 // blocked, rows_b x ceil(K/128) groups
  void* d; int64_t ldd;             // output [rows_a, rows_b], ldd elements per row
  int64_t rows_a, rows_b, k;
  int out;                          // puro::GemmOut
};

// Tensor maps of one GEMM: A, B, the scales of A and B, the output, and B
// again with half-height boxes (m[0..5]).
template <int CG, int BN, int BK, int OUT>
int make_gemm_maps(const GemmArgs& g, CUtensorMap* m) {
  using C = puro::GemmCfg<CG, BN, BK>;
  const int64_t kb = (g.k + 127) / 128;
  int st;
  const CUtensorMapSwizzle sw = BK == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if ((st = make_map_u8(&m[0], g.a, g.k, g.rows_a, g.lda, BK, 128, sw)) != PURO_OK) return st;
  if ((st = make_map_u8(&m[1], g.b, g.k, g.rows_b, g.ldb, BK, C::kBNC, sw)) != PURO_OK) return st;
  // B in half-height boxes, for half-width tiles
  if ((st = make_map_u8(&m[5], g.b, g.k, g.rows_b, g.ldb, BK, C::kBNC / 2, sw)) != PURO_OK) return st;
  if ((st = make_map_scales(&m[2], g.sfa, g.rows_a, kb, 1)) != PURO_OK) return st;
  if ((st = make_map_scales(&m[3], g.sfb, g.rows_b, kb, C::kNB)) != PURO_OK) return st;
  // output [rows_a, rows_b], row stride ldd elements; store boxes of 32 rows
  // x 64 bytes (32 BF16 or 16 FP32 columns)
  const bool f32 = OUT != puro::kOutBf16;
  cuuint64_t dims[2] = {(cuuint64_t)g.rows_b, (cuuint64_t)g.rows_a};
  cuuint64_t strides[1] = {(cuuint64_t)g.ldd * (f32 ? 4 : 2)};
  cuuint32_t box[2] = {f32 ? 16u : 32u, 32};
  cuuint32_t estr[2] = {1, 1};
  if (g_encode(&m[4], f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, g.d,
               dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return PURO_ERR_CUDA;
  return PURO_OK;
}

// Longest-processing-time-first assignment of the two problems' tiles to
// `clusters` clusters: tiles in order of decreasing cost (K blocks plus a
// fixed per-tile share for the epilogue), each to the least-loaded cluster;
// every cluster runs its tiles in the order they were assigned.
void make_schedule(puro::GemmParams& p, int clusters) {
  const int units = p.units;
  std::vector<int> order(units);
  for (int u = 0; u < units; ++u) order[u] = u;
  auto cost = [&](int u) { return p.prob[u >= p.tiles0 ? 1 : 0].kblocks + 2; };  // no split units here
  std::stable_sort(order.begin(), order.end(), [&](int x, int y) { return cost(x) > cost(y); });
  using Slot = std::pair<int64_t, int>;  // (load, cluster), least load first, then lowest index
  std::priority_queue<Slot, std::vector<Slot>, std::greater<Slot>> heap;
  for (int c = 0; c < clusters; ++c) heap.push({0, c});
  std::vector<std::vector<int>> lists(clusters);
  for (int u : order) {
    Slot s = heap.top();
    heap.pop();
    lists[s.second].push_back(u);
    heap.push({s.first + cost(u), s.second});
  }
  int off = 0;
  for (int c = 0; c < clusters; ++c) {
    p.sched_off[c] = (uint16_t)off;
    for (int u : lists[c]) p.sched_unit[off++] = (uint16_t)u;
  }
  p.sched_off[clusters] = (uint16_t)off;
  p.sched = 1;
}

// One launch of the GEMM kernel over one problem (g1 == nullptr) or two
// independent problems that share the launch.
template <int CG, int BN, int BK, int OUT0, int OUT1>
int launch_gemm_cfg(const GemmArgs& g0, const GemmArgs* g1, DeviceInfo* dev, cudaStream_t stream) {
  using C = puro::GemmCfg<CG, BN, BK>;
  CUtensorMap m0[6], m1[6];
  int st;
  if ((st = make_gemm_maps<CG, BN, BK, OUT0>(g0, m0)) != PURO_OK) return st;
  if (g1) {
    if ((st = make_gemm_maps<CG, BN, BK, OUT1>(*g1, m1)) != PURO_OK) return st;
  } else {
    memcpy(m1, m0, sizeof(m0));  // unused by a one-problem launch
  }
  auto kern = puro::gemm_block_scaled_kernel<CG, BN, BK, OUT0, OUT1>;
  // per device, once (threads racing on the first call both store the same value)
  static std::atomic<int> max_clusters[kMaxDevices] = {};
  const int dev_id = dev->index;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;  // the occupancy query below uses the cluster attribute only
  if (max_clusters[dev_id].load(std::memory_order_acquire) == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) !=
        cudaSuccess)
      return PURO_ERR_CUDA;
    int n = 0;
    cfg.gridDim = dim3(CG * (dev->sms / CG));
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) n = dev->sms / CG;
    max_clusters[dev_id].store(n < puro::kMaxSchedClusters ? n : puro::kMaxSchedClusters,
                               std::memory_order_release);
  }
  static thread_local puro::GemmParams p;  // ~4.5 KB: kept off the stack
  memset(&p, 0, sizeof(p));
  const GemmArgs* gs[2] = {&g0, g1};
  p.nprob = g1 ? 2 : 1;
  for (int i = 0; i < p.nprob; ++i) {
    const GemmArgs& g = *gs[i];
    p.prob[i].rows_a = (int32_t)g.rows_a;
    p.prob[i].rows_b = (int32_t)g.rows_b;
    p.prob[i].kblocks = (int32_t)((g.k + BK - 1) / BK);
    p.prob[i].tiles_m = (int32_t)((g.rows_a + C::kBM - 1) / C::kBM);
    p.prob[i].tiles_n = (int32_t)((g.rows_b + BN - 1) / BN);
    // the larger operand is walked in the slower index, so that the tiles
    // running at the same time share its rows and L2 keeps them
    p.prob[i].n_fastest = g.rows_a > g.rows_b ? 1 : 0;
  }
  const int C_max = max_clusters[dev_id].load(std::memory_order_acquire);
  for (int i = 0; i < p.nprob; ++i) {
    const int64_t t = (int64_t)p.prob[i].tiles_m * p.prob[i].tiles_n;
    p.prob[i].split_from = (int32_t)t;
    p.prob[i].units = (int32_t)t;
  }
  if (!g1 && BN == 256) {
    // one GEMM: if the last wave of tiles would fill at most half the clusters,
    // split its tiles into half-width tiles, which then all run at once
    const int64_t t = p.prob[0].split_from;
    const int64_t full = (t / C_max) * C_max, rest = t - full;
    if (rest > 0 && 2 * rest <= C_max) {
      p.prob[0].split_from = (int32_t)full;
      p.prob[0].units = (int32_t)(full + 2 * rest);
    }
  }
  p.tiles0 = p.prob[0].units;
  p.units = p.prob[0].units + (g1 ? p.prob[1].units : 0);
  const int clusters = p.units < C_max ? p.units : C_max;
  if (g1 && p.units <= puro::kMaxSchedUnits) make_schedule(p, clusters);
  cfg.gridDim = dim3(CG * clusters);
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, kern, m0[0], m0[1], m0[2], m0[3], m0[4], m1[0], m1[1], m1[2], m1[3],
                         m1[4], m0[5], m1[5], p) != cudaSuccess)
    return PURO_ERR_CUDA;
  return launch_status();
}

int launch_gemm(const GemmArgs& g, cudaStream_t stream) {
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != PURO_OK) return st;
  if ((st = get_encoder()) != PURO_OK) return st;
  if (g.rows_a == 0 || g.rows_b == 0) return PURO_OK;
  if (g.k == 0) {
    // empty reduction: the product is exactly zero (nothing to add when accumulating)
    if (g.out == puro::kOutF32Add) return PURO_OK;
    const size_t es = g.out == puro::kOutBf16 ? 2 : 4;
    if (cudaMemset2DAsync(g.d, (size_t)g.ldd * es, 0, (size_t)g.rows_b * es, (size_t)g.rows_a,
                          stream) != cudaSuccess)
      return PURO_ERR_CUDA;
    return PURO_OK;
  }
  constexpr int CG = PURO_GEMM_CG, BN = PURO_GEMM_BN, BK = PURO_GEMM_BK;
  switch (g.out) {
    case puro::kOutBf16:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutBf16, puro::kOutBf16>(g, nullptr, dev, stream);
    case puro::kOutF32:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutF32, puro::kOutF32>(g, nullptr, dev, stream);
    case puro::kOutF32Add:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutF32Add, puro::kOutF32Add>(g, nullptr, dev, stream);
    default:
      return PURO_ERR_LAYOUT;
  }
}

// Two independent GEMMs in one launch: g0 with a BF16 output (the data
// gradient) and g1 with any output kind (the weight gradient).  A problem
// that is empty, or has an empty reduction, is run on its own.
int launch_gemm_pair(const GemmArgs& g0, const GemmArgs& g1, cudaStream_t stream) {
  const bool e0 = g0.rows_a == 0 || g0.rows_b == 0 || g0.k == 0;
  const bool e1 = g1.rows_a == 0 || g1.rows_b == 0 || g1.k == 0;
  if (e0 || e1) {
    int st = launch_gemm(g0, stream);
    if (st != PURO_OK) return st;
    return launch_gemm(g1, stream);
  }
  DeviceInfo* dev = nullptr;
  int st = current_device(&dev);
  if (st != PURO_OK) return st;
  if ((st = get_encoder()) != PURO_OK) return st;
  constexpr int CG = PURO_GEMM_CG, BN = PURO_GEMM_BN, BK = PURO_GEMM_BK;
  if (g0.out != puro::kOutBf16) return PURO_ERR_LAYOUT;
  switch (g1.out) {
    case puro::kOutBf16:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutBf16, puro::kOutBf16>(g0, &g1, dev, stream);
    case puro::kOutF32:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutBf16, puro::kOutF32>(g0, &g1, dev, stream);
    case puro::kOutF32Add:
      return launch_gemm_cfg<CG, BN, BK, puro::kOutBf16, puro::kOutF32Add>(g0, &g1, dev, stream);
    default:
      return PURO_ERR_LAYOUT;
  }
}

// Shape/alignment checks shared by the three GEMMs.
int check_mat(const void* p, int64_t ld, int64_t min_ld, int64_t elem_bytes) {
  if (!p) return PURO_ERR_NULL;
  if (!aligned16(p)) return PURO_ERR_ALIGN;
  if (ld < min_ld) return PURO_ERR_SHAPE;
  if ((ld * elem_bytes) % 16) return PURO_ERR_ALIGN;
  return PURO_OK;
}

constexpr int64_t kMaxDim = (int64_t)1 << 31;

}  // namespace

// Argument checks and GEMM mapping of the gradient GEMMs.  They return
// PURO_OK with *g filled in, kNothingToDo when the output is empty, or an
// error status; nothing is launched.
constexpr int kNothingToDo = 1;

int dgrad_args(const void* qdy, int64_t ld_qdy, const void* sdy, const void* qwt, int64_t ld_qwt,
               const void* sw_bwd, void* dx, int64_t ld_dx, int64_t m, int64_t n, int64_t k,
               GemmArgs* g) {
  if (m < 0 || n < 0 || k < 0 || m >= kMaxDim || n >= kMaxDim || k >= kMaxDim) return PURO_ERR_SHAPE;
  if (n % 128 || k % 128) return PURO_ERR_SHAPE;
  if (m == 0 || k == 0) return kNothingToDo;
  int r;
  if ((r = check_mat(dx, ld_dx, k, 2)) != PURO_OK) return r;
  if (n > 0) {
    if ((r = check_mat(qdy, ld_qdy, n, 1)) != PURO_OK) return r;
    if ((r = check_mat(qwt, ld_qwt, n, 1)) != PURO_OK) return r;
    if (!sdy || !sw_bwd) return PURO_ERR_NULL;
    if (!aligned16(sdy) || !aligned16(sw_bwd)) return PURO_ERR_ALIGN;
  }
  *g = GemmArgs{qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, m, k, n, puro::kOutBf16};
  return PURO_OK;
}

int wgrad_args(const void* qdyt, int64_t ld_qdyt, const void* sdyt, const void* qxt, int64_t ld_qxt,
               const void* sxt, void* dw, int64_t ld_dw, int64_t m, int64_t n, int64_t k, int out,
               GemmArgs* g) {
  if (m < 0 || n < 0 || k < 0 || m >= kMaxDim || n >= kMaxDim || k >= kMaxDim) return PURO_ERR_SHAPE;
  if (n % 128 || k % 128) return PURO_ERR_SHAPE;
  if (n == 0 || k == 0) return kNothingToDo;
  int r;
  if ((r = check_mat(dw, ld_dw, k, out == puro::kOutBf16 ? 2 : 4)) != PURO_OK) return r;
  if (m > 0) {
    if ((r = check_mat(qdyt, ld_qdyt, (m + 15) / 16 * 16, 1)) != PURO_OK) return r;
    if ((r = check_mat(qxt, ld_qxt, (m + 15) / 16 * 16, 1)) != PURO_OK) return r;
    if (!sdyt || !sxt) return PURO_ERR_NULL;
    if (!aligned16(sdyt) || !aligned16(sxt)) return PURO_ERR_ALIGN;
  }
  *g = GemmArgs{qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, n, k, m, out};
  return PURO_OK;
}

extern "C" {

const char* puro_fp8_status_string(int status) {
  switch (status) {
    case PURO_OK: return "PURO_OK";
    case PURO_ERR_NULL: return "PURO_ERR_NULL: a required pointer is NULL";
    case PURO_ERR_ALIGN: return "PURO_ERR_ALIGN: pointer or leading dimension not 16-byte aligned";
    case PURO_ERR_SHAPE: return "PURO_ERR_SHAPE: size or leading dimension out of range";
    case PURO_ERR_LAYOUT: return "PURO_ERR_LAYOUT: unknown layout flag";
    case PURO_ERR_CUDA: return "PURO_ERR_CUDA: a CUDA call failed";
    case PURO_ERR_UNSUPPORTED_DEVICE: return "PURO_ERR_UNSUPPORTED_DEVICE: needs sm_100 (B200)";
    case PURO_ERR_DEVICE_TIMEOUT: return "PURO_ERR_DEVICE_TIMEOUT: a bounded device wait expired";
    default: return "unknown puro_status";
  }
}

int64_t puro_fp8_blocked_scale_bytes(int64_t rows, int64_t groups) {
  if (rows <= 0 || groups <= 0) return 0;
  return ((rows + 127) / 128) * g4_of(groups) * 512;
}

int puro_fp8_quant_act(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int layout,
                       void* q, int64_t ld_q, void* s, void* qt, int64_t ld_qt, void* st,
                       uint32_t* tile_counter, void* stream) {
  if (layout != PURO_ROWWISE && layout != PURO_COLWISE && layout != PURO_BOTH)
    return PURO_ERR_LAYOUT;
  if (rows < 0 || cols < 0 || rows >= kMaxDim || cols >= kMaxDim) return PURO_ERR_SHAPE;
  if (cols % 128) return PURO_ERR_SHAPE;
  if (rows == 0 || cols == 0) return PURO_OK;
  if ((cols / 128) * ((rows + 127) / 128) >= kMaxDim) return PURO_ERR_SHAPE;
  int r;
  if ((r = check_mat(x, ld_x, cols, 2)) != PURO_OK) return r;
  const bool row = layout & PURO_ROWWISE, col = layout & PURO_COLWISE;
  if (row) {
    if ((r = check_mat(q, ld_q, cols, 1)) != PURO_OK) return r;
    if (!s) return PURO_ERR_NULL;
    if (!aligned16(s)) return PURO_ERR_ALIGN;
  }
  if (col) {
    if ((r = check_mat(qt, ld_qt, (rows + 15) / 16 * 16, 1)) != PURO_OK) return r;
    if (!st) return PURO_ERR_NULL;
    if (!aligned16(st)) return PURO_ERR_ALIGN;
  }
  if (reinterpret_cast<uintptr_t>(tile_counter) % 8) return PURO_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((r = current_device(&dev)) != PURO_OK) return r;
  puro::QuantParams p{};
  p.ctr = tile_counter;
  p.rows = rows;
  p.cols = cols;
  p.q = static_cast<uint8_t*>(q);
  p.ld_q = ld_q;
  p.s = static_cast<uint8_t*>(s);
  p.s_g4 = g4_of(cols / 128);
  p.qt = static_cast<uint8_t*>(qt);
  p.ld_qt = ld_qt;
  p.st = static_cast<uint8_t*>(st);
  p.st_g4 = g4_of((rows + 127) / 128);
  p.tiles_c = (int32_t)(cols / 128);
  p.tiles = (int32_t)(p.tiles_c * ((rows + 127) / 128));
  cudaStream_t sm = static_cast<cudaStream_t>(stream);
  if (row && col) return launch_quant<true, true, false>(x, ld_x, p, *dev, sm);
  if (row) return launch_quant<true, false, false>(x, ld_x, p, *dev, sm);
  return launch_quant<false, true, false>(x, ld_x, p, *dev, sm);
}

int puro_fp8_quant_weight(const void* w, int64_t n, int64_t k, int64_t ld_w, void* q, int64_t ld_q,
                          void* s, void* qt, int64_t ld_qt, void* s_fwd, void* s_bwd,
                          void* stream) {
  if (n < 0 || k < 0 || n >= kMaxDim || k >= kMaxDim || n % 128 || k % 128) return PURO_ERR_SHAPE;
  if (n == 0 || k == 0) return PURO_OK;
  if ((k / 128) * (n / 128) >= kMaxDim) return PURO_ERR_SHAPE;
  int r;
  if ((r = check_mat(w, ld_w, k, 2)) != PURO_OK) return r;
  if ((r = check_mat(q, ld_q, k, 1)) != PURO_OK) return r;
  if (!s) return PURO_ERR_NULL;
  if (qt && (r = check_mat(qt, ld_qt, n, 1)) != PURO_OK) return r;
  if ((s_fwd && !aligned16(s_fwd)) || (s_bwd && !aligned16(s_bwd))) return PURO_ERR_ALIGN;
  DeviceInfo* dev = nullptr;
  if ((r = current_device(&dev)) != PURO_OK) return r;
  puro::QuantParams p{};
  p.rows = n;
  p.cols = k;
  p.q = static_cast<uint8_t*>(q);
  p.ld_q = ld_q;
  p.qt = static_cast<uint8_t*>(qt);
  p.ld_qt = ld_qt;
  p.sw = static_cast<uint8_t*>(s);
  p.sw_fwd = static_cast<uint8_t*>(s_fwd);
  p.fwd_g4 = g4_of(k / 128);
  p.sw_bwd = static_cast<uint8_t*>(s_bwd);
  p.bwd_g4 = g4_of(n / 128);
  p.tiles_c = (int32_t)(k / 128);
  p.tiles = (int32_t)(p.tiles_c * (n / 128));
  cudaStream_t sm = static_cast<cudaStream_t>(stream);
  if (qt) return launch_quant<true, true, true>(w, ld_w, p, *dev, sm);
  return launch_quant<true, false, true>(w, ld_w, p, *dev, sm);
}

int puro_fp8_gemm_fprop(const void* qx, int64_t ld_qx, const void* sx, const void* qw,
                        int64_t ld_qw, const void* sw_fwd, void* y, int64_t ld_y, int64_t m,
                        int64_t n, int64_t k, void* stream) {
  if (m < 0 || n < 0 || k < 0 || m >= kMaxDim || n >= kMaxDim || k >= kMaxDim) return PURO_ERR_SHAPE;
  if (n % 128 || k % 128) return PURO_ERR_SHAPE;
  if (m == 0 || n == 0) return PURO_OK;
  int r;
  if ((r = check_mat(y, ld_y, n, 2)) != PURO_OK) return r;
  if (k > 0) {
    if ((r = check_mat(qx, ld_qx, k, 1)) != PURO_OK) return r;
    if ((r = check_mat(qw, ld_qw, k, 1)) != PURO_OK) return r;
    if (!sx || !sw_fwd) return PURO_ERR_NULL;
    if (!aligned16(sx) || !aligned16(sw_fwd)) return PURO_ERR_ALIGN;
  }
  GemmArgs g{qx, ld_qx, sx, qw, ld_qw, sw_fwd, y, ld_y, m, n, k, puro::kOutBf16};
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int puro_fp8_gemm_dgrad(const void* qdy, int64_t ld_qdy, const void* sdy, const void* qwt,
                        int64_t ld_qwt, const void* sw_bwd, void* dx, int64_t ld_dx, int64_t m,
                        int64_t n, int64_t k, void* stream) {
  GemmArgs g;
  const int r = dgrad_args(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, m, n, k, &g);
  if (r != PURO_OK) return r == kNothingToDo ? PURO_OK : r;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int puro_fp8_gemm_wgrad(const void* qdyt, int64_t ld_qdyt, const void* sdyt, const void* qxt,
                        int64_t ld_qxt, const void* sxt, void* dw, int64_t ld_dw, int64_t m,
                        int64_t n, int64_t k, void* stream) {
  GemmArgs g;
  const int r = wgrad_args(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, puro::kOutBf16, &g);
  if (r != PURO_OK) return r == kNothingToDo ? PURO_OK : r;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int puro_fp8_gemm_wgrad_f32(const void* qdyt, int64_t ld_qdyt, const void* sdyt, const void* qxt,
                            int64_t ld_qxt, const void* sxt, void* dw, int64_t ld_dw, int64_t m,
                            int64_t n, int64_t k, int accumulate, void* stream) {
  if (accumulate != 0 && accumulate != 1) return PURO_ERR_LAYOUT;
  GemmArgs g;
  const int r = wgrad_args(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k,
                           accumulate ? puro::kOutF32Add : puro::kOutF32, &g);
  if (r != PURO_OK) return r == kNothingToDo ? PURO_OK : r;
  return launch_gemm(g, static_cast<cudaStream_t>(stream));
}

int puro_fp8_gemm_dgrad_wgrad(const void* qdy, int64_t ld_qdy, const void* sdy, const void* qwt,
                              int64_t ld_qwt, const void* sw_bwd, void* dx, int64_t ld_dx,
                              const void* qdyt, int64_t ld_qdyt, const void* sdyt, const void* qxt,
                              int64_t ld_qxt, const void* sxt, void* dw, int64_t ld_dw, int64_t m,
                              int64_t n, int64_t k, int dw_kind, void* stream) {
  if (dw_kind < PURO_DW_BF16 || dw_kind > PURO_DW_F32_ACCUMULATE) return PURO_ERR_LAYOUT;
  const int out = dw_kind == PURO_DW_BF16 ? puro::kOutBf16
                  : dw_kind == PURO_DW_F32 ? puro::kOutF32 : puro::kOutF32Add;
  GemmArgs gd, gw;
  const int rd = dgrad_args(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, m, n, k, &gd);
  if (rd != PURO_OK && rd != kNothingToDo) return rd;
  const int rw = wgrad_args(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, out, &gw);
  if (rw != PURO_OK && rw != kNothingToDo) return rw;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (rd == kNothingToDo) return rw == kNothingToDo ? PURO_OK : launch_gemm(gw, s);
  if (rw == kNothingToDo) return launch_gemm(gd, s);
  return launch_gemm_pair(gd, gw, s);
}

int puro_fp8_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PURO_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, puro::g_status, sizeof(int)) != cudaSuccess) return PURO_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(puro::g_status, &zero, sizeof(int)) != cudaSuccess) return PURO_ERR_CUDA;
  }
  return v;
}

}  // extern "C"

// ------------------------------------------------------------------ self-test

namespace puro {
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
}
}  // namespace puro

extern "C" int puro_fp8_test_schedule(int32_t units0, int32_t kblocks0, int32_t units1,
                                      int32_t kblocks1, int32_t clusters, int32_t* offsets,
                                      int32_t* units) {
  if (!offsets || !units) return PURO_ERR_NULL;
  if (clusters < 1 || clusters > puro::kMaxSchedClusters || units0 < 0 || units1 < 0 ||
      kblocks0 < 0 || kblocks1 < 0 || (int64_t)units0 + units1 > puro::kMaxSchedUnits)
    return PURO_ERR_SHAPE;
  static puro::GemmParams p;  // a few KB: kept off the caller's stack
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  memset(&p, 0, sizeof(p));
  p.nprob = 2;
  p.prob[0].kblocks = kblocks0;
  p.prob[0].units = units0;
  p.prob[1].kblocks = kblocks1;
  p.prob[1].units = units1;
  p.tiles0 = units0;
  p.units = units0 + units1;
  make_schedule(p, clusters);
  for (int c = 0; c <= clusters; ++c) offsets[c] = p.sched_off[c];
  for (int u = 0; u < p.units; ++u) units[u] = p.sched_unit[u];
  return PURO_OK;
}

extern "C" int puro_fp8_test_bounded_wait(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000) limit_ns = 1000;
  if (limit_ns > 5000000000ll) limit_ns = 5000000000ll;
  DeviceInfo* dev = nullptr;
  int r = current_device(&dev);
  if (r != PURO_OK) return r;
  puro::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_ns);
  return launch_status();
}

// ---------------------------------------------------------------- static-scratch entry point
//
// Some callers cannot hand this library any device memory beyond their inputs
// and outputs: an engine that reserves the GPU's memory for its own pool at
// start-up leaves nothing for cudaMalloc (which then fails, or stalls the
// device while the pool gives memory back), and a C caller that only holds
// the buffers it was given has no allocator to ask.  For them, the
// quantizer's tile counter lives in this file-scope array instead: 256
// bytes (one counter pair is used) in the library's own device memory, held
// by every GPU that loads the library until the process exits.  Host code
// needs its device address, which cudaGetSymbolAddress gives once per device
// (the symbol's name is only a host-side stand-in).
namespace {

constexpr size_t kStaticScratchBytes = 256;
static __device__ __align__(256) uint32_t g_static_scratch[kStaticScratchBytes / 4];
uint32_t* g_static_scratch_addr[kMaxDevices] = {};

}  // namespace

extern "C" int puro_fp8_quant_act_static_scratch(const void* x, int64_t rows, int64_t cols,
                                                 int64_t ld_x, int layout, void* q, int64_t ld_q,
                                                 void* s, void* qt, int64_t ld_qt, void* st,
                                                 void* stream) {
  // the sizes this entry point takes (the rest is checked by the common path)
  if (layout != PURO_ROWWISE && layout != PURO_COLWISE && layout != PURO_BOTH)
    return PURO_ERR_LAYOUT;
  if (rows < 0 || cols < 0 || rows >= kMaxDim || cols >= kMaxDim || cols % 128) return PURO_ERR_SHAPE;
  if (rows == 0 || cols == 0) return PURO_OK;
  // the counter's 32-bit tickets: at most one per tile plus one per CTA
  if ((cols / 128) * ((rows + 127) / 128) >= kMaxDim) return PURO_ERR_SHAPE;
  DeviceInfo* dev = nullptr;
  int r = current_device(&dev);
  if (r != PURO_OK) return r;
  uint32_t* ctr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_static_scratch_addr[dev->index]) {
      void* a = nullptr;
      if (cudaGetSymbolAddress(&a, g_static_scratch) != cudaSuccess || a == nullptr)
        return PURO_ERR_CUDA;
      g_static_scratch_addr[dev->index] = static_cast<uint32_t*>(a);
    }
    ctr = g_static_scratch_addr[dev->index];
  }
  // The counter must start at zero.  Each call clears it on its stream before
  // its kernel (the kernel also leaves it zero), so a call that ended early
  // leaves nothing behind; calls that overlap on the GPU share it and race.
  if (cudaMemsetAsync(ctr, 0, 2 * sizeof(uint32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PURO_ERR_CUDA;
  return puro_fp8_quant_act(x, rows, cols, ld_x, layout, q, ld_q, s, qt, ld_qt, st, ctr, stream);
}
