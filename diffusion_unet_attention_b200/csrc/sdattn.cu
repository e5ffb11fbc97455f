// sdattn.cu -- host side of libsdattn: argument checks, TMA tensor maps,
// work partitioning and launches of the sm_100a kernels.  Every entry point is
// declared (and documented) in include/sdattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <mutex>
#include <utility>

#include "sdattn.h"

#include "flash.cuh"
#include "flash_tf32.cuh"
#include "qk_stats.cuh"
#include "row_stats.cuh"
#include "softmax_av.cuh"
#include "unet_ops.cuh"
#include "winograd.cuh"

namespace {

using sdattn::AVCfg;
using sdattn::AVParams;
using sdattn::FlashCfg;
using sdattn::FlashParams;
using sdattn::QKCfg;
using sdattn::QKParams;
using sdattn::RowStatsParams;

constexpr int kMaxDevices = 64;
constexpr int kMaxSplit = 16;
constexpr int kMinBlocksPerSplit = 4;
constexpr int kMinSplitBlocks = 4;   // key tiles per CTA of a cluster-split unit (flash, softmax_av)

// --------------------------------------------------------------------------
// Driver entry point for tensor-map encoding (no link-time libcuda dependency)
// --------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 3-D tiled map: dims {d0 (contiguous), d1, d2}, byte strides of d1 and d2,
// box {b0, b1, 1}, 128-byte swizzle, zero fill outside the tensor.
bool make_map_3d(CUtensorMap* m, const void* ptr, CUtensorMapDataType dt, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// --------------------------------------------------------------------------
// Device facts
// --------------------------------------------------------------------------
int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int sm_count(int dev) {
  static std::atomic<int> cache[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Raises a kernel's dynamic shared-memory limit once per device.
template <typename Kern>
bool ensure_smem(Kern kern, int bytes, std::atomic<uint64_t>& done, int dev) {
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Launch with programmatic stream serialisation: the kernel may begin its
// prologue while the previous kernel of the stream drains (the kernels wait
// for it before touching global memory).
template <typename... KArgs, typename... Args>
bool launch(void (*kern)(KArgs...), int grid, int block, int smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess;
}

// Cluster launch (CTAs of a cluster share work through distributed shared
// memory), with programmatic stream serialisation like every other launch.
template <typename... KArgs, typename... Args>
bool launch_cluster(void (*kern)(KArgs...), int grid, int cluster, int block, int smem, cudaStream_t stream,
                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess;
}

// --------------------------------------------------------------------------
// Validation
// --------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sdattn_status check_desc(const sdattn_desc* d) {
  if (!d) return SDATTN_ERR_INVALID_ARG;
  if (d->B < 1 || d->H < 1 || d->N < 1 || d->M < 1) return SDATTN_ERR_INVALID_ARG;
  if (!std::isfinite(d->scale) || !(d->scale > 0.f)) return SDATTN_ERR_INVALID_ARG;
  if (d->d != 40 && d->d != 80 && d->d != 160) return SDATTN_ERR_UNSUPPORTED;
  if (d->dtype != SDATTN_F16 && d->dtype != SDATTN_BF16) return SDATTN_ERR_UNSUPPORTED;
  const int64_t bh = static_cast<int64_t>(d->B) * d->H;
  if (bh * d->N >= (int64_t(1) << 31) || bh * d->M >= (int64_t(1) << 31)) return SDATTN_ERR_UNSUPPORTED;
  if (bh >= (int64_t(1) << 31)) return SDATTN_ERR_UNSUPPORTED;
  return SDATTN_OK;
}

int64_t a_ld(const sdattn_desc* d) { return (static_cast<int64_t>(d->M) + 3) / 4 * 4; }

// Row stride of fp16-stored A, in elements: 16-byte rows.
int64_t a16_ld(const sdattn_desc* d) { return (static_cast<int64_t>(d->M) + 7) / 8 * 8; }

CUtensorMapDataType elem_type(const sdattn_desc* d) {
  return d->dtype == SDATTN_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

// Column splits of the statistics reduction: the smallest power of two that
// fills the SMs evenly (at least 90% of the last wave), at most kMaxSplit;
// a split that takes the grid past one wave must also shorten the busiest
// CTA's chain (at 32x32, 128 row tiles of 8 blocks: two splits leave 8
// blocks on the busiest CTA and add two hand-offs).
// A split keeps at least kMinBlocksPerSplit column blocks (each split pays a
// partial write and an arrival, which a one-block split cannot hide on a busy
// GPU), except while the doubled grid still fills at most half of the SMs:
// there the shorter chain of blocks per CTA is worth more than the merge.
struct QKPlan {
  int nrt, nb, nsplit, cbs, units;
};

QKPlan plan_qk(const sdattn_desc* d, int nsm) {
  QKPlan pl;
  const int bh = d->B * d->H;
  pl.nrt = (d->N + 127) / 128;
  pl.nb = (d->M + 127) / 128;
  const int64_t base = static_cast<int64_t>(bh) * pl.nrt;
  auto eff = [&](int64_t u) {
    const int64_t waves = (u + nsm - 1) / nsm;
    return static_cast<double>(u) / static_cast<double>(waves * nsm);
  };
  // A CTA's chain, in block times of one epilogue group: its units in turn,
  // each its blocks shared by the epilogue groups plus, when split, the
  // hand-off of the partial statistics (about one block time, measured).
  const int epi = (d->d + 63) / 64 == 3 ? 1 : 2;   // epilogue groups at this head width
  auto chain = [&](int ns) {
    const int cbs = (pl.nb + ns - 1) / ns;
    const int64_t units = base * ((pl.nb + cbs - 1) / cbs);
    return (units + nsm - 1) / nsm * ((cbs + epi - 1) / epi + (ns > 1 ? 1 : 0));
  };
  int ns = 1;
  const int cap = pl.nb < kMaxSplit ? pl.nb : kMaxSplit;
  while (ns * 2 <= cap && (pl.nb / (ns * 2) >= kMinBlocksPerSplit || base * ns * 2 <= nsm / 2) &&
         eff(base * ns) < 0.9 && (base * ns * 2 <= nsm || chain(ns * 2) < chain(ns)))
    ns *= 2;
  pl.cbs = (pl.nb + ns - 1) / ns;
  pl.nsplit = (pl.nb + pl.cbs - 1) / pl.cbs;
  pl.units = static_cast<int>(base * pl.nsplit);
  return pl;
}

// Small calls (every unit has its own CTA) with at most 8 splits per row tile
// merge the splits across a thread-block cluster instead of the workspace.
bool qk_cluster_merge(const QKPlan& pl, int nsm) { return pl.nsplit > 1 && pl.nsplit <= 8 && pl.units <= nsm; }

// Workspace: [tickets: one uint32 per (b, h, row tile), padded to 256 B]
//            [partials: float2 per (b, h, row tile, row, split)]
size_t ws_tickets_bytes(const sdattn_desc* d) {
  const int64_t tiles = static_cast<int64_t>(d->B) * d->H * ((d->N + 127) / 128);
  return static_cast<size_t>((tiles * 4 + 255) / 256 * 256);
}

size_t qk_ws_bytes(const sdattn_desc* d) {
  const int64_t tiles = static_cast<int64_t>(d->B) * d->H * ((d->N + 127) / 128);
  const int nb = (d->M + 127) / 128;
  const int smax = nb < kMaxSplit ? nb : kMaxSplit;
  return ws_tickets_bytes(d) + static_cast<size_t>(tiles) * 128 * smax * sizeof(float2);
}

// Flash workspace, used when a unit's key range is cut between two CTAs:
//   [tickets: one uint32 per (CTA, query tile), padded to 256 B]
//   [partials: per (CTA, query tile, half, row) one row of ROWF floats]
// sized for a grid of one CTA per SM and the most query tiles a CTA runs at d.
int flash_nq_max(int d) { return d == 40 ? 2 : 1; }

size_t flash_ws_tickets_bytes(const sdattn_desc* d, int nsm) {
  return static_cast<size_t>((static_cast<int64_t>(nsm) * flash_nq_max(d->d) * 4 + 255) / 256 * 256);
}

size_t flash_ws_bytes(const sdattn_desc* d, int nsm) {
  const int rowf = (d->d + 3 + 3) / 4 * 4;
  return flash_ws_tickets_bytes(d, nsm) +
         static_cast<size_t>(nsm) * flash_nq_max(d->d) * 2 * 128 * rowf * sizeof(float);
}

// Stand-alone row statistics: one warp per (row, column split).  Rows are
// split over several warps only while there are fewer rows than warps in a
// persistent grid of two CTAs per SM, each split keeping at least 512 columns.
struct RowPlan {
  int64_t rows;
  int nsplit, split_cols, grid;
};

RowPlan plan_rows(const sdattn_desc* d, int nsm) {
  RowPlan pl;
  pl.rows = static_cast<int64_t>(d->B) * d->H * d->N;
  const int64_t warps = static_cast<int64_t>(nsm) * 2 * sdattn::kRowStatsWarps;
  int ns = 1;
  if (pl.rows < warps) {
    const int64_t want = (warps + pl.rows - 1) / pl.rows;
    const int64_t by_len = (d->M + 511) / 512;
    ns = static_cast<int>(std::min<int64_t>(std::min<int64_t>(want, by_len), 64));
    if (ns < 1) ns = 1;
  }
  pl.split_cols = static_cast<int>(((d->M + ns - 1) / ns + 31) / 32 * 32);
  pl.nsplit = (d->M + pl.split_cols - 1) / pl.split_cols;
  const int64_t items = pl.rows * pl.nsplit;
  const int64_t ctas = (items + sdattn::kRowStatsWarps - 1) / sdattn::kRowStatsWarps;
  pl.grid = static_cast<int>(std::min<int64_t>(ctas, static_cast<int64_t>(nsm) * 2));
  return pl;
}

// [tickets: one uint32 per row, padded to 256 B][partials: float2 per (row, split)]
size_t rows_ws_tickets_bytes(const RowPlan& pl) { return static_cast<size_t>((pl.rows * 4 + 255) / 256 * 256); }

size_t rows_ws_bytes(const sdattn_desc* d, int nsm) {
  const RowPlan pl = plan_rows(d, nsm);
  if (pl.nsplit == 1) return 0;
  return rows_ws_tickets_bytes(pl) + static_cast<size_t>(pl.rows) * pl.nsplit * sizeof(float2);
}

size_t ws_bytes(const sdattn_desc* d) {
  const int dev = current_device();
  const size_t qk = qk_ws_bytes(d);
  const int nsm = sm_count(dev < 0 ? 0 : dev);
  const size_t fl = flash_ws_bytes(d, nsm);
  const size_t rs = rows_ws_bytes(d, nsm);
  return std::max(qk, std::max(fl, rs));
}

// --------------------------------------------------------------------------
// Launchers
// --------------------------------------------------------------------------
template <int D, bool BF16, int AMODE = sdattn::kAF32Stats>
sdattn_status launch_qk(const sdattn_desc* d, const void* Q, const void* K, void* A, float* LS, void* ws,
                        cudaStream_t stream) {
  using C = QKCfg<D>;
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  auto kern = sdattn::qk_stats_kernel<D, BF16, AMODE>;
  static std::atomic<uint64_t> smem_done{0};
  if (!ensure_smem(kern, C::SMEM, smem_done, dev)) return SDATTN_ERR_CUDA;

  const int nsm = sm_count(dev);
  const QKPlan pl = plan_qk(d, nsm);
  const uint64_t bh = static_cast<uint64_t>(d->B) * d->H;
  const uint64_t N = d->N, M = d->M;
  CUtensorMap mq, mk, ma;
  if (!make_map_3d(&mq, Q, elem_type(d), D, N, bh, D * 2, N * D * 2, 64, 128)) return SDATTN_ERR_CUDA;
  if (!make_map_3d(&mk, K, elem_type(d), D, M, bh, D * 2, M * D * 2, 64, 128)) return SDATTN_ERR_CUDA;
  if constexpr (AMODE == sdattn::kAF16Stats) {
    const uint64_t lda = a16_ld(d);
    if (!make_map_3d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, M, N, bh, lda * 2, N * lda * 2, 64, 32))
      return SDATTN_ERR_CUDA;
  } else {
    const uint64_t lda = a_ld(d);
    if (!make_map_3d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, N, bh, lda * 4, N * lda * 4, 32, 32))
      return SDATTN_ERR_CUDA;
  }

  QKParams p;
  p.N = d->N;
  p.M = d->M;
  p.BH = static_cast<int>(bh);
  p.nrt = pl.nrt;
  p.nb = pl.nb;
  p.nsplit = pl.nsplit;
  p.cbs = pl.cbs;
  p.units = pl.units;
  p.scale = d->scale;
  p.cmerge = (AMODE != sdattn::kAF32Only && qk_cluster_merge(pl, nsm)) ? 1 : 0;
  p.LS = LS;
  p.tickets = static_cast<uint32_t*>(ws);
  p.part = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + ws_tickets_bytes(d));
  if (p.cmerge)
    return launch_cluster(kern, pl.units, pl.nsplit, C::NTHREADS, C::SMEM, stream, mq, mk, ma, p) ? SDATTN_OK
                                                                                                 : SDATTN_ERR_CUDA;
  const int grid = pl.units < nsm ? pl.units : nsm;
  return launch(kern, grid, C::NTHREADS, C::SMEM, stream, mq, mk, ma, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
}

template <int D, bool BF16, bool AF16 = false>
sdattn_status launch_av(const sdattn_desc* d, const void* A, const float* LS, const void* V, void* O,
                        cudaStream_t stream) {
  using C = AVCfg<D, AF16>;
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  auto kern = sdattn::softmax_av_kernel<D, BF16, AF16>;
  static std::atomic<uint64_t> smem_done{0};
  if (!ensure_smem(kern, C::SMEM, smem_done, dev)) return SDATTN_ERR_CUDA;

  const int nsm = sm_count(dev);
  const uint64_t bh = static_cast<uint64_t>(d->B) * d->H;
  const uint64_t N = d->N, M = d->M;
  CUtensorMap ma, mv;
  if constexpr (AF16) {
    const uint64_t lda = a16_ld(d);
    if (!make_map_3d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, M, N, bh, lda * 2, N * lda * 2, 64, 128))
      return SDATTN_ERR_CUDA;
  } else {
    const uint64_t lda = a_ld(d);
    if (!make_map_3d(&ma, A, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, M, N, bh, lda * 4, N * lda * 4, 32, 128))
      return SDATTN_ERR_CUDA;
  }
  if (!make_map_3d(&mv, V, elem_type(d), D, M, bh, D * 2, M * D * 2, 64, C::BK)) return SDATTN_ERR_CUDA;

  AVParams p;
  p.N = d->N;
  p.M = d->M;
  p.BH = static_cast<int>(bh);
  p.nrt = (d->N + 127) / 128;
  p.nkb = (d->M + C::BK - 1) / C::BK;
  p.units = p.BH * p.nrt;
  p.LS = LS;
  p.O = O;
  // Row tiles filling under half the SMs over long key ranges: a cluster of
  // k CTAs shares each tile's key blocks (k <= 8, k * tiles <= SMs, at least
  // kMinSplitBlocks blocks each: with fewer, merging the k partial tiles of
  // d fp32 columns through distributed shared memory costs more than the
  // blocks it takes off each CTA -- measured on SD's 16x16 calls).
  int k = 1;
  if (2 * p.units <= nsm) k = std::min(std::min(8, p.nkb / kMinSplitBlocks), nsm / p.units);
  if (k < 2) k = 1;
  p.ksplit = k;
  if (k > 1)
    return launch_cluster(kern, p.units * k, k, C::NTHREADS, C::SMEM, stream, ma, mv, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
  const int grid = p.units < nsm ? p.units : nsm;
  return launch(kern, grid, C::NTHREADS, C::SMEM, stream, ma, mv, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
}

template <int D, int NQ, int BN, bool BF16, int NPOLY = 3, bool PREC = false>
sdattn_status launch_flash(const sdattn_desc* d, const void* Q, const void* K, const void* V, void* O, float* LS,
                           void* ws, cudaStream_t stream) {
  using C = FlashCfg<D, NQ, BN, PREC>;
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  auto kern = sdattn::flash_kernel<D, NQ, BN, BF16, NPOLY, PREC>;
  static std::atomic<uint64_t> smem_done{0};
  if (!ensure_smem(kern, C::SMEM, smem_done, dev)) return SDATTN_ERR_CUDA;

  const int nsm = sm_count(dev);
  const uint64_t bh = static_cast<uint64_t>(d->B) * d->H;
  const uint64_t N = d->N, M = d->M;
  CUtensorMap mq, mk, mv, mvt;
  if (!make_map_3d(&mq, Q, elem_type(d), D, N, bh, D * 2, N * D * 2, 64, 128)) return SDATTN_ERR_CUDA;
  if (!make_map_3d(&mk, K, elem_type(d), D, M, bh, D * 2, M * D * 2, 64, BN)) return SDATTN_ERR_CUDA;
  if (!make_map_3d(&mv, V, elem_type(d), D, M, bh, D * 2, M * D * 2, 64, BN)) return SDATTN_ERR_CUDA;
  // V's last column slab is loaded only up to column D, keeping the padding
  // (where the kernel keeps its ones column) untouched
  if (!make_map_3d(&mvt, V, elem_type(d), D, M, bh, D * 2, M * D * 2, C::TAIL, BN)) return SDATTN_ERR_CUDA;

  FlashParams p;
  p.N = d->N;
  p.M = d->M;
  p.BH = static_cast<int>(bh);
  p.tph = (d->N + 128 * NQ - 1) / (128 * NQ);
  p.nkv = (d->M + BN - 1) / BN;
  p.units = p.BH * p.tph;
  p.scale = d->scale;
  p.c = d->scale * 1.4426950408889634f;
  p.O = O;
  p.LS = LS;
  // Test hook for the bounded-wait path: with SDATTN_TEST_INJECT_STALL=1 in
  // the environment, one wait in the kernel can never complete, runs out after
  // about a second, and the call's results are left unwritten.
  const char* stall = std::getenv("SDATTN_TEST_INJECT_STALL");
  p.inject_stall = (stall != nullptr && stall[0] == '1') ? 1 : 0;
  // Whole units leave the last wave of CTAs part-empty when units is just
  // above a multiple of the SM count; then (given a workspace) every CTA
  // takes an equal share of the (unit, key tile) pairs instead, cutting at
  // most one unit at each end of its range.
  const int64_t waves = (p.units + nsm - 1) / nsm;
  const double eff = static_cast<double>(p.units) / static_cast<double>(waves * nsm);
  p.split = (ws != nullptr && p.units > nsm && p.nkv >= 2 && eff < 0.9) ? 1 : 0;
  p.tickets = static_cast<uint32_t*>(ws);
  p.part = ws ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + flash_ws_tickets_bytes(d, nsm)) : nullptr;
  // Units filling under half the SMs over long key ranges (one query tile
  // per CTA): a cluster of k CTAs shares each unit's key tiles (k <= 8,
  // k * units <= SMs, at least kMinSplitBlocks tiles each, as for softmax_av),
  // merged through distributed shared memory.
  p.ksplit = 1;
  if (NQ == 1 && !PREC && 2 * p.units <= nsm) p.ksplit = std::min(std::min(8, p.nkv / kMinSplitBlocks), nsm / p.units);
  if (p.ksplit < 2) p.ksplit = 1;
  if (p.ksplit > 1)
    return launch_cluster(kern, p.units * p.ksplit, p.ksplit, C::NTHREADS, C::SMEM, stream, mq, mk, mv, mvt, p)
               ? SDATTN_OK
               : SDATTN_ERR_CUDA;
  const int grid = p.units < nsm ? p.units : nsm;
  return launch(kern, grid, C::NTHREADS, C::SMEM, stream, mq, mk, mv, mvt, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
}

sdattn_status launch_row_stats(const sdattn_desc* d, const float* A, float* LS, void* ws, size_t ws_size,
                               cudaStream_t stream) {
  const int dev = current_device();
  const RowPlan pl = plan_rows(d, sm_count(dev < 0 ? 0 : dev));
  RowStatsParams p;
  p.A = A;
  p.lda = a_ld(d);
  p.rows = pl.rows;
  p.M = d->M;
  p.nsplit = pl.nsplit;
  p.split_cols = pl.split_cols;
  p.LS = LS;
  p.tickets = nullptr;
  p.part = nullptr;
  if (pl.nsplit > 1) {
    if (!ws || ws_size < rows_ws_tickets_bytes(pl) + static_cast<size_t>(pl.rows) * pl.nsplit * sizeof(float2))
      return SDATTN_ERR_WORKSPACE;
    p.tickets = static_cast<uint32_t*>(ws);
    p.part = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + rows_ws_tickets_bytes(pl));
  }
  if (dev < 0) return SDATTN_ERR_CUDA;
  return launch(sdattn::row_stats_kernel<float>, pl.grid, sdattn::kRowStatsWarps * 32, 0, stream, p)
             ? SDATTN_OK
             : SDATTN_ERR_CUDA;
}

template <int AMODE>
sdattn_status dispatch_qk(const sdattn_desc* d, const void* Q, const void* K, void* A, float* LS, void* ws,
                          cudaStream_t s) {
  const bool bf = d->dtype == SDATTN_BF16;
  switch (d->d) {
    case 40: return bf ? launch_qk<40, true, AMODE>(d, Q, K, A, LS, ws, s) : launch_qk<40, false, AMODE>(d, Q, K, A, LS, ws, s);
    case 80: return bf ? launch_qk<80, true, AMODE>(d, Q, K, A, LS, ws, s) : launch_qk<80, false, AMODE>(d, Q, K, A, LS, ws, s);
    case 160:
      return bf ? launch_qk<160, true, AMODE>(d, Q, K, A, LS, ws, s) : launch_qk<160, false, AMODE>(d, Q, K, A, LS, ws, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

template <bool AF16>
sdattn_status dispatch_av(const sdattn_desc* d, const void* A, const float* LS, const void* V, void* O,
                          cudaStream_t s) {
  const bool bf = d->dtype == SDATTN_BF16;
  switch (d->d) {
    case 40: return bf ? launch_av<40, true, AF16>(d, A, LS, V, O, s) : launch_av<40, false, AF16>(d, A, LS, V, O, s);
    case 80: return bf ? launch_av<80, true, AF16>(d, A, LS, V, O, s) : launch_av<80, false, AF16>(d, A, LS, V, O, s);
    case 160: return bf ? launch_av<160, true, AF16>(d, A, LS, V, O, s) : launch_av<160, false, AF16>(d, A, LS, V, O, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

// Work split of a qk_stats call with statistics: the scratch that its column
// split needs (none for a single split, or for splits merged in a cluster).
size_t qk_split_need(const sdattn_desc* d, const QKPlan& pl, int nsm) {
  if (pl.nsplit == 1 || qk_cluster_merge(pl, nsm)) return 0;
  const int64_t tiles = static_cast<int64_t>(d->B) * d->H * pl.nrt;
  return ws_tickets_bytes(d) + static_cast<size_t>(tiles) * 128 * pl.nsplit * sizeof(float2);
}

// ---- GroupNorm and gated GELU ----
// A group is spread over a cluster of up to kGNMaxCluster CTAs, each holding
// at most kGNThreads x 8 chunks of 8 values.
constexpr int64_t kGNMaxChunks = int64_t(sdattn::kGNThreads) * 8 * sdattn::kGNMaxCluster;

sdattn_status check_gn(const sdattn_gn_desc* d) {
  if (!d) return SDATTN_ERR_INVALID_ARG;
  if (d->B < 1 || d->C < 1 || d->H < 1 || d->W < 1 || d->G < 1 || d->C % d->G != 0) return SDATTN_ERR_INVALID_ARG;
  if (!std::isfinite(d->eps) || d->eps < 0.f) return SDATTN_ERR_INVALID_ARG;
  if (d->dtype != SDATTN_F16 && d->dtype != SDATTN_BF16) return SDATTN_ERR_UNSUPPORTED;
  const int64_t hw = static_cast<int64_t>(d->H) * d->W;
  const int64_t gsize = hw * (d->C / d->G);
  if (hw % 8 != 0 || gsize / 8 > kGNMaxChunks) return SDATTN_ERR_UNSUPPORTED;   // also keeps H*W, gsize in int
  if (static_cast<int64_t>(d->B) * d->C * hw >= (int64_t(1) << 40)) return SDATTN_ERR_UNSUPPORTED;
  return SDATTN_OK;
}

template <int U, bool BF16>
sdattn_status launch_gn_u(const sdattn::GNParams& p, int64_t groups, int cluster, int threads, cudaStream_t s) {
  return launch_cluster(sdattn::group_norm_kernel<U, BF16>, static_cast<int>(groups * cluster), cluster, threads, 0, s, p)
             ? SDATTN_OK
             : SDATTN_ERR_CUDA;
}

template <bool BF16>
sdattn_status launch_gn(const sdattn_gn_desc* d, const void* X, const float* gamma, const float* beta, void* Y,
                        cudaStream_t s) {
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  const int nsm = sm_count(dev);
  sdattn::GNParams p;
  p.X = X;
  p.Y = Y;
  p.gamma = gamma;
  p.beta = beta;
  p.G = d->G;
  p.cpg = d->C / d->G;
  p.HW = d->H * d->W;
  p.gsize = p.HW * p.cpg;
  p.eps = d->eps;
  const int64_t nch = p.gsize / 8;
  const int64_t groups = static_cast<int64_t>(d->B) * d->G;
  // Clusters: as few CTAs per group as hold it in registers, more while the
  // grid would leave SMs idle and each CTA keeps at least a warp of chunks.
  const int64_t cap = int64_t(sdattn::kGNThreads) * 8;
  int k = 1;
  while (k < sdattn::kGNMaxCluster &&
         ((nch + k - 1) / k > cap || (groups * k < nsm && (nch + 2 * k - 1) / (2 * k) >= 32)))
    k *= 2;
  p.cpc = static_cast<int>((nch + k - 1) / k);
  int u = 1;
  while (p.cpc > sdattn::kGNThreads * u) u *= 2;
  const int64_t per = (p.cpc + u - 1) / u;
  const int threads = static_cast<int>(std::min<int64_t>(sdattn::kGNThreads, std::max<int64_t>(32, (per + 31) / 32 * 32)));
  switch (u) {
    case 1: return launch_gn_u<1, BF16>(p, groups, k, threads, s);
    case 2: return launch_gn_u<2, BF16>(p, groups, k, threads, s);
    case 4: return launch_gn_u<4, BF16>(p, groups, k, threads, s);
    case 8: return launch_gn_u<8, BF16>(p, groups, k, threads, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

template <bool BF16>
sdattn_status launch_geglu(int64_t T, int F, const void* X, void* Y, cudaStream_t s) {
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  sdattn::GegluParams p;
  p.X = X;
  p.Y = Y;
  p.T = T;
  p.F = F;
  const int64_t n = T * (F / 8);
  const int64_t want = (n + 2 * 256 - 1) / (2 * 256);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(sm_count(dev)) * 8)));
  return launch(sdattn::geglu_kernel<BF16>, grid, 256, 0, s, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
}

// --------------------------------------------------------------------------
// Winograd F(4x4, 3x3) convolution (winograd.cuh)
// --------------------------------------------------------------------------
sdattn_status check_conv(const sdattn_conv_desc* d) {
  if (!d) return SDATTN_ERR_INVALID_ARG;
  if (d->N < 1 || d->C < 1 || d->K < 1 || d->H < 1 || d->W < 1) return SDATTN_ERR_INVALID_ARG;
  if (d->dtype != SDATTN_F16 && d->dtype != SDATTN_BF16) return SDATTN_ERR_UNSUPPORTED;
  // C % 8: the transformed rows are whole 16-byte units, as TMA needs;
  // W <= 4096: one row of input tiles for one channel fits shared memory
  if (d->C % 8 != 0 || d->W > 4096) return SDATTN_ERR_UNSUPPORTED;
  const int64_t T = int64_t(d->N) * ((d->H + 3) / 4) * ((d->W + 3) / 4);
  const int64_t ldm = (T + 3) / 4 * 4;
  // every index of the 36 planes stays inside 2^31 elements per plane
  if (T * d->C >= (int64_t(1) << 31) || int64_t(d->K) * ldm >= (int64_t(1) << 31) ||
      int64_t(d->K) * d->C >= (int64_t(1) << 31) || int64_t(d->N) * d->C * d->H * d->W >= (int64_t(1) << 40))
    return SDATTN_ERR_UNSUPPORTED;
  return SDATTN_OK;
}

sdattn::WinoGeom wino_geom(const sdattn_conv_desc* d, int nsm) {
  sdattn::WinoGeom g;
  g.N = d->N;
  g.C = d->C;
  g.K = d->K;
  g.H = d->H;
  g.W = d->W;
  g.TH = (d->H + 3) / 4;
  g.TW = (d->W + 3) / 4;
  g.T = g.N * g.TH * g.TW;
  g.ldm = (g.T + 3) / 4 * 4;
  // channels per input-transform CTA: the six rows of each fit in 96 KB, and
  // blocks of at least 16 channels are split further while the grid would
  // give the SMs fewer than four CTAs each (the kernel is latency-bound)
  const int64_t per_c = int64_t(sdattn::WinoRows::of(g.TW).PS) * 4 / 2;   // bytes per channel
  g.CB = 64;
  while (g.CB > 2 && g.CB * per_c > 96 * 1024) g.CB /= 2;   // an even number: channel pairs
  while (g.CB > 16 && int64_t(g.N) * g.TH * ((g.C + g.CB - 1) / g.CB) < 4 * int64_t(nsm)) g.CB /= 2;
  return g;
}

size_t wino_v_bytes(const sdattn::WinoGeom& g) {
  return (size_t(36) * g.T * g.C * 2 + 255) / 256 * 256;
}

size_t wino_ws_bytes(const sdattn::WinoGeom& g) { return wino_v_bytes(g) + size_t(36) * g.K * g.ldm * 4; }

template <bool BF16>
sdattn_status launch_wino(const sdattn_conv_desc* d, const void* X, const void* U, const float* bias, void* Y,
                          void* ws, cudaStream_t s) {
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  const int nsm = sm_count(dev);
  const sdattn::WinoGeom g = wino_geom(d, nsm);
  uint16_t* V = static_cast<uint16_t*>(ws);
  float* M = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + wino_v_bytes(g));
  // input transform
  {
    auto kern = sdattn::wino_input_kernel<BF16>;
    const int smem = (g.CB / 2) * sdattn::WinoRows::of(g.TW).PS * 4;
    static std::atomic<uint64_t> smem_done{0};
    if (!ensure_smem(kern, 96 * 1024, smem_done, dev)) return SDATTN_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(g.N * g.TH), static_cast<unsigned>((g.C + g.CB - 1) / g.CB));
    // one thread per (channel pair, tile) of the CTA's block, 32 to 256
    const int items = (g.CB / 2) * g.TW;
    cfg.blockDim = dim3(static_cast<unsigned>(std::min(256, std::max(32, (items + 31) / 32 * 32))));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, static_cast<const uint16_t*>(X), V, g) != cudaSuccess) return SDATTN_ERR_CUDA;
  }
  // the 36 products
  {
    using C = sdattn::WinoGemmCfg;
    auto kern = sdattn::wino_gemm_kernel<BF16>;
    static std::atomic<uint64_t> smem_done{0};
    if (!ensure_smem(kern, C::SMEM, smem_done, dev)) return SDATTN_ERR_CUDA;
    CUtensorMap mu, mv;
    const CUtensorMapDataType dt = BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!make_map_3d(&mu, U, dt, g.C, g.K, 36, uint64_t(g.C) * 2, uint64_t(g.K) * g.C * 2, 64, 128))
      return SDATTN_ERR_CUDA;
    if (!make_map_3d(&mv, V, dt, g.C, g.T, 36, uint64_t(g.C) * 2, uint64_t(g.T) * g.C * 2, 64, 128))
      return SDATTN_ERR_CUDA;
    CUtensorMap mm;
    if (!make_map_3d(&mm, M, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.ldm, g.K, 36, uint64_t(g.ldm) * 4,
                     uint64_t(g.K) * g.ldm * 4, 32, 32))
      return SDATTN_ERR_CUDA;
    sdattn::WinoGemmParams p;
    p.M = M;
    p.K = g.K;
    p.T = g.T;
    p.ldm = g.ldm;
    p.kbs = (g.K + 127) / 128;
    p.tbs = (g.T + 127) / 128;
    p.units = 36 * p.kbs * p.tbs;
    p.ksteps = (g.C + C::BK - 1) / C::BK;
    const int grid = p.units < nsm ? p.units : nsm;
    if (!launch(kern, grid, C::NTHREADS, C::SMEM, s, mu, mv, mm, p)) return SDATTN_ERR_CUDA;
  }
  // output transform
  {
    const int64_t n = int64_t(g.K) * g.T;
    const int grid = static_cast<int>((n + 255) / 256);
    if (!launch(sdattn::wino_output_kernel<BF16>, grid, 256, 0, s, static_cast<const float*>(M), bias,
                static_cast<uint16_t*>(Y), g))
      return SDATTN_ERR_CUDA;
  }
  return SDATTN_OK;
}

template <bool BF16>
sdattn_status launch_wino_filter(const sdattn_conv_desc* d, const void* w, void* U, cudaStream_t s) {
  const int64_t n = int64_t(d->K) * d->C;
  const int grid = static_cast<int>((n + 255) / 256);
  return launch(sdattn::wino_filter_kernel<BF16>, grid, 256, 0, s, static_cast<const uint16_t*>(w),
                static_cast<uint16_t*>(U), d->K, d->C)
             ? SDATTN_OK
             : SDATTN_ERR_CUDA;
}

// fp32 inputs through tf32 products (flash_tf32.cuh): one query tile per CTA.
template <int D>
sdattn_status launch_flash_tf32(const sdattn_desc* d, const void* Q, const void* K, const void* V, float* O,
                                float* LS, cudaStream_t stream) {
  using C = sdattn::FlashTF32Cfg<D>;
  const int dev = current_device();
  if (dev < 0) return SDATTN_ERR_CUDA;
  auto kern = sdattn::flash_tf32_kernel<D>;
  static std::atomic<uint64_t> smem_done{0};
  if (!ensure_smem(kern, C::SMEM, smem_done, dev)) return SDATTN_ERR_CUDA;
  const int nsm = sm_count(dev);
  const uint64_t bh = static_cast<uint64_t>(d->B) * d->H;
  const uint64_t N = d->N, M = d->M;
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  CUtensorMap mq, mk, mv;
  if (!make_map_3d(&mq, Q, f32, D, N, bh, D * 4, N * D * 4, 32, 128)) return SDATTN_ERR_CUDA;
  if (!make_map_3d(&mk, K, f32, D, M, bh, D * 4, M * D * 4, 32, C::BN)) return SDATTN_ERR_CUDA;
  if (!make_map_3d(&mv, V, f32, D, M, bh, D * 4, M * D * 4, 32, C::BN)) return SDATTN_ERR_CUDA;
  sdattn::FlashTF32Params p;
  p.N = d->N;
  p.M = d->M;
  p.BH = static_cast<int>(bh);
  p.tph = (d->N + 127) / 128;
  p.nkv = (d->M + C::BN - 1) / C::BN;
  p.units = p.BH * p.tph;
  p.scale = d->scale;
  p.c = d->scale * 1.4426950408889634f;
  p.O = O;
  p.LS = LS;
  const int grid = p.units < nsm ? p.units : nsm;
  return launch(kern, grid, C::NTHREADS, C::SMEM, stream, mq, mk, mv, p) ? SDATTN_OK : SDATTN_ERR_CUDA;
}

// The precise variant: every block of rows whole; at d = 40 with enough work,
// two query tiles per CTA over 96-key tiles (tensor memory holds S, P, P's
// residual and O of both), else one query tile over 128-key tiles.
template <bool BF16>
sdattn_status dispatch_flash_f32o(const sdattn_desc* d, const void* Q, const void* K, const void* V, float* O,
                                  float* LS, cudaStream_t s) {
  const int dev = current_device();
  const int nsm = sm_count(dev < 0 ? 0 : dev);
  const int64_t pairs = static_cast<int64_t>(d->B) * d->H * ((d->N + 255) / 256);
  switch (d->d) {
    case 40:
      if (pairs >= nsm) return launch_flash<40, 2, 96, BF16, 3, true>(d, Q, K, V, O, LS, nullptr, s);
      return launch_flash<40, 1, 128, BF16, 3, true>(d, Q, K, V, O, LS, nullptr, s);
    case 80: return launch_flash<80, 1, 128, BF16, 3, true>(d, Q, K, V, O, LS, nullptr, s);
    case 160: return launch_flash<160, 1, 64, BF16, 3, true>(d, Q, K, V, O, LS, nullptr, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

template <bool BF16>
sdattn_status dispatch_flash(const sdattn_desc* d, const void* Q, const void* K, const void* V, void* O, float* LS,
                             void* ws, cudaStream_t s) {
  const int dev = current_device();
  const int nsm = sm_count(dev < 0 ? 0 : dev);
  const int64_t pairs = static_cast<int64_t>(d->B) * d->H * ((d->N + 255) / 256);
  const bool two = pairs >= nsm;   // enough work for two query tiles per CTA
  switch (d->d) {
    case 40:
      // keys that fit one 96-key tile (cross-attention, 77 text tokens): a
      // narrower score tile, so the exponentials, row max and products cover
      // 96 columns instead of 128
      if (d->M <= 96)
        return two ? launch_flash<40, 2, 96, BF16>(d, Q, K, V, O, LS, ws, s)
                   : launch_flash<40, 1, 96, BF16>(d, Q, K, V, O, LS, ws, s);
      return two ? launch_flash<40, 2, 128, BF16>(d, Q, K, V, O, LS, ws, s)
                 : launch_flash<40, 1, 128, BF16>(d, Q, K, V, O, LS, ws, s);
    case 80:
      return launch_flash<80, 1, 128, BF16>(d, Q, K, V, O, LS, ws, s);
    case 160:
      return launch_flash<160, 1, 64, BF16>(d, Q, K, V, O, LS, ws, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

}  // namespace

// ============================================================================
// Allocation-free variant of sdattn_qk_stats (no counterpart in the paper).
//
// Some callers cannot allocate device memory for a workspace: code that runs
// inside a framework whose allocator it may not touch, plug-ins handed only
// input and output buffers, or processes whose memory budget is fixed up front.
// For them the split-reduction scratch of qk_stats lives in this file-scope
// device array instead.  Every GPU that loads this library keeps the array
// (kNoAllocScratchBytes) for the life of the process.
// ============================================================================
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(2) << 20;   // 2 MiB
}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Process-unique id of the calling thread's current context (0 if none or
// unknown).  A device reset ends the primary context; the next one has a new id.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_cur = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// In host code `g_noalloc_scratch` only names the symbol; the device address
// of the array is looked up with the device current, once per device and
// context: after a device reset the array lives in a new context, at an
// address that is looked up anew.
bool noalloc_scratch(int dev, void** out) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return false;
    addr[dev] = p;
    ctx_of[dev] = current_context_id();   // the lookup above made the primary context current
  }
  *out = addr[dev];
  return true;
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

int64_t sdattn_a_ld(const sdattn_desc* desc) {
  if (check_desc(desc) != SDATTN_OK) return -1;
  return a_ld(desc);
}

size_t sdattn_workspace_bytes(const sdattn_desc* desc) {
  if (check_desc(desc) != SDATTN_OK) return 0;
  return ws_bytes(desc);
}

sdattn_status sdattn_qk_stats(const sdattn_desc* desc, const void* Q, const void* K, float* A, float* LS, void* ws,
                              size_t ws_size, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !A || !LS) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(A) || !aligned16(LS)) return SDATTN_ERR_ALIGNMENT;
  if (!ws || ws_size < qk_ws_bytes(desc)) return SDATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return SDATTN_ERR_ALIGNMENT;
  return dispatch_qk<sdattn::kAF32Stats>(desc, Q, K, A, LS, ws, static_cast<cudaStream_t>(stream));
}

sdattn_status sdattn_softmax_av(const sdattn_desc* desc, const float* A, const float* LS, const void* V, void* O,
                                void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!A || !LS || !V || !O) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(LS) || !aligned16(V) || !aligned16(O)) return SDATTN_ERR_ALIGNMENT;
  return dispatch_av<false>(desc, A, LS, V, O, static_cast<cudaStream_t>(stream));
}

sdattn_status sdattn_qk_scores(const sdattn_desc* desc, const void* Q, const void* K, float* A, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !A) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(A)) return SDATTN_ERR_ALIGNMENT;
  return dispatch_qk<sdattn::kAF32Only>(desc, Q, K, A, nullptr, nullptr, static_cast<cudaStream_t>(stream));
}

sdattn_status sdattn_row_stats(const sdattn_desc* desc, const float* A, float* LS, void* ws, size_t ws_size,
                               void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!A || !LS) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(LS)) return SDATTN_ERR_ALIGNMENT;
  if (ws && !aligned16(ws)) return SDATTN_ERR_ALIGNMENT;
  if (!ws && ws_size != 0) return SDATTN_ERR_WORKSPACE;
  return launch_row_stats(desc, A, LS, ws, ws_size, static_cast<cudaStream_t>(stream));
}

int64_t sdattn_a16_ld(const sdattn_desc* desc) {
  if (check_desc(desc) != SDATTN_OK) return -1;
  return a16_ld(desc);
}

sdattn_status sdattn_qk_stats_f16a(const sdattn_desc* desc, const void* Q, const void* K, void* A16, float* LS,
                                   void* ws, size_t ws_size, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !A16 || !LS) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(A16) || !aligned16(LS)) return SDATTN_ERR_ALIGNMENT;
  if (!ws || ws_size < qk_ws_bytes(desc)) return SDATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return SDATTN_ERR_ALIGNMENT;
  return dispatch_qk<sdattn::kAF16Stats>(desc, Q, K, A16, LS, ws, static_cast<cudaStream_t>(stream));
}

sdattn_status sdattn_softmax_av_f16a(const sdattn_desc* desc, const void* A16, const float* LS, const void* V,
                                     void* O, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!A16 || !LS || !V || !O) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(A16) || !aligned16(LS) || !aligned16(V) || !aligned16(O)) return SDATTN_ERR_ALIGNMENT;
  return dispatch_av<true>(desc, A16, LS, V, O, static_cast<cudaStream_t>(stream));
}

sdattn_status sdattn_flash(const sdattn_desc* desc, const void* Q, const void* K, const void* V, void* O,
                           float* LS_or_null, void* ws, size_t ws_size, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !V || !O) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SDATTN_ERR_ALIGNMENT;
  if (LS_or_null && !aligned16(LS_or_null)) return SDATTN_ERR_ALIGNMENT;
  if (ws && !aligned16(ws)) return SDATTN_ERR_ALIGNMENT;
  if (!ws && ws_size != 0) return SDATTN_ERR_WORKSPACE;
  if (ws) {
    const int dev = current_device();
    if (ws_size < flash_ws_bytes(desc, sm_count(dev < 0 ? 0 : dev))) return SDATTN_ERR_WORKSPACE;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return desc->dtype == SDATTN_BF16 ? dispatch_flash<true>(desc, Q, K, V, O, LS_or_null, ws, s)
                                    : dispatch_flash<false>(desc, Q, K, V, O, LS_or_null, ws, s);
}

sdattn_status sdattn_flash_f32o(const sdattn_desc* desc, const void* Q, const void* K, const void* V, float* O,
                                float* LS_or_null, void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !V || !O) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SDATTN_ERR_ALIGNMENT;
  if (LS_or_null && !aligned16(LS_or_null)) return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return desc->dtype == SDATTN_BF16 ? dispatch_flash_f32o<true>(desc, Q, K, V, O, LS_or_null, s)
                                    : dispatch_flash_f32o<false>(desc, Q, K, V, O, LS_or_null, s);
}

sdattn_status sdattn_flash_tf32(const sdattn_desc* desc, const void* Q, const void* K, const void* V, float* O,
                                float* LS_or_null, void* stream) {
  if (!desc) return SDATTN_ERR_INVALID_ARG;
  if (desc->dtype != SDATTN_F32) return SDATTN_ERR_UNSUPPORTED;
  sdattn_desc d16 = *desc;   // every other rule is the 16-bit entry points'
  d16.dtype = SDATTN_F16;
  const sdattn_status st = check_desc(&d16);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !V || !O) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return SDATTN_ERR_ALIGNMENT;
  if (LS_or_null && !aligned16(LS_or_null)) return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (desc->d) {
    case 40: return launch_flash_tf32<40>(desc, Q, K, V, O, LS_or_null, s);
    case 80: return launch_flash_tf32<80>(desc, Q, K, V, O, LS_or_null, s);
    case 160: return launch_flash_tf32<160>(desc, Q, K, V, O, LS_or_null, s);
  }
  return SDATTN_ERR_UNSUPPORTED;
}

sdattn_status sdattn_device_error(uint32_t* detail) {
  if (detail) *detail = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return SDATTN_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, sdattn::g_error_word, sizeof(v)) != cudaSuccess) return SDATTN_ERR_CUDA;
  const uint32_t zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(sdattn::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SDATTN_ERR_CUDA;
  if (detail) *detail = v;
  return v ? SDATTN_ERR_TIMEOUT : SDATTN_OK;
}

sdattn_status sdattn_qk_stats_noalloc(const sdattn_desc* desc, const void* Q, const void* K, float* A, float* LS,
                                      void* stream) {
  const sdattn_status st = check_desc(desc);
  if (st != SDATTN_OK) return st;
  if (!Q || !K || !A || !LS) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(A) || !aligned16(LS)) return SDATTN_ERR_ALIGNMENT;
  // Same work split as sdattn_qk_stats; a single split uses no scratch at all.
  const int dev = current_device();
  const int nsm = sm_count(dev < 0 ? 0 : dev);
  const QKPlan pl = plan_qk(desc, nsm);
  const size_t need = qk_split_need(desc, pl, nsm);
  if (need > kNoAllocScratchBytes) return SDATTN_ERR_WORKSPACE;
  if (dev < 0) return SDATTN_ERR_CUDA;
  void* ws = nullptr;
  if (!noalloc_scratch(dev, &ws)) return SDATTN_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The arrival counters must start at zero; the partials are overwritten.
  if (need > 0 && cudaMemsetAsync(ws, 0, ws_tickets_bytes(desc), s) != cudaSuccess) return SDATTN_ERR_CUDA;
  return dispatch_qk<sdattn::kAF32Stats>(desc, Q, K, A, LS, ws, s);
}

sdattn_status sdattn_group_norm(const sdattn_gn_desc* desc, const void* X, const float* gamma, const float* beta,
                                void* Y, void* stream) {
  const sdattn_status st = check_gn(desc);
  if (st != SDATTN_OK) return st;
  if (!X || !gamma || !beta || !Y) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y) || (reinterpret_cast<uintptr_t>(gamma) & 3u) ||
      (reinterpret_cast<uintptr_t>(beta) & 3u))
    return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return desc->dtype == SDATTN_BF16 ? launch_gn<true>(desc, X, gamma, beta, Y, s)
                                    : launch_gn<false>(desc, X, gamma, beta, Y, s);
}

sdattn_status sdattn_geglu(int64_t T, int32_t F, int32_t dtype, const void* X, void* Y, void* stream) {
  if (T < 1 || F < 8) return SDATTN_ERR_INVALID_ARG;
  if (F % 8 != 0) return SDATTN_ERR_UNSUPPORTED;
  if (dtype != SDATTN_F16 && dtype != SDATTN_BF16) return SDATTN_ERR_UNSUPPORTED;
  if (T > (int64_t(1) << 40) / F) return SDATTN_ERR_UNSUPPORTED;
  if (!X || !Y) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Y)) return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dtype == SDATTN_BF16 ? launch_geglu<true>(T, F, X, Y, s) : launch_geglu<false>(T, F, X, Y, s);
}

size_t sdattn_wino_filter_bytes(const sdattn_conv_desc* desc) {
  if (check_conv(desc) != SDATTN_OK) return 0;
  return size_t(36) * desc->K * desc->C * 2;
}

size_t sdattn_wino_workspace_bytes(const sdattn_conv_desc* desc) {
  if (check_conv(desc) != SDATTN_OK) return 0;
  // the workspace does not depend on the channel blocking
  return wino_ws_bytes(wino_geom(desc, 148));
}

sdattn_status sdattn_wino_filter(const sdattn_conv_desc* desc, const void* w, void* U, void* stream) {
  const sdattn_status st = check_conv(desc);
  if (st != SDATTN_OK) return st;
  if (!w || !U) return SDATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(w) & 1u) || !aligned16(U)) return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return desc->dtype == SDATTN_BF16 ? launch_wino_filter<true>(desc, w, U, s) : launch_wino_filter<false>(desc, w, U, s);
}

sdattn_status sdattn_wino_conv3x3(const sdattn_conv_desc* desc, const void* X, const void* U, const float* bias,
                                  void* Y, void* ws, size_t ws_bytes, void* stream) {
  const sdattn_status st = check_conv(desc);
  if (st != SDATTN_OK) return st;
  if (!X || !U || !Y) return SDATTN_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(U) || !aligned16(Y) || (bias && (reinterpret_cast<uintptr_t>(bias) & 3u)))
    return SDATTN_ERR_ALIGNMENT;
  const sdattn::WinoGeom g = wino_geom(desc, 148);
  if (!ws || ws_bytes < wino_ws_bytes(g)) return SDATTN_ERR_WORKSPACE;
  if (!aligned16(ws)) return SDATTN_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return desc->dtype == SDATTN_BF16 ? launch_wino<true>(desc, X, U, bias, Y, ws, s)
                                    : launch_wino<false>(desc, X, U, bias, Y, ws, s);
}

const char* sdattn_status_string(sdattn_status status) {
  switch (status) {
    case SDATTN_OK: return "ok";
    case SDATTN_ERR_INVALID_ARG: return "invalid argument";
    case SDATTN_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case SDATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SDATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case SDATTN_ERR_CUDA: return "CUDA runtime or driver error";
    case SDATTN_ERR_TIMEOUT: return "kernel wait timed out";
  }
  return "unknown status";
}

int32_t sdattn_version(void) { return 100; }

}  // extern "C"
