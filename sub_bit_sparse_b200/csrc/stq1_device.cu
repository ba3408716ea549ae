// C-ABI entry points of libstq1.so (device side).  Argument checks happen on the
// host before anything is enqueued; every entry point returns an STQ1_* code.
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <utility>

#include <cudaTypedefs.h>
#include <nvtx3/nvToolsExt.h>

#include "device_common.cuh"
#include "encode_device.cuh"
#include "gemv_lut.cuh"
#include "gemv_mma.cuh"
#include "mix_score.cuh"
#include "small_kernels.cuh"
#include "tc_gemm.cuh"

namespace stq1 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kTargetUnits = 444;   // aim for ~3 work units per SM on a 148-SM part
// Two-token units do twice the lookups per chunk and do better with longer K
// pieces (fewer splits): measured on [4096, 7168] and [18432, 7168] at batch 2,
// a quarter of the units is 13-15% faster; one and four tokens keep the full count.
constexpr int kTargetUnitsTwoTokens = kTargetUnits / 4;
constexpr int kMaxExperts = 4096;
// Split-K counters live at a fixed offset (0) of the GEMV workspace so that their
// zero-between-calls invariant does not depend on the shape of earlier calls.
// Split K is used only when tiles x slabs < kTargetUnits, so this bounds them.
constexpr size_t kCounterBytes = 2048;
static_assert(kTargetUnits * sizeof(int) <= kCounterBytes, "counter region too small");

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// An NVTX range around each entry point, so that a profiler's timeline shows
// which library call enqueued which kernels (nearly free without a profiler).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Path selection: 0 = by size, 1 = table kernel, 2 = tensor-core tile kernel,
// 3 = tensor-core decode kernel (mma.sync, few tokens).
// Atomic so that a call on another host thread reads either value, never a torn one.
std::atomic<int> g_path{0};
constexpr int kTcMinBatch = 16;       // stq1_gemv: batches from here use the tile kernel
constexpr int kTcMinPairsPerExpert = 16;
constexpr int kMoeTableTokens = 2;    // MoE decode tiles: pairs per table-kernel unit

// Per-device attribute caches.  Several host threads may make their first
// call at once: a cache slot is an atomic written with the same value by
// whichever thread gets there, so a reader sees 0 (and asks the runtime) or
// the final value.
int device_attr_cached(std::atomic<int>* cache, cudaDeviceAttr attr, int fallback) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fallback;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, attr, dev) != cudaSuccess || v <= 0) v = fallback;
    cache[dev].store(v, std::memory_order_relaxed);
  }
  return v;
}

std::atomic<int> g_sm_count[kMaxDevices];
int sm_count() { return device_attr_cached(g_sm_count, cudaDevAttrMultiProcessorCount, 148); }

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link); a function-local static is initialised once, thread-safely.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

// 2-D map over a row-major activation matrix [rows, K] of bf16 (or, fp8, of
// E4M3 bytes); box = 128 bytes of columns x kTcN rows, 128-byte swizzle,
// out-of-range rows read as zero.
// x tiles of the tile kernel as one 3-D copy per stage: dimension 0 = the
// 128 bytes of one swizzle atom, 1 = rows (row stride K elements), 2 = atoms
// along K (stride 128 bytes); a box is 128 rows x the stage's atoms, which
// land atom after atom, 16 KB apart, as the MMA descriptors expect.
bool make_b_map(CUtensorMap* map, const void* base, long long rows, long long K, bool fp8, int box_rows = kTcN) {
  auto fn = encode_fn();
  if (!fn) return false;
  const int esize = fp8 ? 1 : 2;
  const long long atom = kTcAtomBytes / esize;
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(atom), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(K / atom)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(K) * esize, static_cast<cuuint64_t>(kTcAtomBytes)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(atom), static_cast<cuuint32_t>(box_rows),
                       static_cast<cuuint32_t>(fp8 ? TcGeom<true>::atoms : TcGeom<false>::atoms)};
  cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
            const_cast<void*>(base), gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

// Per-device one-time kernel attribute setup (dynamic shared memory limits).
// The first call on a device holds a lock while it sets the attributes, so a
// call on another host thread never launches before they are in place.
std::atomic<bool> g_configured[kMaxDevices];
std::mutex g_config_mutex;
int ensure_configured() {
  const int dev = current_device();
  if (dev < 0) return STQ1_ERR_CUDA;
  if (g_configured[dev].load(std::memory_order_acquire)) return STQ1_OK;
  std::lock_guard<std::mutex> lock(g_config_mutex);
  if (g_configured[dev].load(std::memory_order_relaxed)) return STQ1_OK;
  if (cudaFuncSetAttribute(lut_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lut_smem_bytes_max(1))) != cudaSuccess ||
      cudaFuncSetAttribute(lut_gemv_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lut_smem_bytes_max(2))) != cudaSuccess ||
      cudaFuncSetAttribute(lut_gemv_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lut_smem_bytes_max(4))) != cudaSuccess ||
      cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           3 * kMaxExperts * 4) != cudaSuccess ||
      cudaFuncSetAttribute(tc_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kTcSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(tc_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kTcSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(encode_smem_bytes_max())) != cudaSuccess ||
      cudaFuncSetAttribute(stq2_encode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(encode_smem_bytes_max())) != cudaSuccess ||
      cudaFuncSetAttribute(hess_score_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kHsSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(hess_score_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kHsSmemBytes) != cudaSuccess ||
      cudaFuncSetAttribute(mma_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(mma_smem_bytes_max())) != cudaSuccess)
    return STQ1_ERR_CUDA;
  // split-K clusters of up to 16 CTAs (above the portable 8); a refusal only
  // disables the cluster path
  cudaFuncSetAttribute(lut_gemv_kernel<1>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(lut_gemv_kernel<2>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(lut_gemv_kernel<4>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(mma_gemv_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaGetLastError();
  g_configured[dev].store(true, std::memory_order_release);
  return STQ1_OK;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? STQ1_OK : STQ1_ERR_CUDA;
}

// Launch with programmatic stream serialization: the kernel may start while the
// previous kernel in the stream drains; it calls griddepcontrol.wait before
// touching anything that kernel may write.  cluster_y > 1 groups CTAs along y.
template <typename... Params, typename... Args>
int launch_pdl_cluster(void (*kernel)(Params...), dim3 grid, unsigned block, size_t smem, cudaStream_t s,
                       unsigned cluster_y, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster_y > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = cluster_y;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess) return STQ1_OK;
  cudaGetLastError();   // clear a refused launch so the caller can fall back
  return STQ1_ERR_CUDA;
}

template <typename... Params, typename... Args>
int launch_pdl(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem, cudaStream_t s,
               Args&&... args) {
  return launch_pdl_cluster(kernel, dim3(grid), block, smem, s, 1u, std::forward<Args>(args)...);
}

int residue_period(long long rowbytes) {
  // rows per residue class of (row * rowbytes) mod 16, for rowbytes % 4 == 0
  const long long g = (rowbytes % 16 == 0) ? 16 : ((rowbytes % 8 == 0) ? 8 : 4);
  return static_cast<int>(16 / g);
}

// Tensor maps over a packed buffer of rows_total rows (table and tile
// kernels): the main map views it as super-rows of P = 2^logP rows (stride
// P * rowbytes, a multiple of 16) and copies boxes of 112 bytes x box_h
// super-rows; the tail map (1-D) covers the last rows_total mod P rows.
// extra_srow: slabs may start inside a super-row (MoE experts with N % P !=
// 0), so boxes take one more.
struct PackedMaps {
  CUtensorMap w, t;
};

int make_packed_maps(PackedMaps* m, PackedGeom* g, const uint8_t* W, long long rows_total, long long rowbytes,
                     bool extra_srow) {
  auto fn = encode_fn();
  if (!fn) return STQ1_ERR_CUDA;
  const int P = residue_period(rowbytes);
  const int logP = P == 1 ? 0 : (P == 2 ? 1 : 2);
  const long long srow_bytes = P * rowbytes;
  const long long main_srows = rows_total >> logP;
  if (main_srows >= (1LL << 31) || srow_bytes + kWindowBytes >= (1LL << 31)) return STQ1_ERR_SHAPE;
  g->rowbytes = rowbytes;
  g->rows_total = rows_total;
  g->tail_row0 = main_srows << logP;
  g->main_srows = static_cast<int>(main_srows);
  g->logP = logP;
  g->box_h = (kSlabRows >> logP) + (extra_srow ? 1 : 0);
  g->buf_bytes = packed_buf_bytes(g->box_h);
  g->stage_bytes = packed_stage_bytes(logP, g->box_h);
  cuuint32_t es[2] = {1, 1};
  {
    // a map that is never read (no full super-row) still has to be valid
    const bool any = main_srows > 0;
    cuuint64_t gdim[2] = {static_cast<cuuint64_t>(any ? srow_bytes : 16),
                          static_cast<cuuint64_t>(any ? main_srows : 1)};
    cuuint64_t gstride[1] = {static_cast<cuuint64_t>(any ? srow_bytes : 16)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(any ? kWindowBytes : 16),
                         static_cast<cuuint32_t>(any ? g->box_h : 1)};
    if (fn(&m->w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(W), gdim, gstride, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return STQ1_ERR_CUDA;
  }
  {
    const long long nt = rows_total - g->tail_row0;
    const uint8_t* base = nt > 0 ? W + g->tail_row0 * rowbytes : W;
    cuuint64_t gdim[1] = {static_cast<cuuint64_t>(nt > 0 ? nt * rowbytes : 16)};
    cuuint64_t gstride[1] = {0};
    cuuint32_t box[1] = {static_cast<cuuint32_t>(nt > 0 ? kWindowBytes : 16)};
    if (fn(&m->t, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, const_cast<uint8_t*>(base), gdim, gstride, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return STQ1_ERR_CUDA;
  }
  return STQ1_OK;
}

// Encoded maps are a pure function of (device, buffer address, rows, row bytes,
// extra super-row): a direct-mapped cache saves re-encoding them on every call
// (a call on the same matrix is the common case).  An entry stays correct even
// if the buffer is freed and the address reused with the same shape, since a
// map only describes an address and a shape.
struct MapCacheEntry {
  const void* base;
  long long rows, rowbytes;
  int dev;
  bool extra, valid;
  PackedMaps maps;
  PackedGeom g;
};
constexpr int kMapCacheSize = 1024;
MapCacheEntry g_map_cache[kMapCacheSize];
std::mutex g_map_mutex;

int packed_maps_cached(PackedMaps* m, PackedGeom* g, const uint8_t* W, long long rows_total, long long rowbytes,
                       bool extra_srow) {
  const int dev = current_device();
  const uint64_t h = (reinterpret_cast<uintptr_t>(W) >> 4) * 0x9E3779B97F4A7C15ull ^
                     static_cast<uint64_t>(rows_total) * 0xC2B2AE3D27D4EB4Full ^ static_cast<uint64_t>(rowbytes) ^
                     (static_cast<uint64_t>(dev) << 1) ^ (extra_srow ? 1u : 0u);
  MapCacheEntry& e = g_map_cache[(h >> 32) % kMapCacheSize];
  {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    if (e.valid && e.base == W && e.rows == rows_total && e.rowbytes == rowbytes && e.dev == dev &&
        e.extra == extra_srow) {
      *m = e.maps;
      *g = e.g;
      return STQ1_OK;
    }
  }
  const int rc = make_packed_maps(m, g, W, rows_total, rowbytes, extra_srow);
  if (rc == STQ1_OK) {
    std::lock_guard<std::mutex> lock(g_map_mutex);
    e.base = W;
    e.rows = rows_total;
    e.rowbytes = rowbytes;
    e.dev = dev;
    e.extra = extra_srow;
    e.maps = *m;
    e.g = *g;
    e.valid = true;
  }
  return rc;
}

// K split of n_chunks chunks into S pieces (split s: cq chunks, one more if s < cr).
void set_split(LutArgs* a, int n_chunks, int S) {
  a->S = S;
  a->cq = n_chunks / S;
  a->cr = n_chunks % S;
}

// Shared-memory stages: two when some split holds at least two chunks.
int lut_stages(const LutArgs& a) { return a.cq + (a.cr > 0 ? 1 : 0) >= 2 ? 2 : 1; }

struct GemvPlan {
  int n_tiles, n_slabs, S, n_chunks, tt;
  size_t partial_bytes, counter_bytes;
  bool table_path, tile_path, mma_path;
};

bool want_tiles(long long nb, long long units) {
  if (nb % 2 != 0) return false;          // the tile kernel needs 4-byte-aligned rows
  if (g_path == 1 || g_path == 3) return false;
  if (g_path == 2) return true;
  return units >= kTcMinBatch;
}

// Plain GEMV from kTcMinBatch tokens on: the tile kernel when it is expected to
// be faster.  Calibrated on [4096, 7168] and [18432, 7168] (CUDA graphs of
// distinct matrices): the table kernel costs about 5.7e-8 us per token and
// weight (its shared-memory lookups grow with the tokens); a tile-kernel wave
// of (128-token, 128-row) items costs about 1.36 us per 256-column block of K.
bool want_tiles_gemv(long long N, long long nb, long long batch) {
  if (!want_tiles(nb, batch)) return false;
  if (g_path == 2) return true;
  const double table_us = 5.7e-8 * static_cast<double>(batch) * static_cast<double>(N) * nb * kBlockWeights;
  const long long items = ((batch + kTcN - 1) / kTcN) * ((N + kTcM - 1) / kTcM);
  const long long waves = (items + sm_count() - 1) / sm_count();
  const double tiles_us = 1.36 * static_cast<double>(waves) * nb;
  return tiles_us < table_us;
}

std::atomic<int> g_smem_per_sm[kMaxDevices];
int smem_per_sm() {
  return device_attr_cached(g_smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, 228 * 1024);
}

// Work split of the table kernel: (token tile, 128-row slab) units, each cut
// into S pieces of K so that there are about kTargetUnits CTAs (a quarter of
// that for two-token units) and, with one_wave, no more than fit on the device
// at once.
void plan_table(GemvPlan* p, long long N, long long K, int batch, bool one_wave) {
  const long long nb = K / kBlockWeights;
  p->tt = batch == 1 ? 1 : (batch == 2 ? 2 : 4);
  p->n_tiles = (batch + kLutMaxTT - 1) / kLutMaxTT;
  p->n_slabs = static_cast<int>((N + kLutRows - 1) / kLutRows);
  p->n_chunks = static_cast<int>(nb / kLutKC);
  const long long units0 = static_cast<long long>(p->n_tiles) * p->n_slabs;
  const long long target = p->tt == 2 ? kTargetUnitsTwoTokens : kTargetUnits;
  long long S = (target + units0 - 1) / units0;
  S = std::max<long long>(1, std::min<long long>(S, std::max(1, p->n_chunks)));
  const int P = residue_period(nb * kBlockBytes);
  const int logP = P == 1 ? 0 : (P == 2 ? 1 : 2);
  const int stage = packed_stage_bytes(logP, kLutRows >> logP);
  const long long slots_sm = smem_per_sm();
  // the split-K partials meet inside one thread-block cluster (at most 16 CTAs)
  if (one_wave) S = std::min<long long>(S, kMaxClusterRanks);
  for (; one_wave && S > 1; --S) {
    const int cq = static_cast<int>(p->n_chunks / S), cr = static_cast<int>(p->n_chunks % S);
    const int stages = cq + (cr > 0 ? 1 : 0) >= 2 ? 2 : 1;
    const long long smem = static_cast<long long>(lut_smem_bytes(p->tt, stages, stage, static_cast<int>(S))) + 1024;
    const long long per_sm = std::min<long long>(lut_min_blocks(p->tt), slots_sm / smem);
    if (units0 * S <= per_sm * sm_count()) break;
  }
  // the fewest splits that keep the longest split as short: n_chunks = 14 and
  // at most 13 splits gives 7 splits of 2 chunks, not 13 with one of 2
  const long long longest = (p->n_chunks + S - 1) / S;
  if (longest > 0) S = (p->n_chunks + longest - 1) / longest;
  p->S = static_cast<int>(std::max<long long>(1, S));
}

// Tensor-core decode kernel for few tokens: 3 .. 15 tokens by default, any
// batch when forced.  Its cost per weight does not depend on the token count;
// the table kernel's grows with it.  Measured (CUDA graphs of distinct
// matrices): on [4096, 7168] 7.7-7.8 us at 1-8 tokens against the table
// kernel's 4.9 / 7.0 / 8.4 / 10.4 / 16.2 us at 1 / 2 / 3 / 4 / 8; on
// [18432, 7168] 21.5-21.8 us against 14.7 / 18.4 / 21.7 / 26.8 / 48.5 us.
// Rows need an even number of blocks (chunks of two).
constexpr int kMmaMinBatch = 3;
bool want_mma(long long nb, int batch) {
  if (nb % 2 != 0) return false;
  const int path = g_path;
  if (path == 3) return true;
  if (path != 0) return false;
  return batch >= kMmaMinBatch;
}

// Work split of the tensor-core decode kernel: (8-token tile, 128-row slab)
// units, each cut into S pieces of K (whole steps of four blocks) so that
// there are about two CTAs per SM, then reduced to the fewest pieces with
// the same longest piece.
void plan_mma(GemvPlan* p, long long N, long long K, int batch) {
  const long long nb = K / kBlockWeights;
  p->n_tiles = (batch + kMmaTokens - 1) / kMmaTokens;
  p->n_slabs = static_cast<int>((N + kMmaRows - 1) / kMmaRows);
  p->n_chunks = static_cast<int>(nb / 2);
  const long long steps = (p->n_chunks + 1) / 2;
  const long long units0 = static_cast<long long>(p->n_tiles) * p->n_slabs;
  const long long slots = 2LL * sm_count();          // two CTAs per SM
  // The K split with the least (waves x steps per piece): a second, partial
  // wave costs a whole piece, so for [18432, 7168] two pieces of 4 steps in
  // one wave beat three of 3 steps in two; ties go to fewer pieces (less to
  // reduce).  Split K only while the arrival counters of the units fit their
  // region (the workspace fallback needs them) and a cluster holds the pieces.
  long long S = 1;
  if (units0 * static_cast<long long>(sizeof(int)) <= static_cast<long long>(kCounterBytes)) {
    long long best = -1;
    for (long long c = 1; c <= std::min<long long>(steps, kMaxClusterRanks); ++c) {
      const long long cost = ((units0 * c + slots - 1) / slots) * ((steps + c - 1) / c);
      if (best < 0 || cost < best) {
        best = cost;
        S = c;
      }
    }
  }
  const long long longest = (steps + S - 1) / S;
  if (longest > 0) S = (steps + longest - 1) / longest;
  p->S = static_cast<int>(S);
}

GemvPlan plan_gemv(long long N, long long K, int batch) {
  GemvPlan p{};
  const long long nb = K / kBlockWeights;
  p.tile_path = want_tiles_gemv(N, nb, batch);
  if (p.tile_path) return p;
  if (want_mma(nb, batch)) {
    p.mma_path = true;
    plan_mma(&p, N, K, batch);
  } else {
    p.table_path = (nb % 2 == 0);
    plan_table(&p, N, K, batch, true);
    if (!p.table_path) p.S = 1;
  }
  if ((p.table_path || p.mma_path) && p.S > 1) {
    p.partial_bytes = static_cast<size_t>(p.S) * batch * N * sizeof(float);
    p.counter_bytes = kCounterBytes;
  }
  return p;
}

size_t round16(size_t b) { return (b + 15) & ~static_cast<size_t>(15); }

}  // namespace
}  // namespace stq1

using namespace stq1;

extern "C" int stq1_dequant(const void* W_packed, uint16_t* W_bf16, int64_t N, int64_t K,
                            void* stream) {
  NvtxRange nvtx_range("stq1_dequant");
  if (!W_packed || !W_bf16) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || K % kBlockWeights) return STQ1_ERR_SHAPE;
  if (!aligned16(W_packed) || !aligned16(W_bf16)) return STQ1_ERR_ALIGN;
  const long long n_groups = N * (K / 4);
  const int threads = 256;
  const long long blocks = std::min<long long>((n_groups + threads - 1) / threads, 148LL * 64);
  dequant_kernel<<<static_cast<unsigned>(blocks), threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(W_packed), W_bf16, n_groups);
  return launch_status();
}

extern "C" size_t stq1_gemv_workspace(int64_t N, int64_t K, int batch) {
  if (N <= 0 || K <= 0 || K % kBlockWeights || batch <= 0) return 0;
  const GemvPlan p = plan_gemv(N, K, batch);
  return p.counter_bytes + round16(p.partial_bytes);
}

namespace {
int gemv_impl(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K, int batch,
              void* workspace, size_t ws_bytes, const void* W_next, int64_t next_bytes, void* stream) {
  if (!W_packed || !x || !y) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || K % kBlockWeights || batch <= 0 || batch > 65535 ||
      N > (1LL << 31) - 1 || K > (1LL << 31) - 1)
    return STQ1_ERR_SHAPE;
  if (!aligned16(W_packed) || !aligned16(x)) return STQ1_ERR_ALIGN;
  const GemvPlan p = plan_gemv(N, K, batch);
  const size_t need = p.counter_bytes + round16(p.partial_bytes);
  if (need > 0 && (!workspace || ws_bytes < need)) return STQ1_ERR_WORKSPACE;
  if (need > 0 && !aligned16(workspace)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long nb = K / kBlockWeights;
  const long long rowbytes = nb * kBlockBytes;
  if (p.tile_path) {
    CUtensorMap map;
    CUtensorMap map_h;                               // half-height boxes for tiles of <= 64 tokens
    if (!make_b_map(&map, x, batch, K, false) || !make_b_map(&map_h, x, batch, K, false, kTcHalfN))
      return STQ1_ERR_CUDA;
    TcArgs t{};
    PackedMaps pm;
    rc = packed_maps_cached(&pm, &t.g, static_cast<const uint8_t*>(W_packed), N, rowbytes, false);
    if (rc != STQ1_OK) return rc;
    t.y = y;
    t.tile_info = nullptr;
    t.n_tiles_dev = nullptr;
    t.pairs = nullptr;
    t.route_w = nullptr;
    t.xscale = nullptr;
    t.n_tiles = (batch + kTcN - 1) / kTcN;
    t.N = static_cast<int>(N);
    t.K = static_cast<int>(K);
    t.nb = static_cast<int>(nb);
    t.n_mtiles = static_cast<int>((N + kTcM - 1) / kTcM);
    t.batch = batch;
    t.flags = 0;
    t.b_rows = batch;
    t.rows_out = batch;
    const long long items = static_cast<long long>(t.n_tiles) * t.n_mtiles;
    const int grid = static_cast<int>(std::min<long long>(items, sm_count()));
    return launch_pdl(tc_gemm_kernel<false>, grid, kTcThreads, kTcSmemBytes, s, map, map_h, pm.w, pm.t, t);
  }
  if (p.mma_path) {
    MmaArgs m{};
    PackedMaps maps;
    rc = packed_maps_cached(&maps, &m.g, static_cast<const uint8_t*>(W_packed), N, rowbytes, false);
    if (rc != STQ1_OK) return rc;
    m.x = x;
    m.y = y;
    m.counters = p.S > 1 ? static_cast<int*>(workspace) : nullptr;
    m.partial = p.S > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes) : nullptr;
    m.N = static_cast<int>(N);
    m.K = static_cast<int>(K);
    m.topk = 1;
    m.batch = batch;
    m.rows_out = batch;
    m.x_rows = batch;
    m.n_slabs = p.n_slabs;
    m.n_chunks = p.n_chunks;
    const int steps = (p.n_chunks + 1) / 2;
    m.S = p.S;
    m.sq = steps / p.S;
    m.sr = steps % p.S;
    m.flags = 0;
    const long long units = static_cast<long long>(p.n_tiles) * p.n_slabs;
    if (units >= (1LL << 31)) return STQ1_ERR_SHAPE;
    const dim3 grid(static_cast<unsigned>(units), static_cast<unsigned>(p.S));
    // split K reduces inside a cluster of the S pieces of a unit (distributed
    // shared memory); if the device refuses such a cluster, through the
    // caller's workspace
    if (p.S > 1 && p.S <= kMaxClusterRanks) {
      m.cluster = 1;
      if (launch_pdl_cluster(mma_gemv_kernel, grid, kMmaThreads, mma_smem_bytes(m.g.stage_bytes, true), s,
                             static_cast<unsigned>(p.S), maps.w, maps.t, m) == STQ1_OK)
        return STQ1_OK;
      m.cluster = 0;
    }
    return launch_pdl_cluster(mma_gemv_kernel, grid, kMmaThreads, mma_smem_bytes(m.g.stage_bytes), s, 1u, maps.w,
                              maps.t, m);
  }
  if (!p.table_path) {
    const long long warps = static_cast<long long>(batch) * N;
    direct_gemv_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(W_packed), 0, 1, x, nullptr, 1, nullptr, 0, y,
        static_cast<int>(N), static_cast<int>(K), batch);
    return launch_status();
  }
  LutArgs a{};
  PackedMaps maps;
  rc = packed_maps_cached(&maps, &a.g, static_cast<const uint8_t*>(W_packed), N, rowbytes, false);
  if (rc != STQ1_OK) return rc;
  a.x = x;
  a.y = y;
  a.counters = p.S > 1 ? static_cast<int*>(workspace) : nullptr;
  a.partial = p.S > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes) : nullptr;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.topk = 1;
  a.batch = batch;
  a.rows_out = batch;
  a.x_rows = batch;
  a.n_slabs = p.n_slabs;
  set_split(&a, p.n_chunks, p.S);
  a.flags = 0;
  a.next = static_cast<const uint8_t*>(W_next);
  a.next_bytes = W_next ? (next_bytes & ~static_cast<int64_t>(15)) : 0;
  if (a.next_bytes <= 0) a.next = nullptr;
  const long long units = static_cast<long long>(p.n_tiles) * p.n_slabs;
  if (units >= (1LL << 31)) return STQ1_ERR_SHAPE;
  const dim3 grid(static_cast<unsigned>(units), static_cast<unsigned>(p.S));
  auto go = [&](int cluster) {
    a.cluster = cluster > 1 ? 1 : 0;
    const size_t smem = lut_smem_bytes(p.tt, lut_stages(a), a.g.stage_bytes, cluster);
    if (p.tt == 1)
      return launch_pdl_cluster(lut_gemv_kernel<1>, grid, kLutThreads, smem, s, cluster, maps.w, maps.t, a);
    if (p.tt == 2)
      return launch_pdl_cluster(lut_gemv_kernel<2>, grid, kLutThreads, smem, s, cluster, maps.w, maps.t, a);
    return launch_pdl_cluster(lut_gemv_kernel<4>, grid, kLutThreads, smem, s, cluster, maps.w, maps.t, a);
  };
  // split K reduces through distributed shared memory inside a cluster of the
  // S units of a slab; if the device refuses such a cluster, through the
  // caller's scratch buffer
  if (p.S > 1 && p.S <= kMaxClusterRanks && go(p.S) == STQ1_OK) return STQ1_OK;
  return go(1);
}
}  // namespace

extern "C" int stq1_gemv(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K,
                         int batch, void* workspace, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("stq1_gemv");
  return gemv_impl(W_packed, x, y, N, K, batch, workspace, ws_bytes, nullptr, 0, stream);
}

extern "C" int stq1_gemv_prefetch(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K,
                                  int batch, void* workspace, size_t ws_bytes, const void* W_next,
                                  int64_t next_bytes, void* stream) {
  NvtxRange nvtx_range("stq1_gemv_prefetch");
  if (next_bytes < 0) return STQ1_ERR_SHAPE;
  if (W_next && !aligned16(W_next)) return STQ1_ERR_ALIGN;
  return gemv_impl(W_packed, x, y, N, K, batch, workspace, ws_bytes, W_next, next_bytes, stream);
}

namespace stq1 {
namespace {
struct MoePlan {
  size_t pairs_off, tiles_off, small_off, ntiles_off, xperm_off, xq_off, sq_off, sperm_off, total;
  int max_tiles, tile_tokens, small_max, max_small;
  bool tiles, fp8, mma;
};
// Decode with the tensor-core kernel: experts with at most this many routed
// pairs go to the lookup-table kernel instead, whose cost per weight is lower
// for one or two tokens (one table load per token and group against a fixed
// decode of about a dozen instructions per group on the tensor-core path).
constexpr int kMoeSmallMax = 2;
MoePlan plan_moe(int T, int topk, int E, long long K, int flags) {
  MoePlan m{};
  const long long n_pairs = static_cast<long long>(T) * topk;
  const long long nb = K / kBlockWeights;
  const long long active = std::min<long long>(E, n_pairs);
  m.tiles = want_tiles(nb, n_pairs >= kTcMinPairsPerExpert * active ? kTcMinBatch : 0);
  m.mma = !m.tiles && nb % 2 == 0 && g_path != 1;
  m.tile_tokens = m.tiles ? kTcN : (m.mma ? kMmaTokens : kMoeTableTokens);
  // Tiles of an expert with c pairs: ceil(c / tile_tokens) <= c / tile_tokens + 1,
  // so at most n_pairs / tile_tokens plus the number of experts with tiles;
  // on the tensor-core decode path only experts with more than kMoeSmallMax
  // pairs have main tiles, at most n_pairs / (kMoeSmallMax + 1) of them.  The
  // grid is sized by this bound (the real count is on the device), and every
  // CTA past the real count exits at once.
  const long long tiled = m.mma ? std::min<long long>(active, n_pairs / (kMoeSmallMax + 1)) : active;
  m.max_tiles = static_cast<int>(std::min<long long>(n_pairs, n_pairs / m.tile_tokens + tiled));
  m.small_max = m.mma ? kMoeSmallMax : 0;
  m.max_small = m.mma ? static_cast<int>(active) : 0;
  size_t off = 0;
  m.pairs_off = off;
  off += round16(n_pairs * sizeof(int));
  m.tiles_off = off;
  off += round16(static_cast<size_t>(m.max_tiles) * 4 * sizeof(int));
  m.small_off = off;
  off += round16(static_cast<size_t>(m.max_small) * 4 * sizeof(int));
  m.ntiles_off = off;
  off += 16;
  m.fp8 = m.tiles && (flags & STQ1_MOE_FP8);
  m.xperm_off = off;
  if (m.tiles) off += round16(static_cast<size_t>(n_pairs) * K * (m.fp8 ? 1 : 2));
  m.xq_off = m.sq_off = m.sperm_off = off;
  if (m.fp8) {
    m.xq_off = off;
    off += round16(static_cast<size_t>(T) * K);
    m.sq_off = off;
    off += round16(static_cast<size_t>(T) * sizeof(float));
    m.sperm_off = off;
    off += round16(static_cast<size_t>(n_pairs) * sizeof(float));
  }
  m.total = off;
  return m;
}
}  // namespace
}  // namespace stq1

extern "C" size_t stq1_moe_workspace(int T, int topk, int E, int64_t N, int64_t K, int flags) {
  (void)N;
  if (T <= 0 || topk <= 0 || E <= 0 || K <= 0 || K % kBlockWeights) return 0;
  return plan_moe(T, topk, E, K, flags).total;
}

namespace stq1 {
namespace {

// Routing tables one MoE call computes once (route_kernel) and its matmuls read.
struct MoeTables {
  int* pairs;         // pair ids grouped by expert
  int* tiles;         // main tile table
  int* tiles_small;   // tiles of experts with few pairs (tensor-core decode path)
  int* ntiles;        // [0] main tiles, [1] pairs with a valid id, [2] small tiles
};

// Device scratch of one matmul over routed pairs on the tile path.
struct MoeScratch {
  void* xperm;        // activation rows in pair order (bf16, or E4M3 bytes)
  uint8_t* xq;        // E4M3 codes of the activation rows (fp8)
  float* sq;          // their per-row scales (fp8)
  float* sperm;       // scales in pair order (fp8)
};

// A second stream per device and host thread, with a fork and a join event,
// for MoE decode calls that split experts between the table and tensor-core
// kernels: the two launches are independent (disjoint output rows, both read
// only the routing tables and x), so they run side by side and fill each
// other's idle issue slots and wave tails.  Created on first use, kept for
// the thread's lifetime.  Under stream capture the fork and join become graph
// edges.  If they cannot be created the two kernels run one after the other.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  bool failed = false;
};
SideStream* side_stream() {
  thread_local SideStream side[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return nullptr;
  SideStream& ss = side[dev];
  if (ss.stream == nullptr && !ss.failed) {
    if (cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      ss.failed = true;
    }
  }
  return ss.failed ? nullptr : &ss;
}

// The matmul over routed pairs, on tables the route kernel already fills.
// `compact` bit 0: pair i of the grouped list writes output row i (else row
// pairs[i]); bit 1: its activation row is row i of x (else pairs[i] / topk).
// x_rows = rows of x (tokens, or the compact rows).  Routing weights are
// always indexed by pair id.
int moe_compute(const MoePlan& m, const MoeTables& tb, const MoeScratch& sc, const void* expert_blocks,
                const uint16_t* x, int x_rows, const float* topk_weights, float* y, int topk, int n_pairs, int E,
                long long N, long long K, int flags, int compact, cudaStream_t s) {
  const long long nb = K / kBlockWeights;
  const long long rowbytes = nb * kBlockBytes;
  int rc;
  if (m.tiles) {
    const void* B = x;
    float* xscale = nullptr;
    if (m.fp8) {
      rc = launch_pdl(quant_e4m3_kernel, static_cast<unsigned>(x_rows), kQuantThreads, 0, s, x, static_cast<int>(K),
                      sc.xq, sc.sq);
      if (rc != STQ1_OK) return rc;
      if (compact & 2) {
        B = sc.xq;                                   // compact rows are already in pair order
        xscale = sc.sq;
      } else {
        rc = launch_pdl(gather_rows8_kernel, static_cast<unsigned>(n_pairs), 256, 0, s,
                        static_cast<const uint8_t*>(sc.xq), static_cast<const float*>(sc.sq),
                        static_cast<const int*>(tb.pairs), static_cast<const int*>(tb.ntiles + 1), n_pairs, topk,
                        static_cast<int>(K), static_cast<uint8_t*>(sc.xperm), sc.sperm);
        if (rc != STQ1_OK) return rc;
        B = sc.xperm;
        xscale = sc.sperm;
      }
    } else if (!(compact & 2)) {
      rc = launch_pdl(gather_rows_kernel, static_cast<unsigned>(n_pairs), 256, 0, s, x,
                      static_cast<const int*>(tb.pairs), static_cast<const int*>(tb.ntiles + 1), n_pairs, topk,
                      static_cast<int>(K), static_cast<uint16_t*>(sc.xperm));
      if (rc != STQ1_OK) return rc;
      B = sc.xperm;
    }
    CUtensorMap map;
    CUtensorMap map_h;                               // half-height boxes for tiles of <= 64 pairs
    if (!make_b_map(&map, B, n_pairs, K, m.fp8) || !make_b_map(&map_h, B, n_pairs, K, m.fp8, kTcHalfN))
      return STQ1_ERR_CUDA;
    TcArgs t{};
    PackedMaps pm;
    rc = packed_maps_cached(&pm, &t.g, static_cast<const uint8_t*>(expert_blocks), static_cast<long long>(E) * N,
                            rowbytes, N % residue_period(rowbytes) != 0);
    if (rc != STQ1_OK) return rc;
    t.y = y;
    t.tile_info = tb.tiles;
    t.n_tiles_dev = tb.ntiles;
    t.pairs = (compact & 1) ? nullptr : tb.pairs;
    t.wpairs = tb.pairs;
    t.route_w = topk_weights;
    t.xscale = xscale;
    t.n_tiles = m.max_tiles;
    t.N = static_cast<int>(N);
    t.K = static_cast<int>(K);
    t.nb = static_cast<int>(nb);
    t.n_mtiles = static_cast<int>((N + kTcM - 1) / kTcM);
    t.batch = 0;
    t.flags = flags;
    t.b_rows = (compact & 2) ? x_rows : n_pairs;
    t.rows_out = n_pairs;
    const long long items = static_cast<long long>(m.max_tiles) * t.n_mtiles;
    const int grid = static_cast<int>(std::min<long long>(items, sm_count()));
    if (m.fp8)
      return launch_pdl(tc_gemm_kernel<true>, grid, kTcThreads, kTcSmemBytes, s, map, map_h, pm.w, pm.t, t);
    return launch_pdl(tc_gemm_kernel<false>, grid, kTcThreads, kTcSmemBytes, s, map, map_h, pm.w, pm.t, t);
  }
  PackedMaps maps;
  PackedGeom geom;
  rc = packed_maps_cached(&maps, &geom, static_cast<const uint8_t*>(expert_blocks), static_cast<long long>(E) * N,
                          rowbytes, N % residue_period(rowbytes) != 0);
  if (rc != STQ1_OK) return rc;
  // lookup-table kernel: every tile (table path) or the experts with few pairs
  LutArgs l{};
  l.g = geom;
  l.x = x;
  l.y = y;
  l.tile_info = m.mma ? tb.tiles_small : tb.tiles;
  l.n_tiles_dev = m.mma ? tb.ntiles + 2 : tb.ntiles;
  l.pairs = tb.pairs;
  l.route_w = topk_weights;
  l.N = static_cast<int>(N);
  l.K = static_cast<int>(K);
  l.topk = topk;
  l.rows_out = n_pairs;
  l.n_slabs = static_cast<int>((N + kLutRows - 1) / kLutRows);
  set_split(&l, static_cast<int>(nb / kLutKC), 1);
  l.flags = flags;
  l.cluster = 0;
  l.compact = compact;
  l.tiles_cap = m.mma ? m.max_small : m.max_tiles;
  l.x_rows = x_rows;
  const long long lunits = static_cast<long long>(m.mma ? m.max_small : m.max_tiles) * l.n_slabs;
  if (lunits >= (1LL << 31)) return STQ1_ERR_SHAPE;
  auto launch_lut = [&](cudaStream_t st) {
    return launch_pdl_cluster(lut_gemv_kernel<kMoeTableTokens>, dim3(static_cast<unsigned>(lunits)), kLutThreads,
                              lut_smem_bytes(kMoeTableTokens, lut_stages(l), l.g.stage_bytes, 1), st, 1u, maps.w,
                              maps.t, l);
  };
  if (!m.mma) return launch_lut(s);
  // tensor-core decode kernel: the other experts, in tiles of up to 8 pairs
  MmaArgs a{};
  a.g = geom;
  a.x = x;
  a.y = y;
  a.tile_info = tb.tiles;
  a.n_tiles_dev = tb.ntiles;
  a.pairs = tb.pairs;
  a.route_w = topk_weights;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.topk = topk;
  a.rows_out = n_pairs;
  a.n_slabs = static_cast<int>((N + kMmaRows - 1) / kMmaRows);
  a.n_chunks = static_cast<int>(nb / 2);
  a.S = 1;
  a.sq = (a.n_chunks + 1) / 2;
  a.sr = 0;
  a.flags = flags;
  a.compact = compact;
  a.tiles_cap = m.max_tiles;
  a.x_rows = x_rows;
  const long long units = static_cast<long long>(m.max_tiles) * a.n_slabs;
  if (units >= (1LL << 31)) return STQ1_ERR_SHAPE;
  auto launch_mma = [&](cudaStream_t st) {
    return launch_pdl_cluster(mma_gemv_kernel, dim3(static_cast<unsigned>(units)), kMmaThreads,
                              mma_smem_bytes(a.g.stage_bytes), st, 1u, maps.w, maps.t, a);
  };
  if (m.max_small == 0) return launch_mma(s);
  // both kernels: fork the tensor-core part onto the side stream, join after
  SideStream* side = side_stream();
  if (side == nullptr) {
    rc = launch_lut(s);
    return rc != STQ1_OK ? rc : launch_mma(s);
  }
  if (cudaEventRecord(side->fork, s) != cudaSuccess || cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess)
    return STQ1_ERR_CUDA;
  rc = launch_mma(side->stream);
  if (rc != STQ1_OK) return rc;
  if (cudaEventRecord(side->join, side->stream) != cudaSuccess) return STQ1_ERR_CUDA;
  rc = launch_lut(s);
  if (rc != STQ1_OK) return rc;
  return cudaStreamWaitEvent(s, side->join, 0) == cudaSuccess ? STQ1_OK : STQ1_ERR_CUDA;
}

}  // namespace
}  // namespace stq1

extern "C" int stq1_moe_gateup(const void* expert_blocks, const uint16_t* x, const int32_t* topk_ids,
                               const float* topk_weights, float* y, int T, int topk, int E, int64_t N,
                               int64_t K, int flags, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("stq1_moe_gateup");
  if (!expert_blocks || !x || !topk_ids || !y) return STQ1_ERR_NULL;
  if ((flags & STQ1_MOE_WEIGHT_UP) && !topk_weights) return STQ1_ERR_NULL;
  if (flags & ~(STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8 | STQ1_MOE_SKIP_FOREIGN)) return STQ1_ERR_ARG;
  // with STQ1_MOE_SKIP_FOREIGN a rank may hold fewer experts than a token picks
  const bool foreign = (flags & STQ1_MOE_SKIP_FOREIGN) != 0;
  if (T <= 0 || topk <= 0 || E <= 0 || (!foreign && topk > E) || E > kMaxExperts || N <= 0 || (N & 1) || K <= 0 ||
      K % kBlockWeights || N > (1LL << 30) || K > (1LL << 30) ||
      static_cast<long long>(T) * topk > (1LL << 30))
    return STQ1_ERR_SHAPE;
  if (!aligned16(expert_blocks) || !aligned16(x)) return STQ1_ERR_ALIGN;
  const MoePlan m = plan_moe(T, topk, E, K, flags);
  if (!ws || ws_bytes < m.total) return STQ1_ERR_WORKSPACE;
  if (!aligned16(ws)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long nb = K / kBlockWeights;
  const long long rowbytes = nb * kBlockBytes;
  const int n_pairs = T * topk;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  MoeTables tb;
  tb.pairs = reinterpret_cast<int*>(wsb + m.pairs_off);
  tb.tiles = reinterpret_cast<int*>(wsb + m.tiles_off);
  tb.tiles_small = reinterpret_cast<int*>(wsb + m.small_off);
  tb.ntiles = reinterpret_cast<int*>(wsb + m.ntiles_off);
  MoeScratch sc;
  sc.xperm = wsb + m.xperm_off;
  sc.xq = wsb + m.xq_off;
  sc.sq = reinterpret_cast<float*>(wsb + m.sq_off);
  sc.sperm = reinterpret_cast<float*>(wsb + m.sperm_off);

  if (nb % 2 != 0) {
    const long long warps = static_cast<long long>(n_pairs) * N;
    direct_gemv_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(expert_blocks), N * rowbytes, E, x, topk_ids, topk, topk_weights,
        flags, y, static_cast<int>(N), static_cast<int>(K), n_pairs);
    return launch_status();
  }

  rc = launch_pdl(route_kernel, 1, kRouteThreads, 3 * E * sizeof(int), s, topk_ids, n_pairs, E, m.tile_tokens,
                  m.small_max, tb.pairs, tb.tiles, tb.tiles_small, tb.ntiles, static_cast<int*>(nullptr), y,
                  static_cast<int>(N), (flags & STQ1_MOE_SKIP_FOREIGN) ? 1 : 0, m.max_tiles, m.max_small);
  if (rc != STQ1_OK) return rc;
  return moe_compute(m, tb, sc, expert_blocks, x, T, topk_weights, y, topk, n_pairs, E, N, K, flags, 0, s);
}

extern "C" int stq1_quantize(const float* W, const float* h, int64_t N, int64_t K, int mode, int rounds,
                             uint8_t* out, void* stream) {
  NvtxRange nvtx_range("stq1_quantize");
  if (!W || !out) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || K % kBlockWeights) return STQ1_ERR_SHAPE;
  if (mode != STQ1_ENC_PLAIN && mode != STQ1_ENC_SHERRY) return STQ1_ERR_ARG;
  if (mode == STQ1_ENC_SHERRY && (rounds < 0 || rounds > 1000)) return STQ1_ERR_ARG;
  if (N > (1LL << 40) / K) return STQ1_ERR_SHAPE;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(out) & 1)) return STQ1_ERR_ALIGN;
  if (mode == STQ1_ENC_SHERRY && h && !aligned16(h)) return STQ1_ERR_ALIGN;   // read as float4
  const long long n_blocks = N * (K / kBlockWeights);
  const long long grid = (n_blocks + kEncThreads - 1) / kEncThreads;
  if (grid >= (1LL << 31)) return STQ1_ERR_SHAPE;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  const int nb = static_cast<int>(K / kBlockWeights);
  const bool staged_h = mode == STQ1_ENC_SHERRY && h && nb <= kEncHMaxCols;
  return launch_pdl(encode_kernel, static_cast<unsigned>(grid), kEncThreads, encode_smem_bytes(nb, staged_h),
                    static_cast<cudaStream_t>(stream), W, h, n_blocks, static_cast<int>(K / kBlockWeights), mode,
                    rounds, out);
}

extern "C" int stq1_quantize_x_e4m3(const uint16_t* x, int64_t T, int64_t K, uint8_t* q, float* scales,
                                    void* stream) {
  NvtxRange nvtx_range("stq1_quantize_x_e4m3");
  if (!x || !q || !scales) return STQ1_ERR_NULL;
  if (T <= 0 || K <= 0 || K % 16 || T > (1LL << 31) - 1) return STQ1_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(q)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  return launch_pdl(quant_e4m3_kernel, static_cast<unsigned>(T), kQuantThreads, 0, static_cast<cudaStream_t>(stream),
                    x, static_cast<int>(K), q, scales);
}

extern "C" int stq1_swiglu(const float* y, uint16_t* act, int64_t P, int64_t N, void* stream) {
  NvtxRange nvtx_range("stq1_swiglu");
  if (!y || !act) return STQ1_ERR_NULL;
  if (P <= 0 || N <= 0 || (N & 1) || N > (1LL << 31) - 1 || P > (1LL << 40) / N) return STQ1_ERR_SHAPE;
  const long long total = P * (N / 2);
  const long long grid = std::min<long long>((total + 255) / 256, 148LL * 16);
  return launch_pdl(swiglu_kernel, static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream), y, act, P,
                    static_cast<int>(N / 2), static_cast<const int*>(nullptr));
}

extern "C" int stq1_moe_combine(const float* y, const float* w, float* out, int64_t T, int topk, int64_t H,
                                void* stream) {
  NvtxRange nvtx_range("stq1_moe_combine");
  if (!y || !out) return STQ1_ERR_NULL;
  if (T <= 0 || topk <= 0 || H <= 0 || H > (1LL << 31) - 1 || T > (1LL << 40) / (H * topk)) return STQ1_ERR_SHAPE;
  const long long total = T * H;
  const long long grid = std::min<long long>((total + 255) / 256, 148LL * 16);
  return launch_pdl(combine_kernel, static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream), y, w, out,
                    static_cast<long long>(T), topk, static_cast<int>(H));
}

namespace stq1 {
namespace {
struct FfnPlan {
  size_t ygu_off, act_off, yd_off, moe_off, moe_bytes, total;
};
FfnPlan plan_ffn(int T, int topk, int E, long long N, long long H, int flags) {
  FfnPlan f{};
  const long long P = static_cast<long long>(T) * topk;
  size_t off = 0;
  f.ygu_off = off;
  off += round16(static_cast<size_t>(P) * N * sizeof(float));
  f.act_off = off;
  off += round16(static_cast<size_t>(P) * (N / 2) * sizeof(uint16_t));
  f.yd_off = off;
  off += round16(static_cast<size_t>(P) * H * sizeof(float));
  f.moe_off = off;
  f.moe_bytes = std::max(plan_moe(T, topk, E, H, flags).total, plan_moe(static_cast<int>(P), 1, E, N / 2, flags).total);
  f.total = off + f.moe_bytes;
  return f;
}
}  // namespace
}  // namespace stq1

extern "C" size_t stq1_moe_ffn_workspace(int T, int topk, int E, int64_t N, int64_t H, int flags) {
  if (T <= 0 || topk <= 0 || E <= 0 || N <= 0 || (N & 1) || H <= 0 || H % kBlockWeights || (N / 2) % kBlockWeights)
    return 0;
  return plan_ffn(T, topk, E, N, H, flags).total;
}

extern "C" int stq1_moe_ffn(const void* gateup_blocks, const void* down_blocks, const uint16_t* x,
                            const int32_t* topk_ids, const float* topk_weights, float* out, int T, int topk, int E,
                            int64_t N, int64_t H, int flags, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("stq1_moe_ffn");
  if (!gateup_blocks || !down_blocks || !x || !topk_ids || !out) return STQ1_ERR_NULL;
  if (flags & ~(STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8 | STQ1_MOE_SKIP_FOREIGN)) return STQ1_ERR_ARG;
  if (T <= 0 || topk <= 0 || E <= 0 || N <= 0 || (N & 1) || H <= 0 || H % kBlockWeights || (N / 2) % kBlockWeights ||
      (H & 1) || static_cast<long long>(T) * topk > (1LL << 30))
    return STQ1_ERR_SHAPE;
  const FfnPlan f = plan_ffn(T, topk, E, N, H, flags);
  if (!ws || ws_bytes < f.total) return STQ1_ERR_WORKSPACE;
  if (!aligned16(ws)) return STQ1_ERR_ALIGN;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  float* ygu = reinterpret_cast<float*>(wsb + f.ygu_off);
  uint16_t* act = reinterpret_cast<uint16_t*>(wsb + f.act_off);
  float* yd = reinterpret_cast<float*>(wsb + f.yd_off);
  const int P = T * topk;
  // gate/up per (token, slot) pair; the routing weight goes on the up half or into the combine
  int rc = stq1_moe_gateup(gateup_blocks, x, topk_ids, topk_weights, ygu, T, topk, E, N, H, flags, wsb + f.moe_off,
                           f.moe_bytes, stream);
  if (rc != STQ1_OK) return rc;
  rc = stq1_swiglu(ygu, act, P, N, stream);
  if (rc != STQ1_OK) return rc;
  // down projection: each pair is its own token (ids [T, topk] read as [P, 1])
  rc = stq1_moe_gateup(down_blocks, act, topk_ids, nullptr, yd, P, 1, E, H, N / 2,
                       flags & (STQ1_MOE_FP8 | STQ1_MOE_SKIP_FOREIGN), wsb + f.moe_off, f.moe_bytes, stream);
  if (rc != STQ1_OK) return rc;
  return stq1_moe_combine(yd, (flags & STQ1_MOE_WEIGHT_UP) ? nullptr : topk_weights, out, T, topk, H, stream);
}

namespace stq1 {
namespace {
// One rank's share of an expert-parallel layer, stored compactly: only the
// pairs routed to this rank's experts are computed and stored, in the order
// of the grouped pair list; inv maps each (token, slot) pair to its row or -1.
struct FfnLocalPlan {
  MoePlan m;                       // routing and matmul plan (gate/up shape; the down shares the tables)
  size_t ids_off, pairs_off, tiles_off, small_off, ntiles_off, inv_off;
  size_t xperm_off, xq_off, sq_off, sperm_off;   // tile-path scratch, sized for both projections
  size_t ygu_off, act_off, yd_off, total;
  bool compact;                    // false: rows with an odd number of blocks (generic kernels)
};
FfnLocalPlan plan_ffn_local(int T, int topk, int E_local, long long N, long long H, int flags) {
  FfnLocalPlan f{};
  const long long P = static_cast<long long>(T) * topk;
  f.compact = (H / kBlockWeights) % 2 == 0 && (N / 2 / kBlockWeights) % 2 == 0;
  f.m = plan_moe(T, topk, E_local, H, flags);
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += round16(bytes); return o; };
  f.ids_off = take(P * sizeof(int32_t));
  f.pairs_off = take(P * sizeof(int));
  f.tiles_off = take(static_cast<size_t>(f.m.max_tiles) * 4 * sizeof(int));
  f.small_off = take(static_cast<size_t>(f.m.max_small) * 4 * sizeof(int));
  f.ntiles_off = take(16);
  f.inv_off = take(P * sizeof(int));
  const long long kmax = std::max(H, N / 2);
  f.xperm_off = f.xq_off = f.sq_off = f.sperm_off = off;
  if (f.m.tiles) {
    f.xperm_off = take(static_cast<size_t>(P) * H * (f.m.fp8 ? 1 : 2));   // gate/up gather
    if (f.m.fp8) {
      f.xq_off = take(static_cast<size_t>(std::max<long long>(T, P)) * kmax);
      f.sq_off = take(static_cast<size_t>(std::max<long long>(T, P)) * sizeof(float));
      f.sperm_off = take(static_cast<size_t>(P) * sizeof(float));
    }
  }
  f.ygu_off = take(static_cast<size_t>(P) * N * sizeof(float));
  f.act_off = take(static_cast<size_t>(P) * (N / 2) * sizeof(uint16_t));
  f.yd_off = take(static_cast<size_t>(P) * H * sizeof(float));
  f.total = off;
  return f;
}
}  // namespace
}  // namespace stq1

extern "C" size_t stq1_moe_ffn_local_workspace(int T, int topk, int E_local, int64_t N, int64_t H, int flags) {
  if (T <= 0 || topk <= 0 || E_local <= 0 || N <= 0 || (N & 1) || H <= 0 || H % kBlockWeights ||
      (N / 2) % kBlockWeights)
    return 0;
  const FfnLocalPlan f = plan_ffn_local(T, topk, E_local, N, H, flags);
  if (f.compact) return f.total;
  // generic shapes: shifted ids, then the whole-layer chain with foreign pairs skipped
  const size_t w = stq1_moe_ffn_workspace(T, topk, E_local, N, H, flags);
  return w ? w + round16(static_cast<size_t>(T) * topk * sizeof(int32_t)) : 0;
}

extern "C" int stq1_moe_ffn_local(const void* gateup_local, const void* down_local, const uint16_t* x,
                                  const int32_t* topk_ids, const float* topk_weights, float* out, int T, int topk,
                                  int E_local, int expert_begin, int64_t N, int64_t H, int flags, void* ws,
                                  size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("stq1_moe_ffn_local");
  if (!gateup_local || !down_local || !x || !topk_ids || !out) return STQ1_ERR_NULL;
  if (!ws) return STQ1_ERR_WORKSPACE;
  if (flags & ~(STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8 | STQ1_MOE_SKIP_FOREIGN)) return STQ1_ERR_ARG;
  if (T <= 0 || topk <= 0 || E_local <= 0 || expert_begin < 0 || E_local > kMaxExperts) return STQ1_ERR_SHAPE;
  const size_t need = stq1_moe_ffn_local_workspace(T, topk, E_local, N, H, flags);
  if (need == 0 || static_cast<long long>(T) * topk > (1LL << 30)) return STQ1_ERR_SHAPE;
  if (ws_bytes < need) return STQ1_ERR_WORKSPACE;
  if (!aligned16(ws) || !aligned16(gateup_local) || !aligned16(down_local) || !aligned16(x)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long n = static_cast<long long>(T) * topk;
  const FfnLocalPlan f = plan_ffn_local(T, topk, E_local, N, H, flags);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  // this rank's view of the routing: ids of its range start at 0, others fall outside [0, E_local)
  int32_t* ids_local = reinterpret_cast<int32_t*>(wsb + (f.compact ? f.ids_off : 0));
  rc = launch_pdl(shift_ids_kernel, static_cast<unsigned>(std::min<long long>((n + 255) / 256, 1024)), 256, 0, s,
                  topk_ids, ids_local, n, expert_begin);
  if (rc != STQ1_OK) return rc;
  if (!f.compact) {
    const size_t ids_bytes = round16(static_cast<size_t>(n) * sizeof(int32_t));
    return stq1_moe_ffn(gateup_local, down_local, x, ids_local, topk_weights, out, T, topk, E_local, N, H,
                        flags | STQ1_MOE_SKIP_FOREIGN, wsb + ids_bytes, ws_bytes - ids_bytes, stream);
  }
  const int P = static_cast<int>(n);
  MoeTables tb;
  tb.pairs = reinterpret_cast<int*>(wsb + f.pairs_off);
  tb.tiles = reinterpret_cast<int*>(wsb + f.tiles_off);
  tb.tiles_small = reinterpret_cast<int*>(wsb + f.small_off);
  tb.ntiles = reinterpret_cast<int*>(wsb + f.ntiles_off);
  int* inv = reinterpret_cast<int*>(wsb + f.inv_off);
  MoeScratch sc;
  sc.xperm = wsb + f.xperm_off;
  sc.xq = wsb + f.xq_off;
  sc.sq = reinterpret_cast<float*>(wsb + f.sq_off);
  sc.sperm = reinterpret_cast<float*>(wsb + f.sperm_off);
  float* ygu = reinterpret_cast<float*>(wsb + f.ygu_off);
  uint16_t* act = reinterpret_cast<uint16_t*>(wsb + f.act_off);
  float* yd = reinterpret_cast<float*>(wsb + f.yd_off);
  // group the local pairs by expert; foreign pairs get no row (inv = -1) and nothing is written for them
  rc = launch_pdl(route_kernel, 1, kRouteThreads, 3 * E_local * sizeof(int), s, static_cast<const int32_t*>(ids_local),
                  P, E_local, f.m.tile_tokens, f.m.small_max, tb.pairs, tb.tiles, tb.tiles_small, tb.ntiles, inv,
                  static_cast<float*>(nullptr), static_cast<int>(N), 1, f.m.max_tiles, f.m.max_small);
  if (rc != STQ1_OK) return rc;
  // gate/up of the local pairs into compact rows (routing weight on the up half with STQ1_MOE_WEIGHT_UP)
  rc = moe_compute(f.m, tb, sc, gateup_local, x, T, topk_weights, ygu, topk, P, E_local, N, H, flags, 1, s);
  if (rc != STQ1_OK) return rc;
  // SwiGLU over the rows in use (their count is on the device)
  const long long half = N / 2;
  const long long grid = std::min<long long>((n * half + 255) / 256, 148LL * 16);
  rc = launch_pdl(swiglu_kernel, static_cast<unsigned>(grid), 256, 0, s, static_cast<const float*>(ygu), act, n,
                  static_cast<int>(half), static_cast<const int*>(tb.ntiles + 1));
  if (rc != STQ1_OK) return rc;
  // down projection on the same tables: compact rows in, compact rows out
  rc = moe_compute(f.m, tb, sc, down_local, act, P, nullptr, yd, 1, P, E_local, H, N / 2,
                   flags & STQ1_MOE_FP8, 3, s);
  if (rc != STQ1_OK) return rc;
  // combine through the pair -> row map (plain sum when the weight went on the up half)
  const long long total = static_cast<long long>(T) * H;
  const long long cgrid = std::min<long long>((total + 255) / 256, 148LL * 16);
  return launch_pdl(combine_compact_kernel, static_cast<unsigned>(cgrid), 256, 0, s, static_cast<const float*>(yd),
                    (flags & STQ1_MOE_WEIGHT_UP) ? static_cast<const float*>(nullptr) : topk_weights,
                    static_cast<const int*>(inv), out, static_cast<long long>(T), topk, static_cast<int>(H), n);
}

extern "C" int stq1_ep_dispatch(const int32_t* topk_ids, const uint16_t* x, const float* topk_weights, int T,
                                int topk, int E, int world, int64_t K, int32_t* order, int32_t* inv, int32_t* counts,
                                int32_t* local_ids, uint16_t* x_send, float* w_send, void* stream) {
  NvtxRange nvtx_range("stq1_ep_dispatch");
  if (!topk_ids || !x || !order || !inv || !counts || !local_ids || !x_send) return STQ1_ERR_NULL;
  if (w_send && !topk_weights) return STQ1_ERR_NULL;
  if (T <= 0 || topk <= 0 || E <= 0 || world <= 0 || world > E || world > 4096 || K <= 0 || K % 8 ||
      static_cast<long long>(T) * topk > (1LL << 30) || K > (1LL << 30))
    return STQ1_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(x_send)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int n = T * topk;
  rc = launch_pdl(ep_dispatch_kernel, 1, kDispatchThreads, 2 * world * sizeof(int), s, topk_ids, n, E, world, order,
                  inv, counts, local_ids);
  if (rc != STQ1_OK) return rc;
  return launch_pdl(ep_gather_kernel, static_cast<unsigned>(n), 256, 0, s, x, w_send ? topk_weights : nullptr,
                    static_cast<const int*>(order), static_cast<const int*>(counts + world), topk,
                    static_cast<int>(K), x_send, w_send, n);
}

extern "C" int stq1_ep_combine(const float* rows, const int32_t* inv, float* out, int64_t T, int topk, int64_t H,
                               void* stream) {
  NvtxRange nvtx_range("stq1_ep_combine");
  if (!rows || !inv || !out) return STQ1_ERR_NULL;
  if (T <= 0 || topk <= 0 || H <= 0 || H > (1LL << 31) - 1 || T > (1LL << 40) / (H * topk)) return STQ1_ERR_SHAPE;
  const long long total = T * H;
  const long long grid = std::min<long long>((total + 255) / 256, 148LL * 16);
  return launch_pdl(combine_compact_kernel, static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream),
                    rows, static_cast<const float*>(nullptr), static_cast<const int*>(inv), out,
                    static_cast<long long>(T), topk, static_cast<int>(H), T * topk);
}

extern "C" int stq1_set_path(int path) {
  if (path < 0 || path > 3) return STQ1_ERR_ARG;
  g_path.store(path);
  return STQ1_OK;
}

extern "C" int stq1_selftest_wait(int arrive, void* stream) {
  NvtxRange nvtx_range("stq1_selftest_wait");
  if (arrive != 0 && arrive != 1) return STQ1_ERR_ARG;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(arrive);
  return launch_status();
}

extern "C" int stq1_selftest_bounds(int index, int bound, void* stream) {
  NvtxRange nvtx_range("stq1_selftest_bounds");
  bounds_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(index, bound);
  return launch_status();
}

extern "C" int stq1_build_flags(void) { return kDebugBuild ? STQ1_BUILD_DEBUG : 0; }

extern "C" int stq1_status(void* stream, int* device_err) {
  NvtxRange nvtx_range("stq1_status");
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return STQ1_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_err, sizeof(int)) != cudaSuccess) return STQ1_ERR_CUDA;
  if (v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_dev_err, &zero, sizeof(int)) != cudaSuccess) return STQ1_ERR_CUDA;
  }
  if (device_err) *device_err = v;
  return v ? STQ1_ERR_DEVICE : STQ1_OK;
}

// ---------------------------------------------------------------------------
// GEMV that allocates nothing (no counterpart on the source pages).
//
// Some callers cannot hand this library a workspace: frameworks and plugin
// hosts that own all device memory and pass in only the input and output
// buffers, and latency-critical code that must not call cudaMalloc, which can
// synchronize the whole device.  For them, stq1_gemv_noalloc runs the table
// GEMV with its split-K scratch (arrival counters and partial sums) in a
// fixed buffer compiled into the library.
// ---------------------------------------------------------------------------
namespace stq1 {
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(1) << 20;   // 1 MiB

// Loaded with the library on every GPU that uses it and kept until the process
// exits.  Host code must not use this name as a device address: it only
// stands in for the symbol; the device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

uint8_t* g_static_scratch_ptr[kMaxDevices] = {};
std::mutex g_static_scratch_mutex;

// One-time set-up per device, with that device current (under a lock: two
// host threads making their first call at once look the address up once).
int static_scratch(uint8_t** out) {
  const int dev = current_device();
  if (dev < 0) return STQ1_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr)
      return STQ1_ERR_CUDA;
    g_static_scratch_ptr[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_static_scratch_ptr[dev];
  return STQ1_OK;
}

}  // namespace
}  // namespace stq1

extern "C" int stq1_gemv_noalloc(const void* W_packed, const uint16_t* x, float* y, int64_t N,
                                 int64_t K, int batch, void* stream) {
  NvtxRange nvtx_range("stq1_gemv_noalloc");
  if (!W_packed || !x || !y) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || K % kBlockWeights || batch <= 0 || batch > 65535 ||
      N > (1LL << 31) - 1 || K > (1LL << 31) - 1)
    return STQ1_ERR_SHAPE;
  if (!aligned16(W_packed) || !aligned16(x)) return STQ1_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long nb = K / kBlockWeights;
  const long long rowbytes = nb * kBlockBytes;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  if (nb % 2 != 0) {
    // rows with an odd number of blocks use the direct kernel, which needs no scratch
    const long long warps = static_cast<long long>(batch) * N;
    direct_gemv_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(W_packed), 0, 1, x, nullptr, 1, nullptr, 0, y,
        static_cast<int>(N), static_cast<int>(K), batch);
    return launch_status();
  }
  // The table path's work split, without its one-wave cap on the K split (a
  // plain launch reduces through the scratch buffer, whatever the split).
  GemvPlan p{};
  plan_table(&p, N, K, batch, false);
  const int n_tiles = p.n_tiles, n_slabs = p.n_slabs, n_chunks = p.n_chunks, S = p.S;
  const long long units0 = static_cast<long long>(n_tiles) * n_slabs;
  const size_t need = S > 1 ? kCounterBytes + static_cast<size_t>(S) * batch * N * sizeof(float) : 0;
  if (need > kStaticScratchBytes) return STQ1_ERR_SCRATCH;
  uint8_t* scratch = nullptr;
  if (S > 1) {
    rc = static_scratch(&scratch);
    if (rc != STQ1_OK) return rc;
    // the array keeps the previous call's contents: the counters must start at zero
    if (cudaMemsetAsync(scratch, 0, kCounterBytes, s) != cudaSuccess) return STQ1_ERR_CUDA;
  }
  LutArgs a{};
  PackedMaps maps;
  rc = packed_maps_cached(&maps, &a.g, static_cast<const uint8_t*>(W_packed), N, rowbytes, false);
  if (rc != STQ1_OK) return rc;
  a.x = x;
  a.y = y;
  a.counters = S > 1 ? reinterpret_cast<int*>(scratch) : nullptr;
  a.partial = S > 1 ? reinterpret_cast<float*>(scratch + kCounterBytes) : nullptr;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.topk = 1;
  a.batch = batch;
  a.rows_out = batch;
  a.x_rows = batch;
  a.n_slabs = n_slabs;
  set_split(&a, n_chunks, S);
  a.flags = 0;
  a.cluster = 0;
  if (units0 >= (1LL << 31)) return STQ1_ERR_SHAPE;
  const dim3 grid(static_cast<unsigned>(units0), static_cast<unsigned>(S));
  const size_t smem = lut_smem_bytes(batch == 1 ? 1 : (batch == 2 ? 2 : 4), lut_stages(a), a.g.stage_bytes, 1);
  if (batch == 1)
    lut_gemv_kernel<1><<<grid, kLutThreads, smem, s>>>(maps.w, maps.t, a);
  else if (batch == 2)
    lut_gemv_kernel<2><<<grid, kLutThreads, smem, s>>>(maps.w, maps.t, a);
  else
    lut_gemv_kernel<4><<<grid, kLutThreads, smem, s>>>(maps.w, maps.t, a);
  return launch_status();
}

// ---------------------------------------------------------------------------
// Mixed-precision allocation: STQ2 encoder, Hessian diagonal, layer error.
// ---------------------------------------------------------------------------

extern "C" int stq1_quantize_stq2(const float* W, const float* h, int64_t N, int64_t K, int rounds, uint8_t* out,
                                  void* stream) {
  NvtxRange nvtx_range("stq1_quantize_stq2");
  if (!W || !out) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || K % kBlockWeights || N > (1LL << 40) / K) return STQ1_ERR_SHAPE;
  if (rounds < 0 || rounds > 1000) return STQ1_ERR_ARG;
  if (!aligned16(W) || (reinterpret_cast<uintptr_t>(out) & 1) || (h && !aligned16(h)))   // h read as float4
    return STQ1_ERR_ALIGN;
  const long long n_blocks = N * (K / kBlockWeights);
  const long long grid = (n_blocks + kEncThreads - 1) / kEncThreads;
  if (grid >= (1LL << 31)) return STQ1_ERR_SHAPE;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  const int nb = static_cast<int>(K / kBlockWeights);
  const bool staged_h = h && nb <= kEncHMaxCols;
  return launch_pdl(stq2_encode_kernel, static_cast<unsigned>(grid), kEncThreads, encode_smem_bytes(nb, staged_h),
                    static_cast<cudaStream_t>(stream), W, h, n_blocks, nb, rounds, out);
}

extern "C" int stq1_hessian_diag(const uint16_t* x, int64_t L, int64_t rows, int64_t K, float* h, void* stream) {
  NvtxRange nvtx_range("stq1_hessian_diag");
  if (!x || !h) return STQ1_ERR_NULL;
  if (L <= 0 || rows <= 0 || K <= 0 || L > 65535 || rows > (1LL << 40) / K || L > (1LL << 40) / (rows * K))
    return STQ1_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x) & 1) || (reinterpret_cast<uintptr_t>(h) & 3)) return STQ1_ERR_ALIGN;
  const long long gx = (K + 255) / 256;
  if (gx >= (1LL << 31)) return STQ1_ERR_SHAPE;
  return launch_pdl_cluster(hess_diag_kernel, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(L)), 256, 0,
                            static_cast<cudaStream_t>(stream), 1u, x, static_cast<long long>(rows),
                            static_cast<long long>(K), h);
}

namespace {

// 3-D map over calibration rows [L][n_cal][K] of bf16: box = 64 columns (one
// 128-byte swizzle atom) x box_rows rows x 1 layer; rows past n_cal read as zero.
bool make_cal_map(CUtensorMap* map, const void* base, long long L, long long n_cal, long long K, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(n_cal), static_cast<cuuint64_t>(L)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(n_cal * K) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kHsKC), static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstride, box, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int stq1_hessian_error(int format, const void* packed, const float* W, const uint16_t* x,
                                  const float* h, int64_t L, int64_t N, int64_t K, int64_t n_cal, double* out,
                                  void* stream) {
  NvtxRange nvtx_range("stq1_hessian_error");
  if (!packed || !W || !x || !h || !out) return STQ1_ERR_NULL;
  if (format != STQ1_FMT_STQ1_0 && format != STQ1_FMT_STQ2) return STQ1_ERR_ARG;
  if (L <= 0 || N <= 0 || n_cal <= 0 || K < kBlockWeights || K % kBlockWeights) return STQ1_ERR_SHAPE;
  if (K > (1LL << 31) - 1 || n_cal > (1LL << 31) - 1 || L > (1LL << 31) - 1) return STQ1_ERR_SHAPE;
  if (N > (1LL << 40) / K || L > (1LL << 40) / (N * K) || L > (1LL << 40) / (n_cal * K)) return STQ1_ERR_SHAPE;
  if (!aligned16(W) || !aligned16(x) || !aligned16(h) || (reinterpret_cast<uintptr_t>(packed) & 1) ||
      (reinterpret_cast<uintptr_t>(out) & 7))
    return STQ1_ERR_ALIGN;
  const long long n_mtiles = (N + kHsM - 1) / kHsM;
  const long long n_cchunks = (n_cal + kHsMaxCal - 1) / kHsMaxCal;
  const long long items = L * n_mtiles * n_cchunks;
  if (items >= (1LL << 31)) return STQ1_ERR_SHAPE;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  const int box_rows = static_cast<int>(std::min<long long>(kHsMaxCal, (n_cal + 15) / 16 * 16));
  CUtensorMap map;
  if (!make_cal_map(&map, x, L, n_cal, K, box_rows)) return STQ1_ERR_CUDA;
  HsArgs a{};
  a.W = W;
  a.packed = static_cast<const uint8_t*>(packed);
  a.h = h;
  a.out = out;
  a.N = N;
  a.K = K;
  a.bb = format == STQ1_FMT_STQ1_0 ? kBlockBytes : kStq2BlockBytes;
  a.n_mtiles = static_cast<int>(n_mtiles);
  a.n_cchunks = static_cast<int>(n_cchunks);
  a.box_rows = box_rows;
  a.tmem_cols = box_rows <= 32 ? 32u : (box_rows <= 64 ? 64u : (box_rows <= 128 ? 128u : 256u));
  a.idesc = hs_idesc(box_rows);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(out, 0, static_cast<size_t>(L) * 2 * sizeof(double), s) != cudaSuccess) return STQ1_ERR_CUDA;
  if (format == STQ1_FMT_STQ1_0)
    return launch_pdl(hess_score_kernel<0>, static_cast<unsigned>(items), kHsThreads, kHsSmemBytes, s, map, a);
  return launch_pdl(hess_score_kernel<1>, static_cast<unsigned>(items), kHsThreads, kHsSmemBytes, s, map, a);
}
