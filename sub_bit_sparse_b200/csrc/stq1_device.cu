// C-ABI entry points of libstq1.so (device side).  Argument checks happen on the
// host before anything is enqueued; every entry point returns an STQ1_* code.
#include <algorithm>
#include <cstdint>
#include <cstdio>

#include "device_common.cuh"
#include "gemv_lut.cuh"
#include "small_kernels.cuh"

namespace stq1 {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kTargetUnits = 444;   // aim for ~3 work units per SM on a 148-SM part
constexpr int kMaxExperts = 4096;
// Split-K counters live at a fixed offset (0) of the GEMV workspace so that their
// zero-between-calls invariant does not depend on the shape of earlier calls.
// Split K is used only when tiles x slabs < kTargetUnits, so this bounds them.
constexpr size_t kCounterBytes = 2048;
static_assert(kTargetUnits * sizeof(int) <= kCounterBytes, "counter region too small");

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

// Per-device one-time kernel attribute setup (dynamic shared memory limits).
int ensure_configured() {
  static bool done[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return STQ1_ERR_CUDA;
  if (done[dev]) return STQ1_OK;
  if (cudaFuncSetAttribute(lut_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lut_smem_bytes(1))) != cudaSuccess ||
      cudaFuncSetAttribute(lut_gemv_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lut_smem_bytes(4))) != cudaSuccess ||
      cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           3 * kMaxExperts * 4) != cudaSuccess)
    return STQ1_ERR_CUDA;
  done[dev] = true;
  return STQ1_OK;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? STQ1_OK : STQ1_ERR_CUDA;
}

int residue_period(long long rowbytes) {
  // rows per residue class of (row * rowbytes) mod 16, for rowbytes % 4 == 0
  const long long g = (rowbytes % 16 == 0) ? 16 : ((rowbytes % 8 == 0) ? 8 : 4);
  return static_cast<int>(16 / g);
}

struct GemvPlan {
  int n_tiles, n_slabs, S, n_chunks;
  size_t partial_bytes, counter_bytes;
  bool table_path;
};

GemvPlan plan_gemv(long long N, long long K, int batch) {
  GemvPlan p{};
  const long long nb = K / kBlockWeights;
  p.table_path = (nb % 2 == 0);
  p.n_tiles = (batch + kLutMaxTT - 1) / kLutMaxTT;
  p.n_slabs = static_cast<int>((N + kLutRows - 1) / kLutRows);
  p.n_chunks = static_cast<int>(nb / kLutKC);
  const long long units0 = static_cast<long long>(p.n_tiles) * p.n_slabs;
  long long S = (kTargetUnits + units0 - 1) / units0;
  S = std::max<long long>(1, std::min<long long>(S, std::max(1, p.n_chunks)));
  p.S = p.table_path ? static_cast<int>(S) : 1;
  if (p.table_path && p.S > 1) {
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

extern "C" int stq1_gemv(const void* W_packed, const uint16_t* x, float* y, int64_t N, int64_t K,
                         int batch, void* workspace, size_t ws_bytes, void* stream) {
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
  if (!p.table_path) {
    const long long warps = static_cast<long long>(batch) * N;
    direct_gemv_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(W_packed), 0, 1, x, nullptr, 1, nullptr, 0, y,
        static_cast<int>(N), static_cast<int>(K), batch);
    return launch_status();
  }
  LutArgs a{};
  a.W = static_cast<const uint8_t*>(W_packed);
  a.W_end = a.W + N * rowbytes;
  a.expert_bytes = 0;
  a.rowbytes = rowbytes;
  a.x = x;
  a.y = y;
  a.counters = p.S > 1 ? static_cast<int*>(workspace) : nullptr;
  a.partial = p.S > 1 ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes) : nullptr;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.nb = static_cast<int>(nb);
  a.topk = 1;
  a.batch = batch;
  a.rows_out = batch;
  a.n_tiles = p.n_tiles;
  a.n_slabs = p.n_slabs;
  a.S = p.S;
  a.n_chunks = p.n_chunks;
  a.P = residue_period(rowbytes);
  a.flags = 0;
  const long long grid = static_cast<long long>(p.n_tiles) * p.n_slabs * p.S;
  if (batch == 1) {
    lut_gemv_kernel<1><<<static_cast<unsigned>(grid), kLutThreads, lut_smem_bytes(1), s>>>(a);
  } else {
    lut_gemv_kernel<4><<<static_cast<unsigned>(grid), kLutThreads, lut_smem_bytes(4), s>>>(a);
  }
  return launch_status();
}

namespace stq1 {
namespace {
struct MoePlan {
  size_t pairs_off, tiles_off, ntiles_off, total;
  int max_tiles;
};
MoePlan plan_moe(int T, int topk, int E) {
  MoePlan m{};
  const long long n_pairs = static_cast<long long>(T) * topk;
  m.max_tiles = static_cast<int>(std::min<long long>(n_pairs, n_pairs / kLutMaxTT + std::min<long long>(E, n_pairs)));
  size_t off = 0;
  m.pairs_off = off;
  off += round16(n_pairs * sizeof(int));
  m.tiles_off = off;
  off += round16(static_cast<size_t>(m.max_tiles) * 4 * sizeof(int));
  m.ntiles_off = off;
  off += 16;
  m.total = off;
  return m;
}
}  // namespace
}  // namespace stq1

extern "C" size_t stq1_moe_workspace(int T, int topk, int E, int64_t N, int64_t K, int flags) {
  (void)N;
  (void)K;
  (void)flags;
  if (T <= 0 || topk <= 0 || E <= 0) return 0;
  return plan_moe(T, topk, E).total;
}

extern "C" int stq1_moe_gateup(const void* expert_blocks, const uint16_t* x, const int32_t* topk_ids,
                               const float* topk_weights, float* y, int T, int topk, int E, int64_t N,
                               int64_t K, int flags, void* ws, size_t ws_bytes, void* stream) {
  if (!expert_blocks || !x || !topk_ids || !y) return STQ1_ERR_NULL;
  if ((flags & STQ1_MOE_WEIGHT_UP) && !topk_weights) return STQ1_ERR_NULL;
  if (flags & ~(STQ1_MOE_WEIGHT_UP | STQ1_MOE_FP8)) return STQ1_ERR_ARG;
  if (T <= 0 || topk <= 0 || E <= 0 || topk > E || E > kMaxExperts || N <= 0 || (N & 1) || K <= 0 ||
      K % kBlockWeights || N > (1LL << 30) || K > (1LL << 30) ||
      static_cast<long long>(T) * topk > (1LL << 30))
    return STQ1_ERR_SHAPE;
  if (!aligned16(expert_blocks) || !aligned16(x)) return STQ1_ERR_ALIGN;
  const MoePlan m = plan_moe(T, topk, E);
  if (!ws || ws_bytes < m.total) return STQ1_ERR_WORKSPACE;
  if (!aligned16(ws)) return STQ1_ERR_ALIGN;
  int rc = ensure_configured();
  if (rc != STQ1_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const long long nb = K / kBlockWeights;
  const long long rowbytes = nb * kBlockBytes;
  const int n_pairs = T * topk;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  int* pairs = reinterpret_cast<int*>(wsb + m.pairs_off);
  int* tiles = reinterpret_cast<int*>(wsb + m.tiles_off);
  int* ntiles = reinterpret_cast<int*>(wsb + m.ntiles_off);

  if (nb % 2 != 0) {
    const long long warps = static_cast<long long>(n_pairs) * N;
    direct_gemv_kernel<<<static_cast<unsigned>((warps + 7) / 8), 256, 0, s>>>(
        static_cast<const uint8_t*>(expert_blocks), N * rowbytes, E, x, topk_ids, topk, topk_weights,
        flags, y, static_cast<int>(N), static_cast<int>(K), n_pairs);
    return launch_status();
  }

  route_kernel<<<1, kRouteThreads, 3 * E * sizeof(int), s>>>(topk_ids, n_pairs, E, kLutMaxTT, pairs,
                                                             tiles, ntiles, y, static_cast<int>(N));
  rc = launch_status();
  if (rc != STQ1_OK) return rc;
  LutArgs a{};
  a.W = static_cast<const uint8_t*>(expert_blocks);
  a.W_end = a.W + static_cast<long long>(E) * N * rowbytes;
  a.expert_bytes = N * rowbytes;
  a.rowbytes = rowbytes;
  a.x = x;
  a.y = y;
  a.partial = nullptr;
  a.counters = nullptr;
  a.tile_info = tiles;
  a.n_tiles_dev = ntiles;
  a.pairs = pairs;
  a.route_w = topk_weights;
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.nb = static_cast<int>(nb);
  a.topk = topk;
  a.batch = 0;
  a.rows_out = n_pairs;
  a.n_tiles = m.max_tiles;
  a.n_slabs = static_cast<int>((N + kLutRows - 1) / kLutRows);
  a.S = 1;
  a.n_chunks = static_cast<int>(nb / kLutKC);
  a.P = residue_period(rowbytes);
  a.flags = flags;
  const long long grid = static_cast<long long>(m.max_tiles) * a.n_slabs;
  lut_gemv_kernel<4><<<static_cast<unsigned>(grid), kLutThreads, lut_smem_bytes(4), s>>>(a);
  return launch_status();
}

extern "C" int stq1_status(void* stream, int* device_err) {
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
