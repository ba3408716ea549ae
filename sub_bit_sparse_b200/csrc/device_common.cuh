// Device helpers shared by the STQ1_0 kernels: block-format constants, the
// codebook, and thin wrappers around the sm_90+/sm_100 PTX the kernels use
// (mbarriers, 1-D bulk copies, shared-memory loads with immediate offsets).
#pragma once

#include <cstdint>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "../../include/stq1.h"

namespace stq1 {

// ---- STQ1_0 block format ("How STQ1_0 works": 42 bytes per 256 weights) ----
constexpr int kBlockWeights = 256;
constexpr int kGroupsPerBlock = 64;
constexpr int kBlockBytes = 42;
constexpr int kOffD = 0;    // fp16 scale
constexpr int kOffQs = 2;   // 32 bytes of 4-bit codes, even group in the low nibble
constexpr int kOffQh = 34;  // 8 bytes of select bits, group g at bit g & 7 of byte g >> 3

// Device error word, read and cleared by stq1_status().
__device__ int g_dev_err;

__device__ __forceinline__ void flag_error(int bits) { atomicOr(&g_dev_err, bits); }

// Bounds checks of the debug build (compiled with -DSTQ1_DEBUG): a failed
// check records STQ1_DEV_BOUNDS in the device error word and the caller skips
// the access it guards.  The release build compiles every check to `true`.
#ifdef STQ1_DEBUG
constexpr bool kDebugBuild = true;
__device__ __forceinline__ bool dbg_check(bool ok) {
  if (!ok) flag_error(STQ1_DEV_BOUNDS);
  return ok;
}
// [addr, addr + bytes) lies inside this CTA's dynamic shared memory.
__device__ __forceinline__ bool dbg_smem_range(uint32_t addr, uint32_t bytes) {
  extern __shared__ __align__(16) uint8_t stq1_dyn_smem[];
  const uint32_t lo = static_cast<uint32_t>(__cvta_generic_to_shared(stq1_dyn_smem));
  uint32_t size;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(size));
  return dbg_check(addr >= lo && addr + bytes <= lo + size);
}
#else
constexpr bool kDebugBuild = false;
__device__ __forceinline__ bool dbg_check(bool) { return true; }
__device__ __forceinline__ bool dbg_smem_range(uint32_t, uint32_t) { return true; }
#endif

// Codebook: code = t << 4 | n; zero lane z = n >> 2; non-zero lanes a < b < c
// carry +1, -(bit1 of n), -(bit0 of n); t = 1 negates them.  Returns the
// lane values in {-1, 0, +1} (lemmy.durstig.online post 66506, "Four weights,
// five bits"; the lane order and table split are this library's layout).
__device__ __forceinline__ void code_pattern(unsigned code, int v[4]) {
  const unsigned n = code & 15u, t = (code >> 4) & 1u;
  const unsigned z = n >> 2;
  const int s = t ? -1 : 1;
  const int la = (z == 0) ? 1 : 0;
  const int lb = (z <= 1) ? 2 : 1;
  const int lc = (z == 3) ? 2 : 3;
  v[0] = v[1] = v[2] = v[3] = 0;
  v[la] = s;
  v[lb] = ((n >> 1) & 1u) ? -s : s;
  v[lc] = (n & 1u) ? -s : s;
}

// Compile-time loop helper: f(IntC<0>{}) ... f(IntC<N-1>{}).
template <int I>
struct IntC {
  static constexpr int value = I;
};
template <typename F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
  (f(IntC<Is>{}), ...);
}
template <int N, typename F>
__device__ __forceinline__ void static_for(F&& f) {
  static_for_impl(f, std::make_integer_sequence<int, N>{});
}

// ---- PTX wrappers ----
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or about `kWaitHintNs` pass, instead of spinning.
constexpr uint32_t kWaitHintNs = 100000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(kWaitHintNs)
      : "memory");
  return done != 0;
}

// Bounded wait on an mbarrier phase: at most 2^14 suspended tries (each ends
// early when the phase completes, or after about the hint), so a few seconds
// at the very most.  Returns false (and flags the device error word) if the
// phase did not complete.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < (1u << 14); ++i)
    if (mbar_try_wait(bar, parity)) return true;
  flag_error(STQ1_DEV_WAIT_LIMIT);
  return false;
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted in bytes
// on `bar`.  dst, src and bytes must all be multiples of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Programmatic dependent launch: wait for the preceding kernel in the stream
// (no-op when the launch did not ask for overlap), and let the next kernel
// start launching.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Thread-block clusters: rank in the cluster, a full cluster barrier, and a
// load from a peer CTA's shared memory (distributed shared memory).
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
constexpr int kMaxClusterRanks = 16;   // largest (non-portable) cluster the kernels use
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// The two halves of a cluster barrier, for work between them.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}
// Cluster barrier without memory ordering: only to keep a CTA (and its shared
// memory) alive until its peers are done reading it.
__device__ __forceinline__ void cluster_sync_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_peer_f32(uint32_t local_addr, uint32_t rank) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

__device__ __forceinline__ void st_peer_f32(uint32_t local_addr, uint32_t rank, float v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local_addr), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(remote), "f"(v) : "memory");
}

// Asynchronous store of one fp32 into the shared memory of cluster CTA
// `rank` (same offset as local_addr), counted as 4 bytes of completed
// transactions on that CTA's mbarrier at local_bar's offset.  The sender does
// not wait for it; the receiver waits on its own mbarrier.
__device__ __forceinline__ void st_async_peer_f32(uint32_t local_addr, uint32_t local_bar, uint32_t rank, float v) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(local_addr), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(local_bar), "r"(rank));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(ra),
               "r"(__float_as_uint(v)), "r"(rb)
               : "memory");
}

// Two fp32 additions in one instruction (the packed f32x2 add of sm_100),
// each lane rounded to nearest as a scalar add: {a.x + b.x, a.y + b.y}.
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\t"
      "mov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}

template <int OFF>
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1+%2];" : "=f"(v) : "r"(addr), "n"(OFF));
  return v;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void sts_v4f(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float(b << 16);
}

}  // namespace stq1
