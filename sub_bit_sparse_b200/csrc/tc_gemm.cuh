// Tensor-core tile path for STQ1_0 at large token counts (sm_100a, tcgen05).
//
// y[p, j] = sum_k W^[j, k] x[tok(p), k] for all pairs p of an expert (or all
// tokens of a plain matmul).  Per 256-column block the weights are
// d_{j,b} * s_{jk} with s in {-1, 0, +1} ("How STQ1_0 works"); s is exact in
// bf16, d is not.  So each tile contracts the +/-1 pattern against bf16
// activations on the tensor cores, one 256-column slab at a time into a TMEM
// accumulator, and CUDA cores add d_{j,b} * slab into an fp32 register
// accumulator (a5 of the hot path, done once per row, slab and token).
//
// Tile: M = 128 weight rows x N = 128 tokens, K in stages of one 256-column
// scale block (bf16: four 128-byte swizzle atoms, 16 MMAs; fp8: two atoms,
// 8 MMAs).
//   warp 0      TMA producer: x tiles (128-byte swizzle) into a shared ring
//               (bf16: 3 stages of 64 KB, fp8: 4 of 32 KB), one 2-D tensor
//               copy per atom, no multicast.
//   warps 1, 19 the two MMA-issuing threads (warp 1 also allocates TMEM):
//               tcgen05.mma.cta_group::1, A from TMEM, B from shared; warp 1
//               issues the even stages, warp 19 the odd ones, so that one
//               thread waits for its next stage's operands while the MMAs the
//               other queued keep the tensor pipe busy.
//   warp 18     TMA producer of the packed weights: per 128-row tile, chunks
//               of two blocks (the super-row tensor copies of
//               packed_copy.cuh) into a shared ring (bf16: 2 stages,
//               fp8: 4).
//   warps 2-9   decoders, two per TMEM lane quadrant: a thread owns one weight
//               row (TMEM lane order = the ring's slot order), copies a
//               chunk's two blocks of codes from shared memory into registers
//               (releasing the stage), expands each group's 5-bit code to four
//               bf16 values through a 32-entry table and stores its half of
//               each stage's columns into TMEM (tcgen05.st), the A operand.
//   warps 10-17 epilogue, two per quadrant (64 token columns each): per slab,
//               tcgen05.ld of the slab accumulator, fp32 FMA with the row's d
//               (read from the packed ring),
//               release of the TMEM buffer; at the end of the tile, coalesced
//               stores of y.
// TMEM (512 columns allocated, one CTA per SM): slab accumulators 2 x 128
// columns, A stages 256 columns (bf16: 2 x 128, fp8: 4 x 64).
// All waits are bounded; a timeout sets the device error word and makes every
// role stop at its next wait, so the CTA always reaches the final barrier and
// frees its TMEM.
//
// fp8 variant (FP8 = true): x rows arrive as E4M3 codes with one fp32 scale
// per row, the pattern is expanded to E4M3 +/-1 and 0 (one byte per weight,
// a 32-bit word per group), the MMA is kind::f8f6f4, and a stage covers 256
// columns (256 bytes, the same 64 TMEM columns and 32 KB x tile as a bf16
// stage of 128 columns), so a scale block is one stage instead of two.
// The row's scale multiplies the finished sum.
#pragma once

#include <cuda.h>
#include <cuda_fp8.h>

#include "device_common.cuh"
#include "packed_copy.cuh"

namespace stq1 {

constexpr int kTcM = 128;
constexpr int kTcN = 128;
constexpr int kTcAtomBytes = 128;             // one 128-byte swizzle atom of x per row
constexpr int kTcMaxBStages = 4;
constexpr int kTcMaxAStages = 4;
constexpr int kTcMaxPkStages = 4;
// Pipeline geometry: a stage is one 256-column scale block of K, i.e. four
// 128-byte atoms of bf16 x (two of E4M3).  bf16: 3 x stages of 64 KB (192
// KB), so that a stage's copy starts one stage earlier than with two (it
// takes about as long as a stage's MMAs), and a 2-stage packed-weight ring;
// fp8: 4 x stages of 32 KB and a 4-stage packed ring (its stages are half
// as long, so the packed chunks need the deeper ring).  256 TMEM columns of
// A give 2 (bf16) or 4 (fp8) A stages.
template <bool FP8>
struct TcGeom {
  static constexpr int atoms = FP8 ? 2 : 4;                  // swizzle atoms per stage
  static constexpr int b_ring_bytes = (FP8 ? 8 : 12) * kTcN * kTcAtomBytes;
  static constexpr int b_stages = b_ring_bytes / (kTcN * kTcAtomBytes * atoms);   // x-tile stages
  static constexpr int a_stages = 8 / atoms;                 // A stages in TMEM
  static constexpr int pk_stages = FP8 ? 4 : 2;              // packed-weight chunks in flight
  static constexpr int kc = kBlockWeights;                   // K per stage
  static constexpr int a_cols = 32 * atoms;                  // TMEM columns of A per stage
  static constexpr int b_stage_bytes = kTcN * kTcAtomBytes * atoms;
  static constexpr int mmas = 4 * atoms;                     // 32 bytes of K per MMA
};

constexpr int kTcThreads = 640;
constexpr int kTcMmaWarp2 = 19;                  // the second MMA issuer (odd stages)
constexpr int kTcDecoders = 256;                 // threads: 8 warps
constexpr int kTcEpilogue = 256;                 // threads: 8 warps
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcColD = 0;               // 2 x 128
constexpr uint32_t kTcColA = 256;             // stages x a_cols = 256
// shared layout (offsets from a 1024-aligned base)
constexpr int kTcOffB = 0;
// x ring then packed-weight ring (per geometry), then the rest at fixed offsets
constexpr int kTcOffTable = (12 * kTcN * kTcAtomBytes + 2 * kPackedStageMax >
                             8 * kTcN * kTcAtomBytes + 4 * kPackedStageMax)
                                ? 12 * kTcN * kTcAtomBytes + 2 * kPackedStageMax
                                : 8 * kTcN * kTcAtomBytes + 4 * kPackedStageMax;   // 2 x 128 B decode tables
static_assert(kTcOffTable % 256 == 0, "decode tables must be 256-aligned");
constexpr int kTcOffBar = kTcOffTable + 256;
constexpr int kTcOffPairs = kTcOffBar + 512;                       // kTcN ints
constexpr int kTcOffScale = kTcOffPairs + kTcN * 4;                // kTcN floats (fp8)
constexpr int kTcOffWrow = kTcOffScale + kTcN * 4;                 // kTcN ints: routing-weight index
constexpr int kTcOffMisc = kTcOffWrow + kTcN * 4;
constexpr int kTcSmemBytes = 1024 + kTcOffMisc + 64;   // > 114 KB: one CTA per SM
static_assert(kTcSmemBytes <= 232448, "shared memory per CTA is at most 227 KB");

struct TcArgs {
  PackedGeom g;              // tensor maps' view of the packed weights
  float* y;                  // [rows_out, N]
  const int* tile_info;      // [tiles, 4] expert, first B row, count, pad (nullptr: plain)
  const int* n_tiles_dev;    // device tile count (MoE) or nullptr
  const int* pairs;          // output row of each B row (MoE) or nullptr (identity)
  const int* wpairs;         // routing-weight index of each B row, or nullptr (the output row)
  const float* route_w;
  const float* xscale;       // fp8: scale of each B row, nullptr otherwise
  int n_tiles;               // plain: token tiles
  int N, K, nb;
  int n_mtiles;
  int batch;                 // plain: tokens
  int flags;
  int b_rows;                // rows of B (debug-build checks)
  int rows_out;              // rows of y (debug-build checks)
};

// ---- tcgen05 / TMA wrappers ----
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]: bf16 x bf16 (kind::f16) or E4M3 x E4M3 (kind::f8f6f4)
template <bool FP8>
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  if constexpr (FP8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

#define STQ1_TMEM_ST32(taddr, v)                                                                  \
  asm volatile(                                                                                   \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),   \
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),    \
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),          \
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),        \
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),        \
      "r"(v[29]), "r"(v[30]), "r"(v[31])                                                         \
      : "memory")

#define STQ1_TMEM_LD32(taddr, v)                                                                  \
  asm volatile(                                                                                   \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"              \
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),      \
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),  \
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),            \
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),            \
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])             \
      : "r"(taddr)                                                                                \
      : "memory")

#define STQ1_TMEM_LD16(taddr, v)                                                                  \
  asm volatile(                                                                                   \
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15}, [%16];"                                                                               \
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),      \
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),  \
        "=r"(v[14]), "=r"(v[15])                                                                   \
      : "r"(taddr)                                                                                \
      : "memory")

#define STQ1_TMEM_ST16(taddr, v)                                                                  \
  asm volatile(                                                                                   \
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14," \
      "%15,%16};" ::"r"(taddr),                                                                    \
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),    \
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),          \
      "r"(v[15])                                                                                   \
      : "memory")

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void named_bar(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), version 1 (sm_100).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor: D f32 (bits 4-5 = 1), A and B types (bits 7-9,
// 10-12: bf16 = 1 for kind::f16, E4M3 = 0 for kind::f8f6f4), both K-major,
// N >> 3 at bit 17, M >> 4 at bit 24.
template <bool FP8>
constexpr uint32_t tc_idesc(int n = kTcN) {
  return (1u << 4) | (FP8 ? 0u : ((1u << 7) | (1u << 10))) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kTcM >> 4) << 24);
}
// Tiles with at most this many pairs (tokens) run half-width: N = 64 MMAs and
// 64-row x boxes.  Accumulator columns 64..127 then keep stale values, which
// belong to no pair and are never stored.
constexpr int kTcHalfN = kTcN / 2;

// bf16 bit patterns of the 32 codes: lanes 0,1 (word 0) and lanes 2,3 (word 1);
// for fp8 one word per code, lane l in byte l (E4M3 +1 = 0x38, -1 = 0xB8).
template <bool FP8>
__device__ __forceinline__ void tc_fill_tables(uint32_t* t0, uint32_t* t1) {
  const int c = threadIdx.x;
  if (c < 32) {
    int v[4];
    code_pattern(static_cast<unsigned>(c), v);
    if constexpr (FP8) {
      uint32_t w = 0;
#pragma unroll
      for (int l = 0; l < 4; ++l) w |= (v[l] == 0 ? 0u : (v[l] > 0 ? 0x38u : 0xB8u)) << (8 * l);
      t0[c] = w;
      t1[c] = 0u;
    } else {
      uint32_t h[4];
#pragma unroll
      for (int l = 0; l < 4; ++l) h[l] = v[l] == 0 ? 0u : (v[l] > 0 ? 0x3F80u : 0xBF80u);
      t0[c] = h[0] | (h[1] << 16);
      t1[c] = h[2] | (h[3] << 16);
    }
  }
}

// Two fp32 fused multiply-adds in one instruction (the packed f32x2 FMA of
// sm_100), each lane rounded once as fmaf: {a.x * b.x + c.x, a.y * b.y + c.y}.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\t"
      "mov.b64 rb, {%4, %5};\n\t"
      "mov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
      "mov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}

// Expands this thread's half of each of the block's stages into 16 TMEM
// columns (bf16: 8 groups x 2 words of each 64-column stage; fp8: 16 groups
// x 1 word of each 128-column stage); for each stage waits for the A stage
// to be free, stores its columns and signals the MMA thread.
template <bool FP8, int HALF>
__device__ __forceinline__ bool tc_decode_slab(const uint32_t (&Q)[8], uint32_t H0, uint32_t H1,
                                               uint32_t tables, uint32_t tmem_a_lane, uint32_t bar_full_a,
                                               uint32_t bar_empty_a, uint32_t& it) {
  using G = TcGeom<FP8>;
  const uint32_t s = it % G::a_stages;
  const uint32_t use = it / G::a_stages;
  bool waited = false;
  // this half's 32 groups (qs words 4 * HALF .. 4 * HALF + 3) in pieces of 32 TMEM
  // columns: bf16 two pieces of 16 groups (2 columns each), fp8 one of 32 groups
#pragma unroll
  for (int piece = 0; piece < (FP8 ? 1 : 2); ++piece) {
    uint32_t v[32];
#pragma unroll
    for (int w = 0; w < (FP8 ? 4 : 2); ++w) {
      const int i = 4 * HALF + (FP8 ? w : 2 * piece + w);      // qs word i: groups 8i .. 8i+7
      const uint32_t hb = (i < 4 ? H0 : H1) >> (8 * (i & 3));
      const uint32_t ce = ((Q[i] << 2) & 0x3C3C3C3Cu) | (((hb & 0x55u) * 0x01041040u) & 0x40404040u);
      const uint32_t co = ((Q[i] >> 2) & 0x3C3C3C3Cu) | (((hb & 0xAAu) * 0x00820820u) & 0x40404040u);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        // the group's (code * 4) byte spliced into the 256-aligned table base
        const uint32_t ae = __byte_perm(ce, tables, 0x7650u | m);
        const uint32_t ao = __byte_perm(co, tables, 0x7650u | m);
        if constexpr (FP8) {
          uint32_t x0, y0;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(ae));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(y0) : "r"(ao));
          v[8 * w + 2 * m] = x0;
          v[8 * w + 2 * m + 1] = y0;
        } else {
          uint32_t x0, x1, y0, y1;
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(x0) : "r"(ae));
          asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(x1) : "r"(ae));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(y0) : "r"(ao));
          asm volatile("ld.shared.u32 %0, [%1+128];" : "=r"(y1) : "r"(ao));
          v[16 * w + 4 * m] = x0;
          v[16 * w + 4 * m + 1] = x1;
          v[16 * w + 4 * m + 2] = y0;
          v[16 * w + 4 * m + 3] = y1;
        }
      }
    }
    if (!waited) {
      if (!mbar_wait_bounded(bar_empty_a + 8 * s, (use & 1) ^ 1)) return false;
      tc_fence_after();
      waited = true;
    }
    STQ1_TMEM_ST32(tmem_a_lane + kTcColA + G::a_cols * s + (G::a_cols / 2) * HALF + 32 * piece, v);
  }
  tmem_wait_st();
  tc_fence_before();
  mbar_arrive(bar_full_a + 8 * s);
  ++it;
  return true;
}

template <bool FP8>
__global__ void __launch_bounds__(kTcThreads, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmap_b, const __grid_constant__ CUtensorMap tmap_bh,
               const __grid_constant__ CUtensorMap wmap,
               const __grid_constant__ CUtensorMap tmap_w, const TcArgs a) {
  using G = TcGeom<FP8>;
  constexpr int KC = G::kc;
  extern __shared__ __align__(16) uint8_t smem_raw[];   // realigned to 1024 below
  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - sraw);
  const uint32_t sB = sbase + kTcOffB;
  const uint32_t sA = sbase + G::b_ring_bytes;        // packed-weight ring
  const uint32_t sTab = sbase + kTcOffTable;
  const uint32_t bar = sbase + kTcOffBar;
  // barriers: full_b[8] @0, full_a[8] @64, empty[8] @128, d_full[2] @192, d_empty[2] @208, drain @224,
  // packed ring full[4] @256, empty[4] @288
  const uint32_t bar_full_b = bar, bar_empty_b = bar + 48;          // up to 6 each (4 used)
  const uint32_t bar_full_a = bar + 96, bar_empty_a = bar + 128;     // kTcMaxAStages each
  const uint32_t bar_d_full = bar + 160, bar_d_empty = bar + 176;
  const uint32_t bar_drain = bar + 192, bar_drain2 = bar + 200;
  const uint32_t bar_pk_full = bar + 256, bar_pk_empty = bar + 288;
  int* s_pairs = reinterpret_cast<int*>(sgen + kTcOffPairs);
  float* s_scale = reinterpret_cast<float*>(sgen + kTcOffScale);
  int* s_wrow = reinterpret_cast<int*>(sgen + kTcOffWrow);
  volatile int* s_misc = reinterpret_cast<volatile int*>(sgen + kTcOffMisc);   // [0] tmem base, [1] abort
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kTcMaxBStages; ++i) {
      mbar_init(bar_full_b + 8 * i, 1);
      mbar_init(bar_empty_b + 8 * i, 1);
    }
    for (int i = 0; i < kTcMaxAStages; ++i) {
      mbar_init(bar_full_a + 8 * i, kTcDecoders);
      mbar_init(bar_empty_a + 8 * i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_d_full + 8 * i, 1);
      mbar_init(bar_d_empty + 8 * i, kTcEpilogue);
    }
    mbar_init(bar_drain, 1);                         // drain barriers (abort path), one per MMA issuer
    mbar_init(bar_drain2, 1);
    for (int i = 0; i < kTcMaxPkStages; ++i) {
      mbar_init(bar_pk_full + 8 * i, 1);
      mbar_init(bar_pk_empty + 8 * i, kTcDecoders + kTcEpilogue);
    }
    s_misc[1] = 0;
    fence_mbar_init();
  }
  tc_fill_tables<FP8>(reinterpret_cast<uint32_t*>(sgen + kTcOffTable),
                      reinterpret_cast<uint32_t*>(sgen + kTcOffTable + 128));
  if (warp == 1) {
    tmem_alloc(sbase + kTcOffMisc, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(s_misc[0]);
  volatile int* abort = s_misc + 1;
  griddep_wait();                                    // inputs may come from the previous kernel
  griddep_launch_dependents();

  int n_tiles = a.n_tiles_dev ? *a.n_tiles_dev : a.n_tiles;
  if constexpr (kDebugBuild) {
    // every tile of the table names an expert of the buffer and B rows that
    // exist; otherwise the CTA does no work
    bool bad = a.n_tiles_dev && n_tiles > a.n_tiles;
    if (a.tile_info && !bad)
      for (int t = threadIdx.x; t < n_tiles; t += blockDim.x) {
        const int e = a.tile_info[4 * t], b = a.tile_info[4 * t + 1], c = a.tile_info[4 * t + 2];
        if (!(e >= 0 && (e + 1LL) * a.N <= a.g.rows_total && c >= 1 && c <= kTcN && b >= 0 && b + c <= a.b_rows))
          bad = true;
      }
    if (__syncthreads_or(bad)) {
      if (threadIdx.x == 0) dbg_check(false);
      n_tiles = 0;
    }
  }
  const long long n_items = static_cast<long long>(n_tiles) * a.n_mtiles;
  const int n_chunks = a.K / KC;
  const int n_slabs = a.nb;
  const int n_pk = a.nb / kChunkBlocks;              // packed chunks per tile (two slabs each)

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      for (long long item = blockIdx.x; item < n_items && !*abort; item += gridDim.x) {
        const int tile = static_cast<int>(item / a.n_mtiles);
        const int b_row = a.tile_info ? a.tile_info[4 * tile + 1] : tile * kTcN;
        const int cnt = a.tile_info ? a.tile_info[4 * tile + 2] : min(kTcN, a.batch - tile * kTcN);
        const bool half_n = cnt <= kTcHalfN;
        for (int kc = 0; kc < n_chunks; ++kc, ++it) {
          const uint32_t s = it % G::b_stages, use = it / G::b_stages;
          if (!mbar_wait_bounded(bar_empty_b + 8 * s, (use & 1) ^ 1)) { *abort = 1; break; }
          mbar_arrive_expect_tx(bar_full_b + 8 * s, half_n ? G::b_stage_bytes / 2 : G::b_stage_bytes);
          // one 3-D copy per stage: (column in atom, row, atom); the atoms land
          // one after another, 16 KB apart (8 KB for a half-height box)
          tma_load_3d(sB + s * G::b_stage_bytes, half_n ? &tmap_bh : &tmap_b, 0, b_row, kc * G::atoms,
                      bar_full_b + 8 * s);
        }
      }
      if (*abort) {
        // let the last tensor copies land before the CTA can exit (bounded)
        for (uint32_t j = it > G::b_stages ? it - G::b_stages : 0; j < it; ++j)
          mbar_wait_bounded(bar_full_b + 8 * (j % G::b_stages), (j / G::b_stages) & 1);
      }
    }
  } else if (warp == 1 || warp == kTcMmaWarp2) {
    // ---------------- MMA issuers ----------------
    // Two threads take alternate stages (warp 1 the even ones, the second
    // issuer warp the odd ones): an issuing thread blocks while the tensor
    // pipe works through the MMAs it has queued, so one issuer alone leaves
    // the pipe idle while it waits for the next stage's operands; with two,
    // one waits while the other's MMAs run.  Each stage has its own
    // accumulator buffer, A and B stage, and its commits track the MMAs of
    // the thread that issued them.
    if (lane == 0) {
      const uint32_t mine = warp == 1 ? 0u : 1u;
      const uint32_t drain = warp == 1 ? bar_drain : bar_drain2;
      uint32_t it = 0;
      for (long long item = blockIdx.x; item < n_items && !*abort; item += gridDim.x) {
        const int tile = static_cast<int>(item / a.n_mtiles);
        const int cnt = a.tile_info ? a.tile_info[4 * tile + 2] : min(kTcN, a.batch - tile * kTcN);
        const bool half_n = cnt <= kTcHalfN;
        const uint32_t idesc = half_n ? tc_idesc<FP8>(kTcHalfN) : tc_idesc<FP8>();
        // a half-height 3-D copy lands its atoms 8 KB apart instead of 16 KB
        const uint32_t atom_bytes = (half_n ? kTcHalfN : kTcN) * kTcAtomBytes;
        for (int slab = 0; slab < n_slabs && !*abort; ++slab, ++it) {
          if ((it & 1u) != mine) continue;
          const uint32_t p = it & 1, puse = it >> 1;
          if (!mbar_wait_bounded(bar_d_empty + 8 * p, (puse & 1) ^ 1)) { *abort = 1; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem + kTcColD + p * kTcN;
          const uint32_t sb = it % G::b_stages, ub = it / G::b_stages;
          const uint32_t sa = it % G::a_stages, ua = it / G::a_stages;
          if (!mbar_wait_bounded(bar_full_b + 8 * sb, ub & 1) ||
              !mbar_wait_bounded(bar_full_a + 8 * sa, ua & 1)) { *abort = 1; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < G::mmas; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(sB + sb * G::b_stage_bytes + (kk >> 2) * atom_bytes) + 2 * (kk & 3);
            tc_mma_ts<FP8>(d_tmem, tmem + kTcColA + G::a_cols * sa + 8 * kk, bdesc, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar_empty_b + 8 * sb);
          tc_commit(bar_empty_a + 8 * sa);
          tc_commit(bar_d_full + 8 * p);
        }
      }
      if (*abort) {
        // all MMAs this thread issued must finish before TMEM is freed (bounded)
        tc_commit(drain);
        mbar_wait_bounded(drain, 0);
      }
    }
  } else if (warp < 10) {
    // ---------------- decoders ----------------
    const int half = (warp - 2) >> 2;               // which half of each stage's groups
    const int quad = warp & 3;                       // TMEM lane quadrant of this warp
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    uint32_t it = 0, ca = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < n_items && ok && !*abort; item += gridDim.x) {
      const int tile = static_cast<int>(item / a.n_mtiles);
      const int mt = static_cast<int>(item - static_cast<long long>(tile) * a.n_mtiles);
      const int e = a.tile_info ? a.tile_info[4 * tile + 0] : 0;
      const long long R0 = static_cast<long long>(e) * a.N + static_cast<long long>(mt) * kTcM;
      // TMEM lane 32 * quad + lane holds the row of slot 32 * quad + lane of the ring
      const PackedRow pr = packed_row(a.g, R0, 32 * quad + lane);
      const bool row_ok = mt * kTcM + pr.rho < a.N;   // rows past N decode zeros: computed, never stored
      for (int c = 0; c < n_pk; ++c, ++ca) {
        const uint32_t sa = ca % G::pk_stages, ause = ca / G::pk_stages;
        if (!mbar_wait_bounded(bar_pk_full + 8 * sa, ause & 1)) { *abort = 1; ok = false; break; }
        BlockCodes b0 = {}, b1 = {};
        if (row_ok) {
          const uint32_t slot = sA + sa * kPackedStageMax + pr.slot;
          const int o = packed_window_offset(a.g, pr.res, c);
          load_chunk_block(slot, o, 0, b0);
          load_chunk_block(slot, o, 1, b1);
        }
        mbar_arrive(bar_pk_empty + 8 * sa);          // the codes are in registers now
        const bool okd =
            (half == 0 ? tc_decode_slab<FP8, 0>(b0.Q, b0.H0, b0.H1, sTab, tmem_lane, bar_full_a, bar_empty_a, it)
                       : tc_decode_slab<FP8, 1>(b0.Q, b0.H0, b0.H1, sTab, tmem_lane, bar_full_a, bar_empty_a, it)) &&
            (half == 0 ? tc_decode_slab<FP8, 0>(b1.Q, b1.H0, b1.H1, sTab, tmem_lane, bar_full_a, bar_empty_a, it)
                       : tc_decode_slab<FP8, 1>(b1.Q, b1.H0, b1.H1, sTab, tmem_lane, bar_full_a, bar_empty_a, it));
        if (!okd) {
          *abort = 1;
          ok = false;
          break;
        }
      }
    }
  } else if (warp < 18) {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;
    const int chalf = (warp - 10) >> 2;              // token columns [64 * chalf, 64 * chalf + 64)
    const uint32_t tmem_lane = tmem + (static_cast<uint32_t>(32 * quad) << 16);
    const int et = threadIdx.x - 320;                // 0..255
    constexpr int kCols = kTcN / 2;
    uint32_t sc = 0, ca = 0;
    for (long long item = blockIdx.x; item < n_items && !*abort; item += gridDim.x) {
      const int tile = static_cast<int>(item / a.n_mtiles);
      const int mt = static_cast<int>(item - static_cast<long long>(tile) * a.n_mtiles);
      const int e = a.tile_info ? a.tile_info[4 * tile + 0] : 0;
      const int b_row = a.tile_info ? a.tile_info[4 * tile + 1] : tile * kTcN;
      const int cnt = a.tile_info ? a.tile_info[4 * tile + 2] : min(kTcN, a.batch - tile * kTcN);
      named_bar(1, kTcEpilogue);                     // previous tile's stores are done
      if (et < kTcN) {
        s_pairs[et] = et < cnt ? (a.pairs ? a.pairs[b_row + et] : b_row + et) : -1;
        s_wrow[et] = et < cnt ? (a.wpairs ? a.wpairs[b_row + et] : s_pairs[et]) : 0;
        // (debug build: a row whose output or routing-weight index is out of range is not stored)
        if (et < cnt && !dbg_check(s_pairs[et] >= 0 && s_pairs[et] < a.rows_out && s_wrow[et] >= 0 &&
                                   s_wrow[et] < a.rows_out))
          s_pairs[et] = -1;
        if constexpr (FP8) s_scale[et] = et < cnt ? a.xscale[b_row + et] : 0.f;
      }
      named_bar(1, kTcEpilogue);
      const long long R0 = static_cast<long long>(e) * a.N + static_cast<long long>(mt) * kTcM;
      const PackedRow pr = packed_row(a.g, R0, 32 * quad + lane);
      const int row = mt * kTcM + pr.rho;
      const bool row_ok = row < a.N;
      float acc[kCols];
#pragma unroll
      for (int j = 0; j < kCols; ++j) acc[j] = 0.f;
      bool ok = true;
      float dpair[2] = {0.f, 0.f};
      for (int slab = 0; slab < n_slabs; ++slab, ++sc) {
        if ((slab & 1) == 0) {
          // the scales of this chunk's two blocks, then release the ring stage
          const uint32_t sa = ca % G::pk_stages, ause = ca / G::pk_stages;
          if (!mbar_wait_bounded(bar_pk_full + 8 * sa, ause & 1)) { *abort = 1; ok = false; break; }
          if (row_ok) {
            const uint32_t w0 = sA + sa * kPackedStageMax + pr.slot +
                                static_cast<uint32_t>(packed_window_offset(a.g, pr.res, slab >> 1));
            unsigned short h0, h1;
            asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h0) : "r"(w0));
            asm volatile("ld.shared.u16 %0, [%1+42];" : "=h"(h1) : "r"(w0));
            dpair[0] = __half2float(__ushort_as_half(h0));
            dpair[1] = __half2float(__ushort_as_half(h1));
          }
          mbar_arrive(bar_pk_empty + 8 * sa);
          ++ca;
        }
        const float d = dpair[slab & 1];
        const uint32_t p = sc & 1, puse = sc >> 1;
        if (!mbar_wait_bounded(bar_d_full + 8 * p, puse & 1)) { *abort = 1; ok = false; break; }
        tc_fence_after();
        if (chalf == 0 || cnt > kTcHalfN) {           // warp-uniform: a half-width tile has no upper columns
#pragma unroll
          for (int c = 0; c < kCols / 16; ++c) {
            uint32_t v[16];
            STQ1_TMEM_LD16(tmem_lane + kTcColD + p * kTcN + kCols * chalf + 16 * c, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; i += 2) {         // two columns per packed fp32x2 FMA
              const float2 r = ffma2(make_float2(d, d), make_float2(__uint_as_float(v[i]), __uint_as_float(v[i + 1])),
                                     make_float2(acc[16 * c + i], acc[16 * c + i + 1]));
              acc[16 * c + i] = r.x;
              acc[16 * c + i + 1] = r.y;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar_d_empty + 8 * p);
      }
      if (!ok) break;
      if (row_ok) {
        const bool up = (a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2;
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
          const int pair = s_pairs[kCols * chalf + j];
          if (pair >= 0) {
            float v = acc[j];
            if constexpr (FP8) v *= s_scale[kCols * chalf + j];
            if (up) v *= a.route_w[s_wrow[kCols * chalf + j]];
            a.y[static_cast<long long>(pair) * a.N + row] = v;
          }
        }
      }
    }
  } else {
    // ---------------- TMA producer of the packed weights (warp 18) ----------------
    if (lane == 0) {
      uint32_t ca = 0;
      for (long long item = blockIdx.x; item < n_items && !*abort; item += gridDim.x) {
        const int tile = static_cast<int>(item / a.n_mtiles);
        const int mt = static_cast<int>(item - static_cast<long long>(tile) * a.n_mtiles);
        const int e = a.tile_info ? a.tile_info[4 * tile + 0] : 0;
        const long long R0 = static_cast<long long>(e) * a.N + static_cast<long long>(mt) * kTcM;
        for (int c = 0; c < n_pk; ++c, ++ca) {
          const uint32_t sa = ca % G::pk_stages, ause = ca / G::pk_stages;
          if (!mbar_wait_bounded(bar_pk_empty + 8 * sa, (ause & 1) ^ 1)) { *abort = 1; break; }
          packed_issue_chunk(a.g, &wmap, &tmap_w, R0, c, sA + sa * kPackedStageMax, bar_pk_full + 8 * sa);
        }
      }
      if (*abort) {
        // let the last chunk copies land before the CTA can exit (bounded)
        for (uint32_t j = ca > G::pk_stages ? ca - G::pk_stages : 0; j < ca; ++j)
          mbar_wait_bounded(bar_pk_full + 8 * (j % G::pk_stages), (j / G::pk_stages) & 1);
      }
    }
  }

  // all roles meet here (every wait above is bounded)
  tc_fence_before();
  __syncthreads();
  if (*abort && threadIdx.x == 0) flag_error(STQ1_DEV_WAIT_LIMIT);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

// x rows gathered into expert order for the tile path's TMA tiles.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint16_t* __restrict__ x, const int* __restrict__ pairs, const int* __restrict__ n_valid,
                   int n_rows, int topk, int K, uint16_t* __restrict__ out) {
  const int r = blockIdx.x;
  griddep_wait();
  griddep_launch_dependents();
  if (r >= n_rows) return;
  const int nv = n_valid ? *n_valid : n_rows;
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<long long>(r) * K);
  // (debug build: a pair id outside the list's range gives a zero row)
  if (r >= nv || !dbg_check(pairs[r] >= 0 && pairs[r] < n_rows)) {
    for (int i = threadIdx.x; i < K / 8; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
    return;
  }
  const int tok = pairs[r] / topk;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(tok) * K);
  for (int i = threadIdx.x; i < K / 8; i += blockDim.x) dst[i] = src[i];
}

// E4M3 codes of x rows with one fp32 scale per row (fp8 variant): inv = 448 /
// amax and s = amax / 448 (IEEE divisions; 0 for an all-zero row), code =
// round-to-nearest-even, saturating, of the fp32 product x * inv.
constexpr int kQuantThreads = 256;
__global__ void __launch_bounds__(kQuantThreads)
quant_e4m3_kernel(const uint16_t* __restrict__ x, int K, uint8_t* __restrict__ q, float* __restrict__ s) {
  __shared__ float s_red[kQuantThreads / 32];
  const long long r = blockIdx.x;
  griddep_wait();
  griddep_launch_dependents();
  const uint16_t* xr = x + r * K;
  float m = 0.f;
  for (int i = threadIdx.x; i < K / 8; i += kQuantThreads) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j)
      m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_f32(w[j] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[j] >> 16))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kQuantThreads / 32; ++i) amax = fmaxf(amax, s_red[i]);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
  if (threadIdx.x == 0) s[r] = __fdiv_rn(amax, 448.f);
  uint8_t* qr = q + r * K;
  for (int i = threadIdx.x; i < K / 8; i += kQuantThreads) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(xr) + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t lo = __nv_cvt_float_to_fp8(__fmul_rn(bf16_bits_to_f32(w[j] & 0xFFFFu), inv), __NV_SATFINITE, __NV_E4M3);
      const uint32_t hi = __nv_cvt_float_to_fp8(__fmul_rn(bf16_bits_to_f32(w[j] >> 16), inv), __NV_SATFINITE, __NV_E4M3);
      o[j >> 1] |= (lo | (hi << 8)) << (16 * (j & 1));
    }
    reinterpret_cast<uint2*>(qr)[i] = make_uint2(o[0], o[1]);
  }
}

// E4M3 rows and their scales gathered into expert order (fp8 variant).
__global__ void __launch_bounds__(256)
gather_rows8_kernel(const uint8_t* __restrict__ q, const float* __restrict__ s, const int* __restrict__ pairs,
                    const int* __restrict__ n_valid, int n_rows, int topk, int K, uint8_t* __restrict__ out,
                    float* __restrict__ s_out) {
  const int r = blockIdx.x;
  griddep_wait();
  griddep_launch_dependents();
  if (r >= n_rows) return;
  const int nv = n_valid ? *n_valid : n_rows;
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<long long>(r) * K);
  if (r >= nv || !dbg_check(pairs[r] >= 0 && pairs[r] < n_rows)) {
    for (int i = threadIdx.x; i < K / 16; i += blockDim.x) dst[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) s_out[r] = 0.f;
    return;
  }
  const int tok = pairs[r] / topk;
  const uint4* src = reinterpret_cast<const uint4*>(q + static_cast<long long>(tok) * K);
  for (int i = threadIdx.x; i < K / 16; i += blockDim.x) dst[i] = src[i];
  if (threadIdx.x == 0) s_out[r] = s[tok];
}

}  // namespace stq1
