// Decode GEMV for STQ1_0 through per-group lookup tables (CUDA cores, sm_100a).
//
// y[t, j] = sum_k W^[j, k] x[t, k] where every group of four weights is one of
// 32 patterns in {-d, 0, +d} with exactly one zero (lemmy.durstig.online post
// 66506, "Four weights, five bits").  For a group of four activations the 32
// possible partial sums sum_l pattern_c[l] * x[l] are tabulated once per CTA in
// shared memory; a weight group then costs one table load and one add, with no
// multiplies on the weight side.  The scale d multiplies each 256-weight block
// sum once (fp32 FMA).
//
// Work unit = (token tile, 128-row slab, K split).  One lane owns one weight row,
// so all 32 lanes of a warp read the same group's table at the same time and
// the 32 distinct codes hit 32 distinct banks.  Weight rows are streamed in
// chunks of two blocks (512 columns, 84 bytes per row) by 1-D bulk copies into
// a two-stage shared-memory ring; one copy per row fetches the 16-byte-aligned
// superset of the row's 84 bytes.  Rows are assigned to lanes so that the
// copied span starts at the same offset (mod 16) for every lane of a warp,
// which lets each warp decode with compile-time byte offsets and
// conflict-free 16-byte shared loads.
//
// Split K: with few rows the K range is divided into S contiguous pieces.  The
// S units of a (tile, slab) normally form one thread-block cluster: each keeps
// its partial sums in its own shared memory and, after a cluster barrier, each
// adds a slice of the rows from all S peers (distributed shared memory) in
// order 0..S-1 and writes y.  Without clusters (a caller-provided scratch
// buffer instead), each unit stores its partials in global memory and the last
// unit to finish adds them in the same order.  Both are deterministic.
#pragma once

#include <utility>

#include "device_common.cuh"

namespace stq1 {

constexpr int kLutRows = 128;                 // rows per unit = threads per CTA
constexpr int kLutThreads = 128;
constexpr int kLutKC = 2;                     // blocks per chunk
constexpr int kLutChunkGroups = kGroupsPerBlock * kLutKC;    // 128
constexpr int kLutGroupBytes = 144;           // 32 fp32 entries + 16-byte pad
constexpr int kLutTokenBytes = kLutChunkGroups * kLutGroupBytes;   // 18432 = 72 * 256
constexpr int kLutSlotBytes = 112;            // 84-byte span + alignment slack, 7 x 16 B
constexpr int kLutStageBytes = kLutRows * kLutSlotBytes;     // 14336
constexpr int kLutMaxTT = 4;                  // tokens per tile

struct LutArgs {
  const uint8_t* W;          // matrix, or expert 0 of a contiguous expert array
  const uint8_t* W_end;      // one past the last byte of the packed buffer
  long long expert_bytes;    // bytes per expert matrix (N * rowbytes)
  long long rowbytes;        // K / 256 * 42
  const uint16_t* x;         // [T, K] bf16 bits
  float* y;                  // [rows_out, N]
  float* partial;            // [S, rows_out, N] (S > 1)
  int* counters;             // [n_tiles, n_slabs] (S > 1), zero between calls
  const int* tile_info;      // MoE: [n_tiles_max, 4] = expert, pair offset, count, pad
  const int* n_tiles_dev;    // MoE: number of valid tiles
  const int* pairs;          // MoE: pair ids grouped by expert
  const float* route_w;      // [rows_out] routing weight per pair (flag WEIGHT_UP)
  int N, K, nb;
  int topk;                  // pairs per token (1 for a plain GEMV)
  int batch;                 // plain GEMV: tokens
  int rows_out;              // rows of y
  int n_tiles;               // tiles in the grid
  int n_slabs;
  int S;
  int n_chunks;
  int P;                     // rows per residue class of (row * rowbytes) mod 16
  int flags;
  int cluster;               // 1: the S splits of a (tile, slab) form one thread-block cluster
};

__device__ __forceinline__ uint32_t win_word(const uint32_t* w, int p) {
  // p is a compile-time constant after unrolling
  return (p & 3) ? __funnelshift_r(w[p >> 2], w[(p >> 2) + 1], 8 * (p & 3)) : w[p >> 2];
}

// Spread bits 0, 2, 4, 6 of x to bit 6 of bytes 0..3 (other bits cleared).
__device__ __forceinline__ uint32_t spread_even_bits(uint32_t x) {
  return ((x & 0x55u) * 0x01041040u) & 0x40404040u;
}

__device__ __forceinline__ float lds_f32_addr(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// Code words of one block, extracted from a 16-byte-aligned register window:
// d (fp32), qs as 8 little-endian words, qh as 2 words.
struct BlockCodes {
  float d;
  uint32_t Q[8];
  uint32_t H0, H1;
};

// Loads the block starting at byte B0 of a slot (B0 compile-time) with 16-byte
// shared loads and extracts its fields.
template <int B0>
__device__ __forceinline__ void load_block_codes(uint32_t slot, BlockCodes& bc) {
  constexpr int C0 = B0 >> 4;
  constexpr int C1 = (B0 + kBlockBytes - 1) >> 4;
  uint32_t w[16];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    if (C0 + c <= C1) {
      const uint4 v = lds_v4(slot + 16u * (C0 + c));
      w[4 * c + 0] = v.x;
      w[4 * c + 1] = v.y;
      w[4 * c + 2] = v.z;
      w[4 * c + 3] = v.w;
    } else {
      w[4 * c + 0] = w[4 * c + 1] = w[4 * c + 2] = w[4 * c + 3] = 0u;
    }
  }
  constexpr int base = B0 - 16 * C0;                // even
  const uint32_t dword = w[base >> 2] >> (8 * (base & 3));
  bc.d = __half2float(__ushort_as_half(static_cast<unsigned short>(dword & 0xFFFFu)));
  bc.H0 = win_word(w, base + kOffQh);
  bc.H1 = win_word(w, base + kOffQh + 4);
#pragma unroll
  for (int i = 0; i < 8; ++i) bc.Q[i] = win_word(w, base + kOffQs + 4 * i);
}

// Compile-time loop helper.
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

// Table lookups of one block's 64 groups for TT tokens; `lut` is the 256-aligned
// base of this block's tables, every offset below it is an immediate of the
// shared load, and the group's code byte is spliced into the base with one
// byte permute.
template <int TT>
__device__ __forceinline__ void lut_block_body(const BlockCodes& bc, uint32_t lut, float (&acc)[kLutMaxTT]) {
  float s[TT][4];
#pragma unroll
  for (int t = 0; t < TT; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
  static_for<8>([&](auto IC) {                       // qs word i: groups 8i .. 8i+7
    constexpr int i = decltype(IC)::value;
    const uint32_t Q = bc.Q[i];
    const uint32_t hb = (i < 4 ? bc.H0 : bc.H1) >> (8 * (i & 3));
    // table byte offsets (t << 6 | n << 2) of the 4 even / 4 odd groups
    const uint32_t ce = ((Q << 2) & 0x3C3C3C3Cu) | (((hb & 0x55u) * 0x01041040u) & 0x40404040u);
    const uint32_t co = ((Q >> 2) & 0x3C3C3C3Cu) | (((hb & 0xAAu) * 0x00820820u) & 0x40404040u);
    static_for<4>([&](auto MC) {
      constexpr int m = decltype(MC)::value;
      constexpr int ge = 8 * i + 2 * m;              // even group's index in the block
      const uint32_t ae = __byte_perm(ce, lut, 0x7650u | m);
      const uint32_t ao = __byte_perm(co, lut, 0x7650u | m);
      s[0][m] += lds_f32<ge * kLutGroupBytes>(ae) + lds_f32<(ge + 1) * kLutGroupBytes>(ao);
      if constexpr (TT > 1)
        s[1][m] += lds_f32<kLutTokenBytes + ge * kLutGroupBytes>(ae) +
                   lds_f32<kLutTokenBytes + (ge + 1) * kLutGroupBytes>(ao);
      if constexpr (TT > 2)
        s[2][m] += lds_f32<2 * kLutTokenBytes + ge * kLutGroupBytes>(ae) +
                   lds_f32<2 * kLutTokenBytes + (ge + 1) * kLutGroupBytes>(ao);
      if constexpr (TT > 3)
        s[3][m] += lds_f32<3 * kLutTokenBytes + ge * kLutGroupBytes>(ae) +
                   lds_f32<3 * kLutTokenBytes + (ge + 1) * kLutGroupBytes>(ao);
    });
  });
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = fmaf(bc.d, (s[t][0] + s[t][1]) + (s[t][2] + s[t][3]), acc[t]);
}

// Activations of this thread's group for chunk `chunk`, TT tokens (8 bytes each).
template <int TT>
__device__ __forceinline__ void lut_load_x(const LutArgs& a, int chunk, const int* xrow, uint2 (&xv)[kLutMaxTT]) {
  const int col = chunk * (kLutKC * kBlockWeights) + 4 * static_cast<int>(threadIdx.x);
#pragma unroll
  for (int t = 0; t < TT; ++t)
    xv[t] = __ldg(reinterpret_cast<const uint2*>(a.x + static_cast<long long>(xrow[t]) * a.K + col));
}

// Tables for one chunk: thread g builds the 32 entries of group g for each token.
// Entry c (code) = (-1)^t * (x_a + (-1)^beta x_b + (-1)^gamma x_c).
template <int TT>
__device__ __forceinline__ void lut_build(const uint2 (&xv)[kLutMaxTT], uint32_t lut) {
  const int g = threadIdx.x;                       // 0 .. 127 = kLutChunkGroups - 1
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    const float x0 = bf16_bits_to_f32(xv[t].x & 0xFFFFu), x1 = bf16_bits_to_f32(xv[t].x >> 16);
    const float x2 = bf16_bits_to_f32(xv[t].y & 0xFFFFu), x3 = bf16_bits_to_f32(xv[t].y >> 16);
    const uint32_t gb = lut + static_cast<uint32_t>(t * kLutTokenBytes + g * kLutGroupBytes);
    // z = 0: a=1 b=2 c=3 ; z = 1: a=0 b=2 c=3 ; z = 2: a=0 b=1 c=3 ; z = 3: a=0 b=1 c=2
    auto put = [&](int z, float xa, float xb, float xc) {
      const float p = xa + xb, q = xa - xb;
      const float e0 = p + xc, e1 = p - xc, e2 = q + xc, e3 = q - xc;
      sts_v4f(gb + 16u * z, e0, e1, e2, e3);
      sts_v4f(gb + 64u + 16u * z, -e0, -e1, -e2, -e3);
    };
    put(0, x1, x2, x3);
    put(1, x0, x2, x3);
    put(2, x0, x1, x3);
    put(3, x0, x1, x2);
  }
}

// One work unit with TT tokens.
template <int TT>
__device__ void lut_unit(const LutArgs& a, const uint8_t* Wm, int slab, int split, int tile_id,
                         const int* xrow, const int* orow, uint8_t* smem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rg = warp;                                           // 32-row group
  const int P = a.P;
  const int rho = P * lane + (rg % P) + 32 * P * (rg / P);       // row within the slab
  const long long row = static_cast<long long>(slab) * kLutRows + rho;
  const bool row_ok = row < a.N;
  const int c0 = static_cast<int>(static_cast<long long>(split) * a.n_chunks / a.S);
  const int c1 = static_cast<int>(static_cast<long long>(split + 1) * a.n_chunks / a.S);

  const uint32_t sbase = smem_u32(smem);
  const uint32_t lut = (sbase + 255u) & ~255u;
  const uint32_t bar0 = lut + TT * kLutTokenBytes;   // 2 mbarriers, then the stages
  const uint32_t stage0 = bar0 + 16;
  const uint32_t my_slot_off = static_cast<uint32_t>(rg * 32 + lane) * kLutSlotBytes;

  if (threadIdx.x == 0) {
    mbar_init(bar0, kLutThreads);
    mbar_init(bar0 + 8, kLutThreads);
    fence_mbar_init();
  }
  __syncthreads();

  // Bulk copy of this lane's row span for chunk c into stage st.
  auto issue = [&](int c, int st) {
    const uint32_t bar = bar0 + 8u * st;
    if (!row_ok) {
      mbar_arrive(bar);
      return;
    }
    const uint8_t* A = Wm + row * a.rowbytes + static_cast<long long>(c) * (kLutKC * kBlockBytes);
    const uintptr_t lo = reinterpret_cast<uintptr_t>(A) & ~static_cast<uintptr_t>(15);
    uintptr_t hi = (reinterpret_cast<uintptr_t>(A) + kLutKC * kBlockBytes + 15) & ~static_cast<uintptr_t>(15);
    const uintptr_t end = reinterpret_cast<uintptr_t>(a.W_end);
    const uint32_t dst = stage0 + st * kLutStageBytes + my_slot_off;
    if (hi > end) {
      // the last row of an unaligned buffer: bulk-copy the aligned part, plain-copy the tail
      const uintptr_t end16 = end & ~static_cast<uintptr_t>(15);
      for (uintptr_t q = end16; q < end; ++q) {
        const uint8_t v = *reinterpret_cast<const uint8_t*>(q);
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(dst + static_cast<uint32_t>(q - lo)), "r"(static_cast<uint32_t>(v)) : "memory");
      }
      hi = end16;
    }
    const uint32_t bytes = static_cast<uint32_t>(hi - lo);
    mbar_arrive_expect_tx(bar, bytes);
    if (bytes) bulk_g2s(dst, reinterpret_cast<const void*>(lo), bytes, bar);
  };

  float acc[kLutMaxTT];
#pragma unroll
  for (int t = 0; t < kLutMaxTT; ++t) acc[t] = 0.f;

  // offset of the warp's spans inside their 16-byte slots (same for every lane)
  const long long row0 = static_cast<long long>(slab) * kLutRows + (rg % P) + 32 * P * (rg / P);
  const uintptr_t wbase = reinterpret_cast<uintptr_t>(Wm) + static_cast<uintptr_t>(row0 * a.rowbytes);

  // Weights do not depend on the previous kernel in the stream: start their
  // copies before waiting for it (programmatic dependent launch), unless the
  // unit itself came from a routing kernel.
  if (a.tile_info == nullptr) {
    if (c0 < c1) issue(c0, 0);
    if (c0 + 1 < c1) issue(c0 + 1, 1);
  }
  griddep_wait();
  if (a.tile_info != nullptr) {
    if (c0 < c1) issue(c0, 0);
    if (c0 + 1 < c1) issue(c0 + 1, 1);
  }
  griddep_launch_dependents();
  uint2 xv[kLutMaxTT];
  if (c0 < c1) lut_load_x<TT>(a, c0, xrow, xv);
  bool failed = false;
  for (int c = c0; c < c1; ++c) {
    const int it = c - c0;
    const int st = it & 1;
    lut_build<TT>(xv, lut);
    if (c + 1 < c1) lut_load_x<TT>(a, c + 1, xrow, xv);   // prefetch the next chunk's activations
    const bool landed = mbar_wait_bounded(bar0 + 8u * st, (it >> 1) & 1);
    // one barrier: tables built, copies landed (agreed by every thread)
    if (!__syncthreads_and(landed)) {
      // A copy did not complete within the bound (the error word is set).
      // Wait (bounded) for the copy already issued into the other stage, so no
      // bulk copy is still writing this CTA's shared memory when it exits.
      if (c + 1 < c1) mbar_wait_bounded(bar0 + 8u * (st ^ 1), ((it + 1) >> 1) & 1);
      failed = true;
      break;
    }
    if (row_ok) {
      const uint32_t slot = stage0 + st * kLutStageBytes + my_slot_off;
      const int o = static_cast<int>((wbase + static_cast<uintptr_t>(c) * (kLutKC * kBlockBytes)) & 15);
      // only the extraction depends on the warp's offset; one copy of the body follows
      BlockCodes b0, b1;
      switch (o) {
        case 0: load_block_codes<0>(slot, b0); load_block_codes<0 + kBlockBytes>(slot, b1); break;
        case 4: load_block_codes<4>(slot, b0); load_block_codes<4 + kBlockBytes>(slot, b1); break;
        case 8: load_block_codes<8>(slot, b0); load_block_codes<8 + kBlockBytes>(slot, b1); break;
        default: load_block_codes<12>(slot, b0); load_block_codes<12 + kBlockBytes>(slot, b1); break;
      }
      // the second block's tables start 64 groups into the chunk's (256-aligned)
      lut_block_body<TT>(b0, lut, acc);
      lut_block_body<TT>(b1, lut + static_cast<uint32_t>(kGroupsPerBlock * kLutGroupBytes), acc);
    }
    __syncthreads();
    if (c + 2 < c1) issue(c + 2, st);                      // this stage is free again
  }
  const bool up = (a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2;
  if (a.S == 1) {
    if (row_ok && !failed) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float v = acc[t];
        if (up) v *= a.route_w[orow[t]];
        a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
      }
    }
    return;
  }

  if (a.cluster) {
    // Every CTA of the cluster reaches both cluster barriers, failed or not.
    const uint32_t red = lut;                          // tables are no longer needed
#pragma unroll
    for (int t = 0; t < TT; ++t)
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(red + 4u * (t * kLutRows + rho)), "f"(acc[t]) : "memory");
    cluster_sync_all();
    const int rank = static_cast<int>(cluster_ctarank());
    const int lo = rank * kLutRows / a.S, hi = (rank + 1) * kLutRows / a.S;
    const int nr = hi - lo;
    for (int idx = threadIdx.x; idx < nr * TT; idx += kLutThreads) {
      const int t = idx / nr, rr = lo + idx % nr;
      float v = 0.f;
      for (int sp = 0; sp < a.S; ++sp) v += ld_peer_f32(red + 4u * (t * kLutRows + rr), sp);
      const long long rrow = static_cast<long long>(slab) * kLutRows + rr;
      if (rrow < a.N) {
        if ((a.flags & STQ1_MOE_WEIGHT_UP) && rrow >= a.N / 2) v *= a.route_w[orow[t]];
        a.y[static_cast<long long>(orow[t]) * a.N + rrow] = v;
      }
    }
    cluster_sync_all();                                // peers may still read this CTA's partials
    return;
  }
  if (failed) return;

  // Scratch mode: publish partials, the last unit of this (tile, slab) reduces.
  // One thread fences after the barrier: the barrier orders the other threads'
  // stores before it, and the gpu-scope fence is cumulative.
  if (row_ok) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
      a.partial[(static_cast<long long>(split) * a.rows_out + orow[t]) * a.N + row] = acc[t];
  }
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(&a.counters[tile_id * a.n_slabs + slab], 1);
    s_last = (old == a.S - 1);
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  if (row_ok) {
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      float v = 0.f;
      for (int sp = 0; sp < a.S; ++sp)
        v += __ldcg(&a.partial[(static_cast<long long>(sp) * a.rows_out + orow[t]) * a.N + row]);
      if (up) v *= a.route_w[orow[t]];
      a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
    }
  }
  if (threadIdx.x == 0) a.counters[tile_id * a.n_slabs + slab] = 0;
}

template <int TTMAX>
__global__ void __launch_bounds__(kLutThreads) lut_gemv_kernel(const LutArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_xrow[kLutMaxTT], s_orow[kLutMaxTT], s_cnt, s_expert;
  const int u = blockIdx.x;
  const int split = u % a.S;
  const int rest = u / a.S;
  const int slab = rest % a.n_slabs;
  const int tile = rest / a.n_slabs;
  if (a.tile_info) {
    griddep_wait();                                  // the tile table comes from the routing kernel
    if (tile >= *a.n_tiles_dev) return;
    if (threadIdx.x == 0) {
      const int e = a.tile_info[4 * tile + 0];
      const int off = a.tile_info[4 * tile + 1];
      const int cnt = a.tile_info[4 * tile + 2];
      s_expert = e;
      s_cnt = cnt;
      for (int t = 0; t < kLutMaxTT; ++t) {
        const int p = a.pairs[off + (t < cnt ? t : 0)];
        s_orow[t] = p;
        s_xrow[t] = p / a.topk;
      }
    }
  } else {
    if (threadIdx.x == 0) {
      const int t0 = tile * kLutMaxTT;
      const int cnt = min(kLutMaxTT, a.batch - t0);
      s_expert = 0;
      s_cnt = cnt;
      for (int t = 0; t < kLutMaxTT; ++t) {
        s_orow[t] = t0 + (t < cnt ? t : 0);
        s_xrow[t] = s_orow[t];
      }
    }
  }
  __syncthreads();
  const uint8_t* Wm = a.W + static_cast<long long>(s_expert) * a.expert_bytes;
  const int cnt = s_cnt;
  if (TTMAX >= 4 && cnt >= 4) {
    lut_unit<(TTMAX >= 4 ? 4 : 1)>(a, Wm, slab, split, tile, s_xrow, s_orow, smem);
  } else if (TTMAX >= 3 && cnt == 3) {
    lut_unit<(TTMAX >= 3 ? 3 : 1)>(a, Wm, slab, split, tile, s_xrow, s_orow, smem);
  } else if (TTMAX >= 2 && cnt == 2) {
    lut_unit<(TTMAX >= 2 ? 2 : 1)>(a, Wm, slab, split, tile, s_xrow, s_orow, smem);
  } else {
    lut_unit<1>(a, Wm, slab, split, tile, s_xrow, s_orow, smem);
  }
}

inline size_t lut_smem_bytes(int ttmax, int stages = 2) {
  return 256 + static_cast<size_t>(ttmax) * kLutTokenBytes + 16 + static_cast<size_t>(stages) * kLutStageBytes;
}

}  // namespace stq1
