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
// Split K: with few rows the K range is divided into S contiguous pieces; each
// unit stores its partial sums and the last unit to finish a (tile, slab)
// adds them in order 0..S-1 (deterministic) and writes y.
#pragma once

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

// Decode the chunk's KC blocks of this lane's row against TT tokens' tables.
// O = byte offset of the row's span inside its 16-byte-aligned slot.
template <int TT, int O>
__device__ __forceinline__ void lut_row_chunk(uint32_t slot, uint32_t lut,
                                              float (&acc)[kLutMaxTT]) {
#pragma unroll
  for (int j = 0; j < kLutKC; ++j) {
    const int B0 = O + kBlockBytes * j;            // block start inside the slot
    const int C0 = B0 >> 4;
    const int C1 = (B0 + kBlockBytes - 1) >> 4;
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
    const int base = B0 - 16 * C0;                 // block start inside the window (even)
    const uint32_t dword = w[base >> 2] >> (8 * (base & 3));
    const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(dword & 0xFFFFu)));
    const uint32_t H0 = win_word(w, base + kOffQh);
    const uint32_t H1 = win_word(w, base + kOffQh + 4);
    float2 s0[TT], s1[TT];
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      s0[t] = make_float2(0.f, 0.f);
      s1[t] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {                  // qs word i: groups 8i .. 8i+7
      const uint32_t Q = win_word(w, base + kOffQs + 4 * i);
      const uint32_t hb = (i < 4 ? H0 : H1) >> (8 * (i & 3));
      // table byte offsets (t << 6 | n << 2) of the 4 even / 4 odd groups
      const uint32_t ce = ((Q << 2) & 0x3C3C3C3Cu) | spread_even_bits(hb);
      const uint32_t co = ((Q >> 2) & 0x3C3C3C3Cu) | spread_even_bits(hb >> 1);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const uint32_t ae = __byte_perm(ce, lut, 0x7650u | m);   // lut is 256-aligned
        const uint32_t ao = __byte_perm(co, lut, 0x7650u | m);
        const int ge = 64 * j + 8 * i + 2 * m;    // even group's index in the chunk
#pragma unroll
        for (int t = 0; t < TT; ++t) {
          const uint32_t off = static_cast<uint32_t>(t * kLutTokenBytes + ge * kLutGroupBytes);
          const float ve = lds_f32_addr(ae + off);
          const float vo = lds_f32_addr(ao + off + kLutGroupBytes);
          if (m & 1)
            s1[t] = __fadd2_rn(s1[t], make_float2(ve, vo));
          else
            s0[t] = __fadd2_rn(s0[t], make_float2(ve, vo));
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      const float sum = (s0[t].x + s0[t].y) + (s1[t].x + s1[t].y);
      acc[t] = fmaf(d, sum, acc[t]);
    }
  }
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
    const float xa[4] = {x1, x0, x0, x0};
    const float xb[4] = {x2, x2, x1, x1};
    const float xc[4] = {x3, x3, x3, x2};
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      const float p = xa[z] + xb[z], q = xa[z] - xb[z];
      const float e0 = p + xc[z], e1 = p - xc[z], e2 = q + xc[z], e3 = q - xc[z];
      sts_v4f(gb + 16u * z, e0, e1, e2, e3);
      sts_v4f(gb + 64u + 16u * z, -e0, -e1, -e2, -e3);
    }
  }
}

// One work unit with TT tokens.
template <int TT>
__device__ void lut_unit(const LutArgs& a, const uint8_t* Wm, int slab, int split, int tile_id,
                         const int* xrow, const int* orow, uint8_t* smem) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = a.P;
  const int rho = P * lane + (warp % P) + 32 * P * (warp / P);   // row within the slab
  const long long row = static_cast<long long>(slab) * kLutRows + rho;
  const bool row_ok = row < a.N;
  const int c0 = static_cast<int>(static_cast<long long>(split) * a.n_chunks / a.S);
  const int c1 = static_cast<int>(static_cast<long long>(split + 1) * a.n_chunks / a.S);

  const uint32_t sbase = smem_u32(smem);
  const uint32_t lut = (sbase + 255u) & ~255u;
  const uint32_t stage0 = lut + TT * kLutTokenBytes;
  const uint32_t bar0 = stage0 + 2 * kLutStageBytes;
  const uint32_t my_slot_off = static_cast<uint32_t>(threadIdx.x) * kLutSlotBytes;

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
  const long long row0 = static_cast<long long>(slab) * kLutRows + (warp % P) + 32 * P * (warp / P);
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
  for (int c = c0; c < c1; ++c) {
    const int it = c - c0;
    const int st = it & 1;
    lut_build<TT>(xv, lut);
    if (c + 1 < c1) lut_load_x<TT>(a, c + 1, xrow, xv);   // prefetch the next chunk's activations
    const bool landed = mbar_wait_bounded(bar0 + 8u * st, (it >> 1) & 1);
    // one barrier: tables built, copies landed (agreed by every thread)
    if (!__syncthreads_and(landed)) {
      // A copy did not complete within the bound.  Wait (bounded) for the copy
      // already issued into the other stage, so no bulk copy is still writing
      // this CTA's shared memory when it exits; the error word is set.
      if (c + 1 < c1) mbar_wait_bounded(bar0 + 8u * (st ^ 1), ((it + 1) >> 1) & 1);
      return;
    }
    if (row_ok) {
      const uint32_t slot = stage0 + st * kLutStageBytes + my_slot_off;
      const int o = static_cast<int>((wbase + static_cast<uintptr_t>(c) * (kLutKC * kBlockBytes)) & 15);
      switch (o) {
        case 0: lut_row_chunk<TT, 0>(slot, lut, acc); break;
        case 4: lut_row_chunk<TT, 4>(slot, lut, acc); break;
        case 8: lut_row_chunk<TT, 8>(slot, lut, acc); break;
        default: lut_row_chunk<TT, 12>(slot, lut, acc); break;
      }
    }
    __syncthreads();
    if (c + 2 < c1) issue(c + 2, st);                      // this stage is free again
  }
  if (a.S == 1) {
    if (row_ok) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float v = acc[t];
        if ((a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2) v *= a.route_w[orow[t]];
        a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
      }
    }
    return;
  }

  // split K: publish partials, the last unit of this (tile, slab) reduces.
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
      for (int s = 0; s < a.S; ++s)
        v += __ldcg(&a.partial[(static_cast<long long>(s) * a.rows_out + orow[t]) * a.N + row]);
      if ((a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2) v *= a.route_w[orow[t]];
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

inline size_t lut_smem_bytes(int ttmax) {
  return 256 + static_cast<size_t>(ttmax) * kLutTokenBytes + 2 * kLutStageBytes + 16;
}

}  // namespace stq1
