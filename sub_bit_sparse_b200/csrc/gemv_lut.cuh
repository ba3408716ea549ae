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
// chunks of two blocks (512 columns, 84 bytes per row) into a shared-memory
// ring by 2-D tensor copies (TMA).  A row's 84 bytes rarely start on the
// 16-byte boundary a tensor copy needs, and a row's stride (K / 256 * 42
// bytes) is rarely a multiple of 16, so the packed buffer is viewed as
// "super-rows" of P consecutive rows, P = 16 / gcd(rowbytes, 16) in {1, 2, 4},
// whose stride P * rowbytes is.  Rows of the same residue r = row mod P start
// their chunk at the same offset mod 16; one copy per residue fetches a
// 112-byte window (the chunk plus lead-in, rounded to 16) of every super-row
// of the slab.  Each warp holds rows of one residue, so it decodes with
// compile-time byte offsets and conflict-free 16-byte shared loads (the
// 112-byte pitch is an odd multiple of 16).  The last rows of the buffer, when
// they do not fill a super-row, come through a second, 1-D tensor map.
//
// Split K: with few rows the K range is divided into S contiguous pieces.  The
// S units of a (tile, slab) normally form one thread-block cluster: each keeps
// its partial sums in its own shared memory and, after a cluster barrier, each
// adds a slice of the rows from all S peers (distributed shared memory) in
// order 0..S-1 and writes y.  Without clusters (a caller-provided scratch
// buffer instead), each unit stores its partials in global memory and the last
// unit to finish adds them in the same order.  Both are deterministic.
#pragma once

#include "device_common.cuh"
#include "packed_copy.cuh"

namespace stq1 {

constexpr int kLutRows = kSlabRows;           // rows per unit
constexpr int kLutThreads = 256;              // two threads per row: one per block of a chunk
constexpr int kLutKC = kChunkBlocks;          // blocks per chunk
constexpr int kLutChunkGroups = kGroupsPerBlock * kLutKC;    // 128
constexpr int kLutGroupBytes = 144;           // 32 fp32 entries + 16-byte pad
constexpr int kLutTokenBytes = kLutChunkGroups * kLutGroupBytes;   // 18432 = 72 * 256
constexpr int kLutMaxTT = 4;                  // tokens per tile

struct LutArgs {
  const uint16_t* x;         // [T, K] bf16 bits
  float* y;                  // [rows_out, N]
  float* partial;            // [S, rows_out, N] (S > 1, no cluster)
  int* counters;             // [n_units] (S > 1, no cluster), zero between calls
  const int* tile_info;      // MoE: [n_tiles_max, 4] = expert, pair offset, count, pad
  const int* n_tiles_dev;    // MoE: number of valid tiles
  const int* pairs;          // MoE: pair ids grouped by expert
  const float* route_w;      // [rows_out] routing weight per pair (flag WEIGHT_UP)
  PackedGeom g;              // tensor maps' view of the packed buffer
  int N, K;
  int topk;                  // pairs per token (1 for a plain GEMV)
  int batch;                 // plain GEMV: tokens
  int rows_out;              // rows of y
  int n_slabs;
  int S, cq, cr;             // K splits; split s has cq chunks, plus one if s < cr
  int flags;
  int cluster;               // 1: the S splits of a (tile, slab) form one thread-block cluster
  const uint8_t* next;       // bytes to bring into L2 for a following call, or nullptr
  long long next_bytes;      // multiple of 16
  int compact;               // MoE: bit 0 = output row of a pair is its position in `pairs`
                             // (else the pair id); bit 1 = its activation row is that position
                             // (else pair id / topk).  Routing weights are always by pair id.
  int tiles_cap;             // MoE: entries the tile table holds (debug-build checks)
  int x_rows;                // rows of x (debug-build checks)
};

// Spread bits 0, 2, 4, 6 of x to bit 6 of bytes 0..3 (other bits cleared).
__device__ __forceinline__ uint32_t spread_even_bits(uint32_t x) {
  return ((x & 0x55u) * 0x01041040u) & 0x40404040u;
}

__device__ __forceinline__ float lds_f32_addr(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// Table lookups of one block's 64 groups for TT tokens; `lut` is the 256-aligned
// base of this block's tables, every offset below it is an immediate of the
// shared load, and the group's code byte is spliced into the base with one
// byte permute.
template <int TT>
__device__ __forceinline__ void lut_block_body(const BlockCodes& bc, uint32_t lut, float (&acc)[kLutMaxTT]) {
  // partial sums of the byte positions m = 0, 1 and m = 2, 3 of each code
  // word, two per packed register: every update adds two lanes at once
  float2 s[TT][2];
#pragma unroll
  for (int t = 0; t < TT; ++t) s[t][0] = s[t][1] = make_float2(0.f, 0.f);
  static_for<8>([&](auto IC) {                       // qs word i: groups 8i .. 8i+7
    constexpr int i = decltype(IC)::value;
    const uint32_t Q = bc.Q[i];
    const uint32_t hb = (i < 4 ? bc.H0 : bc.H1) >> (8 * (i & 3));
    // table byte offsets (t << 6 | n << 2) of the 4 even / 4 odd groups
    const uint32_t ce = ((Q << 2) & 0x3C3C3C3Cu) | (((hb & 0x55u) * 0x01041040u) & 0x40404040u);
    const uint32_t co = ((Q >> 2) & 0x3C3C3C3Cu) | (((hb & 0xAAu) * 0x00820820u) & 0x40404040u);
    static_for<2>([&](auto PC) {
      constexpr int mp = decltype(PC)::value;        // byte positions 2 mp, 2 mp + 1
      constexpr int g0 = 8 * i + 4 * mp;             // even group of position 2 mp
      constexpr int g1 = g0 + 2;                     // even group of position 2 mp + 1
      const uint32_t ae0 = __byte_perm(ce, lut, 0x7650u | (2 * mp));
      const uint32_t ae1 = __byte_perm(ce, lut, 0x7650u | (2 * mp + 1));
      const uint32_t ao0 = __byte_perm(co, lut, 0x7650u | (2 * mp));
      const uint32_t ao1 = __byte_perm(co, lut, 0x7650u | (2 * mp + 1));
      static_for<TT>([&](auto TC) {
        constexpr int t = decltype(TC)::value;
        constexpr int tb = t * kLutTokenBytes;
        const float2 e = make_float2(lds_f32<tb + g0 * kLutGroupBytes>(ae0), lds_f32<tb + g1 * kLutGroupBytes>(ae1));
        const float2 o = make_float2(lds_f32<tb + (g0 + 1) * kLutGroupBytes>(ao0),
                                     lds_f32<tb + (g1 + 1) * kLutGroupBytes>(ao1));
        s[t][mp] = fadd2(s[t][mp], fadd2(e, o));     // s_m += e_m + o_m, lane by lane
      });
    });
  });
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = fmaf(bc.d, (s[t][0].x + s[t][0].y) + (s[t][1].x + s[t][1].y), acc[t]);
}

// Activations of this thread's group for chunk `chunk`, TT tokens (8 bytes each).
template <int TT>
__device__ __forceinline__ void lut_load_x(const uint16_t* const (&xr)[kLutMaxTT], int chunk, uint2 (&xv)[kLutMaxTT]) {
  const int col = chunk * (kLutKC * kBlockWeights) + 4 * static_cast<int>(threadIdx.x & (kLutChunkGroups - 1));
#pragma unroll
  for (int t = 0; t < TT; ++t) xv[t] = __ldg(reinterpret_cast<const uint2*>(xr[t] + col));
}

// Tables for one chunk: threads g and g + 128 build the 32 entries of group g
// for each token (zero lane 0, 1 and zero lane 2, 3 respectively).
// Entry c (code) = (-1)^t * (x_a + (-1)^beta x_b + (-1)^gamma x_c).
template <int TT>
__device__ __forceinline__ void lut_build(const uint2 (&xv)[kLutMaxTT], uint32_t lut) {
  const int g = threadIdx.x & (kLutChunkGroups - 1);
  const bool hi = threadIdx.x >= kLutChunkGroups;   // uniform over a warp
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
    if (!hi) {
      put(0, x1, x2, x3);
      put(1, x0, x2, x3);
    } else {
      put(2, x0, x1, x3);
      put(3, x0, x1, x2);
    }
  }
}

// One work unit with TT tokens.  R0 = first packed-buffer row of the slab
// (expert * N + slab * 128); xr / orow = activation row pointers and output
// rows of the tile's tokens.  Threads q and q + 128 own the same row; the
// first decodes the chunk's first block, the second its second block.
// DB (a one-token unit in a launch sized for two or more tokens): the unused
// second token's table space holds a second table, so chunk c + 1's table is
// built while slower threads still read chunk c's, and a chunk needs one
// barrier instead of two.
template <int TT, bool DB = false>
__device__ __forceinline__ void lut_unit(const LutArgs& a, const CUtensorMap* wmap, const CUtensorMap* tmap, long long R0,
                         int slab, int split, int unit, const uint16_t* const (&xr)[kLutMaxTT],
                         const int (&orow)[kLutMaxTT], const int (&wrow)[kLutMaxTT], uint8_t* smem) {
  const int c0 = split * a.cq + min(split, a.cr);
  const int c1 = c0 + a.cq + (split < a.cr ? 1 : 0);
  const int half = threadIdx.x >> 7;               // block of the chunk this thread decodes
  const int q = threadIdx.x & (kLutRows - 1);

  // ---- this thread's row and window (slots in residue-major order) ----
  const PackedRow pr = packed_row(a.g, R0, q);
  const int res = pr.res;                          // residue, uniform over a warp
  const int rho = pr.rho;                          // row within the slab, 0..127
  const int row = slab * kLutRows + rho;           // output row
  // (debug build: the window of a row that is read lies inside the stage)
  const bool row_ok = row < a.N && dbg_check(pr.slot + kWindowBytes <= static_cast<uint32_t>(a.g.stage_bytes));
  const uint32_t my_slot = pr.slot;

  const uint32_t sbase = smem_u32(smem);
  const uint32_t lut = (sbase + 255u) & ~255u;
  const uint32_t bar0 = lut + (DB ? 2 : TT) * kLutTokenBytes;   // 2 mbarriers
  const uint32_t stage0 = bar0 + 128;                // 128-aligned tensor-copy destinations
  const int NS = (c1 - c0 >= 2) ? 2 : 1;
  // split-K partials pushed by the cluster, at the same offset in every CTA of it
  const uint32_t red = stage0 + ((a.cq + (a.cr > 0 ? 1 : 0)) >= 2 ? 2 : 1) * a.g.stage_bytes;
  const bool push = a.cluster && a.S > 1;

  // split-K partials arrive by asynchronous stores counted on this barrier:
  // 2 halves x S pieces x TT tokens x the rows this CTA owns, 4 bytes each
  const uint32_t bar_red = bar0 + 16;
  if (threadIdx.x == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    mbar_init(bar_red, 1);
    if (push) {
      const int owned = (kLutRows * (split + 1) + a.S - 1) / a.S - (kLutRows * split + a.S - 1) / a.S;
      mbar_arrive_expect_tx(bar_red, static_cast<uint32_t>(2 * a.S * TT * owned * 4));
    }
    fence_mbar_init();
  }
  // Peers may write this CTA's shared memory only once it runs: announce it
  // now, and wait for every peer's announcement before the first push.
  if (push) cluster_arrive_relaxed();
  __syncthreads();

  // Tensor copies of chunk c into stage st (thread 0 only).
  auto issue = [&](int c, int st) {
    packed_issue_chunk(a.g, wmap, tmap, R0, c, stage0 + st * a.g.stage_bytes, bar0 + 8u * st);
  };

  float acc[kLutMaxTT];
#pragma unroll
  for (int t = 0; t < kLutMaxTT; ++t) acc[t] = 0.f;

  // Weights do not depend on the previous kernel in the stream: start their
  // copies before waiting for it (programmatic dependent launch), unless the
  // unit itself came from a routing kernel (which already waited).
  if (threadIdx.x == 0) {
    issue(c0, 0);
    if (NS == 2) issue(c0 + 1, 1);
  }
  // The next call's weights: each CTA asks for its share to be brought into
  // L2 (no completion is tracked; nothing here reads them).
  if (a.next != nullptr && threadIdx.x == 32) {
    const long long n_cta = static_cast<long long>(gridDim.x) * gridDim.y;
    const long long cta = static_cast<long long>(blockIdx.y) * gridDim.x + blockIdx.x;
    const long long share = ((a.next_bytes + n_cta - 1) / n_cta + 15) & ~15LL;
    const long long off = cta * share;
    if (off < a.next_bytes) {
      // the prefetch length is a 32-bit count: a share above 1 GiB is cut
      // there (the rest of it is simply not prefetched)
      const long long len = min(min(share, a.next_bytes - off), 1LL << 30);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.next + off), "r"(static_cast<uint32_t>(len))
                   : "memory");
    }
  }
  if (a.tile_info == nullptr) griddep_wait();
  griddep_launch_dependents();
  uint2 xv[kLutMaxTT];
  lut_load_x<TT>(xr, c0, xv);
  const uint32_t half_off = static_cast<uint32_t>(half * kGroupsPerBlock * kLutGroupBytes);
  bool failed = false;
  for (int c = c0; c < c1; ++c) {
    const int it = c - c0;
    const int st = NS == 2 ? (it & 1) : 0;
    const uint32_t parity = static_cast<uint32_t>(NS == 2 ? (it >> 1) : it) & 1u;
    // DB: chunk c's table goes to the buffer chunk c - 2 used; every thread
    // finished reading that one before it passed chunk c - 1's barrier
    const uint32_t lut_c = DB ? lut + static_cast<uint32_t>((it & 1) * kLutTokenBytes) : lut;
    lut_build<TT>(xv, lut_c);
    if (c + 1 < c1) lut_load_x<TT>(xr, c + 1, xv);   // prefetch the next chunk's activations
    const bool landed = mbar_wait_bounded(bar0 + 8u * st, parity);
    // one barrier: tables built, copies landed (agreed by every thread); with
    // DB also every thread done with chunk c - 1, so its stage is free
    if (!__syncthreads_and(landed)) {
      // A copy did not complete within the bound (the error word is set).
      // Wait (bounded) for the copies already issued into the other stage, so
      // no tensor copy is still writing this CTA's shared memory when it exits.
      // (With DB the next chunk's copy is issued only after this barrier, so
      // the other stage has one in flight only in the first iteration.)
      if (NS == 2 && c + 1 < c1 && (!DB || it == 0))
        mbar_wait_bounded(bar0 + 8u * (st ^ 1), static_cast<uint32_t>((it + 1) >> 1) & 1u);
      failed = true;
      break;
    }
    if (DB && threadIdx.x == 0 && it >= 1 && c + 1 < c1) issue(c + 1, st ^ 1);   // chunk c - 1's stage
    if (row_ok) {
      // only the extraction depends on the block's offset; one copy of the body follows
      BlockCodes b;
      load_chunk_block(stage0 + st * a.g.stage_bytes + my_slot, packed_window_offset(a.g, res, c), half, b);
      lut_block_body<TT>(b, lut_c + half_off, acc);
    }
    if (!DB) {
      __syncthreads();
      if (threadIdx.x == 0 && c + NS < c1) issue(c + NS, st);   // this stage is free again
    }
  }
  if (DB) __syncthreads();                         // every lookup done: the tables are free below

  if (push) {
    // Push both halves' partials into the shared memory of the CTA that owns
    // the row (cluster rank (row * S) / 128, the rank equal to its split) by
    // asynchronous stores counted on its reduction barrier; every CTA pushes,
    // failed or not.  Each CTA then waits (bounded) on its own barrier for
    // the partials of the rows it owns: no cluster-wide release fence.
    cluster_wait();
    const int owner = (rho * a.S) >> 7;
    // the owner's rows are ceil(128 r / S) .. ceil(128 (r + 1) / S) - 1
    const int local = rho - (owner * kLutRows + a.S - 1) / a.S;
    const int per = (kLutRows + a.S - 1) / a.S;      // rows per owner, at most
#pragma unroll
    for (int t = 0; t < TT; ++t)
      st_async_peer_f32(red + 4u * (((t * 2 * a.S) + 2 * split + half) * per + local), bar_red, owner, acc[t]);
    // every thread waits, so the CTA outlives the stores still coming in
    if (!mbar_wait_bounded(bar_red, 0)) return;
    if (half == 0 && owner == split && row_ok) {
      const bool up = (a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2;
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float v = 0.f;
        for (int i = 0; i < 2 * a.S; ++i) v += lds_f32_addr(red + 4u * ((t * 2 * a.S + i) * per + local));
        if (up) v *= a.route_w[wrow[t]];
        a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
      }
    }
    return;
  }

  // Add the second half into the first through shared memory (the tables are
  // free after the loop's last barrier).
  if (half == 1) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(lut + 4u * (t * kLutRows + rho)), "f"(acc[t]) : "memory");
  }
  __syncthreads();
  if (half == 0) {
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] += lds_f32_addr(lut + 4u * (t * kLutRows + rho));
  }
  const bool up = (a.flags & STQ1_MOE_WEIGHT_UP) && row >= a.N / 2;
  if (a.S == 1) {
    if (half == 0 && row_ok && !failed) {
#pragma unroll
      for (int t = 0; t < TT; ++t) {
        float v = acc[t];
        if (up) v *= a.route_w[wrow[t]];
        a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
      }
    }
    return;
  }
  if (failed) return;

  // Scratch mode: publish partials, the last unit of this (tile, slab) reduces.
  // One thread fences after the barrier: the barrier orders the other threads'
  // stores before it, and the gpu-scope fence is cumulative.
  if (half == 0 && row_ok) {
#pragma unroll
    for (int t = 0; t < TT; ++t)
      a.partial[(static_cast<long long>(split) * a.rows_out + orow[t]) * a.N + row] = acc[t];
  }
  __shared__ int s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const int old = atomicAdd(&a.counters[unit], 1);
    s_last = (old == a.S - 1);
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  if (half == 0 && row_ok) {
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      float v = 0.f;
      for (int sp = 0; sp < a.S; ++sp)
        v += __ldcg(&a.partial[(static_cast<long long>(sp) * a.rows_out + orow[t]) * a.N + row]);
      if (up) v *= a.route_w[wrow[t]];
      a.y[static_cast<long long>(orow[t]) * a.N + row] = v;
    }
  }
  if (threadIdx.x == 0) a.counters[unit] = 0;
}

// CTAs per SM the register budget must allow (the host's work split assumes it).
constexpr int lut_min_blocks(int ttmax) { return ttmax == 1 ? 4 : (ttmax == 2 ? 3 : 2); }

// Grid: x = unit = tile * n_slabs + slab, y = K split; clusters of (1, S, 1).
template <int TTMAX>
__global__ void __launch_bounds__(kLutThreads, lut_min_blocks(TTMAX))
lut_gemv_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap tmap, const LutArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int unit = blockIdx.x;
  const int split = blockIdx.y;
  const int tile = unit / a.n_slabs;
  const int slab = unit - tile * a.n_slabs;
  const uint16_t* xr[kLutMaxTT];
  int orow[kLutMaxTT], wrow[kLutMaxTT];
  int cnt, expert = 0;
  if (a.tile_info) {
    griddep_wait();                                  // the tile table comes from the routing kernel
    const int n_tiles = *a.n_tiles_dev;
    if (kDebugBuild && unit == 0 && split == 0 && threadIdx.x == 0) dbg_check(n_tiles <= a.tiles_cap);
    if (tile >= n_tiles) return;                     // whole clusters leave together (same tile)
    expert = a.tile_info[4 * tile + 0];
    const int off = a.tile_info[4 * tile + 1];
    cnt = a.tile_info[4 * tile + 2];
    // (debug build: the tile names an expert of the buffer and pairs of the list;
    // every check depends on the tile only, so a cluster leaves whole)
    if (!dbg_check(expert >= 0 && (expert + 1LL) * a.N <= a.g.rows_total && cnt >= 1 && cnt <= TTMAX &&
                   off >= 0 && off + cnt <= a.rows_out))
      return;
#pragma unroll
    for (int t = 0; t < kLutMaxTT; ++t) {
      const int pos = off + (t < cnt ? t : 0);
      const int p = a.pairs[pos];
      if (!dbg_check(p >= 0 && p < a.rows_out && ((a.compact & 2) ? pos : p / a.topk) < a.x_rows)) return;
      orow[t] = (a.compact & 1) ? pos : p;
      wrow[t] = p;
      xr[t] = a.x + static_cast<long long>((a.compact & 2) ? pos : p / a.topk) * a.K;
    }
  } else {
    const int t0 = tile * kLutMaxTT;
    cnt = min(kLutMaxTT, a.batch - t0);
#pragma unroll
    for (int t = 0; t < kLutMaxTT; ++t) {
      orow[t] = t0 + (t < cnt ? t : 0);
      wrow[t] = orow[t];
      xr[t] = a.x + static_cast<long long>(orow[t]) * a.K;
    }
  }
  const long long R0 = static_cast<long long>(expert) * a.N + static_cast<long long>(slab) * kLutRows;
  if constexpr (TTMAX >= 4) {
    if (cnt >= 4) {
      lut_unit<4>(a, &wmap, &tmap, R0, slab, split, unit, xr, orow, wrow, smem);
      return;
    }
  }
  if constexpr (TTMAX >= 3) {
    if (cnt == 3) {
      lut_unit<3>(a, &wmap, &tmap, R0, slab, split, unit, xr, orow, wrow, smem);
      return;
    }
  }
  if constexpr (TTMAX >= 2) {
    if (cnt == 2) {
      lut_unit<2>(a, &wmap, &tmap, R0, slab, split, unit, xr, orow, wrow, smem);
      return;
    }
  }
  lut_unit<1, (TTMAX >= 2)>(a, &wmap, &tmap, R0, slab, split, unit, xr, orow, wrow, smem);
}

// Dynamic shared memory: tables, barriers, stages and (cluster split K) the
// partials pushed by the S CTAs of the cluster into the CTA that owns a row:
// two per split, token and owned row (ceil(128 / S) rows).
inline size_t lut_smem_bytes(int ttmax, int stages, int stage_bytes, int cluster_S) {
  const size_t per = cluster_S > 1 ? static_cast<size_t>((kLutRows + cluster_S - 1) / cluster_S) : 0;
  return 256 + static_cast<size_t>(ttmax) * kLutTokenBytes + 128 + static_cast<size_t>(stages) * stage_bytes +
         static_cast<size_t>(ttmax) * 2 * cluster_S * per * 4;
}
// Upper bound over every geometry (P = 4 with the extra super-row is the largest stage).
inline size_t lut_smem_bytes_max(int ttmax) {
  return lut_smem_bytes(ttmax, 2, kPackedStageMax, kMaxClusterRanks);
}

}  // namespace stq1
