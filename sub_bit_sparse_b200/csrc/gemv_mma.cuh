// Decode GEMV for a few tokens on the tensor cores (mma.sync m16n8k16, sm_100a).
//
// y[t, j] = sum_k W^[j, k] x[t, k] for up to 8 tokens t at once.  A group of
// four weights is one of 32 patterns in {-d, 0, +d} with one zero lane
// (lemmy.durstig.online post 66506, "Four weights, five bits"), so the
// pattern is exact in bf16 and only d is not.  Each group's 5-bit code is
// expanded once into bf16 values +/-2 and 0 -- two 4-byte loads from two
// 32-entry shared tables that hold, per code, lanes 0-1 and lanes 2-3 as
// ready bf16 pairs (each table is 128 bytes, so a warp's 32 lookups hit 32
// distinct banks), i.e. the two A-operand registers -- and the tensor core
// contracts the pattern against the bf16 activations of all tokens of the
// unit with fp32 accumulation.  The decode cost per weight does not depend
// on the number of tokens, unlike the lookup-table kernel, whose table loads
// grow with them.  Each 256-column block is contracted into its own fp32
// accumulator and added with weight d / 2 (an exact fp32 product), once per
// row, block and token.
//
// Fragment use.  In an m16n8k16 MMA thread (g, q) (g = lane / 4, q = lane % 4)
// holds A for rows g and g + 8 at k slots {2q, 2q+1} and {2q+8, 2q+9}, and B
// for column (token) g at the same k slots.  The contraction does not care
// which weight column a k slot stands for as long as A and B agree, so those
// four slots hold the four lanes of one group: thread q of MMA m owns group
// 16q + m of the block, and a thread's sixteen groups of a block are
// contiguous (8 code bytes, 2 select-bit bytes).  B for group q is simply
// the token's four bf16 activations of that group, 8 bytes.
//
// Work unit = (token tile of <= 8 tokens, 128-row slab, K split), 8 warps.
// Packed rows arrive in chunks of two blocks through the super-row tensor
// copies of packed_copy.cuh (four stages); a step consumes two chunks (four
// blocks).  Warp w takes block w % 4 of the step for rows 64 (w / 4) ..
// + 63 of the slab (four 16-row MMA tiles, each of one residue class, in the
// copies' slot order), so its B fragments (one block of x for eight tokens,
// 32 registers) serve 64 MMAs.  Activations for a step are staged in shared
// memory by all threads, one step ahead, in a layout permuted so that the B
// loads (16 bytes: two MMAs) are free of bank conflicts.  At the end the
// four block-warps' partial sums meet in shared memory (fixed order).  The S
// split-K pieces of a unit normally form one thread-block cluster and push
// their partials into the shared memory of the CTA that owns each row, one
// cluster barrier, and the owner adds them in order 0..S-1; if the device
// refuses the cluster, they meet through the caller's workspace (the last
// piece to finish adds them in order), as in the lookup-table kernel.
#pragma once

#include "device_common.cuh"
#include "packed_copy.cuh"

namespace stq1 {

constexpr int kMmaThreads = 256;
constexpr int kMmaTokens = 8;                    // N of the MMA: tokens per unit
constexpr int kMmaRows = kSlabRows;              // 128 rows per unit
constexpr int kMmaStepBlocks = 4;                // blocks consumed per step (two chunks)
constexpr int kMmaStages = 4;                    // packed-weight chunks in flight
constexpr int kMmaXStepBytes = kMmaStepBlocks * kMmaTokens * kBlockWeights * 2;   // 16 KB
constexpr int kMmaOffTable = 0;                  // 2 x 32 x 4 bytes (256-aligned base)
constexpr int kMmaOffBar = 256;                  // kMmaStages mbarriers
constexpr int kMmaOffX = 512;                    // 2 x 16 KB of staged activations
constexpr int kMmaOffStage = kMmaOffX + 2 * kMmaXStepBytes;
// cluster split K: S x ceil(128 / S) slots x 8 tokens of pushed partials, at
// most (128 + S) x 32 bytes; placed after the stages
constexpr int kMmaRedBytes = (kMmaRows + kMaxClusterRanks) * kMmaTokens * 4;
static_assert(4 * kMmaRows * kMmaTokens * 4 <= 2 * kMmaXStepBytes, "reduction buffer must fit the x buffers");

struct MmaArgs {
  const uint16_t* x;         // [T, K] bf16 bits
  float* y;                  // [rows_out, N]
  float* partial;            // [S, rows_out, N] (S > 1)
  int* counters;             // [units] (S > 1), zero between calls
  const int* tile_info;      // MoE: [tiles, 4] = expert, pair offset, count, pad
  const int* n_tiles_dev;    // MoE: number of valid tiles
  const int* pairs;          // MoE: pair ids grouped by expert
  const float* route_w;      // [rows_out] routing weight per pair (flag WEIGHT_UP)
  PackedGeom g;
  int N, K;
  int topk;                  // pairs per token (1 for a plain GEMV)
  int batch;                 // plain GEMV: tokens
  int rows_out;
  int n_slabs;
  int n_chunks;              // chunks (two blocks each) of K
  int S, sq, sr;             // K splits over steps: split s has sq steps, plus one if s < sr
  int flags;
  int compact;               // MoE: bit 0 = output row of a pair is its position in `pairs`
                             // (else the pair id); bit 1 = its activation row is that position
                             // (else pair id / topk).  Routing weights are always by pair id.
  int tiles_cap;             // MoE: entries the tile table holds (debug-build checks)
  int x_rows;                // rows of x (debug-build checks)
  int cluster;               // 1: the S splits of a unit form one thread-block cluster (1, S, 1)
};

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts_v4u(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Position (in 8-byte group slots) of group 16j + i of token t inside the
// token's 64-slot row of a staged block: pairs (i even, i + 1) stay adjacent
// and the eight threads of a quarter warp (two tokens x four j) read eight
// distinct 16-byte bank groups.
__device__ __forceinline__ int mma_x_pos(int t, int j, int i) {
  return 16 * j + (i ^ (2 * (((t & 1) << 2) | j)));
}

// The code fields a thread needs from one block of one row: fp32 d / 2, the
// eight code bytes of its sixteen groups (Q0: groups 0..7, Q1: 8..15) and
// their sixteen select bits.  `blk` = shared address of the block's first
// byte; H = which block of the chunk (it fixes the alignment of the codes:
// the block starts at 0 (H = 0) or 2 (H = 1) mod 4).
struct QuarterCodes {
  float d;
  uint32_t Q0, Q1, S;
};

template <int H>
__device__ __forceinline__ QuarterCodes load_quarter(uint32_t blk, int q) {
  QuarterCodes c;
  c.d = 0.5f * __half2float(__ushort_as_half(static_cast<unsigned short>(lds_u16(blk + kOffD))));
  const uint32_t qs = blk + kOffQs + 8u * q;
  if constexpr (H == 0) {
    // qs starts 2 bytes past a 4-byte boundary
    const uint32_t w0 = lds_u32(qs - 2), w1 = lds_u32(qs + 2), w2 = lds_u32(qs + 6);
    c.Q0 = __funnelshift_r(w0, w1, 16);
    c.Q1 = __funnelshift_r(w1, w2, 16);
  } else {
    c.Q0 = lds_u32(qs);
    c.Q1 = lds_u32(qs + 4);
  }
  c.S = lds_u16(blk + kOffQh + 2u * q);
  return c;
}

// Table byte offsets (t << 6 | n << 2) of groups 0, 2, 4, 6 (even) and
// 1, 3, 5, 7 (odd) of a code word Q with select bits hb (bit i = group i).
__device__ __forceinline__ void code_offsets(uint32_t Q, uint32_t hb, uint32_t& ce, uint32_t& co) {
  ce = ((Q << 2) & 0x3C3C3C3Cu) | (((hb & 0x55u) * 0x01041040u) & 0x40404040u);
  co = ((Q >> 2) & 0x3C3C3C3Cu) | (((hb & 0xAAu) * 0x00820820u) & 0x40404040u);
}

template <int OFF>
__device__ __forceinline__ uint32_t lds_u32_off(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF));
  return v;
}

// The two A registers (lanes 0, 1 and lanes 2, 3 as bf16 pairs) of the group
// whose table offset is byte m of `c`: the offset is spliced into the
// 256-aligned table base, the second table sits 128 bytes above the first.
__device__ __forceinline__ void decode_group(uint32_t c, int m, uint32_t table, uint32_t& lo, uint32_t& hi) {
  const uint32_t addr = __byte_perm(c, table, 0x7650u | static_cast<uint32_t>(m));
  lo = lds_u32_off<0>(addr);
  hi = lds_u32_off<128>(addr);
}

// One 16-row tile of one block: 16 MMAs into a fresh accumulator, then added
// with each row's d / 2.  cA / cB = code fields of rows g and g + 8 (zero
// patterns for rows outside the matrix); xb = B fragments of the block.
__device__ __forceinline__ void mma_tile_block(const QuarterCodes& cA, const QuarterCodes& cB,
                                               const uint32_t (&xb)[32], uint32_t table, float (&acc)[4]) {
  // two accumulators (even and odd groups) so that consecutive MMAs do not
  // wait on each other
  float blk[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const uint32_t QA = half ? cA.Q1 : cA.Q0, QB = half ? cB.Q1 : cB.Q0;
    // code_offsets looks at bits 0..7 only
    const uint32_t hA = half ? (cA.S >> 8) : cA.S, hB = half ? (cB.S >> 8) : cB.S;
    uint32_t eA, oA, eB, oB;
    code_offsets(QA, hA, eA, oA);
    code_offsets(QB, hB, eB, oB);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int m = 8 * half + i;
      uint32_t a0, a2, a1, a3;
      decode_group((i & 1) ? oA : eA, i >> 1, table, a0, a2);
      decode_group((i & 1) ? oB : eB, i >> 1, table, a1, a3);
      mma_bf16_16816(blk[i & 1], a0, a1, a2, a3, xb[2 * m], xb[2 * m + 1]);
    }
  }
  acc[0] = fmaf(cA.d, blk[0][0] + blk[1][0], acc[0]);
  acc[1] = fmaf(cA.d, blk[0][1] + blk[1][1], acc[1]);
  acc[2] = fmaf(cB.d, blk[0][2] + blk[1][2], acc[2]);
  acc[3] = fmaf(cB.d, blk[0][3] + blk[1][3], acc[3]);
}

// Grid: x = unit = tile * n_slabs + slab, y = K split.
__global__ void __launch_bounds__(kMmaThreads, 2)
mma_gemv_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap tmap, const MmaArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t sbase = (smem_u32(smem_raw) + 255u) & ~255u;
  const uint32_t table = sbase + kMmaOffTable;
  const uint32_t bar0 = sbase + kMmaOffBar;
  const uint32_t xs0 = sbase + kMmaOffX;
  const uint32_t stage0 = sbase + kMmaOffStage;

  const int unit = blockIdx.x;
  const int split = blockIdx.y;
  const int tile = unit / a.n_slabs;
  const int slab = unit - tile * a.n_slabs;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, q = lane & 3;          // MMA row group, thread in group
  const int hb = warp & 3;                         // block of the step
  const int rh = warp >> 2;                        // row half of the slab

  // ---- tokens of the unit ----
  int cnt, expert = 0, off = 0;
  if (a.tile_info) {
    griddep_wait();                                // the tile table comes from the routing kernel
    const int n_tiles = *a.n_tiles_dev;
    if (kDebugBuild && unit == 0 && split == 0 && threadIdx.x == 0) dbg_check(n_tiles <= a.tiles_cap);
    if (tile >= n_tiles) return;
    expert = a.tile_info[4 * tile + 0];
    off = a.tile_info[4 * tile + 1];
    cnt = a.tile_info[4 * tile + 2];
    if constexpr (kDebugBuild) {
      // the tile names an expert of the buffer and pairs of the list, and each
      // pair's activation row exists (uniform over the CTA: it leaves whole)
      bool ok = expert >= 0 && (expert + 1LL) * a.N <= a.g.rows_total && cnt >= 1 && cnt <= kMmaTokens &&
                off >= 0 && off + cnt <= a.rows_out;
      for (int t = 0; ok && t < cnt; ++t) {
        const int p = a.pairs[off + t];
        ok = p >= 0 && p < a.rows_out && ((a.compact & 2) ? off + t : p / a.topk) < a.x_rows;
      }
      if (!dbg_check(ok)) return;
    }
  } else {
    cnt = min(kMmaTokens, a.batch - tile * kMmaTokens);
  }
  auto out_row = [&](int t) -> int {               // output row of token t (< cnt)
    if (!a.tile_info) return tile * kMmaTokens + t;
    return (a.compact & 1) ? off + t : a.pairs[off + t];
  };
  auto x_row = [&](int t) -> const uint16_t* {     // activation row of token t (clamped)
    const int tt = t < cnt ? t : 0;
    int r = tile * kMmaTokens + tt;
    if (a.tile_info) r = (a.compact & 2) ? off + tt : a.pairs[off + tt] / a.topk;
    return a.x + static_cast<long long>(r) * a.K;
  };

  const int s0 = split * a.sq + min(split, a.sr);
  const int s1 = s0 + a.sq + (split < a.sr ? 1 : 0);
  const int c0 = 2 * s0, c1 = min(a.n_chunks, 2 * s1);
  const long long R0 = static_cast<long long>(expert) * a.N + static_cast<long long>(slab) * kMmaRows;

  // ---- set-up: decode table, barriers, first copies ----
  if (threadIdx.x < 32) {
    // bf16 +2 = 0x4000, -2 = 0xC000, 0 = 0x0000; lanes 0, 1 then lanes 2, 3
    int v[4];
    code_pattern(threadIdx.x, v);
    uint32_t h[4];
#pragma unroll
    for (int l = 0; l < 4; ++l) h[l] = v[l] == 0 ? 0u : (v[l] > 0 ? 0x4000u : 0xC000u);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 4u * threadIdx.x), "r"(h[0] | (h[1] << 16)) : "memory");
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(table + 128u + 4u * threadIdx.x), "r"(h[2] | (h[3] << 16))
                 : "memory");
  }
  const bool push = a.cluster != 0 && a.S > 1;
  // cluster split K: the pushed partials arrive by asynchronous stores counted
  // on this barrier (S pieces x 8 tokens x the slots this CTA owns, 4 bytes each)
  const uint32_t bar_red = bar0 + 8u * kMmaStages;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kMmaStages; ++i) mbar_init(bar0 + 8u * i, 1);
    mbar_init(bar_red, 1);
    if (push) {
      const int owned = (kMmaRows * (split + 1) + a.S - 1) / a.S - (kMmaRows * split + a.S - 1) / a.S;
      mbar_arrive_expect_tx(bar_red, static_cast<uint32_t>(a.S * kMmaTokens * owned * 4));
    }
    fence_mbar_init();
  }
  __syncthreads();
  // Cluster split K: peers write this CTA's shared memory only once it runs;
  // announce it now and wait for every peer's announcement before the pushes.
  if (push) cluster_arrive_relaxed();
  auto issue = [&](int c) {
    const int st = (c - c0) % kMmaStages;
    packed_issue_chunk(a.g, &wmap, &tmap, R0, c, stage0 + st * a.g.stage_bytes, bar0 + 8u * st);
  };
  if (threadIdx.x == 0)
    for (int c = c0; c < min(c1, c0 + kMmaStages); ++c) issue(c);
  if (a.tile_info == nullptr) griddep_wait();
  griddep_launch_dependents();

  // ---- this thread's rows: 4 tiles x (g, g + 8) ----
  uint32_t slot[8];
  int res_of_tile[4];
  bool ok[8];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const PackedRow pr = packed_row(a.g, R0, 64 * rh + 16 * rt + gq + 8 * u);
      // (debug build: the window of a row that is read lies inside the stage)
      ok[2 * rt + u] = slab * kMmaRows + pr.rho < a.N &&
                       dbg_check(pr.slot + kWindowBytes <= static_cast<uint32_t>(a.g.stage_bytes));
      // A row outside the matrix has no slot in the stage (its computed slot
      // can lie past the stage's tail slots): read slot 0 instead, whose
      // bytes are in bounds, and give the row scale 0.
      slot[2 * rt + u] = ok[2 * rt + u] ? pr.slot : 0u;
      if (u == 0) res_of_tile[rt] = pr.res;
    }
  }

  // ---- staged activations: step s's four blocks, 8 tokens ----
  // Thread (warp w, lane l) moves, for each block k of the step, the 16-byte
  // pair of groups l of token w: a warp reads 512 contiguous bytes of one
  // token row per block.
  const uint16_t* xr = x_row(warp);
  uint4 xv[4];
  auto load_x = [&](int step) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 2 * step + (k >> 1);
      const int col = c * (2 * kBlockWeights) + (k & 1) * kBlockWeights + 8 * lane;
      xv[k] = c < a.n_chunks ? __ldg(reinterpret_cast<const uint4*>(xr + col)) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto store_x = [&](int step) {
    const uint32_t xb = xs0 + static_cast<uint32_t>(step & 1) * kMmaXStepBytes;
    const int grp = 2 * lane;
    const int pos = mma_x_pos(warp, grp >> 4, grp & 15);
#pragma unroll
    for (int k = 0; k < 4; ++k)
      sts_v4u(xb + static_cast<uint32_t>(((k * kMmaTokens + warp) * 64 + pos) * 8), xv[k]);
  };
  if (s0 < s1) {
    load_x(s0);
    store_x(s0);
  }

  float acc[4][4];
#pragma unroll
  for (int rt = 0; rt < 4; ++rt) acc[rt][0] = acc[rt][1] = acc[rt][2] = acc[rt][3] = 0.f;

  int s_fail = -1;
  for (int s = s0; s < s1; ++s) {
    if (s + 1 < s1) load_x(s + 1);                 // next step's activations, stored after this step
    const int ca = 2 * s, cb = min(2 * s + 1, c1 - 1);
    bool landed = true;
    for (int c = ca; c <= cb; ++c) {
      const int it = c - c0;
      landed &= mbar_wait_bounded(bar0 + 8u * (it % kMmaStages), static_cast<uint32_t>(it / kMmaStages) & 1u);
    }
    // one barrier: this step's copies landed (agreed by every thread) and the
    // activations staged during the previous step are visible
    if (__syncthreads_or(!landed)) {
      s_fail = s;
      break;
    }
    const int c = 2 * s + (hb >> 1);               // this warp's chunk
    if (c < c1) {
      // B fragments of block hb for token gq: pairs of groups (m, m + 1)
      const uint32_t xrow = xs0 + static_cast<uint32_t>(s & 1) * kMmaXStepBytes +
                            static_cast<uint32_t>((hb * kMmaTokens + gq) * 64 * 8);
      uint32_t xb[32];
#pragma unroll
      for (int m = 0; m < 16; m += 2) {
        const uint4 v = lds_v4(xrow + static_cast<uint32_t>(mma_x_pos(gq, q, m) * 8));
        xb[2 * m] = v.x;
        xb[2 * m + 1] = v.y;
        xb[2 * m + 2] = v.z;
        xb[2 * m + 3] = v.w;
      }
      const uint32_t st = stage0 + static_cast<uint32_t>((c - c0) % kMmaStages) * a.g.stage_bytes;
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const uint32_t o = static_cast<uint32_t>(packed_window_offset(a.g, res_of_tile[rt], c));
        QuarterCodes cA, cB;
        if (hb & 1) {
          cA = load_quarter<1>(st + slot[2 * rt] + o + kBlockBytes, q);
          cB = load_quarter<1>(st + slot[2 * rt + 1] + o + kBlockBytes, q);
        } else {
          cA = load_quarter<0>(st + slot[2 * rt] + o, q);
          cB = load_quarter<0>(st + slot[2 * rt + 1] + o, q);
        }
        // rows outside the matrix: scale 0 (their codes are slot 0's bytes)
        if (!ok[2 * rt]) cA.d = 0.f;
        if (!ok[2 * rt + 1]) cB.d = 0.f;
        mma_tile_block(cA, cB, xb, table, acc[rt]);
      }
    }
    if (s + 1 < s1) store_x(s + 1);
    __syncthreads();                               // this step's stages and x buffer s & 1 are free
    if (threadIdx.x == 0)
      for (int cn = 2 * s + kMmaStages; cn < min(c1, 2 * s + kMmaStages + 2); ++cn) issue(cn);
  }
  if (s_fail >= 0) {
    // A copy did not land within the bound (the error word is set).  Wait,
    // bounded, for the copies still in flight (chunks of this step and the
    // next, which were issued) so that no tensor copy writes this CTA's shared
    // memory after it exits.  Waiting on a phase that already completed
    // returns at once.
    if (threadIdx.x == 0) {
      for (int c = 2 * s_fail; c < min(c1, 2 * s_fail + kMmaStages); ++c) {
        const int it = c - c0;
        mbar_wait_bounded(bar0 + 8u * (it % kMmaStages), static_cast<uint32_t>(it / kMmaStages) & 1u);
      }
    }
    __syncthreads();
    if (push) {
      // push zeros so that every owner's count completes; the error word is set
      cluster_wait();
      const uint32_t redc = stage0 + static_cast<uint32_t>(kMmaStages) * a.g.stage_bytes;
      const int per = (kMmaRows + a.S - 1) / a.S;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int idx = threadIdx.x + 256 * k;
        const int sl = idx >> 3, t = idx & 7;
        const int owner = (sl * a.S) >> 7;
        const int local = sl - (owner * kMmaRows + a.S - 1) / a.S;
        st_async_peer_f32(redc + 4u * static_cast<uint32_t>((split * per + local) * kMmaTokens + t), bar_red, owner,
                          0.f);
      }
      mbar_wait_bounded(bar_red, 0);               // this CTA outlives the stores coming in
    }
    return;
  }

  // ---- the four block-warps' partials, in shared memory, fixed order ----
  const uint32_t red = xs0;                        // [4 hb][128 slots][8 tokens] fp32
#pragma unroll
  for (int rt = 0; rt < 4; ++rt) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int sl = 64 * rh + 16 * rt + gq + 8 * u;
#pragma unroll
      for (int v = 0; v < 2; ++v)
        sts_f32(red + 4u * static_cast<uint32_t>((hb * kMmaRows + sl) * kMmaTokens + 2 * q + v),
                acc[rt][2 * u + v]);
    }
  }
  __syncthreads();
  const bool up_flag = (a.flags & STQ1_MOE_WEIGHT_UP) != 0;
  float vals[4];
  int orows[4], rows[4], wrows[4];
  bool good[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int idx = threadIdx.x + 256 * k;         // (slot, token), token fastest
    const int sl = idx >> 3, t = idx & 7;
    float v = 0.f;
#pragma unroll
    for (int h = 0; h < 4; ++h) v += lds_f32_addr(red + 4u * static_cast<uint32_t>((h * kMmaRows + sl) * kMmaTokens + t));
    const PackedRow pr = packed_row(a.g, R0, sl);
    const int row = slab * kMmaRows + pr.rho;
    good[k] = t < cnt && row < a.N;
    rows[k] = row;
    orows[k] = good[k] ? out_row(t) : 0;
    wrows[k] = (good[k] && a.tile_info) ? a.pairs[off + t] : 0;
    vals[k] = v;
  }
  if (a.S == 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (!good[k]) continue;
      float v = vals[k];
      if (up_flag && rows[k] >= a.N / 2) v *= a.route_w[wrows[k]];
      a.y[static_cast<long long>(orows[k]) * a.N + rows[k]] = v;
    }
    return;
  }
  if (push) {
    // Push every (slot, token) partial into the shared memory of the CTA that
    // owns the slot (cluster rank (slot * S) / 128, the rank equal to its
    // split) by asynchronous stores counted on its reduction barrier; each
    // CTA waits (bounded) on its own barrier, then adds its slots' S partials
    // in order 0..S-1.
    const uint32_t redc = stage0 + static_cast<uint32_t>(kMmaStages) * a.g.stage_bytes;
    const int per = (kMmaRows + a.S - 1) / a.S;   // slots per owner, at most
    cluster_wait();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = threadIdx.x + 256 * k;
      const int sl = idx >> 3, t = idx & 7;
      const int owner = (sl * a.S) >> 7;
      const int local = sl - (owner * kMmaRows + a.S - 1) / a.S;
      st_async_peer_f32(redc + 4u * static_cast<uint32_t>((split * per + local) * kMmaTokens + t), bar_red, owner,
                        vals[k]);
    }
    if (!mbar_wait_bounded(bar_red, 0)) return;    // every thread: the CTA outlives the stores coming in
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = threadIdx.x + 256 * k;
      const int sl = idx >> 3, t = idx & 7;
      if (((sl * a.S) >> 7) != split || !good[k]) continue;
      const int local = sl - (split * kMmaRows + a.S - 1) / a.S;
      float v = 0.f;
      for (int sp = 0; sp < a.S; ++sp)
        v += lds_f32_addr(redc + 4u * static_cast<uint32_t>((sp * per + local) * kMmaTokens + t));
      if (up_flag && rows[k] >= a.N / 2) v *= a.route_w[wrows[k]];
      a.y[static_cast<long long>(orows[k]) * a.N + rows[k]] = v;
    }
    return;
  }
  // split K through the workspace: publish the partials; the last piece of
  // the unit adds them in order
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (good[k]) a.partial[(static_cast<long long>(split) * a.rows_out + orows[k]) * a.N + rows[k]] = vals[k];
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
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    if (!good[k]) continue;
    float v = 0.f;
    for (int sp = 0; sp < a.S; ++sp)
      v += __ldcg(&a.partial[(static_cast<long long>(sp) * a.rows_out + orows[k]) * a.N + rows[k]]);
    if (up_flag && rows[k] >= a.N / 2) v *= a.route_w[wrows[k]];
    a.y[static_cast<long long>(orows[k]) * a.N + rows[k]] = v;
  }
  if (threadIdx.x == 0) a.counters[unit] = 0;
}

inline size_t mma_smem_bytes(int stage_bytes, bool cluster = false) {
  return 256 + kMmaOffStage + static_cast<size_t>(kMmaStages) * stage_bytes + (cluster ? kMmaRedBytes : 0);
}
inline size_t mma_smem_bytes_max() { return mma_smem_bytes(kPackedStageMax, true); }

}  // namespace stq1
