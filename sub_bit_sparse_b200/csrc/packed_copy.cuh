// Tensor copies of packed STQ1_0 rows into shared memory, shared by the table
// kernel and the tile kernel.
//
// A row's stride (K / 256 * 42 bytes) is rarely a multiple of 16 and a chunk
// of two blocks (84 bytes) rarely starts on a 16-byte boundary, both of which
// a tensor copy needs.  So the packed buffer is viewed as "super-rows" of
// P = 16 / gcd(rowbytes, 16) consecutive rows (P in {1, 2, 4}), whose stride
// P * rowbytes is a multiple of 16.  Rows of the same residue r = row mod P
// start a chunk at the same offset mod 16; one 2-D copy per residue fetches a
// 112-byte window (the chunk plus up to 12 bytes of lead-in, rounded to 16)
// of every super-row of a 128-row slab.  In shared memory, residue r's windows
// sit one after another at a 112-byte pitch (an odd multiple of 16: 16-byte
// loads by 8 consecutive rows hit distinct banks).  The last rows of the
// buffer, when they do not fill a super-row, come through a 1-D map into
// separate slots.  A slab whose first row is not a multiple of P (MoE experts
// with N % P != 0) takes one more super-row per box.
#pragma once

#include <cudaTypedefs.h>

#include "device_common.cuh"

namespace stq1 {

constexpr int kSlabRows = 128;                 // rows per slab (and per tile-kernel M tile)
constexpr int kChunkBlocks = 2;                // blocks per chunk
constexpr int kChunkBytes = kChunkBlocks * kBlockBytes;    // 84 bytes of a row per chunk
constexpr int kWindowBytes = 112;              // tensor-copy box width: 84 bytes + lead-in, 7 x 16 B
constexpr int kTailSlots = 3;                  // rows of a partial last super-row (P - 1 at most)
constexpr int kTailSlotBytes = 128;

// Geometry of the two tensor maps over one packed buffer (built per call on the host).
struct PackedGeom {
  long long rowbytes;        // K / 256 * 42
  long long tail_row0;       // first buffer row fetched through the tail map
  long long rows_total;      // rows in the packed buffer (N, or E * N)
  int main_srows;            // super-rows in the main map (tail_row0 / P)
  int logP;                  // rows per super-row = 1 << logP
  int box_h;                 // super-rows per box: 128 / P, plus one when N % P != 0
  int buf_bytes;             // shared bytes per residue buffer (box_h * 112, 128-aligned)
  int stage_bytes;           // P * buf_bytes + tail slots
};

inline int packed_buf_bytes(int box_h) { return (box_h * kWindowBytes + 127) & ~127; }
inline int packed_stage_bytes(int logP, int box_h) {
  return (1 << logP) * packed_buf_bytes(box_h) + kTailSlots * kTailSlotBytes;
}
// Largest stage over every geometry (P = 4 with the extra super-row).
constexpr int kPackedStageMax = 4 * ((33 * kWindowBytes + 127) & ~127) + kTailSlots * kTailSlotBytes;

__device__ __forceinline__ void tma_load_w2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tma_load_w1d(uint32_t dst, const CUtensorMap* map, int x, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2}], [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(bar)
      : "memory");
}

// The row a thread owns inside a slab starting at buffer row R0, for slot
// order q in [0, 128) (residue-major), and where its window lands in a stage.
struct PackedRow {
  long long R;      // buffer row
  int rho;          // row within the slab, 0..127
  int res;          // residue R mod P (uniform over 32 consecutive q)
  uint32_t slot;    // byte offset of the window inside a stage
};

__device__ __forceinline__ PackedRow packed_row(const PackedGeom& g, long long R0, int q) {
  PackedRow p;
  const int shift = 7 - g.logP;                    // log2(rows of one residue per slab)
  p.res = q >> shift;
  const int kk = q & ((1 << shift) - 1);
  const int R0mod = static_cast<int>(R0 & ((1 << g.logP) - 1));
  const int br = p.res < R0mod ? 1 : 0;            // residues below R0's start one super-row later
  p.R = (((R0 >> g.logP) + br + kk) << g.logP) + p.res;
  p.rho = static_cast<int>(p.R - R0);
  p.slot = p.R >= g.tail_row0
               ? static_cast<uint32_t>((1 << g.logP) * g.buf_bytes) +
                     static_cast<uint32_t>(p.R - g.tail_row0) * kTailSlotBytes
               : static_cast<uint32_t>(p.res * g.buf_bytes + (br + kk) * kWindowBytes);
  return p;
}

// Offset mod 16 of chunk c's first byte inside the window of a row of residue res.
__device__ __forceinline__ int packed_window_offset(const PackedGeom& g, int res, int c) {
  return ((static_cast<int>(res * g.rowbytes) & 15) + c * kChunkBytes) & 15;
}

// Issues the copies of chunk c of the slab at buffer row R0 into the stage at
// dst, with completion counted on bar (one thread).
__device__ __forceinline__ void packed_issue_chunk(const PackedGeom& g, const CUtensorMap* wmap,
                                                   const CUtensorMap* tmap, long long R0, int c, uint32_t dst,
                                                   uint32_t bar) {
  const int P = 1 << g.logP;
  const int xc = c * kChunkBytes;
  const long long sr0 = R0 >> g.logP;
  const bool main = sr0 < g.main_srows;
  int ntail = 0;
  const long long t0 = g.tail_row0 > R0 ? g.tail_row0 : R0;
  const long long t1 = g.rows_total < R0 + kSlabRows ? g.rows_total : R0 + kSlabRows;
  if (t1 > t0) ntail = static_cast<int>(t1 - t0);
  if constexpr (kDebugBuild) {
    // every box inside the stage's buffers, every tail row in its slot
    const int tfirst = static_cast<int>(t0 - g.tail_row0);
    const bool ok = (!main || dbg_smem_range(dst, static_cast<uint32_t>((P - 1) * g.buf_bytes +
                                                                       g.box_h * kWindowBytes))) &&
                    (ntail == 0 || (dbg_check(tfirst >= 0 && tfirst + ntail <= kTailSlots) &&
                                    dbg_smem_range(dst + P * g.buf_bytes + tfirst * kTailSlotBytes,
                                                   static_cast<uint32_t>(ntail * kTailSlotBytes))));
    if (!ok) {
      mbar_arrive(bar);                            // complete the phase without copies
      return;
    }
  }
  mbar_arrive_expect_tx(bar, (main ? P * g.box_h * kWindowBytes : 0) + ntail * kWindowBytes);
  if (main)
    for (int r = 0; r < P; ++r)
      tma_load_w2d(dst + r * g.buf_bytes, wmap, (static_cast<int>(r * g.rowbytes) + xc) & ~15,
                   static_cast<int>(sr0), bar);
  for (int i = 0; i < ntail; ++i) {
    const int t = static_cast<int>(t0 - g.tail_row0) + i;
    tma_load_w1d(dst + P * g.buf_bytes + t * kTailSlotBytes, tmap,
                 (static_cast<int>(t * g.rowbytes) + xc) & ~15, bar);
  }
}

__device__ __forceinline__ uint32_t win_word(const uint32_t* w, int p) {
  // p is a compile-time constant after unrolling
  return (p & 3) ? __funnelshift_r(w[p >> 2], w[(p >> 2) + 1], 8 * (p & 3)) : w[p >> 2];
}

// Code words of one block, extracted from a 16-byte-aligned register window:
// d (fp32), qs as 8 little-endian words, qh as 2 words.
struct BlockCodes {
  float d;
  uint32_t Q[8];
  uint32_t H0, H1;
};

// Loads the block starting at byte B0 of a window (B0 compile-time) with
// 16-byte shared loads and extracts its fields.
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

// Block `blk` (0 or 1) of a chunk whose window starts at offset o (mod 16, a
// multiple of 4): one of eight compile-time variants.
__device__ __forceinline__ void load_chunk_block(uint32_t slot, int o, int blk, BlockCodes& b) {
  switch (o | (blk << 4)) {
    case 0: load_block_codes<0>(slot, b); break;
    case 4: load_block_codes<4>(slot, b); break;
    case 8: load_block_codes<8>(slot, b); break;
    case 12: load_block_codes<12>(slot, b); break;
    case 16 | 0: load_block_codes<0 + kBlockBytes>(slot, b); break;
    case 16 | 4: load_block_codes<4 + kBlockBytes>(slot, b); break;
    case 16 | 8: load_block_codes<8 + kBlockBytes>(slot, b); break;
    default: load_block_codes<12 + kBlockBytes>(slot, b); break;
  }
}

}  // namespace stq1
