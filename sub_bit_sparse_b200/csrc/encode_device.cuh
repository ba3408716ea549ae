// Device STQ1_0 encoders (plain amax and Sherry), byte-identical to the host
// encoder behind stq1_quantize_ref.
//
// Plain encoder: amax scale ("AngelSlim Shrinks Tencent's 1.5TB Hy4-Preview to
// 214 GiB at 6x Compression", bullet list).  Sherry encoder: alternating
// weighted-least-squares scale fit and importance-weighted zero placement,
// three rounds on the pages (lemmy.durstig.online post 66506, "Scale and zero
// position are fit together").  One thread encodes one 256-weight block; every
// real-valued step is fp64 in the host encoder's order, written with the
// round-to-nearest intrinsics (__dmul_rn, __dadd_rn, ...) so that no multiply
// and add are fused, which is what makes the bytes identical.
#pragma once

#include "device_common.cuh"

namespace stq1 {

constexpr int kEncThreads = 128;                 // blocks per CTA (one thread each)
constexpr int kEncHPitch = kBlockWeights + 4;    // floats per staged importance block (1040 B: 16 B mod 128)
constexpr int kEncHMaxCols = 40;                 // importance rows of at most this many blocks are staged

// fp64 -> IEEE binary16 bits, round to nearest even, saturating at +/-65504:
// 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits, subnormal quantum
// 2^-24; scaling by a power of two (ldexp) is exact and rint rounds ties to even.
__device__ __forceinline__ uint16_t enc_half_bits(double x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  const double a = fabs(x);
  if (a >= 65520.0) return sign | 0x7BFFu;
  if (a == 0.0) return sign;
  int e = 0;
  frexp(a, &e);                                   // a = m * 2^e, m in [0.5, 1)
  int ex = e - 1;
  if (ex >= -14) {
    double q = rint(ldexp(a, 10 - ex));           // in [1024, 2048]
    if (q >= 2048.0) {
      q = 1024.0;
      ex += 1;
    }
    if (ex > 15) return sign | 0x7BFFu;
    return sign | static_cast<uint16_t>(((ex + 15) << 10) | (static_cast<int>(q) - 1024));
  }
  return sign | static_cast<uint16_t>(rint(ldexp(a, 24)));
}

// Code of a group from its zero lane z and the lanes' signs (bit l of neg = lane l
// negative): t = sign of the first non-zero lane, bits 1 / 0 of the 4-bit code =
// whether the second / third non-zero lane differs from it.
__device__ __forceinline__ uint32_t enc_group_code(int z, uint32_t neg) {
  const int la = z == 0 ? 1 : 0;
  const int lb = z <= 1 ? 2 : 1;
  const int lc = z == 3 ? 2 : 3;
  const uint32_t sa = (neg >> la) & 1u, sb = (neg >> lb) & 1u, sc = (neg >> lc) & 1u;
  return (sa << 4) | (static_cast<uint32_t>(z) << 2) | ((sb ^ sa) << 1) | (sc ^ sa);
}

// Lane of least |w| (ties: lowest lane) and the sign mask (-0.0 counts as +).
__device__ __forceinline__ void enc_group_lane(const float* w, int& z, uint32_t& neg) {
  z = 0;
  float best = fabsf(w[0]);
  neg = w[0] < 0.f ? 1u : 0u;
#pragma unroll
  for (int l = 1; l < 4; ++l) {
    const float a = fabsf(w[l]);
    if (a < best) {
      best = a;
      z = l;
    }
    if (w[l] < 0.f) neg |= 1u << l;
  }
}

// Per-block state in registers, processed eight groups at a time by a
// runtime loop of eight iterations: the zero lanes (two bits per group, 128
// bits) and the sign masks (four bits per group, 256 bits) rotate by one
// chunk per iteration, so the chunk in use is always the low 16 bits of z[0]
// and all of neg[0] -- no indexing with a loop variable, hence no
// local-memory arrays.
struct EncState {
  uint32_t z[4];      // zero lanes: chunk c (groups 8c .. 8c+7) in bits 16 (c mod 2) of word c / 2, rotated
  uint32_t neg[8];    // sign masks: chunk c in word c (rotated)
  __device__ __forceinline__ void rotate(uint32_t z16) {   // z16 = the current chunk's (new) zero lanes
    z[0] = (z[0] >> 16) | (z[1] << 16);
    z[1] = (z[1] >> 16) | (z[2] << 16);
    z[2] = (z[2] >> 16) | (z[3] << 16);
    z[3] = (z[3] >> 16) | (z16 << 16);
    const uint32_t n0 = neg[0];
#pragma unroll
    for (int i = 0; i < 7; ++i) neg[i] = neg[i + 1];
    neg[7] = n0;
  }
};

// Sums of the weighted least-squares scale over the non-zero lanes, added in
// ascending k: num = sum h|w|, den = sum h, num1 = sum |w| (for a zero den).
struct WlsSums {
  double num = 0.0, den = 0.0, num1 = 0.0;
  __device__ __forceinline__ void add(double aw, double hk) {
    num = __dadd_rn(num, __dmul_rn(hk, aw));
    den = __dadd_rn(den, hk);
    num1 = __dadd_rn(num1, aw);
  }
  // d = num / den; with a zero denominator the mean |w| over the 192 non-zero lanes
  __device__ __forceinline__ double scale() const {
    if (den == 0.0) return __ddiv_rn(num1, static_cast<double>(kBlockWeights - kGroupsPerBlock));
    return __ddiv_rn(num, den);
  }
};

// Per-warp staging of W.  A warp encodes 32 consecutive blocks, one per lane.
// Chunk c of a block (groups 8c .. 8c+7: 128 bytes) is brought into a
// shared slot by the whole warp with 16-byte asynchronous copies, eight lanes
// per block, so one instruction moves four whole 128-byte lines; each lane
// then reads its own block's slot.  Slots are 144 bytes apart (16 B mod 128),
// so a quarter-warp's 16-byte reads from eight consecutive slots hit distinct
// banks.  A lane reading its own 1 KB global block directly would touch 32
// lines per warp instruction.  Each pass over a block goes through its eight
// chunks in order and the next pass starts again at chunk 0, so the copy of
// the next chunk is always (c + 1) mod 8.
constexpr int kEncWarps = kEncThreads / 32;
constexpr int kEncChunkBytes = 8 * 16;              // eight groups of one block
constexpr int kEncWPitch = kEncChunkBytes + 16;     // bytes per block slot
constexpr int kEncWBufBytes = 32 * kEncWPitch;      // one warp's 32 slots: 4608 B
constexpr int kEncWBufs = 2;                        // chunks in flight per warp
constexpr int kEncWBytes = kEncWarps * kEncWBufs * kEncWBufBytes;

__device__ __forceinline__ void enc_cp_async16(uint32_t dst, const float* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ float4 enc_lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}

struct EncWPipe {
  uint32_t buf;          // shared address of this warp's kEncWBufs buffers
  const float* wbase;    // first weight of the warp's first block
  int nblk;              // the warp's blocks inside the matrix (1..32)
  int lane;
  int q;                 // chunks consumed so far
  int total;             // chunks this warp will consume (8 per pass)

  __device__ __forceinline__ void fetch(int c, int slot) const {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int blk = 4 * j + (lane >> 3), part = lane & 7;
      if (blk < nblk)
        enc_cp_async16(buf + slot * kEncWBufBytes + blk * kEncWPitch + part * 16,
                       wbase + static_cast<long long>(blk) * kBlockWeights + 32 * c + 4 * part);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  __device__ __forceinline__ void start() { q = 0; if (total > 0) fetch(0, 0); }
  // Shared address of this lane's slot of chunk c (the q-th chunk overall).
  // With two buffers, first queue the next chunk into the other one (read
  // last during chunk q - 1, which every lane has released), then wait for
  // chunk c; with one, the next chunk is queued at the release.
  __device__ __forceinline__ uint32_t acquire(int c) {
    if (kEncWBufs == 2 && q + 1 < total) {
      fetch((c + 1) & 7, (q + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncwarp();
    return buf + (q % kEncWBufs) * kEncWBufBytes + lane * kEncWPitch;
  }
  __device__ __forceinline__ void release(int c) {
    __syncwarp();
    if (kEncWBufs == 1 && q + 1 < total) fetch((c + 1) & 7, 0);
    ++q;
  }
};
static_assert(kEncWBufs == 1 || kEncWBufs == 2, "one or two chunks in flight per warp");

// One thread encodes one block.  Its weights come through the warp's staged
// chunks, once per pass; the importances depend only on the column, so a CTA
// copies the whole importance row (up to kEncHMaxCols blocks) into shared
// memory once, at a pitch of 16 B mod 128 (longer rows are read from global
// memory).  Many blocks are in flight per SM, which is what hides the latency
// of the sequential fp64 sums.  Passes: lanes and checks; the scale of the
// initial lanes; then per Sherry round one pass that picks every group's zero
// lane with that round's d and, group by group in the same ascending order,
// adds the group's new non-zero lanes to the sums of the next d.  The
// additions happen in exactly the order of a separate fit over k = 0..255, so
// the bytes do not change.  Every lane of a warp runs every pass (the copies
// are shared); lanes past the matrix or with a non-finite block only skip
// their stores.
__global__ void __launch_bounds__(kEncThreads, 4)
encode_kernel(const float* __restrict__ W, const float* __restrict__ hcol, long long n_blocks, int nb, int mode,
              int rounds, uint8_t* __restrict__ out) {
  extern __shared__ __align__(16) uint8_t enc_smem[];   // [W slots][importance row]
  float4* hs4 = reinterpret_cast<float4*>(enc_smem + kEncWBytes);
  griddep_wait();
  griddep_launch_dependents();
  const bool use_h = mode == STQ1_ENC_SHERRY && hcol;
  const bool staged = use_h && nb <= kEncHMaxCols;
  if (staged) {
    const float4* g4 = reinterpret_cast<const float4*>(hcol);
    for (int i = threadIdx.x; i < nb * (kBlockWeights / 4); i += kEncThreads)
      hs4[(i / (kBlockWeights / 4)) * (kEncHPitch / 4) + i % (kBlockWeights / 4)] = __ldg(g4 + i);
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long bw0 = static_cast<long long>(blockIdx.x) * kEncThreads + 32 * warp;
  if (bw0 >= n_blocks) return;                    // whole warps only
  const long long b = bw0 + lane;
  const bool active = b < n_blocks;
  EncWPipe wp;
  wp.buf = smem_u32(enc_smem) + warp * kEncWBufs * kEncWBufBytes;
  wp.wbase = W + bw0 * kBlockWeights;
  wp.nblk = static_cast<int>(min(32LL, n_blocks - bw0));
  wp.lane = lane;
  wp.total = 8 * (mode == STQ1_ENC_PLAIN ? 1 : 2 + rounds);
  wp.start();
  // generic pointer: shared (staged) or global; read with plain loads
  const float4* h4 = !use_h ? nullptr
                     : staged ? hs4 + (b % nb) * (kEncHPitch / 4)
                              : reinterpret_cast<const float4*>(hcol + (b % nb) * kBlockWeights);

  // pass 1: zero lanes (least |w|), sign masks, amax, checks
  EncState st;
  bool finite = true, hany = false;
  float amax = 0.f;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    const uint32_t ws = wp.acquire(c);
    uint32_t z16 = 0u, n32 = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = enc_lds_f4(ws + 16 * i);
      const float wg[4] = {v.x, v.y, v.z, v.w};
      int zl;
      uint32_t neg;
      enc_group_lane(wg, zl, neg);
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        finite = finite && isfinite(wg[l]);
        amax = fmaxf(amax, fabsf(wg[l]));
      }
      if (h4) {
        const float4 hv = h4[8 * c + i];
        const float hg[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          finite = finite && isfinite(hg[l]) && hg[l] >= 0.f;
          hany = hany || hg[l] != 0.f;
        }
      }
      z16 |= static_cast<uint32_t>(zl) << (2 * i);
      n32 |= neg << (4 * i);
    }
    wp.release(c);
    // fill the rotating state in chunk order: after 8 iterations chunk c sits in its place
    st.neg[0] = n32;
    st.rotate(z16);
  }
  uint16_t* o16 = reinterpret_cast<uint16_t*>(out + b * kBlockBytes);   // 2-byte aligned
  const bool store = active && finite;
  if (active && !finite) {
    flag_error(STQ1_DEV_BAD_VALUE);
    for (int i = 0; i < kBlockBytes / 2; ++i) o16[i] = 0;
  }
  if (!hany) h4 = nullptr;                       // an all-zero importance block uses h = 1

  uint16_t d_bits;
  if (mode == STQ1_ENC_PLAIN) {
    d_bits = enc_half_bits(static_cast<double>(amax));
  } else {
    // pass 2: the scale of the initial lanes
    WlsSums sums;
#pragma unroll 1
    for (int c = 0; c < 8; ++c) {
      const uint32_t ws = wp.acquire(c);
      const uint32_t z16 = st.z[0] & 0xFFFFu;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = enc_lds_f4(ws + 16 * i);
        const float wg[4] = {v.x, v.y, v.z, v.w};
        float hg[4] = {1.f, 1.f, 1.f, 1.f};
        if (h4) {
          const float4 hv = h4[8 * c + i];
          hg[0] = hv.x; hg[1] = hv.y; hg[2] = hv.z; hg[3] = hv.w;
        }
        const int zg = static_cast<int>((z16 >> (2 * i)) & 3u);
#pragma unroll
        for (int l = 0; l < 4; ++l)
          if (l != zg) sums.add(fabs(static_cast<double>(wg[l])), static_cast<double>(hg[l]));
      }
      wp.release(c);
      st.rotate(z16);
    }
    double d = sums.scale();
    // one pass per round: zero lanes at d, and the sums of the next d
#pragma unroll 1
    for (int r = 0; r < rounds; ++r) {
      WlsSums next;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        const uint32_t ws = wp.acquire(c);
        uint32_t z16 = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 v = enc_lds_f4(ws + 16 * i);
          const float wg[4] = {v.x, v.y, v.z, v.w};
          float hg[4] = {1.f, 1.f, 1.f, 1.f};
          if (h4) {
            const float4 hv = h4[8 * c + i];
            hg[0] = hv.x; hg[1] = hv.y; hg[2] = hv.z; hg[3] = hv.w;
          }
          double aw[4];
          int best_l = 0;
          double best = 0.0;
#pragma unroll
          for (int l = 0; l < 4; ++l) {
            aw[l] = fabs(static_cast<double>(wg[l]));
            const double hd = __dmul_rn(static_cast<double>(hg[l]), d);
            const double delta = __dmul_rn(hd, __dsub_rn(__dmul_rn(2.0, aw[l]), d));
            if (l == 0 || delta < best) {
              best = delta;
              best_l = l;
            }
          }
          z16 |= static_cast<uint32_t>(best_l) << (2 * i);
#pragma unroll
          for (int l = 0; l < 4; ++l)
            if (l != best_l) next.add(aw[l], static_cast<double>(hg[l]));
        }
        wp.release(c);
        st.rotate(z16);
      }
      d = next.scale();
    }
    d_bits = enc_half_bits(d);
  }
  if (!store) return;
  // pack: d, qs (even group in the low nibble), qh (group g at bit g & 7 of byte g >> 3);
  // chunk c gives qs bytes 4c .. 4c+3 and qh byte c (the block starts on a 2-byte boundary)
  o16[0] = d_bits;
  uint32_t qh2 = 0u;
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    const uint32_t z16 = st.z[0] & 0xFFFFu;
    const uint32_t n32 = st.neg[0];
    uint32_t qs = 0u, qh = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t code = enc_group_code(static_cast<int>((z16 >> (2 * i)) & 3u), (n32 >> (4 * i)) & 15u);
      qs |= (code & 15u) << (4 * i);
      qh |= ((code >> 4) & 1u) << i;
    }
    o16[1 + 2 * c] = static_cast<uint16_t>(qs & 0xFFFFu);
    o16[2 + 2 * c] = static_cast<uint16_t>(qs >> 16);
    qh2 |= qh << (8 * (c & 1));
    if (c & 1) {
      o16[17 + (c >> 1)] = static_cast<uint16_t>(qh2);
      qh2 = 0u;
    }
    st.rotate(z16);
  }
}

// Dynamic shared memory of a launch: the warps' W slots, then the staged
// importance row, if any.
inline size_t encode_smem_bytes(int nb, bool staged_h) {
  return kEncWBytes + (staged_h ? static_cast<size_t>(nb) * kEncHPitch * sizeof(float) : 0);
}
inline size_t encode_smem_bytes_max() {
  return kEncWBytes + static_cast<size_t>(kEncHMaxCols) * kEncHPitch * sizeof(float);
}

}  // namespace stq1
