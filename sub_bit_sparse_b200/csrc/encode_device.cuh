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

constexpr int kEncThreads = 64;                  // blocks per CTA
constexpr int kEncPitch = kBlockWeights + 1;     // floats per staged block (odd: conflict-free reads)

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

// Weighted least-squares scale over the non-zero lanes, k ascending; with a zero
// denominator the unweighted mean of |w| over the 192 non-zero lanes.
__device__ __forceinline__ double enc_wls(const float* w, const float* h, const uint8_t* z) {
  double num = 0.0, den = 0.0, num1 = 0.0;
  for (int k = 0; k < kBlockWeights; ++k) {
    if ((k & 3) == z[k >> 2]) continue;
    const double aw = fabs(static_cast<double>(w[k]));
    const double hk = h ? static_cast<double>(h[k]) : 1.0;
    num = __dadd_rn(num, __dmul_rn(hk, aw));
    den = __dadd_rn(den, hk);
    num1 = __dadd_rn(num1, aw);
  }
  if (den == 0.0) return __ddiv_rn(num1, static_cast<double>(kBlockWeights - kGroupsPerBlock));
  return __ddiv_rn(num, den);
}

__global__ void __launch_bounds__(kEncThreads)
encode_kernel(const float* __restrict__ W, const float* __restrict__ hcol, long long n_blocks, int nb, int mode,
              int rounds, uint8_t* __restrict__ out) {
  extern __shared__ float sw[];                   // [kEncThreads][kEncPitch]
  const long long b0 = static_cast<long long>(blockIdx.x) * kEncThreads;
  const int nblk = static_cast<int>(min(static_cast<long long>(kEncThreads), n_blocks - b0));
  griddep_wait();
  griddep_launch_dependents();
  // the CTA's blocks are one contiguous span of W (row-major [N, K], blocks in storage order)
  const float4* src = reinterpret_cast<const float4*>(W + b0 * kBlockWeights);
  for (int f = threadIdx.x; f < nblk * (kBlockWeights / 4); f += kEncThreads) {
    const float4 v = __ldg(src + f);
    float* d = sw + (f >> 6) * kEncPitch + 4 * (f & 63);
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
  __syncthreads();
  if (threadIdx.x >= nblk) return;
  const long long b = b0 + threadIdx.x;
  const float* w = sw + threadIdx.x * kEncPitch;
  const float* h = (mode == STQ1_ENC_SHERRY && hcol) ? hcol + (b % nb) * kBlockWeights : nullptr;

  bool finite = true;
  for (int k = 0; k < kBlockWeights; ++k) finite = finite && isfinite(w[k]);
  bool hany = false;
  if (h) {
    for (int k = 0; k < kBlockWeights; ++k) {
      const float hk = h[k];
      finite = finite && isfinite(hk) && hk >= 0.f;
      hany = hany || hk != 0.f;
    }
    if (!hany) h = nullptr;                      // an all-zero importance block uses h = 1
  }
  uint8_t* ob = out + b * kBlockBytes;
  if (!finite) {
    flag_error(STQ1_DEV_BAD_VALUE);
    for (int i = 0; i < kBlockBytes; ++i) ob[i] = 0;
    return;
  }

  uint8_t z[kGroupsPerBlock];
  uint32_t negs[kGroupsPerBlock / 8];             // 4 bits per group
  for (int i = 0; i < kGroupsPerBlock / 8; ++i) negs[i] = 0u;
  for (int g = 0; g < kGroupsPerBlock; ++g) {
    int zl;
    uint32_t neg;
    enc_group_lane(w + 4 * g, zl, neg);
    z[g] = static_cast<uint8_t>(zl);
    negs[g >> 3] |= neg << (4 * (g & 7));
  }
  uint16_t d_bits;
  if (mode == STQ1_ENC_PLAIN) {
    float amax = 0.f;
    for (int k = 0; k < kBlockWeights; ++k) amax = fmaxf(amax, fabsf(w[k]));
    d_bits = enc_half_bits(static_cast<double>(amax));
  } else {
    for (int r = 0; r < rounds; ++r) {
      const double d = enc_wls(w, h, z);
      for (int g = 0; g < kGroupsPerBlock; ++g) {
        int best_l = 0;
        double best = 0.0;
#pragma unroll
        for (int l = 0; l < 4; ++l) {
          const int k = 4 * g + l;
          const double aw = fabs(static_cast<double>(w[k]));
          const double hd = __dmul_rn(h ? static_cast<double>(h[k]) : 1.0, d);
          const double delta = __dmul_rn(hd, __dsub_rn(__dmul_rn(2.0, aw), d));
          if (l == 0 || delta < best) {
            best = delta;
            best_l = l;
          }
        }
        z[g] = static_cast<uint8_t>(best_l);
      }
    }
    d_bits = enc_half_bits(enc_wls(w, h, z));
  }
  // pack: d, qs (even group in the low nibble), qh (group g at bit g & 7 of byte g >> 3)
  uint8_t blk[kBlockBytes];
  blk[0] = static_cast<uint8_t>(d_bits & 0xFF);
  blk[1] = static_cast<uint8_t>(d_bits >> 8);
  for (int i = 2; i < kBlockBytes; ++i) blk[i] = 0;
  for (int g = 0; g < kGroupsPerBlock; ++g) {
    const uint32_t c = enc_group_code(z[g], (negs[g >> 3] >> (4 * (g & 7))) & 15u);
    blk[kOffQs + (g >> 1)] |= static_cast<uint8_t>((c & 15u) << (4 * (g & 1)));
    blk[kOffQh + (g >> 3)] |= static_cast<uint8_t>(((c >> 4) & 1u) << (g & 7));
  }
  // the block starts on a 2-byte boundary: 21 halfword stores
  uint16_t* o16 = reinterpret_cast<uint16_t*>(ob);
  for (int i = 0; i < kBlockBytes / 2; ++i) o16[i] = static_cast<uint16_t>(blk[2 * i] | (blk[2 * i + 1] << 8));
}

inline size_t encode_smem_bytes() { return static_cast<size_t>(kEncThreads) * kEncPitch * sizeof(float); }

}  // namespace stq1
