// Host-side STQ1_0 encoders behind stq1_quantize_ref.
//
// Plain encoder: amax scale ("AngelSlim Shrinks Tencent's 1.5TB Hy4-Preview to
// 214 GiB at 6x Compression", bullet list: the improved encoder replaces amax
// scaling).  Sherry encoder: alternating weighted-least-squares scale fit and
// importance-weighted zero placement, three rounds on the pages
// (lemmy.durstig.online post 66506, "Scale and zero position are fit
// together").  Block format: "How STQ1_0 works" (same AngelSlim page).
//
// Every real-valued step is IEEE fp64 with a fixed evaluation order, and this
// file is compiled with -ffp-contract=off, so the bytes do not depend on the
// compiler or the thread count.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "../../include/stq1.h"

namespace {

constexpr int kBlock = 256;
constexpr int kGroups = 64;
constexpr int kBlockBytes = 42;

// fp64 -> IEEE binary16 bits, round to nearest even, saturating at +/-65504.
// Built from the binary16 definition: 1 sign bit, 5 exponent bits (bias 15),
// 10 fraction bits; subnormals have quantum 2^-24.  Scaling by a power of two
// (ldexp) is exact, and nearbyint rounds ties to even in the default mode.
uint16_t half_bits(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000u : 0u;
  double a = std::fabs(x);
  if (a >= 65520.0) return sign | 0x7BFFu;   // at or past the rounding point to +inf
  if (a == 0.0) return sign;
  int e = 0;
  std::frexp(a, &e);                          // a = m * 2^e, m in [0.5, 1)
  int ex = e - 1;                             // a = 1.f * 2^ex
  if (ex >= -14) {
    double q = std::nearbyint(std::ldexp(a, 10 - ex));   // in [1024, 2048]
    if (q >= 2048.0) { q = 1024.0; ex += 1; }
    if (ex > 15) return sign | 0x7BFFu;
    return sign | static_cast<uint16_t>(((ex + 15) << 10) | (static_cast<int>(q) - 1024));
  }
  double q = std::nearbyint(std::ldexp(a, 24));          // subnormal quantum 2^-24
  return sign | static_cast<uint16_t>(q);                // q == 1024 is the least normal
}

// Code of a group from its zero lane z and the lanes' signs (bit l of neg =
// lane l negative): t = sign of the first non-zero lane, bit 1 / bit 0 of the
// 4-bit code = whether the second / third non-zero lane differs from it.
inline uint8_t group_code(int z, unsigned neg) {
  int lanes[3];
  int m = 0;
  for (int l = 0; l < 4; ++l)
    if (l != z) lanes[m++] = l;
  const unsigned sa = (neg >> lanes[0]) & 1u;
  const unsigned sb = (neg >> lanes[1]) & 1u;
  const unsigned sc = (neg >> lanes[2]) & 1u;
  return static_cast<uint8_t>((sa << 4) | (z << 2) | ((sb ^ sa) << 1) | (sc ^ sa));
}

void pack_block(uint16_t d_bits, const uint8_t* codes, uint8_t* out) {
  std::memset(out, 0, kBlockBytes);
  out[0] = static_cast<uint8_t>(d_bits & 0xFF);
  out[1] = static_cast<uint8_t>(d_bits >> 8);
  for (int g = 0; g < kGroups; ++g) {
    out[2 + (g >> 1)] |= static_cast<uint8_t>((codes[g] & 0xF) << (4 * (g & 1)));
    out[34 + (g >> 3)] |= static_cast<uint8_t>(((codes[g] >> 4) & 1) << (g & 7));
  }
}

// Lane of least |w| in a group; ties go to the lowest lane.
inline int argmin_abs(const float* w) {
  int z = 0;
  float best = std::fabs(w[0]);
  for (int l = 1; l < 4; ++l) {
    const float a = std::fabs(w[l]);
    if (a < best) { best = a; z = l; }
  }
  return z;
}

inline unsigned neg_mask(const float* w) {
  unsigned m = 0;
  for (int l = 0; l < 4; ++l)
    if (w[l] < 0.0f) m |= 1u << l;   // -0.0f < 0 is false: counts as positive
  return m;
}

void encode_block_plain(const float* w, uint8_t* out) {
  float amax = 0.0f;
  for (int k = 0; k < kBlock; ++k) amax = std::max(amax, std::fabs(w[k]));
  uint8_t codes[kGroups];
  for (int g = 0; g < kGroups; ++g)
    codes[g] = group_code(argmin_abs(w + 4 * g), neg_mask(w + 4 * g));
  pack_block(half_bits(static_cast<double>(amax)), codes, out);
}

// Weighted least squares scale over the non-zero lanes (k ascending).
double wls_scale(const double* aw, const double* h, const int* z) {
  double num = 0.0, den = 0.0, num1 = 0.0;
  for (int k = 0; k < kBlock; ++k) {
    if ((k & 3) == z[k >> 2]) continue;
    num += h[k] * aw[k];
    den += h[k];
    num1 += aw[k];
  }
  if (den == 0.0) return num1 / static_cast<double>(kBlock - kGroups);
  return num / den;
}

void encode_block_sherry(const float* w, const float* hcol, int rounds, uint8_t* out) {
  double aw[kBlock], h[kBlock];
  bool any = false;
  for (int k = 0; k < kBlock; ++k) {
    aw[k] = std::fabs(static_cast<double>(w[k]));
    h[k] = hcol ? static_cast<double>(hcol[k]) : 1.0;
    any = any || (h[k] != 0.0);
  }
  if (!any)
    for (int k = 0; k < kBlock; ++k) h[k] = 1.0;
  int z[kGroups];
  for (int g = 0; g < kGroups; ++g) z[g] = argmin_abs(w + 4 * g);
  for (int r = 0; r < rounds; ++r) {
    const double d = wls_scale(aw, h, z);
    for (int g = 0; g < kGroups; ++g) {
      int best_l = 0;
      double best = 0.0;
      for (int l = 0; l < 4; ++l) {
        const int k = 4 * g + l;
        const double hd = h[k] * d;
        const double delta = hd * (2.0 * aw[k] - d);
        if (l == 0 || delta < best) { best = delta; best_l = l; }
      }
      z[g] = best_l;
    }
  }
  const double d = wls_scale(aw, h, z);
  uint8_t codes[kGroups];
  for (int g = 0; g < kGroups; ++g) codes[g] = group_code(z[g], neg_mask(w + 4 * g));
  pack_block(half_bits(d), codes, out);
}

}  // namespace

extern "C" int stq1_quantize_ref(const float* W, const float* h, int64_t N, int64_t K, int mode,
                                 int rounds, uint8_t* out, int threads) {
  if (!W || !out) return STQ1_ERR_NULL;
  if (N <= 0 || K <= 0 || (K % kBlock) != 0) return STQ1_ERR_SHAPE;
  if (mode != STQ1_ENC_PLAIN && mode != STQ1_ENC_SHERRY) return STQ1_ERR_ARG;
  if (mode == STQ1_ENC_SHERRY && (rounds < 0 || rounds > 1000)) return STQ1_ERR_ARG;
  const int64_t total = N * K;
  if (total / K != N) return STQ1_ERR_SHAPE;
  const int64_t nb = K / kBlock;
  const int64_t n_blocks = N * nb;

  int nt = threads > 0 ? threads : static_cast<int>(std::thread::hardware_concurrency());
  nt = std::max(1, std::min<int>(nt, 256));
  nt = static_cast<int>(std::min<int64_t>(nt, std::max<int64_t>(1, n_blocks / 64)));

  if (mode == STQ1_ENC_SHERRY && h) {
    for (int64_t k = 0; k < K; ++k)
      if (!std::isfinite(h[k]) || h[k] < 0.0f) return STQ1_ERR_VALUE;
  }
  std::atomic<int> bad{0};
  auto work = [&](int tid) {
    const int64_t b0 = n_blocks * tid / nt, b1 = n_blocks * (tid + 1) / nt;
    for (int64_t b = b0; b < b1; ++b) {
      const float* wb = W + b * kBlock;   // row-major [N, K]: block b is contiguous
      bool finite = true;
      for (int k = 0; k < kBlock; ++k) finite = finite && std::isfinite(wb[k]);
      if (!finite) { bad.store(1); return; }
      uint8_t* ob = out + b * kBlockBytes;
      if (mode == STQ1_ENC_PLAIN) {
        encode_block_plain(wb, ob);
      } else {
        const float* hb = h ? h + (b % nb) * kBlock : nullptr;
        encode_block_sherry(wb, hb, rounds, ob);
      }
    }
  };
  if (nt == 1) {
    work(0);
  } else {
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int t = 0; t < nt; ++t) pool.emplace_back(work, t);
    for (auto& th : pool) th.join();
  }
  return bad.load() ? STQ1_ERR_VALUE : STQ1_OK;
}

extern "C" int stq1_version(void) { return 100; }
