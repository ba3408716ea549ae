// Routing sort, dequantization and the direct (generic-shape) GEMV.
#pragma once

#include "device_common.cuh"

namespace stq1 {

// ---------------------------------------------------------------------------
// Routing: group token-slot pairs by expert (top-k of E routed experts, lemmy
// post "Precision follows weight sensitivity": 256 routed experts, top-8).
// One CTA: histogram of ids, exclusive scans of pair counts and of tile
// counts, tile table, then a scatter of pair ids into per-expert segments.
// A pair p = t * topk + s.  Pairs with an id outside [0, E) get y = 0 and set
// STQ1_DEV_BAD_EXPERT, unless skip_foreign (expert parallelism: ids of
// experts another rank holds) makes them a silent zero.  Order inside a segment is unspecified (it does not
// change any result: every output row is computed on its own).
// tile_info[4 * i] = expert, first pair offset, pair count (<= tile_tokens), 0.
// n_tiles[0] = number of tiles, n_tiles[1] = number of pairs with a valid id.
// With small_max > 0, an expert with at most small_max pairs gets one tile in
// a second table, tile_small (same format), counted in n_tiles[2]; the other
// experts' tiles go to tile_info as before.  Decode sends the two tables to
// different kernels.
// inv (optional): inv[p] = the position of pair p in pairs_out, or -1 for a
// pair whose id is out of range -- the row of p in outputs that are stored
// compactly, in pairs_out order.  y (optional): the rows of out-of-range
// pairs are zeroed in y [n_pairs, N] (a compact caller passes nullptr).
// tiles_cap / small_cap = entries tile_info / tile_small hold (the debug build
// checks every write against them).
// ---------------------------------------------------------------------------
constexpr int kRouteThreads = 1024;

__global__ void __launch_bounds__(kRouteThreads)
route_kernel(const int32_t* __restrict__ ids, int n_pairs, int E, int tile_tokens, int small_max,
             int* __restrict__ pairs_out, int* __restrict__ tile_info, int* __restrict__ tile_small,
             int* __restrict__ n_tiles, int* __restrict__ inv, float* __restrict__ y, int N, int skip_foreign,
             int tiles_cap, int small_cap) {
  extern __shared__ int sm[];
  __shared__ int s_bad[kRouteThreads];      // out-of-range pairs to zero, this round
  __shared__ int s_nbad;
  griddep_wait();           // ids may come from the previous kernel in the stream
  griddep_launch_dependents();
  int* cnt = sm;            // [E]
  int* off = sm + E;        // [E]
  int* tst = sm + 2 * E;    // [E] first tile of the expert in its table
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  // Rounds of blockDim pairs: count valid ids; the rows of invalid ones are
  // zeroed by the whole block (float4 stores along each row).
  for (int p0 = 0; p0 < n_pairs; p0 += blockDim.x) {
    if (threadIdx.x == 0) s_nbad = 0;
    __syncthreads();
    const int p = p0 + static_cast<int>(threadIdx.x);
    if (p < n_pairs) {
      const int e = ids[p];
      if (e < 0 || e >= E) {
        if (!skip_foreign) flag_error(STQ1_DEV_BAD_EXPERT);
        if (inv) inv[p] = -1;
        if (y) s_bad[atomicAdd(&s_nbad, 1)] = p;
      } else {
        atomicAdd(&cnt[e], 1);
      }
    }
    __syncthreads();
    const int nbad = s_nbad;
    if (nbad > 0) {
      for (long long i = threadIdx.x; i < static_cast<long long>(nbad) * N; i += blockDim.x) {
        const int r = static_cast<int>(i / N);
        const int j = static_cast<int>(i - static_cast<long long>(r) * N);
        y[static_cast<long long>(s_bad[r]) * N + j] = 0.f;
      }
    }
    __syncthreads();
  }
  // tiles of an expert with c pairs: in the small table one (c <= small_max),
  // else ceil(c / tile_tokens) in the main table
  auto big_tiles = [&](int c) { return c > small_max ? (c + tile_tokens - 1) / tile_tokens : 0; };
  auto small_tiles = [&](int c) { return (c > 0 && c <= small_max) ? 1 : 0; };
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int lo = min(E, lane * per), hi = min(E, lo + per);
    int s1 = 0, s2 = 0, s3 = 0;
    for (int e = lo; e < hi; ++e) {
      s1 += cnt[e];
      s2 += big_tiles(cnt[e]);
      s3 += small_tiles(cnt[e]);
    }
    int i1 = s1, i2 = s2, i3 = s3;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v1 = __shfl_up_sync(0xffffffffu, i1, d);
      const int v2 = __shfl_up_sync(0xffffffffu, i2, d);
      const int v3 = __shfl_up_sync(0xffffffffu, i3, d);
      if (lane >= d) { i1 += v1; i2 += v2; i3 += v3; }
    }
    int r1 = i1 - s1, r2 = i2 - s2, r3 = i3 - s3;
    for (int e = lo; e < hi; ++e) {
      off[e] = r1;
      tst[e] = small_tiles(cnt[e]) ? r3 : r2;
      r1 += cnt[e];
      r2 += big_tiles(cnt[e]);
      r3 += small_tiles(cnt[e]);
    }
    if (lane == 31) {
      n_tiles[0] = i2;       // tiles in the main table
      n_tiles[1] = i1;       // pairs with a valid expert id
      n_tiles[2] = i3;       // tiles in the small table
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = cnt[e];
    if (small_tiles(c)) {
      if (!dbg_check(tst[e] >= 0 && tst[e] < small_cap)) continue;
      int* ti = tile_small + 4 * tst[e];
      ti[0] = e;
      ti[1] = off[e];
      ti[2] = c;
      ti[3] = 0;
      continue;
    }
    const int nt = big_tiles(c);
    for (int k = 0; k < nt; ++k) {
      if (!dbg_check(tst[e] + k >= 0 && tst[e] + k < tiles_cap)) break;
      int* ti = tile_info + 4 * (tst[e] + k);
      ti[0] = e;
      ti[1] = off[e] + k * tile_tokens;
      ti[2] = min(tile_tokens, c - k * tile_tokens);
      ti[3] = 0;
    }
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int e = ids[p];
    if (e < 0 || e >= E) continue;
    const int pos = atomicSub(&cnt[e], 1) - 1;
    if (!dbg_check(pos >= 0 && off[e] + pos < n_pairs)) continue;
    pairs_out[off[e] + pos] = p;
    if (inv) inv[p] = off[e] + pos;
  }
}

// ---------------------------------------------------------------------------
// Dequantization: one thread per group of four weights, 8-byte stores.
// W^ = bf16_rne(fp32(d)) with the pattern's sign; zero lanes are +0.0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
dequant_kernel(const uint8_t* __restrict__ W, uint16_t* __restrict__ out, long long n_groups) {
  for (long long gid = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; gid < n_groups;
       gid += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long blk = gid >> 6;
    const int g = static_cast<int>(gid & 63);
    const uint8_t* B = W + blk * kBlockBytes;
    const unsigned short dbits = static_cast<unsigned short>(B[kOffD] | (B[kOffD + 1] << 8));
    const unsigned n = (B[kOffQs + (g >> 1)] >> (4 * (g & 1))) & 15u;
    const unsigned t = (B[kOffQh + (g >> 3)] >> (g & 7)) & 1u;
    const __nv_bfloat16 db = __float2bfloat16_rn(__half2float(__ushort_as_half(dbits)));
    const uint32_t mag = __bfloat16_as_ushort(db);
    int v[4];
    code_pattern(n | (t << 4), v);
    uint32_t o[4];
#pragma unroll
    for (int l = 0; l < 4; ++l) o[l] = v[l] == 0 ? 0u : (v[l] > 0 ? mag : (mag ^ 0x8000u));
    uint2 pk;
    pk.x = o[0] | (o[1] << 16);
    pk.y = o[2] | (o[3] << 16);
    *reinterpret_cast<uint2*>(out + (blk << 8) + 4 * g) = pk;
  }
}

// ---------------------------------------------------------------------------
// Direct GEMV for shapes the table kernel does not take (an odd number of
// blocks per row): one warp per output element, lanes stride over blocks and
// decode each group arithmetically.  Correct for any K % 256 == 0; slow.
// MoE use: ids != nullptr, pair p reads expert ids[p] and token p / topk.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
direct_gemv_kernel(const uint8_t* __restrict__ W, long long expert_bytes, int E,
                   const uint16_t* __restrict__ x, const int32_t* __restrict__ ids, int topk,
                   const float* __restrict__ route_w, int flags, float* __restrict__ y, int N,
                   int K, int rows_out) {
  const bool skip_foreign = (flags & STQ1_MOE_SKIP_FOREIGN) != 0;
  const int nb = K / kBlockWeights;
  const long long gw = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(rows_out) * N) return;
  const int p = static_cast<int>(gw / N);
  const int j = static_cast<int>(gw % N);
  int e = 0;
  if (ids) {
    e = ids[p];
    if (e < 0 || e >= E) {
      if (lane == 0) {
        y[static_cast<long long>(p) * N + j] = 0.f;
        if (!skip_foreign) flag_error(STQ1_DEV_BAD_EXPERT);
      }
      return;
    }
  }
  const int tok = ids ? p / topk : p;
  const uint8_t* Wr = W + e * expert_bytes + static_cast<long long>(j) * nb * kBlockBytes;
  const uint16_t* xr = x + static_cast<long long>(tok) * K;
  float acc = 0.f;
  for (int b = lane; b < nb; b += 32) {
    const uint8_t* B = Wr + static_cast<long long>(b) * kBlockBytes;
    const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(B[0] | (B[1] << 8))));
    float s = 0.f;
    for (int g = 0; g < kGroupsPerBlock; ++g) {
      const unsigned n = (B[kOffQs + (g >> 1)] >> (4 * (g & 1))) & 15u;
      const unsigned t = (B[kOffQh + (g >> 3)] >> (g & 7)) & 1u;
      int v[4];
      code_pattern(n | (t << 4), v);
#pragma unroll
      for (int l = 0; l < 4; ++l) {
        const float xv = bf16_bits_to_f32(xr[b * kBlockWeights + 4 * g + l]);
        if (v[l] > 0) s += xv;
        else if (v[l] < 0) s -= xv;
      }
    }
    acc = fmaf(d, s, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    if ((flags & STQ1_MOE_WEIGHT_UP) && j >= N / 2 && route_w) acc *= route_w[p];
    y[static_cast<long long>(p) * N + j] = acc;
  }
}

// ---------------------------------------------------------------------------
// After gate/up: SwiGLU and the top-k combine.
// ---------------------------------------------------------------------------

// fp64 -> bf16 bits, one rounding (nearest, ties to even): 8 significant bits,
// exponent bias 127, subnormal quantum 2^-133, overflow to infinity.  ldexp is
// exact and rint rounds ties to even.
__device__ __forceinline__ uint16_t bf16_bits_from_f64(double x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  const double a = fabs(x);
  if (isnan(x)) return 0x7FC0u;
  if (a == 0.0) return sign;
  int e = 0;
  frexp(a, &e);                                   // a = m * 2^e, m in [0.5, 1)
  int ex = e - 1;
  if (ex >= -126) {
    double q = rint(ldexp(a, 7 - ex));            // in [128, 256]
    if (q >= 256.0) {
      q = 128.0;
      ex += 1;
    }
    if (ex > 127) return sign | 0x7F80u;
    return sign | static_cast<uint16_t>(((ex + 127) << 7) | (static_cast<int>(q) - 128));
  }
  return sign | static_cast<uint16_t>(rint(ldexp(a, 133)));
}

// act[p, j] = bf16(SiLU(g) * u), g = y[p, j], u = y[p, half + j], SiLU(v) =
// v / (1 + e^-v), in fp64 (the down projection's bf16 input, rounded once).
__global__ void __launch_bounds__(256)
swiglu_kernel(const float* __restrict__ y, uint16_t* __restrict__ act, long long P, int half,
              const int* __restrict__ n_rows) {
  griddep_wait();
  griddep_launch_dependents();
  // n_rows (optional, device): only the first *n_rows rows are in use
  const long long rows = n_rows ? min(P, static_cast<long long>(*n_rows)) : P;
  const long long total = rows * half;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += 256LL * gridDim.x) {
    const long long p = i / half;
    const int j = static_cast<int>(i - p * half);
    const double g = y[p * 2 * half + j];
    const double u = y[p * 2 * half + half + j];
    const double s = g / (1.0 + exp(-g));
    act[i] = bf16_bits_from_f64(s * u);
  }
}

// ids[i] - begin: the routing ids of one rank's expert range (expert parallelism).
__global__ void __launch_bounds__(256)
shift_ids_kernel(const int32_t* __restrict__ ids, int32_t* __restrict__ out, long long n, int begin) {
  griddep_wait();
  griddep_launch_dependents();
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n; i += 256LL * gridDim.x) out[i] = ids[i] - begin;
}

// out[t, h] = sum_s w[t, s] * y[t, s, h] (plain sum without w), fp32 in slot order.
__global__ void __launch_bounds__(256)
combine_kernel(const float* __restrict__ y, const float* __restrict__ w, float* __restrict__ out, long long T,
               int topk, int H) {
  griddep_wait();
  griddep_launch_dependents();
  const long long total = T * H;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += 256LL * gridDim.x) {
    const long long t = i / H;
    const int h = static_cast<int>(i - t * H);
    const float* yt = y + t * topk * H + h;
    float acc = 0.f;
    for (int s = 0; s < topk; ++s) acc = w ? fmaf(w[t * topk + s], yt[static_cast<long long>(s) * H], acc)
                                           : acc + yt[static_cast<long long>(s) * H];
    out[i] = acc;
  }
}

// Combine of one rank's compact outputs: out[t, h] = sum over slots s whose
// pair is local (inv[t * topk + s] >= 0) of w[t, s] * y[inv[...], h] (plain
// sum without w), fp32 in slot order; 0 where no slot is local.
__global__ void __launch_bounds__(256)
combine_compact_kernel(const float* __restrict__ y, const float* __restrict__ w, const int* __restrict__ inv,
                       float* __restrict__ out, long long T, int topk, int H, long long y_rows) {
  griddep_wait();
  griddep_launch_dependents();
  const long long total = T * H;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < total; i += 256LL * gridDim.x) {
    const long long t = i / H;
    const int h = static_cast<int>(i - t * H);
    float acc = 0.f;
    for (int s = 0; s < topk; ++s) {
      const int r = inv[t * topk + s];
      if (r < 0 || !dbg_check(r < y_rows)) continue;   // (debug build: y_rows = rows y holds)
      const float v = y[static_cast<long long>(r) * H + h];
      acc = w ? fmaf(w[t * topk + s], v, acc) : acc + v;
    }
    out[i] = acc;
  }
}

// ---------------------------------------------------------------------------
// Expert parallelism with token dispatch.  The E experts are split into world
// contiguous ranges, the first E % world ranks holding one more (the split of
// sub_bit_sparse_b200.ep.expert_range).  Pairs p = t * topk + s are grouped by
// the rank that owns expert ids[p], in rank order.  Inside a rank's segment
// the order is that of the atomic slot counters; it changes no result, since
// every row is computed on its own and the combine adds a token's rows in
// slot order through inv.
// ---------------------------------------------------------------------------
__device__ __forceinline__ int expert_owner(int e, int E, int world) {
  const int base = E / world, extra = E % world;
  const int split = extra * (base + 1);
  return e < split ? e / (base + 1) : extra + (e - split) / base;
}
__device__ __forceinline__ int expert_begin(int r, int E, int world) {
  const int base = E / world, extra = E % world;
  return r * base + min(r, extra);
}

// order[i] = pair sent i-th; inv[p] = i; counts[r] = pairs sent to rank r,
// counts[world] = all pairs sent; local[i] = the expert id of pair order[i]
// within its owner's range.  Invalid ids (outside [0, E)) are sent nowhere
// (inv = -1) and flagged in the device error word.
constexpr int kDispatchThreads = 1024;
__global__ void __launch_bounds__(kDispatchThreads)
ep_dispatch_kernel(const int32_t* __restrict__ ids, int n_pairs, int E, int world, int* __restrict__ order,
                   int* __restrict__ inv, int* __restrict__ counts, int32_t* __restrict__ local) {
  extern __shared__ int sm[];
  int* cnt = sm;                  // [world]
  int* cur = sm + world;          // [world] next slot of each rank
  griddep_wait();
  griddep_launch_dependents();
  for (int r = threadIdx.x; r < world; r += blockDim.x) cnt[r] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[expert_owner(e, E, world)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int r = 0; r < world; ++r) {
      cur[r] = run;
      counts[r] = cnt[r];
      run += cnt[r];
    }
    counts[world] = run;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) {
    const int e = ids[p];
    if (e < 0 || e >= E) {
      inv[p] = -1;
      flag_error(STQ1_DEV_BAD_EXPERT);
      continue;
    }
    const int r = expert_owner(e, E, world);
    const int i = atomicAdd(&cur[r], 1);
    if (!dbg_check(r >= 0 && r < world && i >= 0 && i < n_pairs)) continue;
    order[i] = p;
    inv[p] = i;
    local[i] = e - expert_begin(r, E, world);
  }
}

// Rows of one dispatch: xs[i] = x[order[i] / topk] (bf16 rows of K), ws[i] =
// w[order[i]] (w optional).  One CTA per sent pair, 16-byte copies (K % 8 == 0).
__global__ void __launch_bounds__(256)
ep_gather_kernel(const uint16_t* __restrict__ x, const float* __restrict__ w, const int* __restrict__ order,
                 const int* __restrict__ n_sent, int topk, int K, uint16_t* __restrict__ xs, float* __restrict__ ws,
                 int n_pairs) {
  griddep_wait();
  griddep_launch_dependents();
  const int i = blockIdx.x;
  if (i >= *n_sent) return;
  const int p = order[i];
  if (!dbg_check(p >= 0 && p < n_pairs)) return;   // (debug build: n_pairs = pairs of the dispatch)
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<long long>(p / topk) * K);
  uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<long long>(i) * K);
  for (int c = threadIdx.x; c < K / 8; c += blockDim.x) dst[c] = src[c];
  if (w && threadIdx.x == 0) ws[i] = w[p];
}

// ---------------------------------------------------------------------------
// Self-test of the failure path: one thread waits, through the same bounded
// wait every kernel uses, on an mbarrier phase that `arrive` completes or
// (arrive = 0) nothing completes.  In the second case the wait gives up after
// its bound and records STQ1_DEV_WAIT_LIMIT; the kernel then returns normally.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) wait_selftest_kernel(int arrive) {
  __shared__ __align__(8) uint64_t bar_storage;
  if (threadIdx.x != 0) return;
  const uint32_t bar = smem_u32(&bar_storage);
  mbar_init(bar, 1);
  fence_mbar_init();
  if (arrive) mbar_arrive(bar);
  mbar_wait_bounded(bar, 0);
}

// The bounds check of the debug build, seen from outside: thread 0 stores
// into a 32-entry shared array at `index` only if 0 <= index < bound passes
// the check.  The store's address is masked to the array, so no build and no
// argument can reach past it: a debug build records STQ1_DEV_BOUNDS for an
// index outside [0, bound) and skips the store; a release build does not
// check.
__global__ void __launch_bounds__(32) bounds_selftest_kernel(int index, int bound) {
  __shared__ volatile int s_buf[32];
  s_buf[threadIdx.x] = 0;
  __syncwarp();
  if (threadIdx.x == 0 && dbg_check(index >= 0 && index < bound)) s_buf[index & 31] = 1;
}

}  // namespace stq1
