// Refit: one warm-started assign + update pass over the whole clustered
// prefix, with Hamerly bounds.
//
// AttentionIndex explainer (paper-daily.com), section "索引怎么边算边建？",
// item 3 and the paragraph after it: every R tokens the whole prefix is
// regrouped, starting from the previous centres plus a few new centres taken
// from recent keys; each key keeps an upper bound to its own centre and a
// lower bound to the others, and only new keys and keys whose bounds no
// longer guarantee their cluster are compared against all centres; one
// round of assignment and update, run on a side CUDA stream.  The kurate.org
// review ("Core Contribution", item 1) names the bounds Elkan/Hamerly-style.
//
// The result equals plain nearest-centre assignment (ties to the lower
// centre id) followed by a mean update: the bounds only skip comparisons
// whose outcome they already prove.  Bounds are kept conservative in fp32
// (rounded outward, with a relative margin), distances are screened in fp32
// and every near tie is decided again in float64.
//
// Bounds.  For a key with centre a: u >= d(x, c_a) at the current centre
// positions, and l is a lower bound on d(x, c_j) for every other centre j
// at the positions before the last update (no drift subtracted).  At the
// next refit the 256 centres that moved most (and the new seeds) form a set
// N handled through the centres: d(x, c_j) >= d(c_a, c_j) - u; every other
// centre moved at most delta_rest, so d(x, c_j) >= l - delta_rest.  A seed
// starts at a single key and moves far in its first update, so it must not
// enter the global drift bound.
//
// Steps (all on the stream given):
//   init      centres = previous refit centres ++ seed keys (float64)
//   far set   the 256 largest previous drifts -> N, delta_rest
//   near far  for each previous centre a: min over N \ {a} of ||c_a - c_j||
//   test      bound test for keys with bounds (tightening u once); failures
//             and new keys are queued for a full scan
//   scan      fp32 distances to all centres (tiled SIMT), best and second
//   recheck   float64 argmin for keys whose best two are within the margin
//   count / tile counts / scan / scatter: CSR by cluster, members in
//             ascending key id (deterministic, no float atomics)
//   update    float64 member means in CSR order, drift, bf16 representatives
//   bounds    u += drift(own centre)
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

constexpr int64_t kTileKeys = 4096;  // keys per CSR tile
constexpr float kRel = 1e-4f;         // relative margin of fp32 distances

__device__ __forceinline__ double kf64(const RefitArgs& a, int64_t s, int i) {
  double v = key_elem(a.keys, a.key_dtype, s, a.d, i);
  if (a.key_dtype == KD_FP8) v *= static_cast<double>(a.key_scale[s]);
  return v;
}
__device__ __forceinline__ float kf32(const RefitArgs& a, int64_t s, int i) {
  float v = key_elem(a.keys, a.key_dtype, s, a.d, i);
  if (a.key_dtype == KD_FP8) v *= a.key_scale[s];  // screening only; near ties are redone in fp64
  return v;
}

// Four consecutive key elements [e, e + 4) as float64 (d % 4 == 0).
__device__ __forceinline__ void load4_f64(const RefitArgs& a, int64_t row, int e, double* x) {
  if (a.key_dtype == KD_BF16) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(a.keys) + row * a.d + e));
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  } else if (a.key_dtype == KD_FP8) {
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint8_t*>(a.keys) + row * a.d + e));
    const double sc = static_cast<double>(__ldg(a.key_scale + row));
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = static_cast<double>(fp8_to_f32(static_cast<uint8_t>(v >> (8 * u)))) * sc;
  } else {
    const float4 v = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.keys) + row * a.d + e));
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  }
}

__global__ void k_init(RefitArgs a) {
  const int64_t n = static_cast<int64_t>(a.K) * a.d;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(e / a.d), i = static_cast<int>(e % a.d);
    double v = j < a.K_prev ? a.prev_centroids[e] : kf64(a, a.seed_ids[j - a.K_prev], i);
    a.cent[e] = v;
    a.cent_old[e] = v;
    a.cent32[e] = static_cast<float>(v);
  }
}

constexpr int kFar = 256;  // previous centres treated through the centres

// Single block: the kFar largest previous drifts (radix select on the bits
// of the non-negative doubles) -> far flags and the list N = far centres ++
// new seeds in nlist; delta_rest (largest drift outside N) -> *rest_bits.
__global__ void __launch_bounds__(1024) k_far_set(RefitArgs a, int32_t* flags, int32_t* nlist,
                                                  int32_t* n_list, unsigned long long* rest_bits) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_need, s_cnt;
  const int K = a.K_prev;
  unsigned long long prefix = 0, mask = 0;
  int need = kFar;
  if (threadIdx.x == 0) s_cnt = 0;
  if (K > kFar) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
      __syncthreads();
      for (int j = threadIdx.x; j < K; j += blockDim.x) {
        const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(a.drift[j]));
        if ((b & mask) == prefix) atomicAdd(&hist[(b >> shift) & 255ull], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int cum = 0, dg = 0;
        for (int d = 255; d >= 0; --d) {
          const int h = static_cast<int>(hist[d]);
          if (cum < need && need <= cum + h) {
            dg = d;
            break;
          }
          cum += h;
        }
        s_need = need - cum;
        s_prefix = prefix | (static_cast<unsigned long long>(dg) << shift);
      }
      __syncthreads();
      need = s_need;
      prefix = s_prefix;
      mask |= 255ull << shift;
      __syncthreads();
    }
  }
  // theta = the kFar-th largest drift; far = drift > theta (fewer than kFar)
  const unsigned long long theta = K > kFar ? prefix : 0ull;
  for (int j = threadIdx.x; j < K; j += blockDim.x) {
    const unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(a.drift[j]));
    const bool far = K <= kFar || b > theta;
    flags[j] = far ? 1 : 0;
    if (far) nlist[atomicAdd(&s_cnt, 1)] = j;
  }
  __syncthreads();
  for (int j = a.K_prev + threadIdx.x; j < a.K; j += blockDim.x) nlist[atomicAdd(&s_cnt, 1)] = j;
  __syncthreads();
  if (threadIdx.x == 0) {
    *n_list = s_cnt;
    *rest_bits = theta;  // largest drift of a centre outside N (0 if none)
  }
}

// One warp per previous centre a: nb(a) = min over N \ {a} of ||c_a - c_j||
// (fp32 with a relative margin, rounded down: a lower bound).
__global__ void k_near_far(RefitArgs a, const int32_t* nlist, const int32_t* n_list) {
  const int ca = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (ca >= a.K_prev) return;
  const int nn = *n_list;
  float best = INFINITY;
  for (int q = 0; q < nn; ++q) {
    const int j = nlist[q];
    if (j == ca) continue;
    float acc = 0.f;
    for (int i = lane; i < a.d; i += 32) {
      const float df = a.cent32[static_cast<int64_t>(ca) * a.d + i] - a.cent32[static_cast<int64_t>(j) * a.d + i];
      acc = fmaf(df, df, acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    best = fminf(best, acc);
  }
  if (lane == 0) a.seed_lb[ca] = isinf(best) ? INFINITY : fmaxf(0.f, __fsub_rd(__fmul_rd(sqrtf(best), 1.f - 1e-4f), 1e-6f));
}

// Exact-ish d(x, c) in fp32 (8-element vector loads), rounded up with a margin.
__device__ __forceinline__ float dist_up(const RefitArgs& a, int64_t x, int c) {
  float acc = 0.f;
  for (int e = 0; e < a.d; e += 4) {
    double v[4];
    load4_f64(a, x, e, v);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float df = static_cast<float>(v[u]) - a.cent32[static_cast<int64_t>(c) * a.d + e + u];
      acc = fmaf(df, df, acc);
    }
  }
  return __fadd_ru(__fmul_ru(sqrtf(acc), 1.f + 1e-4f), 1e-6f);
}

// Bound test.  One thread per key in [S, n_r).
__global__ void k_test(RefitArgs a, const unsigned long long* rest_bits) {
  const int64_t x = a.S + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (x >= a.n_r) return;
  bool scan = true;
  if (x < a.n_old && a.K_prev > 0) {
    const int ca = a.assign[x];
    const float rest = __double2float_ru(__longlong_as_double(static_cast<long long>(*rest_bits)));
    float u = a.ub[x];
    const float lfar = a.seed_lb[ca];
    float l = fminf(__fsub_rd(a.lb[x], rest), __fsub_rd(lfar, u));
    if (u < l) {
      scan = false;
      a.lb[x] = l;
    } else {
      u = dist_up(a, x, ca);  // tighten u once and retest
      l = fminf(__fsub_rd(a.lb[x], rest), __fsub_rd(lfar, u));
      if (u < l) {
        scan = false;
        a.ub[x] = u;
        a.lb[x] = l;
      }
    }
  }
  if (scan) {
    const int pos = atomicAdd(a.n_scan, 1);
    a.scan_list[pos] = static_cast<int32_t>(x);
  }
}

// Full scan in fp32: block = 64 keys x all centres in tiles of 64.  The
// block's 64 key rows are staged once in shared memory (fp32, padded rows);
// centre tiles stream through in 32-column slices.  Thread (r, c) of a
// 16 x 16 grid covers keys 4r..4r+3 and centres 4c..4c+3 of each tile.
constexpr int kSK = 64, kSC = 64, kSD = 32, kMaxD = 128;
__global__ void __launch_bounds__(256) k_scan(RefitArgs a, int32_t* recheck, int32_t* n_recheck) {
  __shared__ float xs[kSK][kMaxD + 1];
  __shared__ float cs[kSC][kSD + 1];
  const int n = *a.n_scan;
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  for (int kb = blockIdx.x * kSK; kb < n; kb += gridDim.x * kSK) {
    for (int e = threadIdx.x; e < kSK * a.d; e += blockDim.x) {
      const int r = e / a.d, i = e % a.d;
      const int kk = kb + r;
      xs[r][i] = kk < n ? kf32(a, a.scan_list[kk], i) : 0.f;
    }
    float best[4], second[4];
    int bid[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      best[r] = INFINITY;
      second[r] = INFINITY;
      bid[r] = 0x7fffffff;
    }
    for (int c0 = 0; c0 < a.K; c0 += kSC) {
      float acc[4][4] = {};
      for (int d0 = 0; d0 < a.d; d0 += kSD) {
        __syncthreads();
        for (int e = threadIdx.x; e < kSC * kSD; e += blockDim.x) {
          const int r = e / kSD, i = e % kSD;
          const int cc = c0 + r;
          cs[r][i] = (cc < a.K && d0 + i < a.d) ? a.cent32[static_cast<int64_t>(cc) * a.d + d0 + i] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int i = 0; i < kSD; ++i) {
          const bool in = d0 + i < a.d;
          float xv[4], cv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) xv[r] = in ? xs[tr * 4 + r][d0 + i] : 0.f;
#pragma unroll
          for (int c = 0; c < 4; ++c) cv[c] = cs[tc * 4 + c][i];
#pragma unroll
          for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float df = xv[r] - cv[c];
              acc[r][c] = fmaf(df, df, acc[r][c]);
            }
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int cc = c0 + tc * 4 + c;
        if (cc >= a.K) continue;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float v = acc[r][c];
          if (v < best[r] || (v == best[r] && cc < bid[r])) {
            second[r] = best[r];
            best[r] = v;
            bid[r] = cc;
          } else if (v < second[r]) {
            second[r] = v;
          }
        }
      }
    }
    // merge across the 16 threads of a row (consecutive lanes)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      for (int o = 8; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best[r], o);
        const float os = __shfl_xor_sync(0xffffffffu, second[r], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bid[r], o);
        if (ob < best[r] || (ob == best[r] && oi < bid[r])) {
          second[r] = fminf(best[r], os);
          best[r] = ob;
          bid[r] = oi;
        } else {
          second[r] = fminf(second[r], ob);
        }
      }
    }
    if (tc == 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int kk = kb + tr * 4 + r;
        if (kk >= n) continue;
        const int32_t x = a.scan_list[kk];
        a.assign[x] = bid[r];
        if (second[r] - best[r] <= kRel * second[r] + 1e-30f) {
          const int p = atomicAdd(n_recheck, 1);
          recheck[p] = x;
        }
        a.ub[x] = __fmul_ru(sqrtf(best[r]), 1.f + kRel);
        a.lb[x] = __fmul_rd(sqrtf(second[r]), 1.f - kRel);
      }
    }
    __syncthreads();
  }
}

// float64 decision for near ties.  A block takes kRkKeys listed keys (one
// warp each); centre rows stream through shared memory in tiles of
// kRkCent, one centre per lane, so each centre is read from L2 once per
// block with coalesced loads.  Per (key, centre) the sum runs over the
// dimensions in order with fma, as in the fp32 screen.
constexpr int kRkKeys = 8, kRkCent = 32;
constexpr int kBand = 16;  // centres listed per flagged key by the band pass
// Entries p < cap whose band has at most kBand centres were decided by
// k_recheck_band; this kernel takes the rest (all of them when cap = 0).
__global__ void __launch_bounds__(256) k_recheck(RefitArgs a, const int32_t* recheck,
                                                 const int32_t* n_recheck, const int32_t* band_cnt,
                                                 int cap) {
  __shared__ double xs[kRkKeys][kMaxD];
  __shared__ double cs[kRkCent][kMaxD + 1];
  const int nr = *n_recheck;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto todo = [&](int p) { return p < nr && (p >= cap || band_cnt[p] > kBand); };
  for (int g0 = blockIdx.x * kRkKeys; g0 < nr; g0 += gridDim.x * kRkKeys) {
    __syncthreads();
    if (!__syncthreads_or(threadIdx.x < kRkKeys && todo(g0 + threadIdx.x))) continue;
    for (int e = threadIdx.x; e < kRkKeys * a.d; e += blockDim.x) {
      const int r = e / a.d, i = e % a.d;
      xs[r][i] = g0 + r < nr ? kf64(a, recheck[g0 + r], i) : 0.0;
    }
    double best = INFINITY, second = INFINITY;
    int bi = 0x7fffffff;
    for (int c0 = 0; c0 < a.K; c0 += kRkCent) {
      __syncthreads();
      for (int e = threadIdx.x; e < kRkCent * a.d; e += blockDim.x) {
        const int r = e / a.d, i = e % a.d;
        cs[r][i] = c0 + r < a.K ? a.cent[static_cast<int64_t>(c0 + r) * a.d + i] : 0.0;
      }
      __syncthreads();
      double acc = 0.0;
      for (int i = 0; i < a.d; ++i) {
        const double df = xs[warp][i] - cs[lane][i];
        acc = fma(df, df, acc);
      }
      const int c = c0 + lane;
      if (c < a.K) {
        if (acc < best || (acc == best && c < bi)) {
          second = best;
          best = acc;
          bi = c;
        } else if (acc < second) {
          second = acc;
        }
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, best, o);
      const double os = __shfl_xor_sync(0xffffffffu, second, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob < best || (ob == best && oi < bi)) {
        second = fmin(best, os);
        best = ob;
        bi = oi;
      } else {
        second = fmin(second, ob);
      }
    }
    if (lane == 0 && todo(g0 + warp)) {
      const int32_t x = recheck[g0 + warp];
      a.assign[x] = bi;
      a.ub[x] = __double2float_ru(sqrt(best) * (1.0 + 1e-6));
      a.lb[x] = __double2float_rd(sqrt(second) * (1.0 - 1e-6));
    }
  }
}

// float64 decision among the band of a flagged key: one warp per key, lanes
// over dimensions.  Centres outside the band are farther than the band's
// best in exact arithmetic; their lower bound (stored by the band pass)
// enters the key's lower bound.
__global__ void k_recheck_band(RefitArgs a, const int32_t* recheck, const int32_t* n_recheck,
                               const float* outside_lb2, const int32_t* band_ids, const int32_t* band_cnt,
                               int cap) {
  const int warp = static_cast<int>((blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>((gridDim.x * static_cast<int64_t>(blockDim.x)) >> 5);
  const int nr = min(*n_recheck, cap);
  for (int p = warp; p < nr; p += nwarps) {
    const int nb = band_cnt[p];
    if (nb > kBand) continue;  // overflow: full decision in k_recheck
    const int32_t x = recheck[p];
    double xv[4];
    const int e = lane * 4;
    if (e < a.d) load4_f64(a, x, e, xv);
    double best = INFINITY, second = INFINITY;
    int bi = 0x7fffffff;
    for (int u = 0; u < nb; ++u) {
      const int c = band_ids[static_cast<int64_t>(p) * kBand + u];
      double acc = 0.0;
      if (e < a.d) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const double df = xv[q] - a.cent[static_cast<int64_t>(c) * a.d + e + q];
          acc = fma(df, df, acc);
        }
      }
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (acc < best || (acc == best && c < bi)) {
        second = best;
        best = acc;
        bi = c;
      } else if (acc < second) {
        second = acc;
      }
    }
    if (lane == 0 && nb > 0) {
      const double out2 = static_cast<double>(outside_lb2[p]);
      const double sec = fmin(second, out2 > 0.0 ? out2 : 0.0);
      a.assign[x] = bi;
      a.ub[x] = __double2float_ru(sqrt(best) * (1.0 + 1e-6));
      a.lb[x] = __double2float_rd(sqrt(sec) * (1.0 - 1e-6));
    }
  }
}

__global__ void k_zero_counts(RefitArgs a) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < a.K; j += gridDim.x * blockDim.x)
    a.counts[j] = 0;
}

__global__ void k_count(RefitArgs a) {
  const int64_t x = a.S + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (x >= a.n_r) return;
  const int c = a.assign[x];
  if (c < 0 || c >= a.K) {
    atomicOr(a.err, DEV_ERR_RANGE);
    return;
  }
  atomicAdd(&a.counts[c], 1);
}

// exclusive scan of counts -> offsets (single block)
// Exclusive prefix sum over j < K of f(counts[j]) into out[0..K] by one
// 1024-thread block; f = identity (chunk = 0) or ceil(v / chunk).
__device__ void block_scan_counts(const int32_t* counts, int K, int chunk, int32_t* out, int* warp_sums,
                                  int* carry) {
  if (threadIdx.x == 0) *carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int base = 0; base < K; base += blockDim.x) {
    const int j = base + threadIdx.x;
    int v = j < K ? counts[j] : 0;
    if (chunk > 0) v = (v + chunk - 1) / chunk;
    int incl = v;
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
      int s = warp_sums[lane];
      int si = s;
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, si, o);
        if (lane >= o) si += n;
      }
      warp_sums[lane] = si - s;
    }
    __syncthreads();
    if (j < K) out[j] = *carry + warp_sums[w] + incl - v;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) *carry += warp_sums[w] + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) out[K] = *carry;
  __syncthreads();
}

// CSR offsets, and the offsets of the update chunks (kUpdChunk members)
constexpr int kUpdChunk = 128;
__global__ void __launch_bounds__(1024) k_offsets(RefitArgs a) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  block_scan_counts(a.counts, a.K, 0, a.offsets, warp_sums, &carry);
  block_scan_counts(a.counts, a.K, kUpdChunk, a.upd_chunk_off, warp_sums, &carry);
}

// per-tile cluster counts: one warp per tile, keys walked in order
__global__ void k_tile_counts(RefitArgs a) {
  extern __shared__ int cnt[];
  const int tile = blockIdx.x;
  const int lane = threadIdx.x;
  for (int j = lane; j < a.K; j += 32) cnt[j] = 0;
  __syncwarp();
  const int64_t x0 = a.S + tile * kTileKeys;
  const int64_t x1 = min(a.n_r, x0 + kTileKeys);
  for (int64_t xb = x0; xb < x1; xb += 32) {
    const int64_t x = xb + lane;
    const bool v = x < x1;
    const int c = v ? a.assign[x] : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    if (v && __ffs(peers) - 1 == lane) cnt[c] += __popc(peers);
    __syncwarp();
  }
  for (int j = lane; j < a.K; j += 32) a.tile_counts[static_cast<int64_t>(tile) * a.K + j] = cnt[j];
}

// tile_counts[t][j] <- offsets[j] + sum of counts of earlier tiles
__global__ void k_tile_base(RefitArgs a, int ntiles) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= a.K) return;
  int run = a.offsets[j];
  for (int t = 0; t < ntiles; ++t) {
    int32_t* p = a.tile_counts + static_cast<int64_t>(t) * a.K + j;
    const int v = *p;
    *p = run;
    run += v;
  }
}

__global__ void k_scatter(RefitArgs a) {
  extern __shared__ int base[];
  const int tile = blockIdx.x;
  const int lane = threadIdx.x;
  for (int j = lane; j < a.K; j += 32) base[j] = a.tile_counts[static_cast<int64_t>(tile) * a.K + j];
  __syncwarp();
  const int64_t x0 = a.S + tile * kTileKeys;
  const int64_t x1 = min(a.n_r, x0 + kTileKeys);
  const unsigned lt = (1u << lane) - 1u;
  for (int64_t xb = x0; xb < x1; xb += 32) {
    const int64_t x = xb + lane;
    const bool v = x < x1;
    const int c = v ? a.assign[x] : -1 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, c);
    if (v) a.members[base[c] + __popc(peers & lt)] = static_cast<int32_t>(x);
    __syncwarp();
    if (v && __ffs(peers) - 1 == lane) base[c] += __popc(peers);
    __syncwarp();
  }
}

// One warp per cluster: float64 member sums in member (CSR) order, lanes
// over 4-element column blocks, member ids fetched 32 at a time and four
// member rows in flight; then mean, drift and the bf16 representative.
// Centre update in two deterministic steps.  k_update_part: one warp per
// chunk of up to kUpdChunk consecutive members of a cluster sums them in
// member order (lane = 4 dimensions); k_update_fin: one warp per cluster
// adds its chunk sums in chunk order, divides by the size (an empty cluster
// keeps its centre) and writes centre, bf16 representative and drift.
__global__ void k_update_part(RefitArgs a) {
  const int q = static_cast<int>((blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  const int32_t* co = a.upd_chunk_off;
  if (q >= co[a.K]) return;
  int lo = 0, hi = a.K;  // co[lo] <= q < co[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (co[mid] <= q) lo = mid;
    else hi = mid;
  }
  const int p0 = a.offsets[lo] + (q - co[lo]) * kUpdChunk;
  const int p1 = min(p0 + kUpdChunk, a.offsets[lo + 1]);
  const int e = lane * 4;
  const bool act = e < a.d;
  double sum[4] = {0.0, 0.0, 0.0, 0.0};
  for (int b0 = p0; b0 < p1; b0 += 32) {
    const int nb = min(32, p1 - b0);
    const int myid = lane < nb ? a.members[b0 + lane] : 0;
    int u = 0;
    for (; u + 8 <= nb; u += 8) {
      double x[8][4];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int id = __shfl_sync(0xffffffffu, myid, u + r);
        if (act) load4_f64(a, id, e, x[r]);
      }
      if (act) {
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 4; ++c) sum[c] += x[r][c];
      }
    }
    for (; u < nb; ++u) {
      const int id = __shfl_sync(0xffffffffu, myid, u);
      if (act) {
        double x[4];
        load4_f64(a, id, e, x);
#pragma unroll
        for (int c = 0; c < 4; ++c) sum[c] += x[c];
      }
    }
  }
  if (act) {
#pragma unroll
    for (int c = 0; c < 4; ++c) a.upd_part[static_cast<int64_t>(q) * a.d + e + c] = sum[c];
  }
}

__global__ void k_update_fin(RefitArgs a, unsigned long long* max_drift_bits) {
  const int j = static_cast<int>((blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (j >= a.K) return;
  const int n = a.offsets[j + 1] - a.offsets[j];
  const int q0 = a.upd_chunk_off[j], q1 = a.upd_chunk_off[j + 1];
  const int e = lane * 4;
  double dr = 0.0;
  if (e < a.d) {
    double sum[4] = {0.0, 0.0, 0.0, 0.0};
    for (int q = q0; q < q1; ++q) {
      const double* pp = a.upd_part + static_cast<int64_t>(q) * a.d + e;
#pragma unroll
      for (int c = 0; c < 4; ++c) sum[c] += pp[c];
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t idx = static_cast<int64_t>(j) * a.d + e + c;
      double v = a.cent[idx];
      if (n > 0) v = sum[c] / static_cast<double>(n);
      const double df = v - a.cent_old[idx];
      dr = fma(df, df, dr);
      a.cent[idx] = v;
      a.reps[idx] = f64_to_bf16_rne(v);
    }
  }
  for (int o = 16; o > 0; o >>= 1) dr += __shfl_xor_sync(0xffffffffu, dr, o);
  if (lane == 0) {
    const double drift = sqrt(dr) * (1.0 + 1e-6);
    a.drift[j] = drift;
    atomicMax(max_drift_bits, static_cast<unsigned long long>(__double_as_longlong(drift)));
  }
}

__global__ void k_bounds(RefitArgs a) {
  const int64_t x = a.S + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (x >= a.n_r) return;
  a.ub[x] = __fadd_ru(a.ub[x], __double2float_ru(a.drift[a.assign[x]]));
}

// ------------------------------------------------- tensor-core full scan
// bf16 keys, d = 128.  Each fp64 centre c is split into bf16 hi + lo
// (hi = rne(c), lo = rne(c - hi); per element |c - hi - lo| <= 2^-16 |c|),
// and one UMMA pair per 128-centre tile accumulates x.hi + x.lo in fp32
// TMEM.  d^2 = ||x||^2 - 2 x.c + ||c||^2 then carries, per key, at most
//   1.5e-5 (split residual) + 3.1e-5 (256-term fp32 accumulation, counted
//   with whole-ulp steps) + 0.8e-5 (||x||^2 in fp32) + rounding of the sum
// times (||x||^2 + max ||c||^2); the kernel takes 1e-4 times that as its
// bound err.  Keys whose best two lie within 2 err of each other are
// re-decided in float64, so the assignment equals the exact one.
constexpr int kTcKeys = 128, kTcCent = 128;
constexpr int kTcBStages = 2;
constexpr int kTcA = kTcKeys * 256;            // 32 KiB per key tile
constexpr int kTcB = 2 * kTcCent * 256;        // hi + lo, 64 KiB per centre tile
constexpr int kTcThreads = 256;
constexpr size_t kTcSmem = 1024 + 2 * kTcA + kTcBStages * kTcB;
constexpr double kTcErr = 1e-4;

__global__ void k_cent_split(RefitArgs a, unsigned long long* ccmax_bits) {
  const int j = blockIdx.x, i = threadIdx.x;  // 128 threads per centre
  const bool live = j < a.K;
  const double c = live ? a.cent[static_cast<int64_t>(j) * 128 + i] : 0.0;
  const uint16_t hb = f64_to_bf16_rne(c);
  const uint16_t lb = f64_to_bf16_rne(c - static_cast<double>(bf16_bits_to_f32(hb)));
  a.cent_hi[static_cast<int64_t>(j) * 128 + i] = hb;
  a.cent_lo[static_cast<int64_t>(j) * 128 + i] = lb;
  __shared__ double red[4];
  double sq = c * c;
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if ((i & 31) == 0) red[i >> 5] = sq;
  __syncthreads();
  if (i == 0) {
    const double t = (red[0] + red[1]) + (red[2] + red[3]);
    a.cent_cc[j] = live ? static_cast<float>(t) : INFINITY;
    if (live) atomicMax(ccmax_bits, static_cast<unsigned long long>(__double_as_longlong(t)));
  }
}

// Warp roles: 0 = centre-tile producer (TMA, lane 0), 1 = UMMA issuer
// (lane 0), 2-3 = key-tile producers (TMA gather4 of the listed keys, 64
// rows each), 4-7 = epilogue (one key row per thread).  Key tiles are
// double-buffered; centre tiles stream through kTcBStages stages; two TMEM
// accumulators of 128 columns alternate between UMMA and epilogue.
// Band pass (kBandPass = true): the same kernel over the keys flagged by
// the scan, with their first-pass best value known, lists every centre
// whose screened d^2 is within 2 err of it (at most kBand; more is marked
// as an overflow).  The screened values are bit-identical in both passes.
struct BandArgs {
  const int32_t* list;  // keys of this pass (scan list, or recheck list)
  const int32_t* n;     // its length (device)
  int32_t* recheck;     // scan: flagged keys out
  int32_t* n_recheck;   // scan: their count
  float* best;          // [cap] screened best d^2 of flagged key p
  int32_t* ids;         // [cap, kBand] band: centre ids
  int32_t* cnt;         // [cap] band: size (> kBand: overflow)
  int cap;              // flagged keys that get a band
};

template <bool kBandPass>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_scan_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap hmap,
              const __grid_constant__ CUtensorMap lmap, RefitArgs a, int K_pad,
              const unsigned long long* ccmax_bits, BandArgs bd) {
  extern __shared__ uint8_t raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = base;             // [2][kTcA]
  uint8_t* sb = base + 2 * kTcA;  // [kTcBStages][kTcB]
  __shared__ uint64_t afull[2], aempty[2], bfull[kTcBStages], bempty[kTcBStages], tfull[2], tempty[2], done;
  __shared__ uint32_t tmem_holder;
  __shared__ int abort_flag;
  volatile int* aborted = &abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = kBandPass ? min(*bd.n, bd.cap) : *bd.n;
  const int ntiles = (n + kTcKeys - 1) / kTcKeys;
  const int nct = K_pad / kTcCent;
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 2);
      mbar_init(&aempty[b], 1 + 128);
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    for (int s2 = 0; s2 < kTcBStages; ++s2) {
      mbar_init(&bfull[s2], 1);
      mbar_init(&bempty[s2], 1);
    }
    mbar_init(&done, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_holder, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_holder;

  if (warp == 0) {
    // ---------------------------------------------- centre-tile producer
    if (lane == 0) {
      uint32_t gj = 0;
      for (int kt = blockIdx.x; kt < ntiles && !*aborted; kt += gridDim.x) {
        for (int ct = 0; ct < nct; ++ct, ++gj) {
          const int s2 = gj % kTcBStages;
          if (gj >= kTcBStages && !mbar_wait(&bempty[s2], ((gj / kTcBStages) & 1) ^ 1, a.err, &abort_flag))
            break;
          uint8_t* dst = sb + s2 * kTcB;
          mbar_arrive_expect_tx(&bfull[s2], kTcB);
          tma_load_2d(dst, &hmap, 0, ct * kTcCent, &bfull[s2]);
          tma_load_2d(dst + kTcCent * 128, &hmap, 64, ct * kTcCent, &bfull[s2]);
          tma_load_2d(dst + 2 * kTcCent * 128, &lmap, 0, ct * kTcCent, &bfull[s2]);
          tma_load_2d(dst + 3 * kTcCent * 128, &lmap, 64, ct * kTcCent, &bfull[s2]);
        }
      }
      if (*aborted)  // let the last copies land before the CTA exits
        for (uint32_t g = gj > kTcBStages ? gj - kTcBStages : 0; g < gj; ++g)
          mbar_drain(&bfull[g % kTcBStages], (g / kTcBStages) & 1);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------- key-tile producers
    uint32_t it = 0;
    for (int kt = blockIdx.x; kt < ntiles; kt += gridDim.x, ++it) {
      const int b = it & 1;
      if (it >= 2 && !mbar_wait(&aempty[b], ((it >> 1) & 1) ^ 1, a.err, &abort_flag)) break;
      if (lane == 0) mbar_arrive_expect_tx(&afull[b], kTcA / 2);
      __syncwarp();
      const int rl = (warp - 2) * 64 + (lane & 15) * 4;  // first of this lane's 4 rows
      const int half = lane >> 4;
      int r[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = kt * kTcKeys + rl + q;
        r[q] = kk < n ? bd.list[kk] : static_cast<int>(a.S);
      }
      tma_gather4(sa + b * kTcA + half * (kTcKeys * 128) + rl * 128, &kmap, half * 64, r[0], r[1], r[2], r[3],
                  &afull[b]);
    }
    if (*aborted)
      for (uint32_t g = it > 2 ? it - 2 : 0; g < it; ++g) mbar_drain(&afull[g & 1], (g >> 1) & 1);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTcKeys, kTcCent);
      uint32_t it = 0, gj = 0;
      bool ok = true;
      for (int kt = blockIdx.x; ok && kt < ntiles; kt += gridDim.x, ++it) {
        const int b = it & 1;
        if (!mbar_wait(&afull[b], (it >> 1) & 1, a.err, &abort_flag)) break;
        tc_fence_after();
        const uint32_t sA = smem_u32(sa + b * kTcA);
        for (int ct = 0; ct < nct; ++ct, ++gj) {
          const int s2 = gj % kTcBStages;
          const int acc = gj & 1;
          if (!mbar_wait(&bfull[s2], (gj / kTcBStages) & 1, a.err, &abort_flag) ||
              (gj >= 2 && !mbar_wait(&tempty[acc], ((gj >> 1) & 1) ^ 1, a.err, &abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sB = smem_u32(sb + s2 * kTcB);
#pragma unroll
          for (int part = 0; part < 2; ++part) {  // x.hi, then x.lo into the same accumulator
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
              umma_bf16(tmem_base + acc * kTcCent, sdesc_sw128(sA + kb * (kTcKeys * 128) + ko),
                        sdesc_sw128(sB + part * (2 * kTcCent * 128) + kb * (kTcCent * 128) + ko), idesc,
                        (part > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&bempty[s2]);
          umma_commit(&tfull[acc]);
        }
        if (ok) umma_commit(&aempty[b]);  // the key tile is free once these UMMAs finish
      }
      umma_commit(&done);  // every UMMA issued above has finished before TMEM is freed
      mbar_drain(&done, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int row = (warp - 4) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const double ccmax = __longlong_as_double(static_cast<long long>(*ccmax_bits));
    uint32_t it = 0, gj = 0;
    bool ok = true;
    for (int kt = blockIdx.x; ok && kt < ntiles; kt += gridDim.x, ++it) {
      const int b = it & 1;
      float xx = 0.f;
      if (!mbar_wait(&afull[b], (it >> 1) & 1, a.err, &abort_flag)) break;
      {
        // ||x||^2 from the staged row (128-byte swizzle: 16-byte chunk c of
        // row r sits at chunk c ^ (r & 7))
        const uint8_t* rowp = sa + b * kTcA + row * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + (c >> 3) * (kTcKeys * 128) +
                                                          (((c & 7) ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float lo = __uint_as_float(w[u] << 16), hi = __uint_as_float(w[u] & 0xFFFF0000u);
            xx = fmaf(lo, lo, xx);
            xx = fmaf(hi, hi, xx);
          }
        }
      }
      mbar_arrive(&aempty[b]);
      const int kk = kt * kTcKeys + row;
      // fp8 keys: the tile holds the codes (exact in bf16), the key is
      // scale * code; ||x||^2 and x.c take the scale (2^-24-level roundings,
      // far inside the bound below)
      float m2 = -2.f;
      if (a.key_dtype == KD_FP8) {
        const float sx = kk < n ? a.key_scale[bd.list[kk]] : 1.f;
        xx = sx * sx * xx;
        m2 = -2.f * sx;
      }
      const float err = static_cast<float>(kTcErr * (static_cast<double>(xx) + ccmax));
      float best = INFINITY, second = INFINITY;
      int bid = 0x7fffffff;
      float thr = 0.f;
      int nb = 0;
      // rounded up: every centre whose exact d^2 can be the minimum is listed
      if (kBandPass) thr = kk < n ? __fadd_ru(bd.best[kk], 2.f * err) : -INFINITY;
      for (int ct = 0; ct < nct; ++ct, ++gj) {
        const int acc = gj & 1;
        if (!mbar_wait(&tfull[acc], (gj >> 1) & 1, a.err, &abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c32 = 0; c32 < kTcCent / 32; ++c32) {
          float v[32];
          tmem_ld32(tmem_base + acc * kTcCent + c32 * 32 + lane_off, v);
          const float4* ccp = reinterpret_cast<const float4*>(a.cent_cc + ct * kTcCent + c32 * 32);
          float cc[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 t = __ldg(ccp + q);
            cc[4 * q] = t.x;
            cc[4 * q + 1] = t.y;
            cc[4 * q + 2] = t.z;
            cc[4 * q + 3] = t.w;
          }
          tmem_ld_wait();
          if (kBandPass) {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float d2 = fmaf(m2, v[q], xx + cc[q]);
              if (d2 <= thr) {
                if (nb < kBand) bd.ids[static_cast<int64_t>(kk) * kBand + nb] = ct * kTcCent + c32 * 32 + q;
                ++nb;
              }
            }
          } else {
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              const float d2 = fmaf(m2, v[q], xx + cc[q]);
              if (d2 < best) {
                second = best;
                best = d2;
                bid = ct * kTcCent + c32 * 32 + q;
              } else if (d2 < second) {
                second = d2;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
      }
      if (!ok) break;
      if (kBandPass) {
        if (kk < n) {
          bd.cnt[kk] = nb;
          bd.best[kk] = __fsub_rd(thr, err);  // exact d^2 of every centre outside the band is above this
        }
      } else if (kk < n && bid < a.K) {
        const int32_t x = bd.list[kk];
        a.assign[x] = bid;
        if (!(second - best > 2.f * err)) {
          const int p = atomicAdd(bd.n_recheck, 1);
          bd.recheck[p] = x;
          if (p < bd.cap) bd.best[p] = best;
        }
        a.ub[x] = __fmul_ru(sqrtf(__fadd_ru(fmaxf(best, 0.f), err)), 1.f + 1e-6f);
        a.lb[x] = __fmul_rd(sqrtf(fmaxf(__fsub_rd(second, err), 0.f)), 1.f - 1e-6f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

}  // namespace

int64_t refit_tile_size() { return kTileKeys; }
int64_t refit_update_chunk() { return kUpdChunk; }

cudaError_t launch_refit(const RefitArgs& a, int64_t max_tiles, cudaStream_t st,
                         int32_t* host_nscan, const RefitTcMaps* tc) {
  const int64_t n = a.n_r - a.S;
  if (n <= 0 || a.K <= 0) return cudaSuccess;
  const int64_t ntiles = (n + kTileKeys - 1) / kTileKeys;
  if (ntiles > max_tiles) return cudaErrorInvalidValue;
  if (static_cast<size_t>(a.K) * 4 > 200 * 1024 || a.d > 128 || a.d % 4 != 0) return cudaErrorInvalidValue;
  // scratch words after n_scan: [1] n_recheck, [2..3] max drift bits,
  // [4..5] drift bound of the centres outside N, [6] size of N, [8..9]
  // largest ||c||^2 (tensor-core scan)
  int32_t* n_recheck = a.n_scan + 1;
  unsigned long long* mdb = reinterpret_cast<unsigned long long*>(a.n_scan + 2);
  unsigned long long* rest_bits = reinterpret_cast<unsigned long long*>(a.n_scan + 4);
  int32_t* n_list = a.n_scan + 6;
  unsigned long long* ccmax_bits = reinterpret_cast<unsigned long long*>(a.n_scan + 8);
  if (tc && ((a.key_dtype != KD_BF16 && a.key_dtype != KD_FP8) || a.d != 128)) return cudaErrorInvalidValue;
  cudaMemsetAsync(a.n_scan, 0, 40, st);
  const int64_t ce = static_cast<int64_t>(a.K) * a.d;
  count_launch();
  k_init<<<static_cast<unsigned>((ce + 255) / 256 < 4096 ? (ce + 255) / 256 : 4096), 256, 0, st>>>(a);
  if (a.K_prev > 0) {
    // far set and centre-to-far-centre bounds (counts and tile_counts are
    // free until the CSR build below)
    count_launch();
    k_far_set<<<1, 1024, 0, st>>>(a, a.counts, a.tile_counts, n_list, rest_bits);
    count_launch();
    k_near_far<<<(a.K_prev * 32 + 255) / 256, 256, 0, st>>>(a, a.tile_counts, n_list);
  }
  const unsigned gk = static_cast<unsigned>((n + 255) / 256);
  count_launch();
  k_test<<<gk, 256, 0, st>>>(a, rest_bits);
  // the scan list length is only known on the device: fixed grids that stride
  if (tc) {
    const int K_pad = (a.K + kTcCent - 1) / kTcCent * kTcCent;
    count_launch();
    k_cent_split<<<K_pad, 128, 0, st>>>(a, ccmax_bits);
    cudaFuncSetAttribute(k_scan_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kTcSmem));
    const int64_t ktiles = (n + kTcKeys - 1) / kTcKeys;
    const int grid = static_cast<int>(ktiles < tc->num_sms ? ktiles : tc->num_sms);
    BandArgs bd{};
    bd.list = a.scan_list;
    bd.n = a.n_scan;
    bd.recheck = a.scan_list + n;
    bd.n_recheck = n_recheck;
    bd.best = a.band_best;
    bd.ids = a.band_ids;
    bd.cnt = a.band_cnt;
    bd.cap = a.band_cap;
    count_launch();
    k_scan_tc<false><<<grid, kTcThreads, kTcSmem, st>>>(tc->keys, tc->hi, tc->lo, a, K_pad, ccmax_bits, bd);
    // the flagged keys again, listing the centres within their error band
    bd.list = a.scan_list + n;
    bd.n = n_recheck;
    cudaFuncSetAttribute(k_scan_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kTcSmem));
    const int bgrid = static_cast<int>((a.band_cap + kTcKeys - 1) / kTcKeys < tc->num_sms
                                           ? (a.band_cap + kTcKeys - 1) / kTcKeys
                                           : tc->num_sms);
    count_launch();
    k_scan_tc<true><<<bgrid, kTcThreads, kTcSmem, st>>>(tc->keys, tc->hi, tc->lo, a, K_pad, ccmax_bits, bd);
    count_launch();
    k_recheck_band<<<static_cast<unsigned>((a.band_cap + 7) / 8 < 1184 ? (a.band_cap + 7) / 8 : 1184), 256, 0,
                     st>>>(a, a.scan_list + n, n_recheck, a.band_best, a.band_ids, a.band_cnt, a.band_cap);
  } else {
    const int64_t sblocks = (n + kSK - 1) / kSK;
    count_launch();
    k_scan<<<static_cast<unsigned>(sblocks < 1184 ? sblocks : 1184), 256, 0, st>>>(a, a.scan_list + n,
                                                                                    n_recheck);
  }
  // recheck list lives after the scan list (capacity n)
  const int64_t rblocks = (n + kRkKeys - 1) / kRkKeys;
  count_launch();
  k_recheck<<<static_cast<unsigned>(rblocks < 1184 ? rblocks : 1184), 256, 0, st>>>(
      a, a.scan_list + n, n_recheck, a.band_cnt, tc ? a.band_cap : 0);
  count_launch();
  k_zero_counts<<<(a.K + 255) / 256, 256, 0, st>>>(a);
  count_launch();
  k_count<<<gk, 256, 0, st>>>(a);
  count_launch();
  k_offsets<<<1, 1024, 0, st>>>(a);
  const size_t sm = static_cast<size_t>(a.K) * 4;
  cudaFuncSetAttribute(k_tile_counts, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  cudaFuncSetAttribute(k_scatter, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm));
  count_launch();
  k_tile_counts<<<static_cast<unsigned>(ntiles), 32, sm, st>>>(a);
  count_launch();
  k_tile_base<<<(a.K + 255) / 256, 256, 0, st>>>(a, static_cast<int>(ntiles));
  count_launch();
  k_scatter<<<static_cast<unsigned>(ntiles), 32, sm, st>>>(a);
  // chunks: at most n / kUpdChunk + K
  const int64_t max_chunks = n / kUpdChunk + a.K;
  count_launch();
  k_update_part<<<static_cast<unsigned>((max_chunks * 32 + 255) / 256), 256, 0, st>>>(a);
  count_launch();
  k_update_fin<<<static_cast<unsigned>((static_cast<int64_t>(a.K) * 32 + 255) / 256), 256, 0, st>>>(a, mdb);
  count_launch();
  k_bounds<<<gk, 256, 0, st>>>(a);
  if (host_nscan) cudaMemcpyAsync(host_nscan, a.n_scan, 8, cudaMemcpyDeviceToHost, st);
  return cudaGetLastError();
}

}  // namespace aiidx
