// Seal: size-capped k-means of each completed W-key window into m clusters.
//
// AttentionIndex explainer (paper-daily.com), section "索引怎么边算边建？",
// item 2: every W open keys are grouped into m clusters, appended to the
// index, and the existing clusters are left alone; the kurate.org review
// ("Core Contribution", item 1) names the method size-capped k-means.  The
// pages give no algorithm; the reading implemented here:
//   init    c_j = x[floor((j + 1/2) W / m)]
//   repeat  at most `iters` times, stopping when the assignment repeats:
//           D_ij = ||x_i - c_j||^2 (float64; evaluated as
//                  ||x||^2 - 2 x.c + ||c||^2, clamped at 0)
//           visit all (i, j) pairs by (D asc, i asc, j asc); key i joins
//           cluster j if i is still free and j has fewer than cap keys
//           c_j = mean of its members (float64, ascending key order)
// Members are stored per cluster in ascending key id; the representative is
// the mean rounded once to bf16 (round to nearest even).
//
// One CTA (512 threads) per window.  The sequential greedy walk over the
// W*m sorted pairs is reproduced exactly in at most m + 1 data-parallel
// rounds: in a round every free key proposes its best pair among the
// clusters that are not full; the first cluster to fill is the one whose
// (cap - count)-th smallest proposal comes first in pair order; every
// proposal up to that pair is final (nothing before it can be refused),
// that cluster is closed, and the remaining keys propose again.  Pair order
// is (distance, key, cluster).
//
// The (cap - count)-th smallest proposal of each cluster is selected with a
// histogram over the cluster's distance range (bins are a monotone function
// of the distance, so the element lies in the bin where the running count
// reaches it) and an exact rank among the few proposals of that one bin.
// The histograms are built from every key's proposal in a pass's first
// round and then kept current by the commit step: a committed key's count
// is removed, and a free key whose cluster has just filled moves its count
// to its next open cluster (the only proposals that change between rounds).
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

constexpr int kThreads = 512;
constexpr int kBins = 1024;  // histogram bins per cluster (32 chunks of 32)

struct SealSmem {
  double* D;         // [m, W] squared distances (cluster-major)
  double* cent;      // [m, d]
  double* cc;        // [m] squared centre norms
  double* dlo;       // [m] smallest distance to the cluster (bin origin)
  double* dsc;       // [m] bins per unit distance
  uint64_t* fk1;     // [m] fill pair of each cluster: distance bits
  int* hist;         // [m, kBins]
  uint32_t* fk2;     // [m] fill pair: (key << 16) | cluster
  int* cnt;          // [m] members so far
  int* tb;           // [m] bin holding the filling proposal (-1: no fill)
  int* cb;           // [m] proposals in the bins before it
  int* cstart;       // [m + 1] member list starts
  int* ncoll;        // [m] proposals collected from the target bin
  int* misc;         // [0] best cluster, [2] free keys, [3] changed
  unsigned long long* fullmask;
  int8_t* prop;      // [W] proposal of each free key (-1: none)
  int16_t* assign;   // [W]
  int16_t* prev;     // [W]
  int16_t* mlist;    // [W] members, grouped by cluster, ascending
  int16_t* coll;     // [m, W] proposals in each cluster's target bin
  uint16_t* bin;     // [m, W] histogram bin of D[j, i] for this pass
  uint32_t* ord;     // [W] (m <= 8) clusters of key i by (D asc, j asc), 4 bits each
};

// Lays the arrays out from p; returns the bytes used.  Shared by the kernel
// and the host-side size computation.
__host__ __device__ inline size_t seal_layout(uint8_t* p, int W, int m, int d, SealSmem* s) {
  size_t o = 0;
  auto take = [&](size_t bytes) {
    uint8_t* q = p + o;
    o += (bytes + 15) & ~size_t(15);
    return q;
  };
  uint8_t* D = take(static_cast<size_t>(W) * m * 8);
  uint8_t* cent = take(static_cast<size_t>(m) * d * 8);
  uint8_t* cc = take(static_cast<size_t>(m) * 8);
  uint8_t* dlo = take(static_cast<size_t>(m) * 8);
  uint8_t* dsc = take(static_cast<size_t>(m) * 8);
  uint8_t* fk1 = take(static_cast<size_t>(m) * 8);
  uint8_t* full = take(8);
  uint8_t* hist = take(static_cast<size_t>(m) * kBins * 4);
  uint8_t* fk2 = take(static_cast<size_t>(m) * 4);
  uint8_t* cnt = take(static_cast<size_t>(m) * 4);
  uint8_t* tb = take(static_cast<size_t>(m) * 4);
  uint8_t* cb = take(static_cast<size_t>(m) * 4);
  uint8_t* cstart = take(static_cast<size_t>(m + 1) * 4);
  uint8_t* ncoll = take(static_cast<size_t>(m) * 4);
  uint8_t* misc = take(16);
  uint8_t* prop = take(static_cast<size_t>(W));
  uint8_t* assign = take(static_cast<size_t>(W) * 2);
  uint8_t* prev = take(static_cast<size_t>(W) * 2);
  uint8_t* mlist = take(static_cast<size_t>(W) * 2);
  uint8_t* coll = take(static_cast<size_t>(W) * m * 2);
  uint8_t* bin = take(static_cast<size_t>(W) * m * 2);
  uint8_t* ord = take(static_cast<size_t>(W) * 4);
  if (s) {
    s->D = reinterpret_cast<double*>(D);
    s->cent = reinterpret_cast<double*>(cent);
    s->cc = reinterpret_cast<double*>(cc);
    s->dlo = reinterpret_cast<double*>(dlo);
    s->dsc = reinterpret_cast<double*>(dsc);
    s->fk1 = reinterpret_cast<uint64_t*>(fk1);
    s->fullmask = reinterpret_cast<unsigned long long*>(full);
    s->hist = reinterpret_cast<int*>(hist);
    s->fk2 = reinterpret_cast<uint32_t*>(fk2);
    s->cnt = reinterpret_cast<int*>(cnt);
    s->tb = reinterpret_cast<int*>(tb);
    s->cb = reinterpret_cast<int*>(cb);
    s->cstart = reinterpret_cast<int*>(cstart);
    s->ncoll = reinterpret_cast<int*>(ncoll);
    s->misc = reinterpret_cast<int*>(misc);
    s->prop = reinterpret_cast<int8_t*>(prop);
    s->assign = reinterpret_cast<int16_t*>(assign);
    s->prev = reinterpret_cast<int16_t*>(prev);
    s->mlist = reinterpret_cast<int16_t*>(mlist);
    s->coll = reinterpret_cast<int16_t*>(coll);
    s->bin = reinterpret_cast<uint16_t*>(bin);
    s->ord = reinterpret_cast<uint32_t*>(ord);
  }
  return o;
}

__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }
__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ double key_f64(const SealArgs& a, int64_t s, int i) {
  double v = key_elem(a.keys, a.key_dtype, s, a.d, i);
  if (a.key_dtype == KD_FP8) v *= static_cast<double>(a.key_scale[s]);
  return v;
}

// Eight consecutive key elements [e0, e0 + 8) as float64 (d % 8 == 0).
__device__ __forceinline__ void load8(const SealArgs& a, int64_t row, int e0, double* x) {
  if (a.key_dtype == KD_BF16) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(a.keys) + row * a.d + e0));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[2 * u] = __uint_as_float(w[u] << 16);
      x[2 * u + 1] = __uint_as_float(w[u] & 0xFFFF0000u);
    }
  } else if (a.key_dtype == KD_FP8) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(
        reinterpret_cast<const uint8_t*>(a.keys) + row * a.d + e0));
    const double sc = static_cast<double>(a.key_scale[row]);
    const uint8_t* b = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
    for (int u = 0; u < 8; ++u) x[u] = static_cast<double>(fp8_to_f32(b[u])) * sc;
  } else {
    const float4* f = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(a.keys) + row * a.d + e0);
    const float4 p0 = __ldg(f), p1 = __ldg(f + 1);
    x[0] = p0.x; x[1] = p0.y; x[2] = p0.z; x[3] = p0.w;
    x[4] = p1.x; x[5] = p1.y; x[6] = p1.z; x[7] = p1.w;
  }
}

// Two consecutive key elements [e, e + 2) as float64 (e even).
__device__ __forceinline__ void load2(const SealArgs& a, int64_t row, int e, double* x) {
  if (a.key_dtype == KD_BF16) {
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(
        reinterpret_cast<const uint16_t*>(a.keys) + row * a.d + e));
    x[0] = __uint_as_float(v << 16);
    x[1] = __uint_as_float(v & 0xFFFF0000u);
  } else if (a.key_dtype == KD_FP8) {
    const uint16_t v = __ldg(reinterpret_cast<const uint16_t*>(
        reinterpret_cast<const uint8_t*>(a.keys) + row * a.d + e));
    const double sc = static_cast<double>(a.key_scale[row]);
    x[0] = static_cast<double>(fp8_to_f32(static_cast<uint8_t>(v & 0xFF))) * sc;
    x[1] = static_cast<double>(fp8_to_f32(static_cast<uint8_t>(v >> 8))) * sc;
  } else {
    const float2 v = __ldg(reinterpret_cast<const float2*>(reinterpret_cast<const float*>(a.keys) + row * a.d + e));
    x[0] = v.x;
    x[1] = v.y;
  }
}

// Pair order (distance, key, cluster): is (d1, i1, j1) <= (d2, i2, j2)?
__device__ __forceinline__ bool pair_le(uint64_t d1, uint32_t i1, uint32_t j1, uint64_t d2,
                                        uint32_t i2, uint32_t j2) {
  if (d1 != d2) return d1 < d2;
  if (i1 != i2) return i1 < i2;
  return j1 <= j2;
}

__device__ __forceinline__ uint64_t dbits(double v) { return static_cast<uint64_t>(__double_as_longlong(v)); }

// Histogram bin of a distance to cluster j: non-decreasing in the distance
// (each rounded step is monotone), so a smaller bin means a smaller distance.
__device__ __forceinline__ int dist_bin(const SealSmem& s, int j, double v) {
  const int b = __double2int_rz((v - s.dlo[j]) * s.dsc[j]);
  return b < 0 ? 0 : (b >= kBins ? kBins - 1 : b);
}

// D[j, i] for all keys of the window, two key rows per thread, the centre
// values read as pairs (the summation order per (i, j) is dimension order).
template <int MM, bool kBf16>
__device__ __forceinline__ void seal_dist(const SealArgs& a, const SealSmem& s, int64_t lo) {
  const int W = a.W, m = a.m, d = a.d;
  for (int i0 = 2 * threadIdx.x; i0 < W; i0 += 2 * blockDim.x) {
    const bool two = i0 + 1 < W;
    double xx0 = 0.0, xx1 = 0.0;
    double acc0[MM], acc1[MM];
#pragma unroll
    for (int j = 0; j < MM; ++j) {
      acc0[j] = 0.0;
      acc1[j] = 0.0;
    }
    // bf16 rows: the next 8-element block of both rows is loaded while the
    // current one is used (the rows come from L2 on every pass)
    const uint4* kp = kBf16 ? reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.keys) +
                                                             (lo + i0) * d)
                            : nullptr;
    uint4 n0 = kBf16 ? __ldg(kp) : make_uint4(0, 0, 0, 0);
    uint4 n1 = kBf16 && two ? __ldg(kp + d / 8) : make_uint4(0, 0, 0, 0);
    for (int e0 = 0; e0 < d; e0 += 8) {
      double x0[8], x1[8];
      if (kBf16) {
        const uint4 v0 = n0, v1 = n1;
        if (e0 + 8 < d) {
          n0 = __ldg(kp + (e0 + 8) / 8);
          if (two) n1 = __ldg(kp + d / 8 + (e0 + 8) / 8);
        }
        const uint32_t w0[4] = {v0.x, v0.y, v0.z, v0.w}, w1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          x0[2 * u] = __uint_as_float(w0[u] << 16);
          x0[2 * u + 1] = __uint_as_float(w0[u] & 0xFFFF0000u);
          x1[2 * u] = __uint_as_float(w1[u] << 16);
          x1[2 * u + 1] = __uint_as_float(w1[u] & 0xFFFF0000u);
        }
      } else {
        load8(a, lo + i0, e0, x0);
        if (two) {
          load8(a, lo + i0 + 1, e0, x1);
        } else {
#pragma unroll
          for (int u = 0; u < 8; ++u) x1[u] = 0.0;
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        xx0 = fma(x0[u], x0[u], xx0);
        xx1 = fma(x1[u], x1[u], xx1);
      }
#pragma unroll
      for (int j = 0; j < MM; ++j) {
        if (j < m) {
          const double2* c2 = reinterpret_cast<const double2*>(s.cent + j * d + e0);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const double2 c = c2[u];
            acc0[j] = fma(x0[2 * u], c.x, acc0[j]);
            acc0[j] = fma(x0[2 * u + 1], c.y, acc0[j]);
            acc1[j] = fma(x1[2 * u], c.x, acc1[j]);
            acc1[j] = fma(x1[2 * u + 1], c.y, acc1[j]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < MM; ++j) {
      if (j < m) {
        s.D[j * W + i0] = fmax(0.0, fma(-2.0, acc0[j], xx0) + s.cc[j]);
        if (two) s.D[j * W + i0 + 1] = fmax(0.0, fma(-2.0, acc1[j], xx1) + s.cc[j]);
      }
    }
  }
}

// Any m: one centre at a time (key row re-read per centre).
__device__ __forceinline__ void seal_dist_any(const SealArgs& a, const SealSmem& s, int64_t lo) {
  const int W = a.W, m = a.m, d = a.d;
  for (int i = threadIdx.x; i < W; i += blockDim.x) {
    double xx = 0.0;
    for (int e0 = 0; e0 < d; e0 += 8) {
      double x[8];
      load8(a, lo + i, e0, x);
#pragma unroll
      for (int u = 0; u < 8; ++u) xx = fma(x[u], x[u], xx);
    }
    for (int j = 0; j < m; ++j) {
      double acc = 0.0;
      for (int e0 = 0; e0 < d; e0 += 8) {
        double x[8];
        load8(a, lo + i, e0, x);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc = fma(x[u], s.cent[j * d + e0 + u], acc);
      }
      s.D[j * W + i] = fmax(0.0, fma(-2.0, acc, xx) + s.cc[j]);
    }
  }
}

__global__ void __launch_bounds__(kThreads) k_seal(SealArgs a) {
  extern __shared__ __align__(16) uint8_t raw[];
  const int W = a.W, m = a.m, d = a.d;
  SealSmem s;
  seal_layout(raw, W, m, d, &s);
  const int win = blockIdx.x;
  const int64_t lo = a.first_key + static_cast<int64_t>(win) * W;
  const int tid = threadIdx.x;
  const int warp = warp_id(), lane = lane_id();
  const int nwarps = blockDim.x >> 5;
  // loop bound over keys rounded up to whole warps (ballots need every lane)
  const int Wr = (W + 31) & ~31;

  // strided initialisation
  for (int e = tid; e < m * d; e += blockDim.x) {
    const int j = e / d, i = e % d;
    s.cent[e] = key_f64(a, lo + ((2 * j + 1) * W) / (2 * m), i);
  }
  for (int i = tid; i < W; i += blockDim.x) s.prev[i] = -1;
  __syncthreads();

  for (int it = 0; it < a.iters; ++it) {
    // squared centre norms for this pass
    for (int j = warp; j < m; j += nwarps) {
      double cc = 0.0;
      for (int e = lane; e < d; e += 32) cc = fma(s.cent[j * d + e], s.cent[j * d + e], cc);
      for (int o = 16; o > 0; o >>= 1) cc += __shfl_xor_sync(0xffffffffu, cc, o);
      if (lane == 0) s.cc[j] = cc;
    }
    __syncthreads();
    if (m <= 8 && a.key_dtype == KD_BF16) seal_dist<8, true>(a, s, lo);
    else if (m <= 8) seal_dist<8, false>(a, s, lo);
    else seal_dist_any(a, s, lo);
    for (int i = tid; i < W; i += blockDim.x) s.assign[i] = -1;
    for (int j = tid; j < m; j += blockDim.x) s.cnt[j] = 0;
    for (int e = tid; e < m * kBins; e += blockDim.x) s.hist[e] = 0;
    if (tid == 0) {
      *s.fullmask = 0ull;
      s.misc[2] = W;
    }
    __syncthreads();
    // per-cluster distance range: the histogram's origin and scale
    for (int j = warp; j < m; j += nwarps) {
      double mn = INFINITY, mx = 0.0;
      for (int i = lane; i < W; i += 32) {
        const double v = s.D[j * W + i];
        mn = fmin(mn, v);
        mx = fmax(mx, v);
      }
      for (int o = 16; o > 0; o >>= 1) {
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      if (lane == 0) {
        s.dlo[j] = mn;
        s.dsc[j] = mx > mn ? static_cast<double>(kBins) / (mx - mn) : 0.0;
      }
    }
    __syncthreads();
    // fixed for the pass: every pair's histogram bin and (m <= 8) every
    // key's clusters in (distance, cluster) order, so that a round only
    // skips the clusters that have filled
    for (int e = tid; e < m * W; e += blockDim.x) s.bin[e] = static_cast<uint16_t>(dist_bin(s, e / W, s.D[e]));
    if (m <= 8) {
      for (int i = tid; i < W; i += blockDim.x) {
        double dv[8];
        int jv[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          dv[j] = j < m ? s.D[j * W + i] : INFINITY;
          jv[j] = j;
        }
        // insertion by (distance, cluster): the order of the first-minimum scan
#pragma unroll
        for (int a1 = 1; a1 < 8; ++a1) {
#pragma unroll
          for (int b1 = a1; b1 > 0; --b1) {
            const bool sw = dv[b1] < dv[b1 - 1];
            const double td = sw ? dv[b1 - 1] : dv[b1];
            const int tj = sw ? jv[b1 - 1] : jv[b1];
            dv[b1 - 1] = sw ? dv[b1] : dv[b1 - 1];
            jv[b1 - 1] = sw ? jv[b1] : jv[b1 - 1];
            dv[b1] = td;
            jv[b1] = tj;
          }
        }
        uint32_t o = 0;
#pragma unroll
        for (int j = 7; j >= 0; --j) o = (o << 4) | static_cast<uint32_t>(jv[j]);
        s.ord[i] = o;
      }
    }
    __syncthreads();

    // greedy capacity assignment in rounds (see the file comment)
    for (int round = 0; round <= m && s.misc[2] > 0; ++round) {
      const unsigned long long fullm = *s.fullmask;
      // B. (first round) proposals: best open cluster of every free key,
      //    counted per bin; later rounds' proposals are kept by step G
      for (int i = tid; i < (round == 0 ? W : 0); i += blockDim.x) {
        int bj = -1;
        if (s.assign[i] < 0) {
          if (m <= 8) {
            // pop the clusters that filled since the last round (they stay full)
            uint32_t o = s.ord[i];
            for (int g = 0; g < m && ((fullm >> (o & 15u)) & 1ull); ++g) o >>= 4;
            s.ord[i] = o;
            const int oj = static_cast<int>(o & 15u);
            bj = (oj < m && !((fullm >> oj) & 1ull)) ? oj : -1;
          } else {
            double bd = 0.0;
            for (int j = 0; j < m; ++j) {
              if ((fullm >> j) & 1ull) continue;
              const double v = s.D[j * W + i];
              if (bj < 0 || v < bd) {
                bj = j;
                bd = v;
              }
            }
          }
        }
        s.prop[i] = static_cast<int8_t>(bj);
        if (bj >= 0) atomicAdd(&s.hist[bj * kBins + s.bin[bj * W + i]], 1);
      }
      if (round == 0) __syncthreads();
      // C. per open cluster, the bin where the running count reaches the
      //    (cap - count)-th proposal (none if the cluster cannot fill now):
      //    32-bin chunk sums, a scan over the chunks, a scan inside the one
      //    chunk.
      for (int j = warp; j < m; j += nwarps) {
        int found = -1, before = 0;
        if (!((fullm >> j) & 1ull)) {
          const int need = a.cap - s.cnt[j];
          int* hj = s.hist + j * kBins;
          // lane l sums chunk l (bins 32 l .. 32 l + 31), reading the bins in
          // a lane-skewed order so the warp's loads hit 32 different banks
          int csum = 0;
#pragma unroll 8
          for (int u = 0; u < 32; ++u) csum += hj[lane * 32 + ((u + lane) & 31)];
          int cin = csum;
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, cin, o);
            if (lane >= o) cin += t;
          }
          const unsigned cb = __ballot_sync(0xffffffffu, cin >= need);
          if (cb) {
            const int c = __ffs(cb) - 1;
            const int base = __shfl_sync(0xffffffffu, cin - csum, c);
            const int v = hj[c * 32 + lane];
            int incl = v;
            for (int o = 1; o < 32; o <<= 1) {
              const int t = __shfl_up_sync(0xffffffffu, incl, o);
              if (lane >= o) incl += t;
            }
            const unsigned bb = __ballot_sync(0xffffffffu, base + incl >= need);
            const int first = __ffs(bb) - 1;
            found = c * 32 + first;
            before = base + __shfl_sync(0xffffffffu, incl - v, first);
          }
        }
        if (lane == 0) {
          s.tb[j] = found;
          s.cb[j] = before;
          s.ncoll[j] = 0;
          s.fk1[j] = ~0ull;
          s.fk2[j] = ~0u;
        }
      }
      __syncthreads();
      // D. collect, per cluster, the proposals lying in its target bin
      for (int i = tid; i < W; i += blockDim.x) {
        const int j = s.prop[i];
        if (j >= 0 && s.tb[j] >= 0 && static_cast<int>(s.bin[j * W + i]) == s.tb[j])
          s.coll[j * W + atomicAdd(&s.ncoll[j], 1)] = static_cast<int16_t>(i);
      }
      __syncthreads();
      // E. exact rank (distance bits, key) inside the target bin, one warp
      //    per cluster: lanes hold entries, the others stream by shuffles
      for (int j = warp; j < m; j += nwarps) {
        const int nc = s.ncoll[j];
        if (s.tb[j] < 0 || nc == 0) continue;
        const int want = a.cap - s.cnt[j] - s.cb[j] - 1;
        const int16_t* cj = s.coll + j * W;
        for (int e0 = 0; e0 < nc; e0 += 32) {
          const int e = e0 + lane;
          const int i = e < nc ? cj[e] : 0;
          const uint64_t di = e < nc ? dbits(s.D[j * W + i]) : ~0ull;
          int r = 0;
          for (int x0 = 0; x0 < nc; x0 += 32) {
            const int xi = x0 + lane < nc ? cj[x0 + lane] : 0;
            const uint64_t xd = x0 + lane < nc ? dbits(s.D[j * W + xi]) : ~0ull;
            const int nx = min(32, nc - x0);
            for (int t = 0; t < nx; ++t) {
              const uint64_t dk = __shfl_sync(0xffffffffu, xd, t);
              const int k2 = __shfl_sync(0xffffffffu, xi, t);
              r += (dk < di || (dk == di && k2 < i)) ? 1 : 0;
            }
          }
          if (e < nc && r == want) {
            s.fk1[j] = di;
            s.fk2[j] = (static_cast<uint32_t>(i) << 16) | static_cast<uint32_t>(j);
          }
        }
      }
      __syncthreads();
      // F. the cluster that fills first closes this round (warp 0: lanes
      //    hold the fill pairs, an argmin in pair order)
      if (warp == 0) {
        uint64_t bd = ~0ull;
        uint32_t bk = ~0u;
        int bj = -1;
        for (int j = lane; j < m; j += 32) {
          if (s.fk2[j] == ~0u) continue;
          const uint64_t d1 = s.fk1[j];
          const uint32_t k1 = s.fk2[j] >> 16;
          if (bj < 0 || pair_le(d1, k1, j, bd, bk, bj)) {
            bd = d1;
            bk = k1;
            bj = j;
          }
        }
        // lanes below m hold the candidates: the first step pairs lanes o0 apart
        int o0 = 1;
        while (2 * o0 < m && o0 < 16) o0 <<= 1;
        for (int o = o0; o > 0; o >>= 1) {
          const uint64_t od = __shfl_xor_sync(0xffffffffu, bd, o);
          const uint32_t ok = __shfl_xor_sync(0xffffffffu, bk, o);
          const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
          if (oj >= 0 && (bj < 0 || pair_le(od, ok, oj, bd, bk, bj))) {
            bd = od;
            bk = ok;
            bj = oj;
          }
        }
        if (lane == 0) {
          s.misc[0] = bj;
          if (bj >= 0) *s.fullmask |= 1ull << bj;
        }
      }
      __syncthreads();
      // G. commit every proposal up to the filling pair (all if none), and
      //    keep the proposals and their counts current for the next round: a
      //    committed key leaves its cluster's histogram (rows of full
      //    clusters are not read again), and a free key whose cluster has
      //    just filled proposes its next open cluster
      const int best = s.misc[0];
      const uint64_t bk1 = best >= 0 ? s.fk1[best] : 0;
      const uint32_t bi = best >= 0 ? (s.fk2[best] >> 16) : 0;
      const unsigned long long fulln = *s.fullmask;  // now includes best
      for (int i0 = warp * 32; i0 < Wr; i0 += blockDim.x) {
        const int i = i0 + lane;
        const int j = i < W ? s.prop[i] : -1;
        bool take = false;
        if (j >= 0)
          take = best < 0 || pair_le(dbits(s.D[j * W + i]), i, j, bk1, bi, static_cast<uint32_t>(best));
        if (take) {
          s.assign[i] = static_cast<int16_t>(j);
          s.prop[i] = -1;
          if (best >= 0 && j != best) atomicSub(&s.hist[j * kBins + s.bin[j * W + i]], 1);
        } else if (j >= 0 && j == best) {
          int bj = -1;
          if (m <= 8) {
            uint32_t o = s.ord[i];
            for (int g = 0; g < m && ((fulln >> (o & 15u)) & 1ull); ++g) o >>= 4;
            s.ord[i] = o;
            const int oj = static_cast<int>(o & 15u);
            bj = (oj < m && !((fulln >> oj) & 1ull)) ? oj : -1;
          } else {
            double bd = 0.0;
            for (int jj = 0; jj < m; ++jj) {
              if ((fulln >> jj) & 1ull) continue;
              const double v = s.D[jj * W + i];
              if (bj < 0 || v < bd) {
                bj = jj;
                bd = v;
              }
            }
          }
          s.prop[i] = static_cast<int8_t>(bj);
          if (bj >= 0) atomicAdd(&s.hist[bj * kBins + s.bin[bj * W + i]], 1);
        }
        const int tj = take ? j : -1;
        const unsigned grp = __match_any_sync(0xffffffffu, tj);
        if (take && lane == __ffs(grp) - 1) atomicAdd(&s.cnt[j], __popc(grp));
        const unsigned nt = __ballot_sync(0xffffffffu, take);
        if (lane == 0 && nt) atomicSub(&s.misc[2], __popc(nt));
      }
      __syncthreads();
    }
    if (tid == 0 && s.misc[2] != 0) atomicOr(a.err, DEV_ERR_CAPACITY);

    // member lists (ascending key order), one warp per cluster
    if (tid == 0) {
      int run = 0;
      for (int j = 0; j < m; ++j) {
        s.cstart[j] = run;
        run += s.cnt[j];
      }
      s.cstart[m] = run;
    }
    __syncthreads();
    for (int j = warp; j < m; j += nwarps) {
      int w = s.cstart[j];
      for (int x0 = 0; x0 < W; x0 += 32) {
        const int x = x0 + lane;
        const bool in = x < W && s.assign[x] == j;
        const unsigned bal = __ballot_sync(0xffffffffu, in);
        if (in) s.mlist[w + __popc(bal & ((1u << lane) - 1u))] = static_cast<int16_t>(x);
        w += __popc(bal);
      }
    }
    __syncthreads();
    // update: float64 mean of the members in ascending key order.  A warp
    // takes (cluster, 64-dim block): each lane sums two dimensions over the
    // members in order, 16 member rows in flight.
    {
      const int nblk = (d + 63) / 64;
      for (int wj = warp; wj < m * nblk; wj += nwarps) {
        const int j = wj / nblk;
        const int e = (wj % nblk) * 64 + 2 * lane;
        const int b0 = s.cstart[j], b1 = s.cstart[j + 1];
        if (b1 == b0 || e >= d) continue;
        double s0 = 0.0, s1 = 0.0;
        int q = b0;
        if (a.key_dtype == KD_BF16) {
          // raw bf16 pairs: the loads of a batch are issued back to back
          const uint32_t* kp = reinterpret_cast<const uint32_t*>(a.keys) + (lo * d + e) / 2;
          // batches of 16 member rows; the next batch is loaded while the
          // current one is summed (in member order)
          uint32_t r[16];
          if (q + 16 <= b1) {
#pragma unroll
            for (int u = 0; u < 16; ++u) r[u] = __ldg(kp + static_cast<int64_t>(s.mlist[q + u]) * (d / 2));
          }
          for (; q + 16 <= b1; q += 16) {
            uint32_t c[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) c[u] = r[u];
            if (q + 32 <= b1) {
#pragma unroll
              for (int u = 0; u < 16; ++u) r[u] = __ldg(kp + static_cast<int64_t>(s.mlist[q + 16 + u]) * (d / 2));
            }
#pragma unroll
            for (int u = 0; u < 16; ++u) {
              s0 += static_cast<double>(__uint_as_float(c[u] << 16));
              s1 += static_cast<double>(__uint_as_float(c[u] & 0xFFFF0000u));
            }
          }
        }
        for (; q + 16 <= b1; q += 16) {
          double v[16][2];
#pragma unroll
          for (int u = 0; u < 16; ++u) load2(a, lo + s.mlist[q + u], e, v[u]);
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            s0 += v[u][0];
            s1 += v[u][1];
          }
        }
        for (; q < b1; ++q) {
          double v[2];
          load2(a, lo + s.mlist[q], e, v);
          s0 += v[0];
          s1 += v[1];
        }
        s.cent[j * d + e] = s0 / static_cast<double>(b1 - b0);
        s.cent[j * d + e + 1] = s1 / static_cast<double>(b1 - b0);
      }
    }
    if (tid == 0) s.misc[3] = 0;
    __syncthreads();
    for (int i = tid; i < W; i += blockDim.x)
      if (s.assign[i] != s.prev[i]) s.misc[3] = 1;
    __syncthreads();
    const bool changed = s.misc[3] != 0;
    for (int i = tid; i < W; i += blockDim.x) s.prev[i] = s.assign[i];
    __syncthreads();
    if (!changed) break;
  }

  // outputs: CSR (members ascending within each cluster), centroids, reps
  const int64_t mem0 = a.mem_base + static_cast<int64_t>(win) * W;
  const int64_t cl0 = a.cl_base + static_cast<int64_t>(win) * m;
  for (int j = tid; j < m; j += blockDim.x) a.offsets[cl0 + j] = static_cast<int32_t>(mem0 + s.cstart[j]);
  for (int x = tid; x < W; x += blockDim.x) a.members[mem0 + x] = static_cast<int32_t>(lo + s.mlist[x]);
  if (win == gridDim.x - 1 && tid == 0)
    a.offsets[a.cl_base + static_cast<int64_t>(gridDim.x) * m] =
        static_cast<int32_t>(a.mem_base + static_cast<int64_t>(gridDim.x) * W);
  for (int e = tid; e < m * d; e += blockDim.x) {
    a.centroids[cl0 * d + e] = s.cent[e];
    a.reps[cl0 * d + e] = f64_to_bf16_rne(s.cent[e]);
  }
}

// Block seal (the contiguous-block baseline): CTA (window, block j) owns
// keys [lo + floor(j W / m), lo + floor((j + 1) W / m)); its representative
// is the float64 mean of those keys in ascending order, rounded once to
// bf16.  Thread e sums dimensions e, e + blockDim, ...
__global__ void __launch_bounds__(128) k_seal_blocks(SealArgs a) {
  const int W = a.W, m = a.m, d = a.d;
  const int win = blockIdx.x / m, j = blockIdx.x % m;
  const int64_t lo = a.first_key + static_cast<int64_t>(win) * W;
  const int b0 = static_cast<int>((static_cast<int64_t>(j) * W) / m);
  const int b1 = static_cast<int>((static_cast<int64_t>(j + 1) * W) / m);
  const int64_t mem0 = a.mem_base + static_cast<int64_t>(win) * W;
  const int64_t cl = a.cl_base + static_cast<int64_t>(win) * m + j;
  for (int i = b0 + threadIdx.x; i < b1; i += blockDim.x) a.members[mem0 + i] = static_cast<int32_t>(lo + i);
  if (threadIdx.x == 0) {
    a.offsets[cl] = static_cast<int32_t>(mem0 + b0);
    if (blockIdx.x == gridDim.x - 1)
      a.offsets[a.cl_base + static_cast<int64_t>(a.n_windows) * m] =
          static_cast<int32_t>(a.mem_base + static_cast<int64_t>(a.n_windows) * W);
  }
  for (int e = threadIdx.x; e < d; e += blockDim.x) {
    double acc = 0.0;
    for (int i = b0; i < b1; ++i) acc += key_f64(a, lo + i, e);
    const double c = b1 > b0 ? acc / static_cast<double>(b1 - b0) : 0.0;
    a.centroids[cl * d + e] = c;
    a.reps[cl * d + e] = f64_to_bf16_rne(c);
  }
}

}  // namespace

size_t seal_smem_bytes(int W, int m, int d) { return seal_layout(nullptr, W, m, d, nullptr) + 16; }

cudaError_t launch_seal(const SealArgs& a, cudaStream_t st) {
  if (a.n_windows <= 0) return cudaSuccess;
  if (a.m < 1 || a.m > 64 || a.W < 1 || a.W > 32767 || a.d % 8 != 0) return cudaErrorInvalidValue;
  if (a.blocks) {
    count_launch();
    k_seal_blocks<<<a.n_windows * a.m, 128, 0, st>>>(a);
    return cudaGetLastError();
  }
  const size_t smem = seal_smem_bytes(a.W, a.m, a.d);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_seal, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  count_launch();
  k_seal<<<a.n_windows, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
