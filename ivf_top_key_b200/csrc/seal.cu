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
// One CTA (1024 threads) per window.  The sequential greedy walk over the
// W*m sorted pairs is reproduced exactly in at most m + 1 data-parallel
// rounds: in a round every free key proposes its best pair among the
// clusters that are not full; the proposals are sorted by (cluster, pair
// order); the first cluster to fill is the one whose (cap - count)-th
// proposal comes first in pair order; every proposal up to that pair is
// final (nothing before it can be refused), that cluster is closed, and the
// remaining keys propose again.  Pair order is (distance, key, cluster).
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

constexpr int kThreads = 1024;

struct SealSmem {
  double* D;         // [W, m] squared distances
  double* cent;      // [m, d]
  double* cc;        // [m] squared centre norms
  uint64_t* bk1;     // [m, NPW] proposal buckets: distance bits
  uint16_t* bk2;     // [m, NPW] proposal buckets: key
  int* wcnt;         // [m, 32] per-(cluster, warp) counts / offsets
  int* bfill;        // [m] bucket sizes
  int* bpass;        // [m]
  int16_t* assign;   // [W]
  int16_t* prev;     // [W]
  int* cnt;          // [m] members so far
  int* tcnt;         // [m] (spare)
  int* tstart;       // [m + 1] (spare)
  int* cstart;       // [m + 1] member list starts
  int16_t* mlist;    // [W] members, grouped by cluster, ascending
  uint64_t* fk1;     // [m] fill pair of each cluster: distance bits
  uint32_t* fk2;     // [m] fill pair: (key << 16) | cluster
  int* flag;         // [4]
  int* red;          // [32] per-warp partial sums
  unsigned long long* fullmask;
};

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

// Pair order (distance, key, cluster): is (d1, i1, j1) <= (d2, i2, j2)?
__device__ __forceinline__ bool pair_le(uint64_t d1, uint32_t i1, uint32_t j1, uint64_t d2,
                                        uint32_t i2, uint32_t j2) {
  if (d1 != d2) return d1 < d2;
  if (i1 != i2) return i1 < i2;
  return j1 <= j2;
}

__global__ void __launch_bounds__(kThreads) k_seal(SealArgs a) {
  extern __shared__ uint8_t raw[];
  const int W = a.W, m = a.m, d = a.d;
  int NPW = 1;
  while (NPW < W) NPW <<= 1;
  SealSmem s;
  uint8_t* p = raw;
  s.D = reinterpret_cast<double*>(p);
  p += static_cast<size_t>(W) * m * 8;
  s.cent = reinterpret_cast<double*>(p);
  p += static_cast<size_t>(m) * d * 8;
  s.cc = reinterpret_cast<double*>(p);
  p += static_cast<size_t>(m) * 8;
  s.bk1 = reinterpret_cast<uint64_t*>(p);
  p += static_cast<size_t>(m) * NPW * 8;
  s.fk1 = reinterpret_cast<uint64_t*>(p);
  p += static_cast<size_t>(m) * 8;
  s.fullmask = reinterpret_cast<unsigned long long*>(p);
  p += 8;
  s.wcnt = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 32 * 4;
  s.bfill = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 4;
  s.bpass = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 4;
  s.fk2 = reinterpret_cast<uint32_t*>(p);
  p += static_cast<size_t>(m) * 4;
  s.cnt = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 4;
  s.tcnt = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 4;
  s.tstart = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m + 1) * 4;
  s.cstart = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m + 1) * 4;
  s.flag = reinterpret_cast<int*>(p);
  p += 16;
  s.red = reinterpret_cast<int*>(p);
  p += 128;
  s.assign = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W) * 2;
  s.prev = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W) * 2;
  s.mlist = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W) * 2;
  s.bk2 = reinterpret_cast<uint16_t*>(p);

  const int win = blockIdx.x;
  const int64_t lo = a.first_key + static_cast<int64_t>(win) * W;
  const int tid = threadIdx.x;

  // strided initialisation
  for (int e = tid; e < m * d; e += blockDim.x) {
    const int j = e / d, i = e % d;
    s.cent[e] = key_f64(a, lo + ((2 * j + 1) * W) / (2 * m), i);
  }
  for (int i = tid; i < W; i += blockDim.x) s.prev[i] = -1;
  __syncthreads();

  for (int it = 0; it < a.iters; ++it) {
    // squared centre norms for this pass
    for (int j = warp_id(); j < m; j += blockDim.x >> 5) {
      double cc = 0.0;
      for (int e = lane_id(); e < d; e += 32) cc = fma(s.cent[j * d + e], s.cent[j * d + e], cc);
      for (int o = 16; o > 0; o >>= 1) cc += __shfl_xor_sync(0xffffffffu, cc, o);
      if (lane_id() == 0) s.cc[j] = cc;
    }
    __syncthreads();
    // distances ||x||^2 - 2 x.c + ||c||^2 (float64, clamped at 0): one key
    // row per thread, read once, 32 elements per batch of loads
    for (int i = tid; i < W; i += blockDim.x) {
      const int64_t row = lo + i;
      double xx = 0.0;
      if (m <= 16) {
        double acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0.0;
        for (int e0 = 0; e0 < d; e0 += 8) {
          double x[8];
          load8(a, row, e0, x);
#pragma unroll
          for (int u = 0; u < 8; ++u) xx = fma(x[u], x[u], xx);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < m) {
              const double* c = s.cent + j * d + e0;
#pragma unroll
              for (int u = 0; u < 8; ++u) acc[j] = fma(x[u], c[u], acc[j]);
            }
          }
        }
        for (int j = 0; j < m; ++j) s.D[i * m + j] = fmax(0.0, fma(-2.0, acc[j], xx) + s.cc[j]);
      } else {
        for (int e0 = 0; e0 < d; e0 += 8) {
          double x[8];
          load8(a, row, e0, x);
#pragma unroll
          for (int u = 0; u < 8; ++u) xx = fma(x[u], x[u], xx);
        }
        for (int j = 0; j < m; ++j) {
          double acc = 0.0;
          for (int e0 = 0; e0 < d; e0 += 8) {
            double x[8];
            load8(a, row, e0, x);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc = fma(x[u], s.cent[j * d + e0 + u], acc);
          }
          s.D[i * m + j] = fmax(0.0, fma(-2.0, acc, xx) + s.cc[j]);
        }
      }
      s.assign[i] = -1;
    }
    for (int j = tid; j < m; j += blockDim.x) s.cnt[j] = 0;
    if (tid == 0) *s.fullmask = 0ull;
    __syncthreads();

    // greedy capacity assignment in rounds (see the file comment)
    int n_free = W;
    const int warp = tid >> 5, lane = tid & 31;
    const int nwarps = blockDim.x >> 5;
    for (int round = 0; round <= m && n_free > 0; ++round) {
      const unsigned long long fullm = *s.fullmask;
      // 1. proposals, bucketed by cluster without atomics: per-warp ballot
      //    counts -> (cluster, warp) offsets -> scatter
      for (int j = tid; j < m; j += blockDim.x) s.bfill[j] = 0;
      __syncthreads();
      for (int i0 = 0; i0 < W; i0 += blockDim.x) {
        const int i = i0 + tid;
        int bj = -1;
        double bd = 0.0;
        if (i < W && s.assign[i] < 0) {
          for (int j = 0; j < m; ++j) {
            if ((fullm >> j) & 1ull) continue;
            const double v = s.D[i * m + j];
            if (bj < 0 || v < bd) {
              bj = j;
              bd = v;
            }
          }
        }
        for (int j = 0; j < m; ++j) {
          const unsigned bal = __ballot_sync(0xffffffffu, bj == j);
          if (lane == 0) s.wcnt[j * nwarps + warp] = __popc(bal);
        }
        __syncthreads();
        // exclusive offsets of (cluster j, warp w) within this pass
        if (tid < m) {
          int run = 0;
          for (int w = 0; w < nwarps; ++w) {
            const int c = s.wcnt[tid * nwarps + w];
            s.wcnt[tid * nwarps + w] = run;
            run += c;
          }
          s.bpass[tid] = run;
        }
        __syncthreads();
        for (int j = 0; j < m; ++j) {
          const unsigned bal = __ballot_sync(0xffffffffu, bj == j);
          if (bj == j) {
            const int slot = s.bfill[j] + s.wcnt[j * nwarps + warp] + __popc(bal & ((1u << lane) - 1u));
            s.bk1[j * NPW + slot] = static_cast<uint64_t>(__double_as_longlong(bd));
            s.bk2[j * NPW + slot] = static_cast<uint16_t>(i);
          }
        }
        __syncthreads();
        if (tid < m) s.bfill[tid] += s.bpass[tid];
        __syncthreads();
      }
      // 2. the proposal that would fill each open cluster: the need-th
      //    smallest (distance, key) of its bucket, found by counting ranks
      //    (all threads; one entry each, compared against its bucket)
      if (tid == 0) {
        int run = 0;
        for (int j = 0; j < m; ++j) {
          s.tstart[j] = run;
          run += s.bfill[j];
        }
        s.tstart[m] = run;
      }
      for (int j = tid; j < m; j += blockDim.x) {
        s.fk1[j] = ~0ull;
        s.fk2[j] = ~0u;
      }
      __syncthreads();
      for (int e = tid; e < s.tstart[m]; e += blockDim.x) {
        int j = 0;
        while (j + 1 < m && s.tstart[j + 1] <= e) ++j;
        const int need = a.cap - s.cnt[j];
        const int nb = s.bfill[j];
        if (((fullm >> j) & 1ull) || nb < need || need <= 0) continue;
        const uint64_t* k1 = s.bk1 + j * NPW;
        const uint16_t* k2 = s.bk2 + j * NPW;
        const int me = e - s.tstart[j];
        const uint64_t a1 = k1[me];
        const uint16_t a2 = k2[me];
        int rank = 0;
        for (int x = 0; x < nb; ++x) {
          const uint64_t b1 = k1[x];
          rank += (b1 < a1 || (b1 == a1 && k2[x] < a2)) ? 1 : 0;
        }
        if (rank == need - 1) {
          s.fk1[j] = a1;
          s.fk2[j] = (static_cast<uint32_t>(a2) << 16) | static_cast<uint32_t>(j);
        }
      }
      __syncthreads();
      if (tid == 0) {
        int best = -1;
        for (int j = 0; j < m; ++j) {
          if (s.fk1[j] == ~0ull && s.fk2[j] == ~0u) continue;
          if (best < 0 || pair_le(s.fk1[j], s.fk2[j] >> 16, s.fk2[j] & 0xFFFFu, s.fk1[best],
                                  s.fk2[best] >> 16, s.fk2[best] & 0xFFFFu))
            best = j;
        }
        s.flag[2] = best;
      }
      __syncthreads();
      const int best = s.flag[2];
      const uint64_t bk1 = best >= 0 ? s.fk1[best] : 0;
      const uint32_t bi = best >= 0 ? (s.fk2[best] >> 16) : 0;
      // 3. commit every proposal up to the filling pair (all if none)
      for (int i = tid; i < W; i += blockDim.x) {
        if (s.assign[i] >= 0) continue;
        int bj = -1;
        double bd = 0.0;
        for (int j = 0; j < m; ++j) {
          if ((fullm >> j) & 1ull) continue;
          const double v = s.D[i * m + j];
          if (bj < 0 || v < bd) {
            bj = j;
            bd = v;
          }
        }
        if (bj >= 0 && (best < 0 || pair_le(static_cast<uint64_t>(__double_as_longlong(bd)), i, bj, bk1, bi,
                                            static_cast<uint32_t>(best))))
          s.assign[i] = static_cast<int16_t>(bj);
      }
      if (tid == 0 && best >= 0) *s.fullmask |= 1ull << best;
      __syncthreads();
      // member counts and keys still free (ballots, no shared atomics)
      {
        int mine = 0;
        for (int i = tid; i < W; i += blockDim.x) mine += s.assign[i] < 0 ? 1 : 0;
        for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
        if (lane == 0) s.red[warp] = mine;
        for (int j = 0; j < m; ++j) {
          int cj = 0;
          for (int i0 = 0; i0 < W; i0 += blockDim.x) {
            const int i = i0 + tid;
            cj += __popc(__ballot_sync(0xffffffffu, i < W && s.assign[i] == j));
          }
          if (lane == 0) s.wcnt[j * nwarps + warp] = cj;
        }
        __syncthreads();
        n_free = 0;
        for (int w = 0; w < nwarps; ++w) n_free += s.red[w];
        if (tid < m) {
          int c = 0;
          for (int w = 0; w < nwarps; ++w) c += s.wcnt[tid * nwarps + w];
          s.cnt[tid] = c;
        }
        __syncthreads();
      }
    }
    if (tid == 0 && n_free != 0) atomicOr(a.err, DEV_ERR_CAPACITY);

    // member lists (ascending key order), one warp per cluster
    {
      const int warp = tid >> 5, lane = tid & 31;
      if (tid == 0) {
        int run = 0;
        for (int j = 0; j < m; ++j) {
          s.cstart[j] = run;
          run += s.cnt[j];
        }
        s.cstart[m] = run;
      }
      __syncthreads();
      for (int j = warp; j < m; j += blockDim.x >> 5) {
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
      // update: float64 mean of the members in ascending key order; the
      // (cluster, 32-dim block) pairs are spread over all warps
      const int nblk = (d + 31) / 32;
      for (int wj = warp; wj < m * nblk; wj += blockDim.x >> 5) {
        const int j = wj / nblk;
        const int b0 = s.cstart[j], b1 = s.cstart[j + 1];
        if (b1 == b0) continue;
        for (int e = (wj % nblk) * 32 + lane; e < d && e < (wj % nblk) * 32 + 32; e += 32) {
          double sum = 0.0;
          int q = b0;
          for (; q + 4 <= b1; q += 4) {
            const double v0 = key_f64(a, lo + s.mlist[q], e);
            const double v1 = key_f64(a, lo + s.mlist[q + 1], e);
            const double v2 = key_f64(a, lo + s.mlist[q + 2], e);
            const double v3 = key_f64(a, lo + s.mlist[q + 3], e);
            sum += v0;
            sum += v1;
            sum += v2;
            sum += v3;
          }
          for (; q < b1; ++q) sum += key_f64(a, lo + s.mlist[q], e);
          s.cent[j * d + e] = sum / static_cast<double>(b1 - b0);
        }
      }
    }
    if (tid == 0) s.flag[0] = 0;
    __syncthreads();
    for (int i = tid; i < W; i += blockDim.x)
      if (s.assign[i] != s.prev[i]) s.flag[0] = 1;
    __syncthreads();
    const bool changed = s.flag[0] != 0;
    for (int i = tid; i < W; i += blockDim.x) s.prev[i] = s.assign[i];
    __syncthreads();
    if (!changed) break;
  }

  // outputs: CSR (members ascending within each cluster), centroids, reps
  const int64_t mem0 = a.mem_base + static_cast<int64_t>(win) * W;
  const int64_t cl0 = a.cl_base + static_cast<int64_t>(win) * m;
  if (tid < m) a.offsets[cl0 + tid] = static_cast<int32_t>(mem0 + s.cstart[tid]);
  for (int x = tid; x < W; x += blockDim.x) a.members[mem0 + x] = static_cast<int32_t>(lo + s.mlist[x]);
  if (win == gridDim.x - 1 && tid == 0)
    a.offsets[a.cl_base + static_cast<int64_t>(gridDim.x) * m] =
        static_cast<int32_t>(a.mem_base + static_cast<int64_t>(gridDim.x) * W);
  for (int e = tid; e < m * d; e += blockDim.x) {
    a.centroids[cl0 * d + e] = s.cent[e];
    a.reps[cl0 * d + e] = f64_to_bf16_rne(s.cent[e]);
  }
}

}  // namespace

size_t seal_smem_bytes(int W, int m, int d) {
  int NPW = 1;
  while (NPW < W) NPW <<= 1;
  // D, centres, proposal buckets (m x NPW of u64 + u16), counters, key lists
  return static_cast<size_t>(W) * m * 8 + static_cast<size_t>(m) * d * 8 +
         static_cast<size_t>(m) * NPW * 10 + static_cast<size_t>(m) * 12 + 8 +
         static_cast<size_t>(m) * 32 * 4 + static_cast<size_t>(m) * 8 +
         static_cast<size_t>(m + 1) * 8 + 16 + 128 + static_cast<size_t>(W) * 6 +
         static_cast<size_t>(m) * 32 + 256 + static_cast<size_t>(m) * 8;
}

cudaError_t launch_seal(const SealArgs& a, cudaStream_t st) {
  if (a.n_windows <= 0) return cudaSuccess;
  if (a.m > 64 || a.W > 65535 || a.d % 8 != 0) return cudaErrorInvalidValue;
  const size_t smem = seal_smem_bytes(a.W, a.m, a.d);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_seal, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  count_launch();
  k_seal<<<a.n_windows, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
