// Seal: size-capped k-means of each completed W-key window into m clusters.
//
// AttentionIndex explainer (paper-daily.com), section "索引怎么边算边建？",
// item 2: every W open keys are grouped into m clusters, appended to the
// index, and the existing clusters are left alone; the kurate.org review
// ("Core Contribution", item 1) names the method size-capped k-means.  The
// pages give no algorithm; the reading implemented here:
//   init    c_j = x[floor((j + 1/2) W / m)]
//   repeat  at most `iters` times, stopping when the assignment repeats:
//           D_ij = ||x_i - c_j||^2 (float64)
//           visit all (i, j) pairs by (D asc, i asc, j asc); key i joins
//           cluster j if i is still free and j has fewer than cap keys
//           c_j = mean of its members (float64, ascending key order)
// Members are stored per cluster in ascending key id; the representative is
// the mean rounded once to bf16 (round to nearest even).
//
// One CTA (1024 threads) per window.  The W*m distances are sorted with a
// shared-memory bitonic sort of (distance bits, pair index); the greedy walk
// is done by one warp, 32 sorted pairs at a time: within a batch the first
// live pair of each key is the only one that can win, pairs of one cluster
// are ranked in order, and the batch is committed up to the first pair
// refused for lack of room (which happens at most m times per pass), so the
// result equals the sequential walk.
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

constexpr int kThreads = 1024;

struct SealSmem {
  uint64_t* dkey;    // [NP] distance bits
  uint16_t* pidx;    // [NP] pair index i*m + j
  double* cent;      // [m, d]
  int16_t* assign;   // [W]
  int16_t* prev;     // [W]
  uint8_t* taken;    // [W]
  int* cnt;          // [m]
  int* cstart;       // [m + 1] member list starts
  int16_t* mlist;    // [W] members, grouped by cluster, ascending
  int* flag;         // [2]
};

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

__device__ __forceinline__ bool pair_less(uint64_t d1, uint16_t p1, uint64_t d2, uint16_t p2) {
  return d1 < d2 || (d1 == d2 && p1 < p2);
}

__global__ void __launch_bounds__(kThreads) k_seal(SealArgs a) {
  extern __shared__ uint8_t raw[];
  const int W = a.W, m = a.m, d = a.d;
  const int np_pairs = W * m;
  int NP = 1;
  while (NP < np_pairs) NP <<= 1;
  SealSmem s;
  uint8_t* p = raw;
  s.dkey = reinterpret_cast<uint64_t*>(p);
  p += static_cast<size_t>(NP) * 8;
  s.cent = reinterpret_cast<double*>(p);
  p += static_cast<size_t>(m) * d * 8;
  s.pidx = reinterpret_cast<uint16_t*>(p);
  p += static_cast<size_t>(NP) * 2;
  s.assign = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W) * 2;
  s.prev = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W) * 2;
  s.taken = p;
  p += (W + 15) / 16 * 16;
  s.cnt = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m) * 4;
  s.cstart = reinterpret_cast<int*>(p);
  p += static_cast<size_t>(m + 1) * 4;
  s.mlist = reinterpret_cast<int16_t*>(p);
  p += static_cast<size_t>(W + 8) / 8 * 16;
  s.flag = reinterpret_cast<int*>(p);

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
    // distances: one key row per thread, read once in 8-element chunks,
    // against all m centres (m <= 16 in registers, else one centre at a time)
    for (int i = tid; i < W; i += blockDim.x) {
      const int64_t row = lo + i;
      if (m <= 16) {
        double acc[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[j] = 0.0;
        for (int e0 = 0; e0 < d; e0 += 8) {
          double x[8];
          load8(a, row, e0, x);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < m) {
              const double* c = s.cent + j * d + e0;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const double df = x[u] - c[u];
                acc[j] = fma(df, df, acc[j]);
              }
            }
          }
        }
        for (int j = 0; j < m; ++j) {
          s.dkey[i * m + j] = static_cast<uint64_t>(__double_as_longlong(acc[j]));
          s.pidx[i * m + j] = static_cast<uint16_t>(i * m + j);
        }
      } else {
        for (int j = 0; j < m; ++j) {
          double acc = 0.0;
          for (int e0 = 0; e0 < d; e0 += 8) {
            double x[8];
            load8(a, row, e0, x);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const double df = x[u] - s.cent[j * d + e0 + u];
              acc = fma(df, df, acc);
            }
          }
          s.dkey[i * m + j] = static_cast<uint64_t>(__double_as_longlong(acc));
          s.pidx[i * m + j] = static_cast<uint16_t>(i * m + j);
        }
      }
    }
    for (int q = np_pairs + tid; q < NP; q += blockDim.x) {
      s.dkey[q] = ~0ull;
      s.pidx[q] = 0xFFFFu;
    }
    for (int i = tid; i < W; i += blockDim.x) s.taken[i] = 0;
    for (int j = tid; j < m; j += blockDim.x) s.cnt[j] = 0;
    __syncthreads();
    // bitonic sort by (distance, pair index)
    for (int k = 2; k <= NP; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int q = tid; q < NP; q += blockDim.x) {
          const int r = q ^ j;
          if (r > q) {
            const uint64_t d1 = s.dkey[q], d2 = s.dkey[r];
            const uint16_t p1 = s.pidx[q], p2 = s.pidx[r];
            const bool up = (q & k) == 0;
            if (pair_less(d2, p2, d1, p1) == up) {
              s.dkey[q] = d2;
              s.dkey[r] = d1;
              s.pidx[q] = p2;
              s.pidx[r] = p1;
            }
          }
        }
        __syncthreads();
      }
    }
    // greedy capacity assignment (warp 0)
    if (tid < 32) {
      const int lane = tid;
      const unsigned lt = (1u << lane) - 1u;
      int pos = 0, n_free = W;
      while (pos < np_pairs && n_free > 0) {
        const int q = pos + lane;
        const bool valid = q < np_pairs;
        const int pi = valid ? s.pidx[q] : 0;
        const int i = pi / m, j = pi % m;
        const bool live = valid && !s.taken[i] && s.cnt[j] < a.cap;
        const unsigned mi = __match_any_sync(0xffffffffu, live ? i : -1 - lane);
        const bool leader = live && (__ffs(mi) - 1 == lane);
        const unsigned mj = __match_any_sync(0xffffffffu, leader ? j : -1 - lane);
        const int rank = __popc(mj & lt);
        const bool ok = leader && (s.cnt[j] + rank < a.cap);
        const unsigned bad = __ballot_sync(0xffffffffu, leader && !ok);
        const int limit = bad ? __ffs(bad) - 1 : 32;
        const bool acc = ok && lane < limit;
        const unsigned accj = __match_any_sync(0xffffffffu, acc ? j : -1 - lane);
        __syncwarp();
        if (acc) {
          s.taken[i] = 1;
          s.assign[i] = static_cast<int16_t>(j);
          if (__ffs(accj) - 1 == lane) s.cnt[j] += __popc(accj);
        }
        n_free -= __popc(__ballot_sync(0xffffffffu, acc));
        __syncwarp();
        pos += bad ? limit + 1 : 32;
      }
      if (lane == 0) s.flag[1] = n_free;
    }
    __syncthreads();
    if (tid == 0 && s.flag[1] != 0) atomicOr(a.err, DEV_ERR_CAPACITY);
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
      // update: float64 mean of the members in ascending key order
      for (int j = warp; j < m; j += blockDim.x >> 5) {
        const int b0 = s.cstart[j], b1 = s.cstart[j + 1];
        if (b1 == b0) continue;
        for (int e = lane; e < d; e += 32) {
          double sum = 0.0;
          int p = b0;
          for (; p + 4 <= b1; p += 4) {
            const double v0 = key_f64(a, lo + s.mlist[p], e);
            const double v1 = key_f64(a, lo + s.mlist[p + 1], e);
            const double v2 = key_f64(a, lo + s.mlist[p + 2], e);
            const double v3 = key_f64(a, lo + s.mlist[p + 3], e);
            sum += v0;
            sum += v1;
            sum += v2;
            sum += v3;
          }
          for (; p < b1; ++p) sum += key_f64(a, lo + s.mlist[p], e);
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
  int NP = 1;
  while (NP < W * m) NP <<= 1;
  return static_cast<size_t>(NP) * 10 + static_cast<size_t>(m) * d * 8 + static_cast<size_t>(W) * 4 +
         (W + 15) / 16 * 16 + static_cast<size_t>(m) * 4 + static_cast<size_t>(m + 1) * 4 +
         static_cast<size_t>(W + 8) / 8 * 16 + 16;
}

cudaError_t launch_seal(const SealArgs& a, cudaStream_t st) {
  if (a.n_windows <= 0) return cudaSuccess;
  if (a.m > 64 || a.W * a.m > 65535 || a.W > 32767 || a.d % 8 != 0) return cudaErrorInvalidValue;
  const size_t smem = seal_smem_bytes(a.W, a.m, a.d);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_seal, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  count_launch();
  k_seal<<<a.n_windows, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
