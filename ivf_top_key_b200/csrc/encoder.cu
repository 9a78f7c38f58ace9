// Learned representative correction (one bounded correction per cluster).
//
// AttentionIndex explainer (paper-daily.com), section "代表向量为什么要学？":
// one small network per layer reads a cluster's member mean, the log of its
// size, and the mean and max of a learned per-key transform of its members;
// it outputs a bounded correction that is added to the mean, is zero at
// initialisation, and runs only when clusters are sealed or refit.  The
// kurate.org review calls it a DeepSets encoder.  Reading implemented here
// (float64 throughout, weights given as float32):
//   phi(k) = ReLU(A k + a)
//   f      = [mean phi ; max phi ; mu ; ln n]            (3d + 1 inputs)
//   h      = ReLU(B1 f + b1);   t = tanh(B2 h + b2)
//   corr   = t * min(1, 0.25 ||mu|| / ||t||)  (0 if t = 0)
//   rep    = bf16(mu + corr)
// One CTA of d threads per cluster; thread o owns output feature o.  The
// per-key transform phi is computed once per key when it is appended
// (k_phi) and pooled from that cache at every seal and refit.
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

constexpr int kEncThreads = 128;
constexpr int kBatch = 8;

// One CTA per cluster, thread o owns output feature o (d <= 128).  A is
// staged in shared memory with padded rows (conflict-free column walks);
// members are transformed 8 at a time; the MLP rows are read coalesced by
// whole warps.
__global__ void __launch_bounds__(kEncThreads) k_encoder(EncoderArgs a) {
  const int c = a.cl_begin + blockIdx.x;
  if (c >= a.cl_end) return;
  const int d = a.d, o = threadIdx.x;
  const int lane = o & 31, warp = o >> 5;
  const int F = 3 * d + 1;
  extern __shared__ double sh[];
  double* keyb = sh;                      // [kBatch][d]
  double* f = keyb + kBatch * d;          // [3d + 1]
  double* hv = f + F;                     // [d]
  double* red = hv + d;                   // [8]
  float* As = reinterpret_cast<float*>(red + 8);  // [d][d + 1]
  const float* A = a.wts;
  const float* av = A + d * d;
  const float* B1 = av + d;
  const float* b1 = B1 + static_cast<int64_t>(d) * F;
  const float* B2 = b1 + d;
  const float* b2 = B2 + d * d;
  const int o0 = a.offsets[c], o1 = a.offsets[c + 1];
  const int n = o1 - o0;
  const bool act = o < d;
  const double mu = act ? a.centroids[static_cast<int64_t>(c) * d + o] : 0.0;
  if (n <= 0) {
    if (act) a.reps[static_cast<int64_t>(c) * d + o] = f64_to_bf16_rne(mu);
    return;
  }
  double psum = 0.0, pmax = 0.0;  // phi >= 0, so 0 starts the max
  if (a.phi) {
    // phi of every key was computed when it arrived (launch_phi, same
    // arithmetic): pool the members' rows in member order
    if (act) {
      for (int p0 = o0; p0 < o1; p0 += kBatch) {
        double ph[kBatch];
#pragma unroll
        for (int r = 0; r < kBatch; ++r)
          ph[r] = p0 + r < o1 ? a.phi[static_cast<int64_t>(a.members[p0 + r]) * d + o] : 0.0;
#pragma unroll
        for (int r = 0; r < kBatch; ++r) {
          if (p0 + r < o1) {
            psum += ph[r];
            pmax = ph[r] > pmax ? ph[r] : pmax;
          }
        }
      }
    }
  } else {
  for (int e = o; e < d * d; e += blockDim.x) As[(e / d) * (d + 1) + (e % d)] = A[e];
  const double ao = act ? static_cast<double>(av[o]) : 0.0;
  for (int p0 = o0; p0 < o1; p0 += kBatch) {
    const int nb = min(kBatch, o1 - p0);
    __syncthreads();
    for (int e = o; e < nb * d; e += blockDim.x) {
      const int r = e / d, i = e % d;
      const int64_t s = a.members[p0 + r];
      double v = key_elem(a.keys, a.key_dtype, s, d, i);
      if (a.key_dtype == KD_FP8) v *= static_cast<double>(a.key_scale[s]);
      keyb[r * d + i] = v;
    }
    __syncthreads();
    if (act) {
      double z[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r) z[r] = ao;
      for (int i = 0; i < d; ++i) {
        const double w = static_cast<double>(As[o * (d + 1) + i]);
#pragma unroll
        for (int r = 0; r < kBatch; ++r) z[r] = fma(w, keyb[r * d + i], z[r]);
      }
      for (int r = 0; r < nb; ++r) {
        const double ph = z[r] > 0.0 ? z[r] : 0.0;
        psum += ph;
        pmax = ph > pmax ? ph : pmax;
      }
    }
  }
  }  // phi computed here
  __syncthreads();
  if (act) {
    f[o] = psum / static_cast<double>(n);
    f[d + o] = pmax;
    f[2 * d + o] = mu;
  }
  if (o == 0) f[3 * d] = log(static_cast<double>(n));
  __syncthreads();
  // h = ReLU(B1 f + b1): one warp per output row, lanes over the row
  for (int r = warp; r < d; r += blockDim.x >> 5) {
    double acc = 0.0;
    for (int j = lane; j < F; j += 32)
      acc = fma(static_cast<double>(B1[static_cast<int64_t>(r) * F + j]), f[j], acc);
    for (int s2 = 16; s2 > 0; s2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s2);
    if (lane == 0) {
      const double h = acc + static_cast<double>(b1[r]);
      hv[r] = h > 0.0 ? h : 0.0;
    }
  }
  __syncthreads();
  // z = B2 h + b2, t = tanh(z)
  for (int r = warp; r < d; r += blockDim.x >> 5) {
    double acc = 0.0;
    for (int j = lane; j < d; j += 32) acc = fma(static_cast<double>(B2[r * d + j]), hv[j], acc);
    for (int s2 = 16; s2 > 0; s2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s2);
    if (lane == 0) f[r] = tanh(acc + static_cast<double>(b2[r]));  // reuse f[0..d) for t
  }
  __syncthreads();
  const double t = act ? f[o] : 0.0;
  // ||t|| and ||mu|| (block reductions)
  double tt = t * t, mm = mu * mu;
  for (int s2 = 16; s2 > 0; s2 >>= 1) {
    tt += __shfl_xor_sync(0xffffffffu, tt, s2);
    mm += __shfl_xor_sync(0xffffffffu, mm, s2);
  }
  if (lane == 0) {
    red[warp] = tt;
    red[4 + warp] = mm;
  }
  __syncthreads();
  double tn2 = 0.0, mn2 = 0.0;
  for (int w = 0; w < (kEncThreads >> 5); ++w) {
    tn2 += red[w];
    mn2 += red[4 + w];
  }
  const double tn = sqrt(tn2);
  double corr = 0.0;
  if (tn > 0.0) {
    const double bound = 0.25 * sqrt(mn2);
    corr = t * (bound / tn < 1.0 ? bound / tn : 1.0);
  }
  if (act) a.reps[static_cast<int64_t>(c) * d + o] = f64_to_bf16_rne(mu + corr);
}

// phi(k) = ReLU(A k + a) for 64 keys per CTA (thread o = output feature),
// 8 at a time, with exactly the arithmetic of k_encoder's own loop (same
// float64 FMA order), so cached and recomputed values are identical.
constexpr int kPhiKeys = 64;
__global__ void __launch_bounds__(kEncThreads) k_phi(const void* keys, const float* key_scale, int key_dtype,
                                                     int d, const float* wts, int64_t s0, int64_t s1,
                                                     double* phi) {
  extern __shared__ double sh[];
  double* keyb = sh;                                        // [kBatch][d]
  float* As = reinterpret_cast<float*>(keyb + kBatch * d);  // [d][d + 1]
  const int o = threadIdx.x;
  const bool act = o < d;
  const int64_t b0 = s0 + static_cast<int64_t>(blockIdx.x) * kPhiKeys;
  const int64_t b1 = b0 + kPhiKeys < s1 ? b0 + kPhiKeys : s1;
  for (int e = o; e < d * d; e += blockDim.x) As[(e / d) * (d + 1) + (e % d)] = wts[e];
  const double ao = act ? static_cast<double>(wts[d * d + o]) : 0.0;
  for (int64_t p0 = b0; p0 < b1; p0 += kBatch) {
    const int nb = static_cast<int>(b1 - p0 < kBatch ? b1 - p0 : kBatch);
    __syncthreads();
    for (int e = o; e < nb * d; e += blockDim.x) {
      const int r = e / d, i = e % d;
      const int64_t s = p0 + r;
      double v = key_elem(keys, key_dtype, s, d, i);
      if (key_dtype == KD_FP8) v *= static_cast<double>(key_scale[s]);
      keyb[r * d + i] = v;
    }
    __syncthreads();
    if (act) {
      double z[kBatch];
#pragma unroll
      for (int r = 0; r < kBatch; ++r) z[r] = ao;
      for (int i = 0; i < d; ++i) {
        const double w = static_cast<double>(As[o * (d + 1) + i]);
#pragma unroll
        for (int r = 0; r < kBatch; ++r) z[r] = fma(w, keyb[r * d + i], z[r]);
      }
      for (int r = 0; r < nb; ++r) phi[(p0 + r) * d + o] = z[r] > 0.0 ? z[r] : 0.0;
    }
  }
}

}  // namespace

cudaError_t launch_phi(const void* keys, const float* key_scale, int key_dtype, int d, const float* wts,
                       int64_t s0, int64_t s1, double* phi, cudaStream_t st) {
  if (s1 <= s0) return cudaSuccess;
  if (d > kEncThreads) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(kBatch) * d * 8 + static_cast<size_t>(d) * (d + 1) * 4;
  const cudaError_t e = cudaFuncSetAttribute(k_phi, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t blocks = (s1 - s0 + kPhiKeys - 1) / kPhiKeys;
  count_launch();
  k_phi<<<static_cast<unsigned>(blocks), kEncThreads, smem, st>>>(keys, key_scale, key_dtype, d, wts, s0, s1, phi);
  return cudaGetLastError();
}

cudaError_t launch_encoder(const EncoderArgs& a, cudaStream_t st) {
  const int n = a.cl_end - a.cl_begin;
  if (n <= 0) return cudaSuccess;
  if (a.d > kEncThreads) return cudaErrorInvalidValue;
  // with cached phi the weight staging is not needed: a smaller footprint
  // lets the encoder share SMs with other kernels
  const size_t smem = static_cast<size_t>(kBatch * a.d + 3 * a.d + 1 + a.d + 8) * 8 +
                      (a.phi ? 0 : static_cast<size_t>(a.d) * (a.d + 1) * 4);
  const cudaError_t e = cudaFuncSetAttribute(k_encoder, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  count_launch();
  k_encoder<<<n, kEncThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
