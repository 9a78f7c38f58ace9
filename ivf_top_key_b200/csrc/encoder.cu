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
// One CTA of d threads per cluster; thread o owns output feature o.
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

__global__ void k_encoder(EncoderArgs a) {
  const int c = a.cl_begin + blockIdx.x;
  if (c >= a.cl_end) return;
  const int d = a.d, o = threadIdx.x;
  const int F = 3 * d + 1;
  extern __shared__ double sh[];
  double* key = sh;          // [d]
  double* f = sh + d;        // [3d + 1]
  double* hv = f + F;        // [d]
  double* red = hv + d;      // [d] reduction scratch
  const float* A = a.wts;
  const float* av = A + d * d;
  const float* B1 = av + d;
  const float* b1 = B1 + static_cast<int64_t>(d) * F;
  const float* B2 = b1 + d;
  const float* b2 = B2 + d * d;
  const int o0 = a.offsets[c], o1 = a.offsets[c + 1];
  const int n = o1 - o0;
  const double mu = a.centroids[static_cast<int64_t>(c) * d + o];
  if (n <= 0) {
    a.reps[static_cast<int64_t>(c) * d + o] = f64_to_bf16_rne(mu);
    return;
  }
  double psum = 0.0, pmax = 0.0;  // phi >= 0, so 0 is a valid start for the max
  for (int p = o0; p < o1; ++p) {
    const int64_t s = a.members[p];
    __syncthreads();
    double v = key_elem(a.keys, a.key_dtype, s, d, o);
    if (a.key_dtype == KD_FP8) v *= static_cast<double>(a.key_scale[s]);
    key[o] = v;
    __syncthreads();
    double z = static_cast<double>(av[o]);
    for (int i = 0; i < d; ++i) z = fma(static_cast<double>(A[o * d + i]), key[i], z);
    z = z > 0.0 ? z : 0.0;
    psum += z;
    pmax = z > pmax ? z : pmax;
  }
  __syncthreads();
  f[o] = psum / static_cast<double>(n);
  f[d + o] = pmax;
  f[2 * d + o] = mu;
  if (o == 0) f[3 * d] = log(static_cast<double>(n));
  __syncthreads();
  double h = static_cast<double>(b1[o]);
  for (int j = 0; j < F; ++j) h = fma(static_cast<double>(B1[static_cast<int64_t>(o) * F + j]), f[j], h);
  hv[o] = h > 0.0 ? h : 0.0;
  __syncthreads();
  double z = static_cast<double>(b2[o]);
  for (int j = 0; j < d; ++j) z = fma(static_cast<double>(B2[o * d + j]), hv[j], z);
  const double t = tanh(z);
  // ||t|| and ||mu||
  red[o] = t * t;
  __syncthreads();
  double tn2 = 0.0;
  for (int j = 0; j < d; ++j) tn2 += red[j];
  __syncthreads();
  red[o] = mu * mu;
  __syncthreads();
  double mn2 = 0.0;
  for (int j = 0; j < d; ++j) mn2 += red[j];
  const double tn = sqrt(tn2);
  double corr = 0.0;
  if (tn > 0.0) {
    const double bound = 0.25 * sqrt(mn2);
    corr = t * (bound / tn < 1.0 ? bound / tn : 1.0);
  }
  a.reps[static_cast<int64_t>(c) * d + o] = f64_to_bf16_rne(mu + corr);
}

}  // namespace

cudaError_t launch_encoder(const EncoderArgs& a, cudaStream_t st) {
  const int n = a.cl_end - a.cl_begin;
  if (n <= 0) return cudaSuccess;
  if (a.d > 1024) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(a.d * 3 + 3 * a.d + 1) * 8;
  count_launch();
  k_encoder<<<n, a.d, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
