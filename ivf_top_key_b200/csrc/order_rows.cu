// Output order of the route+refine top-k: each query's k selected ids (and
// their scores), written by the refine kernel in candidate-slot order, are
// put in the order that defines the top-k: score descending, key id
// ascending (AttentionIndex explainer, paper-daily.com, section
// "查询时怎么挑候选？": the k highest-scoring candidates are kept).
//
// One CTA per query row.  The valid entries (a prefix of the row; -1
// padding follows) become 64-bit keys (~f2key(score) << 32 | id), which sort
// ascending into exactly that order.  A counting sort: keys are grouped by
// bin of their order-preserving score key over the row's [min, max] (equal
// integer ranges, about constant relative width), then each key's final
// position is its bin's start plus its rank among the bin's keys.  A bin
// holding more than kMaxBin keys (near-equal scores) sends the row through a
// bitonic sort instead.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxK = 2048;
constexpr int kBins = 2048;
constexpr int kMaxBin = 64;

__global__ void __launch_bounds__(kThreads) k_order_rows(OrderRowsArgs a) {
  __shared__ uint64_t A[kMaxK];      // keys in row order
  __shared__ uint64_t B[kMaxK];      // keys grouped by bin
  __shared__ uint32_t hist[kBins];   // counts, then bin starts / ends
  __shared__ uint32_t red[2 * (kThreads / 32)];
  __shared__ int nvalid, binmax;
  const int k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t row = blockIdx.x;
  const int32_t* ids = a.ids_in + row * k;
  const float* sc = a.scores_in + row * k;
  // keys, the number of valid entries and the score-key range
  if (tid == 0) nvalid = 0;
  for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
  __syncthreads();
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  int nv = 0;
  for (int j = tid; j < k; j += kThreads) {
    const int32_t id = ids[j];
    const float v = sc[j];
    const bool ok = id >= 0;
    A[j] = ok ? order_key(v, id) : kOrderPad;
    if (ok) {
      const uint32_t fk = f2key(v);
      kmin = min(kmin, fk);
      kmax = max(kmax, fk);
      ++nv;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    nv += __shfl_xor_sync(0xffffffffu, nv, o);
  }
  if (lane == 0) {
    red[warp] = kmin;
    red[kThreads / 32 + warp] = kmax;
    atomicAdd(&nvalid, nv);
  }
  __syncthreads();
  kmin = red[0];
  kmax = red[kThreads / 32];
  for (int w = 1; w < kThreads / 32; ++w) {
    kmin = min(kmin, red[w]);
    kmax = max(kmax, red[kThreads / 32 + w]);
  }
  const int n = nvalid;  // valid entries form a prefix of the row
  const uint32_t range = kmax - kmin;
  int shift = 0;
  while (shift < 32 && (static_cast<uint64_t>(range) >> shift) >= static_cast<uint64_t>(kBins)) ++shift;
  // bin of a key, highest score first (bin 0 = largest scores)
  auto bin = [=](uint64_t x) -> int {
    const uint32_t d = kmax - ~static_cast<uint32_t>(x >> 32);  // kmax - f2key(score)
    const uint32_t b = shift < 32 ? d >> shift : 0u;
    return b < static_cast<uint32_t>(kBins) ? static_cast<int>(b) : kBins - 1;
  };
  for (int j = tid; j < n; j += kThreads) atomicAdd(&hist[bin(A[j])], 1u);
  __syncthreads();
  // exclusive scan of the counts (thread t owns bins 8t .. 8t + 7), largest bin
  int c8[8], loc = 0, cmax = 0;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    c8[u] = static_cast<int>(hist[8 * tid + u]);
    loc += c8[u];
    cmax = max(cmax, c8[u]);
  }
  int incl = loc;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
  if (lane == 31) red[warp] = static_cast<uint32_t>(incl);
  if (lane == 0) red[kThreads / 32 + warp] = static_cast<uint32_t>(cmax);
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += static_cast<int>(red[w]);
  if (tid == 0) {
    int m = 0;
    for (int w = 0; w < kThreads / 32; ++w) m = max(m, static_cast<int>(red[kThreads / 32 + w]));
    binmax = m;
  }
  int run = before + incl - loc;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    hist[8 * tid + u] = static_cast<uint32_t>(run);  // start of bin 8 tid + u
    run += c8[u];
  }
  __syncthreads();
  int32_t* ids_out = a.ids_out + row * k;
  float* sc_out = a.scores_out ? a.scores_out + row * k : nullptr;
  if (binmax <= kMaxBin) {
    // group by bin; afterwards bin b spans [start(b), hist[b]) with
    // start(b) = hist[b - 1] (0 for b = 0)
    for (int j = tid; j < n; j += kThreads) {
      const uint64_t x = A[j];
      B[atomicAdd(&hist[bin(x)], 1u)] = x;
    }
    __syncthreads();
    for (int p = tid; p < n; p += kThreads) {
      const uint64_t x = B[p];
      const int b = bin(x);
      const int lo = b == 0 ? 0 : static_cast<int>(hist[b - 1]);
      const int hi = static_cast<int>(hist[b]);
      int r = lo;
      for (int q = lo; q < hi; ++q) r += B[q] < x ? 1 : 0;
      ids_out[r] = order_key_id(x);
      if (sc_out) sc_out[r] = order_key_score(x);
    }
  } else {
    int np = 1;
    while (np < n) np <<= 1;
    for (int j = n + tid; j < np; j += kThreads) A[j] = kOrderPad;
    __syncthreads();
    block_sort_u64(A, np);
    for (int j = tid; j < n; j += kThreads) {
      ids_out[j] = order_key_id(A[j]);
      if (sc_out) sc_out[j] = order_key_score(A[j]);
    }
  }
  for (int j = n + tid; j < k; j += kThreads) {
    ids_out[j] = -1;
    if (sc_out) sc_out[j] = -INFINITY;
  }
}

}  // namespace

cudaError_t launch_order_rows(const OrderRowsArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  if (a.k <= 0 || a.k > kMaxK) return cudaErrorInvalidValue;
  count_launch();
  k_order_rows<<<a.T, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
