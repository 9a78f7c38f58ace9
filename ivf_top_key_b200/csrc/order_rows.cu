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
#include "../../include/ai_index.h"
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxK = 2048;

// Slots for the valid entries of a merge row: all P * k, and room for the
// power of two the bitonic fallback of emit_sorted_prefix sorts in place.
__host__ __device__ inline int merge_items_cap(int P, int k) {
  const int L = P * k;
  int np = 1;
  while (np < (L < 8192 ? L : 8192)) np <<= 1;
  return L > np ? L : np;
}
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

// Merge of P partial top-k lists per row (the shards of a sharded rescore,
// or the parts of a divided one): the valid (id >= 0) entries of the row's
// P lists are compacted into shared memory as order keys, and the block
// writes the first k of them in order (score desc, id asc), padded with -1.
// The partial lists hold disjoint ids, and each holds its part's top k, so
// the union holds the row's top k.  Up to kMergeSort valid entries are
// ordered by the counting sort of emit_sorted_prefix; more take a radix
// select of the top k and a bitonic sort.
constexpr int kMergeSort = 8192;

__global__ void __launch_bounds__(1024) k_merge_rows(const int32_t* __restrict__ ids,
                                                    const float* __restrict__ scores, int P, int T, int k,
                                                    int32_t* out, float* out_scores) {
  extern __shared__ __align__(16) uint8_t raw[];
  const int L = P * k;
  const int cap = merge_items_cap(P, k);
  uint64_t* items = reinterpret_cast<uint64_t*>(raw);       // [cap] valid entries
  uint64_t* grp = items + cap;                              // [kMergeSort] grouping / output sort
  uint32_t* hist = reinterpret_cast<uint32_t*>(grp + kMergeSort);  // [kPrefixBins]
  __shared__ BlockScratch bs;
  __shared__ int s_n;
  const int row = blockIdx.x, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) s_n = 0;
  __syncthreads();
  const int Lr = (L + 31) & ~31;  // whole warps for the ballots
  for (int e = threadIdx.x; e < Lr; e += blockDim.x) {
    int32_t id = -1;
    float v = 0.f;
    if (e < L) {
      const int p = e / k, j = e % k;
      const int64_t o = (static_cast<int64_t>(p) * T + row) * k + j;
      id = ids[o];
      v = scores[o];
    }
    const bool ok = id >= 0;
    const unsigned bal = __ballot_sync(0xffffffffu, ok);
    int base = 0;
    if (bal) {
      const int lead = __ffs(bal) - 1;
      if (lane == lead) base = atomicAdd(&s_n, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, lead);
    }
    if (ok) items[base + __popc(bal & ((1u << lane) - 1u))] = order_key(v, id);
  }
  __syncthreads();
  const int n = s_n;
  int32_t* o_ids = out + static_cast<int64_t>(row) * k;
  float* o_sc = out_scores ? out_scores + static_cast<int64_t>(row) * k : nullptr;
  if (n <= kMergeSort) {
    const int nw = n < k ? n : k;
    emit_sorted_prefix(items, n, nw, grp, hist, o_ids, o_sc);
    for (int j = nw + threadIdx.x; j < k; j += blockDim.x) {
      o_ids[j] = -1;
      if (o_sc) o_sc[j] = -INFINITY;
    }
  } else {
    topk_select_emit(
        n, [&](int i) -> float { return order_key_score(items[i]); },
        [&](int i) -> int32_t { return order_key_id(items[i]); }, k, o_ids, o_sc, bs, grp);
  }
}

}  // namespace

size_t merge_smem_bytes(int P, int k) {
  return static_cast<size_t>(merge_items_cap(P, k)) * 8 + static_cast<size_t>(kMergeSort) * 8 +
         static_cast<size_t>(kPrefixBins) * 4;
}

cudaError_t launch_merge_rows(const int32_t* ids, const float* scores, int P, int T, int k, int32_t* out,
                              float* out_scores, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  const size_t smem = merge_smem_bytes(P, k);
  if (P < 1 || k < 1 || k > kTcMaxK || smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_merge_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  count_launch();
  k_merge_rows<<<T, 1024, smem, st>>>(ids, scores, P, T, k, out, out_scores);
  return cudaGetLastError();
}

cudaError_t launch_order_rows(const OrderRowsArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  if (a.k <= 0 || a.k > kMaxK) return cudaErrorInvalidValue;
  count_launch();
  k_order_rows<<<a.T, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx

// ------------------------------------------------------------------ C ABI
extern "C" int ai_merge_topk(const int32_t* ids_dev, const float* scores_dev, int32_t n_parts, int32_t T,
                             int32_t k, int32_t* out_dev, float* out_scores_dev, void* cuda_stream) {
  using namespace aiidx;
  if (!ids_dev || !scores_dev || !out_dev) {
    set_last_error("null pointer argument");
    return AI_ERR_ARG;
  }
  if (n_parts < 1 || T < 0 || k < 1 || k > kTcMaxK) {
    set_last_error("n_parts >= 1, T >= 0 and 1 <= k <= 2048 required");
    return AI_ERR_ARG;
  }
  const size_t smem = merge_smem_bytes(n_parts, k);
  if (smem > 227 * 1024) {
    set_last_error("n_parts * k too large for one block (n_parts * k <= 19840)");
    return AI_ERR_ARG;
  }
  if (T == 0) return AI_OK;
  const cudaError_t e = launch_merge_rows(ids_dev, scores_dev, n_parts, T, k, out_dev, out_scores_dev,
                                          static_cast<cudaStream_t>(cuda_stream));
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return AI_ERR_CUDA;
  }
  return AI_OK;
}
