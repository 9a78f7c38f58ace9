// Exhaustive ("Full DSA") selection, second half: the top k of each query's
// row of indexer scores over keys 0..t (AttentionIndex explainer,
// paper-daily.com, section "它到底在解决什么问题？": the indexer scores every
// key before the query and the k highest are kept).  One CTA per row;
// radix select on the order-preserving float key, ties to the lower key id,
// ids written by (score desc, id asc).
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

__global__ void __launch_bounds__(1024) k_row_topk(RowTopkArgs a) {
  __shared__ BlockScratch bs;
  __shared__ uint64_t sbuf[kRowTopkMaxK];  // output sort
  const int qi = blockIdx.x;
  const int64_t t = a.q_pos0 + qi;
  const int64_t n64 = t + 1 < a.n_keys ? t + 1 : a.n_keys;
  const int n = static_cast<int>(n64 < 0 ? 0 : n64);
  const float* row = a.scores + static_cast<int64_t>(qi) * a.ld;
  topk_select_emit(
      n, [&](int i) -> float { return row[i]; }, [&](int i) -> int32_t { return i; }, a.k,
      a.out + static_cast<int64_t>(qi) * a.k,
      a.out_scores ? a.out_scores + static_cast<int64_t>(qi) * a.k : nullptr, bs, sbuf);
}

}  // namespace

cudaError_t launch_row_topk(const RowTopkArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  if (a.k <= 0 || a.k > kRowTopkMaxK) return cudaErrorInvalidValue;
  count_launch();
  k_row_topk<<<a.T, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
