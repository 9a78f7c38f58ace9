// Exhaustive ("Full DSA") selection, second half: the top k of each query's
// row of indexer scores over keys 0..t (AttentionIndex explainer,
// paper-daily.com, section "它到底在解决什么问题？": the indexer scores every
// key before the query and the k highest are kept), written by (score
// desc, id asc).
//
// One CTA per row.  A row of n scores (up to the whole key store) is read
// once:
//  1. a threshold theta from a strided sample of the row: the r-th largest
//     of n_s sampled scores, with r set so that about 1.5 k keys of the row
//     are expected at or above it;
//  2. one vectorised pass collects every key whose score is >= theta as a
//     64-bit order key (~f2key(score) << 32 | id) into shared memory;
//  3. if at least k and at most kCand keys were collected, the top k of the
//     row are exactly the top k of the collected keys (every key scoring at
//     least the k-th score is >= theta); they are sorted and written.
// Otherwise (a sample far off the row's distribution) the row takes a
// radix select over all its items instead.  Rows of at most kCand keys are
// collected whole.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kThreads = 1024;
constexpr int kCand = 8192;     // collected keys held in shared memory
constexpr int kSample = 16384;  // sampled scores (share the same buffer)
static_assert(kCand >= kRowTopkMaxK, "the fallback sorts k keys in the same buffer");
constexpr size_t kSmem = static_cast<size_t>(kCand) * 8;

__global__ void __launch_bounds__(kThreads) k_row_topk(RowTopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw);
  uint32_t* samp = reinterpret_cast<uint32_t*>(smem_raw);  // sample keys (phase 1 only)
  __shared__ BlockScratch bs;
  __shared__ int s_cnt;
  const int qi = blockIdx.x;
  const int64_t t = a.q_pos0 + qi;
  const int64_t n64 = t + 1 < a.n_keys ? t + 1 : a.n_keys;
  const int n = static_cast<int>(n64 < 0 ? 0 : n64);
  const int k = a.k;
  const float* row = a.scores + static_cast<int64_t>(qi) * a.ld;
  int32_t* out = a.out + static_cast<int64_t>(qi) * k;
  float* outs = a.out_scores ? a.out_scores + static_cast<int64_t>(qi) * k : nullptr;
  const int tid = threadIdx.x, lane = tid & 31;

  // 1. threshold (order-preserving key) from a strided sample
  uint32_t ktheta = 0;  // every key is >= 0: collect all
  if (n > kCand) {
    const int ns = n < kSample ? n : kSample;
    for (int i = tid; i < ns; i += kThreads)
      samp[i] = f2key(row[static_cast<int64_t>(i) * n / ns]);
    __syncthreads();
    int64_t r = (3 * static_cast<int64_t>(k) * ns + 2 * static_cast<int64_t>(n) - 1) / (2 * static_cast<int64_t>(n)) + 8;
    r = r > ns ? ns : r;
    uint64_t above = 0;
    ktheta = radix_select(
        ns, [&](int i) -> uint32_t { return samp[i]; }, [](int) { return true; }, [](int) -> uint32_t { return 1u; },
        static_cast<uint64_t>(r), &above, bs);
    __syncthreads();  // the sample buffer becomes the candidate buffer
  }
  // 2. one pass: every key scoring >= theta (16-byte loads where aligned)
  if (tid == 0) s_cnt = 0;
  __syncthreads();
  auto push = [&](bool take, uint64_t key) {
    const unsigned bal = __ballot_sync(0xffffffffu, take);
    if (!bal) return;
    const int lead = __ffs(bal) - 1;
    int base = 0;
    if (lane == lead) base = atomicAdd(&s_cnt, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, lead);
    const int pos = base + __popc(bal & ((1u << lane) - 1u));
    if (take && pos < kCand) cand[pos] = key;
  };
  const int n4 = (reinterpret_cast<uintptr_t>(row) % 16 == 0) ? n / 4 : 0;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  const int n4r = (n4 + kThreads - 1) / kThreads * kThreads;  // whole warps for the ballots
  for (int i = tid; i < n4r; i += 2 * kThreads) {
    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
    const bool ok0 = i < n4, ok1 = i + kThreads < n4;
    if (ok0) v0 = row4[i];
    if (ok1) v1 = row4[i + kThreads];
    const float e0[4] = {v0.x, v0.y, v0.z, v0.w}, e1[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) push(ok0 && f2key(e0[u]) >= ktheta, order_key(e0[u], 4 * i + u));
#pragma unroll
    for (int u = 0; u < 4; ++u)
      push(ok1 && f2key(e1[u]) >= ktheta, order_key(e1[u], 4 * (i + kThreads) + u));
  }
  const int rest0 = 4 * n4;
  for (int j0 = rest0; j0 < n; j0 += kThreads) {
    const int j = j0 + tid;
    const float v = j < n ? row[j] : 0.f;
    push(j < n && f2key(v) >= ktheta, order_key(v, j));
  }
  __syncthreads();
  const int c = s_cnt;
  if (c >= (k < n ? k : n) && c <= kCand) {
    // 3. exact top k of the collected keys, sorted
    int np = 1;
    while (np < c) np <<= 1;
    for (int j = c + tid; j < np; j += kThreads) cand[j] = kOrderPad;
    __syncthreads();
    block_sort_u64(cand, np);
    const int nw = k < c ? k : c;
    for (int j = tid; j < k; j += kThreads) {
      const bool v = j < nw;
      out[j] = v ? order_key_id(cand[j]) : -1;
      if (outs) outs[j] = v ? order_key_score(cand[j]) : -INFINITY;
    }
    __syncthreads();
  } else {
    topk_select_emit(
        n, [&](int i) -> float { return row[i]; }, [&](int i) -> int32_t { return i; }, k, out, outs, bs, cand);
  }
}

}  // namespace

cudaError_t launch_row_topk(const RowTopkArgs& a, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  if (a.k <= 0 || a.k > kRowTopkMaxK) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_row_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmem));
  count_launch();
  k_row_topk<<<a.T, kThreads, kSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace aiidx
