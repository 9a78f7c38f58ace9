// Exhaustive ("Full DSA") selection, second half: the top k of each query's
// row of indexer scores over keys 0..t (AttentionIndex explainer,
// paper-daily.com, section "它到底在解决什么问题？": the indexer scores every
// key before the query and the k highest are kept), written by (score
// desc, id asc).
//
// One CTA per row.  A row of n scores (up to the whole key store) is read
// once:
//  1. a threshold theta from kSample scores at evenly strided positions (8
//     per thread, held in registers): the largest key such that at least r
//     sampled keys lie at or above it, resolved to a key range of width at
//     most 2^-22 of the sample's spread by two histogram levels over the
//     key's distance below the sample maximum.  r is set so that about
//     1.5 k keys of the row are expected at or above theta;
//  2. one vectorised pass collects every key whose score is >= theta as a
//     64-bit order key (~f2key(score) << 32 | id) into shared memory (one
//     warp vote per 8 scores; the rare hits are compacted by ballots);
//  3. if at least min(k, n) and at most kCand keys were collected, the top
//     k of the row are exactly the first k of the collected keys in order
//     (every key scoring at least the k-th score is >= theta).  They are
//     put in order by a counting sort over bins of the score key and a rank
//     by comparison inside each bin (a bitonic sort when a bin is crowded,
//     e.g. by equal scores), and the first k are written.
// Otherwise (a sample far off the row's distribution) the row takes a
// radix select over all its items instead.  Rows of at most kCand keys are
// collected whole.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kThreads = 1024;
constexpr int kCand = 8192;                  // collected keys held in shared memory
constexpr int kPerThread = 8;                // sampled scores per thread
constexpr int kSample = kThreads * kPerThread;
constexpr int kBins = kPrefixBins;          // histogram bins (2 per thread)
static_assert(kCand >= kRowTopkMaxK, "the fallback sorts k keys in the same buffer");
constexpr size_t kSmem = static_cast<size_t>(kCand) * 8 * 2 + static_cast<size_t>(kBins) * 4;

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Bin of hist[0 .. kBins) where the running count from bin 0 first reaches
// target (1 <= target <= total), and the count before that bin.  All
// threads call it; wt: 32 words of scratch.
__device__ __forceinline__ void hist_find(const uint32_t* hist, uint32_t target, uint32_t* wt, int* s_bin,
                                          uint32_t* s_before, int* bin, uint32_t* before) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t c0 = hist[2 * tid], c1 = hist[2 * tid + 1];
  const uint32_t loc = c0 + c1;
  uint32_t incl = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wt[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = wt[lane];
    uint32_t in2 = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_up_sync(0xffffffffu, in2, o);
      if (lane >= o) in2 += t;
    }
    wt[lane] = in2 - v;  // exclusive
  }
  __syncthreads();
  const uint32_t pre = wt[warp] + incl - loc;
  if (pre < target && pre + loc >= target) {
    const bool first = pre + c0 >= target;
    *s_bin = first ? 2 * tid : 2 * tid + 1;
    *s_before = first ? pre : pre + c0;
  }
  __syncthreads();
  *bin = *s_bin;
  *before = *s_before;
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads) k_row_topk(RowTopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw);  // [kCand] collected keys
  uint64_t* grp = cand + kCand;                            // [kCand] keys grouped by bin
  uint32_t* hist = reinterpret_cast<uint32_t*>(grp + kCand);  // [kBins]
  __shared__ BlockScratch bs;
  __shared__ uint32_t s_wt[32], s_red[2][32];
  __shared__ int s_cnt, s_bin;
  __shared__ uint32_t s_before;
  const int qi = blockIdx.x;
  const int64_t t = a.q_pos0 + qi;
  const int64_t n64 = t + 1 < a.n_keys ? t + 1 : a.n_keys;
  const int n = static_cast<int>(n64 < 0 ? 0 : n64);
  const int k = a.k;
  const float* row = a.scores + static_cast<int64_t>(qi) * a.ld;
  int32_t* out = a.out + static_cast<int64_t>(qi) * k;
  float* outs = a.out_scores ? a.out_scores + static_cast<int64_t>(qi) * k : nullptr;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // 1. threshold (order-preserving key) from the strided sample
  uint32_t ktheta = 0;  // every key is >= 0: collect all
  if (n > kCand) {
    uint32_t sk[kPerThread];
    uint32_t kmn = 0xffffffffu, kmx = 0u;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) {
      const int64_t i = tid + j * kThreads;
      sk[j] = f2key(__ldg(row + i * n / kSample));
      kmn = min(kmn, sk[j]);
      kmx = max(kmx, sk[j]);
    }
    for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      kmn = min(kmn, __shfl_xor_sync(0xffffffffu, kmn, o));
      kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, o));
    }
    if (lane == 0) {
      s_red[0][warp] = kmn;
      s_red[1][warp] = kmx;
    }
    __syncthreads();
    kmn = s_red[0][0];
    kmx = s_red[1][0];
    for (int w = 1; w < kThreads / 32; ++w) {
      kmn = min(kmn, s_red[0][w]);
      kmx = max(kmx, s_red[1][w]);
    }
    int64_t r = (3 * static_cast<int64_t>(k) * kSample + 2 * static_cast<int64_t>(n) - 1) / (2 * static_cast<int64_t>(n)) + 8;
    r = r > kSample ? kSample : r;
    // level 1: distance below the maximum, (kmx - kmn) >> sh1 < kBins
    const uint32_t range = kmx - kmn;
    int sh1 = 0;
    while (sh1 < 32 && (static_cast<uint64_t>(range) >> sh1) >= static_cast<uint64_t>(kBins)) ++sh1;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) atomicAdd(&hist[(kmx - sk[j]) >> sh1], 1u);
    __syncthreads();
    int b1;
    uint32_t cb1;
    hist_find(hist, static_cast<uint32_t>(r), s_wt, &s_bin, &s_before, &b1, &cb1);
    // level 2: inside bin b1, sub-bins of width 2^sh2
    uint64_t dhi;  // largest distance below the maximum that is collected
    if (sh1 > 0) {
      const int sh2 = sh1 > 11 ? sh1 - 11 : 0;
      for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
      __syncthreads();
      const uint32_t lo1 = static_cast<uint32_t>(b1) << sh1;
#pragma unroll
      for (int j = 0; j < kPerThread; ++j) {
        const uint32_t dd = kmx - sk[j];
        if ((dd >> sh1) == static_cast<uint32_t>(b1)) atomicAdd(&hist[(dd - lo1) >> sh2], 1u);
      }
      __syncthreads();
      int b2;
      uint32_t cb2;
      hist_find(hist, static_cast<uint32_t>(r) - cb1, s_wt, &s_bin, &s_before, &b2, &cb2);
      dhi = static_cast<uint64_t>(lo1) + ((static_cast<uint64_t>(b2) + 1) << sh2) - 1;
    } else {
      dhi = static_cast<uint64_t>(b1);
    }
    ktheta = dhi >= kmx ? 0u : kmx - static_cast<uint32_t>(dhi);
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
  const int n4r = (n4 + kThreads - 1) / kThreads * kThreads;  // whole warps for the votes
  for (int i = tid; i < n4r; i += 2 * kThreads) {
    // the rows come from DRAM: the lines two iterations ahead are requested
    // into L2 now, so more of the row is in flight than the loads below hold
    if (i + 4 * kThreads < n4) prefetch_l2(row4 + i + 4 * kThreads);
    if (i + 5 * kThreads < n4) prefetch_l2(row4 + i + 5 * kThreads);
    float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0;
    const bool ok0 = i < n4, ok1 = i + kThreads < n4;
    if (ok0) v0 = row4[i];
    if (ok1) v1 = row4[i + kThreads];
    const float e[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    unsigned hits = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) hits |= (f2key(e[u]) >= ktheta ? 1u : 0u) << u;
    hits &= (ok0 ? 0x0fu : 0u) | (ok1 ? 0xf0u : 0u);
    if (__any_sync(0xffffffffu, hits != 0)) {
#pragma unroll
      for (int u = 0; u < 4; ++u) push((hits >> u) & 1u, order_key(e[u], 4 * i + u));
#pragma unroll
      for (int u = 0; u < 4; ++u) push((hits >> (4 + u)) & 1u, order_key(e[4 + u], 4 * (i + kThreads) + u));
    }
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
    // 3. the first k collected keys in order
    const int nw = k < c ? k : c;
    emit_sorted_prefix(cand, c, nw, grp, hist, out, outs);
    for (int j = nw + tid; j < k; j += kThreads) {
      out[j] = -1;
      if (outs) outs[j] = -INFINITY;
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
