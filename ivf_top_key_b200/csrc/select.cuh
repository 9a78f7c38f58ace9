// Block-wide selection helpers: ordered compaction and radix select.
//
// Used by the per-query top-k (candidate scores in shared memory), the
// exhaustive row top-k (scores in global memory) and the size-weighted
// cluster threshold of the candidate fill.
#pragma once

#include <cstddef>

#include "common.cuh"

namespace aiidx {

// 16-byte aligned: bcast[2 .. 3] also holds a 64-bit value (offset 1192),
// which needs an 8-byte aligned address whatever else the block declares.
struct __align__(16) BlockScratch {
  uint32_t hist[256];     // radix histogram (counts or weights)
  int warp_tot[40];       // per-warp totals for ordered compaction
  int bcast[8];           // broadcast slots
};
static_assert(offsetof(BlockScratch, bcast) % 8 == 0, "bcast[2] holds a 64-bit value");

// Exclusive prefix of `pred` over the block in thread order.  Returns this
// thread's rank among the threads with pred set; *total receives the count.
// Every thread of the block must call it.
__device__ __forceinline__ int block_rank(bool pred, int* total, BlockScratch& bs) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = (blockDim.x + 31) >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, pred);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) bs.warp_tot[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    int v = lane < nwarps ? bs.warp_tot[lane] : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane < nwarps) bs.warp_tot[lane] = incl - v;  // exclusive
    if (lane == 31) bs.bcast[7] = incl;
  }
  __syncthreads();
  const int r = bs.warp_tot[warp] + in_warp;
  *total = bs.bcast[7];
  __syncthreads();
  return r;
}

// Radix select over n items with 32-bit keys: find theta, the key of the
// k-th largest item among those with pred(i), with weights wt(i) (the
// k-th unit of weight).  Returns theta and *above = weight strictly above
// theta.  If the total weight is <= k, returns 0 and *above = total.
// key(i), pred(i), wt(i) are functors; all threads call it.
template <class KeyF, class PredF, class WtF>
__device__ uint32_t radix_select(int n, KeyF key, PredF pred, WtF wt, uint64_t k, uint64_t* above,
                                 BlockScratch& bs, uint64_t* tot_out = nullptr) {
  uint32_t prefix = 0, mask = 0;
  uint64_t need = k;
  uint64_t above_acc = 0;
  // total weight
  __shared__ unsigned long long s_tot;
  if (threadIdx.x == 0) s_tot = 0;
  __syncthreads();
  {
    unsigned long long loc = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x)
      if (pred(i)) loc += wt(i);
    for (int o = 16; o > 0; o >>= 1) loc += __shfl_xor_sync(0xffffffffu, loc, o);
    if ((threadIdx.x & 31) == 0 && loc) atomicAdd(&s_tot, loc);
  }
  __syncthreads();
  const uint64_t total = s_tot;
  if (tot_out) *tot_out = total;
  if (total <= k) {
    *above = total;
    __syncthreads();
    return 0;
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) bs.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      if (!pred(i)) continue;
      const uint32_t kk = key(i);
      if ((kk & mask) != prefix) continue;
      atomicAdd(&bs.hist[(kk >> shift) & 255u], static_cast<uint32_t>(wt(i)));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // scan digits from 255 down; lane l owns digits 255-8l .. 248-8l
      const int lane = threadIdx.x;
      uint64_t loc[8];
      uint64_t lsum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        loc[j] = bs.hist[255 - (lane * 8 + j)];
        lsum += loc[j];
      }
      uint64_t incl = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        uint64_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      uint64_t run = incl - lsum;  // weight of digits above this lane's range
      int found = -1;
      uint64_t before = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (found < 0 && run + loc[j] >= need && run < need) {
          found = 255 - (lane * 8 + j);
          before = run;
        }
        run += loc[j];
      }
      const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
      const int src = __ffs(who) - 1;
      const int dg = __shfl_sync(0xffffffffu, found, src);
      const uint64_t bf = __shfl_sync(0xffffffffu, before, src);
      if (lane == 0) {
        bs.bcast[0] = dg;
        reinterpret_cast<unsigned long long*>(&bs.bcast[2])[0] = bf;
      }
    }
    __syncthreads();
    const uint32_t dg = static_cast<uint32_t>(bs.bcast[0]);
    const uint64_t bf = reinterpret_cast<unsigned long long*>(&bs.bcast[2])[0];
    need -= bf;
    above_acc += bf;
    prefix |= dg << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  *above = above_acc;
  return prefix;
}

// ------------------------------------------------------- output ordering
// Every top-k result is written in the order that defines it: score
// descending, then key id ascending.  One 64-bit key per selected item,
// (~f2key(score) << 32) | id, sorts ascending into exactly that order (ids
// are non-negative), and its score is recovered exactly by key2f.
__device__ __forceinline__ uint64_t order_key(float v, int32_t id) {
  return (static_cast<uint64_t>(~f2key(v)) << 32) | static_cast<uint32_t>(id);
}
__device__ __forceinline__ int32_t order_key_id(uint64_t x) { return static_cast<int32_t>(x & 0xffffffffu); }
__device__ __forceinline__ float order_key_score(uint64_t x) {
  return key2f(~static_cast<uint32_t>(x >> 32));
}
constexpr uint64_t kOrderPad = ~0ull;  // sorts after every real key

// Bitonic sort, ascending, of buf[0 .. np) (np a power of two) by all
// threads of the block.
__device__ __forceinline__ void block_sort_u64(uint64_t* buf, int np) {
  for (int kk = 2; kk <= np; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int p = threadIdx.x; p < (np >> 1); p += blockDim.x) {
        const int i = 2 * j * (p / j) + (p % j);  // lower element of pair p
        const uint64_t x = buf[i], y = buf[i + j];
        const bool asc = (i & kk) == 0;
        if ((x > y) == asc) {
          buf[i] = y;
          buf[i + j] = x;
        }
      }
      __syncthreads();
    }
  }
}

// Top-k of n items (score(i), id(i)) by (score desc, id asc).  Writes the
// selected ids (and scores) in that order, then pads with -1 / -inf up to
// k.  sbuf: shared memory for the next power of two >= k keys.  All
// threads call it.
template <class ScoreF, class IdF>
__device__ void topk_select_emit(int n, ScoreF score, IdF id, int k, int32_t* out, float* outs,
                                 BlockScratch& bs, uint64_t* sbuf) {
  auto skey = [&](int i) -> uint32_t { return f2key(score(i)); };
  auto all = [&](int) -> bool { return true; };
  auto one = [&](int) -> uint32_t { return 1u; };
  uint64_t above = 0, tot = 0;
  const uint32_t theta = radix_select(n, skey, all, one, static_cast<uint64_t>(k), &above, bs, &tot);
  const bool take_all = tot <= static_cast<uint64_t>(k);
  uint32_t theta_id = 0;
  bool ties_all = true;
  if (!take_all) {
    const uint64_t need_eq = k - above;
    auto idkey = [&](int i) -> uint32_t { return ~static_cast<uint32_t>(id(i)); };
    auto tie = [&](int i) -> bool { return skey(i) == theta; };
    uint64_t above2 = 0, tot2 = 0;
    theta_id = radix_select(n, idkey, tie, one, need_eq, &above2, bs, &tot2);
    ties_all = tot2 <= need_eq;
  }
  int written = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + threadIdx.x;
    bool p = false;
    float sv = 0.f;
    if (i < n) {
      sv = score(i);
      if (take_all) {
        p = true;
      } else {
        const uint32_t kk = f2key(sv);
        p = kk > theta || (kk == theta && (ties_all || (~static_cast<uint32_t>(id(i))) >= theta_id));
      }
    }
    int total;
    const int r = block_rank(p, &total, bs);
    if (p && written + r < k) sbuf[written + r] = order_key(sv, id(i));
    written += total;
  }
  const int nw = min(written, k);
  int np = 1;
  while (np < nw) np <<= 1;
  for (int j = nw + threadIdx.x; j < np; j += blockDim.x) sbuf[j] = kOrderPad;
  __syncthreads();
  block_sort_u64(sbuf, np);
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const bool v = j < nw;
    const uint64_t x = v ? sbuf[j] : kOrderPad;
    out[j] = v ? order_key_id(x) : -1;
    if (outs) outs[j] = v ? order_key_score(x) : -INFINITY;
  }
  __syncthreads();
}

// ------------------------------------------- sorted prefix of a key set
// For blocks of exactly 1024 threads.  keys[0 .. c) hold c distinct order
// keys (any order); their first nw (nw <= c) in ascending order -- score
// descending, id ascending -- are written to out[0 .. nw) (ids) and
// outs[0 .. nw) (scores, if outs).  A counting sort: the keys are grouped
// by bin of their score key over the set's range (kPrefixBins equal integer
// ranges of the order-preserving key, about constant relative width), and a
// key's position is its bin's start plus its rank among the bin's keys;
// only the bins that start before nw are grouped and ranked.  One of those
// holding more than 64 keys (near-equal scores) sends the block to a
// bitonic sort of keys instead, which needs keys to hold the next power of
// two >= c slots.  grp: c slots of scratch; hist: kPrefixBins words.  Ends
// with the block synchronised; keys and grp are clobbered.
constexpr int kPrefixBins = 2048;

__device__ inline void emit_sorted_prefix(uint64_t* keys, int c, int nw, uint64_t* grp, uint32_t* hist, int32_t* out,
                                   float* outs) {
  constexpr int kMaxBin = 64;
  __shared__ uint32_t s_wt[32], s_red[2][32];
  __shared__ int s_bmax, s_bend, s_nbin;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // score-key range of the keys (high words: ~f2key(score))
  uint32_t hmn = 0xffffffffu, hmx = 0u;
  for (int j = tid; j < c; j += 1024) {
    const uint32_t h = static_cast<uint32_t>(keys[j] >> 32);
    hmn = min(hmn, h);
    hmx = max(hmx, h);
  }
  for (int i = tid; i < kPrefixBins; i += 1024) hist[i] = 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    hmn = min(hmn, __shfl_xor_sync(0xffffffffu, hmn, o));
    hmx = max(hmx, __shfl_xor_sync(0xffffffffu, hmx, o));
  }
  if (lane == 0) {
    s_red[0][warp] = hmn;
    s_red[1][warp] = hmx;
  }
  __syncthreads();
  hmn = s_red[0][0];
  hmx = s_red[1][0];
  for (int w = 1; w < 32; ++w) {
    hmn = min(hmn, s_red[0][w]);
    hmx = max(hmx, s_red[1][w]);
  }
  // Keys are binned by (hi - hmn) >> sh over [hmn, hhi]; keys above hhi
  // (lower scores) get bin kPrefixBins.  After the first histogram the
  // first nw keys are known to lie in bins [0, b_end); when that is a small
  // part of the range (a wide range: outliers, scores of both signs) the
  // histogram is taken once more over just that part.
  uint32_t hhi = hmx;
  int sh = 0;
  auto bin = [&](uint64_t x) -> int {
    const uint32_t h = static_cast<uint32_t>(x >> 32);
    return h > hhi ? kPrefixBins : static_cast<int>((h - hmn) >> sh);
  };
  for (int round = 0;; ++round) {
    sh = 0;
    while (sh < 32 && (static_cast<uint64_t>(hhi - hmn) >> sh) >= static_cast<uint64_t>(kPrefixBins)) ++sh;
    if (round > 0) {
      for (int i = tid; i < kPrefixBins; i += 1024) hist[i] = 0;
      __syncthreads();
    }
    for (int j = tid; j < c; j += 1024) {
      const int b = bin(keys[j]);
      if (b < kPrefixBins) atomicAdd(&hist[b], 1u);
    }
    __syncthreads();
    // exclusive scan of the counts (thread t owns bins 2t, 2t + 1)
    const uint32_t c0 = hist[2 * tid], c1 = hist[2 * tid + 1];
    const uint32_t loc = c0 + c1;
    uint32_t incl = loc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t tt = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += tt;
    }
    if (lane == 31) s_wt[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t v = s_wt[lane];
      uint32_t in2 = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t tt = __shfl_up_sync(0xffffffffu, in2, o);
        if (lane >= o) in2 += tt;
      }
      s_wt[lane] = in2 - v;
    }
    __syncthreads();
    const uint32_t st0 = s_wt[warp] + incl - loc, st1 = st0 + c0;  // bin starts
    // Only the bins starting before nw hold any of the first nw keys (bins
    // run from the highest scores down): b_end is the first bin starting at
    // or after nw, and the largest count among the bins before it decides
    // between the counting sort and the bitonic sort.
    uint32_t cm = max(st0 < static_cast<uint32_t>(nw) ? c0 : 0u, st1 < static_cast<uint32_t>(nw) ? c1 : 0u);
    uint32_t be = st0 >= static_cast<uint32_t>(nw) ? 2 * tid
                                                    : (st1 >= static_cast<uint32_t>(nw) ? 2 * tid + 1 : kPrefixBins);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, o));
      be = min(be, __shfl_xor_sync(0xffffffffu, be, o));
    }
    if (lane == 0) {
      s_red[0][warp] = cm;
      s_red[1][warp] = be;
    }
    if (tid == 1023) s_nbin = static_cast<int>(st1 + c1);  // keys binned (hi <= hhi)
    hist[2 * tid] = st0;
    hist[2 * tid + 1] = st1;
    __syncthreads();
    if (warp == 0) {
      uint32_t m2 = s_red[0][lane], b2 = s_red[1][lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        m2 = max(m2, __shfl_xor_sync(0xffffffffu, m2, o));
        b2 = min(b2, __shfl_xor_sync(0xffffffffu, b2, o));
      }
      if (lane == 0) {
        s_bmax = static_cast<int>(m2);
        s_bend = static_cast<int>(b2);
      }
    }
    __syncthreads();
    const int be_all = s_bend;
    if (round > 0 || sh == 0 || be_all > kPrefixBins / 4) break;
    // the keys of bins [0, be_all) span hi in [hmn, hmn + (be_all << sh) - 1]
    const uint64_t top = static_cast<uint64_t>(hmn) + (static_cast<uint64_t>(be_all) << sh) - 1;
    hhi = top < hhi ? static_cast<uint32_t>(top) : hhi;
    __syncthreads();  // every thread has read s_bend before the next round
  }
  const int b_end = s_bend;
  // keys of bins [0, b_end) fill grp[0 .. n_rel) after grouping (keys
  // above hhi are in no bin)
  const int n_rel = b_end < kPrefixBins ? static_cast<int>(hist[b_end]) : s_nbin;
  if (s_bmax <= kMaxBin) {
    // group the keys of bins before b_end; afterwards such a bin b spans
    // [end(b - 1), hist[b]) with end(-1) = 0
    for (int j = tid; j < c; j += 1024) {
      const uint64_t x = keys[j];
      const int b = bin(x);
      if (b < b_end) grp[atomicAdd(&hist[b], 1u)] = x;
    }
    __syncthreads();
    for (int p = tid; p < n_rel; p += 1024) {
      const uint64_t x = grp[p];
      const int b = bin(x);
      if (b >= b_end) continue;  // (every grouped key is in a bin before b_end)
      const int lo = b == 0 ? 0 : static_cast<int>(hist[b - 1]);
      const int hi = static_cast<int>(hist[b]);
      int rk = lo;
      for (int q = lo; q < hi; ++q) rk += grp[q] < x ? 1 : 0;
      if (rk < nw) {
        out[rk] = order_key_id(x);
        if (outs) outs[rk] = order_key_score(x);
      }
    }
  } else {
    int np = 1;
    while (np < c) np <<= 1;
    for (int j = c + tid; j < np; j += 1024) keys[j] = kOrderPad;
    __syncthreads();
    block_sort_u64(keys, np);
    for (int j = tid; j < nw; j += 1024) {
      out[j] = order_key_id(keys[j]);
      if (outs) outs[j] = order_key_score(keys[j]);
    }
  }
  __syncthreads();
}

}  // namespace aiidx
