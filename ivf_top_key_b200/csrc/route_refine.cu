// Per-query candidate fill, exact rescore and top-k (one fused kernel).
//
// AttentionIndex explainer (paper-daily.com), section "查询时怎么挑候选？":
// each query ranks the clusters by the indexer score of their
// representatives, fills a candidate budget C with the sink keys and the
// open (not yet clustered) window first and then with whole member lists in
// rank order, truncating the last list that does not fit; the candidates
// are rescored with the indexer score and the top k are kept.  The version
// paragraph of "索引怎么边算边建？" fixes which clusters and which open window
// a query at position t may use (passed in as a small version table).
//
// Persistent CTAs (two per SM) walk queries.  Per query:
//  1. candidate build: the route-score range and a size-weighted histogram
//     (two levels) find the budget threshold over the visible non-empty
//     clusters; the clusters at or above it are ranked by (score desc, id
//     asc) and their member runs are copied, after the sinks and the open
//     window, into the candidate list (shared memory or global scratch);
//  2. exact rescore, 128 candidates per tile: TMA tile::gather4 brings the
//     bf16 rows (for fp8 keys, the bf16 copy of the codes) into the
//     128-byte-swizzled UMMA layout, one tcgen05 UMMA (M = 128 candidates,
//     N = H heads, K = 128) per tile accumulates in TMEM, and four epilogue
//     warps apply ReLU, the head weights and the fp8 scale, keeping the
//     scores in TMEM (SIMT FMA path for fp32 keys);
//  3. top-k: a histogram over the score range locates the k-th score's bin,
//     whose items are sorted to read the exact threshold; ties at the
//     threshold go to the lower key id; ids are written in a fixed order,
//     padded with -1.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kSortCap = 2048;  // ranked clusters per query (size-capped at ~W/m keys each)
constexpr int kTile = 128;
constexpr int kStages = 3;
constexpr int kTcThreads = 288;   // 9 warps; each tensor-core kernel lists its warp roles
constexpr int kSimtThreads = 256;

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// The threads that run the candidate build: the whole block, or a
// warp-aligned group of 128 threads synchronised by a named barrier.
struct BlockGrp {
  __device__ int tid() const { return threadIdx.x; }
  __device__ int size() const { return blockDim.x; }
  __device__ void sync() const { __syncthreads(); }
};
struct SubGrp128 {
  int first, bar;  // first thread of the group, named barrier id
  __device__ int tid() const { return threadIdx.x - first; }
  __device__ int size() const { return 128; }
  __device__ void sync() const { named_bar(bar, 128); }
};

template <class G>
__device__ __forceinline__ void bitonic_sort_u64(uint64_t* buf, int n, const G& g) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = g.tid(); i < n; i += g.size()) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t x = buf[i], y = buf[ixj];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            buf[i] = y;
            buf[ixj] = x;
          }
        }
      }
      g.sync();
    }
  }
}

// Work item q of this CTA in the pipelined kernel: query qi, and (split > 1)
// the part sp of its list that this item rescores.  Items run query-major:
// the split parts of a query go to neighbouring CTAs.
struct RefineItem {
  int qi, sp;
};
__device__ __forceinline__ int refine_split(const RefineArgs& a) { return a.split > 1 ? a.split : 1; }
__device__ __forceinline__ RefineItem refine_item(const RefineArgs& a, int q) {
  const int S = refine_split(a);
  const int v = static_cast<int>(blockIdx.x) + q * static_cast<int>(gridDim.x);
  return RefineItem{v / S, v % S};
}

// The share of a candidate list of n slots that one item rescores: the
// whole list, or a contiguous range of its 128-slot tiles when the list is
// divided among shards (ranks; n_shards > 1) and, inside this launch, among
// the split parts of the query (part sp of split).  The rescore and the
// top-k run on the list shifted to that range.
__device__ __forceinline__ void shard_span(const RefineArgs& a, int sp, int n, int* off, int* n_loc) {
  const int S = refine_split(a);
  const int parts = (a.n_shards > 1 ? a.n_shards : 1) * S;
  if (parts <= 1) {
    *off = 0;
    *n_loc = n;
    return;
  }
  const int part = (a.n_shards > 1 ? a.shard : 0) * S + sp;
  const int tiles = (n + kTile - 1) / kTile;
  const int t0 = static_cast<int>(static_cast<int64_t>(part) * tiles / parts);
  const int t1 = static_cast<int>(static_cast<int64_t>(part + 1) * tiles / parts);
  const int e = n < t1 * kTile ? n : t1 * kTile;
  *off = t0 * kTile;
  *n_loc = e > t0 * kTile ? e - t0 * kTile : 0;
}

__device__ __forceinline__ void version_of(const VersionTable& vt, int64_t t, int* nC,
                                           int64_t* n_v) {
  int idx = 0;
  for (int i = 1; i < vt.n; ++i)
    if (vt.seg[i].first_pos <= t) idx = i;
  *nC = vt.seg[idx].nC;
  *n_v = vt.seg[idx].n_v;
}

// Phase 1: candidate list of query qi (position t).  Returns its length.
//
// Sinks and the open window come first.  Then clusters in rank order
// (score desc, id asc) until C slots are filled, the last one truncated.
// Only the clusters that can reach the budget are ranked: a weighted
// 2048-bin histogram of the cluster scores over [min, max] (weights =
// cluster sizes) finds the bin where the size-weighted count from the top
// crosses the remaining budget; clusters in that bin or above are sorted
// exactly and the fill stops at C.
constexpr int kNB1 = 2048;
constexpr int kLightBin = 512;  // members in a boundary bin taken whole (no level-2 pass)
struct P1Smem {
  union {                    // the histogram is dead before the offsets are written
    int32_t coff[kSortCap];  // member offset of each ranked cluster
    uint32_t hist[kNB1];
  };
  float fred[32];
  unsigned long long wred[16];
  int scal[4];
};

// Warp 0 scans the weighted histogram ps.hist from the top for the bin
// where the weight reaches `need`: its index and the weight above it.
// All threads of the group call it (it ends with a barrier).
template <class G>
__device__ __forceinline__ void p1_find_bin(P1Smem& ps, int need, int* bstar, int* above, const G& g) {
  const int lane = threadIdx.x & 31;
  if (g.tid() < 32) {
    uint32_t lsum = 0;
    for (int b = 0; b < 64; ++b) lsum += ps.hist[lane * 64 + b];
    uint32_t incl = lsum;  // sum over lanes >= this one
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += v;
    }
    uint32_t cum = incl - lsum;
    int found = -1;
    uint32_t ab = 0;
    for (int b = lane * 64 + 63; b >= lane * 64; --b) {
      const uint32_t h = ps.hist[b];
      if (found < 0 && cum < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= cum + h) {
        found = b;
        ab = cum;
      }
      cum += h;
    }
    const unsigned who = __ballot_sync(0xffffffffu, found >= 0);
    const int src = who ? __ffs(who) - 1 : 0;
    const int fb = __shfl_sync(0xffffffffu, found, src);
    const uint32_t fa = __shfl_sync(0xffffffffu, ab, src);
    if (lane == 0) {
      ps.scal[0] = who ? fb : 0;
      ps.scal[2] = static_cast<int>(fa);
    }
  }
  g.sync();
  *bstar = ps.scal[0];
  *above = ps.scal[2];
  g.sync();
}

// f(c, score, size) for every cluster c < nC: blocks of four clusters with
// 16-byte loads of their offsets and route scores (both arrays 16-byte
// aligned), two blocks in flight per thread, then the ragged tail.
template <class F>
__device__ __forceinline__ void for_clusters(const int32_t* off, const float* rs, int nC, int tid, int nthr,
                                             F f) {
  const int nb = nC >> 2;
  for (int i0 = tid; i0 < nb; i0 += 2 * nthr) {
    int4 o[2];
    int o4[2];
    float4 v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * nthr;
      o[u] = make_int4(0, 0, 0, 0);
      o4[u] = 0;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < nb) {
        o[u] = __ldg(reinterpret_cast<const int4*>(off) + i);
        o4[u] = __ldg(off + 4 * i + 4);
        v[u] = __ldg(reinterpret_cast<const float4*>(rs) + i);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * nthr;
      if (i < nb) {
        f(4 * i, v[u].x, o[u].y - o[u].x);
        f(4 * i + 1, v[u].y, o[u].z - o[u].y);
        f(4 * i + 2, v[u].z, o[u].w - o[u].z);
        f(4 * i + 3, v[u].w, o4[u] - o[u].w);
      }
    }
  }
  for (int c = 4 * nb + tid; c < nC; c += nthr) f(c, __ldg(rs + c), __ldg(off + c + 1) - __ldg(off + c));
}

// The list is written to shared memory (kGlobal = false) or to the CTA's
// global scratch row (kGlobal = true).
template <bool kGlobal, class G>
__device__ int build_candidates(const RefineArgs& a, int qi, int64_t t, int nC, int64_t n_v,
                                int32_t* cand, uint64_t* sortbuf, int32_t* pref, const G& g) {
  const int C = a.C;
  const int tid = g.tid(), lane = tid & 31, warp = tid >> 5;
  const int nthr = g.size();
  const int nwarps = (nthr + 31) >> 5;
  const int n_s = static_cast<int>(min64(a.n_sinks, t + 1));
  const int64_t open_lo = max64(n_v, a.n_sinks);
  const int64_t n_open64 = open_lo <= t ? t + 1 - open_lo : 0;
  const int fixed = static_cast<int>(min64(C, n_s + n_open64));
  for (int i = tid; i < fixed; i += nthr)
    cand[i] = i < n_s ? i : static_cast<int32_t>(open_lo + (i - n_s));
  const int rem = C - fixed;
  if (rem <= 0 || nC == 0) {
    g.sync();
    return fixed;
  }
  // scratch after the sort buffer and prefix array
  P1Smem& ps = *reinterpret_cast<P1Smem*>(
      (reinterpret_cast<uintptr_t>(pref + kSortCap + 1) + 15) & ~uintptr_t(15));
  const float* rs = a.route + static_cast<int64_t>(qi) * a.ld_route;
  const int32_t* off = a.offsets;
  float vmin = INFINITY, vmax = -INFINITY;
  unsigned long long wsum = 0;
  if (a.route_kmin) {
    // score range from the route GEMM (over all clusters of the buffer: a
    // superset of this query's visible ones, which only widens the bins)
    // and the total size of the visible clusters (telescoping offsets)
    const uint4 mn4 = __ldg(reinterpret_cast<const uint4*>(a.route_kmin) + qi);
    const uint4 mx4 = __ldg(reinterpret_cast<const uint4*>(a.route_kmax) + qi);
    vmin = key2f(min(min(mn4.x, mn4.y), min(mn4.z, mn4.w)));
    vmax = key2f(max(max(mx4.x, mx4.y), max(mx4.z, mx4.w)));
    wsum = static_cast<unsigned long long>(__ldg(off + nC) - __ldg(off));
    for (int i = tid; i < kNB1; i += nthr) ps.hist[i] = 0;
    g.sync();
  } else {
    // pass A: score range and total size of the non-empty clusters
#pragma unroll 4
    for (int c = tid; c < nC; c += nthr) {
      const int sz = __ldg(off + c + 1) - __ldg(off + c);
      const float v = __ldg(rs + c);
      if (sz > 0) {
        vmin = fminf(vmin, v);
        vmax = fmaxf(vmax, v);
        wsum += static_cast<unsigned long long>(sz);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
      vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
    }
    if (lane == 0) {
      ps.fred[warp] = vmin;
      ps.fred[16 + warp] = vmax;
      ps.wred[warp] = wsum;
    }
    for (int i = tid; i < kNB1; i += nthr) ps.hist[i] = 0;
    g.sync();
    vmin = INFINITY;
    vmax = -INFINITY;
    wsum = 0;
    for (int w = 0; w < nwarps; ++w) {
      vmin = fminf(vmin, ps.fred[w]);
      vmax = fmaxf(vmax, ps.fred[16 + w]);
      wsum += ps.wred[w];
    }
  }
  const bool take_all = wsum <= static_cast<unsigned long long>(rem);
  const float scale = vmax > vmin ? static_cast<float>(kNB1) / (vmax - vmin) : 0.f;
  // bin positions use explicitly rounded operations (no FMA contraction), so
  // every pass computes the same bin for the same score
  auto pos1 = [=](float v) -> float { return __fmul_rn(__fsub_rn(v, vmin), scale); };
  auto binof = [=](float v) -> int {
    const int b = static_cast<int>(pos1(v));
    return b < kNB1 - 1 ? b : kNB1 - 1;
  };
  int bstar = 0, bstar2 = 0;
  auto bin2 = [=](float v, int b1) -> int {
    const int b = static_cast<int>(__fmul_rn(__fsub_rn(pos1(v), static_cast<float>(b1)),
                                             static_cast<float>(kNB1)));
    return b < 0 ? 0 : (b < kNB1 - 1 ? b : kNB1 - 1);
  };
  if (!take_all) {
    // pass B: size-weighted histogram; the bin where the weight from the top
    // reaches the remaining budget
    for_clusters(off, rs, nC, tid, nthr, [&](int, float v, int sz) {
      if (sz > 0) atomicAdd(&ps.hist[binof(v)], static_cast<uint32_t>(sz));
    });
    g.sync();
    int above1 = 0;
    p1_find_bin(ps, rem, &bstar, &above1, g);
    // pass B2: the boundary bin split into kNB1 sub-bins (a long score tail
    // leaves most clusters in few level-1 bins).  A light boundary bin (few
    // members, hence few clusters) is instead taken whole: the exact sort
    // below ranks its clusters.
    const bool light = ps.hist[bstar] <= static_cast<uint32_t>(kLightBin);
    g.sync();
    if (!light) {
    for (int i = tid; i < kNB1; i += nthr) ps.hist[i] = 0;
    g.sync();
    for_clusters(off, rs, nC, tid, nthr, [&](int, float v, int sz) {
      if (sz > 0 && binof(v) == bstar) atomicAdd(&ps.hist[bin2(v, bstar)], static_cast<uint32_t>(sz));
    });
    g.sync();
    int above2 = 0;
    p1_find_bin(ps, rem - above1, &bstar2, &above2, g);
    }  // !light (else bstar2 = 0: every cluster of the boundary bin)
  }
  auto selected = [=](float v) -> bool {
    if (take_all) return true;
    const int b = binof(v);
    if (b != bstar) return b > bstar;
    return bin2(v, bstar) >= bstar2;
  };
  // pass C: clusters at or above the boundary bin (any order: sorted next)
  if (tid == 0) ps.scal[1] = 0;
  g.sync();
  for_clusters(off, rs, nC, tid, nthr, [&](int c, float v, int sz) {
    if (sz > 0 && selected(v)) {
      const int pos = atomicAdd(&ps.scal[1], 1);
      if (pos < kSortCap) sortbuf[pos] = (static_cast<uint64_t>(~f2key(v)) << 32) | static_cast<uint32_t>(c);
    }
  });
  g.sync();
  int nsel = ps.scal[1];
  if (nsel > kSortCap) {
    if (tid == 0) atomicOr(a.err, DEV_ERR_CAPACITY);
    nsel = kSortCap;
  }
  // rank order (score descending, then cluster id): small selections by
  // counting (keys are distinct, so ranks are a permutation), larger ones
  // by a bitonic sort in place
  const uint64_t* sorted = sortbuf;
  if (nsel <= kSortCap / 4) {
    uint64_t* dst = sortbuf + kSortCap / 2;
    for (int i = tid; i < nsel; i += nthr) {
      const uint64_t x = sortbuf[i];
      int r = 0;
      for (int j = 0; j < nsel; ++j) r += sortbuf[j] < x ? 1 : 0;
      dst[r] = x;
    }
    g.sync();
    sorted = dst;
  } else {
    int np = 1;
    while (np < nsel) np <<= 1;
    for (int i = nsel + tid; i < np; i += nthr) sortbuf[i] = ~0ull;
    g.sync();
    bitonic_sort_u64(sortbuf, np, g);
  }
  // member offsets and sizes of the ranked clusters (parallel loads), then
  // the exclusive prefix of sizes in rank order
  int32_t* coff = ps.coff;
  for (int r = tid; r < nsel; r += nthr) {
    const int c = static_cast<int>(sorted[r] & 0xffffffffu);
    const int o0 = off[c];
    coff[r] = o0;
    pref[r] = off[c + 1] - o0;
  }
  g.sync();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < nsel; base += 32) {
      const int r = base + lane;
      const int v = r < nsel ? pref[r] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (r < nsel) pref[r] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) pref[nsel] = carry;
  }
  g.sync();
  const int len = static_cast<int>(min64(C, static_cast<int64_t>(fixed) + pref[nsel]));
  if (kGlobal) {
    // fill of a list in global memory: one warp per ranked cluster, four
    // clusters per warp at a time (their run bounds are independent shared
    // loads, their first 128 members sixteen coalesced loads per lane in
    // flight), cut at C
    for (int r0 = warp; r0 < nsel; r0 += 4 * nwarps) {
      int d0[4], sz[4], src[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = r0 + u * nwarps;
        d0[u] = 0;
        sz[u] = 0;
        src[u] = 0;
        if (r < nsel) {
          d0[u] = fixed + pref[r];
          sz[u] = min(pref[r + 1] - pref[r], len - d0[u]);
          src[u] = coff[r];
        }
      }
      // the first 128 members of the four clusters: 16 loads in flight per
      // lane (clusters hold ~W/m = 128 keys after a seal)
      int32_t v[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int l = lane + 32 * h;
          v[u][h] = l < sz[u] ? __ldg(a.members + src[u] + l) : 0;
        }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int l = lane + 32 * h;
          if (l < sz[u]) cand[d0[u] + l] = v[u][h];
        }
      // larger (refit) clusters: the rest, four loads in flight per lane
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        for (int l0 = 128; l0 < sz[u]; l0 += 128) {
          int32_t w4[4];
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int l = l0 + lane + 32 * h;
            w4[h] = l < sz[u] ? __ldg(a.members + src[u] + l) : 0;
          }
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const int l = l0 + lane + 32 * h;
            if (l < sz[u]) cand[d0[u] + l] = w4[h];
          }
        }
      }
    }
  } else {
    // fill of a list in shared memory: one warp per ranked cluster copies
    // its member run with 4-byte asynchronous copies (all in flight at
    // once), cut at C
    for (int r = warp; r < nsel; r += nwarps) {
      const int d0 = fixed + pref[r];
      if (d0 >= len) continue;
      const int sz = min(pref[r + 1] - pref[r], len - d0);
      const int32_t* src = a.members + coff[r];
      for (int l = lane; l < sz; l += 32) cp_async4(cand + d0 + l, src + l);
    }
    cp_async_wait_all();
  }
  g.sync();
  return len;
}

// Phase 3: top-k of score[0..n) with ids cand[]; ties go to the lower id.
// sbuf: shared memory for the output sort (next power of two >= k keys).
__device__ __forceinline__ void topk_emit(const RefineArgs& a, int qi, const float* score,
                                          const int32_t* cand, int n, BlockScratch& bs, uint64_t* sbuf) {
  int32_t* out = a.out + static_cast<int64_t>(qi) * a.k;
  float* outs = a.out_scores ? a.out_scores + static_cast<int64_t>(qi) * a.k : nullptr;
  topk_select_emit(
      n, [&](int i) -> float { return score[i]; }, [&](int i) -> int32_t { return cand[i]; }, a.k,
      out, outs, bs, sbuf);
}

struct Layout {
  float* score;
  int32_t* cand;
  uint8_t* region;   // phase-1 sort scratch; phase-2 stages + q tile
  uint64_t* sortbuf;
  int32_t* pref;
  float* wsh;        // [H]
  float* qf;         // SIMT: [H * d] fp32 query
  uint64_t* bars;    // full[kStages], empty[kStages], tfull[2], tempty[2]
  uint32_t* tmem;
  int* abort;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline size_t region_bytes(int H, int d, bool tc) {
  size_t p1 = static_cast<size_t>(kSortCap) * 8 + (kSortCap + 1) * 4 + sizeof(P1Smem) + 16;
  size_t p2 = tc ? static_cast<size_t>(kStages) * kTile * 256 + static_cast<size_t>(H) * 256
                 : static_cast<size_t>(H) * d * 4;
  return align_up(p1 > p2 ? p1 : p2, 1024);
}

__device__ inline Layout carve(uint8_t* raw, int C, int H, int d, bool tc) {
  Layout L;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  L.region = p;
  p += region_bytes(H, d, tc);
  L.sortbuf = reinterpret_cast<uint64_t*>(L.region);
  L.pref = reinterpret_cast<int32_t*>(L.region + static_cast<size_t>(kSortCap) * 8);
  L.qf = reinterpret_cast<float*>(L.region);
  L.score = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(C) * 4, 16);
  L.cand = reinterpret_cast<int32_t*>(p);
  p += align_up(static_cast<size_t>(C) * 4, 16);
  L.wsh = reinterpret_cast<float*>(p);
  p += align_up(static_cast<size_t>(H) * 4, 16);
  L.bars = reinterpret_cast<uint64_t*>(p);
  p += (2 * kStages + 4) * 8;
  L.tmem = reinterpret_cast<uint32_t*>(p);
  L.abort = reinterpret_cast<int*>(p + 4);
  return L;
}

// ------------------------------------------------------------- SIMT kernel
__global__ void __launch_bounds__(kSimtThreads) k_refine_simt(RefineArgs a, VersionTable vt) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ BlockScratch bs;
  Layout L = carve(smem_raw, a.C, a.H, a.d, false);
  const int H = a.H, d = a.d;
  for (int qi = blockIdx.x; qi < a.T; qi += gridDim.x) {
    const int64_t t = a.pos0 + qi;
    int nC;
    int64_t n_v;
    version_of(vt, t, &nC, &n_v);
    const int n = build_candidates<false>(a, qi, t, nC, n_v, L.cand, L.sortbuf, L.pref, BlockGrp{});
    if (a.cand_out) {
      for (int i = threadIdx.x; i < a.C; i += blockDim.x)
        a.cand_out[static_cast<int64_t>(qi) * a.C + i] = i < n ? L.cand[i] : -1;
    }
    // query row to shared fp32
    for (int i = threadIdx.x; i < H * d; i += blockDim.x) {
      const int64_t o = static_cast<int64_t>(qi) * H * d + i;
      L.qf[i] = a.q_is_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(a.q)[o])
                            : reinterpret_cast<const float*>(a.q)[o];
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) L.wsh[h] = a.w[static_cast<int64_t>(qi) * H + h];
    __syncthreads();
    for (int slot = threadIdx.x; slot < n; slot += blockDim.x) {
      const int32_t s = L.cand[slot];
      float sc = -INFINITY;
      if (s >= 0 && s <= t) {
        sc = 0.f;
        for (int h = 0; h < H; ++h) {
          float dot = 0.f;
          for (int i = 0; i < d; ++i) dot = fmaf(L.qf[h * d + i], key_elem(a.keys, a.key_dtype, s, d, i), dot);
          sc = fmaf(L.wsh[h], fmaxf(dot, 0.f), sc);
        }
        if (a.key_scale) sc *= a.key_scale[s];
      } else {
        atomicOr(a.err, DEV_ERR_RANGE);
      }
      L.score[slot] = sc;
    }
    __syncthreads();
    // the query row in the region is dead now: it holds the output sort
    topk_emit(a, qi, L.score, L.cand, n, bs, L.sortbuf);
    __syncthreads();
  }
}

// ---------------------------------------------------------- tcgen05 kernel

// ------------------------------------------------- top-k by the epilogue warps
// The 128 epilogue threads hold the candidate scores in TMEM: thread
// (quarter q, lane l) owns row r = 32 q + l, i.e. slots j * 128 + r, in
// columns scol + j.  Selection: a 2048-bin linear histogram over
// [min, max] locates the bin of the k-th score; the bin's items are sorted
// to get the exact threshold; rare overflow and tie cases use a radix
// select over the same items.  Ties at the threshold go to the lower key id.
constexpr int kNB = 2048;     // histogram bins
constexpr int kCapB = 2048;   // items of the threshold bin sorted in smem (>= k/2)

struct P3Smem {
  uint32_t hist[kNB];
  uint64_t buf[kCapB];
  float fred[8];
  int ired[8];
  int scal[8];
  int cnt32;   // items of the threshold bin appended so far
};

struct P3Ctx {
  uint32_t tcol;   // TMEM address of this thread's first score column
  int row, ntiles, n;
  const int32_t* cand;
};

template <class F>
__device__ __forceinline__ void p3_for_each(const P3Ctx& c, F f) {
  for (int c0 = 0; c0 < c.ntiles; c0 += 16) {
    float v[16];
    tmem_ld16(c.tcol + c0, v);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = c0 + u;
      const int slot = j * 128 + c.row;
      if (j < c.ntiles && slot < c.n) f(v[u], slot);
    }
  }
}

// Every item of the thread's columns (16 at a time), with its validity as
// an int: bodies fold it into branch-free arithmetic (a data-dependent
// branch per item costs far more than the arithmetic).
template <class F>
__device__ __forceinline__ void p3_for_each_all(const P3Ctx& c, F f) {
  for (int c0 = 0; c0 < c.ntiles; c0 += 16) {
    float v[16];
    tmem_ld16(c.tcol + c0, v);
    tmem_ld_wait();
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = c0 + u;
      const int slot = j * 128 + c.row;
      f(v[u], slot, static_cast<int>(j < c.ntiles) & static_cast<int>(slot < c.n));
    }
  }
}

// Exclusive prefix over the 128 epilogue threads (et = 0..127).
__device__ __forceinline__ int p3_scan(int v, int et, int* total, P3Smem& ps) {
  const int lane = et & 31, w = et >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ps.ired[w] = incl;
  named_bar(1, 128);
  int before = 0, tot = 0;
  for (int i = 0; i < 4; ++i) {
    if (i < w) before += ps.ired[i];
    tot += ps.ired[i];
  }
  named_bar(1, 128);
  *total = tot;
  return before + incl - v;
}

// Radix select over the items passing pred: the value of key(v, slot) of
// the need-th largest item, and how many items lie strictly above it.
template <class Pred, class Key>
__device__ __forceinline__ uint32_t p3_radix(const P3Ctx& c, int et, Pred pred, Key key, int need, int* above,
                             int* eq, P3Smem& ps) {
  uint32_t prefix = 0, mask = 0;
  int needr = need, ab = 0, last = 0;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = et; i < 256; i += 128) ps.hist[i] = 0;
    named_bar(1, 128);
    p3_for_each(c, [&, pred, key](float v, int slot) {
      if (!pred(v, slot)) return;
      const uint32_t kk = key(v, slot);
      if ((kk & mask) == prefix) atomicAdd(&ps.hist[(kk >> shift) & 255u], 1u);
    });
    named_bar(1, 128);
    if (et == 0) {
      int cum = 0, dg = 0;
      for (int d = 255; d >= 0; --d) {
        const int h = static_cast<int>(ps.hist[d]);
        if (cum < needr && needr <= cum + h) {
          dg = d;
          ps.scal[5] = h;
          break;
        }
        cum += h;
      }
      ps.scal[3] = dg;
      ps.scal[4] = cum;
    }
    named_bar(1, 128);
    const uint32_t dg = static_cast<uint32_t>(ps.scal[3]);
    needr -= ps.scal[4];
    ab += ps.scal[4];
    last = ps.scal[5];
    prefix |= dg << shift;
    mask |= 255u << shift;
    named_bar(1, 128);
  }
  *above = ab;
  *eq = last;
  return prefix;
}

// The bin of ps.hist (kNB bins, scanned from the top) holding the k-th
// item: its index, the count above it, and its own count.  All 128
// epilogue threads call it; thread et owns bins [16 et, 16 et + 16).
__device__ __forceinline__ void p3_find_bin(P3Smem& ps, int et, int k, int* bstar, int* above, int* nb) {
  int tsum = 0;
  for (int b = 0; b < 16; ++b) tsum += static_cast<int>(ps.hist[16 * et + b]);
  int tot;
  const int before = p3_scan(tsum, et, &tot, ps);
  int cum = tot - before - tsum;
  for (int b = 16 * et + 15; b >= 16 * et; --b) {
    const int h = static_cast<int>(ps.hist[b]);
    if (cum < k && k <= cum + h) {
      ps.scal[0] = b;
      ps.scal[1] = cum;
      ps.scal[2] = h;
    }
    cum += h;
  }
  named_bar(1, 128);
  *bstar = ps.scal[0];
  *above = ps.scal[1];
  *nb = ps.scal[2];
  named_bar(1, 128);
}

__device__ void p3_topk(const RefineArgs& a, int orow, const P3Ctx& c, int et, P3Smem& ps) {
  const int k = a.k;
  int32_t* out = a.out + static_cast<int64_t>(orow) * k;
  float* outs = a.out_scores ? a.out_scores + static_cast<int64_t>(orow) * k : nullptr;
  // range of the valid scores
  float vmin = INFINITY, vmax = -INFINITY;
  p3_for_each(c, [&](float v, int) {
    vmin = fminf(vmin, v);
    vmax = fmaxf(vmax, v);
  });
  for (int o = 16; o > 0; o >>= 1) {
    vmin = fminf(vmin, __shfl_xor_sync(0xffffffffu, vmin, o));
    vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  }
  if ((et & 31) == 0) {
    ps.fred[et >> 5] = vmin;
    ps.fred[4 + (et >> 5)] = vmax;
  }
  named_bar(1, 128);
  vmin = fminf(fminf(ps.fred[0], ps.fred[1]), fminf(ps.fred[2], ps.fred[3]));
  vmax = fmaxf(fmaxf(ps.fred[4], ps.fred[5]), fmaxf(ps.fred[6], ps.fred[7]));
  named_bar(1, 128);
  const bool take_all = c.n <= k;
  float theta = -INFINITY;
  int theta_id = 0x7fffffff;
  bool ties_all = true;
  if (!take_all) {
    const float scale = vmax > vmin ? static_cast<float>(kNB) / (vmax - vmin) : 0.f;
    // explicitly rounded (never contracted): the same score always lands in
    // the same bin in every pass
    auto pos1 = [=](float v) -> float { return __fmul_rn(__fsub_rn(v, vmin), scale); };
    auto binof = [=](float v) -> int {
      const int b = static_cast<int>(pos1(v));
      return b < 0 ? 0 : (b < kNB - 1 ? b : kNB - 1);
    };
    // level 1 over [vmin, vmax]; level 2 splits the level-1 bin that holds
    // the k-th score into kNB sub-bins (a long score tail leaves the bulk
    // in few level-1 bins)
    for (int i = et; i < kNB; i += 128) ps.hist[i] = 0;
    if (et == 0) ps.cnt32 = 0;
    named_bar(1, 128);
    // (an add of 0 for slots past the list keeps the body branch-free)
    p3_for_each_all(c, [&ps, binof](float v, int, int ok) {
      atomicAdd(&ps.hist[binof(v)], static_cast<uint32_t>(ok));
    });
    named_bar(1, 128);
    int above_b = 0, bstar = 0, nb = 0;
    p3_find_bin(ps, et, k, &bstar, &above_b, &nb);
    const float b1f = static_cast<float>(bstar);
    auto bin2 = [=](float v) -> int {
      const int b = static_cast<int>(__fmul_rn(__fsub_rn(pos1(v), b1f), static_cast<float>(kNB)));
      return b < 0 ? 0 : (b < kNB - 1 ? b : kNB - 1);
    };
    // The items of the threshold bin (bin bstar, or its sub-bin bstar2 when
    // the bin is too full) are gathered and sorted; the k-th score is
    // read off the sorted list.
    int bsel2 = -1, nsel = nb, above_in = 0, eq = 0;
    if (nb > kCapB) {
      // level 2: the bin split into kNB sub-bins
      for (int i = et; i < kNB; i += 128) ps.hist[i] = 0;
      named_bar(1, 128);
      // few items per warp fall in the bin: a warp-uniform test skips the rest
      p3_for_each_all(c, [&ps, binof, bin2, bstar](float v, int, int ok) {
        const int f = ok & static_cast<int>(binof(v) == bstar);
        if (__any_sync(0xffffffffu, f)) {
          if (f) atomicAdd(&ps.hist[bin2(v)], 1u);
        }
      });
      named_bar(1, 128);
      int above2 = 0;
      p3_find_bin(ps, et, k - above_b, &bsel2, &above2, &nsel);
      above_b += above2;
    }
    auto in_b = [=](float v) -> bool { return binof(v) == bstar && (bsel2 < 0 || bin2(v) == bsel2); };
    const int need = k - above_b;
    uint32_t tkey;
    if (nsel <= kCapB) {
      // append of the items of the threshold (sub-)bin: flags for 16 items
      // at a time without branches, then a warp-uniform test; the rare hits
      // are appended warp-aggregated
      for (int c0 = 0; c0 < c.ntiles; c0 += 16) {
        float v[16];
        tmem_ld16(c.tcol + c0, v);
        tmem_ld_wait();
        uint32_t m = 0;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int j = c0 + u;
          const int slot = j * 128 + c.row;
          const int f = static_cast<int>(j < c.ntiles) & static_cast<int>(slot < c.n) &
                        static_cast<int>(binof(v[u]) == bstar) &
                        (static_cast<int>(bsel2 < 0) | static_cast<int>(bin2(v[u]) == bsel2));
          m |= static_cast<uint32_t>(f) << u;
        }
        if (__any_sync(0xffffffffu, m != 0u)) {
          // one scan of the per-thread hit counts and one counter update per
          // warp; each thread then writes its hits with predicated stores
          const int lane = threadIdx.x & 31;
          const int h = __popc(m);
          int incl = h;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t2 = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t2;
          }
          int base = 0;
          if (lane == 31) base = atomicAdd(&ps.cnt32, incl);
          int pos = __shfl_sync(0xffffffffu, base, 31) + incl - h;
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const bool f = (m >> u) & 1u;
            if (f)
              ps.buf[pos] = (static_cast<uint64_t>(~f2key(v[u])) << 32) |
                            static_cast<uint32_t>((c0 + u) * 128 + c.row);
            pos += f ? 1 : 0;
          }
        }
      }
      named_bar(1, 128);
      int np = 1;
      while (np < nsel) np <<= 1;
      for (int i = nsel + et; i < np; i += 128) ps.buf[i] = ~0ull;
      named_bar(1, 128);
      for (int kk = 2; kk <= np; kk <<= 1) {
        for (int j = kk >> 1; j > 0; j >>= 1) {
          for (int i = et; i < np; i += 128) {
            const int ixj = i ^ j;
            if (ixj > i) {
              const uint64_t x = ps.buf[i], y = ps.buf[ixj];
              if ((x > y) == ((i & kk) == 0)) {
                ps.buf[i] = y;
                ps.buf[ixj] = x;
              }
            }
          }
          named_bar(1, 128);
        }
      }
      tkey = ~static_cast<uint32_t>(ps.buf[need - 1] >> 32);
      if (et == 0) {
        int i0 = need - 1;
        while (i0 > 0 && ~static_cast<uint32_t>(ps.buf[i0 - 1] >> 32) == tkey) --i0;
        int i1 = need - 1;
        while (i1 + 1 < nsel && ~static_cast<uint32_t>(ps.buf[i1 + 1] >> 32) == tkey) ++i1;
        ps.scal[6] = i0;
        ps.scal[7] = i1 - i0 + 1;
      }
      named_bar(1, 128);
      above_in = ps.scal[6];
      eq = ps.scal[7];
    } else {
      tkey = p3_radix(
          c, et, [=](float v, int) { return in_b(v); }, [](float v, int) { return f2key(v); }, need,
          &above_in, &eq, ps);
    }
    theta = key2f(tkey);
    const int need_eq = k - above_b - above_in;  // above_b spans both levels
    if (eq > need_eq) {
      ties_all = false;
      int ab2 = 0, eq2 = 0;
      const uint32_t idk = p3_radix(
          c, et, [=](float v, int) { return v == theta; },
          [cd = c.cand](float, int slot) { return ~static_cast<uint32_t>(cd[slot]); }, need_eq, &ab2, &eq2,
          ps);
      theta_id = static_cast<int>(~idk);
    }
  }
  // emission: ids (and scores) staged in shared memory in thread-major
  // order, then written out coalesced; a follow-up kernel (order_rows.cu)
  // puts every row in the output order.  Selection is v >= theta
  // (everything when all items are kept), except when only some of the
  // items tied at theta are kept: then v > theta or (v == theta and id <=
  // theta_id).  Bodies are branch-free; unselected items write to a
  // per-thread dummy slot.
  const bool partial_ties = !take_all && !ties_all;
  const float th = take_all ? -INFINITY : theta;
  const int thid = theta_id;
  const int32_t* cd = c.cand;
  const int nlast = c.n - 1;  // slots past the list read entry 0 instead (their result is unused)
  int mine = 0;
  if (!partial_ties) {
    p3_for_each_all(c, [&mine, th](float v, int, int ok) { mine += ok & static_cast<int>(v >= th); });
  } else {
    // rare: the id decides among the items tied at theta
    p3_for_each_all(c, [&mine, th, thid, cd, nlast](float v, int slot, int ok) {
      const int sl = slot <= nlast ? slot : 0;
      mine += ok & (static_cast<int>(v > th) | (v == th ? static_cast<int>(cd[sl] <= thid) : 0));
    });
  }
  int total;
  int pos = p3_scan(mine, et, &total, ps);
  int32_t* sid = reinterpret_cast<int32_t*>(ps.buf);          // [k] slots
  float* ssc = reinterpret_cast<float*>(ps.buf) + kCapB;       // [k] scores
  int32_t* dump_id = reinterpret_cast<int32_t*>(ps.hist) + et;
  float* dump_sc = reinterpret_cast<float*>(ps.hist) + 128 + et;
  auto stage = [&pos, sid, ssc, dump_id, dump_sc, k](float v, int slot, int f) {
    const bool w = (f & static_cast<int>(pos < k)) != 0;
    int32_t* pi = w ? sid + pos : dump_id;
    float* pv = w ? ssc + pos : dump_sc;
    *pi = slot;
    *pv = v;
    pos += f;
  };
  if (!partial_ties) {
    p3_for_each_all(c, [stage, th](float v, int slot, int ok) mutable {
      stage(v, slot, ok & static_cast<int>(v >= th));
    });
  } else {
    p3_for_each_all(c, [stage, th, thid, cd, nlast](float v, int slot, int ok) mutable {
      const int sl = slot <= nlast ? slot : 0;
      stage(v, slot, ok & (static_cast<int>(v > th) | (v == th ? static_cast<int>(cd[sl] <= thid) : 0)));
    });
  }
  named_bar(1, 128);
  const int nw = min(total, k);
  // the ids of a thread's outputs are all loaded before any is stored (the
  // stores could alias the list, so the compiler would not reorder them)
  for (int j0 = et; j0 < k; j0 += 8 * 128) {
    int32_t id[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 128;
      id[u] = j < nw ? cd[sid[j]] : -1;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * 128;
      if (j < k) {
        out[j] = id[u];
        if (outs) outs[j] = j < nw ? ssc[j] : -INFINITY;
      }
    }
  }
  named_bar(1, 128);
}

// Indexer score of one candidate row from its H head dot products in TMEM
// (columns acc .. acc + H - 1 of this thread's lane): sum_h w_h ReLU(dot_h).
// Four interleaved partial sums (head h goes to sum h mod 4, combined as
// (s0 + s1) + (s2 + s3)) keep the dependent chain short; every tensor-core
// kernel uses this same order, so their scores agree bit for bit.  The
// weights are read four at a time from shared memory (16-byte aligned).
template <int H>
__device__ __forceinline__ float head_sum(uint32_t acc, const float* wsh) {
  float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int c = 0; c < H / 32; ++c) {
    float v[32];
    tmem_ld32(acc + c * 32, v);
    tmem_ld_wait();
#pragma unroll
    for (int h4 = 0; h4 < 8; ++h4) {
      const float4 w4 = reinterpret_cast<const float4*>(wsh)[c * 8 + h4];
      s[0] = fmaf(w4.x, fmaxf(v[4 * h4 + 0], 0.f), s[0]);
      s[1] = fmaf(w4.y, fmaxf(v[4 * h4 + 1], 0.f), s[1]);
      s[2] = fmaf(w4.z, fmaxf(v[4 * h4 + 2], 0.f), s[2]);
      s[3] = fmaf(w4.w, fmaxf(v[4 * h4 + 3], 0.f), s[3]);
    }
  }
  return (s[0] + s[1]) + (s[2] + s[3]);
}

// Layout of the tensor-core kernel (one region reused by the three phases).
constexpr int kStages2 = 2;
__host__ __device__ inline size_t tc_region_bytes() {
  size_t p1 = static_cast<size_t>(kSortCap) * 8 + (kSortCap + 1) * 4 + sizeof(P1Smem) + 16;
  size_t p2 = static_cast<size_t>(kStages2) * kTile * 256;
  size_t p3 = sizeof(P3Smem);
  size_t m = p1 > p2 ? p1 : p2;
  return align_up(m > p3 ? m : p3, 1024);
}
constexpr int kTcSlack = 128;  // alignment slack of the dynamic shared memory
constexpr int kTcCtasPerSm = 2;  // launch bound: CTAs per SM the registers allow
// global_cand: the candidate list lives in a global scratch row (for large
// budgets whose list would leave room for one CTA per SM only)
__host__ __device__ inline size_t tc_smem_bytes(int C, int H, bool global_cand) {
  return kTcSlack + tc_region_bytes() + static_cast<size_t>(H) * 256 +
         (global_cand ? 0 : align_up(static_cast<size_t>(C) * 4, 16)) + align_up(static_cast<size_t>(H) * 4, 16) +
         (2 * kStages2 + 5) * 8 + 16;
}
__host__ __device__ inline int tc_tmem_cols(int C, int H) {
  const int sc = ((C + 127) / 128 + 15) / 16 * 16;
  int need = 2 * H + sc, cols = 32;
  while (cols < need) cols <<= 1;
  return cols;
}

// Block-sequential tensor-core kernel: one query at a time per CTA.  All
// warps build the candidate list; then warps 0-3 gather the rows (TMA
// gather4), warp 4 issues the UMMAs and warps 5-8 run the epilogue into
// TMEM score columns and, after the last tile, the top-k.
template <int H, bool kGC>
__global__ void __launch_bounds__(kTcThreads, kTcCtasPerSm)
    k_refine_tc(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                RefineArgs a, VersionTable vt) {
  // 1024-byte alignment (128-byte swizzle atoms) is requested from the
  // runtime; the launch adds kTcSlack bytes, and a base that would need
  // more than that is reported instead of overrunning the allocation
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (base - smem_raw > kTcSlack) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_RANGE);
    return;
  }
  uint8_t* region = base;
  uint8_t* qtile = region + tc_region_bytes();
  // the candidate list of the query in flight: in shared memory, or (kGC)
  // this CTA's row of the global scratch
  int32_t* cand = kGC ? a.cand_scratch + static_cast<int64_t>(blockIdx.x) * a.C
                      : reinterpret_cast<int32_t*>(qtile + H * 256);
  float* wsh = reinterpret_cast<float*>(qtile + H * 256 + (kGC ? 0 : align_up(static_cast<size_t>(a.C) * 4, 16)));
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(wsh) + align_up(H * 4, 16));
  uint64_t* qfull = bars + 2 * kStages2 + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages2 + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages2;
  uint64_t* tfull = bars + 2 * kStages2;
  uint64_t* tempty = bars + 2 * kStages2 + 2;
  uint64_t* sortbuf = reinterpret_cast<uint64_t*>(region);
  int32_t* pref = reinterpret_cast<int32_t*>(region + static_cast<size_t>(kSortCap) * 8);
  P3Smem& ps = *reinterpret_cast<P3Smem*>(region);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = tc_tmem_cols(a.C, H);
  const bool fp8 = a.key_dtype == KD_FP8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&full[s], 4);
      mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&tfull[c], 1);
      mbar_init(&tempty[c], 128);
    }
    mbar_init(qfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_holder, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  uint32_t g = 0;      // tiles processed so far by this CTA (barrier parity)
  uint32_t qiter = 0;  // queries processed so far by this CTA

  for (int qi = blockIdx.x; qi < a.T; qi += gridDim.x, ++qiter) {
    const int64_t t = a.pos0 + qi;
    // the query's heads (UMMA B operand) arrive by TMA while the
    // candidate list is built
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(qfull, H * 256);
      tma_load_2d(qtile, &qmap, 0, qi * H, qfull);
      tma_load_2d(qtile + H * 128, &qmap, 64, qi * H, qfull);
    }
    int nC;
    int64_t n_v;
    version_of(vt, t, &nC, &n_v);
    const int n = build_candidates<kGC>(a, qi, t, nC, n_v, cand, sortbuf, pref, BlockGrp{});
    if (a.cand_out) {
      for (int i = threadIdx.x; i < a.C; i += blockDim.x)
        a.cand_out[static_cast<int64_t>(qi) * a.C + i] = i < n ? cand[i] : -1;
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) wsh[h] = a.w[static_cast<int64_t>(qi) * H + h];
    fence_proxy_async_smem();
    __syncthreads();

    const int ntiles = (n + kTile - 1) / kTile;
    if (warp < 4) {
      // ------------------------------------------- TMA gather4 producers
      // Four warps share a tile (32 rows each): a single issuing warp
      // limits gather4 throughput, so the issue is spread out.
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j;
        const int s = gj % kStages2;
        if (gj >= kStages2 && !mbar_wait(&empty[s], ((gj / kStages2) & 1) ^ 1, a.err, abort_flag)) break;
        if (lane == 0) mbar_arrive_expect_tx(&full[s], kTile * 256 / 4);
        __syncwarp();
        if (lane < 16) {
          const int rl = warp * 32 + (lane & 7) * 4;  // first of this lane's 4 rows
          int r[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int slot = j * kTile + rl + i;
            int id = slot < n ? cand[slot] : 0;
            if (id < 0 || id > t) {
              atomicOr(a.err, DEV_ERR_RANGE);
              id = 0;
            }
            r[i] = id;
          }
          const int half = lane >> 3;
          uint8_t* dst = region + s * (kTile * 256) + half * (kTile * 128) + rl * 128;
          tma_gather4(dst, &kmap, half * 64, r[0], r[1], r[2], r[3], &full[s]);
        }
      }
    } else if (warp == 4) {
      // ------------------------------------------------------ UMMA issue
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(kTile, H);
        const uint32_t sb = smem_u32(qtile);
        // wait for this query's head tile (every query, so phases stay paired)
        const bool qok = mbar_wait(qfull, qiter & 1, a.err, abort_flag);
        for (int j = 0; qok && j < ntiles; ++j) {
          const uint32_t gj = g + j;
          const int s = gj % kStages2;
          const int acc = gj & 1;
          if (!mbar_wait(&full[s], (gj / kStages2) & 1, a.err, abort_flag)) break;
          if (gj >= 2 && !mbar_wait(&tempty[acc], ((gj >> 1) & 1) ^ 1, a.err, abort_flag)) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(region + s * (kTile * 256));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
            umma_bf16(tmem_base + acc * H, sdesc_sw128(sa + kb * (kTile * 128) + ko),
                      sdesc_sw128(sb + kb * (H * 128) + ko), idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          umma_commit(&tfull[acc]);
        }
      }
    } else if (warp >= 5) {
      // ------------------------------------------ epilogue -> TMEM scores
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j;
        const int acc = gj & 1;
        if (!mbar_wait(&tfull[acc], (gj >> 1) & 1, a.err, abort_flag)) break;
        tc_fence_after();
        float sc = head_sum<H>(tmem_base + acc * H + lane_off, wsh);
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        const int slot = j * kTile + row;
        if (fp8 && slot < n) sc *= a.key_scale[cand[slot]];
        tmem_st1(tmem_base + 2 * H + j + lane_off, sc);
      }
      tmem_st_wait();
    }
    g += ntiles;
    __syncthreads();
    if (*abort_flag) break;
    fence_proxy_async_smem();  // the region is rewritten by generic stores next
    // ----------------------------------------------------------- top-k
    if (warp >= 5) {
      const int quarter = warp & 3;
      P3Ctx c;
      c.row = quarter * 32 + lane;
      c.tcol = tmem_base + 2 * H + (static_cast<uint32_t>(quarter * 32) << 16);
      c.ntiles = ntiles;
      c.n = n;
      c.cand = cand;
      p3_topk(a, qi, c, c.row, ps);  // threads ordered by row: the emission order
    }
    __syncthreads();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

// ------------------------------------------------- pipelined tcgen05 kernel
// The three phases of consecutive queries overlap inside one CTA:
//   warps 0-3   gather candidate rows of query i (TMA gather4) and run the
//               epilogue (ReLU, head weights) into TMEM score columns
//   warps 4-7   build the candidate list of query i+1, then select the
//               top-k of query i-1 from its score columns
//   warps 8-11  (NGW = 8 only) gather rows
//   last warp   loads query i's head tile and issues the UMMAs
// Gather throughput grows with the number of warps issuing gather4
// (each warp's ops are issued one after another), so NGW = 8 splits a
// tile's 128 rows over eight warps, 16 rows each.  The roles sit on
// warpgroup boundaries so that, with NGW = 8, the gather-only warpgroup
// hands registers to the build / top-k warpgroup (setmaxnreg): launched
// at 72 per thread, 416 threads hold 29,952; afterwards 128 x 72
// (gather + epilogue) + 128 x 96 (build / top-k) + 128 x 40 (gather only)
// + 32 x 72 (UMMA) = 28,928 are in use.
// Candidate lists live in two global scratch rows per CTA and score
// columns in two TMEM buffers, so the build and the top-k of neighbouring
// queries run while the gather of query i keeps the copy engine busy.
// Synchronisation (all mbarriers, every wait bounded):
//   full[s]    tile rows landed in stage s (TMA transaction count)
//   tfull[a]   UMMAs of a tile done: accumulator a written, its stage free
//   tempty[a]  epilogue has read accumulator a
//   qfull      head tile landed;  qempty  UMMAs of the previous query done
//   cready[b]  list b built;  sready[b]  score columns b written;
//   sfree[b]   score columns b read by the top-k;
//   mread[b]   list b's length read by the UMMA warp
__host__ __device__ inline size_t pipe_bg_bytes() {
  const size_t p1 = align_up(static_cast<size_t>(kSortCap) * 8 + (kSortCap + 1) * 4, 16) + sizeof(P1Smem);
  const size_t p3 = sizeof(P3Smem);
  return align_up(p1 > p3 ? p1 : p3, 16);
}
// the top-k's shared memory (with the output sort) fits in the build's, so
// the pipelined kernel keeps two CTAs per SM
static_assert(sizeof(P3Smem) <= ((static_cast<size_t>(kSortCap) * 8 + (kSortCap + 1) * 4 + 15) & ~size_t(15)) +
                                    sizeof(P1Smem),
              "top-k shared memory grew past the candidate build's");
constexpr int kPipeBars = 16;
// Gathering warps of the pipelined kernel (4 or 8).  Eight measured
// slower on B200 (128K bf16: 2.21M vs 2.40M query tokens/s): the SM's
// gather4 throughput, not the issuing warps, bounds the rescore there.
#ifndef AI_PIPE_NGW
#define AI_PIPE_NGW 4
#endif
constexpr int kPipeNgw = AI_PIPE_NGW;
__host__ __device__ inline size_t pipe_smem_bytes(int H) {
  return kTcSlack + static_cast<size_t>(kStages2) * kTile * 256 + static_cast<size_t>(H) * 256 + pipe_bg_bytes() +
         align_up(static_cast<size_t>(H) * 4, 16) + 16 + kPipeBars * 8 + 8;
}
__host__ __device__ inline int pipe_sc_cols(int C) { return ((C + 127) / 128 + 15) / 16 * 16; }
// TMEM columns: two H-column accumulators and nsb score buffers
__host__ __device__ inline int pipe_tmem_cols(int C, int H, int nsb) {
  const int need = 2 * H + nsb * pipe_sc_cols(C);
  int cols = 32;
  while (cols < need) cols <<= 1;
  return cols;
}

constexpr int pipe_threads(int ngw) { return kTcThreads + (ngw - 4) * 32; }
constexpr int kPipeRegsLaunch = 72, kPipeRegsBuild = 96, kPipeRegsGather = 40;
static_assert(128 * kPipeRegsLaunch + 128 * kPipeRegsBuild + 128 * kPipeRegsGather + 32 * kPipeRegsLaunch <=
                  416 * kPipeRegsLaunch,
              "register split above the launch allocation");
static_assert(65536 / (2 * 416) / 8 * 8 == kPipeRegsLaunch, "launch allocation of the NGW = 8 kernel");
__device__ __forceinline__ void regs_inc96() { asm volatile("setmaxnreg.inc.sync.aligned.u32 96;\n" ::: "memory"); }
__device__ __forceinline__ void regs_dec40() { asm volatile("setmaxnreg.dec.sync.aligned.u32 40;\n" ::: "memory"); }

// NSB score buffers: 2 lets the epilogue of query i run while the top-k of
// query i-1 reads its columns; 1 (large budgets, where two buffers would
// need all 512 TMEM columns) makes the epilogue's first score store wait
// for that top-k, the gather and the build still overlapping.
template <int H, int NGW, int NSB>
__global__ void __launch_bounds__(pipe_threads(NGW), kTcCtasPerSm)
    k_refine_pipe(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                  RefineArgs a, VersionTable vt) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (base - smem_raw > kTcSlack) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_RANGE);
    return;
  }
  uint8_t* stages = base;
  uint8_t* qtile = stages + kStages2 * kTile * 256;
  uint8_t* bg = qtile + H * 256;
  float* wsh = reinterpret_cast<float*>(bg + pipe_bg_bytes());
  int* meta = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(wsh) + align_up(H * 4, 16));  // list lengths [2]
  uint64_t* bars = reinterpret_cast<uint64_t*>(meta + 4);
  uint64_t* full = bars;
  uint64_t* tfull = bars + 2;
  uint64_t* tempty = bars + 4;
  uint64_t* qfull = bars + 6;
  uint64_t* qempty = bars + 7;
  uint64_t* cready = bars + 8;
  uint64_t* sready = bars + 10;
  uint64_t* sfree = bars + 12;
  uint64_t* mread = bars + 14;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + kPipeBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_holder + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kMmaWarp = NGW + 4;
  const int tcols = pipe_tmem_cols(a.C, H, NSB);
  const int sc_cols = pipe_sc_cols(a.C);
  int32_t* rows = a.cand_scratch + static_cast<int64_t>(2 * blockIdx.x) * a.C;  // this CTA's two lists

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], NGW);  // one arrive.expect_tx per gathering warp
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 128);
      mbar_init(&cready[i], 128);
      mbar_init(&sready[i], 128);
      mbar_init(&sfree[i], 128);
      mbar_init(&mread[i], 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n_items = a.T * refine_split(a);
  const int nq = static_cast<int>(blockIdx.x) < n_items ? (n_items - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

  // Gathering warp gw (0 .. NGW-1) owns rows [gw * RPW, gw * RPW + RPW) of
  // every tile; lane l holds the id of row gw * RPW + l % RPW and lanes
  // below 2 * RPW / 4 issue one gather4 (4 rows, one 64-column half) each.
  constexpr int RPW = kTile / NGW;
  constexpr int GPH = RPW / 4;  // gather4 ops per half
  auto next_gid = [&](int j, int gw, int n, const int32_t* cl) -> int {
    const int slot = (j + 1) * kTile + gw * RPW + lane % RPW;
    return slot < n ? cl[slot] : 0;
  };
  auto issue_rows = [&](uint32_t gj, int j, int gid, int gw, int n, int64_t t, const int32_t* cl) {
    (void)cl;
    int id = gid;
    if (j * kTile + gw * RPW + lane % RPW < n && (id < 0 || id > t)) {
      atomicOr(a.err, DEV_ERR_RANGE);
      id = 0;
    }
    int r[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = __shfl_sync(0xffffffffu, id, ((lane % GPH) * 4 + i) % RPW);
    if (lane == 0) mbar_arrive_expect_tx(&full[gj & 1], kTile * 256 / NGW);
    __syncwarp();
    if (lane < 2 * GPH) {
      const int half = lane / GPH;
      const int rl = gw * RPW + (lane % GPH) * 4;
      uint8_t* dst = stages + (gj & 1) * (kTile * 256) + half * (kTile * 128) + rl * 128;
      tma_gather4(dst, &kmap, half * 64, r[0], r[1], r[2], r[3], &full[gj & 1]);
    }
  };

  if (warp < 4) {
    // --------------------------------------------- gather + epilogue (0-3)
    const int row = warp * 32 + lane;  // tile row == TMEM lane of this thread
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool fp8 = a.key_dtype == KD_FP8;
    uint32_t g = 0;           // tiles issued by this CTA so far
    int64_t last_issued = -1;
    bool dead = false;
    for (int q = 0; q < nq; ++q) {
      const RefineItem it = refine_item(a, q);
      const int qi = it.qi;
      const int64_t t = a.pos0 + qi;
      const int b = q & 1;
      const bool ok = !dead && mbar_wait(&cready[b], (q >> 1) & 1, a.err, abort_flag);
      // every thread of the group takes the same way out; the barrier also
      // orders the previous query's reads of wsh before its rewrite
      if (!named_bar_and(3, 128, ok)) break;
      tc_fence_after();
      int off, n;
      shard_span(a, it.sp, meta[b], &off, &n);
      const int nt = (n + kTile - 1) / kTile;
      const int32_t* cl = rows + static_cast<int64_t>(b) * a.C + off;
      for (int h = row; h < H; h += 128) wsh[h] = a.w[static_cast<int64_t>(qi) * H + h];
      named_bar(3, 128);
      const int sb = q % NSB;  // score buffer of this query
      const uint32_t scol = tmem_base + 2 * H + sb * sc_cols + lane_off;
      int myid = fp8 && row < n ? cl[row] : 0;  // this thread's epilogue row of tile 0 (fp8 scale)
      int gid = next_gid(-1, warp, n, cl);      // this lane's gather row of tile 0
      float sc0 = 1.f, sc1 = 1.f;          // fp8 scales of the tiles in flight (by tile parity)
      // iteration j issues tile j and finishes the epilogue of tile j-2
      auto step = [&](int j, float& s_slot) -> bool {
        const uint32_t gj = g + j;
        const int acc = gj & 1;
        if (j >= 2) {
          // UMMAs of tile j-2 done: its accumulator is ready and stage
          // gj & 1 is free
          const bool w = mbar_wait(&tfull[acc], ((gj - 2) >> 1) & 1, a.err, abort_flag);
          if (!__all_sync(0xffffffffu, w)) return false;
          tc_fence_after();
        }
        const float s_ep = s_slot;  // scale of tile j-2
        if (j < nt) {
          issue_rows(gj, j, gid, warp, n, t, cl);
          last_issued = gj;
          if (fp8) {
            // consumed two iterations later: the load stays in flight
            int id = myid;
            if (row + j * kTile >= n || id < 0 || id > t) id = 0;
            s_slot = a.key_scale[id];
            const int nslot = (j + 1) * kTile + row;
            myid = (j + 1 < nt && nslot < n) ? cl[nslot] : 0;
          }
          gid = next_gid(j, warp, n, cl);
        }
        if (j == 2 && q >= NSB) {
          // the first score store of this query: the top-k of query q - NSB
          // has finished reading the buffer
          const bool w = mbar_wait(&sfree[sb], ((q - NSB) / NSB) & 1, a.err, abort_flag);
          if (!__all_sync(0xffffffffu, w)) return false;
          tc_fence_after();
        }
        if (j >= 2) {
          float sc = head_sum<H>(tmem_base + acc * H + lane_off, wsh);
          tc_fence_before();
          mbar_arrive(&tempty[acc]);
          tmem_st1(scol + (j - 2), sc * s_ep);
        }
        return true;
      };
      bool good = true;
      for (int j = 0; good && j < nt + 2; j += 2) {
        good = step(j, sc0);
        if (good && j + 1 < nt + 2) good = step(j + 1, sc1);
      }
      if (!good) {
        dead = true;
        continue;  // the next barrier takes every thread of the group out
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sready[b]);
      g += nt;
    }
    if (*abort_flag && lane == 0 && last_issued >= 0) {
      // copies this warp issued may still be landing: bounded wait
      for (int64_t e = last_issued > 0 ? last_issued - 1 : 0; e <= last_issued; ++e)
        mbar_drain(&full[e & 1], (e >> 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------- UMMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTile, H);
      const uint32_t sb = smem_u32(qtile);
      uint32_t g = 0;
      int commits = 0;
      for (int q = 0; q < nq; ++q) {
        const RefineItem it = refine_item(a, q);
        const int qi = it.qi;
        const int b = q & 1;
        if (!mbar_wait(&cready[b], (q >> 1) & 1, a.err, abort_flag)) break;
        int off, n_loc;
        shard_span(a, it.sp, meta[b], &off, &n_loc);
        const int nt = (n_loc + kTile - 1) / kTile;
        mbar_arrive(&mread[b]);  // the slot's length is read; it may be rebuilt
        // the head tile is rewritten once the previous query's UMMAs are done
        if (q > 0 && !mbar_wait(qempty, (commits - 1) & 1, a.err, abort_flag)) break;
        mbar_arrive_expect_tx(qfull, H * 256);
        tma_load_2d(qtile, &qmap, 0, qi * H, qfull);
        tma_load_2d(qtile + H * 128, &qmap, 64, qi * H, qfull);
        if (!mbar_wait(qfull, q & 1, a.err, abort_flag)) {
          mbar_drain(qfull, q & 1);
          break;
        }
        bool good = true;
        for (int j = 0; j < nt; ++j) {
          const uint32_t gj = g + j;
          const int s = gj & 1;
          if (!mbar_wait(&full[s], (gj >> 1) & 1, a.err, abort_flag) ||
              (gj >= 2 && !mbar_wait(&tempty[s], ((gj >> 1) & 1) ^ 1, a.err, abort_flag))) {
            good = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + s * (kTile * 256));
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
            umma_bf16(tmem_base + s * H, sdesc_sw128(sa + kb * (kTile * 128) + ko),
                      sdesc_sw128(sb + kb * (H * 128) + ko), idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&tfull[s]);
        }
        umma_commit(qempty);
        ++commits;
        g += nt;
        if (!good) break;
      }
      // every UMMA issued has completed before the TMEM is released
      if (commits > 0) mbar_drain(qempty, (commits - 1) & 1);
    }
  } else if (warp >= 8) {
    // ------------------------------------------------ gather only (8-11)
    if (NGW == 8) regs_dec40();
    const int gw = warp - 4;
    uint32_t g = 0;
    int64_t last_issued = -1;
    for (int q = 0; q < nq; ++q) {
      const RefineItem it = refine_item(a, q);
      const int qi = it.qi;
      const int64_t t = a.pos0 + qi;
      const int b = q & 1;
      const bool ok = mbar_wait(&cready[b], (q >> 1) & 1, a.err, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      int off, n;
      shard_span(a, it.sp, meta[b], &off, &n);
      const int nt = (n + kTile - 1) / kTile;
      const int32_t* cl = rows + static_cast<int64_t>(b) * a.C + off;
      int gid = next_gid(-1, gw, n, cl);
      bool good = true;
      for (int j = 0; j < nt; ++j) {
        const uint32_t gj = g + j;
        if (gj >= 2) {
          // stage gj & 1 is free once the UMMAs of tile gj - 2 are done
          const bool w = mbar_wait(&tfull[gj & 1], ((gj - 2) >> 1) & 1, a.err, abort_flag);
          if (!__all_sync(0xffffffffu, w)) {
            good = false;
            break;
          }
        }
        issue_rows(gj, j, gid, gw, n, t, cl);
        last_issued = gj;
        gid = next_gid(j, gw, n, cl);
      }
      if (!good) break;
      g += nt;
    }
    if (*abort_flag && lane == 0 && last_issued >= 0) {
      for (int64_t e = last_issued > 0 ? last_issued - 1 : 0; e <= last_issued; ++e)
        mbar_drain(&full[e & 1], (e >> 1) & 1);
    }
  } else {
    // ------------------------------------------- candidate build + top-k (4-7)
    if (NGW == 8) regs_inc96();
    const SubGrp128 grp{128, 2};
    const int et = threadIdx.x - 128;
    uint64_t* sortbuf = reinterpret_cast<uint64_t*>(bg);
    int32_t* pref = reinterpret_cast<int32_t*>(bg + static_cast<size_t>(kSortCap) * 8);
    P3Smem& ps = *reinterpret_cast<P3Smem*>(bg);
    // returns false (every thread alike) when a wait gave up
    auto build = [&](int q) -> bool {
      if (q >= 2) {
        // slot q & 1 last held query q - 2: the gathering warps and the
        // top-k are done with it (sready, sequence), and the UMMA warp must
        // have read its length, which nothing else orders when that query
        // had no tiles
        const bool w = mbar_wait(&mread[q & 1], ((q - 2) >> 1) & 1, a.err, abort_flag);
        if (!named_bar_and(2, 128, w)) return false;
      }
      const RefineItem it = refine_item(a, q);
      const int qi = it.qi;
      const int64_t t = a.pos0 + qi;
      int nC;
      int64_t n_v;
      version_of(vt, t, &nC, &n_v);
      int32_t* cl = rows + static_cast<int64_t>(q & 1) * a.C;
      const int n = build_candidates<true>(a, qi, t, nC, n_v, cl, sortbuf, pref, grp);
      if (a.cand_out && it.sp == 0) {
        for (int i = et; i < a.C; i += 128) a.cand_out[static_cast<int64_t>(qi) * a.C + i] = i < n ? cl[i] : -1;
      }
      if (et == 0) meta[q & 1] = n;
      mbar_arrive(&cready[q & 1]);  // after this thread's own list stores
      return true;
    };
    const bool started = nq > 0 && build(0);
    for (int q = 0; started && q < nq; ++q) {
      const RefineItem it = refine_item(a, q);
      const int qi = it.qi;
      if (q + 1 < nq && !build(q + 1)) break;
      const bool ok = mbar_wait(&sready[q & 1], (q >> 1) & 1, a.err, abort_flag);
      if (!named_bar_and(1, 128, ok)) break;
      tc_fence_after();
      const int quarter = warp & 3;
      P3Ctx c;
      c.row = quarter * 32 + lane;
      c.tcol = tmem_base + 2 * H + (q % NSB) * sc_cols + (static_cast<uint32_t>(quarter * 32) << 16);
      int off;
      shard_span(a, it.sp, meta[q & 1], &off, &c.n);
      c.ntiles = (c.n + kTile - 1) / kTile;
      c.cand = rows + static_cast<int64_t>(q & 1) * a.C + off;
      // output row: the query's, or (split) its part's row of [split, T, k]
      p3_topk(a, it.sp * a.T + qi, c, c.row, ps);  // c.row == et: rows in thread order
      tc_fence_before();
      mbar_arrive(&sfree[q % NSB]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tcols);
  }
}

// CTAs per SM of a tensor-core refine launch: bounded by shared memory
// (228 KiB per SM, 1 KiB reserved per CTA; the carveout is set to the
// maximum), by TMEM (512 columns) and by the registers.
int per_sm_for(size_t smem, int tmem_cols) {
  int p = static_cast<int>((228 * 1024) / (smem + 1024));
  const int tm = 512 / tmem_cols;
  p = p < tm ? p : tm;
  p = p < kTcCtasPerSm ? p : kTcCtasPerSm;
  return p < 1 ? 1 : p;
}

}  // namespace

int pick_refine_kernel(int C, int H, bool has_scratch) {
  // the pipelined kernel where it keeps two CTAs per SM; else the
  // block-sequential one, its list in shared memory unless that costs the
  // second CTA
  constexpr size_t kMaxSmem = 227 * 1024;
  const size_t sm_local = tc_smem_bytes(C, H, false), sm_pipe = pipe_smem_bytes(H);
  if (has_scratch && sm_pipe <= kMaxSmem && per_sm_for(sm_pipe, pipe_tmem_cols(C, H, 2)) >= kTcCtasPerSm)
    return REFINE_PIPE;
  if (has_scratch && sm_pipe <= kMaxSmem && per_sm_for(sm_pipe, pipe_tmem_cols(C, H, 1)) >= kTcCtasPerSm)
    return REFINE_PIPE_1BUF;
  if (sm_local <= kMaxSmem && per_sm_for(sm_local, tc_tmem_cols(C, H)) >= kTcCtasPerSm) return REFINE_SEQ_SMEM;
  return has_scratch ? REFINE_SEQ_GLOBAL : REFINE_SEQ_SMEM;
}

size_t refine_smem_bytes(int C, int H, int d, bool tc) {
  if (tc) return tc_smem_bytes(C, H, true);  // the smaller layout; the launch picks
  return 1024 + region_bytes(H, d, false) + 2 * align_up(static_cast<size_t>(C) * 4, 16) +
         align_up(static_cast<size_t>(H) * 4, 16) + (2 * kStages + 4) * 8 + 16;
}

cudaError_t launch_refine(const RefineArgs& a, const VersionTable& vt, const CUtensorMap* kmap,
                          const CUtensorMap* qmap, int num_sms, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const bool tc = kmap != nullptr && qmap != nullptr;
  const size_t smem = refine_smem_bytes(a.C, a.H, a.d, tc);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (tc) {
    if (a.d != 128 || !a.q_is_bf16 || (a.key_dtype != KD_BF16 && a.key_dtype != KD_FP8))
      return cudaErrorInvalidValue;
    if (a.H != 32 && a.H != 64) return cudaErrorInvalidValue;
    if (a.k > kTcMaxK) return cudaErrorInvalidValue;
    const size_t sm_local = tc_smem_bytes(a.C, a.H, false), sm_glob = tc_smem_bytes(a.C, a.H, true);
    const size_t sm_pipe = pipe_smem_bytes(a.H);
    constexpr size_t kMaxSmem = 227 * 1024;
    const int kind = a.refine_kernel == REFINE_AUTO ? pick_refine_kernel(a.C, a.H, a.cand_scratch != nullptr)
                                                    : a.refine_kernel;
    if (kind < REFINE_SEQ_SMEM || kind > REFINE_PIPE_1BUF) return cudaErrorInvalidValue;
    const bool pipe = kind == REFINE_PIPE || kind == REFINE_PIPE_1BUF;
    if ((a.n_shards > 1 || a.split > 1) && !pipe) return cudaErrorInvalidValue;  // pipelined kernels only
    if ((kind == REFINE_SEQ_GLOBAL || pipe) && !a.cand_scratch) return cudaErrorInvalidValue;
    const int tm = pipe ? pipe_tmem_cols(a.C, a.H, kind == REFINE_PIPE ? 2 : 1) : tc_tmem_cols(a.C, a.H);
    const size_t smem_tc = kind == REFINE_SEQ_SMEM ? sm_local : kind == REFINE_SEQ_GLOBAL ? sm_glob : sm_pipe;
    if (smem_tc > kMaxSmem || tm > 512) return cudaErrorInvalidValue;
    const int per_sm = per_sm_for(smem_tc, tm);
    const int items = pipe ? a.T * (a.split > 1 ? a.split : 1) : a.T;
    const int grid = items < num_sms * per_sm ? items : num_sms * per_sm;
    if (grid <= 0) return cudaSuccess;
#define AI_LAUNCH_REFINE(KERNEL)                                                                         \
  do {                                                                                                   \
    cudaFuncSetAttribute(KERNEL, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem_tc)); \
    cudaFuncSetAttribute(KERNEL, cudaFuncAttributePreferredSharedMemoryCarveout, 100);                   \
    count_launch();                                                                                      \
    KERNEL<<<grid, pipe ? pipe_threads(kPipeNgw) : kTcThreads, smem_tc, st>>>(*kmap, *qmap, a, vt);      \
  } while (0)
    if (a.H == 32) {
      if (kind == REFINE_PIPE) AI_LAUNCH_REFINE((k_refine_pipe<32, kPipeNgw, 2>));
      else if (kind == REFINE_PIPE_1BUF) AI_LAUNCH_REFINE((k_refine_pipe<32, kPipeNgw, 1>));
      else if (kind == REFINE_SEQ_GLOBAL) AI_LAUNCH_REFINE((k_refine_tc<32, true>));
      else AI_LAUNCH_REFINE((k_refine_tc<32, false>));
    } else {
      if (kind == REFINE_PIPE) AI_LAUNCH_REFINE((k_refine_pipe<64, kPipeNgw, 2>));
      else if (kind == REFINE_PIPE_1BUF) AI_LAUNCH_REFINE((k_refine_pipe<64, kPipeNgw, 1>));
      else if (kind == REFINE_SEQ_GLOBAL) AI_LAUNCH_REFINE((k_refine_tc<64, true>));
      else AI_LAUNCH_REFINE((k_refine_tc<64, false>));
    }
#undef AI_LAUNCH_REFINE
  } else {
    if (a.n_shards > 1 || a.split > 1) return cudaErrorInvalidValue;
    // the output sort reuses the phase-1 region: room for kRowTopkMaxK keys
    if (a.k > kRowTopkMaxK || region_bytes(a.H, a.d, false) < static_cast<size_t>(kRowTopkMaxK) * 8)
      return cudaErrorInvalidValue;
    cudaFuncSetAttribute(k_refine_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    int per_sm = 1;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_refine_simt, kSimtThreads, smem);
    if (per_sm < 1) per_sm = 1;
    const int grid = a.T < num_sms * per_sm ? a.T : num_sms * per_sm;
    count_launch();
    k_refine_simt<<<grid, kSimtThreads, smem, st>>>(a, vt);
  }
  return cudaGetLastError();
}

}  // namespace aiidx
