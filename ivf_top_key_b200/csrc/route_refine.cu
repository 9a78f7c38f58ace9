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
// One persistent CTA per SM walks queries.  Per query:
//  1. size-weighted radix select of the budget threshold over the cluster
//     scores of the visible, non-empty clusters; the clusters at or above it
//     are sorted by (score desc, id asc) and their member lists are copied,
//     after sinks and the open window, into a shared-memory candidate list;
//  2. exact rescore of the candidates, 128 at a time: the key rows are
//     gathered into the 128-byte-swizzled UMMA layout (cp.async for bf16,
//     fp8 codes widened to bf16 in registers), one tcgen05 UMMA
//     (M = 128 candidates, N = H heads, K = 128) per tile accumulates in
//     TMEM, and four epilogue warps apply ReLU, the head weights and the fp8
//     scale (SIMT FMA path for fp32 keys);
//  3. radix select of the k-th score; ties at the threshold go to the lower
//     key id; ids are written in candidate-slot order, padded with -1.
#include "common.cuh"
#include "kernels.h"
#include "select.cuh"

namespace aiidx {
namespace {

constexpr int kSortCap = 4096;
constexpr int kTile = 128;
constexpr int kStages = 3;
constexpr int kTcThreads = 288;   // warps 0-3 gather, 4 UMMA, 5-8 epilogue
constexpr int kSimtThreads = 256;

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

__device__ __forceinline__ void bitonic_sort_u64(uint64_t* buf, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
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
      __syncthreads();
    }
  }
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
__device__ int build_candidates(const RefineArgs& a, int qi, int64_t t, int nC, int64_t n_v,
                                int32_t* cand, uint64_t* sortbuf, int32_t* pref,
                                BlockScratch& bs) {
  const int C = a.C;
  const int n_s = static_cast<int>(min64(a.n_sinks, t + 1));
  const int64_t open_lo = max64(n_v, a.n_sinks);
  const int64_t n_open64 = open_lo <= t ? t + 1 - open_lo : 0;
  const int fixed = static_cast<int>(min64(C, n_s + n_open64));
  for (int i = threadIdx.x; i < fixed; i += blockDim.x)
    cand[i] = i < n_s ? i : static_cast<int32_t>(open_lo + (i - n_s));
  const int rem = C - fixed;
  if (rem <= 0 || nC == 0) {
    __syncthreads();
    return fixed;
  }
  const float* rs = a.route + static_cast<int64_t>(qi) * a.ld_route;
  const int32_t* off = a.offsets;
  auto size = [&](int c) -> uint32_t { return static_cast<uint32_t>(off[c + 1] - off[c]); };
  auto key = [&](int c) -> uint32_t { return f2key(rs[c]); };
  auto pred = [&](int c) -> bool { return off[c + 1] > off[c]; };
  uint64_t above = 0, tot = 0;
  const uint32_t theta = radix_select(nC, key, pred, size, static_cast<uint64_t>(rem), &above, bs, &tot);
  const bool take_all = tot <= static_cast<uint64_t>(rem);
  int nsel = 0;
  for (int base = 0; base < nC; base += blockDim.x) {
    const int c = base + threadIdx.x;
    const bool p = c < nC && pred(c) && (take_all || key(c) >= theta);
    int total;
    const int r = block_rank(p, &total, bs);
    if (p && nsel + r < kSortCap)
      sortbuf[nsel + r] = (static_cast<uint64_t>(~key(c)) << 32) | static_cast<uint32_t>(c);
    nsel += total;
  }
  if (nsel > kSortCap) {
    if (threadIdx.x == 0) atomicOr(a.err, DEV_ERR_CAPACITY);
    nsel = kSortCap;
  }
  int np = 1;
  while (np < nsel) np <<= 1;
  for (int i = nsel + threadIdx.x; i < np; i += blockDim.x) sortbuf[i] = ~0ull;
  __syncthreads();
  bitonic_sort_u64(sortbuf, np);
  // exclusive prefix of member counts in rank order
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int carry = 0;
    for (int base = 0; base < nsel; base += 32) {
      const int r = base + lane;
      const int v = r < nsel ? static_cast<int>(size(static_cast<int>(sortbuf[r] & 0xffffffffu))) : 0;
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
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int r = warp; r < nsel; r += nwarps) {
    const int slot0 = fixed + pref[r];
    if (slot0 >= C) continue;
    const int c = static_cast<int>(sortbuf[r] & 0xffffffffu);
    const int o = off[c];
    const int n = min(static_cast<int>(size(c)), C - slot0);
    for (int j = lane; j < n; j += 32) cand[slot0 + j] = a.members[o + j];
  }
  const int len = static_cast<int>(min64(C, static_cast<int64_t>(fixed) + pref[nsel]));
  __syncthreads();
  return len;
}

// Phase 3: top-k of score[0..n) with ids cand[]; ties go to the lower id.
__device__ __forceinline__ void topk_emit(const RefineArgs& a, int qi, const float* score,
                                          const int32_t* cand, int n, BlockScratch& bs) {
  int32_t* out = a.out + static_cast<int64_t>(qi) * a.k;
  float* outs = a.out_scores ? a.out_scores + static_cast<int64_t>(qi) * a.k : nullptr;
  topk_select_emit(
      n, [&](int i) -> float { return score[i]; }, [&](int i) -> int32_t { return cand[i]; }, a.k,
      out, outs, bs);
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
  size_t p1 = static_cast<size_t>(kSortCap) * 8 + (kSortCap + 1) * 4;
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
    const int n = build_candidates(a, qi, t, nC, n_v, L.cand, L.sortbuf, L.pref, bs);
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
    topk_emit(a, qi, L.score, L.cand, n, bs);
  }
}

// ---------------------------------------------------------- tcgen05 kernel
// Gather one 128-row tile of candidate keys into the swizzled bf16 layout.
// Thread r (0..127) of the gather warps; rows handled per warp: 32.
__device__ __forceinline__ void gather_tile_bf16(const RefineArgs& a, const int32_t* cand, int n,
                                                 int slot0, int64_t t, uint8_t* stage) {
  const int gt = threadIdx.x;  // 0..127
  const int gw = gt >> 5, lane = gt & 31;
  const int chunk = lane & 15;
  const uint16_t* keys = reinterpret_cast<const uint16_t*>(a.keys);
#pragma unroll 4
  for (int p = 0; p < 16; ++p) {
    const int row = gw * 32 + 2 * p + (lane >> 4);
    const int slot = slot0 + row;
    int32_t id = slot < n ? cand[slot] : -1;
    if (id > t) {
      atomicOr(a.err, DEV_ERR_RANGE);
      id = -1;
    }
    uint8_t* dst = stage + (chunk >> 3) * (kTile * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
    const void* src = id >= 0 ? static_cast<const void*>(keys + static_cast<int64_t>(id) * 128 + chunk * 8)
                              : static_cast<const void*>(keys);
    const uint32_t sz = id >= 0 ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(sz)
                 : "memory");
  }
}

__device__ __forceinline__ void gather_tile_fp8(const RefineArgs& a, const int32_t* cand, int n,
                                                int slot0, int64_t t, uint8_t* stage) {
  const int gt = threadIdx.x;
  const int gw = gt >> 5, lane = gt & 31;
  const int c8 = lane & 7;  // 16-code chunk of the 128-code row
  const uint8_t* keys = reinterpret_cast<const uint8_t*>(a.keys);
  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int row = gw * 32 + 4 * p + (lane >> 3);
    const int slot = slot0 + row;
    int32_t id = slot < n ? cand[slot] : -1;
    if (id > t) {
      atomicOr(a.err, DEV_ERR_RANGE);
      id = -1;
    }
    v[p] = id >= 0 ? __ldg(reinterpret_cast<const uint4*>(keys + static_cast<int64_t>(id) * 128) + c8)
                   : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int row = gw * 32 + 4 * p + (lane >> 3);
    const uint8_t* b = reinterpret_cast<const uint8_t*>(&v[p]);
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      __nv_fp8x2_e4m3 pr;
      pr.__x = static_cast<__nv_fp8x2_storage_t>(b[2 * j] | (b[2 * j + 1] << 8));
      __nv_bfloat162 h2 = __float22bfloat162_rn(static_cast<float2>(pr));
      w[j] = *reinterpret_cast<uint32_t*>(&h2);
    }
    // codes 16*c8 .. 16*c8+15 -> bf16 chunks 2*c8 and 2*c8+1 (8 values each)
#pragma unroll
    for (int hlf = 0; hlf < 2; ++hlf) {
      const int chunk = 2 * c8 + hlf;
      uint8_t* dst = stage + (chunk >> 3) * (kTile * 128) + row * 128 + (((chunk & 7) ^ (row & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[4 * hlf], w[4 * hlf + 1], w[4 * hlf + 2], w[4 * hlf + 3]);
    }
  }
}

template <int H>
__global__ void __launch_bounds__(kTcThreads, 1) k_refine_tc(RefineArgs a, VersionTable vt) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ BlockScratch bs;
  Layout L = carve(smem_raw, a.C, H, 128, true);
  uint64_t* full = L.bars;
  uint64_t* empty = L.bars + kStages;
  uint64_t* tfull = L.bars + 2 * kStages;
  uint64_t* tempty = L.bars + 2 * kStages + 2;
  uint8_t* stages = L.region;
  uint8_t* qtile = L.region + kStages * kTile * 256;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kTmemCols = 2 * H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 128);
      mbar_init(&empty[s], 1);
    }
    for (int c = 0; c < 2; ++c) {
      mbar_init(&tfull[c], 1);
      mbar_init(&tempty[c], 128);
    }
    *L.abort = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(L.tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *L.tmem;
  uint32_t g = 0;  // tiles processed by this CTA so far (for barrier parity)

  for (int qi = blockIdx.x; qi < a.T; qi += gridDim.x) {
    const int64_t t = a.pos0 + qi;
    int nC;
    int64_t n_v;
    version_of(vt, t, &nC, &n_v);
    const int n = build_candidates(a, qi, t, nC, n_v, L.cand, L.sortbuf, L.pref, bs);
    if (a.cand_out) {
      for (int i = threadIdx.x; i < a.C; i += blockDim.x)
        a.cand_out[static_cast<int64_t>(qi) * a.C + i] = i < n ? L.cand[i] : -1;
    }
    // query heads -> swizzled UMMA B tile (H rows x 128 bf16), weights -> smem
    const uint16_t* qg = reinterpret_cast<const uint16_t*>(a.q) + static_cast<int64_t>(qi) * H * 128;
    for (int i = threadIdx.x; i < H * 16; i += blockDim.x) {
      const int h = i >> 4, chunk = i & 15;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(qg + h * 128) + chunk);
      uint8_t* dst = qtile + (chunk >> 3) * (H * 128) + h * 128 + (((chunk & 7) ^ (h & 7)) << 4);
      *reinterpret_cast<uint4*>(dst) = v;
    }
    for (int h = threadIdx.x; h < H; h += blockDim.x) L.wsh[h] = a.w[static_cast<int64_t>(qi) * H + h];
    fence_proxy_async_smem();
    __syncthreads();

    const int ntiles = (n + kTile - 1) / kTile;
    if (warp < 4) {
      // ------------------------------------------------------------ gather
      if (a.key_dtype == KD_BF16) {
        for (int j = 0; j < ntiles; ++j) {
          const uint32_t gj = g + j;
          const int s = gj % kStages;
          if (gj >= kStages && !mbar_wait(&empty[s], ((gj / kStages) & 1) ^ 1, a.err, L.abort)) break;
          gather_tile_bf16(a, L.cand, n, j * kTile, t, stages + s * (kTile * 256));
          cp_async_commit();
          if (j >= kStages - 1) {
            cp_async_wait<kStages - 1>();
            fence_proxy_async_smem();
            mbar_arrive(&full[(g + j - (kStages - 1)) % kStages]);
          }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        for (int j = max(0, ntiles - (kStages - 1)); j < ntiles; ++j) mbar_arrive(&full[(g + j) % kStages]);
      } else {
        for (int j = 0; j < ntiles; ++j) {
          const uint32_t gj = g + j;
          const int s = gj % kStages;
          if (gj >= kStages && !mbar_wait(&empty[s], ((gj / kStages) & 1) ^ 1, a.err, L.abort)) break;
          gather_tile_fp8(a, L.cand, n, j * kTile, t, stages + s * (kTile * 256));
          fence_proxy_async_smem();
          mbar_arrive(&full[s]);
        }
      }
    } else if (warp == 4) {
      // -------------------------------------------------------- UMMA issue
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(kTile, H);
        const uint32_t sb = smem_u32(qtile);
        for (int j = 0; j < ntiles; ++j) {
          const uint32_t gj = g + j;
          const int s = gj % kStages;
          const int acc = gj & 1;
          if (!mbar_wait(&full[s], (gj / kStages) & 1, a.err, L.abort)) break;
          if (gj >= 2 && !mbar_wait(&tempty[acc], ((gj >> 1) & 1) ^ 1, a.err, L.abort)) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + s * (kTile * 256));
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
    } else {
      // ---------------------------------------------------------- epilogue
      const int quarter = warp & 3;
      const int row = quarter * 32 + lane;
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      for (int j = 0; j < ntiles; ++j) {
        const uint32_t gj = g + j;
        const int acc = gj & 1;
        if (!mbar_wait(&tfull[acc], (gj >> 1) & 1, a.err, L.abort)) break;
        tc_fence_after();
        float sc = 0.f;
#pragma unroll
        for (int c = 0; c < H / 32; ++c) {
          float v[32];
          tmem_ld32(tmem_base + acc * H + c * 32 + lane_off, v);
          tmem_ld_wait();
#pragma unroll
          for (int h = 0; h < 32; ++h) sc = fmaf(L.wsh[c * 32 + h], fmaxf(v[h], 0.f), sc);
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        const int slot = j * kTile + row;
        if (slot < n) {
          if (a.key_scale) sc *= a.key_scale[L.cand[slot]];
          L.score[slot] = sc;
        }
      }
    }
    g += ntiles;
    __syncthreads();
    fence_proxy_async_smem();  // the region is rewritten by generic stores next
    if (*L.abort) break;
    topk_emit(a, qi, L.score, L.cand, n, bs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

size_t refine_smem_bytes(int C, int H, int d, bool tc) {
  return 1024 + region_bytes(H, d, tc) + 2 * align_up(static_cast<size_t>(C) * 4, 16) +
         align_up(static_cast<size_t>(H) * 4, 16) + (2 * kStages + 4) * 8 + 16;
}

cudaError_t launch_refine(const RefineArgs& a, const VersionTable& vt, bool tc, int num_sms,
                          cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  const size_t smem = refine_smem_bytes(a.C, a.H, a.d, tc);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  if (tc) {
    if (a.d != 128 || !a.q_is_bf16 || (a.key_dtype != KD_BF16 && a.key_dtype != KD_FP8))
      return cudaErrorInvalidValue;
    const int grid = a.T < num_sms ? a.T : num_sms;
    if (a.H == 32) {
      cudaFuncSetAttribute(k_refine_tc<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      count_launch();
      k_refine_tc<32><<<grid, kTcThreads, smem, st>>>(a, vt);
    } else if (a.H == 64) {
      cudaFuncSetAttribute(k_refine_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      count_launch();
      k_refine_tc<64><<<grid, kTcThreads, smem, st>>>(a, vt);
    } else {
      return cudaErrorInvalidValue;
    }
  } else {
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
