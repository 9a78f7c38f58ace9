// Indexer score matrices: out[q, a] = sum_h w[q,h] * ReLU(q_h . A_a).
//
// The DSA indexer score (AttentionIndex explainer, paper-daily.com, section
// "代表向量为什么要学？": per-head inner products, ReLU, head-weighted sum)
// evaluated for a block of queries against a set of rows A.  Used twice:
//   * routing: A = cluster representatives (bf16), out = [T, nC] cluster
//     scores (explainer, "查询时怎么挑候选？": every query scores every
//     representative with the indexer's own formula);
//   * exhaustive selection: A = the key store, with the causal mask
//     key position > query position -> -inf.
//
// tcgen05 path (bf16 rows, d = 128, H in {32, 64}): persistent CTAs, one
// per SM, walk work items.  An item is 256 / H queries (the whole N = 256 of
// one UMMA: query x head rows, K-major) against a range of 128-row A tiles.
// Consecutive items share their A range, so CTAs running side by side
// stream the same A tiles (L2 reuse), each starting at its own offset.  Warp 0 issues TMA: the next item's
// query tile and head weights go into the other half of a double buffer
// while the current item runs, A tiles through a 3-deep ring.  Warp 1 owns
// TMEM and issues the UMMAs (M = 128, N = 256, K = 16 x 8) into one of two
// 256-column accumulators.  Warps 4-11 read an accumulator back (TMEM lane
// = one A row; warp w serves lanes 32 (w mod 4) .. + 31 and half of the
// item's queries), apply ReLU and the head weights, and write the scores.
// fp8 rows are given as bf16 copies of their codes; the per-row scale
// multiplies the score (a positive scale commutes with ReLU).
//
// SIMT path (fp32 rows/queries or other shapes): plain tiled FMA kernel.
#include "common.cuh"
#include "kernels.h"

namespace aiidx {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kK = 128;
constexpr int kAStages = 3;
constexpr int kATile = kBM * kK * 2;  // 32 KiB
constexpr int kBTile = kBN * kK * 2;  // 64 KiB
constexpr int kThreads = 384;         // 12 warps: TMA, UMMA, 2 idle, 8 epilogue
constexpr int kEpiWarp0 = 4;
constexpr int kEpiThreads = 256;
constexpr int kSlack = 128;           // alignment slack of the dynamic shared memory
constexpr int kBars = 2 + 2 + 2 * kAStages + 2 + 2;
constexpr int kSmemBytes = kSlack + 2 * kBTile + kAStages * kATile + 2 * kBN * 4 + kBars * 8 + 16;
static_assert(kSmemBytes <= 227 * 1024, "scores GEMM shared memory");

struct GemmSmem {
  uint8_t* b;        // 2 x [2 K-blocks][256 rows][128 B]
  uint8_t* a;        // kAStages x [2 K-blocks][128 rows][128 B]
  float* w;          // 2 x [256] head weights of the item's queries
  uint64_t* bars;    // bfull[2], bempty[2], afull[kAStages], aempty[kAStages], tfull[2], tempty[2]
  uint32_t* tmem;    // allocated TMEM base
  int* abort;
};

__device__ __forceinline__ GemmSmem carve(uint8_t* p) {
  GemmSmem s;
  s.b = p;
  s.a = p + 2 * kBTile;
  s.w = reinterpret_cast<float*>(s.a + kAStages * kATile);
  s.bars = reinterpret_cast<uint64_t*>(s.w + 2 * kBN);
  s.tmem = reinterpret_cast<uint32_t*>(s.bars + kBars);
  s.abort = reinterpret_cast<int*>(s.tmem + 1);
  return s;
}

// 1-D bulk copy global -> shared, completion counted on an mbarrier
// (addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Work item `it`: A range it / n_qb, query block it % n_qb.  Tile range
// [*tb, *te) (empty when the causal mask hides the whole range).
struct ItemMap {
  int n_qb, n_atiles, apc, QPT;
  int64_t n_items;
  __device__ void at(const ScoreArgs& a, int64_t it, int* q0, int* tb, int* te) const {
    const int r = static_cast<int>(it / n_qb);
    const int qb = static_cast<int>(it % n_qb);
    *q0 = qb * QPT;
    *tb = r * apc;
    int e = min(n_atiles, *tb + apc);
    if (a.causal) {
      // last key row any query of the block may see
      const int64_t qlast = a.q_pos0 + min(*q0 + QPT, a.T) - 1;
      const int64_t alast = qlast - a.a_pos0;
      const int lim = alast < 0 ? 0 : static_cast<int>(alast / kBM) + 1;
      e = min(e, lim);
    }
    *te = e;
  }
};

// The jj-th A tile a CTA processes in the range [tb, te): the range rotated
// by up to 32 tiles per CTA, so that CTAs running side by side read
// different tiles at a time (no L2 hot spot) yet stay within a few MiB of
// one another (L2 reuse).
__device__ __forceinline__ int rotated_tile(int tb, int te, int jj) {
  const int n = te - tb;
  const int rot = static_cast<int>(blockIdx.x) % (n < 32 ? n : 32);
  const int r = jj + rot;
  return tb + (r < n ? r : r - n);
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    k_scores_tc(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                ScoreArgs args) {
  constexpr int QPT = kBN / H;       // queries per item
  constexpr int QPW = QPT / 2;       // queries per epilogue warp
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (base - smem_raw > kSlack) {
    if (threadIdx.x == 0) atomicOr(args.err, DEV_ERR_RANGE);
    return;
  }
  GemmSmem sm = carve(base);
  uint64_t* bfull = sm.bars;
  uint64_t* bempty = sm.bars + 2;
  uint64_t* afull = sm.bars + 4;
  uint64_t* aempty = sm.bars + 4 + kAStages;
  uint64_t* tfull = sm.bars + 4 + 2 * kAStages;
  uint64_t* tempty = sm.bars + 4 + 2 * kAStages + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  ItemMap im;
  im.QPT = QPT;
  im.n_qb = (args.T + QPT - 1) / QPT;
  im.n_atiles = (args.nA + kBM - 1) / kBM;
  im.apc = args.a_tiles_per_cta;
  im.n_items = static_cast<int64_t>((im.n_atiles + im.apc - 1) / im.apc) * im.n_qb;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bfull[b], 1);
      // released by the UMMA warp's commit (its last tile of the item) and by
      // every epilogue thread (done with the item's weights)
      mbar_init(&bempty[b], 1 + kEpiThreads);
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiThreads);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    *sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      uint32_t k = 0, g = 0;  // items and A tiles issued by this CTA
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < im.n_items; it += gridDim.x) {
        int q0, tb, te;
        im.at(args, it, &q0, &tb, &te);
        if (te <= tb || q0 >= args.T) continue;
        const int b = k & 1;
        if (k >= 2 && !mbar_wait(&bempty[b], ((k >> 1) & 1) ^ 1, args.err, sm.abort)) break;
        const int nq = min(QPT, args.T - q0);
        mbar_arrive_expect_tx(&bfull[b], kBTile + nq * H * 4);
        tma_load_2d(sm.b + b * kBTile, &mapB, 0, q0 * H, &bfull[b]);
        tma_load_2d(sm.b + b * kBTile + kBN * 128, &mapB, 64, q0 * H, &bfull[b]);
        bulk_load(sm.w + b * kBN, args.w + static_cast<int64_t>(q0) * H, nq * H * 4, &bfull[b]);
        for (int jj = 0; jj < te - tb; ++jj, ++g) {
          const int i = rotated_tile(tb, te, jj);
          const int s = g % kAStages;
          if (g >= kAStages && !mbar_wait(&aempty[s], ((g / kAStages) & 1) ^ 1, args.err, sm.abort)) {
            ok = false;
            break;
          }
          uint8_t* dst = sm.a + s * kATile;
          mbar_arrive_expect_tx(&afull[s], kATile);
          tma_load_2d(dst, &mapA, 0, i * kBM, &afull[s]);
          tma_load_2d(dst + kBM * 128, &mapA, 64, i * kBM, &afull[s]);
        }
        ++k;
      }
      if (*sm.abort) {
        // copies this thread issued may still be landing: bounded waits
        for (uint32_t e = g > kAStages ? g - kAStages : 0; e < g; ++e)
          mbar_drain(&afull[e % kAStages], (e / kAStages) & 1);
        if (k > 0) mbar_drain(&bfull[(k - 1) & 1], ((k - 1) >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- UMMA issue
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      uint32_t k = 0, g = 0;
      bool ok = true;
      for (int64_t it = blockIdx.x; ok && it < im.n_items; it += gridDim.x) {
        int q0, tb, te;
        im.at(args, it, &q0, &tb, &te);
        if (te <= tb || q0 >= args.T) continue;
        const int b = k & 1;
        if (!mbar_wait(&bfull[b], (k >> 1) & 1, args.err, sm.abort)) break;
        const uint32_t sb = smem_u32(sm.b + b * kBTile);
        for (int jj = 0; jj < te - tb; ++jj, ++g) {
          const int s = g % kAStages;
          const int acc = g & 1;
          if (!mbar_wait(&afull[s], (g / kAStages) & 1, args.err, sm.abort) ||
              (g >= 2 && !mbar_wait(&tempty[acc], ((g >> 1) & 1) ^ 1, args.err, sm.abort))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm.a + s * kATile);
          const uint32_t d = tmem_base + acc * kBN;
#pragma unroll
          for (int kk = 0; kk < kK / 16; ++kk) {
            const uint32_t kb = kk >> 2, ko = (kk & 3) * 32;
            umma_bf16(d, sdesc_sw128(sa + kb * (kBM * 128) + ko),
                      sdesc_sw128(sb + kb * (kBN * 128) + ko), idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&aempty[s]);
          umma_commit(&tfull[acc]);
        }
        umma_commit(&bempty[b]);  // the item's UMMAs no longer read its query tile
        ++k;
      }
      // every UMMA issued has completed before the TMEM is released
      if (g > 0) mbar_drain(&tfull[(g - 1) & 1], ((g - 1) >> 1) & 1);
    }
  } else if (warp >= kEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int qh = (warp - kEpiWarp0) >> 2;         // which half of the item's queries
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t k = 0, g = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; ok && it < im.n_items; it += gridDim.x) {
      int q0, tb, te;
      im.at(args, it, &q0, &tb, &te);
      if (te <= tb || q0 >= args.T) continue;
      const int b = k & 1;
      // the weights land with the query tile
      if (!mbar_wait(&bfull[b], (k >> 1) & 1, args.err, sm.abort)) break;
      const float* wk = sm.w + b * kBN + qh * QPW * H;
      uint32_t kmn[QPW], kmx[QPW];
#pragma unroll
      for (int qi = 0; qi < QPW; ++qi) {
        kmn[qi] = 0xffffffffu;
        kmx[qi] = 0u;
      }
      for (int jj = 0; jj < te - tb; ++jj, ++g) {
        const int i = rotated_tile(tb, te, jj);
        const int acc = g & 1;
        if (!mbar_wait(&tfull[acc], (g >> 1) & 1, args.err, sm.abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t tbase = tmem_base + acc * kBN + qh * QPW * H + lane_off;
        float res[QPW];
        // two 32-column loads in flight per wait
#pragma unroll
        for (int c0 = 0; c0 < QPW * H / 32; c0 += 2) {
          float v[2][32];
          tmem_ld32(tbase + c0 * 32, v[0]);
          tmem_ld32(tbase + (c0 + 1) * 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int c = c0 + u;           // 32-column group: query c*32/H, heads (c*32) mod H ..
            const float4* w4 = reinterpret_cast<const float4*>(wk + c * 32);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int h4 = 0; h4 < 8; ++h4) {
              const float4 ww = w4[h4];
              s0 = fmaf(ww.x, fmaxf(v[u][4 * h4 + 0], 0.f), s0);
              s1 = fmaf(ww.y, fmaxf(v[u][4 * h4 + 1], 0.f), s1);
              s0 = fmaf(ww.z, fmaxf(v[u][4 * h4 + 2], 0.f), s0);
              s1 = fmaf(ww.w, fmaxf(v[u][4 * h4 + 3], 0.f), s1);
            }
            const int qi = (c * 32) / H;
            if ((c * 32) % H == 0) res[qi] = s0 + s1;
            else res[qi] += s0 + s1;
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[acc]);
        const int a = i * kBM + row_in_tile;
        const float sc = a < args.nA && args.row_scale ? args.row_scale[a] : 1.f;
        if (a < args.nA) {
#pragma unroll
          for (int qi = 0; qi < QPW; ++qi) {
            const int q = q0 + qh * QPW + qi;
            if (q < args.T) {
              float v = res[qi] * sc;
              if (args.causal && args.a_pos0 + a > args.q_pos0 + q) v = -INFINITY;
              args.out[static_cast<int64_t>(q) * args.ld_out + a] = v;
            }
          }
        }
        // running per-query score range (order-preserving keys) over the
        // item's rows; reduced once at the end of the item
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const uint32_t key = f2key(res[qi] * sc);
          const bool ok = a < args.nA;
          kmn[qi] = ok && key < kmn[qi] ? key : kmn[qi];
          kmx[qi] = ok && key > kmx[qi] ? key : kmx[qi];
        }
      }
      mbar_arrive(&bempty[b]);  // done with this item's weights
      // (after an aborted wait the warp skips the range: the call reports
      // the timeout and its outputs are not used)
      if (__all_sync(0xffffffffu, ok) && args.row_kmin) {
#pragma unroll
        for (int qi = 0; qi < QPW; ++qi) {
          const int q = q0 + qh * QPW + qi;
          const uint32_t mn = __reduce_min_sync(0xffffffffu, kmn[qi]);
          const uint32_t mx = __reduce_max_sync(0xffffffffu, kmx[qi]);
          // one slot per (query, lane quarter): a plain store when this item
          // is the query's only one, else an atomic into a pre-set slot
          if (lane == 0 && q < args.T) {
            uint32_t* pmn = args.row_kmin + static_cast<int64_t>(q) * 4 + quarter;
            uint32_t* pmx = args.row_kmax + static_cast<int64_t>(q) * 4 + quarter;
            if (im.apc >= im.n_atiles) {
              *pmn = mn;
              *pmx = mx;
            } else {
              atomicMin(pmn, mn);
              atomicMax(pmx, mx);
            }
          }
        }
      }
      ++k;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------- SIMT path
// Block: 64 A rows x 16 queries; thread (ty, tx) computes 4 rows x 1 query.
constexpr int kSimtRows = 64;
constexpr int kSimtQ = 16;

__global__ void __launch_bounds__(256) k_scores_simt(const void* A, int a_dtype, const void* Q,
                                                     int q_is_bf16, int d, int H, ScoreArgs args) {
  extern __shared__ float sh[];
  float* sq = sh;                    // [kSimtQ][H][d]
  float* sa = sh + kSimtQ * H * d;   // [kSimtRows][d]
  const int a0 = blockIdx.x * kSimtRows;
  const int qb = blockIdx.y * kSimtQ;
  for (int i = threadIdx.x; i < kSimtQ * H * d; i += blockDim.x) {
    int qi = i / (H * d);
    int q = qb + qi;
    float v = 0.f;
    if (q < args.T) {
      int64_t off = static_cast<int64_t>(q) * H * d + (i % (H * d));
      v = q_is_bf16 ? bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(Q)[off])
                    : reinterpret_cast<const float*>(Q)[off];
    }
    sq[i] = v;
  }
  for (int i = threadIdx.x; i < kSimtRows * d; i += blockDim.x) {
    int r = i / d;
    int a = a0 + r;
    sa[i] = (a < args.nA) ? key_elem(A, a_dtype, a, d, i % d) : 0.f;
  }
  __syncthreads();
  const int qi = threadIdx.x % kSimtQ;
  const int rg = threadIdx.x / kSimtQ;  // 0..15 -> rows rg*4 .. rg*4+3
  const int q = qb + qi;
  if (q >= args.T) return;
  for (int rr = 0; rr < 4; ++rr) {
    const int r = rg * 4 + rr;
    const int a = a0 + r;
    if (a >= args.nA) continue;
    float s = 0.f;
    for (int h = 0; h < H; ++h) {
      const float* qh = sq + (qi * H + h) * d;
      const float* ar = sa + r * d;
      float dot = 0.f;
      for (int i = 0; i < d; ++i) dot = fmaf(qh[i], ar[i], dot);
      s = fmaf(args.w[static_cast<int64_t>(q) * H + h], fmaxf(dot, 0.f), s);
    }
    if (args.row_scale) s *= args.row_scale[a];
    if (args.causal && args.a_pos0 + a > args.q_pos0 + q) s = -INFINITY;
    args.out[static_cast<int64_t>(q) * args.ld_out + a] = s;
  }
}

}  // namespace

int scores_smem_bytes() { return kSmemBytes; }

int scores_tiles_per_item(int64_t nA, int T, int H, int num_sms) {
  // one A range per query block unless there are too few query blocks to
  // give every CTA several items
  const int64_t atiles = (nA + kBM - 1) / kBM;
  const int64_t n_qb = (T + (kBN / H) - 1) / (kBN / H);
  int64_t ranges = (4 * static_cast<int64_t>(num_sms) + n_qb - 1) / n_qb;
  ranges = ranges < 1 ? 1 : (ranges > atiles ? atiles : ranges);
  const int64_t apc = (atiles + ranges - 1) / ranges;
  return static_cast<int>(apc < 1 ? 1 : apc);
}

cudaError_t launch_scores_tc(const CUtensorMap& mapA, const CUtensorMap& mapB, int H,
                             const ScoreArgs& args, int a_tiles_per_cta, cudaStream_t st) {
  ScoreArgs a = args;
  if (a.T <= 0 || a.nA <= 0) return cudaSuccess;
  if (a_tiles_per_cta < 1) return cudaErrorInvalidValue;
  // the head weights are fetched by a bulk copy: 16-byte aligned source
  if (reinterpret_cast<uintptr_t>(a.w) % 16 != 0) return cudaErrorMisalignedAddress;
  a.a_tiles_per_cta = a_tiles_per_cta;
  const int QPT = kBN / H;
  const int64_t n_atiles = (a.nA + kBM - 1) / kBM;
  const int64_t n_items = (n_atiles + a_tiles_per_cta - 1) / a_tiles_per_cta * ((a.T + QPT - 1) / QPT);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = static_cast<int>(n_items < sms ? n_items : sms);
  if (H == 32) {
    cudaFuncSetAttribute(k_scores_tc<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    count_launch();
    k_scores_tc<32><<<grid, kThreads, kSmemBytes, st>>>(mapA, mapB, a);
  } else if (H == 64) {
    cudaFuncSetAttribute(k_scores_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    count_launch();
    k_scores_tc<64><<<grid, kThreads, kSmemBytes, st>>>(mapA, mapB, a);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_scores_simt(const void* A, int a_dtype, const void* Q, int q_is_bf16, int d,
                               int H, const ScoreArgs& args, cudaStream_t st) {
  size_t smem = static_cast<size_t>(kSimtQ * H * d + kSimtRows * d) * sizeof(float);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  cudaFuncSetAttribute(k_scores_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  int64_t last = args.nA;
  if (args.causal) {
    int64_t alast = args.q_pos0 + args.T - 1 - args.a_pos0 + 1;
    if (alast < last) last = alast < 0 ? 0 : alast;
  }
  if (last <= 0 || args.T <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>((last + kSimtRows - 1) / kSimtRows), (args.T + kSimtQ - 1) / kSimtQ);
  count_launch();
  k_scores_simt<<<grid, 256, smem, st>>>(A, a_dtype, Q, q_is_bf16, d, H, args);
  return cudaGetLastError();
}

}  // namespace aiidx
