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
// tcgen05 path (bf16 rows, d = 128, H in {32, 64}): one CTA owns 256 / H
// queries, i.e. the whole N = 256 of one UMMA (query x head rows, K-major),
// loaded once by TMA, and streams 128-row A tiles through a 4-deep TMA ring.
// Warp 0 issues TMA, warp 1 owns TMEM and issues the UMMAs
// (M = 128, N = 256, K = 16 x 8) into one of two 256-column accumulators,
// warps 4-7 read the accumulator back (one TMEM lane = one A row per
// thread), apply ReLU and the head weights, and write 256 / H scores per
// row.  fp8 rows are given as bf16 copies of their codes; the per-row scale
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
constexpr int kStages = 4;
constexpr int kATile = kBM * kK * 2;  // 32 KiB
constexpr int kBTile = kBN * kK * 2;  // 64 KiB
constexpr int kThreads = 256;
constexpr int kSmemBytes = 1024 /*align slack*/ + kBTile + kStages * kATile + kBN * 4 + 256;

struct GemmSmem {
  uint8_t* b;        // [2 K-blocks][256 rows][128 B]
  uint8_t* a;        // kStages x [2 K-blocks][128 rows][128 B]
  float* w;          // [256]
  uint64_t* bars;    // bfull, afull[kStages], aempty[kStages], tfull[2], tempty[2]
  uint32_t* tmem;    // allocated TMEM base
  int* abort;
};

__device__ __forceinline__ GemmSmem carve(uint8_t* raw) {
  GemmSmem s;
  uint8_t* p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.b = p;
  s.a = p + kBTile;
  s.w = reinterpret_cast<float*>(s.a + kStages * kATile);
  s.bars = reinterpret_cast<uint64_t*>(s.w + kBN);
  s.tmem = reinterpret_cast<uint32_t*>(s.bars + 1 + 2 * kStages + 4);
  s.abort = reinterpret_cast<int*>(s.tmem + 1);
  return s;
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    k_scores_tc(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                ScoreArgs args) {
  constexpr int QPT = kBN / H;  // queries per CTA
  extern __shared__ uint8_t smem_raw[];
  GemmSmem sm = carve(smem_raw);
  uint64_t* bfull = sm.bars;
  uint64_t* afull = sm.bars + 1;
  uint64_t* aempty = sm.bars + 1 + kStages;
  uint64_t* tfull = sm.bars + 1 + 2 * kStages;
  uint64_t* tempty = sm.bars + 1 + 2 * kStages + 2;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.y * QPT;
  const int n_atiles = (args.nA + kBM - 1) / kBM;
  int t_begin = blockIdx.x * args.a_tiles_per_cta;
  int t_end = min(n_atiles, t_begin + args.a_tiles_per_cta);
  if (args.causal) {
    // last key row any query of this CTA may see
    int64_t qlast = args.q_pos0 + min(q0 + QPT, args.T) - 1;
    int64_t alast = qlast - args.a_pos0;
    int lim = alast < 0 ? 0 : static_cast<int>(alast / kBM) + 1;
    t_end = min(t_end, lim);
  }
  const int ntiles = t_end - t_begin;
  if (ntiles <= 0 || q0 >= args.T) return;

  if (threadIdx.x == 0) {
    mbar_init(bfull, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    *sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem, 512);
    tmem_relinquish();
  }
  // head weights of this CTA's queries (zero for queries past T)
  for (int j = threadIdx.x; j < kBN; j += kThreads) {
    int q = q0 + j / H;
    sm.w[j] = (q < args.T) ? args.w[static_cast<int64_t>(q0) * H + j] : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------- producer
      mbar_arrive_expect_tx(bfull, kBTile);
      tma_load_2d(sm.b, &mapB, 0, q0 * H, bfull);
      tma_load_2d(sm.b + kBN * 128, &mapB, 64, q0 * H, bfull);
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % kStages;
        const uint32_t ph = (i / kStages) & 1;
        if (i >= kStages && !mbar_wait(&aempty[s], ph ^ 1, args.err, sm.abort)) break;
        uint8_t* dst = sm.a + s * kATile;
        const int row = (t_begin + i) * kBM;
        mbar_arrive_expect_tx(&afull[s], kATile);
        tma_load_2d(dst, &mapA, 0, row, &afull[s]);
        tma_load_2d(dst + kBM * 128, &mapA, 64, row, &afull[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // --------------------------------------------------------- UMMA issue
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      if (mbar_wait(bfull, 0, args.err, sm.abort)) {
        const uint32_t sb = smem_u32(sm.b);
        for (int i = 0; i < ntiles; ++i) {
          const int s = i % kStages;
          const uint32_t ph = (i / kStages) & 1;
          const int acc = i & 1;
          const uint32_t aph = (i >> 1) & 1;
          if (!mbar_wait(&afull[s], ph, args.err, sm.abort)) break;
          if (i >= 2 && !mbar_wait(&tempty[acc], aph ^ 1, args.err, sm.abort)) break;
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
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int row_in_tile = (warp - 4) * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    for (int i = 0; i < ntiles; ++i) {
      const int acc = i & 1;
      const uint32_t aph = (i >> 1) & 1;
      if (!mbar_wait(&tfull[acc], aph, args.err, sm.abort)) break;
      tc_fence_after();
      float res[QPT];
      const uint32_t tbase = tmem_base + acc * kBN + lane_off;
#pragma unroll
      for (int qi = 0; qi < QPT; ++qi) {
        float sacc = 0.f;
#pragma unroll
        for (int c = 0; c < H / 32; ++c) {
          float v[32];
          tmem_ld32(tbase + qi * H + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) sacc = fmaf(sm.w[qi * H + c * 32 + j], fmaxf(v[j], 0.f), sacc);
        }
        res[qi] = sacc;
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      const int a = (t_begin + i) * kBM + row_in_tile;
      if (a < args.nA) {
        const float sc = args.row_scale ? args.row_scale[a] : 1.f;
#pragma unroll
        for (int qi = 0; qi < QPT; ++qi) {
          const int q = q0 + qi;
          if (q < args.T) {
            float v = res[qi] * sc;
            if (args.causal && args.a_pos0 + a > args.q_pos0 + q) v = -INFINITY;
            args.out[static_cast<int64_t>(q) * args.ld_out + a] = v;
          }
        }
      }
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

cudaError_t launch_scores_tc(const CUtensorMap& mapA, const CUtensorMap& mapB, int H,
                             const ScoreArgs& args, int a_tiles_per_cta, cudaStream_t st) {
  ScoreArgs a = args;
  a.a_tiles_per_cta = a_tiles_per_cta;
  const int QPT = kBN / H;
  const int n_atiles = (a.nA + kBM - 1) / kBM;
  dim3 grid((n_atiles + a_tiles_per_cta - 1) / a_tiles_per_cta, (a.T + QPT - 1) / QPT);
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
