// Exhaustive top-k selection that allocates no memory.
//
// Some callers cannot call cudaMalloc: an inference server or framework
// that hands out all device memory from its own pre-reserved pool (a stray
// cudaMalloc would sit outside that pool's accounting and can fail once the
// pool has taken the device), or a latency-critical path that must not hit
// the implicit device synchronisation cudaMalloc/cudaFree can cause.  This
// variant of ai_select_exhaustive keeps its only scratch (the rows of
// indexer scores) in a fixed, file-scope device array that every process
// loading the library holds until it exits, and computes the same result
// with the same kernels as the handle-based call, on keys the caller owns.
#include <cudaTypedefs.h>

#include <mutex>
#include <string>

#include "../../include/ai_index.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// 16 MiB of score rows (4 Mi floats); 256 bytes in front hold the device
// error word.  Shared by every call on the device.
constexpr size_t kScratchFloats = size_t(1) << 22;
constexpr int64_t kMaxKeys = int64_t(1) << 20;  // 4 score rows per pass at the maximum
__device__ __align__(256) float g_noalloc_scratch[64 + kScratchFloats];

std::mutex g_mu;
float* g_scratch_ptr[128] = {};

int fail_na(int code, const char* msg) {
  aiidx::set_last_error(msg);
  return code;
}

// Device address of the static scratch for the current device, looked up
// once per device (host code cannot use the symbol itself as a pointer).
int scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128)
    return fail_na(AI_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return fail_na(AI_ERR_CUDA, "cudaGetSymbolAddress failed");
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return AI_OK;
}

bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int ai_select_exhaustive_noalloc(const void* keys_dev, int32_t key_dtype, int64_t n_keys,
                                            int32_t d, int32_t H, const void* q_dev, const float* w_dev,
                                            int64_t pos0, int32_t T, int32_t k, int32_t* out_dev,
                                            float* out_scores_dev, int32_t* status_dev,
                                            void* cuda_stream) {
  using namespace aiidx;
  const bool tc = key_dtype == AI_BF16 && d == 128 && (H == 32 || H == 64);
  const bool simt = key_dtype == AI_FP32 && d > 0 && d % 8 == 0 && H > 0 && H <= 64 &&
                    static_cast<size_t>(16 * H * d + 64 * d) * 4 <= 200 * 1024;
  if (!keys_dev || !q_dev || !w_dev || !out_dev) return fail_na(AI_ERR_ARG, "null pointer argument");
  if (!tc && !simt)
    return fail_na(AI_ERR_ARG, "keys must be bf16 (d = 128, H in {32, 64}) or fp32 (queries of the same type)");
  if (n_keys <= 0 || n_keys > kMaxKeys) return fail_na(AI_ERR_ARG, "n_keys must be in [1, 1048576] (static scratch)");
  if (T <= 0 || k <= 0 || pos0 < 0) return fail_na(AI_ERR_ARG, "bad T, k or pos0");
  if (k > kRowTopkMaxK) return fail_na(AI_ERR_ARG, "k above 4096");
  if (pos0 + T > n_keys) return fail_na(AI_ERR_CAUSALITY, "query positions beyond the keys");
  if (tc && (reinterpret_cast<uintptr_t>(q_dev) % 16 != 0 || reinterpret_cast<uintptr_t>(w_dev) % 16 != 0))
    return fail_na(AI_ERR_ARG, "q_dev and w_dev must be 16-byte aligned (bf16 keys)");
  float* scratch = nullptr;
  int rc = scratch_for_current_device(&scratch);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int* err = reinterpret_cast<int*>(scratch);  // error word in the first 256 bytes
  float* rows = scratch + 64;
  // the only state that must start at zero
  if (cudaMemsetAsync(err, 0, sizeof(int), st) != cudaSuccess) return fail_na(AI_ERR_CUDA, "memset failed");
  const int64_t ld = (n_keys + 3) / 4 * 4;
  const int64_t per_pass = static_cast<int64_t>(kScratchFloats) / ld;
  const size_t qrow = static_cast<size_t>(H) * d * (tc ? 2 : 4);
  for (int64_t b0 = 0; b0 < T; b0 += per_pass) {
    const int tb = static_cast<int>(per_pass < T - b0 ? per_pass : T - b0);
    const void* qb = static_cast<const uint8_t*>(q_dev) + b0 * qrow;
    const float* wb = w_dev + b0 * H;
    const int64_t nA = pos0 + b0 + tb < n_keys ? pos0 + b0 + tb : n_keys;
    ScoreArgs sa{};
    sa.nA = static_cast<int>(nA);
    sa.T = tb;
    sa.w = wb;
    sa.row_scale = nullptr;
    sa.out = rows;
    sa.ld_out = ld;
    sa.causal = 1;
    sa.a_pos0 = 0;
    sa.q_pos0 = pos0 + b0;
    sa.err = err;
    cudaError_t e;
    if (tc) {
      CUtensorMap ma, mb;
      if (!map_rows(&ma, keys_dev, nA, 128) || !map_rows(&mb, qb, static_cast<int64_t>(tb) * H, 256))
        return fail_na(AI_ERR_CUDA, "tensor map encoding failed");
      int sms = 148;
      int dev = 0;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      e = launch_scores_tc(ma, mb, H, sa, scores_tiles_per_item(nA, tb, H, sms), st);
    } else {
      e = launch_scores_simt(keys_dev, KD_FP32, qb, 0, d, H, sa, st);
    }
    if (e != cudaSuccess) return fail_na(AI_ERR_CUDA, cudaGetErrorString(e));
    RowTopkArgs ta{};
    ta.scores = rows;
    ta.ld = ld;
    ta.T = tb;
    ta.q_pos0 = pos0 + b0;
    ta.n_keys = n_keys;
    ta.k = k;
    ta.out = out_dev + b0 * k;
    ta.out_scores = out_scores_dev ? out_scores_dev + b0 * k : nullptr;
    ta.err = err;
    e = launch_row_topk(ta, st);
    if (e != cudaSuccess) return fail_na(AI_ERR_CUDA, cudaGetErrorString(e));
  }
  // the call's device flags (bounded-wait timeout, range, capacity) go to
  // the caller's status word, in stream order: a 4-byte device-to-device
  // copy, no allocation
  if (status_dev &&
      cudaMemcpyAsync(status_dev, err, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return fail_na(AI_ERR_CUDA, "status copy failed");
  return AI_OK;
}
