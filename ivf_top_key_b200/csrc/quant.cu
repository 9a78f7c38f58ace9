// Storage-format kernels for fp8 key stores.
//
// Per-token scale = amax / 448 (float32), code = E4M3(key / scale) with
// round-to-nearest-even and saturation to +-448; an all-zero row gets scale
// 1.  The bf16 copy of codes (exact) feeds the bf16 tensor-core score GEMM;
// the scale is applied to the score, which is valid because ReLU commutes
// with a positive factor.
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

__global__ void k_quantize(const uint16_t* keys, int64_t n, int d, uint8_t* codes, float* scales) {
  const int64_t row = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n) return;
  const uint16_t* kr = keys + row * d;
  float amax = 0.f;
  for (int i = lane; i < d; i += 32) amax = fmaxf(amax, fabsf(bf16_bits_to_f32(kr[i])));
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  for (int i = lane; i < d; i += 32) {
    const float q = __fdiv_rn(bf16_bits_to_f32(kr[i]), scale);
    codes[row * d + i] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
  }
  if (lane == 0) scales[row] = scale;
}

__global__ void k_codes_to_bf16(const uint8_t* codes, int64_t n_elem, uint16_t* out) {
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n_elem;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    __nv_bfloat16 b = __float2bfloat16_rn(fp8_to_f32(codes[e]));
    out[e] = *reinterpret_cast<uint16_t*>(&b);
  }
}

}  // namespace

cudaError_t launch_quantize_fp8(const uint16_t* keys_bf16, int64_t n, int d, uint8_t* codes,
                                float* scales, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  const int64_t threads = n * 32;
  count_launch();
  k_quantize<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(keys_bf16, n, d, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_fp8_codes_to_bf16(const uint8_t* codes, int64_t n, int d, uint16_t* out,
                                     cudaStream_t st) {
  const int64_t e = n * d;
  if (e <= 0) return cudaSuccess;
  int64_t blocks = (e + 255) / 256;
  if (blocks > 65535 * 8) blocks = 65535 * 8;
  count_launch();
  k_codes_to_bf16<<<static_cast<unsigned>(blocks), 256, 0, st>>>(codes, e, out);
  return cudaGetLastError();
}

}  // namespace aiidx
