// Failure-path test hook: the bounded mbarrier wait used by the pipelined
// kernels, run against a barrier that never completes.  The wait gives up
// after the given number of polls, records DEV_ERR_TIMEOUT in a status word
// and the kernel returns normally, so the context stays usable and the host
// reads the status (nothing is in flight: the kernel issues no copies).
#include "../../include/ai_index.h"
#include "common.cuh"
#include "kernels.h"

namespace aiidx {
namespace {

__global__ void k_wait_timeout(int spin_limit, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);  // one arrival expected; none ever comes
  fence_mbar_init();
  bool done = false;
  for (int i = 0; i < spin_limit && !done; ++i) done = mbar_try_wait(&bar, 0);
  if (!done) atomicOr(status, DEV_ERR_TIMEOUT);
}

}  // namespace
}  // namespace aiidx

extern "C" int ai_debug_wait_timeout(int32_t spin_limit, int32_t* status_out, void* cuda_stream) {
  using namespace aiidx;
  if (!status_out || spin_limit < 1 || spin_limit > (1 << 26)) {
    set_last_error("spin_limit must be in [1, 2^26] and status_out non-null");
    return AI_ERR_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int* status = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void**>(&status), sizeof(int), st) != cudaSuccess) {
    set_last_error("cudaMallocAsync failed");
    return AI_ERR_CUDA;
  }
  cudaMemsetAsync(status, 0, sizeof(int), st);
  count_launch();
  k_wait_timeout<<<1, 32, 0, st>>>(spin_limit, status);
  int host = 0;
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFreeAsync(status, st);
  if (e != cudaSuccess) {
    set_last_error(cudaGetErrorString(e));
    return AI_ERR_CUDA;
  }
  *status_out = host;
  return AI_OK;
}
