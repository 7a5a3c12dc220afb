// Self-test of the kernels' failure path: a bounded mbarrier wait that runs
// out reports SVDQ_ERR_TIMEOUT to the host and leaves the context usable.
// The wait is on a barrier that nothing arrives on, so it ends by its own
// limit (no fault, no trap, no unbounded spin).
#include "internal.h"
#include "ptx.cuh"

namespace svdq {
namespace {

__device__ int g_selftest_status;

__global__ void bounded_wait_selftest_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none is made
    abort_flag = 0;
    fence_mbar_init();
    const bool done = mbar_wait(&bar, 0, &abort_flag);
    g_selftest_status = done ? static_cast<int>(SVDQ_OK) : static_cast<int>(SVDQ_ERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace svdq

using namespace svdq;

extern "C" {

svdq_status svdq_selftest_bounded_wait(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (svdq_check_device(dev) != SVDQ_OK) return SVDQ_ERR_UNSUPPORTED_DEVICE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int init = -1;
  if (cudaMemcpyToSymbolAsync(g_selftest_status, &init, sizeof(int), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;
  int v = -1;
  if (cudaMemcpyFromSymbolAsync(&v, g_selftest_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SVDQ_ERR_CUDA;
  return v < 0 ? SVDQ_ERR_CUDA : static_cast<svdq_status>(v);
}

}  // extern "C"
