// svdq_linear_forward_noalloc: the layer forward for callers that cannot
// allocate device memory (see include/svdq.h).  Its intermediates (codes,
// scales, lora_act) live in one file-scope device array instead of a
// caller-provided workspace; nothing here allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace svdq {
namespace {

// Maximum scratch of one call; svdq_workspace_bytes(w, M) must fit in it
// after the start is rounded up to 1024 bytes.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

// Shared by every call on a device; every GPU that loads this library keeps
// it until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDev = 64;
void* g_scratch_addr[kMaxDev] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the array for the current device.  The name of the
// array in host code is only a host-side stand-in, so the address comes
// from cudaGetSymbolAddress, looked up once per device with that device
// current (the first call on each device does this set-up).
svdq_status scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SVDQ_OK;
}

}  // namespace
}  // namespace svdq

extern "C" svdq_status svdq_linear_forward_noalloc(const svdq_weights* w, const uint16_t* X, int32_t M, float g_x,
                                                   void* Y, int32_t out_dtype, void* stream) {
  using namespace svdq;
  // the same argument errors as svdq_linear_forward, before the size check
  if (!w || w->desc.precision == SVDQ_AWQ_W4A16) return SVDQ_ERR_INVALID_ARG;
  if (M < 0) return SVDQ_ERR_SHAPE;
  if (M == 0) return SVDQ_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SVDQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDev) return SVDQ_ERR_INVALID_ARG;
  // the scratch used is the current device's copy of the array: the weights
  // must live on that device too
  if (w->device != dev) return SVDQ_ERR_INVALID_ARG;
  const size_t need = svdq_workspace_bytes(w, M);
  if (need == 0 || need + 1024 > kNoAllocScratchBytes) return SVDQ_ERR_WORKSPACE;
  svdq_status st = svdq_check_device(dev);
  if (st != SVDQ_OK) return st;
  void* base = nullptr;
  if ((st = scratch_address(dev, &base)) != SVDQ_OK) return st;
  // the forward wants a 1024-byte aligned workspace: round the start up
  const uintptr_t a = (reinterpret_cast<uintptr_t>(base) + 1023) & ~uintptr_t(1023);
  const size_t avail = kNoAllocScratchBytes - (a - reinterpret_cast<uintptr_t>(base));
  return svdq_linear_forward(w, X, M, g_x, Y, out_dtype, reinterpret_cast<void*>(a), avail, stream);
}
