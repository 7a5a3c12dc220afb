// INT4 (group 64) variant of the 4-bit GEMM; see launch_gemm_int4.
#include "internal.h"

namespace svdq {

cudaError_t launch_gemm_int4(const svdq_weights*, const uint8_t*, const void*, const float*, int, void*, int,
                             cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace svdq
