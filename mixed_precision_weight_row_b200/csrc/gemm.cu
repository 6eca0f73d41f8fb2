// Prefill GEMM on tcgen05 tensor cores (not built yet: every shape goes to
// the decode kernel).
#include <cuda_runtime.h>
#include <stdint.h>

#include "mpw_internal.h"

namespace mpw {

bool gemm_supported(int64_t, int64_t, int64_t) { return false; }

cudaError_t launch_gemm(const uint16_t*, const uint8_t*, const float*, int, int64_t, int64_t,
                        int64_t, uint16_t*, int32_t*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace mpw
