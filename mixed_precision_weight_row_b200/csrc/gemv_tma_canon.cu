// Decode linear on the per-tile TMA kernel: the canonical-layout dispatch
// (compiled apart from the paired one, in parallel).
#include "gemv_tma_dispatch.cuh"

namespace mpw {

cudaError_t tma_dispatch_canonical(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits,
                                   int N, int K, uint16_t* y, bool norm, bool pdl, int flags, int32_t* err,
                                   cudaStream_t stream) {
  return tma_layout<false>(x, M, packed, scales, bits, N, K, y, norm, pdl, flags, err, stream);
}

}  // namespace mpw
