// Decode linear for M <= 32 tokens on the per-tile TMA kernel of
// gemv_tma.cuh: the paired-layout dispatch and the C-level entry.
#include "gemv_tma_dispatch.cuh"

namespace mpw {

cudaError_t tma_dispatch_paired(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits,
                                int N, int K, uint16_t* y, bool norm, bool pdl, int flags, int32_t* err,
                                cudaStream_t stream) {
  return tma_layout<true>(x, M, packed, scales, bits, N, K, y, norm, pdl, flags, err, stream);
}

bool gemv_tma_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm) {
  // TMA of x needs a 16-byte aligned base and a row pitch that is a multiple
  // of 16 bytes
  return M >= 1 && M <= 32 && (!norm || M <= kNormMaxM) && N >= 1 && K >= 1 && N < (1 << 30) &&
         K % 8 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 && tensor_map_encoder() != nullptr;
}

cudaError_t launch_gemv_tma(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, bool pdl,
                            unsigned qflags, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  int32_t* err = device_error_word();
  const bool x_ready = (qflags & kQlinearXReady) != 0;
  const int flags = (x_ready ? kXReady : 0) | (x_ready && (qflags & kQlinearYFree) ? kYFree : 0);
  if (layout == kLayoutPaired)
    return tma_dispatch_paired(x, m, packed, scales, bits, n, k, y, norm, pdl, flags, err, stream);
  return tma_dispatch_canonical(x, m, packed, scales, bits, n, k, y, norm, pdl, flags, err, stream);
}

}  // namespace mpw
