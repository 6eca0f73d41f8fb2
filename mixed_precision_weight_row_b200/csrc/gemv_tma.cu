// Decode linear for M <= 32 tokens on the per-tile TMA kernel of
// gemv_tma.cuh: dispatch over bit widths, token tiles and layouts, with one
// fp32 scale per row.
#include "gemv_tma.cuh"

namespace mpw {
namespace {

template <int B, bool PAIRED>
cudaError_t tma_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                     uint16_t* y, bool norm, bool pdl, int flags, int32_t* err, cudaStream_t stream) {
  // one token: the token count is a compile-time constant
  if (norm && M == 1) return run_tma<B, 1, 1, PAIRED, false, 1>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (norm) return run_tma<B, 1, kNormMaxM, PAIRED>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M == 1) return run_tma<B, 1, 0, PAIRED, false, 1>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M <= 8) return run_tma<B, 1, 0, PAIRED>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M <= 16) return run_tma<B, 2, 0, PAIRED>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  return run_tma<B, 4, 0, PAIRED>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
}

template <bool PAIRED>
cudaError_t tma_layout(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits, int N,
                       int K, uint16_t* y, bool norm, bool pdl, int flags, int32_t* err,
                       cudaStream_t stream) {
  switch (bits) {
    case 4: return tma_bits<4, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 5: return tma_bits<5, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 6: return tma_bits<6, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 7: return tma_bits<7, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 8: return tma_bits<8, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 9: return tma_bits<9, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 10: return tma_bits<10, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 11: return tma_bits<11, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 12: return tma_bits<12, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 13: return tma_bits<13, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 14: return tma_bits<14, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    case 15: return tma_bits<15, PAIRED>(x, M, packed, scales, N, K, y, norm, pdl, flags, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

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
    return tma_layout<true>(x, m, packed, scales, bits, n, k, y, norm, pdl, flags, err, stream);
  return tma_layout<false>(x, m, packed, scales, bits, n, k, y, norm, pdl, flags, err, stream);
}

}  // namespace mpw
