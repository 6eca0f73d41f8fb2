// Decode linear with group-wise scales: one fp32 scale per group of g
// consecutive codes of a row (g = 128, 256, 512 or 1024), on the per-tile
// TMA kernel of gemv_tma.cuh.
//   y[m, n] = bf16(sum_j s_nj * sum_{k in group j} x[m, k] * q[n, k])
//
// Quantization tutorial, exercises, item 1: one scale per 128 weights instead
// of one per channel (32, 64, 128 and 256 compared).  A 128-code chunk of the
// decode kernel lies inside one group when g is a multiple of 128, so the
// chunk's products are summed on their own (fp32, on the tensor cores) and
// enter the accumulator multiplied by the group's scale.  Smaller groups
// would split the four 32-code groups that one tensor-core step mixes; the
// quantizer takes them, this kernel does not.
#include "gemv_tma.cuh"

namespace mpw {
namespace {

template <int B, bool PAIRED>
cudaError_t grp_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                     uint16_t* y, int flags, int32_t* err, cudaStream_t stream, int gstride, int gshift) {
  if (M <= 8)
    return run_tma<B, 1, 0, PAIRED, true>(x, M, packed, scales, N, K, y, true, flags, err, stream, gstride, gshift);
  if (M <= 16)
    return run_tma<B, 2, 0, PAIRED, true>(x, M, packed, scales, N, K, y, true, flags, err, stream, gstride, gshift);
  return run_tma<B, 4, 0, PAIRED, true>(x, M, packed, scales, N, K, y, true, flags, err, stream, gstride, gshift);
}

template <bool PAIRED>
cudaError_t grp_layout(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits, int N,
                       int K, uint16_t* y, int flags, int32_t* err, cudaStream_t stream, int gstride, int gshift) {
  switch (bits) {
    case 4: return grp_bits<4, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 5: return grp_bits<5, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 6: return grp_bits<6, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 7: return grp_bits<7, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 8: return grp_bits<8, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 9: return grp_bits<9, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 10: return grp_bits<10, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 11: return grp_bits<11, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 12: return grp_bits<12, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 13: return grp_bits<13, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 14: return grp_bits<14, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    case 15: return grp_bits<15, PAIRED>(x, M, packed, scales, N, K, y, flags, err, stream, gstride, gshift);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool gemv_groups_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, int64_t group) {
  const bool pow2 = group >= 128 && group <= 1024 && (group & (group - 1)) == 0;
  return pow2 && M >= 1 && gemv_tma_supported(x, M < 32 ? M : 32, N, K, false);
}

cudaError_t launch_gemv_groups(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                               int64_t group, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                               cudaStream_t stream, unsigned qflags) {
  // MPW_QLINEAR_X_READY / _Y_UNSHARED as for the per-row decode kernel; with
  // more than one pass of 32 tokens the later passes follow a launch of the
  // same call, which writes another part of y and not x, so the flags hold
  const bool x_ready = (qflags & kQlinearXReady) != 0;
  const int flags = (x_ready ? kXReady : 0) | (x_ready && (qflags & kQlinearYFree) ? kYFree : 0);
  int gshift = 0;
  while ((static_cast<int64_t>(kChunk) << gshift) < group) ++gshift;
  const int gstride = static_cast<int>((K + group - 1) / group);
  int32_t* err = device_error_word();
  for (int64_t m0 = 0; m0 < M; m0 += 32) {
    const int mt = static_cast<int>(M - m0 < 32 ? M - m0 : 32);
    const cudaError_t e =
        layout == kLayoutPaired
            ? grp_layout<true>(x + m0 * K, mt, packed, scales, bits, static_cast<int>(N), static_cast<int>(K),
                               y + m0 * N, flags, err, stream, gstride, gshift)
            : grp_layout<false>(x + m0 * K, mt, packed, scales, bits, static_cast<int>(N), static_cast<int>(K),
                                y + m0 * N, flags, err, stream, gstride, gshift);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace mpw
