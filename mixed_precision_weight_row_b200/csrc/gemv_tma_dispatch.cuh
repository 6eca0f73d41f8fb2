// Dispatch of the per-tile decode kernel over bit widths, token tiles, row
// tiles and input kinds, for one packed layout (included by gemv_tma.cu and
// gemv_tma_canon.cu, one layout each, so the two compile in parallel).
#pragma once

#include "gemv_tma.cuh"

namespace mpw {
namespace {

// 16-row tiles per CTA for a pass of M tokens: with several tokens the x
// chunks of a stage are as large as its weights or larger, and tiles that
// share them save that traffic (MPW_GEMV_RT sets it in a tuning build).
// M = 1 takes the one-token build, always with one tile.
inline int row_tiles_for(int M) {
  static const int forced = [] {
    const char* e = tuning_env("MPW_GEMV_RT");
    const int v = e ? atoi(e) : 0;
    return (v == 1 || v == 2 || v == 4) ? v : 0;
  }();
  if (forced > 0) return forced;
  // measured on 4096x4096 (b = 4, 6) and the 27B-class gate/down matrices:
  // two tiles win from M = 4 to 32 (e.g. M = 8, b = 6: 48 -> 55% of HBM),
  // four lose (too few CTAs per SM to hide latency; built in tuning builds
  // only)
  return M == 1 ? 1 : 2;
}

// 128-code chunks per ring stage for a pass of M tokens: eight, or four when
// the x chunks make stages so large that shared memory holds few CTAs
// (MPW_GEMV_SC sets it in a tuning build).
inline int stage_chunks_for(int M) {
  static const int forced = [] {
    const char* e = tuning_env("MPW_GEMV_SC");
    const int v = e ? atoi(e) : 0;
    return (v == 4 || v == 8) ? v : 0;
  }();
  if (forced > 0) return forced;
  // measured (two row tiles): four chunks from M = 4 (4096x4096 b = 6: M = 4
  // / 8 / 16 from 78 / 55 / 28 to 87 / 67 / 38% of HBM; gate 17408x5120 M = 8
  // from 59 to 66%, down 5120x17408 from 52 to 60%), where stages of eight
  // chunks leave shared memory for only two CTAs per SM
  return M >= 4 ? 4 : 8;
}

template <int B, bool PAIRED, int NT, int SC>
cudaError_t tma_rt_sc(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                      uint16_t* y, bool pdl, int flags, int32_t* err, cudaStream_t stream) {
  // fewer row tiles when a ring of two stages would not fit one CTA's shared
  // memory (wide codes with many tokens)
  const int rt = row_tiles_for(M);
  bool too_big = false;
#ifdef MPW_TUNING_KNOBS
  if (rt == 4) {
    const cudaError_t e = run_tma<B, NT, 0, PAIRED, false, 0, 4, SC>(x, M, packed, scales, N, K, y, pdl, flags,
                                                                      err, stream, 0, 0, &too_big);
    if (e != cudaSuccess || !too_big) return e;
  }
#endif
  if (rt >= 2) {
    const cudaError_t e = run_tma<B, NT, 0, PAIRED, false, 0, 2, SC>(x, M, packed, scales, N, K, y, pdl, flags,
                                                                      err, stream, 0, 0, &too_big);
    if (e != cudaSuccess || !too_big) return e;
  }
  return run_tma<B, NT, 0, PAIRED, false, 0, 1, SC>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
}

template <int B, bool PAIRED, int NT>
cudaError_t tma_rt(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                   uint16_t* y, bool pdl, int flags, int32_t* err, cudaStream_t stream) {
  if (stage_chunks_for(M) == 4)
    return tma_rt_sc<B, PAIRED, NT, 4>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  return tma_rt_sc<B, PAIRED, NT, 8>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
}

template <int B, bool PAIRED>
cudaError_t tma_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                     uint16_t* y, bool norm, bool pdl, int flags, int32_t* err, cudaStream_t stream) {
  // one token: the token count is a compile-time constant
  if (norm && M == 1) return run_tma<B, 1, 1, PAIRED, false, 1>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (norm) return run_tma<B, 1, kNormMaxM, PAIRED>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M == 1) return run_tma<B, 1, 0, PAIRED, false, 1>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M <= 8) return tma_rt<B, PAIRED, 1>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  if (M <= 16) return tma_rt<B, PAIRED, 2>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
  return tma_rt<B, PAIRED, 4>(x, M, packed, scales, N, K, y, pdl, flags, err, stream);
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

// The dispatch for one layout (defined in gemv_tma.cu for paired rows, in
// gemv_tma_canon.cu for canonical rows).
cudaError_t tma_dispatch_paired(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits,
                                int N, int K, uint16_t* y, bool norm, bool pdl, int flags, int32_t* err,
                                cudaStream_t stream);
cudaError_t tma_dispatch_canonical(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits,
                                   int N, int K, uint16_t* y, bool norm, bool pdl, int flags, int32_t* err,
                                   cudaStream_t stream);

}  // namespace mpw
