// Re-ordering of packed rows between the canonical layout and the
// paired-halves layout that the decode kernels read fastest.
//
// Canonical: code k of a row occupies bits [k*b, k*b+b) of the row read as a
// little-endian integer (DynaQuant, "Status": bit pack / unpack; the bit
// order is this library's reading).  Paired halves (K % 32 == 0): in each
// group of 32 codes the even codes form one b-bit stream and the odd codes
// another; word h of the group holds half-word h of the even stream in its
// low 16 bits and half-word h of the odd stream in its high 16 bits.  Both
// layouts give a group exactly b words at word offset g*b of the row and the
// same row stride, so the re-ordering is a permutation of the bits inside
// each group and may run in place.
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "mpw_internal.h"

namespace mpw {
namespace {

constexpr int kRThreads = 256;

// Code j's b-bit field (two's complement bits, not sign-extended).
template <int B, bool PAIRED, int J>
__device__ __forceinline__ uint32_t field_of(const uint32_t (&w)[B + 1]) {
  constexpr uint32_t mask = (1u << B) - 1u;
  if constexpr (PAIRED) {
    constexpr int o = (J >> 1) * B;
    constexpr int h = o >> 4, r = o & 15;
    const uint32_t win = __byte_perm(w[h], w[h + 1], (J & 1) ? 0x7632 : 0x5410);
    return (win >> r) & mask;
  } else {
    constexpr int o = J * B;
    constexpr int i = o >> 5, r = o & 31;
    return (r == 0 ? w[i] : __funnelshift_r(w[i], w[i + 1], r)) & mask;
  }
}

// Writes code j's field u into the group's words of the given layout.
template <int B, bool PAIRED, int J>
__device__ __forceinline__ void put_field(uint32_t (&o)[B + 1], uint32_t u) {
  if constexpr (PAIRED) {
    constexpr int off = (J >> 1) * B;
    constexpr int h = off >> 4, r = off & 15;
    constexpr int sh = 16 * (J & 1);
    o[h] |= ((u << r) & 0xFFFFu) << sh;
    if constexpr (r + B > 16) o[h + 1] |= (u >> (16 - r)) << sh;
  } else {
    constexpr int off = J * B;
    constexpr int i = off >> 5, r = off & 31;
    o[i] |= u << r;
    if constexpr (r + B > 32) o[i + 1] |= u >> (32 - r);
  }
}

template <int B, bool TO_PAIRED, int... J>
__device__ __forceinline__ void move_all(const uint32_t (&w)[B + 1], uint32_t (&o)[B + 1],
                                         std::integer_sequence<int, J...>) {
  (put_field<B, TO_PAIRED, J>(o, field_of<B, !TO_PAIRED, J>(w)), ...);
}

// One thread per (row, 32-code group); the thread of a row's last group also
// zeroes the row's padding words.
template <int B, bool TO_PAIRED>
__global__ void __launch_bounds__(kRThreads)
repack_kernel(const uint32_t* in, uint32_t* out, int64_t N, int G, int rw) {
  const int64_t total = N * G;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = idx / G;
    const int g = static_cast<int>(idx - n * G);
    const uint32_t* src = in + n * rw + static_cast<int64_t>(g) * B;
    uint32_t w[B + 1], o[B + 1];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      w[i] = src[i];
      o[i] = 0u;
    }
    w[B] = 0u;
    o[B] = 0u;
    move_all<B, TO_PAIRED>(w, o, std::make_integer_sequence<int, 32>{});
    uint32_t* dst = out + n * rw + static_cast<int64_t>(g) * B;
#pragma unroll
    for (int i = 0; i < B; ++i) dst[i] = o[i];
    if (g == G - 1)
      for (int i = G * B; i < rw; ++i) out[n * rw + i] = 0u;
  }
}

template <int B>
cudaError_t run_repack(const uint8_t* in, int64_t N, int64_t K, uint8_t* out, bool to_paired,
                       cudaStream_t stream) {
  const int rw = static_cast<int>(row_words(K, B));
  const int G = static_cast<int>(K / 32);
  const int64_t work = N * G;
  const int64_t cap = static_cast<int64_t>(device_info().num_sms) * 16;
  int64_t blocks = (work + kRThreads - 1) / kRThreads;
  blocks = blocks < 1 ? 1 : (blocks > cap ? cap : blocks);
  const uint32_t* src = reinterpret_cast<const uint32_t*>(in);
  uint32_t* dst = reinterpret_cast<uint32_t*>(out);
  if (to_paired)
    repack_kernel<B, true><<<static_cast<unsigned>(blocks), kRThreads, 0, stream>>>(src, dst, N, G, rw);
  else
    repack_kernel<B, false><<<static_cast<unsigned>(blocks), kRThreads, 0, stream>>>(src, dst, N, G, rw);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_repack(const uint8_t* in, int64_t N, int64_t K, int bits, uint8_t* out, bool to_paired,
                          cudaStream_t stream) {
  switch (bits) {
    case 4: return run_repack<4>(in, N, K, out, to_paired, stream);
    case 5: return run_repack<5>(in, N, K, out, to_paired, stream);
    case 6: return run_repack<6>(in, N, K, out, to_paired, stream);
    case 7: return run_repack<7>(in, N, K, out, to_paired, stream);
    case 8: return run_repack<8>(in, N, K, out, to_paired, stream);
    case 9: return run_repack<9>(in, N, K, out, to_paired, stream);
    case 10: return run_repack<10>(in, N, K, out, to_paired, stream);
    case 11: return run_repack<11>(in, N, K, out, to_paired, stream);
    case 12: return run_repack<12>(in, N, K, out, to_paired, stream);
    case 13: return run_repack<13>(in, N, K, out, to_paired, stream);
    case 14: return run_repack<14>(in, N, K, out, to_paired, stream);
    case 15: return run_repack<15>(in, N, K, out, to_paired, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mpw
