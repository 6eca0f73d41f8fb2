// Per-row symmetric INT-b quantization, canonical bit packing, unpacking and
// dequantization.
//
// Quantization tutorial (aiknowledge.cn), "How quantization works" and
// "Step 1: symmetric quantization": s = max|w| / Q with Q = 2^(b-1) - 1,
// q = round(w / s) with round half to even, a zero channel takes 1 / Q.
// DynaQuant, "Status": bit pack / unpack tools; "Custom kernel architecture":
// packed N-bit storage.
//
// Layout of the work: one CTA per weight row.  The row is staged once in
// shared memory (a single HBM read), reduced to its absolute maximum with warp
// shuffles, then each thread turns one group of 32 consecutive codes into
// exactly `B` 32-bit words (32 codes * B bits = B words), so no two threads
// ever touch the same output word.  The packed row is assembled in shared
// memory and written out with 16-byte stores.  Rows too long for shared
// memory take a two-pass variant that re-reads the row from L2.
#include <cuda_runtime.h>
#include <stdint.h>

#include "mpw_internal.h"

namespace mpw {
namespace {

constexpr int kQThreads = 256;

template <int B>
struct Code {
  static constexpr int Q = (1 << (B - 1)) - 1;
  static constexpr uint32_t MASK = (1u << B) - 1u;
};

// Shared-memory index of element k of a staged row: one pad word after every
// 32 elements, so that thread g reading element 32g+j hits bank (g+j) % 32.
__device__ __forceinline__ int padded(int k) { return k + (k >> 5); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// q = clamp(rint(fl32(w / s)), -Q, Q).  __fdiv_rn is the IEEE quotient and
// __float2int_rn rounds half to even; a NaN quotient (0 / 0 after the scale
// underflowed) converts to 0 and +-inf saturates before the clamp.
template <int B>
__device__ __forceinline__ uint32_t code_bits(float w, float s) {
  int q = __float2int_rn(__fdiv_rn(w, s));
  q = max(-Code<B>::Q, min(Code<B>::Q, q));
  return static_cast<uint32_t>(q) & Code<B>::MASK;
}

// Packs codes j = 0..31 of one group into B words, LSB-first.
template <int B, typename Load>
__device__ __forceinline__ void pack_group(float s, Load load, uint32_t (&w)[B]) {
#pragma unroll
  for (int i = 0; i < B; ++i) w[i] = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t u = code_bits<B>(load(j), s);
    const int o = j * B;
    const int i = o >> 5, r = o & 31;
    w[i] |= u << r;
    if (r + B > 32) w[i + 1] |= u >> (32 - r);
  }
}

template <int B>
__device__ __forceinline__ float row_scale(float m) {
  return m == 0.0f ? __fdiv_rn(1.0f, static_cast<float>(Code<B>::Q))
                   : __fdiv_rn(m, static_cast<float>(Code<B>::Q));
}

// Block-wide max over kQThreads threads; every thread gets the result.
__device__ __forceinline__ float block_max(float m, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  m = warp_max(m);
  if (lane == 0) red[warp] = m;
  __syncthreads();
  float v = lane < (kQThreads / 32) ? red[lane] : 0.0f;
  v = warp_max(v);
  __syncthreads();
  return v;
}

// STAGED: the row (and its packed image) lives in shared memory.
// Otherwise: two passes over global memory (row re-read mostly hits L2).
template <int B, bool STAGED>
__global__ void __launch_bounds__(kQThreads)
quantize_pack_kernel(const float* __restrict__ W, int K, int rw, uint8_t* __restrict__ packed,
                     float* __restrict__ scales, int32_t* __restrict__ flag, bool vec4) {
  extern __shared__ __align__(16) float qsmem[];
  __shared__ float red[kQThreads / 32];
  const int n = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = W + static_cast<size_t>(n) * K;
  uint32_t* out_g = reinterpret_cast<uint32_t*>(packed + static_cast<size_t>(n) * rw * 4);
  const int G = (K + 31) >> 5;

  float* srow = qsmem;
  const int pad_floats = ((K + G + 3) & ~3);
  uint32_t* sout = reinterpret_cast<uint32_t*>(qsmem + pad_floats);

  // ---- pass 1: |w| max (and the row into shared memory) ----
  float m = 0.0f;
  bool bad = false;
  if (vec4) {
    const float4* r4 = reinterpret_cast<const float4*>(row);
    for (int k4 = tid; k4 < (K >> 2); k4 += kQThreads) {
      const float4 v = __ldg(r4 + k4);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
      bad |= !(isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w));
      if (STAGED) {
        const int k = k4 << 2;
        srow[padded(k)] = v.x;
        srow[padded(k + 1)] = v.y;
        srow[padded(k + 2)] = v.z;
        srow[padded(k + 3)] = v.w;
      }
    }
  } else {
    for (int k = tid; k < K; k += kQThreads) {
      const float v = __ldg(row + k);
      m = fmaxf(m, fabsf(v));
      bad |= !isfinite(v);
      if (STAGED) srow[padded(k)] = v;
    }
  }
  if (bad && flag != nullptr) *flag = 1;
  m = block_max(m, red);  // includes the barrier that publishes srow
  const float s = row_scale<B>(m);
  if (tid == 0) scales[n] = s;

  // ---- pass 2: codes -> words ----
  for (int g = tid; g < G; g += kQThreads) {
    uint32_t w[B];
    const int k0 = g << 5;
    if (STAGED) {
      pack_group<B>(s, [&](int j) { return (k0 + j < K) ? srow[padded(k0 + j)] : 0.0f; }, w);
    } else {
      pack_group<B>(s, [&](int j) { return (k0 + j < K) ? __ldg(row + k0 + j) : 0.0f; }, w);
    }
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int idx = g * B + i;
      if (idx < rw) {
        if (STAGED) sout[idx] = w[i];
        else out_g[idx] = w[i];
      }
    }
  }
  // zero the words past the last group (padding up to the 16-byte row stride)
  for (int idx = G * B + tid; idx < rw; idx += kQThreads) {
    if (STAGED) sout[idx] = 0u;
    else out_g[idx] = 0u;
  }
  if (STAGED) {
    __syncthreads();
    const uint4* s4 = reinterpret_cast<const uint4*>(sout);
    uint4* o4 = reinterpret_cast<uint4*>(out_g);
    for (int i = tid; i < (rw >> 2); i += kQThreads) o4[i] = s4[i];
  }
}

// ---------------------------------------------------------------------------
// group-wise scales: one scale per g consecutive weights of a row
// ---------------------------------------------------------------------------

// Quantization tutorial, exercises, item 1 (one scale per 128 weights; 32,
// 64, 128 and 256 compared), with the per-channel formula of "How
// quantization works" applied to each group.  One warp covers 1024
// consecutive weights of a row: lane l quantizes the 32-code unit l (its 32
// weights in registers) into exactly B words.  A group is 1 << gu_log2 units
// (g = 32 .. 1024, a power of two), so groups never straddle warps and a
// group's maximum is a butterfly over its lanes.  Units past K hold zeros.
template <int B>
__global__ void __launch_bounds__(256)
quantize_pack_groups_kernel(const float* __restrict__ W, int64_t N, int K, int rw, int gu_log2, int G,
                            uint8_t* __restrict__ packed, float* __restrict__ scales,
                            int32_t* __restrict__ flag, bool vec4) {
  const int lane = threadIdx.x & 31;
  const int U = (K + 31) >> 5;           // 32-code units per row
  const int wpr = (U + 31) >> 5;         // warps per row
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  if (wid >= N * wpr) return;            // the whole warp leaves together
  const int64_t n = wid / wpr;
  const int wr = static_cast<int>(wid - n * wpr);
  const int u = wr * 32 + lane;
  const int k0 = u * 32;
  const float* row = W + n * K;
  float v[32];
  if (vec4 && k0 + 32 <= K) {
    const float4* r4 = reinterpret_cast<const float4*>(row + k0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 t = __ldg(r4 + i);
      v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = (k0 + j < K) ? __ldg(row + k0 + j) : 0.0f;
  }
  float m = 0.0f;
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    m = fmaxf(m, fabsf(v[j]));
    bad |= !isfinite(v[j]);
  }
  if (bad && flag != nullptr) *flag = 1;
  for (int o = 1; o < (1 << gu_log2); o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const float s = row_scale<B>(m);
  if (u < U && (lane & ((1 << gu_log2) - 1)) == 0) scales[n * G + (u >> gu_log2)] = s;
  uint32_t w[B];
  pack_group<B>(s, [&](int j) { return v[j]; }, w);
  uint32_t* out = reinterpret_cast<uint32_t*>(packed + static_cast<size_t>(n) * rw * 4);
  if (u < U) {
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int idx = u * B + i;
      if (idx < rw) out[idx] = w[i];
    }
  }
  // zero the words past the last unit (padding up to the 16-byte row stride)
  if (wr == wpr - 1)
    for (int idx = U * B + lane; idx < rw; idx += 32) out[idx] = 0u;
}

// ---------------------------------------------------------------------------
// unpack / dequantize: one thread per group of 32 codes
// ---------------------------------------------------------------------------

template <int B>
__device__ __forceinline__ int extract_code(const uint32_t (&w)[B + 1], int j) {
  const int o = j * B;
  const int i = o >> 5, r = o & 31;
  const uint32_t t = (r + B <= 32) ? (w[i] >> r) : __funnelshift_r(w[i], w[i + 1], r);
  return static_cast<int>(t << (32 - B)) >> (32 - B);
}

template <int B, bool DEQ>
__global__ void __launch_bounds__(256)
unpack_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ scales, int64_t N,
              int K, int rw, int16_t* __restrict__ codes, float* __restrict__ w_hat) {
  const int G = (K + 31) >> 5;
  const int64_t total = N * G;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t n = t / G;
    const int g = static_cast<int>(t - n * G);
    const uint32_t* rowp = reinterpret_cast<const uint32_t*>(packed) + n * rw;
    uint32_t w[B + 1];
#pragma unroll
    for (int i = 0; i < B; ++i) {
      const int idx = g * B + i;
      w[i] = idx < rw ? __ldg(rowp + idx) : 0u;
    }
    w[B] = 0u;
    const float s = DEQ ? scales[n] : 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int k = (g << 5) + j;
      if (k < K) {
        const int q = extract_code<B>(w, j);
        if (DEQ) w_hat[n * K + k] = __fmul_rn(static_cast<float>(q), s);
        else codes[n * K + k] = static_cast<int16_t>(q);
      }
    }
  }
}

template <template <int> class F, typename... Args>
cudaError_t dispatch_bits(int bits, Args... args) {
  switch (bits) {
    case 4: return F<4>::run(args...);
    case 5: return F<5>::run(args...);
    case 6: return F<6>::run(args...);
    case 7: return F<7>::run(args...);
    case 8: return F<8>::run(args...);
    case 9: return F<9>::run(args...);
    case 10: return F<10>::run(args...);
    case 11: return F<11>::run(args...);
    case 12: return F<12>::run(args...);
    case 13: return F<13>::run(args...);
    case 14: return F<14>::run(args...);
    case 15: return F<15>::run(args...);
    default: return cudaErrorInvalidValue;
  }
}

// Shared-memory budget for staging one row: leaves room for two CTAs per SM
// at the largest rows of the 27B-class shapes (K = 17408 -> ~72 KB).
constexpr size_t kStageBudget = 200 * 1024;

template <int B>
struct QuantizeLaunch {
  static cudaError_t run(const float* W, int64_t N, int64_t K, uint8_t* packed, float* scales,
                         int32_t* flag, cudaStream_t stream) {
    const int rw = static_cast<int>(row_words(K, B));
    const int G = static_cast<int>((K + 31) / 32);
    const size_t pad_floats = (static_cast<size_t>(K) + G + 3) & ~static_cast<size_t>(3);
    const size_t smem = (pad_floats + rw) * 4;
    const bool vec4 = (K % 4 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
    const DeviceInfo& di = device_info();
    if (smem <= kStageBudget && smem <= static_cast<size_t>(di.max_smem_optin)) {
      auto kern = quantize_pack_kernel<B, true>;
      cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kStageBudget);
      if (e != cudaSuccess) return e;
      kern<<<static_cast<unsigned>(N), kQThreads, smem, stream>>>(W, static_cast<int>(K), rw, packed,
                                                                 scales, flag, vec4);
    } else {
      quantize_pack_kernel<B, false><<<static_cast<unsigned>(N), kQThreads, 0, stream>>>(
          W, static_cast<int>(K), rw, packed, scales, flag, vec4);
    }
    return cudaGetLastError();
  }
};

template <int B>
struct QuantizeGroupsLaunch {
  static cudaError_t run(const float* W, int64_t N, int64_t K, int64_t group, uint8_t* packed, float* scales,
                         int32_t* flag, cudaStream_t stream) {
    const int rw = static_cast<int>(row_words(K, B));
    int gl = 0;
    while ((int64_t{32} << gl) < group) ++gl;
    const int G = static_cast<int>((K + group - 1) / group);
    const int64_t wpr = ((K + 31) / 32 + 31) / 32;
    const int64_t blocks = (N * wpr * 32 + 255) / 256;
    const bool vec4 = (K % 4 == 0) && (reinterpret_cast<uintptr_t>(W) % 16 == 0);
    quantize_pack_groups_kernel<B><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        W, N, static_cast<int>(K), rw, gl, G, packed, scales, flag, vec4);
    return cudaGetLastError();
  }
};

unsigned grid_for(int64_t work, int threads) {
  const int64_t blocks = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_info().num_sms) * 16;
  return static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

template <int B>
struct UnpackLaunch {
  static cudaError_t run(const uint8_t* packed, const float* scales, int64_t N, int64_t K,
                         int16_t* codes, float* w_hat, cudaStream_t stream) {
    const int rw = static_cast<int>(row_words(K, B));
    const int64_t work = N * ((K + 31) / 32);
    if (w_hat != nullptr)
      unpack_kernel<B, true><<<grid_for(work, 256), 256, 0, stream>>>(packed, scales, N, static_cast<int>(K), rw,
                                                                      nullptr, w_hat);
    else
      unpack_kernel<B, false><<<grid_for(work, 256), 256, 0, stream>>>(packed, nullptr, N, static_cast<int>(K), rw,
                                                                       codes, nullptr);
    return cudaGetLastError();
  }
};

}  // namespace

cudaError_t launch_quantize_pack(const float* W, int64_t N, int64_t K, int bits, uint8_t* packed,
                                 float* scales, int32_t* flag, cudaStream_t stream) {
  return dispatch_bits<QuantizeLaunch>(bits, W, N, K, packed, scales, flag, stream);
}

cudaError_t launch_quantize_pack_groups(const float* W, int64_t N, int64_t K, int bits, int64_t group,
                                        uint8_t* packed, float* scales, int32_t* flag, cudaStream_t stream) {
  return dispatch_bits<QuantizeGroupsLaunch>(bits, W, N, K, group, packed, scales, flag, stream);
}

cudaError_t launch_unpack(const uint8_t* packed, int64_t N, int64_t K, int bits, int16_t* codes,
                          cudaStream_t stream) {
  return dispatch_bits<UnpackLaunch>(bits, packed, static_cast<const float*>(nullptr), N, K, codes,
                                     static_cast<float*>(nullptr), stream);
}

cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int64_t N, int64_t K,
                              int bits, float* W_hat, cudaStream_t stream) {
  return dispatch_bits<UnpackLaunch>(bits, packed, scales, N, K, static_cast<int16_t*>(nullptr), W_hat,
                                     stream);
}

}  // namespace mpw
