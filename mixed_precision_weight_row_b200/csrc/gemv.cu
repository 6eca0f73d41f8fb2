// Decode GEMV: y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k]) for a few tokens.
//
// DynaQuant, "Custom kernel architecture": the packed N-bit weights are read
// from memory once, expanded in registers and multiplied; in decode the
// saving in bytes is the speedup because the layer is bandwidth-bound
// (quantization tutorial, closing note: decode is memory-bound).
//
// Code expansion (both kernels): one 32-code group of one row is exactly B
// 32-bit words of the packed stream.  A code is isolated with one funnel
// shift; its b-bit two's-complement field, sign bit flipped, is OR-ed into
// the mantissa of 2^23 (one LOP3) and one FADD removes 2^23 + 2^(b-1), which
// leaves the code as an exact fp32 integer.  Products accumulate in fp32 (four
// partial sums per row and token); the row scale is applied once, after the
// sum.
//
// gemv_xreg_kernel (K <= 32768, the decode shapes): lane l of warp w owns the
// group g = 32w + l of K for the whole kernel, so its 32 x values stay in
// registers.  A CTA (ceil(K/32) lanes) walks a contiguous range of rows in
// batches of 4, double-buffering the next batch's packed words in registers
// (vector loads, streaming cache hint) while it computes the current one;
// per-row partials are reduced with warp shuffles and one shared-memory pass.
//
// gemv_generic_kernel (any K): warps own rows, lanes walk the row; x is staged
// in shared memory (per K-chunk when it does not fit).
//
// With norm_input the output is scaled by r_m = 1 / sqrt(mean_k x^2 + 1e-6)
// (fp32, one fixed reduction order per kernel) after the dot product.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>

#include "mpw_internal.h"

namespace mpw {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr size_t kXSmemBudget = 150 * 1024;

__device__ __forceinline__ float bf16_bits_to_float(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Code j (0..31) of a group held in w[0..B-1] as an exact fp32 integer.
template <int B>
__device__ __forceinline__ float code_f32(const uint32_t (&w)[B + 1], int j) {
  const int o = j * B;
  const int i = o >> 5, r = o & 31;
  uint32_t t;
  if (r == 0) t = w[i];
  else if (r + B <= 32) t = w[i] >> r;
  else t = __funnelshift_r(w[i], w[i + 1], r);
  constexpr uint32_t kMask = (1u << B) - 1u;
  constexpr uint32_t kMagic = 0x4B000000u | (1u << (B - 1));  // 2^23, sign bit flip
  constexpr float kOffset = 8388608.0f + static_cast<float>(1 << (B - 1));
  return __uint_as_float((t & kMask) ^ kMagic) - kOffset;
}

// Float index of element (group gl, j) of one token in the transposed x tile.
__device__ __forceinline__ int xs_index(int gl, int j) {
  return (((gl >> 5) * 8 + (j >> 2)) * 32 + (gl & 31)) * 4 + (j & 3);
}

// Stage tokens [0, MT) of x, groups [gb, gb + gc) into xs (zeros past K / mt).
template <int MT, bool NORM>
__device__ __forceinline__ void stage_x(float* xs, const uint16_t* __restrict__ x, int ldx, int mt,
                                        int K, int gb, int gc, const float* inv_rms) {
  const int elems = gc * 32;
  for (int t = 0; t < MT; ++t) {
    float* dst = xs + t * elems;
    const uint16_t* src = x + static_cast<size_t>(t) * ldx;
    for (int idx = threadIdx.x; idx < elems; idx += kThreads) {
      const int k = gb * 32 + idx;
      float v = 0.0f;
      if (t < mt && k < K) {
        v = bf16_bits_to_float(__ldg(src + k));
      }
      dst[xs_index(idx >> 5, idx & 31)] = v;
    }
  }
}

// 1 / sqrt(mean(x^2) + 1e-6) per token, fp32, fixed reduction order (every
// CTA computes the same value bit for bit).
template <int MT>
__device__ void token_inv_rms(const uint16_t* __restrict__ x, int ldx, int mt, int K, float* out,
                              float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int t = 0; t < MT; ++t) {
    float ss = 0.0f;
    if (t < mt)
      for (int k = threadIdx.x; k < K; k += kThreads) {
        const float v = bf16_bits_to_float(__ldg(x + static_cast<size_t>(t) * ldx + k));
        ss = fmaf(v, v, ss);
      }
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
      float tot = 0.0f;
      for (int w = 0; w < kWarps; ++w) tot += red[w];
      out[t] = 1.0f / sqrtf(tot / static_cast<float>(K) + 1e-6f);
    }
    __syncthreads();
  }
}

template <int B, int R, int MT, bool NORM>
__global__ void __launch_bounds__(kThreads)
gemv_generic_kernel(const uint16_t* __restrict__ x, int mt, const uint8_t* __restrict__ packed,
            const float* __restrict__ scales, int N, int K, int rw, uint16_t* __restrict__ y,
            int gc, int num_tasks) {
  extern __shared__ __align__(16) float xs[];
  __shared__ float inv_rms[MT];
  __shared__ float red[kWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = (K + 31) >> 5;
  const int nchunks = (G + gc - 1) / gc;
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);

  if (NORM) token_inv_rms<MT>(x, K, mt, K, inv_rms, red);

  for (int task = blockIdx.x; task < num_tasks; task += gridDim.x) {
    const int row0 = (task * kWarps + warp) * R;
    float acc[R][MT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[r][t][a] = 0.0f;

    for (int c = 0; c < nchunks; ++c) {
      const int gb = c * gc;
      const int ge = min(G, gb + gc);
      if (nchunks > 1 || task == static_cast<int>(blockIdx.x)) {
        __syncthreads();
        stage_x<MT, NORM>(xs, x, K, mt, K, gb, gc, inv_rms);
        __syncthreads();
      }
      for (int g = gb + lane; g < ge; g += 32) {
        const int gl = g - gb;
        uint32_t w[R][B + 1];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int n = row0 + r;
          const uint32_t* rowp = pw + static_cast<size_t>(n) * rw + static_cast<size_t>(g) * B;
          const bool full = n < N && (g + 1) * B <= rw;
#pragma unroll
          for (int i = 0; i < B; ++i)
            w[r][i] = full ? __ldg(rowp + i) : ((n < N && g * B + i < rw) ? __ldg(rowp + i) : 0u);
          w[r][B] = 0u;
        }
        float xv[MT][32];
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const float4* x4 = reinterpret_cast<const float4*>(xs + t * gc * 32);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const float4 v = x4[((gl >> 5) * 8 + jj) * 32 + (gl & 31)];
            xv[t][4 * jj + 0] = v.x;
            xv[t][4 * jj + 1] = v.y;
            xv[t][4 * jj + 2] = v.z;
            xv[t][4 * jj + 3] = v.w;
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) {
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const float q = code_f32<B>(w[r], j);
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[r][t][j & 3] = fmaf(xv[t][j], q, acc[r][t][j & 3]);
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int n = row0 + r;
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        float v = (acc[r][t][0] + acc[r][t][1]) + (acc[r][t][2] + acc[r][t][3]);
        v = warp_sum(v);
        if (lane == 0 && n < N && t < mt) {
          const float outv = v * __ldg(scales + n) * (NORM ? inv_rms[t] : 1.0f);
          y[static_cast<size_t>(t) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(outv));
        }
      }
    }
  }
}

template <int B, int R, int MT, bool NORM>
cudaError_t run_gemv_generic(const uint16_t* x, int mt, const uint8_t* packed, const float* scales, int N,
                     int K, uint16_t* y, cudaStream_t stream) {
  const int rw = static_cast<int>(row_words(K, B));
  const int G = (K + 31) / 32;
  const int g_round = (G + 31) / 32 * 32;
  int gc = static_cast<int>(kXSmemBudget / (static_cast<size_t>(MT) * 32 * 4)) / 32 * 32;
  if (gc > g_round) gc = g_round;
  const size_t smem = static_cast<size_t>(MT) * gc * 32 * 4;
  auto kern = gemv_generic_kernel<B, R, MT, NORM>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kXSmemBudget);
  if (e != cudaSuccess) return e;
  const int rows_per_task = kWarps * R;
  const int num_tasks = (N + rows_per_task - 1) / rows_per_task;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int resident = per_sm * device_info().num_sms;
  const int grid = num_tasks < resident ? num_tasks : resident;
  kern<<<grid, kThreads, smem, stream>>>(x, mt, packed, scales, N, K, rw, y, gc, num_tasks);
  return cudaGetLastError();
}


// ---------------------------------------------------------------------------
// x in registers, persistent row ranges
// ---------------------------------------------------------------------------

// Rows per batch: two batches of packed words plus the x slice must fit the
// registers that __launch_bounds__ leaves (96 per thread when 17 warps share
// the four SM sub-partitions); the thresholds keep every width spill-free.
template <int B, int MT>
constexpr int rows_per_batch() {
  return (8 * (B + 1) + 32 * MT <= 88) ? 4 : ((4 * (B + 1) + 32 * MT <= 80) ? 2 : 1);
}
constexpr int kXregMaxThreads = 544;  // K <= 17408

template <int B>
__device__ __forceinline__ void load_words(const uint32_t* __restrict__ p, bool full, int avail,
                                           uint32_t (&w)[B + 1]) {
  if (full) {
    if constexpr (B % 4 == 0) {
#pragma unroll
      for (int i = 0; i < B / 4; ++i) {
        const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + i);
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
      }
    } else if constexpr (B % 2 == 0) {
#pragma unroll
      for (int i = 0; i < B / 2; ++i) {
        const uint2 v = __ldcs(reinterpret_cast<const uint2*>(p) + i);
        w[2 * i] = v.x; w[2 * i + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < B; ++i) w[i] = __ldcs(p + i);
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = i < avail ? __ldcs(p + i) : 0u;
  }
  w[B] = 0u;
}

template <int B, int MT, bool NORM>
__global__ void __launch_bounds__(kXregMaxThreads, 1)
gemv_xreg_kernel(const uint16_t* __restrict__ x, int mt, const uint8_t* __restrict__ packed,
                 const float* __restrict__ scales, int N, int K, int rw, uint16_t* __restrict__ y) {
  constexpr int kRB = rows_per_batch<B, MT>();
  __shared__ float part[2][kRB][MT][32];
  __shared__ float red[MT][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const int G = (K + 31) >> 5;
  const int g = warp * 32 + lane;
  const bool gact = g < G;
  const int avail = gact ? min(B, rw - g * B) : 0;   // words of this group inside the row
  const bool full = avail == B;

  const int r_begin = static_cast<int>((static_cast<int64_t>(N) * blockIdx.x) / gridDim.x);
  const int r_end = static_cast<int>((static_cast<int64_t>(N) * (blockIdx.x + 1)) / gridDim.x);
  const uint32_t* base = reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(g) * B;

  // first batch of packed words goes out before x is touched
  uint32_t wa[kRB][B + 1], wb[kRB][B + 1];
#pragma unroll
  for (int i = 0; i < kRB; ++i) {
    const int n = r_begin + i;
    if (n < r_end && avail > 0) load_words<B>(base + static_cast<size_t>(n) * rw, full, avail, wa[i]);
    else {
#pragma unroll
      for (int q = 0; q <= B; ++q) wa[i][q] = 0u;
    }
  }

  // this lane's slice of x, as fp32
  float xr[MT][32];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const uint16_t* xt = x + static_cast<size_t>(t) * K + static_cast<size_t>(g) * 32;
    const bool vec = gact && t < mt && (g + 1) * 32 <= K && (reinterpret_cast<uintptr_t>(xt) & 15) == 0;
    if (vec) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(xt) + i);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          xr[t][8 * i + 2 * c] = __uint_as_float(u[c] << 16);
          xr[t][8 * i + 2 * c + 1] = __uint_as_float(u[c] & 0xffff0000u);
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int k = g * 32 + j;
        xr[t][j] = (gact && t < mt && k < K) ? bf16_bits_to_float(__ldg(xt + j)) : 0.0f;
      }
    }
  }
  float inv[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) inv[t] = 1.0f;
  if (NORM) {
    // 1 / sqrt(mean(x^2) + 1e-6) per token, same reduction order in every CTA
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float ss = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) ss = fmaf(xr[t][j], xr[t][j], ss);
      ss = warp_sum(ss);
      if (lane == 0) red[t][warp] = ss;
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float tot = 0.0f;
      for (int w = 0; w < nwarps; ++w) tot += red[t][w];
      inv[t] = 1.0f / sqrtf(tot / static_cast<float>(K) + 1e-6f);
    }
  }

  auto compute = [&](const uint32_t (&w)[kRB][B + 1], int r0, int par) {
#pragma unroll
    for (int i = 0; i < kRB; ++i) {
      float acc[MT][4];
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.0f;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float q = code_f32<B>(w[i], j);
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t][j & 3] = fmaf(xr[t][j], q, acc[t][j & 3]);
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const float v = warp_sum((acc[t][0] + acc[t][1]) + (acc[t][2] + acc[t][3]));
        if (lane == 0) part[par][i][t][warp] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < kRB * MT) {
      const int i = threadIdx.x / MT, t = threadIdx.x % MT;
      const int n = r0 + i;
      if (n < r_end && t < mt) {
        float v = 0.0f;
        for (int w = 0; w < nwarps; ++w) v += part[par][i][t][w];
        const float sc = __ldg(scales + n) * (NORM ? inv[t] : 1.0f);
        y[static_cast<size_t>(t) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(v * sc));
      }
    }
  };
  auto load_batch = [&](uint32_t (&w)[kRB][B + 1], int r0) {
#pragma unroll
    for (int i = 0; i < kRB; ++i) {
      const int n = r0 + i;
      if (n < r_end && avail > 0) load_words<B>(base + static_cast<size_t>(n) * rw, full, avail, w[i]);
    }
  };

  for (int r = r_begin; r < r_end; r += 2 * kRB) {
    load_batch(wb, r + kRB);
    compute(wa, r, 0);
    load_batch(wa, r + 2 * kRB);
    if (r + kRB < r_end) compute(wb, r + kRB, 1);
  }
}

template <int B, int MT, bool NORM>
cudaError_t run_gemv_xreg(const uint16_t* x, int mt, const uint8_t* packed, const float* scales, int N,
                          int K, uint16_t* y, cudaStream_t stream) {
  const int rw = static_cast<int>(row_words(K, B));
  const int G = (K + 31) / 32;
  const int threads = (G + 31) / 32 * 32;
  auto kern = gemv_xreg_kernel<B, MT, NORM>;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int grid = per_sm * device_info().num_sms;
  if (grid > N) grid = N;
  kern<<<grid, threads, 0, stream>>>(x, mt, packed, scales, N, K, rw, y);
  return cudaGetLastError();
}

template <int B>
cudaError_t gemv_bits(const uint16_t* x, int64_t M, const uint8_t* packed, const float* scales,
                      int64_t N, int64_t K, uint16_t* y, bool norm, cudaStream_t stream) {
  const bool xreg = K <= kXregMaxThreads * 32;  // one group per lane
  // passes over the tokens: 2 at a time, a last single one if M is odd
  for (int64_t m0 = 0; m0 < M; m0 += 2) {
    const int mt = static_cast<int>(M - m0 >= 2 ? 2 : 1);
    const uint16_t* xp = x + m0 * K;
    uint16_t* yp = y + m0 * N;
    const int n = static_cast<int>(N), k = static_cast<int>(K);
    cudaError_t e;
    if (xreg) {
      if (mt == 2)
        e = norm ? run_gemv_xreg<B, 2, true>(xp, mt, packed, scales, n, k, yp, stream)
                 : run_gemv_xreg<B, 2, false>(xp, mt, packed, scales, n, k, yp, stream);
      else
        e = norm ? run_gemv_xreg<B, 1, true>(xp, mt, packed, scales, n, k, yp, stream)
                 : run_gemv_xreg<B, 1, false>(xp, mt, packed, scales, n, k, yp, stream);
    } else {
      if (mt == 2)
        e = norm ? run_gemv_generic<B, 2, 2, true>(xp, mt, packed, scales, n, k, yp, stream)
                 : run_gemv_generic<B, 2, 2, false>(xp, mt, packed, scales, n, k, yp, stream);
      else
        e = norm ? run_gemv_generic<B, 4, 1, true>(xp, mt, packed, scales, n, k, yp, stream)
                 : run_gemv_generic<B, 4, 1, false>(xp, mt, packed, scales, n, k, yp, stream);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

size_t gemv_workspace_bytes(const uint16_t* x_or_null, int bits, int layout, int64_t M, int64_t N, int64_t K,
                            bool norm_input) {
  const int64_t pass = norm_input ? 8 : 32;
  const int64_t m1 = M < pass ? M : pass;
  // alignment of x is the caller's business here: assume the kernel takes it
  const uint16_t* xa = x_or_null != nullptr ? x_or_null : reinterpret_cast<const uint16_t*>(256);
  if (!gemv_sk_supported(xa, m1, N, K, norm_input)) return 0;
  size_t b = gemv_sk_workspace_bytes(bits, layout, m1, N, K, norm_input);
  const int64_t last = M % pass;
  if (M > pass && last != 0) {
    const size_t b2 = gemv_sk_workspace_bytes(bits, layout, last, N, K, norm_input);
    if (b2 > b) b = b2;
  }
  return b;
}

cudaError_t launch_gemv(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                        int layout, int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm_input,
                        void* ws, size_t ws_bytes, cudaStream_t stream, unsigned qflags) {
  // Tensor-core decode kernels in passes of up to 32 tokens (8 with
  // norm_input): the stream-K kernel when a workspace is given, else the
  // per-tile TMA kernel.  MPW_GEMV_KERNEL=mma selects the register-streaming
  // variant for canonical rows (tuning aid).
  static const bool use_mma = [] {
    const char* e = tuning_env("MPW_GEMV_KERNEL");
    return e != nullptr && e[0] == 'm';
  }();
  static const bool use_tc = [] {
    const char* e = tuning_env("MPW_GEMV_KERNEL");
    return e != nullptr && e[0] == 't' && e[1] == 'c';
  }();
  // MPW_GEMV_KERNEL=tma: never the tensor-memory kernel (tuning aid)
  static const bool no_tc = [] {
    const char* e = tuning_env("MPW_GEMV_KERNEL");
    return e != nullptr && e[0] == 't' && e[1] == 'm';
  }();
  // Tensor-memory kernel (passes of 32 tokens) where it is the faster one
  // (MPW_GEMV_KERNEL=tc forces it, a tuning aid).
  {
    const int64_t m1 = M < 32 ? M : 32;
    if (ws == nullptr && !use_mma && !no_tc && gemv_tc_supported(x, m1, N, K, norm_input) &&
        (use_tc || gemv_tc_preferred(bits, m1, N, K))) {
      for (int64_t m0 = 0; m0 < M; m0 += 32) {
        const int64_t mt = M - m0 < 32 ? M - m0 : 32;
        cudaError_t e = launch_gemv_tc(x + m0 * K, packed, scales, bits, layout, mt, N, K, y + m0 * N, norm_input,
                                       stream);
        if (e != cudaSuccess) return e;
      }
      return cudaGetLastError();
    }
  }
  const int64_t pass = norm_input ? 8 : 32;
  const int64_t m1 = M < pass ? M : pass;
  const bool paired = layout == kLayoutPaired;
  const bool sk = ws != nullptr && !use_mma && gemv_sk_supported(x, m1, N, K, norm_input);
  const bool tma = (paired || !use_mma) && gemv_tma_supported(x, m1, N, K, norm_input);
  if (paired && !tma) return cudaErrorInvalidValue;
  if (sk || tma || gemv_mma_supported(m1, N, K, norm_input)) {
    for (int64_t m0 = 0; m0 < M; m0 += pass) {
      const int64_t mt = M - m0 < pass ? M - m0 : pass;
      bool used = false;
      cudaError_t e = cudaSuccess;
      if (sk)
        e = launch_gemv_sk(x + m0 * K, packed, scales, bits, layout, mt, N, K, y + m0 * N, norm_input, ws,
                           ws_bytes, stream, &used);
      if (e != cudaSuccess) return e;
      if (!used)
        e = tma ? launch_gemv_tma(x + m0 * K, packed, scales, bits, layout, mt, N, K, y + m0 * N, norm_input,
                                  /*pdl=*/true, qflags, stream)
                : launch_gemv_mma(x + m0 * K, packed, scales, bits, mt, N, K, y + m0 * N, norm_input,
                                  /*pdl=*/true, stream);
      if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
  }
  return launch_gemv_cuda_core(x, packed, scales, bits, M, N, K, y, norm_input, stream);
}

cudaError_t launch_gemv_cuda_core(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                                  int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm_input,
                                  cudaStream_t stream) {
  switch (bits) {
    case 4: return gemv_bits<4>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 5: return gemv_bits<5>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 6: return gemv_bits<6>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 7: return gemv_bits<7>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 8: return gemv_bits<8>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 9: return gemv_bits<9>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 10: return gemv_bits<10>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 11: return gemv_bits<11>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 12: return gemv_bits<12>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 13: return gemv_bits<13>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 14: return gemv_bits<14>(x, M, packed, scales, N, K, y, norm_input, stream);
    case 15: return gemv_bits<15>(x, M, packed, scales, N, K, y, norm_input, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mpw
