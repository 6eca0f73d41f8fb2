// Prefill GEMM on tcgen05 tensor cores:
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k]),  M tokens x N weight rows.
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are loaded,
// expanded in registers to a tensor-core format and fed to the tensor cores;
// codes of 9-15 bits go to the BF16 tensor cores.  Quantization tutorial,
// closing note: prefill is compute-bound.
//
// One CTA computes a 128-row (W) x 256-token (x) tile of y^T with
// tcgen05.mma.cta_group::1.kind::f16, M=128, N=256, K=16:
//   * A = 128 weight rows x 16 codes, held in TENSOR MEMORY.  Converter warps
//     (8 warps, one weight row per thread per half k-block) read the packed
//     row straight from global memory, expand each b-bit code to an exact
//     bf16 value and store it with tcgen05.st, so the expanded weights never
//     touch shared memory.  Codes up to 9 bits are exact in bf16; wider codes
//     are split q = 256*hi + lo (lo = q & 255, both parts exact in bf16) and
//     issued as two MMAs into the same accumulator.
//   * B = 256 tokens x 16 of x, loaded by TMA (128-byte swizzle, K-major) into
//     a 6-stage shared-memory ring.
//   * D = fp32 accumulator, 128 lanes x 256 columns of tensor memory.
// Warp roles: 0 = TMA producer, 1 = MMA issuer, 2 = tensor-memory allocator,
// 4..11 = converters, then the epilogue (tcgen05.ld, row scale, bf16 store).
// Every mbarrier wait is bounded; on time-out the kernel records an error in
// the device error word and every role falls through to the final barrier.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace mpw {
namespace {

constexpr int BM = 128;          // weight rows per CTA (MMA M)
constexpr int BN = 256;          // tokens per CTA (MMA N)
constexpr int BK = 64;           // codes per k-block (one 128-byte swizzle atom of bf16)
constexpr int SX = 6;            // x stages in shared memory
constexpr int SA = 4;            // A stages in tensor memory
constexpr int kThreads = 384;    // 12 warps
constexpr int kConvWarp0 = 4;    // first converter warp
constexpr uint32_t kXStageBytes = BN * BK * 2;   // 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = BN;                // fp32 accumulator columns
constexpr size_t kSmemBytes = SX * kXStageBytes + 1024 /*align slack*/ + 256 /*barriers*/;

template <int B>
struct GemmCode {
  static constexpr bool HL = B > 9;                    // hi/lo split needed
  static constexpr uint32_t ACOLS = HL ? 64 : 32;      // tensor-memory columns per A stage
};

// Code j (0..31) of a 32-code group as an exact fp32 integer.
template <int B>
__device__ __forceinline__ float code_f32(const uint32_t (&w)[B + 1], int j) {
  const int o = j * B;
  const int i = o >> 5, r = o & 31;
  uint32_t t;
  if (r == 0) t = w[i];
  else if (r + B <= 32) t = w[i] >> r;
  else t = __funnelshift_r(w[i], w[i + 1], r);
  constexpr uint32_t kMask = (1u << B) - 1u;
  constexpr uint32_t kMagic = 0x4B000000u | (1u << (B - 1));
  constexpr float kOffset = 8388608.0f + static_cast<float>(1 << (B - 1));
  return __uint_as_float((t & kMask) ^ kMagic) - kOffset;
}

// Code j (0..31) of a 32-code group of a paired-halves row: even codes form
// the stream in the low half-words, odd codes the stream in the high ones.
template <int B>
__device__ __forceinline__ float code_f32_paired(const uint32_t (&w)[B + 1], int j) {
  const int o = (j >> 1) * B;
  const int h = o >> 4, r = o & 15;
  // half-words h and h+1 of the code's stream as one 32-bit window
  const uint32_t win = __byte_perm(w[h], w[h + 1], (j & 1) ? 0x7632 : 0x5410);
  constexpr uint32_t kMask = (1u << B) - 1u;
  constexpr uint32_t kMagic = 0x4B000000u | (1u << (B - 1));
  constexpr float kOffset = 8388608.0f + static_cast<float>(1 << (B - 1));
  return __uint_as_float(((win >> r) & kMask) ^ kMagic) - kOffset;
}

template <int B, bool PAIRED>
__device__ __forceinline__ float code_at(const uint32_t (&w)[B + 1], int j) {
  if constexpr (PAIRED) return code_f32_paired<B>(w, j);
  else return code_f32<B>(w, j);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <int B>
__device__ __forceinline__ void load_group(const uint32_t* __restrict__ rowp, int g, int rw,
                                           bool row_ok, uint32_t (&w)[B + 1]) {
  const bool full = row_ok && (g + 1) * B <= rw;
#pragma unroll
  for (int i = 0; i < B; ++i) {
    const int idx = g * B + i;
    w[i] = full ? __ldg(rowp + idx) : ((row_ok && idx < rw) ? __ldg(rowp + idx) : 0u);
  }
  w[B] = 0u;
}

template <int B, bool PAIRED>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const uint8_t* __restrict__ packed,
            const float* __restrict__ scales, uint16_t* __restrict__ y, int M, int N, int K, int rw,
            int32_t* err) {
  using C = GemmCode<B>;
  extern __shared__ uint8_t gsmem_raw[];
  const uint32_t raw = ptx::smem_addr(gsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;       // 1024-aligned for the 128-byte swizzle
  uint8_t* gsmem = gsmem_raw + (base - raw);
  const uint32_t xs0 = base;                           // SX x stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(gsmem + SX * kXStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SX + 2 * SA + 1);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full_x = [&](int s) { return bar0 + 8u * s; };
  auto empty_x = [&](int s) { return bar0 + 8u * (SX + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * SX + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * SX + SA + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * SX + 2 * SA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BM;
  const int m0 = blockIdx.y * BN;
  const int KB = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      ptx::mbar_init(full_x(s), 1);
      ptx::mbar_init(empty_x(s), 1);
    }
    for (int s = 0; s < SA; ++s) {
      ptx::mbar_init(full_a(s), 32 * (kThreads / 32 - kConvWarp0));
      ptx::mbar_init(empty_a(s), 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_fence_init();
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_addr(tmem_slot), kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_acc = tmem;
  const uint32_t tmem_a = tmem + kAccCols;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % SX;
        const uint32_t ph = (kb / SX) & 1;
        if (!ptx::mbar_wait(empty_x(s), ph ^ 1, err)) break;
        ptx::mbar_arrive_expect_tx(full_x(s), kXStageBytes);
        ptx::tma_load_2d(xs0 + s * kXStageBytes, &tmap_x, full_x(s), kb * BK, m0);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
      bool ok = true;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int sx = kb % SX, sa = kb % SA;
        ok = ptx::mbar_wait(full_x(sx), (kb / SX) & 1, err) &&
             ptx::mbar_wait(full_a(sa), (kb / SA) & 1, err);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bdesc = ptx::sw128_kmajor_desc(xs0 + sx * kXStageBytes);
        const uint32_t a_stage = tmem_a + sa * C::ACOLS;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = bdesc + static_cast<uint64_t>(2 * kk);  // +32 bytes along K
          if (C::HL) {
            ptx::mma_ts(tmem_acc, a_stage + kk * 8, bd, idesc, (kb | kk) != 0);
            ptx::mma_ts(tmem_acc, a_stage + 32 + kk * 8, bd, idesc, 1u);
          } else {
            ptx::mma_ts(tmem_acc, a_stage + kk * 8, bd, idesc, (kb | kk) != 0);
          }
        }
        ptx::mma_commit(empty_x(sx));
        ptx::mma_commit(empty_a(sa));
      }
      ptx::mma_commit(acc_full);
    }
  } else if (warp >= kConvWarp0) {
    // ---------------- converters, then epilogue ----------------
    const int wg = (warp - kConvWarp0) >> 2;       // which half of each k-block
    const int quad = warp & 3;                     // tensor-memory lane quadrant
    const int r = quad * 32 + lane;                // weight row within the tile
    const int n = n0 + r;
    const bool row_ok = n < N;
    const uint32_t* rowp = reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(row_ok ? n : 0) * rw;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    uint32_t wcur[B + 1], wnext[B + 1];
    load_group<B>(rowp, wg, rw, row_ok, wcur);
    for (int kb = 0; kb < KB; ++kb) {
      const int s = kb % SA;
      if (kb + 1 < KB) load_group<B>(rowp, 2 * (kb + 1) + wg, rw, row_ok, wnext);
      uint32_t va[16], vb[16];
      if (C::HL) {
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float q0 = code_at<B, PAIRED>(wcur, 2 * p), q1 = code_at<B, PAIRED>(wcur, 2 * p + 1);
          const int i0 = static_cast<int>(q0), i1 = static_cast<int>(q1);
          const float l0 = static_cast<float>(i0 & 255), l1 = static_cast<float>(i1 & 255);
          va[p] = pack_bf16x2(q0 - l0, q1 - l1);   // 256 * hi, exact
          vb[p] = pack_bf16x2(l0, l1);             // lo in [0, 255], exact
        }
      } else {
#pragma unroll
        for (int p = 0; p < 16; ++p) va[p] = pack_bf16x2(code_at<B, PAIRED>(wcur, 2 * p), code_at<B, PAIRED>(wcur, 2 * p + 1));
      }
      ok = ptx::mbar_wait(empty_a(s), ((kb / SA) & 1) ^ 1, err);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t col = kAccCols + s * C::ACOLS + wg * 16;
      ptx::tmem_st16(tmem + lane_addr + col, va);
      if (C::HL) ptx::tmem_st16(tmem + lane_addr + col + 32, vb);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(full_a(s));
#pragma unroll
      for (int i = 0; i <= B; ++i) wcur[i] = wnext[i];
    }
    if (ok) ok = ptx::mbar_wait(acc_full, 0, err);
    if (ok) {
      ptx::tc_fence_after();
      const float sn = row_ok ? __ldg(scales + n) : 0.0f;
#pragma unroll 1
      for (int c = 0; c < BN / 2 / 32; ++c) {
        const int col = wg * (BN / 2) + c * 32;
        uint32_t v[32];
        ptx::tmem_ld32(tmem + lane_addr + col, v);
        ptx::tmem_wait_ld(v);
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int t = m0 + col + i;
            if (t < M) {
              const float o = __uint_as_float(v[i]) * sn;
              y[static_cast<size_t>(t) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
            }
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int B, bool PAIRED>
cudaError_t run_gemm(const uint16_t* x, const uint8_t* packed, const float* scales, int64_t M,
                     int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, BN};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides,
                       box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = gemm_kernel<B, PAIRED>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), kSmemBytes);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((N + BM - 1) / BM), static_cast<unsigned>((M + BN - 1) / BN));
  kern<<<grid, kThreads, kSmemBytes, stream>>>(tmap, packed, scales, y, static_cast<int>(M),
                                               static_cast<int>(N), static_cast<int>(K),
                                               static_cast<int>(row_words(K, B)), err);
  return cudaGetLastError();
}

}  // namespace

bool gemm_supported(int64_t M, int64_t N, int64_t K) {
  // TMA needs the x row stride (K * 2 bytes) to be a multiple of 16 bytes.
  return K % 8 == 0 && M >= 1 && N >= 1 && (M + BN - 1) / BN <= 65535;
}

template <bool PAIRED>
cudaError_t gemm_layout(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int64_t M,
                        int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  switch (bits) {
    case 4: return run_gemm<4, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 5: return run_gemm<5, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 6: return run_gemm<6, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 7: return run_gemm<7, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 8: return run_gemm<8, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 9: return run_gemm<9, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 10: return run_gemm<10, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 11: return run_gemm<11, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 12: return run_gemm<12, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 13: return run_gemm<13, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 14: return run_gemm<14, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 15: return run_gemm<15, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemm(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* err,
                        cudaStream_t stream) {
  if (layout == kLayoutPaired) return gemm_layout<true>(x, packed, scales, bits, M, N, K, y, err, stream);
  return gemm_layout<false>(x, packed, scales, bits, M, N, K, y, err, stream);
}

}  // namespace mpw
