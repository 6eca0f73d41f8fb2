// Prefill GEMM on FP8 (E4M3) tensor cores for codes of 4 and 5 bits:
//   y[m, n] = bf16(s_n * sx_m * sum_k xq[m, k] * q[n, k]),
// with xq / sx the per-token E4M3 activations (quantize_x_fp8 below).
//
// DynaQuant, "Custom kernel architecture": codes of 5-7 bits are expanded to
// FP8 E4M3 and fed to FP8 tensor cores.  E4M3 holds integers exactly up to 16
// in magnitude, so codes of b <= 5 bits (|q| <= 15) reach the tensor cores
// unrounded; the product needs the activations in FP8 too, quantized per
// token with the symmetric formula of the quantization tutorial ("How
// quantization works") and E4M3's largest finite value 448 as max_int.
//
// One CTA computes a 128-row (W) x 256-token tile of y^T with
// tcgen05.mma.cta_group::1.kind::f8f6f4, M=128, N=256, K=32:
//   * packed weights move in blocks of 128 codes (16*B bytes per row), one 2D
//     TMA per block into a 4-stage ring (64-byte swizzle for 4-bit rows);
//   * A = 128 rows x 128 codes per block in TENSOR MEMORY (32 columns): two
//     groups of four converter warps take alternate blocks, one row per
//     thread; each pair of codes becomes an exact f16 pair (bit-field magic
//     number 1024 and one f16x2 subtraction), converted to an E4M3 pair
//     (exact) and stored with tcgen05.st;
//   * B = 256 tokens x 128 E4M3 values of x per stage (one 128-byte swizzle
//     row per token) by TMA into a 4-stage ring;
//   * D = fp32 accumulator, 128 lanes x 256 columns of tensor memory; the
//     epilogue applies s_n and sx_m and stores bf16.
// Warp roles as in the bf16 prefill GEMM: 0 = x producer, 1 = MMA issuer,
// 2 = tensor-memory allocator, 3 = weight producer, 4..11 = converters and
// epilogue.  Every mbarrier wait is bounded.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "expand.cuh"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace mpw {
namespace {

using namespace dec;

constexpr int BM = 128;          // weight rows per CTA (MMA M)
constexpr int BK = 128;          // codes per block and per x stage (128 bytes of E4M3)
constexpr int SX = 4;            // x stages
constexpr int SW = 4;            // weight stages
constexpr int kThreads = 384;
constexpr int kConvWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACols = BK / 4;                      // one A stage: 128 bytes per row
constexpr float kE4M3Max = 448.0f;

// BN: tokens per CTA (the MMA's N), 256 or 192 (chosen per shape so that the
// tiles fill the SMs in whole waves).
template <int B, int BN>
struct F8Code {
  static constexpr uint32_t kXStageBytes = BN * BK;      // 32 KB at BN = 256
  static constexpr uint32_t kAccCols = BN;               // fp32 accumulator columns
  static constexpr int SA = static_cast<int>((kTmemCols - kAccCols) / kACols);
  static constexpr uint32_t PITCH = 16u * B;
  static constexpr uint32_t WSTAGE = BM * PITCH;
  static constexpr CUtensorMapSwizzle WSWZ = B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
  // byte offset of 16-byte unit u of row r inside a weight stage
  static __device__ __forceinline__ uint32_t unit(int r, int u) {
    if constexpr (B == 4) return r * 64u + 16u * (static_cast<uint32_t>(u) ^ ((r >> 1) & 3));
    else return r * PITCH + 16u * u;
  }
  static constexpr size_t SMEM = SX * kXStageBytes + SW * WSTAGE + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(SMEM <= 232448, "shared memory per block");
};

// Codes 2I, 2I+1 of a 32-code group as an E4M3 pair (16 bits, code 2I in the
// low byte): 1024 + (q + 2^(B-1)) as f16 by OR-ing the offset-binary field
// into the mantissa of 1024.0, one f16x2 subtraction, one conversion.
template <int B, bool PAIRED, int I>
__device__ __forceinline__ uint32_t e4m3_pair(const uint32_t (&w)[B + 1]) {
  constexpr uint32_t fm = ((1u << B) - 1u) * 0x10001u;
  constexpr uint32_t xm = 0x64006400u | (1u << (B - 1)) * 0x10001u;   // 1024.0 pair, sign bit flipped
  const uint32_t h = and_xor(pair_window<B, PAIRED, I>(w), fm, xm);
  const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&h),
                            __halves2half2(__ushort_as_half(static_cast<unsigned short>(0x6400u | (1u << (B - 1)))),
                                           __ushort_as_half(static_cast<unsigned short>(0x6400u | (1u << (B - 1))))));
  __half2_raw raw = static_cast<__half2_raw>(v);
  return static_cast<uint32_t>(__nv_cvt_halfraw2_to_fp8x2(raw, __NV_SATFINITE, __NV_E4M3));
}

template <int B, bool PAIRED, int... I>
__device__ __forceinline__ void e4m3_all(const uint32_t (&w)[B + 1], uint32_t (&o)[8],
                                         std::integer_sequence<int, I...>) {
  ((o[I] = e4m3_pair<B, PAIRED, 2 * I>(w) | (e4m3_pair<B, PAIRED, 2 * I + 1>(w) << 16)), ...);
}

// One 32-code group -> 8 words of E4M3 codes in k order.
template <int B, bool PAIRED>
__device__ __forceinline__ void e4m3_group(const uint32_t (&w)[B + 1], uint32_t (&o)[8]) {
  e4m3_all<B, PAIRED>(w, o, std::make_integer_sequence<int, 8>{});
}

template <int B, bool PAIRED, int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const float* __restrict__ scales, const float* __restrict__ sx, uint16_t* __restrict__ y, int M,
                int N, int K, int32_t* err) {
  using C = F8Code<B, BN>;
  constexpr uint32_t kXStageBytes = C::kXStageBytes;
  constexpr uint32_t kAccCols = C::kAccCols;
  constexpr int SA = C::SA;
  extern __shared__ uint8_t fsmem_raw[];
  __shared__ float sx_s[BN];
  const uint32_t raw = ptx::smem_addr(fsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;       // 1024-aligned for the 128-byte swizzle
  uint8_t* fsmem = fsmem_raw + (base - raw);
  const uint32_t xs0 = base;
  const uint32_t ws0 = base + SX * kXStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(fsmem + SX * kXStageBytes + SW * C::WSTAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SX + 2 * SW + 2 * SA + 1);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full_x = [&](int s) { return bar0 + 8u * s; };
  auto empty_x = [&](int s) { return bar0 + 8u * (SX + s); };
  auto full_w = [&](int s) { return bar0 + 8u * (2 * SX + s); };
  auto empty_w = [&](int s) { return bar0 + 8u * (2 * SX + SW + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + SA + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * SX + 2 * SW + 2 * SA);
  constexpr int32_t kW = ptx::kWaitGemmFp8;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // token tiles run fastest (CTAs resident together share weight rows)
  const int m0 = blockIdx.x * BN;
  const int n0 = blockIdx.y * BM;
  const int KB = (K + BK - 1) / BK;      // blocks (one x stage and one weight block each)

  if (threadIdx.x < BN) sx_s[threadIdx.x] = m0 + static_cast<int>(threadIdx.x) < M ? sx[m0 + threadIdx.x] : 0.0f;
  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      ptx::mbar_init(full_x(s), 1);
      ptx::mbar_init(empty_x(s), 1);
    }
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(full_w(s), 1);
      ptx::mbar_init(empty_w(s), 128);      // one converter group
    }
    for (int s = 0; s < SA; ++s) {
      ptx::mbar_init(full_a(s), 128);       // one converter group
      ptx::mbar_init(empty_a(s), 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::mbar_fence_init();
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_w);
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
    // ---------------- x producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % SX;
        if (!ptx::mbar_wait(empty_x(s), ((kb / SX) & 1) ^ 1, err, ptx::wait_code(kW, ptx::kWaitXEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_x(s), kXStageBytes);
        ptx::tma_load_2d(xs0 + s * kXStageBytes, &tmap_x, full_x(s), kb * BK, m0);
        issued = kb + 1;
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int kb = max(0, issued - SX); kb < issued; ++kb)
        ptx::mbar_wait(full_x(kb % SX), (kb / SX) & 1, err, ptx::wait_code(kW, ptx::kWaitXTail));
    }
  } else if (warp == 3) {
    // ---------------- weight producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int wb = 0; wb < KB; ++wb) {
        const int s = wb % SW;
        if (!ptx::mbar_wait(empty_w(s), ((wb / SW) & 1) ^ 1, err, ptx::wait_code(kW, ptx::kWaitWEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_w(s), C::WSTAGE);
        ptx::tma_load_2d(ws0 + s * C::WSTAGE, &tmap_w, full_w(s), wb * 16 * B, n0);
        issued = wb + 1;
      }
      for (int wb = max(0, issued - SW); wb < issued; ++wb)
        ptx::mbar_wait(full_w(wb % SW), (wb / SW) & 1, err, ptx::wait_code(kW, ptx::kWaitWTail));
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_e4m3_f32(BM, BN);
      bool ok = true;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int sx_ = kb % SX, sa = kb % SA;
        ok = ptx::mbar_wait(full_x(sx_), (kb / SX) & 1, err, ptx::wait_code(kW, ptx::kWaitFull));
        if (ok) ok = ptx::mbar_wait(full_a(sa), (kb / SA) & 1, err, ptx::wait_code(kW, ptx::kWaitAFull));
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bdesc = ptx::sw128_kmajor_desc(xs0 + sx_ * kXStageBytes);
        const uint32_t a_cols = tmem_a + sa * kACols;
#pragma unroll
        for (int kk = 0; kk < BK / 32; ++kk)
          ptx::mma_ts_f8(tmem_acc, a_cols + kk * 8, bdesc + static_cast<uint64_t>(2 * kk), idesc, (kb | kk) != 0);
        ptx::mma_commit(empty_x(sx_));
        ptx::mma_commit(empty_a(sa));
      }
      ptx::mma_commit(acc_full);
    }
  } else if (warp >= kConvWarp0) {
    // ---------------- converters, then epilogue ----------------
    const int wg = (warp - kConvWarp0) >> 2;       // which blocks (even / odd)
    const int quad = warp & 3;                     // tensor-memory lane quadrant
    const int r = quad * 32 + lane;                // weight row within the tile
    const int n = n0 + r;
    const bool row_ok = n < N;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int wb = wg; wb < KB; wb += 2) {
      const int ws = wb % SW, sa = wb % SA;
      ok = ptx::mbar_wait(full_w(ws), (wb / SW) & 1, err, ptx::wait_code(kW, ptx::kWaitWFull));
      if (!ok) break;
      uint32_t w[4 * B + 1];
      const uint8_t* stage = fsmem + SX * kXStageBytes + ws * C::WSTAGE;
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + C::unit(r, i));
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
      }
      w[4 * B] = 0u;
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(empty_w(ws));
      ok = ptx::mbar_wait(empty_a(sa), ((wb / SA) & 1) ^ 1, err, ptx::wait_code(kW, ptx::kWaitAEmpty));
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t col = tmem + lane_addr + kAccCols + sa * kACols;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t o[16];
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
          const int g4 = 2 * h2 + g2;
          uint32_t gw[B + 1];
#pragma unroll
          for (int i = 0; i <= B; ++i) gw[i] = w[g4 * B + i];
          uint32_t og[8];
          e4m3_group<B, PAIRED>(gw, og);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[8 * g2 + i] = og[i];
        }
        ptx::tmem_st16(col + 16 * h2, o);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(full_a(sa));
    }
    if (ok) ok = ptx::mbar_wait(acc_full, 0, err, ptx::wait_code(kW, ptx::kWaitAcc));
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
              const float o = __uint_as_float(v[i]) * sn * sx_s[col + i];
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

// ---------------------------------------------------------------------------
// per-token E4M3 activations: one CTA per token
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// sx = fl32(max |x| / 448) (a zero token: fl32(1 / 448)); xq = E4M3_rn(fl32(x / sx)),
// saturating.  K % 16 == 0, x 16-byte aligned (checked by the caller).
__global__ void __launch_bounds__(256)
quantize_x_fp8_kernel(const uint16_t* __restrict__ x, int K, uint8_t* __restrict__ xq, float* __restrict__ sx) {
  __shared__ float red[8];
  const int m = blockIdx.x;
  const uint4* row = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K);
  const int n8 = K >> 3;
  float amax = 0.0f;
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(u[j])), fabsf(bf16_hi(u[j]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = amax == 0.0f ? __fdiv_rn(1.0f, kE4M3Max) : __fdiv_rn(amax, kE4M3Max);
  if (threadIdx.x == 0) sx[m] = s;
  uint2* out = reinterpret_cast<uint2*>(xq + static_cast<size_t>(m) * K);
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = __ldg(row + i);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 a = make_float2(__fdiv_rn(bf16_lo(u[2 * j]), s), __fdiv_rn(bf16_hi(u[2 * j]), s));
      const float2 b = make_float2(__fdiv_rn(bf16_lo(u[2 * j + 1]), s), __fdiv_rn(bf16_hi(u[2 * j + 1]), s));
      const uint32_t pa = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
      const uint32_t pb = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
      o[j] = (pa & 0xFFFFu) | (pb << 16);
    }
    out[i] = make_uint2(o[0], o[1]);
  }
}

template <int B, bool PAIRED, int BN>
cudaError_t run_fp8(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales, int64_t M,
                    int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  using C = F8Code<B, BN>;
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  const cuuint32_t box[2] = {BK, BN};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(xq), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int64_t rb = 16 * ((K * B + 127) / 128);
  CUtensorMap tmap_w;
  {
    const cuuint64_t wdims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(N)};
    const cuuint64_t wstrides[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t wbox[2] = {static_cast<cuuint32_t>(16 * B), static_cast<cuuint32_t>(BM)};
    if (encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), wdims, wstrides, wbox,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, C::WSWZ, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = gemm_fp8_kernel<B, PAIRED, BN>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((M + BN - 1) / BN), static_cast<unsigned>((N + BM - 1) / BM));
  kern<<<grid, kThreads, C::SMEM, stream>>>(tmap, tmap_w, scales, sx, y, static_cast<int>(M), static_cast<int>(N),
                                            static_cast<int>(K), err);
  return cudaGetLastError();
}

// Fraction of the SMs' tile slots that do useful work with token tiles of
// bn (whole waves of one CTA per SM, less the padding of the last token tile).
double fp8_tile_efficiency(int64_t M, int64_t N, int bn, int sms) {
  const int64_t mt = (M + bn - 1) / bn, tiles = mt * ((N + BM - 1) / BM);
  const int64_t rounds = (tiles + sms - 1) / sms;
  return static_cast<double>(tiles) / static_cast<double>(rounds * sms) *
         static_cast<double>(M) / static_cast<double>(mt * bn);
}

template <int B, bool PAIRED>
cudaError_t fp8_bn(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales, int64_t M,
                   int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  const int sms = device_info().num_sms;
  if (fp8_tile_efficiency(M, N, 192, sms) > fp8_tile_efficiency(M, N, 256, sms) + 0.05)
    return run_fp8<B, PAIRED, 192>(xq, sx, packed, scales, M, N, K, y, err, stream);
  return run_fp8<B, PAIRED, 256>(xq, sx, packed, scales, M, N, K, y, err, stream);
}

}  // namespace

cudaError_t launch_quantize_x_fp8(const uint16_t* x, int64_t M, int64_t K, uint8_t* xq, float* sx,
                                  cudaStream_t stream) {
  quantize_x_fp8_kernel<<<static_cast<unsigned>(M), 256, 0, stream>>>(x, static_cast<int>(K), xq, sx);
  return cudaGetLastError();
}

cudaError_t launch_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales,
                            int bits, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                            cudaStream_t stream) {
  int32_t* err = device_error_word();
  const bool paired = layout == kLayoutPaired;
  if (bits == 4)
    return paired ? fp8_bn<4, true>(xq, sx, packed, scales, M, N, K, y, err, stream)
                  : fp8_bn<4, false>(xq, sx, packed, scales, M, N, K, y, err, stream);
  if (bits == 5)
    return paired ? fp8_bn<5, true>(xq, sx, packed, scales, M, N, K, y, err, stream)
                  : fp8_bn<5, false>(xq, sx, packed, scales, M, N, K, y, err, stream);
  return cudaErrorInvalidValue;
}

}  // namespace mpw
