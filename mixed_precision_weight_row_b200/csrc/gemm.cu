// Prefill GEMM on tcgen05 tensor cores:
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k]),  M tokens x N weight rows.
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are loaded,
// expanded in registers to a tensor-core format and fed to the tensor cores;
// codes of 9-15 bits go to the BF16 tensor cores.  Quantization tutorial,
// closing note: prefill is compute-bound.
//
// One CTA computes a 128-row (W) x 256-token (x) tile of y^T with
// tcgen05.mma.cta_group::1.kind::f16, M=128, N=256, K=16 (192-token tiles,
// N=192, on shapes where 256-token tiles would leave a mostly empty last
// wave of CTAs):
//   * Packed weights move in blocks of 128 codes (16*B bytes per row), one 2D
//     TMA per block ({16*B bytes x 128 rows}) into a 3-stage ring; rows past
//     N and bytes past the row read as zeros.  The converters read a row's
//     16-byte units; for b = 4 and b = 8 the TMA's 64- and 128-byte swizzle
//     spreads eight consecutive rows over all banks, odd b are conflict-free
//     as they are, and the other even b cost two to four ways.
//   * A = 128 weight rows x 16 codes, held in TENSOR MEMORY.  Converter warps
//     (two groups of four, alternating weight blocks; one row per thread)
//     expand each pair of codes to an exact bf16x2 value with a bit-field
//     magic number and one bf16x2 FMA (expand.cuh) and store it with
//     tcgen05.st.  Codes up to 9 bits are fed whole; wider codes as
//     lo7 + 128*hi, two MMAs into the same accumulator, so no code is ever
//     rounded.
//   * B = 256 tokens x 64 of x, loaded by TMA (128-byte swizzle, K-major)
//     into a 4- or 5-stage ring.
//   * D = fp32 accumulator, 128 lanes x 256 columns of tensor memory.
// Warp roles: 0 = x TMA producer, 1 = MMA issuer, 2 = tensor-memory
// allocator, 3 = weight producer, 4..11 = converters, then the epilogue
// (tcgen05.ld, row scale, bf16 store).  Every mbarrier wait is bounded; on
// time-out the kernel records an error in the device error word and every
// role falls through to the final barrier.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "expand.cuh"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace mpw {
namespace {

using namespace dec;

constexpr int BM = 128;          // weight rows per CTA (MMA M)
constexpr int BK = 64;           // codes per x stage (one 128-byte swizzle atom of bf16)
constexpr int WB = 128;          // codes per weight block
constexpr int SW = 3;            // weight stages in shared memory
constexpr int kThreads = 384;    // 12 warps
constexpr int kConvWarp0 = 4;    // first converter warp
constexpr uint32_t kTmemCols = 512;

// BN: tokens per CTA (the MMA's N), 256 or 192 (chosen per shape so that the
// tiles fill the SMs in whole waves).
template <int B, int BN>
struct GemmCode {
  static constexpr uint32_t kXStageBytes = BN * BK * 2;   // 32 KB at BN = 256
  static constexpr uint32_t kAccCols = BN;                // fp32 accumulator columns
  // x stages in shared memory: as many as fit beside the weight stages
  static constexpr int SX = BN == 256 ? (B <= 8 ? 5 : 4) : (B <= 8 ? 6 : 5);
  static constexpr int P = GemmParts<B>::parts;              // MMAs per k-step
  static constexpr uint32_t ACOLS = 64u * P;                 // tensor-memory columns per A stage
  static constexpr int SA = static_cast<int>((kTmemCols - kAccCols) / ACOLS);
  // a weight stage is the TMA box: 128 rows of 16*B bytes
  static constexpr uint32_t PITCH = 16u * B;
  static constexpr uint32_t WSTAGE = BM * PITCH;
  static constexpr CUtensorMapSwizzle WSWZ =
      B == 8 ? CU_TENSOR_MAP_SWIZZLE_128B : (B == 4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE);
  // byte offset of 16-byte unit u of row r inside a weight stage
  static __device__ __forceinline__ uint32_t unit(int r, int u) {
    if constexpr (B == 8) return r * 128u + 16u * (static_cast<uint32_t>(u) ^ (r & 7));
    else if constexpr (B == 4) return r * 64u + 16u * (static_cast<uint32_t>(u) ^ ((r >> 1) & 3));
    else return r * PITCH + 16u * u;
  }
  static constexpr size_t SMEM = SX * kXStageBytes + SW * WSTAGE + 1024 /*align*/ + 256 /*barriers*/;
  static_assert(SMEM <= 232448, "shared memory per block");
};


template <int B, bool PAIRED, int BN>
__global__ void __launch_bounds__(kThreads, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
            const float* __restrict__ scales, uint16_t* __restrict__ y, int M, int N, int K, int rb,
            int32_t* err) {
  using C = GemmCode<B, BN>;
  constexpr int P = C::P;
  constexpr int SA = C::SA;
  constexpr int SX = C::SX;
  constexpr uint32_t kXStageBytes = C::kXStageBytes;
  constexpr uint32_t kAccCols = C::kAccCols;
  extern __shared__ uint8_t gsmem_raw[];
  const uint32_t raw = ptx::smem_addr(gsmem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;       // 1024-aligned for the 128-byte swizzle
  uint8_t* gsmem = gsmem_raw + (base - raw);
  const uint32_t xs0 = base;                           // SX x stages
  const uint32_t ws0 = base + SX * kXStageBytes;       // SW weight stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(gsmem + SX * kXStageBytes + SW * C::WSTAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SX + 2 * SW + 2 * SA + 1);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full_x = [&](int s) { return bar0 + 8u * s; };
  auto empty_x = [&](int s) { return bar0 + 8u * (SX + s); };
  auto full_w = [&](int s) { return bar0 + 8u * (2 * SX + s); };
  auto empty_w = [&](int s) { return bar0 + 8u * (2 * SX + SW + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + SA + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * SX + 2 * SW + 2 * SA);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // token tiles run fastest: the CTAs resident together share weight rows,
  // which then come from L2 after the first of them has read them
  const int m0 = blockIdx.x * BN;
  const int n0 = blockIdx.y * BM;
  const int KB = (K + BK - 1) / BK;      // x stages
  const int WBs = (K + WB - 1) / WB;     // weight blocks

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
    // ---------------- x TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % SX;
        if (!ptx::mbar_wait(empty_x(s), ((kb / SX) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitXEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_x(s), kXStageBytes);
        ptx::tma_load_2d(xs0 + s * kXStageBytes, &tmap_x, full_x(s), kb * BK, m0);
        issued = kb + 1;
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int kb = max(0, issued - SX); kb < issued; ++kb) ptx::mbar_wait(full_x(kb % SX), (kb / SX) & 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitXTail));
    }
  } else if (warp == 3) {
    // ---------------- weight producer: one TMA per block ----------------
    if (lane == 0) {
      int issued = 0;
      for (int wb = 0; wb < WBs; ++wb) {
        const int s = wb % SW;
        if (!ptx::mbar_wait(empty_w(s), ((wb / SW) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitWEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_w(s), C::WSTAGE);
        ptx::tma_load_2d(ws0 + s * C::WSTAGE, &tmap_w, full_w(s), wb * 16 * B, n0);
        issued = wb + 1;
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int wb = max(0, issued - SW); wb < issued; ++wb) ptx::mbar_wait(full_w(wb % SW), (wb / SW) & 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitWTail));
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
      bool ok = true;
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int sx = kb % SX;
        const int wb = kb >> 1, h = kb & 1, sa = wb % SA;
        ok = ptx::mbar_wait(full_x(sx), (kb / SX) & 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitFull));
        if (ok && h == 0) ok = ptx::mbar_wait(full_a(sa), (wb / SA) & 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitAFull));
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bdesc = ptx::sw128_kmajor_desc(xs0 + sx * kXStageBytes);
        const uint32_t a_cols = tmem_a + sa * C::ACOLS + h * 32;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = bdesc + static_cast<uint64_t>(2 * kk);  // +32 bytes along K
          ptx::mma_ts(tmem_acc, a_cols + kk * 8, bd, idesc, (kb | kk) != 0);
          if constexpr (P == 2) ptx::mma_ts(tmem_acc, a_cols + 64 + kk * 8, bd, idesc, 1u);
        }
        ptx::mma_commit(empty_x(sx));
        if (h == 1 || kb == KB - 1) ptx::mma_commit(empty_a(sa));
      }
      ptx::mma_commit(acc_full);
    }
  } else if (warp >= kConvWarp0) {
    // ---------------- converters, then epilogue ----------------
    const int wg = (warp - kConvWarp0) >> 2;       // which weight blocks (even / odd)
    const int quad = warp & 3;                     // tensor-memory lane quadrant
    const int r = quad * 32 + lane;                // weight row within the tile
    const int n = n0 + r;
    const bool row_ok = n < N;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int wb = wg; wb < WBs; wb += 2) {
      const int ws = wb % SW, sa = wb % SA;
      ok = ptx::mbar_wait(full_w(ws), (wb / SW) & 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitWFull));
      if (!ok) break;
      // the row's 4 groups: 16*B bytes, read as 16-byte units
      uint32_t w[4 * B + 1];
      const uint8_t* stage = gsmem + SX * kXStageBytes + ws * C::WSTAGE;
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + C::unit(r, i));
        w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
      }
      w[4 * B] = 0u;
      // the async-proxy refill of this stage must not overtake these reads
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(empty_w(ws));
      ok = ptx::mbar_wait(empty_a(sa), ((wb / SA) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitAEmpty));
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t col = tmem + lane_addr + kAccCols + sa * C::ACOLS;
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        uint32_t gw[B + 1];
#pragma unroll
        for (int i = 0; i <= B; ++i) gw[i] = w[g4 * B + i];
        uint32_t v[P][16];
        gemm_expand_group<B, PAIRED>(gw, v);
        ptx::tmem_st16(col + g4 * 16, v[0]);
        if constexpr (P == 2) ptx::tmem_st16(col + 64 + g4 * 16, v[1]);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(full_a(sa));
    }
    if (ok) ok = ptx::mbar_wait(acc_full, 0, err, ptx::wait_code(ptx::kWaitGemm, ptx::kWaitAcc));
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

template <int B, bool PAIRED, int BN>
cudaError_t run_gemm(const uint16_t* x, const uint8_t* packed, const float* scales, int64_t M,
                     int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  using C = GemmCode<B, BN>;
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
  auto kern = gemm_kernel<B, PAIRED, BN>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>((M + BN - 1) / BN), static_cast<unsigned>((N + BM - 1) / BM));
  kern<<<grid, kThreads, C::SMEM, stream>>>(tmap, tmap_w, scales, y, static_cast<int>(M), static_cast<int>(N),
                                            static_cast<int>(K), static_cast<int>(rb), err);
  return cudaGetLastError();
}

// Fraction of the SMs' tile slots that do useful work with token tiles of
// bn: whole waves of one CTA per SM, less the padding of the last token tile.
double tile_efficiency(int64_t M, int64_t N, int bn, int sms) {
  const int64_t mt = (M + bn - 1) / bn, tiles = mt * ((N + BM - 1) / BM);
  const int64_t rounds = (tiles + sms - 1) / sms;
  return static_cast<double>(tiles) / static_cast<double>(rounds * sms) *
         static_cast<double>(M) / static_cast<double>(mt * bn);
}

template <int B, bool PAIRED>
cudaError_t gemm_bn(const uint16_t* x, const uint8_t* packed, const float* scales, int64_t M, int64_t N,
                    int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  // 256-token tiles convert each weight block for more tokens; 192-token
  // tiles only when they fill the SMs clearly better
  const int sms = device_info().num_sms;
  if (tile_efficiency(M, N, 192, sms) > tile_efficiency(M, N, 256, sms) + 0.05)
    return run_gemm<B, PAIRED, 192>(x, packed, scales, M, N, K, y, err, stream);
  return run_gemm<B, PAIRED, 256>(x, packed, scales, M, N, K, y, err, stream);
}

template <bool PAIRED>
cudaError_t gemm_layout(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int64_t M,
                        int64_t N, int64_t K, uint16_t* y, int32_t* err, cudaStream_t stream) {
  switch (bits) {
    case 4: return gemm_bn<4, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 5: return gemm_bn<5, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 6: return gemm_bn<6, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 7: return gemm_bn<7, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 8: return gemm_bn<8, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 9: return gemm_bn<9, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 10: return gemm_bn<10, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 11: return gemm_bn<11, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 12: return gemm_bn<12, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 13: return gemm_bn<13, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 14: return gemm_bn<14, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    case 15: return gemm_bn<15, PAIRED>(x, packed, scales, M, N, K, y, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool gemm_supported(int64_t M, int64_t N, int64_t K) {
  // TMA needs the x row stride (K * 2 bytes) to be a multiple of 16 bytes.
  return K % 8 == 0 && M >= 1 && N >= 1 && (N + BM - 1) / BM <= 65535;
}

cudaError_t launch_gemm(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int32_t* err,
                        cudaStream_t stream) {
  if (layout == kLayoutPaired) return gemm_layout<true>(x, packed, scales, bits, M, N, K, y, err, stream);
  return gemm_layout<false>(x, packed, scales, bits, M, N, K, y, err, stream);
}

}  // namespace mpw
