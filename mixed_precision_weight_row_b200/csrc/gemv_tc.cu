// Decode linear for M <= 32 tokens on tcgen05 tensor cores with the
// accumulator in tensor memory:
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k])
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are read from
// memory once, expanded in registers to a tensor-core format and multiplied;
// in decode the bytes saved are the speedup (quantization tutorial, closing
// note: the layer is bandwidth-bound).
//
// One CTA owns 128 weight rows (the MMA's M) and a K slice; a cluster of KC
// CTAs splits the K range of a row tile when there are few tiles.  The
// structure is that of the prefill GEMM with a 32-token tile:
//   * warp 3 streams the slice's 128-code weight blocks (16*B bytes per row)
//     with one 2D TMA per block ({16*B bytes x 128 rows}) into a deep ring
//     (64/128-byte swizzle for 4- and 8-bit rows, so that the converters'
//     16-byte reads spread over all banks);
//   * warp 0 loads x, 64 codes x 32 tokens per stage, by TMA (128-byte
//     swizzle, K-major; tokens past M read as zeros) after
//     griddepcontrol.wait;
//   * four groups of four converter warps (two for b > 7) take weight blocks
//     in turn, one row per thread, and write exact bf16x2 pairs of codes
//     into tensor memory (expand.cuh), codes of more than 9 bits as
//     lo7 + 128*hi;
//   * one thread of warp 1 issues tcgen05.mma kind::f16, M=128, N=32, K=16,
//     A from tensor memory, B (x) from shared memory;
//   * with norm_input, warp 2 sums the squares of each token's x from the
//     same stages;
//   * at the end the cluster's partial sums (128 rows x M tokens) and sums of
//     squares are gathered in the first CTA through distributed shared
//     memory, which applies the row scale (and the rms scale) and writes y.
// The weight loads of the first blocks are issued before
// griddepcontrol.wait (programmatic dependent launch); the next kernel in
// the stream may launch once that wait has returned.  Every mbarrier wait
// is bounded; on time-out the kernel records an error in the device error
// word and every role falls through to the final barriers.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>

#include "expand.cuh"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace cg = cooperative_groups;

namespace mpw {
namespace {

using namespace dec;

constexpr int BM = 128;          // weight rows per CTA (MMA M)
constexpr int BN = 32;           // tokens per CTA (MMA N)
constexpr int BK = 64;           // codes per x stage
constexpr int WB = 128;          // codes per weight block
constexpr int SX = 8;            // x stages
constexpr int kConvWarp0 = 4;
constexpr uint32_t kXStageBytes = BN * BK * 2;   // 4 KB
constexpr uint32_t kTmemCols = 512;
constexpr int kNAcc = 4;                          // accumulators used in rotation
constexpr uint32_t kAccCols = kNAcc * BN;
constexpr int kMaxCluster = 8;

template <int B>
struct TcCode {
  static constexpr int P = GemmParts<B>::parts;
  // converter groups of four warps (one row per thread); wide codes need
  // more registers per thread, so fewer groups
  static constexpr int NG = B <= 7 ? 4 : 2;
  static constexpr int THREADS = 128 + 128 * NG;
  static constexpr uint32_t ACOLS = 64u * P;
  static constexpr int SA = NG;   // one A stage per group
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
  // weight stages: as many as fit (up to 8) in about 200 KB
  static constexpr int SWF = static_cast<int>((200u * 1024u - SX * kXStageBytes) / WSTAGE);
  static constexpr int SW = SWF < 2 ? 2 : (SWF > 8 ? 8 : SWF);
  static constexpr uint32_t RINGS = SX * kXStageBytes + SW * WSTAGE;
  static constexpr size_t SMEM = RINGS + 1024 /*align*/ + 512 /*barriers*/;
  static_assert(kAccCols + SA * ACOLS <= kTmemCols, "tensor memory");
  static_assert(SMEM <= 232448, "shared memory per block");
};


template <int B, bool PAIRED, bool NORM>
__global__ void __launch_bounds__(TcCode<B>::THREADS, 1)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const float* __restrict__ scales, uint16_t* __restrict__ y, int M, int N, int K, int rb,
               int32_t* err) {
  using C = TcCode<B>;
  constexpr int P = C::P;
  constexpr int SA = C::SA;
  constexpr int SW = C::SW;
  extern __shared__ uint8_t tc_smem_raw[];
  __shared__ float ss_part[kMaxCluster][BN];   // sums of squares of x per CTA (gathered in rank 0)
  const uint32_t raw = ptx::smem_addr(tc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = tc_smem_raw + (base - raw);
  const uint32_t xs0 = base;
  const uint32_t ws0 = base + SX * kXStageBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::RINGS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * SX + 2 * SW + 2 * SA + 1);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full_x = [&](int s) { return bar0 + 8u * s; };
  auto empty_x = [&](int s) { return bar0 + 8u * (SX + s); };
  auto full_w = [&](int s) { return bar0 + 8u * (2 * SX + s); };
  auto empty_w = [&](int s) { return bar0 + 8u * (2 * SX + SW + s); };
  auto full_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + s); };
  auto empty_a = [&](int s) { return bar0 + 8u * (2 * SX + 2 * SW + SA + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * SX + 2 * SW + 2 * SA);

  cg::cluster_group cluster = cg::this_cluster();
  const int KC = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int tile = blockIdx.x / KC;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = tile * BM;
  // this CTA's weight blocks [wb0, wb1) and x stages [2*wb0, kb1)
  const int WBs = (K + WB - 1) / WB;
  const int wb0 = (WBs * cr) / KC, wb1 = (WBs * (cr + 1)) / KC;
  const int nwb = wb1 - wb0;
  const int KB = (K + BK - 1) / BK;
  const int kb0 = 2 * wb0, kb1 = min(KB, 2 * wb1);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      ptx::mbar_init(full_x(s), 1);
      ptx::mbar_init(empty_x(s), NORM ? 2 : 1);
    }
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(full_w(s), 1);
      ptx::mbar_init(empty_w(s), 128);
    }
    for (int s = 0; s < SA; ++s) {
      ptx::mbar_init(full_a(s), 128);
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

  float acc_row[BN];            // converter group 0: this row's sums for the 32 tokens
  float ss_tok = 0.0f;          // warp 2 with norm_input: this lane's token's sum of squares

  if (warp == 0) {
    // ---------------- x producer ----------------
    if (lane == 0) {
      ptx::grid_dep_wait_then_release();
      int issued = 0;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % SX;
        if (!ptx::mbar_wait(empty_x(s), ((i / SX) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitXEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_x(s), kXStageBytes);
        ptx::tma_load_2d(xs0 + s * kXStageBytes, &tmap_x, full_x(s), (kb0 + i) * BK, 0);
        issued = i + 1;
      }
      for (int i = max(0, issued - SX); i < issued; ++i) ptx::mbar_wait(full_x(i % SX), (i / SX) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitXTail));
    }
  } else if (warp == 3) {
    // ---------------- weight producer: one TMA per block ----------------
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nwb; ++i) {
        const int s = i % SW;
        if (!ptx::mbar_wait(empty_w(s), ((i / SW) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitWEmpty))) break;
        ptx::mbar_arrive_expect_tx(full_w(s), C::WSTAGE);
        ptx::tma_load_2d(ws0 + s * C::WSTAGE, &tmap_w, full_w(s), (wb0 + i) * 16 * B, n0);
        issued = i + 1;
      }
      for (int i = max(0, issued - SW); i < issued; ++i) ptx::mbar_wait(full_w(i % SW), (i / SW) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitWTail));
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
      bool ok = true;
      for (int i = 0; i < nkb && ok; ++i) {
        const int sx = i % SX;
        const int wl = i >> 1, h = i & 1, sa = wl % SA;
        ok = ptx::mbar_wait(full_x(sx), (i / SX) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitFull));
        if (ok && h == 0) ok = ptx::mbar_wait(full_a(sa), (wl / SA) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitAFull));
        if (!ok) break;
        ptx::tc_fence_after();
        const uint64_t bdesc = ptx::sw128_kmajor_desc(xs0 + sx * kXStageBytes);
        const uint32_t a_cols = tmem_a + sa * C::ACOLS + h * 32;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = bdesc + static_cast<uint64_t>(2 * kk);
          // four accumulators in rotation, so that consecutive MMAs do not
          // wait for one another; each starts from zero on its first use
          if constexpr (P == 1) {
            ptx::mma_ts(tmem_acc + kk * BN, a_cols + kk * 8, bd, idesc, i != 0);
          } else {
            const int a0 = (2 * kk) & 3, a1 = (2 * kk + 1) & 3;
            const bool first = i == 0 && kk < 2;
            ptx::mma_ts(tmem_acc + a0 * BN, a_cols + kk * 8, bd, idesc, !first);
            ptx::mma_ts(tmem_acc + a1 * BN, a_cols + 64 + kk * 8, bd, idesc, !first);
          }
        }
        ptx::mma_commit(empty_x(sx));
        if (h == 1 || i == nkb - 1) ptx::mma_commit(empty_a(sa));
      }
      ptx::mma_commit(acc_full);
    }
  } else if (warp == 2) {
    // ---------------- sums of squares of x (norm_input) ----------------
    if (NORM) {
      // x stage: 32 token rows of 128 bytes (64 values) under the 128-byte
      // swizzle, which permutes 16-byte units inside a row: a row's sum is
      // the same in any order
      for (int i = 0; i < nkb; ++i) {
        const int s = i % SX;
        if (!ptx::mbar_wait(full_x(s), (i / SX) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitSquares))) break;
        const uint4* row = reinterpret_cast<const uint4*>(smem + s * kXStageBytes + lane * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = row[q];
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = __uint_as_float(w4[e] << 16), b = __uint_as_float(w4[e] & 0xFFFF0000u);
            ss_tok = fmaf(a, a, fmaf(b, b, ss_tok));
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(empty_x(s));
      }
    }
  } else {
    // ---------------- converters, then the accumulator readout ----------------
    const int wg = (warp - kConvWarp0) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    bool ok = true;
    for (int i = wg; i < nwb; i += C::NG) {
      const int ws = i % SW, sa = i % SA;
      ok = ptx::mbar_wait(full_w(ws), (i / SW) & 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitWFull));
      if (!ok) break;
      uint32_t w[4 * B + 1];
      const uint8_t* stage = smem + SX * kXStageBytes + ws * C::WSTAGE;
#pragma unroll
      for (int j = 0; j < B; ++j) {
        const uint4 v = *reinterpret_cast<const uint4*>(stage + C::unit(r, j));
        w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
      }
      w[4 * B] = 0u;
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(empty_w(ws));
      ok = ptx::mbar_wait(empty_a(sa), ((i / SA) & 1) ^ 1, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitAEmpty));
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t col = tmem + lane_addr + kAccCols + sa * C::ACOLS;
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {
        uint32_t gw[B + 1];
#pragma unroll
        for (int j = 0; j <= B; ++j) gw[j] = w[g4 * B + j];
        uint32_t v[P][16];
        gemm_expand_group<B, PAIRED>(gw, v);
        ptx::tmem_st16(col + g4 * 16, v[0]);
        if constexpr (P == 2) ptx::tmem_st16(col + 64 + g4 * 16, v[1]);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(full_a(sa));
    }
    if (wg == 0) {
      if (ok) ok = ptx::mbar_wait(acc_full, 0, err, ptx::wait_code(ptx::kWaitGemvTc, ptx::kWaitAcc));
#pragma unroll
      for (int t = 0; t < BN; ++t) acc_row[t] = 0.0f;
      if (ok) {
        ptx::tc_fence_after();
#pragma unroll
        for (int a = 0; a < kNAcc; ++a) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem + lane_addr + a * BN, v);
          ptx::tmem_wait_ld(v);
#pragma unroll
          for (int t = 0; t < BN; ++t) acc_row[t] += __uint_as_float(v[t]);
        }
      }
    }
  }

  // ---- gather the cluster's partial sums in rank 0 and write y ----
  ptx::tc_fence_before();
  if (KC > 1) cluster.sync();   // every CTA is done with its rings
  else __syncthreads();
  const bool reader = warp >= kConvWarp0 && ((warp - kConvWarp0) >> 2) == 0;
  float* red = reinterpret_cast<float*>(smem);   // the rings, free now: [KC-1][128][M]
  if (KC > 1 && cr != 0) {
    if (reader) {
      float* dst = cluster.map_shared_rank(red, 0);
      const int r = (warp & 3) * 32 + lane;
#pragma unroll
      for (int t = 0; t < BN; ++t)
        if (t < M) dst[((cr - 1) * BM + r) * M + t] = acc_row[t];
    }
    if (NORM && warp == 2) cluster.map_shared_rank(&ss_part[0][0], 0)[cr * BN + lane] = ss_tok;
  }
  if (NORM && warp == 2 && cr == 0) ss_part[0][lane] = ss_tok;
  if (KC > 1) cluster.sync();
  else __syncthreads();
  if (cr == 0 && reader) {
    const int r = (warp & 3) * 32 + lane;
    const int n = n0 + r;
    for (int c = 1; c < KC; ++c) {
#pragma unroll
      for (int t = 0; t < BN; ++t)
        if (t < M) acc_row[t] += red[((c - 1) * BM + r) * M + t];
    }
    if (n < N) {
      const float sn = __ldg(scales + n);
      // y may be read by the previous kernel in the stream
      asm volatile("griddepcontrol.wait;" ::: "memory");
#pragma unroll
      for (int t = 0; t < BN; ++t) {
        if (t < M) {
          float inv = 1.0f;
          if (NORM) {
            float sst = 0.0f;
            for (int c = 0; c < KC; ++c) sst += ss_part[c][t];
            inv = 1.0f / sqrtf(sst / static_cast<float>(K) + 1e-6f);
          }
          y[static_cast<size_t>(t) * N + n] =
              __bfloat16_as_ushort(__float2bfloat16_rn(acc_row[t] * sn * inv));
        }
      }
    }
  }
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Cluster size: one CTA per SM, a row tile split over KC CTAs so that the
// grid fills the SMs without a second wave, each CTA keeping at least two
// weight blocks; the gathered partial sums must fit in the rings.
template <int B>
int tc_cluster(int tiles, int wbs, int M, int num_sms) {
  static const int forced = [] {
    const char* e = tuning_env("MPW_GEMV_TC_CLUSTER");
    const int v = e ? atoi(e) : 0;
    return v >= 1 && v <= kMaxCluster ? v : 0;
  }();
  int kc = forced > 0 ? forced : num_sms / tiles;
  kc = kc < 1 ? 1 : (kc > kMaxCluster ? kMaxCluster : kc);
  while (kc > 1 && (wbs / kc < 2 || static_cast<size_t>(kc - 1) * BM * M * 4 > TcCode<B>::RINGS)) --kc;
  return kc;
}

template <int B, bool PAIRED, bool NORM>
cudaError_t run_tc(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                   uint16_t* y, int32_t* err, cudaStream_t stream) {
  using C = TcCode<B>;
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {BK, BN};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int64_t rb = 16 * ((static_cast<int64_t>(K) * B + 127) / 128);
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
  auto kern = gemv_tc_kernel<B, PAIRED, NORM>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM);
  if (e != cudaSuccess) return e;
  const int tiles = (N + BM - 1) / BM;
  const int wbs = (K + WB - 1) / WB;
  const int kc = tc_cluster<B>(tiles, wbs, M, device_info().num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * kc));
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeClusterDimension;
  attrs[0].val.clusterDim.x = static_cast<unsigned>(kc);
  attrs[0].val.clusterDim.y = 1;
  attrs[0].val.clusterDim.z = 1;
  attrs[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmap, tmap_w, scales, y, M, N, K, static_cast<int>(rb), err);
}

template <bool PAIRED, bool NORM>
cudaError_t tc_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits, int N, int K,
                    uint16_t* y, int32_t* err, cudaStream_t s) {
  switch (bits) {
    case 4: return run_tc<4, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 5: return run_tc<5, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 6: return run_tc<6, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 7: return run_tc<7, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 8: return run_tc<8, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 9: return run_tc<9, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 10: return run_tc<10, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 11: return run_tc<11, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 12: return run_tc<12, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 13: return run_tc<13, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 14: return run_tc<14, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    case 15: return run_tc<15, PAIRED, NORM>(x, M, packed, scales, N, K, y, err, s);
    default: return cudaErrorInvalidValue;
  }
}

template <int B>
bool tc_preferred(int64_t M, int64_t N, int64_t K) {
  // measured: this kernel wins over the per-tile decode kernel (two row
  // tiles, four-chunk stages) above 16 tokens when each CTA streams a long K
  // slice (gate 17408x5120 / down 5120x17408, b = 6, M = 32: 29 / 21%
  // against 20 / 19% of HBM), not at 16 (30 / 24% against 37 / 35%); with a
  // short slice its fixed costs (tensor-memory set-up, pipeline fill, cluster
  // gather) dominate
  if (M <= 16) return false;
  const int tiles = static_cast<int>((N + BM - 1) / BM);
  const int wbs = static_cast<int>((K + WB - 1) / WB);
  const int kc = tc_cluster<B>(tiles, wbs, static_cast<int>(M < BN ? M : BN), device_info().num_sms);
  return wbs / kc >= 24;
}

}  // namespace

bool gemv_tc_preferred(int bits, int64_t M, int64_t N, int64_t K) {
  switch (bits) {
    case 4: return tc_preferred<4>(M, N, K);
    case 5: return tc_preferred<5>(M, N, K);
    case 6: return tc_preferred<6>(M, N, K);
    case 7: return tc_preferred<7>(M, N, K);
    case 8: return tc_preferred<8>(M, N, K);
    case 9: return tc_preferred<9>(M, N, K);
    case 10: return tc_preferred<10>(M, N, K);
    case 11: return tc_preferred<11>(M, N, K);
    case 12: return tc_preferred<12>(M, N, K);
    case 13: return tc_preferred<13>(M, N, K);
    case 14: return tc_preferred<14>(M, N, K);
    case 15: return tc_preferred<15>(M, N, K);
    default: return false;
  }
}

bool gemv_tc_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm) {
  return M >= 1 && M <= BN && N >= 1 && K >= 1 && N < (1 << 30) && K % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(x) & 15) == 0 && (!norm || M <= BN) && tensor_map_encoder() != nullptr;
}

cudaError_t launch_gemv_tc(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                           int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  int32_t* err = device_error_word();
  const bool paired = layout == kLayoutPaired;
  if (paired && norm) return tc_bits<true, true>(x, m, packed, scales, bits, n, k, y, err, stream);
  if (paired) return tc_bits<true, false>(x, m, packed, scales, bits, n, k, y, err, stream);
  if (norm) return tc_bits<false, true>(x, m, packed, scales, bits, n, k, y, err, stream);
  return tc_bits<false, false>(x, m, packed, scales, bits, n, k, y, err, stream);
}

}  // namespace mpw
