// Decode linear for M <= 32 tokens: packed weights streamed by TMA into a
// shared-memory ring, expanded in registers, multiplied on tensor cores.
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k])
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are read from
// memory once, expanded in registers to a tensor-core format and multiplied;
// in decode the bytes saved are the speedup (the layer is bandwidth-bound:
// quantization tutorial, closing note).
//
// A CTA owns a 16-row tile of W (one cluster of 1..8 CTAs splits the tile's K
// range).  Warp 4 is the producer: one lane walks the CTA's chunks (128 codes
// = 16*B bytes per row) and issues one 2D TMA per chunk, {16*B bytes x 16
// rows}, into a ring of S stages of four chunks each (mbarrier completion,
// rows past N and bytes past the row read as zeros).  Warps 0..3 consume: warp
// w takes chunk 4s+w of stage s, reads the 32-code group of lane tig for rows
// g and g+8 from shared memory (B words per row), expands it to exact bf16
// (expand.cuh) and issues mma.sync m16n8k16 against its x fragment (token g,
// read through L1).  The stage is released to the producer as soon as its
// words are in registers, so the memory system always has S stages of the
// tile in flight independent of how many loads the warps themselves could
// keep outstanding.  Partial sums of the K slices are reduced through shared
// memory and distributed shared memory into the cluster's first CTA, which
// applies the row scale (and the rms scale with norm_input) and writes bf16.
//
// Programmatic dependent launch: every thread lets the next kernel launch at
// once; the producer's TMA loads read only W and never wait, the consumers
// wait (griddepcontrol.wait) before touching x or y.  In a chain of linears
// the next layer's weights stream in while the previous kernel drains.  Every mbarrier wait is bounded (2 s), after which
// the kernel records an error in the device error word and winds down.
#include <cooperative_groups.h>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <cstdlib>

#include "expand.cuh"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace cg = cooperative_groups;

namespace mpw {
namespace {

using namespace dec;

constexpr int kCW = 4;                 // consumer warps
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kChunk = 128;            // codes per chunk
constexpr int kNormMaxM = 8;

// Read-only zeros for lanes without a token (past M).
__device__ __align__(16) uint32_t g_tma_zero_page[16];

template <int B>
constexpr int ring_stages() {
  // one stage = 4 chunks x 16 rows x 16*B bytes = 1 KB * B
  return B <= 6 ? 6 : (B <= 10 ? 4 : 3);
}

template <int B>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t (&w)[B + 1]) {
  if constexpr (B % 4 == 0) {
#pragma unroll
    for (int i = 0; i < B / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
    }
  } else if constexpr (B % 2 == 0) {
#pragma unroll
    for (int i = 0; i < B / 2; ++i) {
      const uint2 v = reinterpret_cast<const uint2*>(p)[i];
      w[2 * i] = v.x; w[2 * i + 1] = v.y;
    }
  } else {
#pragma unroll
    for (int i = 0; i < B; ++i) w[i] = reinterpret_cast<const uint32_t*>(p)[i];
  }
  w[B] = 0u;
}

template <int B, int NT, bool NORM>
__global__ void __launch_bounds__(kThreads)
gemv_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint16_t* __restrict__ x, int M,
                const float* __restrict__ scales, int N, int K, uint16_t* __restrict__ y, int32_t* err) {
  constexpr int P = Exp<B>::parts;
  constexpr int NS = NORM ? kNormMaxM : 1;
  constexpr int S = ring_stages<B>();
  constexpr uint32_t kChunkBytes = 16u * 16u * B;   // 16 rows x 16*B bytes
  constexpr uint32_t kStageBytes = 4u * kChunkBytes;
  extern __shared__ __align__(128) uint8_t tsmem[];
  __shared__ __align__(8) uint64_t bars[2 * S];
  __shared__ float red[kCW][NT][32][4];
  __shared__ float cl_red[8][NT][32][4];
  __shared__ float ss_red[kCW][NS];
  __shared__ float cl_ss[8][NS];

  // The next kernel in the stream may launch right away: it only streams its
  // own weights until its consumers pass griddepcontrol.wait.
  asm volatile("griddepcontrol.launch_dependents;");
  cg::cluster_group cluster = cg::this_cluster();
  const int KC = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int tile = blockIdx.x / KC;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int chunks = (K + kChunk - 1) / kChunk;
  const int cpc = (chunks + KC - 1) / KC;
  const int cb = cr * cpc;
  const int ce = min(chunks, cb + cpc);
  const int n_stages = ce > cb ? (ce - cb + 3) / 4 : 0;
  const int r0 = tile * 16;
  const uint32_t base = ptx::smem_addr(tsmem);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kCW * 32);
    }
    ptx::mbar_fence_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_w);
      int issued = 0;
      for (int s = 0; s < n_stages; ++s) {
        const int slot = s % S;
        if (!ptx::mbar_wait(empty(slot), ((s / S) & 1) ^ 1, err)) break;
        const int c_first = cb + 4 * s;
        const int nvalid = min(4, ce - c_first);
        ptx::mbar_arrive_expect_tx(full(slot), nvalid * kChunkBytes);
        for (int j = 0; j < nvalid; ++j)
          ptx::tma_load_2d(base + slot * kStageBytes + j * kChunkBytes, &tmap_w, full(slot),
                           (c_first + j) * 16 * B, r0);
        issued = s + 1;
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int s = max(0, issued - S); s < issued; ++s) ptx::mbar_wait(full(s % S), (s / S) & 1, err);
    }
  } else {
    // ---------------- consumers ----------------
    // x (and y) may belong to the previous kernel in the stream
    asm volatile("griddepcontrol.wait;" ::: "memory");
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
    float ss[NS];
#pragma unroll
    for (int t = 0; t < NS; ++t) ss[t] = 0.0f;

    const bool xvec = (K % 8) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0;
    const uint16_t* zero_x = reinterpret_cast<const uint16_t*>(g_tma_zero_page);
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % S;
      const int c = cb + 4 * s + warp;
      const bool active = c < ce;
      // x fragments of this chunk (independent of the ring: issued first)
      uint32_t xw[NT][16];
      const int grp = 4 * c + tig;
      const int k0 = grp * 32;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int tok = g + 8 * nt;
        const bool on = active && tok < M;
        if (xvec && k0 + 32 <= K) {
          const uint4* p = reinterpret_cast<const uint4*>(on ? x + static_cast<size_t>(tok) * K + k0 : zero_x);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = __ldg(p + q);
            xw[nt][4 * q] = v.x; xw[nt][4 * q + 1] = v.y; xw[nt][4 * q + 2] = v.z; xw[nt][4 * q + 3] = v.w;
          }
        } else {
          const uint16_t* xr = x + static_cast<size_t>(tok < M ? tok : 0) * K;
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const int k = k0 + 2 * m;
            const uint32_t lo = (on && k < K) ? __ldg(xr + k) : 0u;
            const uint32_t hi = (on && k + 1 < K) ? __ldg(xr + k + 1) : 0u;
            xw[nt][m] = lo | (hi << 16);
          }
        }
      }
      if (NORM && active) {
        // squares of x for the rms scale: 4 of the chunk's 128 values per lane
        const int kk = c * kChunk + 4 * lane;
#pragma unroll
        for (int t = 0; t < NS; ++t) {
          if (t < M) {
            const uint16_t* xr = x + static_cast<size_t>(t) * K;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (kk + e < K) {
                const float v = __uint_as_float(static_cast<uint32_t>(__ldg(xr + kk + e)) << 16);
                ss[t] = fmaf(v, v, ss[t]);
              }
            }
          }
        }
      }
      // packed words of rows g and g+8 from the ring
      if (!ptx::mbar_wait(full(slot), (s / S) & 1, err)) break;
      uint32_t wa[B + 1], wb[B + 1];
      const uint8_t* st = tsmem + slot * kStageBytes + warp * kChunkBytes + tig * 4 * B;
      lds_words<B>(st + g * 16 * B, wa);
      lds_words<B>(st + (g + 8) * 16 * B, wb);
      uint32_t va[P][16], vb[P][16];
      expand_group<B>(wa, va);
      expand_group<B>(wb, vb);
      // Release the stage only once the words are consumed, and order this
      // thread's generic-proxy reads before the TMA (async-proxy) writes that
      // will refill the slot.  Without the fence a refill was observed to land
      // before the reads of the previous stage in this slot had completed.
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(empty(slot));
      if (active) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) permute_x<B>(xw[nt]);
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
#pragma unroll
          for (int part = 0; part < P; ++part)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
              mma_bf16(acc[nt], va[part][2 * s2], vb[part][2 * s2], va[part][2 * s2 + 1],
                       vb[part][2 * s2 + 1], xw[nt][2 * s2], xw[nt][2 * s2 + 1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) red[warp][nt][lane][q] = acc[nt][q];
    if (NORM) {
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        float v = ss[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) ss_red[warp][t] = v;
      }
    }
  }
  __syncthreads();

  // ---- reduce the K slices: warps, then the cluster ----
  if (warp == 0) {
    float acc[NT][4];
    float ss[NS];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v = red[0][nt][lane][q];
#pragma unroll
        for (int w2 = 1; w2 < kCW; ++w2) v += red[w2][nt][lane][q];
        acc[nt][q] = v;
      }
#pragma unroll
    for (int t = 0; t < NS; ++t) {
      float v = 0.0f;
      if (NORM) {
        v = ss_red[0][t];
#pragma unroll
        for (int w2 = 1; w2 < kCW; ++w2) v += ss_red[w2][t];
      }
      ss[t] = v;
    }
    if (KC > 1) {
      float* dst = cluster.map_shared_rank(&cl_red[0][0][0][0], 0);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[((cr * NT + nt) * 32 + lane) * 4 + q] = acc[nt][q];
      if (NORM && lane == 0) {
        float* dss = cluster.map_shared_rank(&cl_ss[0][0], 0);
#pragma unroll
        for (int t = 0; t < NS; ++t) dss[cr * NS + t] = ss[t];
      }
    }
    if (KC > 1) cluster.sync();
    if (cr == 0) {
      if (KC > 1) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v = cl_red[0][nt][lane][q];
            for (int r = 1; r < KC; ++r) v += cl_red[r][nt][lane][q];
            acc[nt][q] = v;
          }
        if (NORM) {
#pragma unroll
          for (int t = 0; t < NS; ++t) {
            float v = cl_ss[0][t];
            for (int r = 1; r < KC; ++r) v += cl_ss[r][t];
            ss[t] = v;
          }
        }
      }
      float inv[2] = {1.0f, 1.0f};
      if (NORM) {
        // this lane writes tokens 2*tig and 2*tig+1 (NT == 1 when NORM)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = 0.0f;
#pragma unroll
          for (int t = 0; t < NS; ++t) v = (t == 2 * tig + e) ? ss[t] : v;
          inv[e] = 1.0f / sqrtf(v / static_cast<float>(K) + 1e-6f);
        }
      }
      const int ra = r0 + g, rb = r0 + g + 8;
      const float sca = ra < N ? __ldg(scales + ra) : 0.0f;
      const float scb = rb < N ? __ldg(scales + rb) : 0.0f;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int tok = 8 * nt + 2 * tig + (q & 1);
          const int row = (q < 2) ? ra : rb;
          if (tok < M && row < N) {
            const float o = acc[nt][q] * ((q < 2) ? sca : scb) * inv[q & 1];
            y[static_cast<size_t>(tok) * N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
          }
        }
    }
    // keep the cluster's shared memory alive until the leader has read it
    if (KC > 1) cluster.sync();
  } else if (KC > 1) {
    // the other warps take part in the cluster barriers too
    cluster.sync();
    cluster.sync();
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

// Cluster size: each 16-row tile is one cluster of kc CTAs.  Time is modelled
// as (CTAs per SM) x (chunks per consumer warp + a fixed cost of three chunks
// for start-up and the reduction).
int cluster_size(int tiles, int chunks, int num_sms) {
  int best = 1;
  double best_t = 1e300;
  for (int kc = 1; kc <= 8; kc *= 2) {
    if (kc > 1 && kCW * kc > chunks) break;
    const double per_sm = std::ceil(static_cast<double>(tiles) * kc / num_sms);
    const double cpw = std::ceil(static_cast<double>(chunks) / (kCW * kc));
    const double t = per_sm * (cpw + 3.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = kc;
    }
  }
  static const int forced = [] {
    const char* e = getenv("MPW_GEMV_CLUSTER");
    const int v = e ? atoi(e) : 0;
    return (v == 1 || v == 2 || v == 4 || v == 8) ? v : 0;
  }();
  if (forced > 0 && kCW * forced <= chunks) best = forced;
  return best;
}

template <int B, int NT, bool NORM>
cudaError_t run_tma(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                    uint16_t* y, bool pdl, int32_t* err, cudaStream_t stream) {
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  const int64_t rb = 16 * ((static_cast<int64_t>(K) * B + 127) / 128);
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(N)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(16 * B), 16};
  const cuuint32_t estr[2] = {1, 1};
  CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides,
                       box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  auto kern = gemv_tma_kernel<B, NT, NORM>;
  const size_t smem = static_cast<size_t>(ring_stages<B>()) * 4 * 16 * 16 * B;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
  const int tiles = (N + 15) / 16;
  const int chunks = (K + kChunk - 1) / kChunk;
  const int kc = cluster_size(tiles, chunks, device_info().num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * kc));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = static_cast<unsigned>(kc);
  attrs[na].val.clusterDim.y = 1;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, tmap, x, M, scales, N, K, y, err);
}

template <int B>
cudaError_t tma_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                     uint16_t* y, bool norm, bool pdl, int32_t* err, cudaStream_t stream) {
  if (norm) return run_tma<B, 1, true>(x, M, packed, scales, N, K, y, pdl, err, stream);  // M <= 8
  if (M <= 8) return run_tma<B, 1, false>(x, M, packed, scales, N, K, y, pdl, err, stream);
  if (M <= 16) return run_tma<B, 2, false>(x, M, packed, scales, N, K, y, pdl, err, stream);
  return run_tma<B, 4, false>(x, M, packed, scales, N, K, y, pdl, err, stream);
}

}  // namespace

bool gemv_tma_supported(int64_t M, int64_t N, int64_t K, bool norm) {
  return M >= 1 && M <= 32 && (!norm || M <= kNormMaxM) && N >= 1 && K >= 1 && N < (1 << 30) &&
         tensor_map_encoder() != nullptr;
}

cudaError_t launch_gemv_tma(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, bool pdl,
                            cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  int32_t* err = device_error_word();
  switch (bits) {
    case 4: return tma_bits<4>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 5: return tma_bits<5>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 6: return tma_bits<6>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 7: return tma_bits<7>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 8: return tma_bits<8>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 9: return tma_bits<9>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 10: return tma_bits<10>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 11: return tma_bits<11>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 12: return tma_bits<12>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 13: return tma_bits<13>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 14: return tma_bits<14>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    case 15: return tma_bits<15>(x, m, packed, scales, n, k, y, norm, pdl, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mpw
