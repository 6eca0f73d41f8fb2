// Decode linear for M <= 32 tokens on register-fed tensor cores:
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k]).
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are read from
// memory once, expanded in registers to a tensor-core format and fed to the
// tensor cores; in decode the bytes saved are the speedup (the layer is
// bandwidth-bound: quantization tutorial, closing note).
//
// Why this shape.  At M = 1 the packed stream arrives at ~13 G codes/s at
// 4 bits, which leaves about three lane-instructions per code on the whole
// GPU.  A CUDA-core dot product alone costs four (isolate, expand, subtract,
// FMA), so the multiply-accumulate goes to the tensor pipe
// (mma.sync m16n8k16, bf16 x bf16 -> fp32) and the integer pipe only expands
// codes:
//   * b = 4: the nibbles of codes k and k+4 sit exactly 16 bits apart in a
//     packed word, so one shift and one LOP3 give two bf16 values 128 + u'
//     (u' = offset-binary code, OR-ed into the mantissa of 128.0);
//   * b = 8: likewise for the low and the high nibbles of bytes k and k+2;
//     q = 16*hi + lo, both parts fed to the same accumulator;
//   * b = 5..7: codes k and k+1 are brought to bits 0 and 16 with one funnel
//     shift, one shift and two LOP3s;
//   * b >= 9: the offset-binary code is split into 7-bit fields (weights 1,
//     128, 16384), each field exact in bf16, one MMA per field.
// A bf16x2 FMA on the otherwise idle FMA pipe removes the 128 offset (and
// applies the field weight), so every A operand is the exact code value and
// the fp32 accumulator holds sum_k x_k q_k as the tensor core computes it.
// The order of k inside a 16-wide MMA step is free; the x fragments are
// permuted to match (PRMT for the nibble schemes).
//
// Work layout.  A warp owns 16 weight rows (MMA rows g and g+8 of lane
// g*4+tig) and a K-slice; lane tig takes the 32-code group 4c+tig of every
// 128-code chunk c of its slice, so one group of one row is B aligned words
// and the four lanes of a row read 16*B contiguous bytes.  The K range of a
// 16-row tile is split over the 4 warps of a CTA and over the CTAs of a
// thread-block cluster (1..8 CTAs, chosen so the tiles spread evenly over the
// SMs); partial accumulators are reduced through shared memory and then
// distributed shared memory into the cluster's first CTA, which applies the
// row scale and writes bf16.  The packed words of the next two chunks of a
// warp's slice and the next chunk's x fragments are in flight while the
// current chunk is expanded.  Launches use programmatic dependent launch:
// each CTA allows its dependent launch as soon as it starts and waits for its
// predecessor only before the first read of x, so in a chain of linears the
// next kernel's CTAs are resident while this one drains.
#include <cooperative_groups.h>
#include <math.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cmath>
#include <cstdlib>

#include "expand.cuh"
#include "mpw_internal.h"

namespace cg = cooperative_groups;

namespace mpw {
namespace {

using namespace dec;

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 128;  // codes per chunk (4 groups of 32)

// ---------------------------------------------------------------------------
// kernel
// ---------------------------------------------------------------------------

// With NORM (M <= 8) the output is also scaled by r_m = 1/sqrt(mean_k x^2 + 1e-6):
// every lane adds the squares of 4 of the chunk's 128 x values per token, and
// the sums are reduced with the accumulators (one fixed order per launch).
constexpr int kNormMaxM = 8;

// Read-only zeros: lanes without a row (past N) or a token (past M) load
// from here, so the main loop has no predicated loads and no branches.
__device__ __align__(16) uint32_t g_zero_page[32];

template <int B>
__device__ __forceinline__ void load_words_vec(const uint32_t* __restrict__ p, uint32_t (&w)[B + 1]) {
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
  w[B] = 0u;
}

__device__ __forceinline__ void load_x_vec(const uint16_t* __restrict__ p, uint32_t (&xw)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p) + q);
    xw[4 * q] = v.x; xw[4 * q + 1] = v.y; xw[4 * q + 2] = v.z; xw[4 * q + 3] = v.w;
  }
}

template <int B, int NT, bool NORM>
__global__ void __launch_bounds__(kThreads)
gemv_mma_kernel(const uint16_t* __restrict__ x, int M, const uint8_t* __restrict__ packed,
                const float* __restrict__ scales, int N, int K, int rw, uint16_t* __restrict__ y,
                int tiles) {
  constexpr int P = Exp<B>::parts;
  constexpr int NS = NORM ? kNormMaxM : 1;
  constexpr int kStepWords = kWarps * 4 * B;    // packed words between a warp's chunks
  constexpr int kStepX = kWarps * kChunk;       // x elements between a warp's chunks
  __shared__ float red[kWarps][NT][32][4];
  __shared__ float cl_red[8][NT][32][4];
  __shared__ float ss_red[kWarps][NS];
  __shared__ float cl_ss[8][NS];

  cg::cluster_group cluster = cg::this_cluster();
  const int KC = static_cast<int>(cluster.num_blocks());
  const int cr = static_cast<int>(cluster.block_rank());
  const int tile = blockIdx.x / KC;  // one 16-row tile per cluster

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int chunks = (K + kChunk - 1) / kChunk;
  // chunks whose four groups lie inside the row and whose x lies inside K
  const int chunks_main = min(rw / (4 * B), K / kChunk);
  const bool xvec = (K % 8) == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0;
  // this CTA's contiguous chunk range; its warps interleave inside it
  const int cpc = (chunks + KC - 1) / KC;
  const int cb = cr * cpc;
  const int ce = min(chunks, cb + cpc);
  const int r0 = tile * 16;
  const int ra = r0 + g, rb = r0 + g + 8;
  const bool ra_ok = ra < N, rb_ok = rb < N;

  // ---- stream this CTA's share of the tile's packed rows into L2 ----
  if (warp == 0 && lane < 16 && r0 + lane < N && ce > cb) {
    const int w0 = cb * 4 * B;
    const int w1 = min(rw, ce * 4 * B);
    if (w1 > w0) {
      const uint8_t* src = packed + (static_cast<size_t>(r0 + lane) * rw + w0) * 4;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"((w1 - w0) * 4) : "memory");
    }
  }

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
  float ss[NS];
#pragma unroll
  for (int t = 0; t < NS; ++t) ss[t] = 0.0f;

  // this warp's chunks: c = c0 + 4i; the first n_main of them are complete
  const int c0 = cb + warp;
  const int n_my = c0 < ce ? (ce - c0 + kWarps - 1) / kWarps : 0;
  const int lim = min(ce, chunks_main);
  int n_main = c0 < lim ? (lim - c0 + kWarps - 1) / kWarps : 0;
  if (!xvec) n_main = 0;

  const uint32_t* zero_w = g_zero_page;
  const uint16_t* zero_x = reinterpret_cast<const uint16_t*>(g_zero_page);
  const uint32_t* pa = ra_ok ? reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(ra) * rw +
                                   static_cast<size_t>(4 * c0 + tig) * B
                             : zero_w;
  const uint32_t* pb = rb_ok ? reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(rb) * rw +
                                   static_cast<size_t>(4 * c0 + tig) * B
                             : zero_w;
  const int sa = ra_ok ? kStepWords : 0, sb = rb_ok ? kStepWords : 0;
  const uint16_t* px[NT];
  int sx[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int tok = g + 8 * nt;
    const bool on = tok < M;
    px[nt] = on ? x + static_cast<size_t>(tok) * K + static_cast<size_t>(4 * c0 + tig) * 32 : zero_x;
    sx[nt] = on ? kStepX : 0;
  }

  auto compute = [&](const uint32_t (&wa)[B + 1], const uint32_t (&wb)[B + 1], uint32_t (&xw)[NT][16]) {
    uint32_t va[P][16], vb[P][16];
    expand_group<B>(wa, va);
    expand_group<B>(wb, vb);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) permute_x<B>(xw[nt]);
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2)
#pragma unroll
      for (int part = 0; part < P; ++part)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
          mma_bf16(acc[nt], va[part][2 * s2], vb[part][2 * s2], va[part][2 * s2 + 1], vb[part][2 * s2 + 1],
                   xw[nt][2 * s2], xw[nt][2 * s2 + 1]);
  };
  auto norm_squares = [&](int c) {
    if (NORM) {
      // squares of x for the rms scale: 4 of the chunk's 128 values per lane
      const int k0 = c * kChunk + 4 * lane;
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        if (t < M) {
          const uint16_t* xr = x + static_cast<size_t>(t) * K;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (k0 + e < K) {
              const float v = __uint_as_float(static_cast<uint32_t>(__ldg(xr + k0 + e)) << 16);
              ss[t] = fmaf(v, v, ss[t]);
            }
          }
        }
      }
    }
  };

  // ---- main loop over complete chunks: two-slot rings for packed words and x ----
  uint32_t w0a[B + 1], w0b[B + 1], w1a[B + 1], w1b[B + 1];
  uint32_t x0[NT][16], x1[NT][16];
  if (n_main > 0) {
    load_words_vec<B>(pa, w0a);
    load_words_vec<B>(pb, w0b);
  }
  if (n_main > 1) {
    load_words_vec<B>(pa + sa, w1a);
    load_words_vec<B>(pb + sb, w1b);
  }
  // everything above reads only the weights; x may still be being written by
  // the previous kernel in the stream.  The next kernel may launch once this
  // wait has returned.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (n_main > 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) load_x_vec(px[nt], x0[nt]);
  }
  for (int i = 0; i < n_main; i += 2) {
    // chunk i: slot 0
    if (i + 1 < n_main) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) load_x_vec(px[nt] + sx[nt], x1[nt]);
    }
    norm_squares(c0 + i * kWarps);
    compute(w0a, w0b, x0);
    pa += 2 * sa;
    pb += 2 * sb;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) px[nt] += 2 * sx[nt];
    if (i + 2 < n_main) {
      load_words_vec<B>(pa, w0a);
      load_words_vec<B>(pb, w0b);
    }
    // chunk i + 1: slot 1
    if (i + 1 < n_main) {
      if (i + 2 < n_main) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) load_x_vec(px[nt], x0[nt]);
      }
      norm_squares(c0 + (i + 1) * kWarps);
      compute(w1a, w1b, x1);
      if (i + 3 < n_main) {
        load_words_vec<B>(pa + sa, w1a);
        load_words_vec<B>(pb + sb, w1b);
      }
    }
  }

  // ---- the ragged tail (K not a multiple of 128, or unaligned x): guarded ----
  for (int i = n_main; i < n_my; ++i) {
    const int c = c0 + i * kWarps;
    const int grp = 4 * c + tig;
    const int avail = max(0, min(B, rw - grp * B));
    uint32_t wa[B + 1], wb[B + 1], xw[NT][16];
    const uint32_t* qa = reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(ra_ok ? ra : 0) * rw + static_cast<size_t>(grp) * B;
    const uint32_t* qb = reinterpret_cast<const uint32_t*>(packed) + static_cast<size_t>(rb_ok ? rb : 0) * rw + static_cast<size_t>(grp) * B;
#pragma unroll
    for (int q = 0; q < B; ++q) {
      wa[q] = (ra_ok && q < avail) ? __ldcs(qa + q) : 0u;
      wb[q] = (rb_ok && q < avail) ? __ldcs(qb + q) : 0u;
    }
    wa[B] = 0u;
    wb[B] = 0u;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int tok = g + 8 * nt;
      const uint16_t* xr = x + static_cast<size_t>(tok < M ? tok : 0) * K;
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        const int k = grp * 32 + 2 * m;
        const uint32_t lo = (tok < M && k < K) ? __ldg(xr + k) : 0u;
        const uint32_t hi = (tok < M && k + 1 < K) ? __ldg(xr + k + 1) : 0u;
        xw[nt][m] = lo | (hi << 16);
      }
    }
    norm_squares(c);
    compute(wa, wb, xw);
  }

  // ---- reduce the K slices: warps, then the cluster ----
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
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v = red[0][nt][lane][q];
#pragma unroll
        for (int w2 = 1; w2 < kWarps; ++w2) v += red[w2][nt][lane][q];
        acc[nt][q] = v;
      }
    if (NORM) {
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        float v = ss_red[0][t];
#pragma unroll
        for (int w2 = 1; w2 < kWarps; ++w2) v += ss_red[w2][t];
        ss[t] = v;
      }
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
  }
  if (KC > 1) cluster.sync();
  if (cr == 0 && warp == 0) {
    if (KC > 1) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v = cl_red[0][nt][lane][q];
          for (int r = 1; r < KC; ++r) v += cl_red[r][nt][lane][q];
          acc[nt][q] = v;
        }
    }
    float inv[2] = {1.0f, 1.0f};
    if (NORM) {
      if (KC > 1) {
#pragma unroll
        for (int t = 0; t < NS; ++t) {
          float v = cl_ss[0][t];
          for (int r = 1; r < KC; ++r) v += cl_ss[r][t];
          ss[t] = v;
        }
      }
      // this lane writes tokens 2*tig and 2*tig+1 (NT == 1 when NORM)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = 0.0f;
#pragma unroll
        for (int t = 0; t < NS; ++t) v = (t == 2 * tig + e) ? ss[t] : v;
        inv[e] = 1.0f / sqrtf(v / static_cast<float>(K) + 1e-6f);
      }
    }
    const float sca = ra_ok ? __ldg(scales + ra) : 0.0f;
    const float scb = rb_ok ? __ldg(scales + rb) : 0.0f;
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
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct Plan {
  int kc;        // CTAs per cluster (K split across 4 * kc warps)
};

// Cluster size: each 16-row tile is one cluster of kc CTAs.  The time is
// modelled as (CTAs per SM) x (chunks per warp + a fixed reduction cost of
// three chunks), which favours few clusters per tile unless there are too few
// tiles to spread over the SMs.
Plan plan_for(int tiles, int chunks, int num_sms) {
  Plan best{1};
  double best_t = 1e300;
  for (int kc = 1; kc <= 8; kc *= 2) {
    if (kc > 1 && kWarps * kc > chunks) break;
    const double per_sm = std::ceil(static_cast<double>(tiles) * kc / num_sms);
    const double cpw = std::ceil(static_cast<double>(chunks) / (kWarps * kc));
    const double t = per_sm * (cpw + 3.0);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = Plan{kc};
    }
  }
  return best;
}

template <int B, int NT, bool NORM>
cudaError_t run_mma(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                    uint16_t* y, bool pdl, cudaStream_t stream) {
  auto kern = gemv_mma_kernel<B, NT, NORM>;
  const DeviceInfo& di = device_info();
  const int tiles = (N + 15) / 16;
  const int chunks = (K + kChunk - 1) / kChunk;
  Plan pl = plan_for(tiles, chunks, di.num_sms);
  // MPW_GEMV_CLUSTER=1|2|4|8 overrides the cluster size (tuning aid)
  static const int forced = [] {
    const char* e = tuning_env("MPW_GEMV_CLUSTER");
    const int v = e ? atoi(e) : 0;
    return (v == 1 || v == 2 || v == 4 || v == 8) ? v : 0;
  }();
  if (forced > 0 && kWarps * forced <= chunks) pl.kc = forced;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * pl.kc));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = static_cast<unsigned>(pl.kc);
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
  const int rw = static_cast<int>(row_words(K, B));
  return cudaLaunchKernelEx(&cfg, kern, x, M, packed, scales, N, K, rw, y, tiles);
}

template <int B>
cudaError_t mma_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                     uint16_t* y, bool norm, bool pdl, cudaStream_t stream) {
  if (norm) return run_mma<B, 1, true>(x, M, packed, scales, N, K, y, pdl, stream);  // M <= 8
  if (M <= 8) return run_mma<B, 1, false>(x, M, packed, scales, N, K, y, pdl, stream);
  if (M <= 16) return run_mma<B, 2, false>(x, M, packed, scales, N, K, y, pdl, stream);
  return run_mma<B, 4, false>(x, M, packed, scales, N, K, y, pdl, stream);
}

}  // namespace

bool gemv_mma_supported(int64_t M, int64_t N, int64_t K, bool norm) {
  return M >= 1 && M <= 32 && (!norm || M <= kNormMaxM) && N >= 1 && K >= 1 && N < (1 << 30);
}

cudaError_t launch_gemv_mma(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, bool pdl,
                            cudaStream_t stream) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (bits) {
    case 4: return mma_bits<4>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 5: return mma_bits<5>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 6: return mma_bits<6>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 7: return mma_bits<7>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 8: return mma_bits<8>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 9: return mma_bits<9>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 10: return mma_bits<10>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 11: return mma_bits<11>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 12: return mma_bits<12>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 13: return mma_bits<13>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 14: return mma_bits<14>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    case 15: return mma_bits<15>(x, m, packed, scales, n, k, y, norm, pdl, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace mpw
