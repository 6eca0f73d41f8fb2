// Decode linear for M <= 32 tokens: packed weights and x streamed by TMA into
// a shared-memory ring, weights expanded in registers, multiplied on tensor
// cores.
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k])
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are read from
// memory once, expanded in registers to a tensor-core format and multiplied;
// in decode the bytes saved are the speedup (the layer is bandwidth-bound:
// quantization tutorial, closing note).
//
// A CTA owns a 16-row tile of W (a cluster of 1..8 CTAs splits the tile's K
// range).  The last warp is the producer: one lane fills a ring of stages of
// SC (8, or 4) 128-code chunks each (mbarrier completion).  When K % 128 == 0 a
// stage is two 3D TMAs: the packed rows viewed as [chunk][row][16*B bytes]
// ({16*B x 16 rows x SC chunks}) and x viewed as [chunk][token][128 values]
// ({128 x M x SC chunks}); rows past N and chunks past K read as zeros.  One
// thread issuing many small copies is slow (tens of nanoseconds each), so
// large boxes matter.  Other K take one 2D TMA per chunk and operand (bytes
// past the row and values past K read as zeros).  Shared memory holds the
// same [chunk][row] and [chunk][token] layout either way.  Consumer warp w takes SC / 4 consecutive
// chunks of each stage: per chunk, the 32-code group of lane tig for rows g
// and g+8 (B words per row) and its x fragment for token g, both from shared
// memory; it expands the codes to exact bf16 (expand.cuh; canonical or
// paired-halves layout) and issues mma.sync m16n8k16 into two alternating
// fp32 accumulators, releasing the stage once its last words are read.  Partial sums of the K slices are reduced through shared
// memory and distributed shared memory into the cluster's first CTA, which
// applies the row scale (and the rms scale with norm_input) and writes bf16.
//
// Programmatic dependent launch: the producer issues the weight loads of the
// first stages before griddepcontrol.wait and the x loads after it, then
// lets the next kernel in the stream launch; the thread that writes y waits
// too.  In a chain of linears the next layer's weights stream in while this
// kernel computes.  Because a CTA lets the next kernel launch only after its
// own wait has returned, every launch before that wait's kernel is complete
// when the next kernel starts.  With kXReady the caller states that x was
// written before the launch that precedes the current run of such calls;
// the kernel then lets the next one launch at once and loads x with the
// weights, without waiting, so that consecutive calls overlap in full; only
// the write of y waits for the predecessor.  With kYFree as well (no call of
// the run, nor the launch before it, reads or writes y) only the first CTA
// waits before writing, which keeps completions in launch order, and every
// other CTA writes y and exits at once.  Every mbarrier wait is bounded
// (2 s), after which the kernel records an error in the device error word
// and winds down.
#pragma once

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

constexpr int kCW = 4;                  // consumer warps
constexpr int kCH = 2;                  // chunks per consumer warp and stage
constexpr int kSC = kCW * kCH;          // chunks per stage
constexpr int kThreads = (kCW + 1) * 32;
constexpr int kChunk = 128;             // codes per chunk and row
constexpr int kNormMaxM = 8;
constexpr int kMaxStages = 8;
constexpr int kXReady = 1;              // flags: x is not written by the preceding launch
constexpr int kStageBoxes = 2;          // flags: one 3D TMA per stage and operand
constexpr int kYFree = 4;               // flags: no call of the run touches y

// Bytes of one stage: SC weight chunks (16*RT rows x 16*B bytes) followed
// by SC x chunks (M tokens x 128 bf16).
__host__ __device__ constexpr uint32_t stage_bytes(int B, int M, int RT = 1, int SC = kSC) {
  return static_cast<uint32_t>(SC) * 256u * static_cast<uint32_t>(B * RT + M);
}

// Ring depth.  When the grid fits on the SMs in one wave, a CTA whose whole
// K slice fits in kWholeSlice bytes puts every stage of it in flight at once
// (latency decides).  Otherwise the register-limited number of resident CTAs
// per SM decides (CTAs of the next launches become resident early and stream
// their weights): the ring takes as many stages (at least two) as keep that
// many CTAs in shared memory, and no more than the CTA's slice needs.
// `fixed` is the shared memory a CTA needs besides its ring.
// MPW_GEMV_RING_KB replaces the rule by a fixed budget (tuning aid).
constexpr uint32_t kWholeSlice = 64u * 1024u;

int ring_stages(int B, int M, int stages_per_cta, bool few_ctas, int ctas_by_regs, uint32_t fixed, int RT = 1,
                int SC = kSC) {
  static const uint32_t budget = [] {
    const char* e = tuning_env("MPW_GEMV_RING_KB");
    const int v = e ? atoi(e) : 0;
    return v >= 8 && v <= 192 ? static_cast<uint32_t>(v) * 1024u : 0u;
  }();
  const uint32_t st = stage_bytes(B, M, RT, SC);
  int s;
  if (budget != 0) {
    s = static_cast<int>(budget / st);
  } else if (few_ctas && static_cast<uint32_t>(stages_per_cta) * st <= kWholeSlice) {
    s = stages_per_cta;
  } else {
    const DeviceInfo& d = device_info();
    const int per_cta = ctas_by_regs > 0 ? d.smem_per_sm / ctas_by_regs - d.smem_reserved : 0;
    s = per_cta > static_cast<int>(fixed) ? static_cast<int>((per_cta - fixed) / st) : 2;
    if (s > stages_per_cta) s = stages_per_cta;
  }
  return s < 2 ? 2 : (s > kMaxStages ? kMaxStages : s);
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

// CTAs per SM the register budget is sized for: wide codes and many tokens
// need more registers per thread (spill-free), narrow ones leave room for
// four CTAs.
template <int B, int NT>
constexpr int min_ctas() {
  return NT == 1 ? (B <= 7 ? 4 : 3) : (NT == 2 ? 2 : 1);
}

// Parts (MMAs per k step) of a code: paired rows take the combined scheme of
// the prefill GEMM (one part up to b = 9, lo7 + 128 * hi above), canonical
// rows the decode schemes of expand.cuh.
template <int B, bool PAIRED>
constexpr int dec_parts() {
  return PAIRED ? GemmParts<B>::parts : Exp<B>::parts;
}

// Paired rows with one part and one token tile fit in 56 registers up to
// b = 7 (seven CTAs per SM, no spills) and 64 at b = 8, 9 (six); with group
// scales (GRP) they need up to 64 (six; at 56 they would spill); the
// rms-scaled variant for one token needs a few more (five CTAs), the one for
// up to eight tokens keeps eight sums of squares and stays at four.
template <int B, int NT, int NSQ, bool PAIRED, bool GRP = false>
constexpr int min_ctas_for() {
  return PAIRED && dec_parts<B, PAIRED>() == 1 && NT == 1
             ? (NSQ > 1 ? 4 : (NSQ == 1 ? 5 : (B <= 7 && !GRP ? 7 : 6)))
             : min_ctas<B, NT>();
}

// NSQ: 0 = plain input; 1 or kNormMaxM = rms-scaled input for up to that
// many tokens (sums of squares kept per token).
// GRP: one scale per group of 128 << gshift consecutive codes of a row
// (scales [N, gstride]) instead of one per row: each 128-code chunk lies in
// one group, so a chunk's products are summed on their own and join the
// accumulator multiplied by the group's scale (fp32).
// MC: the number of tokens when it is fixed at compile time (1 for the one-
// token decode step), else 0 and M is read at run time.
// RT: 16-row tiles per CTA.  The RT tiles share each stage's x chunks (x is
// loaded once for 16*RT rows instead of once per 16), which matters when
// several tokens make x as large as the weights; consumer warp w takes tile
// w % RT and (SC / 4) * RT of the stage's chunks.
// SC: 128-code chunks per stage (8, or 4 when x makes stages so large that
// shared memory would hold too few CTAs).
template <int B, int NT, int NSQ, bool PAIRED, bool GRP = false, int MC = 0, int RT = 1, int SC = kSC>
__global__ void __launch_bounds__(kThreads, min_ctas_for<B, NT, NSQ, PAIRED, GRP>())
gemv_tma_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                int M_, const float* __restrict__ scales, int N, int K, uint16_t* __restrict__ y, int S,
                int flags, int32_t* err, int gstride, int gshift) {
  const int M = MC > 0 ? MC : M_;
  static_assert(!GRP || NSQ == 0, "group scales with the plain input only");
  constexpr int P = dec_parts<B, PAIRED>();
  constexpr bool NORM = NSQ > 0;
  constexpr int NS = NSQ > 0 ? NSQ : 1;
  static_assert(RT == 1 || RT == 2 || RT == 4, "row tiles per CTA");
  static_assert(SC == 4 || SC == 8, "chunks per stage");
  constexpr uint32_t kWChunk = 256u * B * RT;   // 16*RT rows x 16*B bytes
  constexpr int kCHW = (SC / kCW) * RT;         // chunks per consumer warp and stage
  const uint32_t x_chunk = 256u * M;            // M tokens x 128 bf16
  const uint32_t w_part = SC * kWChunk;
  const uint32_t st_bytes = stage_bytes(B, M, RT, SC);
  // dynamic: the ring (S stages), then, in clusters, the partial sums of the
  // cluster's CTAs
  extern __shared__ __align__(128) uint8_t tsmem[];
  __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
  __shared__ float red[kCW][NT][32][4];
  __shared__ float ss_red[kCW][NS];
  __shared__ float cl_ss[8][NS];
  __shared__ __align__(16) uint4 zero_x[4];   // x fragment of lanes without a token
  // cluster partial sums: [cluster rank][row tile][NT][32][4]
  auto cl_red = reinterpret_cast<float (*)[RT][NT][32][4]>(tsmem + static_cast<uint32_t>(S) * stage_bytes(B, M, RT, SC));

  if (flags & kXReady) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
  const int n_stages = ce > cb ? (ce - cb + SC - 1) / SC : 0;
  const int r0 = tile * 16 * RT;
  const uint32_t base = ptx::smem_addr(tsmem);
  const uint32_t bar0 = ptx::smem_addr(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kMaxStages + s); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kCW * 32);
    }
    ptx::mbar_fence_init();
  }
  if (threadIdx.x < 4) zero_x[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();

  if (warp == kCW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      ptx::prefetch_tmap(&tmap_w);
      ptx::prefetch_tmap(&tmap_x);
      const bool boxes = (flags & kStageBoxes) != 0;
      auto nvalid = [&](int s) { return min(SC, ce - (cb + SC * s)); };
      auto issue_w = [&](int s, int slot) {
        const int c0 = cb + SC * s, nv = nvalid(s);
        if (boxes) {
          // a box lands whole (zeros past the tensor); chunks past this
          // CTA's range are loaded and not read
          ptx::mbar_arrive_expect_tx(full(slot), st_bytes);
          ptx::tma_load_3d(base + slot * st_bytes, &tmap_w, full(slot), 0, r0, c0);
          return;
        }
        ptx::mbar_arrive_expect_tx(full(slot), nv * (kWChunk + x_chunk));
        for (int j = 0; j < nv; ++j)
          ptx::tma_load_2d(base + slot * st_bytes + j * kWChunk, &tmap_w, full(slot), (c0 + j) * 16 * B, r0);
      };
      auto issue_x = [&](int s, int slot) {
        const int c0 = cb + SC * s, nv = nvalid(s);
        if (boxes) {
          ptx::tma_load_3d(base + slot * st_bytes + w_part, &tmap_x, full(slot), 0, 0, c0);
          return;
        }
        for (int j = 0; j < nv; ++j)
          ptx::tma_load_2d(base + slot * st_bytes + w_part + j * x_chunk, &tmap_x, full(slot),
                           (c0 + j) * kChunk, 0);
      };
      const int pre = min(S, n_stages);
      // weights do not depend on the previous kernel in the stream; x does
      // unless the caller says otherwise
      if (flags & kXReady) {
        for (int s = 0; s < pre; ++s) {
          issue_w(s, s);
          issue_x(s, s);
        }
      } else {
        for (int s = 0; s < pre; ++s) issue_w(s, s);
        ptx::grid_dep_wait_then_release();
        for (int s = 0; s < pre; ++s) issue_x(s, s);
      }
      int issued = pre;
      int slot = 0;
      uint32_t phase = 0;   // phase of empty(slot) that frees it for stage s
      for (int s = pre; s < n_stages; ++s) {
        if (!ptx::mbar_wait(empty(slot), phase, err, ptx::wait_code(ptx::kWaitGemvTma, ptx::kWaitWEmpty))) break;
        issue_w(s, slot);
        issue_x(s, slot);
        issued = s + 1;
        if (++slot == S) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int s = max(0, issued - S); s < issued; ++s) ptx::mbar_wait(full(s % S), (s / S) & 1, err, ptx::wait_code(ptx::kWaitGemvTma, ptx::kWaitWTail));
    }
  } else {
    // ---------------- consumers ----------------
    float acc[2][NT][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[a][nt][0] = acc[a][nt][1] = acc[a][nt][2] = acc[a][nt][3] = 0.0f;
    float ss[NS];
#pragma unroll
    for (int t = 0; t < NS; ++t) ss[t] = 0.0f;

    // lanes without a token read a zero area (an address select, not a value
    // select per register)
    uint32_t x_lane[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) x_lane[nt] = (g + 8 * nt) * 256 + tig * 64;
    // this warp's row tile and its share of each stage's chunks
    const int rt = warp % RT, wsub = warp / RT;
    const uint32_t w_lane = rt * 256u * B + tig * 4 * B + g * 16 * B;
    // rows of this lane's accumulator entries (0, 1: row g; 2, 3: row g + 8)
    const int row_a = r0 + 16 * rt + g, row_b = row_a + 8;

    // One chunk (global index c): B words of rows g and g+8, the x fragment
    // of token g, expand, (release the stage after its last chunk), MMAs.
    auto chunk = [&](const uint8_t* st, int jc, int c, bool active, bool release, uint32_t rel_bar) {
      float gsa = 0.0f, gsb = 0.0f;   // group scales of rows g and g+8 (GRP)
      if constexpr (GRP) {
        if (active) {
          const int j = c >> gshift;
          if (row_a < N) gsa = __ldg(scales + static_cast<size_t>(row_a) * gstride + j);
          if (row_b < N) gsb = __ldg(scales + static_cast<size_t>(row_b) * gstride + j);
        }
      }
      uint32_t wa[B + 1], wb[B + 1];
      const uint8_t* wr = st + jc * kWChunk + w_lane;
      lds_words<B>(wr, wa);
      lds_words<B>(wr + 8 * 16 * B, wb);
      const uint8_t* xc = st + w_part + jc * x_chunk;
      uint32_t xw[NT][16];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4* px = g + 8 * nt < M ? reinterpret_cast<const uint4*>(xc + x_lane[nt]) : zero_x;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = px[q];
          xw[nt][4 * q] = v.x; xw[nt][4 * q + 1] = v.y; xw[nt][4 * q + 2] = v.z; xw[nt][4 * q + 3] = v.w;
        }
      }
      if (NORM && active && rt == 0) {
        // squares of x for the rms scale (the warps of the first row tile see
        // every chunk once): 4 of the chunk's 128 values per lane
#pragma unroll
        for (int t = 0; t < NS; ++t) {
          if (t < M) {
            const uint2 v = *reinterpret_cast<const uint2*>(xc + t * 256 + lane * 8);
            const float a0 = __uint_as_float(v.x << 16), a1 = __uint_as_float(v.x & 0xFFFF0000u);
            const float a2 = __uint_as_float(v.y << 16), a3 = __uint_as_float(v.y & 0xFFFF0000u);
            ss[t] = fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, fmaf(a3, a3, ss[t]))));
          }
        }
      }
      uint32_t va[P][16], vb[P][16];
      if constexpr (PAIRED) {
        gemm_expand_group<B, true>(wa, va);
        gemm_expand_group<B, true>(wb, vb);
      } else {
        expand_group<B>(wa, va);
        expand_group<B>(wb, vb);
      }
      if (release) {
        // Release the stage once its words are in registers, ordering this
        // thread's generic-proxy reads before the TMA (async-proxy) writes
        // that will refill the slot.
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(rel_bar);
      }
      if (active) {
        if constexpr (!PAIRED) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) permute_x<B>(xw[nt]);
        }
        if constexpr (GRP) {
          // the chunk's own sums, then scaled into the accumulator
          float pc[2][NT][4];
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) pc[a][nt][0] = pc[a][nt][1] = pc[a][nt][2] = pc[a][nt][3] = 0.0f;
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
#pragma unroll
            for (int part = 0; part < P; ++part)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_bf16(pc[(s2 * P + part) & 1][nt], va[part][2 * s2], vb[part][2 * s2], va[part][2 * s2 + 1],
                         vb[part][2 * s2 + 1], xw[nt][2 * s2], xw[nt][2 * s2 + 1]);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q)
              acc[0][nt][q] = fmaf(pc[0][nt][q] + pc[1][nt][q], q < 2 ? gsa : gsb, acc[0][nt][q]);
        } else {
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
#pragma unroll
            for (int part = 0; part < P; ++part)
#pragma unroll
              for (int nt = 0; nt < NT; ++nt)
                mma_bf16(acc[(s2 * P + part) & 1][nt], va[part][2 * s2], vb[part][2 * s2], va[part][2 * s2 + 1],
                         vb[part][2 * s2 + 1], xw[nt][2 * s2], xw[nt][2 * s2 + 1]);
        }
      }
    };

    int slot = 0;
    uint32_t phase = 0;
    uint32_t st_off = 0;
    for (int s = 0; s < n_stages; ++s) {
      if (!ptx::mbar_wait(full(slot), phase, err, ptx::wait_code(ptx::kWaitGemvTma, ptx::kWaitFull))) break;
      const uint8_t* st = tsmem + st_off;
      const int c_first = cb + SC * s + wsub * kCHW;
      if (cb + SC * (s + 1) <= ce) {
        // a whole stage: every chunk is in range
#pragma unroll
        for (int h = 0; h < kCHW; ++h) chunk(st, wsub * kCHW + h, c_first + h, true, h == kCHW - 1, empty(slot));
      } else {
#pragma unroll
        for (int h = 0; h < kCHW; ++h)
          chunk(st, wsub * kCHW + h, c_first + h, c_first + h < ce, h == kCHW - 1, empty(slot));
      }
      st_off += st_bytes;
      if (++slot == S) {
        slot = 0;
        phase ^= 1u;
        st_off = 0;
      }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) red[warp][nt][lane][q] = acc[0][nt][q] + acc[1][nt][q];
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

  // ---- reduce the K slices: warps, then the cluster; warp t finishes row
  // tile t ----
  if (warp < RT) {
    const int t_row = warp;
    float acc[NT][4];
    float ss[NS];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v = red[t_row][nt][lane][q];
#pragma unroll
        for (int w2 = t_row + RT; w2 < kCW; w2 += RT) v += red[w2][nt][lane][q];
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
      float* dst = cluster.map_shared_rank(&cl_red[0][0][0][0][0], 0);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[(((cr * RT + t_row) * NT + nt) * 32 + lane) * 4 + q] = acc[nt][q];
      if (NORM && t_row == 0 && lane == 0) {
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
            float v = cl_red[0][t_row][nt][lane][q];
            for (int r = 1; r < KC; ++r) v += cl_red[r][t_row][nt][lane][q];
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
      const int ra = r0 + 16 * t_row + g, rb = ra + 8;
      // with group scales the chunks were scaled as they were summed
      const float sca = GRP ? 1.0f : (ra < N ? __ldg(scales + ra) : 0.0f);
      const float scb = GRP ? 1.0f : (rb < N ? __ldg(scales + rb) : 0.0f);
      // y may be read or written by the previous kernel in the stream; with
      // kYFree it is not, and the first CTA's wait alone keeps this kernel
      // from completing before its predecessor
      if (!(flags & kYFree) || blockIdx.x == 0) asm volatile("griddepcontrol.wait;" ::: "memory");
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

// Cluster size: each tile is one cluster of kc CTAs.  One token: time is
// modelled as (CTAs per SM) x (chunks per consumer warp + a fixed cost of
// three chunks for start-up and the reduction), which splits K where the
// tiles alone leave SMs idle (down 5120x17408: two CTAs per tile; a recipe
// pass of dependent launches is 9% faster for it).  Several tokens: one CTA
// per tile (measured on gate 17408x5120 and down 5120x17408 at M = 4, 8, 16
// with two-tile CTAs: every split was slower, down M = 8 b = 6 60 against 66%
// of HBM).  The choice depends on the shape and M only, never on the call's
// flags, so that flagged and unflagged calls give the same bits.
int cluster_size(int tiles, int chunks, int num_sms, int M) {
  int best = 1;
  double best_t = 1e300;
  for (int kc = 1; kc <= (M == 1 ? 8 : 1); kc *= 2) {
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
    const char* e = tuning_env("MPW_GEMV_CLUSTER");
    const int v = e ? atoi(e) : 0;
    return (v == 1 || v == 2 || v == 4 || v == 8) ? v : 0;
  }();
  if (forced > 0 && kCW * forced <= chunks) best = forced;
  return best;
}

// gstride, gshift: group scales (GRP; see the kernel), else unused.
// MC, RT, SC: as for the kernel (M must equal MC when MC > 0).
// too_big: if not null, set (and nothing launched) when the configuration's
// shared memory would not fit one CTA, so that the caller can take fewer row
// tiles.
template <int B, int NT, int NSQ, bool PAIRED, bool GRP = false, int MC = 0, int RT = 1, int SC = kSC>
cudaError_t run_tma(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                    uint16_t* y, bool pdl, int flags, int32_t* err, cudaStream_t stream, int gstride = 0,
                    int gshift = 0, bool* too_big = nullptr) {
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  const int64_t rb = 16 * ((static_cast<int64_t>(K) * B + 127) / 128);
  const int chunks = (K + kChunk - 1) / kChunk;
  CUtensorMap tmap_w, tmap_x;
  // Whole-stage boxes need every chunk of a row inside the row (K % 128 ==
  // 0: rb == chunks * 16 * B), so that no in-bounds coordinate of the 3D
  // views addresses past the buffers.
  bool boxes = K % kChunk == 0;
  if (boxes) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(16 * B), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(chunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(16 * B)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(16 * B), static_cast<cuuint32_t>(16 * RT),
                               static_cast<cuuint32_t>(SC)};
    const cuuint32_t estr[3] = {1, 1, 1};
    boxes = encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(packed), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  if (boxes) {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kChunk), static_cast<cuuint64_t>(M),
                                static_cast<cuuint64_t>(chunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K) * 2, static_cast<cuuint64_t>(kChunk) * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(kChunk), static_cast<cuuint32_t>(M),
                               static_cast<cuuint32_t>(SC)};
    const cuuint32_t estr[3] = {1, 1, 1};
    boxes = encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  }
  if (boxes) {
    flags |= kStageBoxes;
  } else {
    // one 2D TMA per chunk: {16*B bytes x 16*RT rows} of W, {128 values x M} of x
    const cuuint64_t wdims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(N)};
    const cuuint64_t wstrides[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t wbox[2] = {static_cast<cuuint32_t>(16 * B), static_cast<cuuint32_t>(16 * RT)};
    const cuuint64_t xdims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t xstrides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t xbox[2] = {static_cast<cuuint32_t>(kChunk), static_cast<cuuint32_t>(M)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), wdims, wstrides, wbox,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), xdims, xstrides, xbox,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = gemv_tma_kernel<B, NT, NSQ, PAIRED, GRP, MC, RT, SC>;
  const int tiles = (N + 16 * RT - 1) / (16 * RT);
  const int kc = cluster_size(tiles, chunks, device_info().num_sms, M);
  const int per_cta = ((chunks + kc - 1) / kc + SC - 1) / SC;
  // resident CTAs per SM that registers and static shared memory allow
  static const int ctas_by_regs = [] {
    int n = 0;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, gemv_tma_kernel<B, NT, NSQ, PAIRED, GRP, MC, RT, SC>,
                                                         kThreads, 0) ==
                   cudaSuccess
               ? n
               : 0;
  }();
  const uint32_t cl_bytes = kc > 1 ? static_cast<uint32_t>(kc) * RT * NT * 32 * 4 * sizeof(float) : 0u;
  const uint32_t fixed = cl_bytes + static_cast<uint32_t>(sizeof(float)) * kCW * NT * 32 * 4 + 1024u;
  const int S = ring_stages(B, M, per_cta, tiles * kc <= device_info().num_sms, ctas_by_regs, fixed, RT, SC);
  const size_t smem = static_cast<size_t>(S) * stage_bytes(B, M, RT, SC) + cl_bytes;
  if (too_big != nullptr) {
    static const size_t static_smem = [] {
      cudaFuncAttributes a;
      return cudaFuncGetAttributes(&a, gemv_tma_kernel<B, NT, NSQ, PAIRED, GRP, MC, RT, SC>) == cudaSuccess
                 ? a.sharedSizeBytes
                 : size_t{16384};
    }();
    *too_big = smem + static_smem > static_cast<size_t>(device_info().max_smem_optin);
    if (*too_big) return cudaSuccess;
  }
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), smem);
  if (e != cudaSuccess) return e;
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
  return cudaLaunchKernelEx(&cfg, kern, tmap_w, tmap_x, M, scales, N, K, y, S, flags, err, gstride, gshift);
}

}  // namespace
}  // namespace mpw
