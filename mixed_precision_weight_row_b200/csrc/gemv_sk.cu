// Decode linear for M <= 32 tokens with an even split of the work over a
// persistent grid ("stream-K"):
//   y[m, n] = bf16(s_n * sum_k x[m, k] * q[n, k])
//
// DynaQuant, "Custom kernel architecture": packed N-bit weights are read from
// memory once, expanded in registers to a tensor-core format and multiplied;
// in decode the bytes saved are the speedup (quantization tutorial, closing
// note: the layer is bandwidth-bound).
//
// The work is U = T * C units: chunk c (128 codes of 16 rows) of 16-row tile
// t.  A grid of G CTAs, all resident, gives CTA b the contiguous units
// [b*U/G, (b+1)*U/G), so every SM streams the same number of bytes whatever
// the matrix shape.  Workspace layout: kCounterWords int32 counters (one per
// tile, the first T used), then T x kmax partial-sum slots.  A CTA's range is a sequence of tile segments; its
// producer warp streams them without a break through one TMA ring (weights
// box {16*B bytes x 16 rows} and x box {128 values x M tokens} per chunk)
// and its four consumer warps expand and multiply exactly as the per-tile
// decode kernel does (expand.cuh, mma.sync m16n8k16).  At the end of a
// segment the consumer warps reduce their partial sums through shared
// memory; a segment that covers its whole tile writes y at once.  A tile
// split between CTAs is combined through the caller's workspace: each
// contributor stores its partial sums in the tile's slot j (its rank among
// the tile's CTAs) and increments the tile's counter; the CTA that brings the
// counter to the number of contributors adds the slots in the order
// j = 0, 1, ... (the same order whichever CTA arrives last), writes y and
// resets the counter to zero for the next call.  No CTA ever waits for
// another.
//
// Programmatic dependent launch: the producer issues the weight loads of the
// first stages before griddepcontrol.wait and the x loads after it, and lets
// the next kernel in the stream launch once the wait has returned; the thread
// that writes y or the workspace waits first.  Every mbarrier wait is bounded (2 s); on
// time-out the kernel records an error in the device error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdlib>
#include <mutex>
#include <type_traits>

#include "expand.cuh"
#include "mpw.h"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

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
constexpr uint32_t kWholeSlice = 64u * 1024u;
// The workspace starts with a counter per tile at a fixed place, so that the
// partial sums of one call never land on the counters of another; calls with
// more tiles than this use the per-tile kernel.
constexpr int kCounterWords = 65536;

__host__ __device__ constexpr uint32_t stage_bytes(int B, int M) {
  return static_cast<uint32_t>(kSC) * 256u * static_cast<uint32_t>(B + M);
}

// floats in one partial-sum slot: the per-lane MMA fragments of a 16-row
// tile (NT x 32 lanes x 4) and the tokens' sums of squares (norm_input)
template <int NT>
__host__ __device__ constexpr int slot_floats() {
  return NT * 128 + kNormMaxM;
}

__device__ __forceinline__ int64_t range_begin(int b, int64_t U, int G) { return (U * b) / G; }

// The CTA whose range holds unit u.
__device__ __forceinline__ int owner_of(int64_t u, int64_t U, int G) {
  int b = static_cast<int>((u * G) / U);
  while (b + 1 < G && range_begin(b + 1, U, G) <= u) ++b;
  while (b > 0 && range_begin(b, U, G) > u) --b;
  return b;
}

// Walks a CTA's units stage by stage; a stage never crosses a tile.
struct StageIt {
  int64_t u, u1;
  int C;
  int t, c, c0, cend;   // tile, first chunk of the stage, first chunk of the segment, end of the segment
  __device__ void init(int64_t u0_, int64_t u1_, int C_) {
    u = u0_;
    u1 = u1_;
    C = C_;
    load();
  }
  __device__ void load() {
    if (u < u1) {
      t = static_cast<int>(u / C);
      c = static_cast<int>(u - static_cast<int64_t>(t) * C);
      c0 = c;
      const int64_t left = u1 - u;
      cend = left < C - c ? c + static_cast<int>(left) : C;
    }
  }
  __device__ bool valid() const { return u < u1; }
  __device__ int nv() const { return min(kSC, cend - c); }
  __device__ bool ends_segment() const { return c + kSC >= cend; }
  __device__ void next() {
    const int n = nv();
    u += n;
    c += n;
    if (c >= cend) load();
  }
};

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

template <int B, int NT, bool PAIRED>
constexpr int min_ctas_for() {
  return dec_parts<B, PAIRED>() == 1 && NT == 1 ? 4 : min_ctas<B, NT>();
}

template <int B, int NT, bool NORM, bool PAIRED>
__global__ void __launch_bounds__(kThreads, min_ctas_for<B, NT, PAIRED>())
gemv_sk_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x, int M,
               const float* __restrict__ scales, int N, int K, uint16_t* __restrict__ y, int S, int64_t U,
               int kmax, float* __restrict__ ws_part, int* __restrict__ ws_cnt, int32_t* err) {
  constexpr int P = dec_parts<B, PAIRED>();
  constexpr int NS = NORM ? kNormMaxM : 1;
  constexpr int SLOT = slot_floats<NT>();
  constexpr uint32_t kWChunk = 256u * B;        // 16 rows x 16*B bytes
  const uint32_t x_chunk = 256u * M;            // M tokens x 128 bf16
  const uint32_t w_part = kSC * kWChunk;
  const uint32_t st_bytes = stage_bytes(B, M);
  extern __shared__ __align__(128) uint8_t tsmem[];
  __shared__ __align__(8) uint64_t bars[2 * kMaxStages];
  __shared__ float red[2][kCW][NT][32][4];
  __shared__ float ss_red[2][kCW][NS];
  __shared__ __align__(16) uint4 zero_x[4];   // x fragment of lanes without a token

  const int G = static_cast<int>(gridDim.x);
  const int b = static_cast<int>(blockIdx.x);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const int C = (K + kChunk - 1) / kChunk;
  const int64_t u0 = range_begin(b, U, G), u1 = range_begin(b + 1, U, G);
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
      auto issue_w = [&](const StageIt& it, int slot) {
        const int nv = it.nv();
        ptx::mbar_arrive_expect_tx(full(slot), nv * (kWChunk + x_chunk));
        for (int j = 0; j < nv; ++j)
          ptx::tma_load_2d(base + slot * st_bytes + j * kWChunk, &tmap_w, full(slot), (it.c + j) * 16 * B,
                           it.t * 16);
      };
      auto issue_x = [&](const StageIt& it, int slot) {
        const int nv = it.nv();
        for (int j = 0; j < nv; ++j)
          ptx::tma_load_2d(base + slot * st_bytes + w_part + j * x_chunk, &tmap_x, full(slot),
                           (it.c + j) * kChunk, 0);
      };
      // weights of the first S stages do not depend on the previous kernel
      StageIt it;
      it.init(u0, u1, C);
      int pre = 0;
      for (; pre < S && it.valid(); ++pre, it.next()) issue_w(it, pre);
      ptx::grid_dep_wait_then_release();
      StageIt ix;
      ix.init(u0, u1, C);
      for (int s = 0; s < pre; ++s, ix.next()) issue_x(ix, s);
      int issued = pre;
      int slot = 0;
      uint32_t phase = 0;
      for (; it.valid(); it.next()) {
        if (!ptx::mbar_wait(empty(slot), phase, err, ptx::wait_code(ptx::kWaitGemvSk, ptx::kWaitWEmpty))) break;
        issue_w(it, slot);
        issue_x(it, slot);
        ++issued;
        if (++slot == S) {
          slot = 0;
          phase ^= 1u;
        }
      }
      // nothing may still be landing in shared memory when the CTA exits
      for (int s = max(0, issued - S); s < issued; ++s) ptx::mbar_wait(full(s % S), (s / S) & 1, err, ptx::wait_code(ptx::kWaitGemvSk, ptx::kWaitWTail));
    }
    return;
  }

  // ---------------- consumers ----------------
  float acc[2][NT][4];
  float ss[NS];
  auto clear = [&]() {
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) acc[a][nt][0] = acc[a][nt][1] = acc[a][nt][2] = acc[a][nt][3] = 0.0f;
#pragma unroll
    for (int t = 0; t < NS; ++t) ss[t] = 0.0f;
  };
  clear();
  uint32_t x_lane[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) x_lane[nt] = (g + 8 * nt) * 256 + tig * 64;
  const uint32_t w_lane = tig * 4 * B + g * 16 * B;

  auto chunk = [&](const uint8_t* st, int jc, bool active, bool release, uint32_t rel_bar) {
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
    if (NORM && active) {
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
      ptx::fence_proxy_async_smem();
      ptx::mbar_arrive(rel_bar);
    }
    if (active) {
      if constexpr (!PAIRED) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) permute_x<B>(xw[nt]);
      }
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
#pragma unroll
        for (int part = 0; part < P; ++part)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
            mma_bf16(acc[(s2 * P + part) & 1][nt], va[part][2 * s2], vb[part][2 * s2], va[part][2 * s2 + 1],
                     vb[part][2 * s2 + 1], xw[nt][2 * s2], xw[nt][2 * s2 + 1]);
    }
  };

  // y for the 16 rows of tile t from the tile's sums (warp 0's fragments)
  auto write_y = [&](int t, const float (&tot)[NT][4], const float (&sst)[NS]) {
    float inv[2] = {1.0f, 1.0f};
    if (NORM) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float v = 0.0f;
#pragma unroll
        for (int q = 0; q < NS; ++q) v = (q == 2 * tig + e) ? sst[q] : v;
        inv[e] = 1.0f / sqrtf(v / static_cast<float>(K) + 1e-6f);
      }
    }
    const int ra = t * 16 + g, rb = t * 16 + g + 8;
    const float sca = ra < N ? __ldg(scales + ra) : 0.0f;
    const float scb = rb < N ? __ldg(scales + rb) : 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int tok = 8 * nt + 2 * tig + (q & 1);
        const int row = (q < 2) ? ra : rb;
        if (tok < M && row < N) {
          const float o = tot[nt][q] * ((q < 2) ? sca : scb) * inv[q & 1];
          y[static_cast<size_t>(tok) * N + row] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        }
      }
  };

  StageIt it;
  it.init(u0, u1, C);
  int slot = 0;
  uint32_t phase = 0;
  uint32_t st_off = 0;
  int seg = 0;
  bool waited = false;
  // After a wait gives up the warp stops waiting and computing but still
  // walks every segment, so that all consumer warps meet at every barrier.
  bool ok = true;
  for (; it.valid(); it.next()) {
    if (ok && !ptx::mbar_wait(full(slot), phase, err, ptx::wait_code(ptx::kWaitGemvSk, ptx::kWaitFull))) ok = false;
    const uint8_t* st = tsmem + st_off;
    const int nv = it.nv();
    if (ok) {
#pragma unroll
      for (int h = 0; h < kCH; ++h)
        chunk(st, warp * kCH + h, warp * kCH + h < nv, h == kCH - 1, empty(slot));
    }
    st_off += st_bytes;
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
      st_off = 0;
    }
    if (!it.ends_segment()) continue;

    // ---- end of a tile segment: reduce the four warps' sums ----
    const int p = seg & 1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) red[p][warp][nt][lane][q] = acc[0][nt][q] + acc[1][nt][q];
    if (NORM) {
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        float v = ss[t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) ss_red[p][warp][t] = v;
      }
    }
    clear();
    asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
    if (warp == 0 && ok) {
      float tot[NT][4];
      float sst[NS];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v = red[p][0][nt][lane][q];
#pragma unroll
          for (int w2 = 1; w2 < kCW; ++w2) v += red[p][w2][nt][lane][q];
          tot[nt][q] = v;
        }
#pragma unroll
      for (int t = 0; t < NS; ++t) {
        float v = 0.0f;
        if (NORM) {
          v = ss_red[p][0][t];
#pragma unroll
          for (int w2 = 1; w2 < kCW; ++w2) v += ss_red[p][w2][t];
        }
        sst[t] = v;
      }
      if (!waited) {
        // y and the workspace may still be in use by the previous kernel
        asm volatile("griddepcontrol.wait;" ::: "memory");
        waited = true;
      }
      const int t = it.t;
      if (it.c0 == 0 && it.cend == C) {
        write_y(t, tot, sst);
      } else {
        const int64_t first = static_cast<int64_t>(t) * C;
        const int b0 = owner_of(first, U, G);
        const int nctb = owner_of(first + C - 1, U, G) - b0 + 1;
        float* mine = ws_part + (static_cast<int64_t>(t) * kmax + (b - b0)) * SLOT;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int q = 0; q < 4; ++q) mine[(nt * 32 + lane) * 4 + q] = tot[nt][q];
        if (NORM && lane < NS) {
          float v = 0.0f;
#pragma unroll
          for (int q = 0; q < NS; ++q) v = (q == lane) ? sst[q] : v;
          mine[NT * 128 + lane] = v;
        }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(ws_cnt + t, 1) == nctb - 1;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          __threadfence();
          // every contributor's slot, in slot order
#pragma unroll
          for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) tot[nt][q] = 0.0f;
#pragma unroll
          for (int q = 0; q < NS; ++q) sst[q] = 0.0f;
          const float* s0 = ws_part + static_cast<int64_t>(t) * kmax * SLOT;
          for (int j = 0; j < nctb; ++j) {
            const float* sj = s0 + static_cast<int64_t>(j) * SLOT;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
              for (int q = 0; q < 4; ++q) tot[nt][q] += __ldcg(sj + (nt * 32 + lane) * 4 + q);
            if (NORM) {
#pragma unroll
              for (int q = 0; q < NS; ++q) sst[q] += __ldcg(sj + NT * 128 + q);
            }
          }
          write_y(t, tot, sst);
          if (lane == 0) ws_cnt[t] = 0;
        }
      }
    }
    ++seg;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct OccEntry {
  const void* kernel;
  int device;
  size_t smem;
  int occ;
};
OccEntry g_occ[512];
int g_num_occ = 0;
std::mutex g_occ_mutex;

int occupancy(const void* kernel, size_t smem) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(g_occ_mutex);
  for (int i = 0; i < g_num_occ; ++i)
    if (g_occ[i].kernel == kernel && g_occ[i].device == dev && g_occ[i].smem == smem) return g_occ[i].occ;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, kThreads, smem) != cudaSuccess || occ < 1) occ = 1;
  if (g_num_occ < 512) g_occ[g_num_occ++] = OccEntry{kernel, dev, smem, occ};
  return occ;
}

struct SkPlan {
  int T, C, G, kmax, S;
  int64_t U;
  size_t smem;
};

int ring_depth(int B, int M, int stages_per_cta) {
  const uint32_t st = stage_bytes(B, M);
  int s = static_cast<uint32_t>(stages_per_cta) * st <= kWholeSlice ? stages_per_cta : 2;
  return s < 2 ? 2 : (s > kMaxStages ? kMaxStages : s);
}

// The grid: every SM holds `occ` CTAs (MPW_GEMV_SK_CTAS caps CTAs per SM,
// a tuning aid); no CTA gets fewer than kSC units unless there are fewer.
template <int B, int NT, bool NORM, bool PAIRED>
SkPlan plan_for(int M, int64_t N, int64_t K) {
  SkPlan p;
  p.T = static_cast<int>((N + 15) / 16);
  p.C = static_cast<int>((K + kChunk - 1) / kChunk);
  p.U = static_cast<int64_t>(p.T) * p.C;
  const int sms = device_info().num_sms;
  static const int cap = [] {
    const char* e = tuning_env("MPW_GEMV_SK_CTAS");
    const int v = e ? atoi(e) : 0;
    return v >= 1 && v <= 16 ? v : 0;
  }();
  // first guess of the per-CTA share, for the ring depth
  int64_t G = static_cast<int64_t>(sms) * 4;
  int64_t per = (p.U + G - 1) / G;
  p.S = ring_depth(B, M, static_cast<int>((per + kSC - 1) / kSC));
  p.smem = static_cast<size_t>(p.S) * stage_bytes(B, M);
  const void* kern = reinterpret_cast<const void*>(gemv_sk_kernel<B, NT, NORM, PAIRED>);
  int occ = ensure_smem_attr(kern, p.smem) == cudaSuccess ? occupancy(kern, p.smem) : 1;
  if (cap > 0 && occ > cap) occ = cap;
  G = static_cast<int64_t>(sms) * occ;
  const int64_t g_min_units = (p.U + kSC - 1) / kSC;   // at least kSC units per CTA
  if (G > g_min_units) G = g_min_units;
  if (G < 1) G = 1;
  p.G = static_cast<int>(G);
  const int64_t L = p.U / p.G;                         // shortest range
  p.kmax = static_cast<int>((p.C + L - 1) / L) + 1;
  return p;
}

template <int NT>
size_t workspace_bytes_for(const SkPlan& p) {
  if (p.T > kCounterWords) return 0;
  return static_cast<size_t>(kCounterWords) * 4 +
         static_cast<size_t>(p.T) * p.kmax * slot_floats<NT>() * sizeof(float);
}

template <int B, int NT, bool NORM, bool PAIRED>
cudaError_t run_sk(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K,
                   uint16_t* y, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t stream, bool* used) {
  *used = false;
  const SkPlan p = plan_for<B, NT, NORM, PAIRED>(M, N, K);
  const size_t need = workspace_bytes_for<NT>(p);
  if (ws == nullptr || need == 0 || ws_bytes < need) return cudaSuccess;   // caller falls back
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaSuccess;
  const int64_t rb = 16 * ((static_cast<int64_t>(K) * B + 127) / 128);
  CUtensorMap tmap_w, tmap_x;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(rb), static_cast<cuuint64_t>(N)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(16 * B), 16};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(packed), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kChunk), static_cast<cuuint32_t>(M)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(x), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = gemv_sk_kernel<B, NT, NORM, PAIRED>;
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kern), p.smem);
  if (e != cudaSuccess) return e;
  int* cnt = static_cast<int*>(ws);
  float* part = reinterpret_cast<float*>(cnt + kCounterWords);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.G));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  *used = true;
  return cudaLaunchKernelEx(&cfg, kern, tmap_w, tmap_x, M, scales, N, K, y, p.S, p.U, p.kmax, part, cnt, err);
}

template <int B, bool PAIRED>
cudaError_t sk_bits(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int N, int K, uint16_t* y,
                    bool norm, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t s, bool* used) {
  if (norm) return run_sk<B, 1, true, PAIRED>(x, M, packed, scales, N, K, y, ws, ws_bytes, err, s, used);
  if (M <= 8) return run_sk<B, 1, false, PAIRED>(x, M, packed, scales, N, K, y, ws, ws_bytes, err, s, used);
  if (M <= 16) return run_sk<B, 2, false, PAIRED>(x, M, packed, scales, N, K, y, ws, ws_bytes, err, s, used);
  return run_sk<B, 4, false, PAIRED>(x, M, packed, scales, N, K, y, ws, ws_bytes, err, s, used);
}

template <bool PAIRED>
cudaError_t sk_layout(const uint16_t* x, int M, const uint8_t* packed, const float* scales, int bits, int N, int K,
                      uint16_t* y, bool norm, void* ws, size_t ws_bytes, int32_t* err, cudaStream_t s,
                      bool* used) {
  switch (bits) {
    case 4: return sk_bits<4, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 5: return sk_bits<5, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 6: return sk_bits<6, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 7: return sk_bits<7, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 8: return sk_bits<8, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 9: return sk_bits<9, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 10: return sk_bits<10, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 11: return sk_bits<11, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 12: return sk_bits<12, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 13: return sk_bits<13, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 14: return sk_bits<14, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    case 15: return sk_bits<15, PAIRED>(x, M, packed, scales, N, K, y, norm, ws, ws_bytes, err, s, used);
    default: return cudaErrorInvalidValue;
  }
}

template <int B>
size_t ws_bits(int64_t M, int64_t N, int64_t K, bool norm, bool paired) {
  auto one = [&](auto nt_tag, auto norm_tag) -> size_t {
    constexpr int NT = decltype(nt_tag)::value;
    constexpr bool NORM_ = decltype(norm_tag)::value;
    if (paired) return workspace_bytes_for<NT>(plan_for<B, NT, NORM_, true>(static_cast<int>(M), N, K));
    return workspace_bytes_for<NT>(plan_for<B, NT, NORM_, false>(static_cast<int>(M), N, K));
  };
  using I1 = std::integral_constant<int, 1>;
  using I2 = std::integral_constant<int, 2>;
  using I4 = std::integral_constant<int, 4>;
  using T_ = std::true_type;
  using F_ = std::false_type;
  if (norm) return one(I1{}, T_{});
  if (M <= 8) return one(I1{}, F_{});
  if (M <= 16) return one(I2{}, F_{});
  return one(I4{}, F_{});
}

}  // namespace

bool gemv_sk_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm) {
  return M >= 1 && M <= 32 && (!norm || M <= kNormMaxM) && N >= 1 && K >= 1 && N < (1 << 30) && K % 8 == 0 &&
         (reinterpret_cast<uintptr_t>(x) & 15) == 0 && tensor_map_encoder() != nullptr;
}

size_t gemv_sk_workspace_bytes(int bits, int layout, int64_t M, int64_t N, int64_t K, bool norm) {
  const bool paired = layout == kLayoutPaired;
  switch (bits) {
    case 4: return ws_bits<4>(M, N, K, norm, paired);
    case 5: return ws_bits<5>(M, N, K, norm, paired);
    case 6: return ws_bits<6>(M, N, K, norm, paired);
    case 7: return ws_bits<7>(M, N, K, norm, paired);
    case 8: return ws_bits<8>(M, N, K, norm, paired);
    case 9: return ws_bits<9>(M, N, K, norm, paired);
    case 10: return ws_bits<10>(M, N, K, norm, paired);
    case 11: return ws_bits<11>(M, N, K, norm, paired);
    case 12: return ws_bits<12>(M, N, K, norm, paired);
    case 13: return ws_bits<13>(M, N, K, norm, paired);
    case 14: return ws_bits<14>(M, N, K, norm, paired);
    case 15: return ws_bits<15>(M, N, K, norm, paired);
    default: return 0;
  }
}

cudaError_t launch_gemv_sk(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                           int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, void* ws, size_t ws_bytes,
                           cudaStream_t stream, bool* used) {
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  int32_t* err = device_error_word();
  if (layout == kLayoutPaired)
    return sk_layout<true>(x, m, packed, scales, bits, n, k, y, norm, ws, ws_bytes, err, stream, used);
  return sk_layout<false>(x, m, packed, scales, bits, n, k, y, norm, ws, ws_bytes, err, stream, used);
}

}  // namespace mpw

// ---------------------------------------------------------------------------
// mpw_qlinear_noalloc: the stream-K decode linear with its workspace in a
// fixed device array, for callers that cannot allocate device memory.
// ---------------------------------------------------------------------------

namespace mpw {

// Zero-initialised when the library is loaded; every device holds a copy.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MPW_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of the array on the current device, looked up once per
// device (with that device current).  nullptr if the lookup failed.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace mpw

extern "C" MPW_API mpw_status mpw_qlinear_noalloc(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                                          int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                          mpw_stream_t stream) {
  using namespace mpw;
  auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) != 0; };
  if (bits < kMinBits || bits > kMaxBits) return MPW_E_UNSUPPORTED_BITS;
  if (x == nullptr || packed == nullptr || scales == nullptr || y == nullptr) return MPW_E_INVALID_ARG;
  if (M < 1 || M > 32 || N < 1 || K < 1 || N > 0x7fffffff || K > 0x3fffffff) return MPW_E_INVALID_ARG;
  if (layout != kLayoutCanonical && layout != kLayoutPaired) return MPW_E_INVALID_ARG;
  if (layout == kLayoutPaired && K % 32 != 0) return MPW_E_INVALID_ARG;
  if (misaligned(packed, 16) || misaligned(x, 16) || misaligned(y, 2) || misaligned(scales, 4))
    return MPW_E_MISALIGNED;
  if (!gemv_sk_supported(x, M, N, K, false)) return MPW_E_INVALID_ARG;
  const size_t need = gemv_sk_workspace_bytes(bits, layout, M, N, K, false);
  if (need == 0 || need > MPW_NOALLOC_SCRATCH_BYTES) return MPW_E_SCRATCH_LIMIT;
  void* ws = noalloc_scratch();
  if (ws == nullptr) return MPW_E_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the counters of the call's tiles (first in the workspace) must start at zero
  const size_t counter_bytes = static_cast<size_t>((N + 15) / 16) * 4;
  if (cudaMemsetAsync(ws, 0, counter_bytes, s) != cudaSuccess) return MPW_E_CUDA;
  bool used = false;
  const cudaError_t e = launch_gemv_sk(x, packed, scales, bits, layout, M, N, K, y, false, ws,
                                       MPW_NOALLOC_SCRATCH_BYTES, s, &used);
  if (e != cudaSuccess || !used) return MPW_E_CUDA;
  return MPW_OK;
}
