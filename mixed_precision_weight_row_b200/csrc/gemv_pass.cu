// A whole decode pass (one token) over a stack of linears in ONE persistent
// kernel:  for each linear l in order, y_l[n] = bf16(s_n * r * sum_k x_l[k] q_l[n, k])
// with r the rms scale of x_l when the linear reads its input normalised.
//
// DynaQuant, "Custom kernel architecture" and "Step 3" (every matrix of the
// stack carries its own bit width): in decode the packed bytes streamed are
// the cost, so the pass is as fast as the weights can be streamed.  Launched
// one kernel per linear, every linear that depends on its predecessor starts
// with the GPU nearly idle (a lone grid at two or three CTAs per SM streams
// far below the copy bandwidth).  Here every SM keeps streaming across the
// linears: while a CTA waits for the linears its next item depends on, its
// ring already holds that item's weights.
//
// Work items are (linear, 16-row tile, K part), numbered linear after linear,
// tile-major; CTA c of G takes items c, c + G, c + 2G, ...  A linear's K range
// is split into `parts` runs of whole stages when its tiles alone would leave
// CTAs idle; the parts' partial sums (and sums of squares of x) go to a
// record each, and the part that finishes last adds the records in part
// order, so the result does not depend on which CTA arrives last.
//
// Each CTA has one producer warp and four consumer warps, as the per-tile
// decode kernel (gemv_tma.cuh): a ring of S stages of eight 128-code chunks,
// the packed rows by one 3D TMA per stage ({16*B bytes x 16 rows x 8 chunks},
// tensor maps in global memory, one per linear) and x by one bulk copy
// (M = 1: the stage's 8 x 128 values are contiguous).  Consumers expand the
// paired-halves codes to exact bf16 (expand.cuh) and multiply on tensor cores
// (mma.sync m16n8k16); the bit width is read per item (b = 4..8).
//
// Dependencies.  The host lists for every linear the earlier linears that
// write bytes it reads, or read or write bytes it writes, minus those that
// another listed one already depends on (transitively).  A linear's item
// loads x only after each listed linear has finished all its tiles: every
// tile's last writer bumps the linear's `done` counter (release) after its y
// stores and a proxy fence; the producer polls the counters (acquire), fences
// the async proxy and then issues the x copies.  Items wait only on items of
// earlier linears, which come earlier in every CTA's sequence, and all CTAs
// are resident at once (the grid is sized by the occupancy calculator), so
// the earliest unfinished item can always proceed.  Every wait is bounded
// and ends early once another wait has set the error word.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "expand.cuh"
#include "mpw.h"
#include "mpw_internal.h"
#include "tc_ptx.cuh"

namespace mpw {
namespace {

using namespace dec;

constexpr int kPW = 4;                    // consumer warps (0..3)
constexpr int kProducerWarp = kPW;        // warp 4: TMA producer
constexpr int kEpilogueWarp = kPW + 1;    // warp 5: finishes items
constexpr int kPThreads = (kPW + 2) * 32;
constexpr int kPSC = 8;                   // chunks per stage (two per consumer warp)
constexpr int kPMaxStages = 8;
constexpr int kPassCtas = 4;              // CTAs per SM the kernel is compiled for
constexpr int kRecFloats = 32;            // one partial-sum record: 16 rows, the sum of squares, padding
constexpr int kEQ = 3;                    // items the epilogue warp may lag behind the consumers
// item descriptors in flight: the producer runs at most (ring stages) items
// ahead of the consumers, which run at most kEQ items ahead of the epilogue
constexpr int kDQ = kPMaxStages + kEQ + 2;

struct PassLinear {
  const uint16_t* x;          // input, K values
  uint16_t* y;                // output, N values
  const float* scales;        // [N]
  const CUtensorMap* tmap;    // packed rows as [chunk][row][16*B bytes]
  long long item0;            // first item of this linear
  long long rec0;             // first partial-sum record (parts > 1)
  int N, K, bits, norm;
  int tiles, parts, stages;   // 16-row tiles, K parts per tile, stages per row
  int dep0, ndep;             // deps[dep0 .. dep0 + ndep)
  int cnt0;                   // first tile counter (parts > 1)
};

struct PassParams {
  const PassLinear* lin;
  const int32_t* deps;
  int32_t* done;              // [L]: tiles of each linear finished
  int32_t* tile_cnt;          // parts of each split tile finished
  float* rec;                 // partial-sum records
  long long items;
  int L;
  int S;
  uint32_t slot_bytes;
  int32_t* err;
  int32_t* abort;             // set when a wait gives up (zeroed with the counters before each run)
};

// What the consumers and the epilogue warp need of an item; written by the
// producer before it issues the item's first stage.
struct ItemDesc {
  long long rec;              // first record of the item's tile (parts > 1)
  int l, tile, part, parts;
  int n, cb, chunks, bits;    // stages, first chunk, chunks per row, width
  int norm, N, K, cnt;        // cnt: the tile's counter (parts > 1)
};

// Shared memory of the kernel, at namespace scope so that the per-width item
// functions reach it without pointer arguments.
extern __shared__ __align__(128) uint8_t pring[];           // the ring: S slots
__shared__ __align__(8) uint64_t pbars[2 * kPMaxStages];     // full[s], empty[s]
__shared__ __align__(8) uint64_t pebars[2 * kEQ];            // epilogue queue: filled[e], free[e]
__shared__ float pred[kEQ][kPW][8][2];                       // queue entry, warp, g: rows g and g + 8
__shared__ float pss[kEQ][kPW];                              // queue entry, warp: sums of squares
__shared__ ItemDesc pdesc[kDQ];
__shared__ __align__(16) uint4 pzero[4];                     // x fragment of lanes without a token

__device__ __forceinline__ int part_stage(int part, int stages, int parts) { return (part * stages) / parts; }

template <int B>
__device__ __forceinline__ void pass_lds(const uint8_t* p, uint32_t (&w)[B + 1]) {
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

// The consumer side of one item of width B: n stages from the ring starting
// at (slot, phase), then the warp's sums for token 0 (rows g and g + 8) and,
// with norm, its sum of squares of x into epilogue queue entry e (once the
// epilogue warp has freed it: parity ephase).  A separate function per width
// (not inlined), so that each keeps its own registers.  Returns false if a
// wait gave up.
template <int B>
__device__ __noinline__ bool pass_item(uint32_t slot_bytes, int S, int n, int chunk_begin, int chunks, bool norm,
                                       int slot, uint32_t phase, int e, uint32_t ephase, bool ewait, int32_t* err,
                                       int32_t* abort) {
  static_assert(GemmParts<B>::parts == 1, "one operand per code");
  constexpr uint32_t kWChunk = 256u * B;           // 16 rows x 16*B bytes
  constexpr uint32_t w_part = kPSC * kWChunk;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, tig = lane & 3;
  const uint32_t w_lane = tig * 4u * B + g * 16u * B;
  const uint32_t bar0 = ptx::smem_addr(pbars);
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  float ss = 0.0f;
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    if (!ptx::mbar_wait_abortable(bar0 + 8u * slot, phase, err,
                                  ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitFull), abort))
      return false;
    const uint8_t* st = pring + static_cast<uint32_t>(slot) * slot_bytes;
    const int nvalid = chunks - (chunk_begin + kPSC * i);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int jc = 2 * warp + h;
      const bool active = jc < nvalid;
      uint32_t wa[B + 1], wb[B + 1];
      const uint8_t* wr = st + jc * kWChunk + w_lane;
      pass_lds<B>(wr, wa);
      pass_lds<B>(wr + 8 * 16 * B, wb);
      const uint8_t* xc = st + w_part + jc * 256;
      uint32_t xw[16];
      const uint4* px = g == 0 ? reinterpret_cast<const uint4*>(xc + tig * 64) : pzero;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = px[q];
        xw[4 * q] = v.x; xw[4 * q + 1] = v.y; xw[4 * q + 2] = v.z; xw[4 * q + 3] = v.w;
      }
      if (norm && active) {
        // squares of x for the rms scale: 4 of the chunk's 128 values per lane
        const uint2 v = *reinterpret_cast<const uint2*>(xc + lane * 8);
        const float a0 = __uint_as_float(v.x << 16), a1 = __uint_as_float(v.x & 0xFFFF0000u);
        const float a2 = __uint_as_float(v.y << 16), a3 = __uint_as_float(v.y & 0xFFFF0000u);
        ss = fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, fmaf(a3, a3, ss))));
      }
      uint32_t va[1][16], vb[1][16];
      gemm_expand_group<B, true>(wa, va);
      gemm_expand_group<B, true>(wb, vb);
      if (h == 1) {
        // release the slot once its words are in registers (generic reads
        // ordered before the async-proxy writes that refill it)
        ptx::fence_proxy_async_smem();
        ptx::mbar_arrive(bar0 + 8u * (kPMaxStages + slot));
      }
      if (active) {
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2)
          mma_bf16(acc[s2 & 1], va[0][2 * s2], vb[0][2 * s2], va[0][2 * s2 + 1], vb[0][2 * s2 + 1], xw[2 * s2],
                   xw[2 * s2 + 1]);
      }
    }
    if (++slot == S) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (norm) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  }
  const uint32_t ebar0 = ptx::smem_addr(pebars);
  if (ewait && !ptx::mbar_wait_abortable(ebar0 + 8u * (kEQ + e), ephase, err,
                                         ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitAcc), abort))
    return false;
  // token 0 sits in accumulator entries 0 (row g) and 2 (row g + 8) of the
  // lanes with tig == 0
  if (tig == 0) {
    pred[e][warp][g][0] = acc[0][0] + acc[1][0];
    pred[e][warp][g][1] = acc[0][2] + acc[1][2];
  }
  if (norm && lane == 0) pss[e][warp] = ss;
  ptx::mbar_arrive(ebar0 + 8u * e);
  return true;
}

// Item j -> (linear, tile, part); `l` only moves forward.
struct ItemPos {
  int tile, part;
};

__device__ __forceinline__ ItemPos locate(const PassLinear* lin, long long j, int& l) {
  while (j >= lin[l].item0 + static_cast<long long>(lin[l].tiles) * lin[l].parts) ++l;
  const long long local = j - lin[l].item0;
  const int parts = lin[l].parts;
  return ItemPos{static_cast<int>(local / parts), static_cast<int>(local % parts)};
}

__global__ void __launch_bounds__(kPThreads, kPassCtas) gemv_pass_kernel(const __grid_constant__ PassParams p) {
  const int S = p.S;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t base = ptx::smem_addr(pring);
  const uint32_t bar0 = ptx::smem_addr(pbars);
  const uint32_t ebar0 = ptx::smem_addr(pebars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kPMaxStages + s); };
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), kPW * 32);
    }
    for (int e = 0; e < kEQ; ++e) {
      ptx::mbar_init(ebar0 + 8u * e, kPW * 32);   // filled by the consumer threads
      ptx::mbar_init(ebar0 + 8u * (kEQ + e), 1);  // freed by the epilogue warp
    }
    ptx::mbar_fence_init();
  }
  if (threadIdx.x < 4) pzero[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  const long long G = gridDim.x;

  if (warp == kProducerWarp) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    int slot = 0;
    uint32_t phase = 0;
    long long issued = 0;
    bool dead = false;
    int l = 0;
    int l_ready = -1;  // the last linear whose dependencies this thread saw finished
    long long k = 0;   // this CTA's item count
    for (long long j = blockIdx.x; j < p.items && !dead; j += G, ++k) {
      const ItemPos pos = locate(p.lin, j, l);
      const PassLinear& L = p.lin[l];
      const int B = L.bits, chunks = L.K / 128;
      const int sb = part_stage(pos.part, L.stages, L.parts), se = part_stage(pos.part + 1, L.stages, L.parts);
      const int n = se - sb;
      const uint32_t w_part = 2048u * B;
      const uint8_t* xg = reinterpret_cast<const uint8_t*>(L.x);
      {
        ItemDesc& d = pdesc[k % kDQ];
        d.rec = L.rec0 + static_cast<long long>(pos.tile) * L.parts;
        d.l = l;
        d.tile = pos.tile;
        d.part = pos.part;
        d.parts = L.parts;
        d.n = n;
        d.cb = sb * kPSC;
        d.chunks = chunks;
        d.bits = B;
        d.norm = L.norm;
        d.N = L.N;
        d.K = L.K;
        d.cnt = L.cnt0 + pos.tile;
      }
      {
        // the descriptor of this CTA's next item, for the TMA unit
        int l2 = l;
        const long long j2 = j + G;
        if (j2 < p.items) {
          while (j2 >= p.lin[l2].item0 + static_cast<long long>(p.lin[l2].tiles) * p.lin[l2].parts) ++l2;
          if (l2 != l) ptx::prefetch_tmap(p.lin[l2].tmap);
        }
      }
      // x is ready when every linear this one depends on has finished (seen
      // once per linear: the counters only grow)
      bool ready = l == l_ready;
      if (!ready) {
        ready = true;
        for (int d = 0; d < L.ndep && ready; ++d) {
          const int dl = p.deps[L.dep0 + d];
          ready = ptx::ld_acquire_gpu(p.done + dl) >= p.lin[dl].tiles;
        }
        if (ready) {
          ptx::fence_proxy_async_global();
          l_ready = l;
        }
      }
      int nd = 0;
      int dslot[kPMaxStages], dc0[kPMaxStages];
      for (int i = 0; i < n; ++i) {
        if (issued >= S && !ptx::mbar_wait_abortable(empty(slot), phase ^ 1u, p.err,
                                                      ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitWEmpty),
                                                      p.abort)) {
          // complete the stages already issued, so that their copies can be
          // waited for below
          for (int e = 0; e < nd; ++e)
            ptx::bulk_load(base + static_cast<uint32_t>(dslot[e]) * p.slot_bytes + w_part,
                           xg + static_cast<size_t>(dc0[e]) * 256, 256u * min(kPSC, chunks - dc0[e]), full(dslot[e]));
          dead = true;
          break;
        }
        const int c0 = (sb + i) * kPSC;
        const int nv = min(kPSC, chunks - c0);
        const uint32_t dst = base + static_cast<uint32_t>(slot) * p.slot_bytes;
        ptx::mbar_arrive_expect_tx(full(slot), w_part + 256u * nv);
        ptx::tma_load_3d(dst, L.tmap, full(slot), 0, pos.tile * 16, c0);
        if (ready) {
          ptx::bulk_load(dst + w_part, xg + static_cast<size_t>(c0) * 256, 256u * nv, full(slot));
        } else {
          dslot[nd] = slot;
          dc0[nd] = c0;
          ++nd;
        }
        ++issued;
        if (++slot == S) {
          slot = 0;
          phase ^= 1u;
        }
        if (!ready && (nd == S || i == n - 1)) {
          // the weights of the first stages are in flight; now wait for x
          for (int d = 0; d < L.ndep; ++d) {
            const int dl = p.deps[L.dep0 + d];
            if (!ptx::counter_wait(p.done + dl, p.lin[dl].tiles, p.err,
                                   ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitDeps), p.abort))
              dead = true;
          }
          ptx::fence_proxy_async_global();
          ready = true;
          l_ready = l;
          // issued even after a failed wait: the stages' barriers expect the bytes
          for (int e = 0; e < nd; ++e) {
            const int nv2 = min(kPSC, chunks - dc0[e]);
            ptx::bulk_load(base + static_cast<uint32_t>(dslot[e]) * p.slot_bytes + w_part,
                           xg + static_cast<size_t>(dc0[e]) * 256, 256u * nv2, full(dslot[e]));
          }
          nd = 0;
          if (dead) break;
        }
      }
    }
    // nothing may still be landing in shared memory when the CTA exits (every
    // issued stage has all its copies issued, so these waits end)
    for (long long t = issued - S > 0 ? issued - S : 0; t < issued; ++t)
      ptx::mbar_wait(full(static_cast<int>(t % S)), static_cast<uint32_t>((t / S) & 1), p.err,
                     ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitWTail));
    return;
  }

  if (warp == kEpilogueWarp) {
    // ---------------- epilogue: finish items in order ----------------
    const int r = lane & 15;   // lane r < 16 finishes row r of the tile
    long long k = 0;
    for (long long j = blockIdx.x; j < p.items; j += G, ++k) {
      const int e = static_cast<int>(k % kEQ);
      if (!ptx::mbar_wait_abortable(ebar0 + 8u * e, static_cast<uint32_t>((k / kEQ) & 1), p.err,
                                    ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitAcc), p.abort))
        return;
      const ItemDesc& d = pdesc[k % kDQ];
      const bool norm = d.norm != 0;
      float v = 0.0f, sq = 0.0f;
#pragma unroll
      for (int w = 0; w < kPW; ++w) {
        v += pred[e][w][r & 7][r >> 3];   // [g][0]: row g, [g][1]: row g + 8
        if (norm) sq += pss[e][w];
      }
      const int l = d.l, row = d.tile * 16 + r, parts = d.parts, N = d.N, K = d.K;
      const long long rec = d.rec;
      const int part = d.part, cnt = d.cnt;
      // the entry may be refilled once its values are in registers
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(ebar0 + 8u * (kEQ + e));
      bool finish = true;
      if (parts > 1) {
        float* mine = p.rec + (rec + part) * kRecFloats;
        if (lane < 16) mine[r] = v;
        if (lane == 16) mine[16] = sq;
        __syncwarp();
        // the increment releases this warp's record stores (ordered before
        // it by the warp barrier) and acquires those of the parts before
        int prior = 0;
        if (lane == 0) prior = ptx::atom_add_acq_rel_gpu(p.tile_cnt + cnt, 1);
        prior = __shfl_sync(0xffffffffu, prior, 0);
        __syncwarp();   // the other lanes' loads below come after lane 0's acquire
        finish = prior == parts - 1;
        if (finish) {
          const float* r0 = p.rec + rec * kRecFloats;
          v = 0.0f;
          sq = 0.0f;
          for (int q = 0; q < parts; ++q) {
            v += __ldcg(r0 + q * kRecFloats + r);
            sq += __ldcg(r0 + q * kRecFloats + 16);
          }
        }
      }
      if (finish) {
        const float inv = norm ? 1.0f / sqrtf(sq / static_cast<float>(K) + 1e-6f) : 1.0f;
        if (lane < 16 && row < N) {
          const PassLinear& L = p.lin[l];
          const float o = v * __ldg(L.scales + row) * inv;
          L.y[row] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        }
        __syncwarp();
        // release (cumulative over the warp's y stores, which the warp
        // barrier orders before it): the tile counts as finished only once
        // they are visible at gpu scope; readers fence their async proxy
        if (lane == 0) ptx::red_release_gpu_add(p.done + l, 1);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  long long gs = 0;       // stages of this CTA's sequence consumed so far
  long long k = 0;
  for (long long j = blockIdx.x; j < p.items; j += G, ++k) {
    const int slot = static_cast<int>(gs % S);
    const uint32_t phase = static_cast<uint32_t>((gs / S) & 1);
    // the item's first stage is loaded: its descriptor was written before
    if (!ptx::mbar_wait_abortable(full(slot), phase, p.err, ptx::wait_code(ptx::kWaitGemvPass, ptx::kWaitFull),
                                  p.abort))
      return;
    const ItemDesc& d = pdesc[k % kDQ];
    const int n = d.n, cb = d.cb, chunks = d.chunks, bits = d.bits;
    const bool norm = d.norm != 0;
    const int e = static_cast<int>(k % kEQ);
    const uint32_t ephase = static_cast<uint32_t>(((k / kEQ) - 1) & 1);
    const bool ewait = k >= kEQ;
    bool ok;
    switch (bits) {
      case 4: ok = pass_item<4>(p.slot_bytes, S, n, cb, chunks, norm, slot, phase, e, ephase, ewait, p.err, p.abort); break;
      case 5: ok = pass_item<5>(p.slot_bytes, S, n, cb, chunks, norm, slot, phase, e, ephase, ewait, p.err, p.abort); break;
      case 6: ok = pass_item<6>(p.slot_bytes, S, n, cb, chunks, norm, slot, phase, e, ephase, ewait, p.err, p.abort); break;
      case 7: ok = pass_item<7>(p.slot_bytes, S, n, cb, chunks, norm, slot, phase, e, ephase, ewait, p.err, p.abort); break;
      default: ok = pass_item<8>(p.slot_bytes, S, n, cb, chunks, norm, slot, phase, e, ephase, ewait, p.err, p.abort); break;
    }
    // a wait that gave up: the error word and the abort word are set; the
    // other roles give up at their next wait
    if (!ok) return;
    gs += n;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

struct Range {
  uintptr_t lo, hi;
  bool overlaps(const Range& o) const { return lo < o.hi && o.lo < hi; }
};

}  // namespace

struct PassPlan {
  void* dev = nullptr;          // one allocation: descriptors, tensor maps, deps, counters, records
  PassParams params{};
  size_t counter_bytes = 0;     // done + tile counters, zeroed before every run
  int32_t* counters = nullptr;
  int grid = 0;
  size_t smem = 0;
};

bool gemv_pass_dependencies(const PassLayer* layers, int64_t count, std::vector<int32_t>& deps,
                            std::vector<int32_t>& dep0) {
  // conflicting earlier linears, minus those another listed one already
  // covers (ancestor sets as bitsets; scanned from the nearest linear back)
  const int L = static_cast<int>(count);
  const int words = (L + 63) / 64;
  std::vector<uint64_t> anc(static_cast<size_t>(L) * words, 0ull);
  deps.clear();
  dep0.assign(static_cast<size_t>(L) + 1, 0);
  for (int i = 0; i < L; ++i) {
    const PassLayer& A = layers[i];
    const Range in{reinterpret_cast<uintptr_t>(A.x), reinterpret_cast<uintptr_t>(A.x) + 2u * A.K};
    const Range outr{reinterpret_cast<uintptr_t>(A.y), reinterpret_cast<uintptr_t>(A.y) + 2u * A.N};
    if (in.overlaps(outr)) return false;
    uint64_t* mine = anc.data() + static_cast<size_t>(i) * words;
    dep0[static_cast<size_t>(i)] = static_cast<int32_t>(deps.size());
    for (int jx = i - 1; jx >= 0; --jx) {
      if (mine[jx / 64] >> (jx % 64) & 1ull) continue;   // covered already
      const PassLayer& Bj = layers[jx];
      const Range bin{reinterpret_cast<uintptr_t>(Bj.x), reinterpret_cast<uintptr_t>(Bj.x) + 2u * Bj.K};
      const Range bout{reinterpret_cast<uintptr_t>(Bj.y), reinterpret_cast<uintptr_t>(Bj.y) + 2u * Bj.N};
      if (!(bout.overlaps(in) || bin.overlaps(outr) || bout.overlaps(outr))) continue;
      deps.push_back(jx);
      const uint64_t* theirs = anc.data() + static_cast<size_t>(jx) * words;
      for (int w = 0; w < words; ++w) mine[w] |= theirs[w];
      mine[jx / 64] |= 1ull << (jx % 64);
    }
  }
  dep0[static_cast<size_t>(L)] = static_cast<int32_t>(deps.size());
  return true;
}

bool gemv_pass_layer_ok(int bits, int layout, int64_t N, int64_t K) {
  return layout == kLayoutPaired && bits >= 4 && bits <= 8 && K >= 128 && K % 128 == 0 && N >= 1 &&
         N < (1LL << 30) && K < (1LL << 30);
}

cudaError_t gemv_pass_create(const PassLayer* layers, int64_t count, PassPlan** out) {
  *out = nullptr;
  auto encode = tensor_map_encoder();
  if (encode == nullptr) return cudaErrorNotSupported;
  const DeviceInfo& d = device_info();
  const int L = static_cast<int>(count);
  int bmax = 4;
  for (int i = 0; i < L; ++i) bmax = std::max(bmax, layers[i].bits);
  const uint32_t slot_bytes = 2048u * static_cast<uint32_t>(bmax + 1);
  // ring depth: as many stages as keep kPassCtas CTAs per SM in shared memory
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, gemv_pass_kernel);
  if (e != cudaSuccess) return e;
  const int per_cta = d.smem_per_sm / kPassCtas - d.smem_reserved - static_cast<int>(fa.sharedSizeBytes);
  int S = per_cta > 0 ? per_cta / static_cast<int>(slot_bytes) : 0;
  S = std::min(std::max(S, 2), kPMaxStages);
  const size_t smem = static_cast<size_t>(S) * slot_bytes;
  e = ensure_smem_attr(reinterpret_cast<const void*>(gemv_pass_kernel), smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, gemv_pass_kernel, kPThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const long long G = static_cast<long long>(occ) * d.num_sms;

  std::vector<int32_t> deps, dep0;
  if (!gemv_pass_dependencies(layers, count, deps, dep0)) return cudaErrorInvalidValue;
  std::vector<PassLinear> lin(static_cast<size_t>(L));
  long long items = 0, recs = 0;
  int cnts = 0;
  for (int i = 0; i < L; ++i) {
    const PassLayer& A = layers[i];
    PassLinear& P = lin[static_cast<size_t>(i)];
    P.x = A.x;
    P.y = A.y;
    P.scales = A.scales;
    P.N = static_cast<int>(A.N);
    P.K = static_cast<int>(A.K);
    P.bits = A.bits;
    P.norm = A.norm ? 1 : 0;
    P.tiles = static_cast<int>((A.N + 15) / 16);
    P.stages = static_cast<int>((A.K / 128 + kPSC - 1) / kPSC);
    // split K into as many parts as keep the linear's items within one
    // round of the grid (a second, partial round would double its time)
    long long parts = G / P.tiles;
    parts = std::min<long long>(std::max<long long>(parts, 1), P.stages);
    P.parts = static_cast<int>(parts);
    P.dep0 = dep0[static_cast<size_t>(i)];
    P.ndep = dep0[static_cast<size_t>(i) + 1] - dep0[static_cast<size_t>(i)];
    P.item0 = items;
    items += static_cast<long long>(P.tiles) * P.parts;
    P.rec0 = recs;
    P.cnt0 = cnts;
    if (P.parts > 1) {
      recs += static_cast<long long>(P.tiles) * P.parts;
      cnts += P.tiles;
    }
  }

  // one device allocation: [descriptors][tensor maps][deps][done][tile counters][records]
  auto up = [](size_t v, size_t a) { return (v + a - 1) / a * a; };
  const size_t off_lin = 0;
  const size_t off_map = up(off_lin + sizeof(PassLinear) * L, 128);
  const size_t off_dep = up(off_map + sizeof(CUtensorMap) * L, 128);
  const size_t off_cnt = up(off_dep + sizeof(int32_t) * std::max<size_t>(deps.size(), 1), 128);
  // [abort word, done[L], tile counters], zeroed before every run
  const size_t counter_bytes = sizeof(int32_t) * (1 + static_cast<size_t>(L) + static_cast<size_t>(cnts));
  const size_t off_rec = up(off_cnt + counter_bytes, 128);
  const size_t total = off_rec + sizeof(float) * kRecFloats * static_cast<size_t>(std::max<long long>(recs, 1));
  PassPlan* plan = new PassPlan();
  e = cudaMalloc(&plan->dev, total);
  if (e != cudaSuccess) {
    delete plan;
    return e;
  }
  uint8_t* dev = static_cast<uint8_t*>(plan->dev);
  std::vector<CUtensorMap> maps(static_cast<size_t>(L));
  for (int i = 0; i < L; ++i) {
    const PassLayer& A = layers[i];
    const int B = A.bits;
    const int chunks = static_cast<int>(A.K / 128);
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(16 * B), static_cast<cuuint64_t>(A.N),
                                static_cast<cuuint64_t>(chunks)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(16 * B) * chunks, static_cast<cuuint64_t>(16 * B)};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(16 * B), 16u, static_cast<cuuint32_t>(kPSC)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&maps[static_cast<size_t>(i)], CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(A.packed), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      cudaFree(plan->dev);
      delete plan;
      return cudaErrorInvalidValue;
    }
    lin[static_cast<size_t>(i)].tmap = reinterpret_cast<const CUtensorMap*>(dev + off_map) + i;
  }
  e = cudaMemcpy(dev + off_lin, lin.data(), sizeof(PassLinear) * L, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(dev + off_map, maps.data(), sizeof(CUtensorMap) * L, cudaMemcpyHostToDevice);
  if (e == cudaSuccess && !deps.empty())
    e = cudaMemcpy(dev + off_dep, deps.data(), sizeof(int32_t) * deps.size(), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(plan->dev);
    delete plan;
    return e;
  }
  PassParams& P = plan->params;
  P.lin = reinterpret_cast<const PassLinear*>(dev + off_lin);
  P.deps = reinterpret_cast<const int32_t*>(dev + off_dep);
  P.abort = reinterpret_cast<int32_t*>(dev + off_cnt);
  P.done = P.abort + 1;
  P.tile_cnt = P.done + L;
  P.rec = reinterpret_cast<float*>(dev + off_rec);
  P.items = items;
  P.L = L;
  P.S = S;
  P.slot_bytes = slot_bytes;
  P.err = device_error_word();
  plan->counters = P.abort;
  plan->counter_bytes = counter_bytes;
  plan->grid = static_cast<int>(std::min<long long>(G, items));
  plan->smem = smem;
  *out = plan;
  return cudaSuccess;
}

cudaError_t gemv_pass_run(const PassPlan* plan, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(plan->counters, 0, plan->counter_bytes, stream);
  if (e != cudaSuccess) return e;
  e = ensure_smem_attr(reinterpret_cast<const void*>(gemv_pass_kernel), plan->smem);
  if (e != cudaSuccess) return e;
  gemv_pass_kernel<<<plan->grid, kPThreads, plan->smem, stream>>>(plan->params);
  return cudaGetLastError();
}

void gemv_pass_destroy(PassPlan* plan) {
  if (plan == nullptr) return;
  cudaFree(plan->dev);
  delete plan;
}

void gemv_pass_info(const PassPlan* plan, int64_t* info) {
  info[0] = plan->grid;
  info[1] = plan->params.S;
  info[2] = plan->params.items;
  info[3] = static_cast<int64_t>(plan->smem);
}

}  // namespace mpw
