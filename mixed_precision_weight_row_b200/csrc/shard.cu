// Output-row (N) sharding of a linear layer over several GPUs: the re-ordering
// of the gathered outputs.
//
// No page describes tensor parallelism; this is the library's own partition.
// Each of `world` ranks owns Nl consecutive weight rows (rows r * Nl ..
// r * Nl + Nl - 1 of W, zero rows past N) with their scales and computes
// y_r = x @ W_r^T, [M, Nl], for the replicated input x.  An all-gather of the
// y_r (NCCL, in the caller) leaves them rank after rank: blocks [world, M, Nl].
// The full output y [M, N] takes column n from block n / Nl, column n % Nl.
// For M = 1 the blocks already are y; for M > 1 this kernel interleaves them.
#include <cuda_runtime.h>
#include <stdint.h>

#include "mpw_internal.h"

namespace mpw {
namespace {

__global__ void __launch_bounds__(256)
gather_shards_kernel(const uint16_t* __restrict__ blocks, int64_t M, int64_t Nl, int64_t N,
                     uint16_t* __restrict__ y) {
  const int64_t total = M * N;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / N, n = i - m * N;
    const int64_t r = n / Nl, j = n - r * Nl;
    y[i] = blocks[(r * M + m) * Nl + j];
  }
}

}  // namespace

cudaError_t launch_gather_shards(const uint16_t* blocks, int64_t M, int64_t Nl, int64_t N, uint16_t* y,
                                 cudaStream_t stream) {
  const int64_t total = M * N;
  int64_t grid = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_info().num_sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  gather_shards_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(blocks, M, Nl, N, y);
  return cudaGetLastError();
}

}  // namespace mpw
