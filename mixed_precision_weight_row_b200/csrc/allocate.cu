// Per-matrix bit allocation under a byte budget (host code, no device work).
//
// DynaQuant, "Step 2: bit allocation": water filling over a max-heap of
// marginal bit upgrades -- every step raises one weight matrix to its next
// bit level, the priority being the marginal quality gain per byte of cost --
// in two modes, hardware-native {4, 8, 16} and full {4, 5, ..., 16}.
//
// The page leaves the gain and the cost open; this library takes:
//   * loss of a matrix at b bits D(b) = sens / Q_b^2, Q_b = 2^(b-1) - 1 (the
//     quantization step is max|w| / Q_b; rounding noise has variance step^2
//     / 12, whose constants drop out of the ordering); 16 bits keeps the
//     bf16 matrix, D = 0;
//   * cost = the bytes this library stores: N rows of 16 * ceil(K*b/128)
//     bytes and a 4-byte scale per row, or 2*N*K bytes at 16 bits;
//   * every matrix starts at 4 bits; upgrades are taken by gain / extra bytes
//     (fp64), ties to the lower matrix index, an upgrade that adds no bytes
//     first; one that no longer fits is dropped for good and the filling
//     goes on with the other matrices.
#include <stdint.h>

#include <cmath>
#include <queue>
#include <vector>

#include "mpw.h"

namespace {

constexpr int kNative[] = {4, 8, 16};
constexpr int kFull[] = {4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16};

uint64_t stored_bytes(int64_t N, int64_t K, int b) {
  const uint64_t n = static_cast<uint64_t>(N), k = static_cast<uint64_t>(K);
  if (b == 16) return 2u * n * k;
  return n * (16u * ((k * static_cast<uint64_t>(b) + 127u) / 128u)) + 4u * n;
}

double matrix_loss(double sens, int b) {
  if (b == 16) return 0.0;
  const double q = static_cast<double>((1 << (b - 1)) - 1);
  return sens / (q * q);
}

struct Upgrade {
  double priority;  // loss removed per extra byte
  int64_t matrix;
  int64_t extra;    // bytes the upgrade adds (<= 0 for very short rows)
};

// max-heap order: larger priority first, then the lower matrix index
struct Later {
  bool operator()(const Upgrade& a, const Upgrade& b) const {
    return a.priority < b.priority || (a.priority == b.priority && a.matrix > b.matrix);
  }
};

}  // namespace

extern "C" {

mpw_status mpw_allocate_bits(const double* sens, const int64_t* N, const int64_t* K, int64_t count,
                             uint64_t budget, int mode, int32_t* bits, uint64_t* total) {
  if (sens == nullptr || N == nullptr || K == nullptr || bits == nullptr || count < 1 || count > (1 << 24))
    return MPW_E_INVALID_ARG;
  if (mode != MPW_ALLOC_NATIVE && mode != MPW_ALLOC_FULL) return MPW_E_INVALID_ARG;
  const int* lv = mode == MPW_ALLOC_NATIVE ? kNative : kFull;
  const int nlv = mode == MPW_ALLOC_NATIVE ? 3 : 13;
  uint64_t spent = 0;
  for (int64_t i = 0; i < count; ++i) {
    if (N[i] < 1 || K[i] < 1 || N[i] >= (int64_t{1} << 31) || K[i] >= (int64_t{1} << 31)) return MPW_E_INVALID_ARG;
    if (!std::isfinite(sens[i]) || sens[i] < 0.0) return MPW_E_INVALID_ARG;
    const uint64_t c = stored_bytes(N[i], K[i], lv[0]);
    if (spent > UINT64_MAX - c) return MPW_E_INVALID_ARG;
    spent += c;
  }
  if (spent > budget) return MPW_E_INVALID_ARG;

  std::vector<int> level(static_cast<size_t>(count), 0);
  std::priority_queue<Upgrade, std::vector<Upgrade>, Later> heap;
  auto push = [&](int64_t i) {
    const int l = level[static_cast<size_t>(i)];
    if (l + 1 >= nlv) return;
    const double gain = matrix_loss(sens[i], lv[l]) - matrix_loss(sens[i], lv[l + 1]);
    const int64_t extra = static_cast<int64_t>(stored_bytes(N[i], K[i], lv[l + 1])) -
                          static_cast<int64_t>(stored_bytes(N[i], K[i], lv[l]));
    // an upgrade that adds no bytes (bf16 can take no more room than padded
    // codes and scales when rows are very short) goes first
    const double priority = extra <= 0 ? INFINITY : gain / static_cast<double>(extra);
    heap.push(Upgrade{priority, i, extra});
  };
  for (int64_t i = 0; i < count; ++i) push(i);
  while (!heap.empty()) {
    const Upgrade u = heap.top();
    heap.pop();
    if (u.extra > 0 && static_cast<uint64_t>(u.extra) > budget - spent) continue;  // dropped for good
    spent = static_cast<uint64_t>(static_cast<int64_t>(spent) + u.extra);
    ++level[static_cast<size_t>(u.matrix)];
    push(u.matrix);
  }
  for (int64_t i = 0; i < count; ++i) bits[i] = lv[level[static_cast<size_t>(i)]];
  if (total != nullptr) *total = spent;
  return MPW_OK;
}

mpw_status mpw_allocate_frontier(const double* sens, const int64_t* N, const int64_t* K, int64_t count, int mode,
                                 uint64_t* bytes, double* loss, int64_t max_points, int64_t* n_points) {
  if (sens == nullptr || N == nullptr || K == nullptr || n_points == nullptr || count < 1 || count > (1 << 24))
    return MPW_E_INVALID_ARG;
  if (max_points > 0 && (bytes == nullptr || loss == nullptr)) return MPW_E_INVALID_ARG;
  if (mode != MPW_ALLOC_NATIVE && mode != MPW_ALLOC_FULL) return MPW_E_INVALID_ARG;
  const int* lv = mode == MPW_ALLOC_NATIVE ? kNative : kFull;
  const int nlv = mode == MPW_ALLOC_NATIVE ? 3 : 13;
  uint64_t spent = 0, top = 0;
  double total = 0.0;
  for (int64_t i = 0; i < count; ++i) {
    if (N[i] < 1 || K[i] < 1 || N[i] >= (int64_t{1} << 31) || K[i] >= (int64_t{1} << 31)) return MPW_E_INVALID_ARG;
    if (!std::isfinite(sens[i]) || sens[i] < 0.0) return MPW_E_INVALID_ARG;
    // every point's bytes lie between the lowest and the highest level's
    const uint64_t hi = stored_bytes(N[i], K[i], lv[nlv - 1]) > stored_bytes(N[i], K[i], lv[0])
                            ? stored_bytes(N[i], K[i], lv[nlv - 1])
                            : stored_bytes(N[i], K[i], lv[0]);
    if (top > (UINT64_MAX >> 1) - hi) return MPW_E_INVALID_ARG;
    top += hi;
    spent += stored_bytes(N[i], K[i], lv[0]);
    total += matrix_loss(sens[i], lv[0]);
  }
  // the unbounded filling: every upgrade, in priority order
  std::vector<int> level(static_cast<size_t>(count), 0);
  std::priority_queue<Upgrade, std::vector<Upgrade>, Later> heap;
  auto push = [&](int64_t i) {
    const int l = level[static_cast<size_t>(i)];
    if (l + 1 >= nlv) return;
    const double gain = matrix_loss(sens[i], lv[l]) - matrix_loss(sens[i], lv[l + 1]);
    const int64_t extra = static_cast<int64_t>(stored_bytes(N[i], K[i], lv[l + 1])) -
                          static_cast<int64_t>(stored_bytes(N[i], K[i], lv[l]));
    const double priority = extra <= 0 ? INFINITY : gain / static_cast<double>(extra);
    heap.push(Upgrade{priority, i, extra});
  };
  for (int64_t i = 0; i < count; ++i) push(i);
  int64_t n = 0;
  auto emit = [&]() {
    if (n < max_points) {
      bytes[n] = spent;
      loss[n] = total;
    }
    ++n;
  };
  emit();
  while (!heap.empty()) {
    const Upgrade u = heap.top();
    heap.pop();
    const int l = level[static_cast<size_t>(u.matrix)];
    total -= matrix_loss(sens[u.matrix], lv[l]) - matrix_loss(sens[u.matrix], lv[l + 1]);
    spent = static_cast<uint64_t>(static_cast<int64_t>(spent) + u.extra);
    ++level[static_cast<size_t>(u.matrix)];
    push(u.matrix);
    emit();
  }
  *n_points = n;
  return MPW_OK;
}

}  // extern "C"
