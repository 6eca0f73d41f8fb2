// C ABI of libmpw.so: argument validation and kernel dispatch.  See mpw.h for
// the contract of every entry point.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "mpw.h"
#include "mpw_internal.h"

namespace mpw {

static_assert(MPW_LAYOUT_CANONICAL == kLayoutCanonical && MPW_LAYOUT_PAIRED == kLayoutPaired,
              "layout values of the C ABI and the kernels agree");

// Device-side error word: set by bounded waits that give up.
__device__ int32_t g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_info[kMaxDevices];
std::mutex g_mutex;

struct AttrEntry {
  const void* kernel;
  int device;
  size_t bytes;
};
AttrEntry g_attrs[1024];
int g_num_attrs = 0;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

mpw_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MPW_OK : MPW_E_CUDA; }

bool bits_ok(int bits) { return bits >= kMinBits && bits <= kMaxBits; }

bool layout_ok(int layout) { return layout == MPW_LAYOUT_CANONICAL || layout == MPW_LAYOUT_PAIRED; }

}  // namespace

const DeviceInfo& device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  DeviceInfo& d = g_info[dev];
  if (d.device != dev) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (d.device != dev) {
      int sms = 0, smem = 0, per_sm = 0, reserved = 0;
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
      cudaDeviceGetAttribute(&per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
      cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
      d.num_sms = sms > 0 ? sms : 1;
      d.max_smem_optin = smem;
      d.smem_per_sm = per_sm;
      d.smem_reserved = reserved;
      d.device = dev;
    }
  }
  return d;
}

cudaError_t ensure_smem_attr(const void* kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mutex);
  for (int i = 0; i < g_num_attrs; ++i)
    if (g_attrs[i].kernel == kernel && g_attrs[i].device == dev && g_attrs[i].bytes >= bytes)
      return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  if (g_num_attrs < 1024) g_attrs[g_num_attrs++] = AttrEntry{kernel, dev, bytes};
  return cudaSuccess;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int32_t* device_error_word() {
  // looked up once per device (with that device current) and kept for the
  // life of the process, like the kernels' shared-memory attributes
  static std::atomic<int32_t*> addr[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  int32_t* a = addr[dev].load(std::memory_order_acquire);
  if (a == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
    a = static_cast<int32_t*>(p);
    addr[dev].store(a, std::memory_order_release);
  }
  return a;
}

}  // namespace mpw

using namespace mpw;

extern "C" {

const char* mpw_status_str(int status) {
  switch (status) {
    case MPW_OK: return "ok";
    case MPW_E_INVALID_ARG: return "invalid argument";
    case MPW_E_UNSUPPORTED_BITS: return "bit width outside 4..15";
    case MPW_E_MISALIGNED: return "misaligned pointer";
    case MPW_E_CUDA: return "CUDA error";
    case MPW_E_NONFINITE: return "non-finite input";
    case MPW_E_TIMEOUT: return "device-side wait timed out";
    case MPW_E_SCRATCH_LIMIT: return "call needs more than the fixed scratch of mpw_qlinear_noalloc";
    case MPW_E_IO: return "file cannot be opened, read or written";
    case MPW_E_FORMAT: return "not a valid packed-weight file, or a checksum differs";
    case MPW_E_UNSUPPORTED: return "the planned decode pass does not take these linears (use mpw_recipe_run)";
    default: return "unknown status";
  }
}

int mpw_version(void) { return 300; }

size_t mpw_packed_row_bytes(int64_t K, int bits) {
  if (!bits_ok(bits) || K < 1) return 0;
  return static_cast<size_t>(16 * ((K * bits + 127) / 128));
}

mpw_status mpw_quantize_pack(const float* W, int64_t N, int64_t K, int bits, uint8_t* packed,
                             float* scales, int32_t* nonfinite_flag, mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if (W == nullptr || packed == nullptr || scales == nullptr || N < 1 || K < 1) return MPW_E_INVALID_ARG;
  if (N > 0x7fffffff || K > 0x3fffffff) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(W, 4) || !aligned(scales, 4) ||
      (nonfinite_flag != nullptr && !aligned(nonfinite_flag, 4)))
    return MPW_E_MISALIGNED;
  return from_cuda(launch_quantize_pack(W, N, K, bits, packed, scales, nonfinite_flag,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_unpack(const uint8_t* packed, int64_t N, int64_t K, int bits, int16_t* codes,
                      mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if (packed == nullptr || codes == nullptr || N < 1 || K < 1) return MPW_E_INVALID_ARG;
  if (K > 0x3fffffff) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(codes, 2)) return MPW_E_MISALIGNED;
  return from_cuda(launch_unpack(packed, N, K, bits, codes, reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_dequantize(const uint8_t* packed, const float* scales, int64_t N, int64_t K, int bits,
                          float* W_hat, mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if (packed == nullptr || scales == nullptr || W_hat == nullptr || N < 1 || K < 1)
    return MPW_E_INVALID_ARG;
  if (K > 0x3fffffff) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(scales, 4) || !aligned(W_hat, 4)) return MPW_E_MISALIGNED;
  return from_cuda(
      launch_dequantize(packed, scales, N, K, bits, W_hat, reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_repack(const uint8_t* in, int64_t N, int64_t K, int bits, int layout_in, int layout_out,
                      uint8_t* out, mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if (in == nullptr || out == nullptr || N < 1 || K < 1 || K > 0x3fffffff || K % 32 != 0)
    return MPW_E_INVALID_ARG;
  if (!layout_ok(layout_in) || !layout_ok(layout_out) || layout_in == layout_out) return MPW_E_INVALID_ARG;
  if (!aligned(in, 16) || !aligned(out, 16)) return MPW_E_MISALIGNED;
  if (in != out) {
    // the kernel may run in place, but not on partly overlapping rows
    const size_t bytes = static_cast<size_t>(N) * mpw_packed_row_bytes(K, bits);
    const uintptr_t a = reinterpret_cast<uintptr_t>(in), b = reinterpret_cast<uintptr_t>(out);
    if (a < b + bytes && b < a + bytes) return MPW_E_INVALID_ARG;
  }
  return from_cuda(launch_repack(in, N, K, bits, out, layout_out == MPW_LAYOUT_PAIRED,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_quantize_pack_groups(const float* W, int64_t N, int64_t K, int bits, int64_t group, uint8_t* packed,
                                    float* scales, int32_t* nonfinite_flag, mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if (W == nullptr || packed == nullptr || scales == nullptr || N < 1 || K < 1) return MPW_E_INVALID_ARG;
  if (group < 32 || group > 1024 || (group & (group - 1)) != 0) return MPW_E_INVALID_ARG;
  if (N > 0x7fffffff || K > 0x3fffffff) return MPW_E_INVALID_ARG;
  // one warp per 1024 weights of a row, 8 warps per block: under 2^31 blocks
  if (N * (((K + 31) / 32 + 31) / 32) >= (int64_t{1} << 34)) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(W, 4) || !aligned(scales, 4) ||
      (nonfinite_flag != nullptr && !aligned(nonfinite_flag, 4)))
    return MPW_E_MISALIGNED;
  return from_cuda(launch_quantize_pack_groups(W, N, K, bits, group, packed, scales, nonfinite_flag,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_qlinear_groups(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int64_t group,
                              int layout, int64_t M, int64_t N, int64_t K, uint16_t* y, unsigned flags,
                              mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if ((flags & ~static_cast<unsigned>(MPW_QLINEAR_X_READY | MPW_QLINEAR_Y_UNSHARED)) != 0) return MPW_E_INVALID_ARG;
  if ((flags & MPW_QLINEAR_Y_UNSHARED) && !(flags & MPW_QLINEAR_X_READY)) return MPW_E_INVALID_ARG;
  if (x == nullptr || packed == nullptr || scales == nullptr || y == nullptr || M < 1 || N < 1 || K < 1)
    return MPW_E_INVALID_ARG;
  if (N > 0x7fffffff || K > 0x3fffffff || M > 0x7fffffff || !layout_ok(layout)) return MPW_E_INVALID_ARG;
  if (group < 128 || group > 1024 || (group & (group - 1)) != 0) return MPW_E_INVALID_ARG;
  if (K % 8 != 0 || (layout == MPW_LAYOUT_PAIRED && K % 32 != 0)) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(x, 16) || !aligned(y, 2) || !aligned(scales, 4)) return MPW_E_MISALIGNED;
  if (!gemv_groups_supported(x, M, N, K, group)) return MPW_E_CUDA;   // no tensor-map encoder
  return from_cuda(launch_gemv_groups(x, packed, scales, bits, group, layout, M, N, K, y,
                                      reinterpret_cast<cudaStream_t>(stream), flags));
}

mpw_status mpw_quantize_x_fp8(const uint16_t* x, int64_t M, int64_t K, uint8_t* xq, float* sx, mpw_stream_t stream) {
  if (x == nullptr || xq == nullptr || sx == nullptr || M < 1 || K < 16) return MPW_E_INVALID_ARG;
  if (M > 0x7fffffff || K > 0x3fffffff || K % 16 != 0) return MPW_E_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(xq, 16) || !aligned(sx, 4)) return MPW_E_MISALIGNED;
  return from_cuda(launch_quantize_x_fp8(x, M, K, xq, sx, reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_qlinear_fp8(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales, int bits,
                           int layout, int64_t M, int64_t N, int64_t K, uint16_t* y, mpw_stream_t stream) {
  if (bits != 4 && bits != 5) return MPW_E_UNSUPPORTED_BITS;
  if (xq == nullptr || sx == nullptr || packed == nullptr || scales == nullptr || y == nullptr || M < 1 || N < 1 ||
      K < 16)
    return MPW_E_INVALID_ARG;
  if (M > 0x7fffffff || N > 0x7fffffff || K > 0x3fffffff || K % 16 != 0 || !layout_ok(layout)) return MPW_E_INVALID_ARG;
  if (layout == MPW_LAYOUT_PAIRED && K % 32 != 0) return MPW_E_INVALID_ARG;
  if ((M + 255) / 256 > 65535) return MPW_E_INVALID_ARG;
  if (!aligned(xq, 16) || !aligned(packed, 16) || !aligned(sx, 4) || !aligned(scales, 4) || !aligned(y, 2))
    return MPW_E_MISALIGNED;
  return from_cuda(launch_gemm_fp8(xq, sx, packed, scales, bits, layout, M, N, K, y,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_gather_shards(const uint16_t* blocks, int64_t world, int64_t M, int64_t Nl, int64_t N, uint16_t* y,
                             mpw_stream_t stream) {
  if (blocks == nullptr || y == nullptr || world < 1 || M < 1 || Nl < 1 || N < 1) return MPW_E_INVALID_ARG;
  if (world > 0x10000 || M > 0x7fffffff || Nl > 0x7fffffff || N > world * Nl) return MPW_E_INVALID_ARG;
  if (!aligned(blocks, 2) || !aligned(y, 2)) return MPW_E_MISALIGNED;
  return from_cuda(launch_gather_shards(blocks, M, Nl, N, y, reinterpret_cast<cudaStream_t>(stream)));
}

namespace {

mpw_status qlinear_impl(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                        int64_t M, int64_t N, int64_t K, uint16_t* y, int path, void* ws, size_t ws_bytes,
                        unsigned flags, mpw_stream_t stream) {
  if (!bits_ok(bits)) return MPW_E_UNSUPPORTED_BITS;
  if ((flags & ~static_cast<unsigned>(MPW_QLINEAR_X_READY | MPW_QLINEAR_Y_UNSHARED)) != 0) return MPW_E_INVALID_ARG;
  if ((flags & MPW_QLINEAR_Y_UNSHARED) && !(flags & MPW_QLINEAR_X_READY)) return MPW_E_INVALID_ARG;
  if (x == nullptr || packed == nullptr || scales == nullptr || y == nullptr || M < 1 || N < 1 ||
      K < 1)
    return MPW_E_INVALID_ARG;
  if (N > 0x7fffffff || K > 0x3fffffff || M > 0x7fffffff) return MPW_E_INVALID_ARG;
  if (path < MPW_PATH_AUTO || path > MPW_PATH_GEMM || !layout_ok(layout)) return MPW_E_INVALID_ARG;
  const bool paired = layout == MPW_LAYOUT_PAIRED;
  if (paired && K % 32 != 0) return MPW_E_INVALID_ARG;
  if (!aligned(packed, 16) || !aligned(x, paired ? 16 : 2) || !aligned(y, 2) || !aligned(scales, 4))
    return MPW_E_MISALIGNED;
  if (ws != nullptr && !aligned(ws, 16)) return MPW_E_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool want_gemm = path == MPW_PATH_GEMM || (path == MPW_PATH_AUTO && M > 32);
  if (want_gemm && gemm_supported(M, N, K) && aligned(x, 16)) {
    return from_cuda(launch_gemm(x, packed, scales, bits, layout, M, N, K, y, device_error_word(), s));
  }
  if (path == MPW_PATH_GEMM) return MPW_E_INVALID_ARG;  // shape the GEMM does not take
  if (ws != nullptr && ws_bytes < gemv_workspace_bytes(x, bits, layout, M, N, K, false)) return MPW_E_INVALID_ARG;
  static_assert(MPW_QLINEAR_X_READY == kQlinearXReady && MPW_QLINEAR_Y_UNSHARED == kQlinearYFree,
                "flag values");
  return from_cuda(launch_gemv(x, packed, scales, bits, layout, M, N, K, y, false, ws, ws_bytes, s, flags));
}

}  // namespace

size_t mpw_qlinear_workspace_bytes(int bits, int layout, int64_t M, int64_t N, int64_t K) {
  if (!bits_ok(bits) || !layout_ok(layout) || M < 1 || N < 1 || K < 1 || M > 32) return 0;
  if (N > 0x7fffffff || K > 0x3fffffff) return 0;
  return gemv_workspace_bytes(nullptr, bits, layout, M, N, K, false);
}

mpw_status mpw_qlinear_ws(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                          int64_t M, int64_t N, int64_t K, uint16_t* y, int path, void* workspace,
                          size_t workspace_bytes, mpw_stream_t stream) {
  return qlinear_impl(x, packed, scales, bits, layout, M, N, K, y, path, workspace, workspace_bytes, 0u, stream);
}

mpw_status mpw_qlinear_flags(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                             int64_t M, int64_t N, int64_t K, uint16_t* y, int path, unsigned flags,
                             mpw_stream_t stream) {
  return qlinear_impl(x, packed, scales, bits, layout, M, N, K, y, path, nullptr, 0, flags, stream);
}

mpw_status mpw_qlinear_ex(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                          int64_t M, int64_t N, int64_t K, uint16_t* y, int path, mpw_stream_t stream) {
  return qlinear_impl(x, packed, scales, bits, layout, M, N, K, y, path, nullptr, 0, 0u, stream);
}

mpw_status mpw_qlinear_path(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, int path,
                            mpw_stream_t stream) {
  return mpw_qlinear_ex(x, packed, scales, bits, MPW_LAYOUT_CANONICAL, M, N, K, y, path, stream);
}

mpw_status mpw_qlinear(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                       int64_t M, int64_t N, int64_t K, uint16_t* y, mpw_stream_t stream) {
  return mpw_qlinear_ex(x, packed, scales, bits, MPW_LAYOUT_CANONICAL, M, N, K, y, MPW_PATH_AUTO, stream);
}

namespace {

mpw_status recipe_check(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t num_slots,
                        int64_t M) {
  if (layers == nullptr || slots == nullptr || count < 1 || num_slots < 1 || M < 1 || M > 32)
    return MPW_E_INVALID_ARG;
  for (int64_t i = 0; i < count; ++i) {
    const mpw_linear& L = layers[i];
    if (!bits_ok(L.bits)) return MPW_E_UNSUPPORTED_BITS;
    if (L.packed == nullptr || L.scales == nullptr || L.N < 1 || L.K < 1 || L.N > 0x7fffffff ||
        L.K > 0x3fffffff)
      return MPW_E_INVALID_ARG;
    if (L.in_slot < 0 || L.in_slot >= num_slots || L.out_slot < 0 || L.out_slot >= num_slots ||
        L.in_slot == L.out_slot)
      return MPW_E_INVALID_ARG;
    if (!layout_ok(L.layout) || L.reserved != 0) return MPW_E_INVALID_ARG;
    if (L.layout == MPW_LAYOUT_PAIRED && L.K % 32 != 0) return MPW_E_INVALID_ARG;
    if (slots[L.in_slot] == nullptr || slots[L.out_slot] == nullptr) return MPW_E_INVALID_ARG;
    if (!aligned(L.packed, 16) || !aligned(L.scales, 4)) return MPW_E_MISALIGNED;
    if (L.layout == MPW_LAYOUT_PAIRED && !aligned(slots[L.in_slot], 16)) return MPW_E_MISALIGNED;
  }
  return MPW_OK;
}

// The MPW_QLINEAR_* flags each linear of a recipe run is launched with.  A
// linear whose input was written neither by the linear before the current
// run of x-ready linears nor by one inside it joins the run (X_READY): k and
// v after q, up after gate; when its output is also neither read nor written
// by the run and that linear, it writes it without waiting (Y_UNSHARED).
// Inputs and outputs are compared as byte ranges, so slots that alias are
// safe.  The first linear follows whatever the caller launched before: never.
void recipe_flags(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t M, uint32_t* flags) {
  constexpr int kRunMax = 8;
  // inputs and outputs of the run and of the linear before it
  uintptr_t in_lo[kRunMax], in_hi[kRunMax], out_lo[kRunMax], out_hi[kRunMax];
  int nrun = 0;
  auto overlaps = [&](const uintptr_t* lo, const uintptr_t* hi, uintptr_t a, uintptr_t b) {
    for (int r = 0; r < nrun; ++r)
      if (a < hi[r] && lo[r] < b) return true;
    return false;
  };
  for (int64_t i = 0; i < count; ++i) {
    const mpw_linear& L = layers[i];
    const uintptr_t xa = reinterpret_cast<uintptr_t>(slots[L.in_slot]);
    const uintptr_t xb = xa + static_cast<uintptr_t>(M * L.K) * 2u;
    const uintptr_t ya = reinterpret_cast<uintptr_t>(slots[L.out_slot]);
    const uintptr_t yb = ya + static_cast<uintptr_t>(M * L.N) * 2u;
    const bool xr = i > 0 && nrun < kRunMax && !overlaps(out_lo, out_hi, xa, xb);
    const bool yf = xr && !overlaps(out_lo, out_hi, ya, yb) && !overlaps(in_lo, in_hi, ya, yb);
    if (!xr) nrun = 0;
    in_lo[nrun] = xa;
    in_hi[nrun] = xb;
    out_lo[nrun] = ya;
    out_hi[nrun] = yb;
    ++nrun;
    flags[i] = (xr ? kQlinearXReady : 0u) | (yf ? kQlinearYFree : 0u);
  }
}

size_t recipe_ws_bytes(const mpw_linear* layers, int64_t count, int64_t M) {
  size_t b = 0;
  for (int64_t i = 0; i < count; ++i) {
    const mpw_linear& L = layers[i];
    const size_t need = gemv_workspace_bytes(nullptr, L.bits, L.layout, M, L.N, L.K, L.norm_input != 0);
    if (need > b) b = need;
  }
  return b;
}

}  // namespace

size_t mpw_recipe_workspace_bytes(const mpw_linear* layers, int64_t count, int64_t M) {
  if (layers == nullptr || count < 1 || M < 1 || M > 32) return 0;
  for (int64_t i = 0; i < count; ++i)
    if (!bits_ok(layers[i].bits) || !layout_ok(layers[i].layout) || layers[i].N < 1 || layers[i].K < 1) return 0;
  return recipe_ws_bytes(layers, count, M);
}

mpw_status mpw_recipe_run_ws(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t num_slots,
                             int64_t M, void* workspace, size_t workspace_bytes, mpw_stream_t stream) {
  const mpw_status st = recipe_check(layers, count, slots, num_slots, M);
  if (st != MPW_OK) return st;
  if (workspace != nullptr) {
    if (!aligned(workspace, 16)) return MPW_E_MISALIGNED;
    if (workspace_bytes < recipe_ws_bytes(layers, count, M)) return MPW_E_INVALID_ARG;
  }
  std::vector<uint32_t> flags(static_cast<size_t>(count));
  recipe_flags(layers, count, slots, M, flags.data());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  for (int64_t i = 0; i < count; ++i) {
    const mpw_linear& L = layers[i];
    if (launch_gemv(slots[L.in_slot], L.packed, L.scales, L.bits, L.layout, M, L.N, L.K, slots[L.out_slot],
                    L.norm_input != 0, workspace, workspace_bytes, s, flags[static_cast<size_t>(i)]) != cudaSuccess)
      return MPW_E_CUDA;
  }
  return MPW_OK;
}

mpw_status mpw_recipe_plan(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t num_slots,
                           int64_t M, uint32_t* flags) {
  if (flags == nullptr) return MPW_E_INVALID_ARG;
  const mpw_status st = recipe_check(layers, count, slots, num_slots, M);
  if (st != MPW_OK) return st;
  recipe_flags(layers, count, slots, M, flags);
  return MPW_OK;
}

mpw_status mpw_recipe_run(const mpw_linear* layers, int64_t count, uint16_t* const* slots,
                          int64_t num_slots, int64_t M, mpw_stream_t stream) {
  return mpw_recipe_run_ws(layers, count, slots, num_slots, M, nullptr, 0, stream);
}

// The planned pass's view of a recipe: one PassLayer per linear (host only).
mpw_status pass_layers(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t num_slots,
                       int64_t M, std::vector<mpw::PassLayer>& pl) {
  const mpw_status st = recipe_check(layers, count, slots, num_slots, M);
  if (st != MPW_OK) return st;
  if (M != 1 || count > (1 << 20)) return MPW_E_UNSUPPORTED;
  pl.assign(static_cast<size_t>(count), mpw::PassLayer{});
  for (int64_t i = 0; i < count; ++i) {
    const mpw_linear& L = layers[i];
    if (!mpw::gemv_pass_layer_ok(L.bits, L.layout, L.N, L.K)) return MPW_E_UNSUPPORTED;
    mpw::PassLayer& P = pl[static_cast<size_t>(i)];
    P.x = slots[L.in_slot];
    P.y = slots[L.out_slot];
    P.packed = L.packed;
    P.scales = L.scales;
    P.N = L.N;
    P.K = L.K;
    P.bits = L.bits;
    P.norm = L.norm_input != 0;
    // a linear whose input and output bytes overlap cannot be ordered
    const uintptr_t xa = reinterpret_cast<uintptr_t>(P.x), ya = reinterpret_cast<uintptr_t>(P.y);
    if (xa < ya + 2u * static_cast<uintptr_t>(P.N) && ya < xa + 2u * static_cast<uintptr_t>(P.K))
      return MPW_E_INVALID_ARG;
  }
  return MPW_OK;
}

mpw_status mpw_pass_dependencies(const mpw_linear* layers, int64_t count, uint16_t* const* slots,
                                 int64_t num_slots, int64_t M, int32_t* offsets, int32_t* deps,
                                 int64_t deps_capacity) {
  if (offsets == nullptr || deps_capacity < 0 || (deps == nullptr && deps_capacity > 0)) return MPW_E_INVALID_ARG;
  std::vector<mpw::PassLayer> pl;
  const mpw_status st = pass_layers(layers, count, slots, num_slots, M, pl);
  if (st != MPW_OK) return st;
  std::vector<int32_t> d, d0;
  if (!mpw::gemv_pass_dependencies(pl.data(), count, d, d0)) return MPW_E_INVALID_ARG;
  for (int64_t i = 0; i <= count; ++i) offsets[i] = d0[static_cast<size_t>(i)];
  if (static_cast<int64_t>(d.size()) > deps_capacity) return MPW_E_INVALID_ARG;
  for (size_t i = 0; i < d.size(); ++i) deps[i] = d[i];
  return MPW_OK;
}

mpw_status mpw_pass_create(const mpw_linear* layers, int64_t count, uint16_t* const* slots, int64_t num_slots,
                           int64_t M, mpw_pass** pass) {
  if (pass == nullptr) return MPW_E_INVALID_ARG;
  *pass = nullptr;
  std::vector<mpw::PassLayer> pl;
  const mpw_status st = pass_layers(layers, count, slots, num_slots, M, pl);
  if (st != MPW_OK) return st;
  mpw::PassPlan* plan = nullptr;
  const cudaError_t e = mpw::gemv_pass_create(pl.data(), count, &plan);
  if (e != cudaSuccess) return MPW_E_CUDA;
  *pass = reinterpret_cast<mpw_pass*>(plan);
  return MPW_OK;
}

mpw_status mpw_pass_run(const mpw_pass* pass, mpw_stream_t stream) {
  if (pass == nullptr) return MPW_E_INVALID_ARG;
  return from_cuda(mpw::gemv_pass_run(reinterpret_cast<const mpw::PassPlan*>(pass),
                                      reinterpret_cast<cudaStream_t>(stream)));
}

mpw_status mpw_pass_info(const mpw_pass* pass, int64_t* info) {
  if (pass == nullptr || info == nullptr) return MPW_E_INVALID_ARG;
  mpw::gemv_pass_info(reinterpret_cast<const mpw::PassPlan*>(pass), info);
  return MPW_OK;
}

void mpw_pass_destroy(mpw_pass* pass) { mpw::gemv_pass_destroy(reinterpret_cast<mpw::PassPlan*>(pass)); }

mpw_status mpw_device_error(int32_t* code) {
  if (code == nullptr) return MPW_E_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MPW_E_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return MPW_E_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return MPW_E_CUDA;
  *code = v;
  return v != 0 ? MPW_E_TIMEOUT : MPW_OK;
}

}  // extern "C"
