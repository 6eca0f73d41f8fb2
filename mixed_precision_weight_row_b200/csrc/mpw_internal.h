// Internal declarations shared by the translation units of libmpw.so.
// Launchers validate nothing: the C-ABI layer (api.cu) has checked every
// argument before it calls them.  Each returns the cudaError_t of its launch.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace mpw {

constexpr int kMinBits = 4;
constexpr int kMaxBits = 15;

// Words (uint32) of one canonical packed row: 4 * ceil(K*b/128).
inline int64_t row_words(int64_t K, int bits) { return 4 * ((K * bits + 127) / 128); }

// Per-device properties cached on first use.
struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int max_smem_optin = 0;  // bytes of dynamic shared memory a block may opt into
};
const DeviceInfo& device_info();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device (once per kernel and device).
cudaError_t ensure_smem_attr(const void* kernel, size_t bytes);

// quantize.cu
cudaError_t launch_quantize_pack(const float* W, int64_t N, int64_t K, int bits,
                                 uint8_t* packed, float* scales, int32_t* flag,
                                 cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t* packed, int64_t N, int64_t K, int bits,
                          int16_t* codes, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int64_t N,
                              int64_t K, int bits, float* W_hat, cudaStream_t stream);

// gemv.cu: y[M, N] for any M, in passes of at most kGemvMaxTokens rows of x.
cudaError_t launch_gemv(const uint16_t* x, const uint8_t* packed, const float* scales,
                        int bits, int64_t M, int64_t N, int64_t K, uint16_t* y,
                        bool norm_input, cudaStream_t stream);

// gemm.cu: tcgen05 prefill GEMM; returns cudaErrorNotSupported for shapes it
// does not take (the caller then uses the GEMV path).
cudaError_t launch_gemm(const uint16_t* x, const uint8_t* packed, const float* scales,
                        int bits, int64_t M, int64_t N, int64_t K, uint16_t* y,
                        int32_t* dev_error, cudaStream_t stream);
bool gemm_supported(int64_t M, int64_t N, int64_t K);

}  // namespace mpw
