// Internal declarations shared by the translation units of libmpw.so.
// Launchers validate nothing: the C-ABI layer (api.cu) has checked every
// argument before it calls them.  Each returns the cudaError_t of its launch.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <vector>

namespace mpw {

constexpr int kMinBits = 4;
constexpr int kMaxBits = 15;

// Packed layouts (the values of mpw_layout): canonical LSB-first stream, and
// the paired-halves re-ordering of the same bits (K % 32 == 0).
constexpr int kLayoutCanonical = 0;
constexpr int kLayoutPaired = 1;

// Words (uint32) of one canonical packed row: 4 * ceil(K*b/128).
inline int64_t row_words(int64_t K, int bits) { return 4 * ((K * bits + 127) / 128); }

// Tuning aids for measurement: the MPW_GEMV_* environment variables are read
// only in a library built with -DMPW_TUNING_KNOBS; the default build ignores
// them, so the environment never changes which kernel runs or how.
inline const char* tuning_env(const char* name) {
#ifdef MPW_TUNING_KNOBS
  return getenv(name);
#else
  (void)name;
  return nullptr;
#endif
}

// Per-device properties cached on first use.
struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  int max_smem_optin = 0;  // bytes of dynamic shared memory a block may opt into
  int smem_per_sm = 0;     // bytes of shared memory per SM
  int smem_reserved = 0;   // bytes the system reserves per resident block
};
const DeviceInfo& device_info();

// cuTensorMapEncodeTiled from the driver (nullptr if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Device address of the library's device-side error word.
int32_t* device_error_word();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device (once per kernel and device).
cudaError_t ensure_smem_attr(const void* kernel, size_t bytes);

// quantize.cu
cudaError_t launch_quantize_pack(const float* W, int64_t N, int64_t K, int bits,
                                 uint8_t* packed, float* scales, int32_t* flag,
                                 cudaStream_t stream);
// Group-wise scales: one per `group` consecutive weights of a row (a power of
// two in 32..1024); scales [N, ceil(K / group)].
cudaError_t launch_quantize_pack_groups(const float* W, int64_t N, int64_t K, int bits, int64_t group,
                                        uint8_t* packed, float* scales, int32_t* flag, cudaStream_t stream);
cudaError_t launch_unpack(const uint8_t* packed, int64_t N, int64_t K, int bits,
                          int16_t* codes, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* packed, const float* scales, int64_t N,
                              int64_t K, int bits, float* W_hat, cudaStream_t stream);
// Canonical <-> paired-halves re-ordering (K % 32 == 0; in == out allowed).
cudaError_t launch_repack(const uint8_t* in, int64_t N, int64_t K, int bits, uint8_t* out,
                          bool to_paired, cudaStream_t stream);

// gemv.cu: decode linear y[M, N] for any M (tensor-core kernels in passes of
// 32 tokens; CUDA-core kernels for canonical shapes they do not take).  The
// paired layout needs a shape the TMA kernel takes (checked by the caller).
// qflags: kQlinearXReady = x was written before the launch that precedes the
// current run of such calls on the stream (MPW_QLINEAR_X_READY): the per-tile
// kernel then releases its successor at once and loads x without waiting;
// kQlinearYFree (with it) = no call of the run, nor the launch before it,
// reads or writes y (MPW_QLINEAR_Y_UNSHARED): y is written without waiting.
constexpr unsigned kQlinearXReady = 1u;
constexpr unsigned kQlinearYFree = 2u;
cudaError_t launch_gemv(const uint16_t* x, const uint8_t* packed, const float* scales,
                        int bits, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                        bool norm_input, void* ws, size_t ws_bytes, cudaStream_t stream,
                        unsigned qflags = 0u);
// Workspace bytes launch_gemv uses for these arguments (0 if none).
size_t gemv_workspace_bytes(const uint16_t* x_or_null, int bits, int layout, int64_t M, int64_t N,
                            int64_t K, bool norm_input);
// The CUDA-core decode kernels alone (x in registers for K <= 17408, else x
// staged in shared memory), in passes of two tokens.
cudaError_t launch_gemv_cuda_core(const uint16_t* x, const uint8_t* packed, const float* scales,
                                  int bits, int64_t M, int64_t N, int64_t K, uint16_t* y,
                                  bool norm_input, cudaStream_t stream);

// gemv_mma.cu: decode linear on register-fed tensor cores for M <= 32
// (M <= 8 with norm_input); pdl = launch with programmatic dependent launch.
bool gemv_mma_supported(int64_t M, int64_t N, int64_t K, bool norm);
cudaError_t launch_gemv_mma(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                            int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, bool pdl,
                            cudaStream_t stream);

// gemv_tma.cu: decode linear with the packed stream and x staged by TMA in a
// shared-memory ring (the default decode kernel for M <= 32; needs K % 8 == 0
// and a 16-byte aligned x).  qflags as for launch_gemv.
bool gemv_tma_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm);
cudaError_t launch_gemv_tma(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                            int layout, int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm,
                            bool pdl, unsigned qflags, cudaStream_t stream);

// gemv_sk.cu: decode linear with the (tile, chunk) units split evenly over
// a persistent grid; split tiles are combined in a caller workspace (zeroed
// before its first use; the kernel leaves its counters at zero).  *used is
// set when the kernel was launched; it is left false (and nothing launched)
// when the workspace is missing or smaller than gemv_sk_workspace_bytes.
bool gemv_sk_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm);
size_t gemv_sk_workspace_bytes(int bits, int layout, int64_t M, int64_t N, int64_t K, bool norm);
cudaError_t launch_gemv_sk(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                           int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, void* ws, size_t ws_bytes,
                           cudaStream_t stream, bool* used);

// gemv_tc.cu: decode linear for M <= 32 on tcgen05 tensor cores (weights
// expanded into tensor memory, 128-row tiles, K split over a cluster when
// there are few tiles).
bool gemv_tc_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, bool norm);
// Whether the shape is one where this kernel beats the per-tile decode kernel.
bool gemv_tc_preferred(int bits, int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemv_tc(const uint16_t* x, const uint8_t* packed, const float* scales, int bits, int layout,
                           int64_t M, int64_t N, int64_t K, uint16_t* y, bool norm, cudaStream_t stream);

// gemv_group.cu: decode linear with group-wise scales (group a power of two
// in 128..1024; scales [N, ceil(K / group)]) on the per-tile TMA kernel, in
// passes of 32 tokens.
bool gemv_groups_supported(const uint16_t* x, int64_t M, int64_t N, int64_t K, int64_t group);
cudaError_t launch_gemv_groups(const uint16_t* x, const uint8_t* packed, const float* scales, int bits,
                               int64_t group, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                               cudaStream_t stream, unsigned qflags = 0u);

// shard.cu: gathered output blocks [world, M, Nl] -> y [M, N] (N <= world * Nl).
cudaError_t launch_gather_shards(const uint16_t* blocks, int64_t M, int64_t Nl, int64_t N, uint16_t* y,
                                 cudaStream_t stream);

// gemm_fp8.cu: per-token E4M3 activations (K % 16 == 0) and the E4M3 prefill
// GEMM for codes of 4 or 5 bits.
cudaError_t launch_quantize_x_fp8(const uint16_t* x, int64_t M, int64_t K, uint8_t* xq, float* sx,
                                  cudaStream_t stream);
cudaError_t launch_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* packed, const float* scales,
                            int bits, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                            cudaStream_t stream);

// gemm.cu: tcgen05 prefill GEMM; returns cudaErrorNotSupported for shapes it
// does not take (the caller then uses the GEMV path).
cudaError_t launch_gemm(const uint16_t* x, const uint8_t* packed, const float* scales,
                        int bits, int layout, int64_t M, int64_t N, int64_t K, uint16_t* y,
                        int32_t* dev_error, cudaStream_t stream);
bool gemm_supported(int64_t M, int64_t N, int64_t K);

// gemv_pass.cu: a decode pass (one token) over a stack of linears as one
// persistent kernel.  A plan owns its device memory (descriptors, tensor maps,
// dependency lists, counters, partial sums); the pointers in the layers must
// stay valid while it is used.
struct PassLayer {
  const uint16_t* x;       // input, K values
  uint16_t* y;             // output, N values
  const uint8_t* packed;   // paired rows
  const float* scales;
  int64_t N, K;
  int bits;
  bool norm;
};
struct PassPlan;
bool gemv_pass_layer_ok(int bits, int layout, int64_t N, int64_t K);
// Host only: for every linear the earlier linears it waits for (deps
// [dep0[i], dep0[i+1])); false if a linear's input and output overlap.
bool gemv_pass_dependencies(const PassLayer* layers, int64_t count, std::vector<int32_t>& deps,
                            std::vector<int32_t>& dep0);
cudaError_t gemv_pass_create(const PassLayer* layers, int64_t count, PassPlan** out);
cudaError_t gemv_pass_run(const PassPlan* plan, cudaStream_t stream);
void gemv_pass_destroy(PassPlan* plan);
// grid size, ring stages, work items, dynamic shared memory bytes
void gemv_pass_info(const PassPlan* plan, int64_t* info);

}  // namespace mpw
