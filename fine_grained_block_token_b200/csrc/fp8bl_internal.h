// Internal launch interface between the C-ABI layer (api.cu) and the
// kernel translation units.  Every launcher assumes the arguments were
// validated by the C-ABI layer.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

namespace fp8bl {

// Per-device state is kept in arrays indexed by the device ordinal.
constexpr int kMaxDevices = 64;

// Runs `init(dev)` once for each device -- the current device at the call --
// and returns the status it recorded for that device (kernel attributes such
// as the shared-memory opt-in belong to one device).  *dev_out receives the
// ordinal when given.
template <class Init>
cudaError_t once_per_device(std::once_flag* flags, cudaError_t* status, Init init,
                            int* dev_out = nullptr) {
  int dev = -1;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(flags[dev], [&] { status[dev] = init(dev); });
  if (dev_out) *dev_out = dev;
  return status[dev];
}

// Launch attribute for programmatic dependent launch: the kernel may begin
// while the previous kernel on the stream finishes; every kernel launched
// this way calls ptx::grid_dep_wait() before touching global memory that
// another kernel writes or reads.
inline void set_programmatic_serialization(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}

struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  int major = 0, minor = 0;
  size_t max_smem_optin = 0;
  int* error_flag = nullptr;   // device address of the kernel error word
};

// Per-device facts and the error-flag address (cached, thread-safe).
// Returns nullptr if the current device cannot be queried.
const DeviceInfo* device_info();

// Activation quantization, bf16 [M,K] -> e4m3 [M,K] + fp32 [M,K/128].
cudaError_t launch_act_quant(const void* x, int64_t M, int64_t K, void* q, float* s,
                             int sm_count, cudaStream_t st);

// Weight quantization, bf16 [N,K] -> e4m3 [N,K] + fp32 [N/128,K/128].
cudaError_t launch_weight_quant(const void* w, int64_t N, int64_t K, void* q, float* s,
                                cudaStream_t st);

// Static activation scale ("DeepGEMM fast path" section): q = e4m3(x / s)
// with the given fp32 scale *s_given (device), s[M, K/128] filled with it.
cudaError_t launch_act_quant_static(const void* x, int64_t M, int64_t K, const float* s_given,
                                    void* q, float* s, int sm_count, cudaStream_t st);

// UE8M0 variants of both ("UE8M0 scale format"): one byte per scale, the
// code e + 127 of the power-of-two scale 2^e.
cudaError_t launch_act_quant_ue8m0(const void* x, int64_t M, int64_t K, void* q, uint8_t* s,
                                   int sm_count, cudaStream_t st);
cudaError_t launch_weight_quant_ue8m0(const void* w, int64_t N, int64_t K, void* q, uint8_t* s,
                                      cudaStream_t st);

// Block-scaled GEMM with UE8M0 scales on the hardware block-scaled MMA
// (tcgen05.mma kind::mxf8f6f4.block_scale); no workspace.
cudaError_t launch_block_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                      const uint8_t* s_w, void* y, int64_t M, int64_t N,
                                      int64_t K, const DeviceInfo& dev, cudaStream_t st);

// UE8M0 block-scaled GEMM on CTA pairs (M > 128), plain (offsets = null,
// E = 1) or grouped: the workspace holds the scale factors rewritten in the
// tensor core's order.
constexpr int kMaxExperts = 1024;
bool ue8m0_use_pairs(int64_t M);
size_t ue8m0_pair_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E);
cudaError_t launch_linear_ue8m0_pairs(const void* q_a, const uint8_t* s_a, const void* q_w,
                                      const uint8_t* s_w, const int* offsets, void* y, int64_t M,
                                      int64_t N, int64_t K, int64_t E, void* workspace,
                                      const DeviceInfo& dev, cudaStream_t st);

// Row-wise e4m3 quantization ("BFL (fp8r / nvfp4)"): bf16 [R, K] -> e4m3
// [R, K] + one fp32 scale per row; K % 16 == 0.
cudaError_t launch_rowwise_quant(const void* x, int64_t R, int64_t K, void* q, float* s,
                                 cudaStream_t st);

// Row-wise scaled linear: y = bf16(s_a[m] s_w[n] sum_k q_a[m,k] q_w[n,k]),
// K and N multiples of 16; no workspace.
cudaError_t launch_linear_rowwise(const void* q_a, const float* s_a, const void* q_w,
                                  const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                  const DeviceInfo& dev, cudaStream_t st);

// Grouped (MoE expert) UE8M0 linear: row segments [off[e], off[e+1]) of
// q_a times expert e's weights, q_w [E, N, K], s_w [E, N/128, K/128].
cudaError_t launch_grouped_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                        const uint8_t* s_w, const int32_t* offsets, void* y,
                                        int64_t M, int64_t N, int64_t K, int64_t E,
                                        const DeviceInfo& dev, cudaStream_t st);

// Largest M served by the decode (swap-AB, stream-K) schedule.
constexpr int64_t kDecodeMaxM = 64;

// GEMM schedule, chosen on the host from the sizes.
struct GemmPlan {
  int kind = 0;          // 0 = prefill tile kernel, 1 = decode (swap-AB) kernel,
                         // 2 = fused prefill kernel (activation quantization in the tiles)
  int split_k = 1;       // number of K slices (decode / small grids)
  size_t workspace = 0;  // bytes of scratch the plan needs
  // fused plans: true when the in-GEMM quantization kernel (kind 2, no
  // workspace) may serve a call whose workspace is smaller than `workspace`
  bool in_kernel_ok = false;
};

GemmPlan plan_block_linear(int64_t M, int64_t N, int64_t K, int sm_count, bool fused);

// Block-scaled GEMM on CTA pairs (256 x 256 tiles), used for M > 128.
bool block_linear_use_pairs(int64_t M);
cudaError_t launch_block_linear_pairs(const void* q_a, const float* s_a, const void* q_w,
                                      const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                      const DeviceInfo& dev, cudaStream_t st);

cudaError_t launch_block_linear(const void* q_a, const float* s_a, const void* q_w,
                                const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                const GemmPlan& plan, void* workspace, const DeviceInfo& dev,
                                cudaStream_t st);

// Decode schedule (M <= kDecodeMaxM): scratch bytes and launch.
size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count);
cudaError_t launch_block_linear_decode(const void* q_a, const float* s_a, const void* q_w,
                                       const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                       void* workspace, const DeviceInfo& dev, cudaStream_t st);

// 2-D TMA map over a row-major byte matrix [rows, cols], box box_rows x
// box_cols, 128-byte swizzle unless told otherwise; out-of-range elements
// read as zero (and are not written by stores).
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, uint32_t box_cols,
                  CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B);

cudaError_t launch_block_linear_fused(const void* x, const void* q_w, const float* s_w, void* y,
                                      int64_t M, int64_t N, int64_t K, const GemmPlan& plan,
                                      void* workspace, const DeviceInfo& dev, cudaStream_t st);

// Fused prefill kernel (plan kind 2): activation quantization inside the
// GEMM's tiles; no workspace.
cudaError_t launch_block_linear_fused_tiles(const void* x, const void* q_w, const float* s_w,
                                            void* y, int64_t M, int64_t N, int64_t K,
                                            const DeviceInfo& dev, cudaStream_t st);

// Error codes a kernel writes into the error word (first error wins).
enum KernelError : int {
  kErrNone = 0,
  kErrTimeoutProducer = 1,
  kErrTimeoutMma = 2,
  kErrTimeoutEpilogue = 3,
  kErrTimeoutSelftest = 4,
};

}  // namespace fp8bl
