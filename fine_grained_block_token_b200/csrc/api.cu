// C-ABI entry points of libfp8bl (declared in include/fp8bl.h): argument
// validation on the host, schedule choice, launch on the caller's stream,
// and status reporting.  No call allocates device memory.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/fp8bl.h"
#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"

namespace fp8bl {
namespace {

// Error word written by kernels whose bounded waits ran out.  One int per
// device image of this library; read and cleared by fp8bl_check().
__device__ int g_kernel_error;

DeviceInfo g_info[kMaxDevices];
std::once_flag g_once[kMaxDevices];

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

bool dim_ok(int64_t v, bool allow_zero) {
  return (allow_zero ? v >= 0 : v > 0) && v <= FP8BL_MAX_DIM;
}

cudaStream_t as_cuda(fp8bl_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

fp8bl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8BL_OK : FP8BL_ERR_CUDA; }

// Common checks: device architecture; returns the device facts.
fp8bl_status current_device(const DeviceInfo** out) {
  const DeviceInfo* d = device_info();
  if (!d) return FP8BL_ERR_CUDA;
  if (d->major != 10 || d->minor != 0) return FP8BL_ERR_ARCH;
  *out = d;
  return FP8BL_OK;
}

}  // namespace

const DeviceInfo* device_info() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_once[dev], [dev] {
    DeviceInfo& d = g_info[dev];
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return;
    d.sm_count = v;
    cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.max_smem_optin = static_cast<size_t>(v);
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kernel_error) != cudaSuccess) return;
    d.error_flag = static_cast<int*>(p);
    d.device = dev;
  });
  const DeviceInfo* d = &g_info[dev];
  return d->device == dev ? d : nullptr;
}

}  // namespace fp8bl

using namespace fp8bl;

extern "C" {

int fp8bl_version(void) { return 100; }

const char* fp8bl_status_string(fp8bl_status s) {
  switch (s) {
    case FP8BL_OK: return "ok";
    case FP8BL_ERR_NULL: return "a required pointer is NULL";
    case FP8BL_ERR_SHAPE: return "invalid sizes (need K, N multiples of 128, within limits)";
    case FP8BL_ERR_ALIGN: return "pointer not 16-byte aligned (4-byte for fp32 scales)";
    case FP8BL_ERR_ARCH: return "current device is not compute capability 10.0 (sm_100)";
    case FP8BL_ERR_CUDA: return "CUDA call failed";
    case FP8BL_ERR_TIMEOUT: return "a kernel wait ran out of time";
    case FP8BL_ERR_WORKSPACE: return "workspace smaller than required";
    case FP8BL_ERR_OVERLAP: return "an output buffer overlaps an input buffer";
  }
  return "unknown status";
}

fp8bl_status fp8_quant_act(const void* x_bf16, int64_t M, int64_t K, void* q_e4m3, float* s,
                           fp8bl_stream_t stream) {
  if (!dim_ok(M, true) || !dim_ok(K, false) || K % FP8BL_BLOCK) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!x_bf16 || !q_e4m3 || !s) return FP8BL_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 16) || !aligned(s, 4)) return FP8BL_ERR_ALIGN;
  const size_t nx = static_cast<size_t>(M * K) * 2, nq = static_cast<size_t>(M * K),
               ns = static_cast<size_t>(M * (K / 128)) * 4;
  if (overlap(x_bf16, nx, q_e4m3, nq) || overlap(x_bf16, nx, s, ns) || overlap(q_e4m3, nq, s, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(launch_act_quant(x_bf16, M, K, q_e4m3, s, d->sm_count, as_cuda(stream)));
}

fp8bl_status fp8_quant_act_static(const void* x_bf16, int64_t M, int64_t K, const float* s_given,
                                  void* q_e4m3, float* s, fp8bl_stream_t stream) {
  if (!dim_ok(M, true) || !dim_ok(K, false) || K % FP8BL_BLOCK) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!x_bf16 || !s_given || !q_e4m3 || !s) return FP8BL_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 16) || !aligned(s, 4) || !aligned(s_given, 4))
    return FP8BL_ERR_ALIGN;
  const size_t nx = static_cast<size_t>(M * K) * 2, nq = static_cast<size_t>(M * K),
               ns = static_cast<size_t>(M * (K / 128)) * 4;
  if (overlap(x_bf16, nx, q_e4m3, nq) || overlap(x_bf16, nx, s, ns) || overlap(q_e4m3, nq, s, ns) ||
      overlap(s_given, 4, q_e4m3, nq) || overlap(s_given, 4, s, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(
      launch_act_quant_static(x_bf16, M, K, s_given, q_e4m3, s, d->sm_count, as_cuda(stream)));
}

fp8bl_status fp8_quant_weight(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3, float* s,
                              fp8bl_stream_t stream) {
  if (!dim_ok(N, false) || !dim_ok(K, false) || N % FP8BL_BLOCK || K % FP8BL_BLOCK)
    return FP8BL_ERR_SHAPE;
  if (!w_bf16 || !q_e4m3 || !s) return FP8BL_ERR_NULL;
  if (!aligned(w_bf16, 16) || !aligned(q_e4m3, 16) || !aligned(s, 4)) return FP8BL_ERR_ALIGN;
  const size_t nw = static_cast<size_t>(N * K) * 2, nq = static_cast<size_t>(N * K),
               ns = static_cast<size_t>((N / 128) * (K / 128)) * 4;
  if (overlap(w_bf16, nw, q_e4m3, nq) || overlap(w_bf16, nw, s, ns) || overlap(q_e4m3, nq, s, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(launch_weight_quant(w_bf16, N, K, q_e4m3, s, as_cuda(stream)));
}

static bool linear_dims_ok(int64_t M, int64_t N, int64_t K) {
  return dim_ok(M, true) && dim_ok(N, false) && dim_ok(K, false) && N % FP8BL_BLOCK == 0 &&
         K % FP8BL_BLOCK == 0;
}

size_t fp8_block_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (!linear_dims_ok(M, N, K)) return 0;
  const DeviceInfo* d = device_info();
  return plan_block_linear(M, N, K, d ? d->sm_count : 148, false).workspace;
}

size_t fp8_block_linear_fused_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (!linear_dims_ok(M, N, K)) return 0;
  const DeviceInfo* d = device_info();
  return plan_block_linear(M, N, K, d ? d->sm_count : 148, true).workspace;
}

fp8bl_status fp8_block_linear(const void* q_a, const float* s_a, const void* q_w,
                              const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                              void* workspace, size_t workspace_bytes, fp8bl_stream_t stream) {
  if (!linear_dims_ok(M, N, K)) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(q_a, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16) || !aligned(s_a, 4) ||
      !aligned(s_w, 4) || !aligned(workspace, 16))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (overlap(y_bf16, ny, q_a, static_cast<size_t>(M * K)) ||
      overlap(y_bf16, ny, q_w, static_cast<size_t>(N * K)) ||
      overlap(y_bf16, ny, s_a, static_cast<size_t>(M * (K / 128)) * 4) ||
      overlap(y_bf16, ny, s_w, static_cast<size_t>((N / 128) * (K / 128)) * 4))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  const GemmPlan plan = plan_block_linear(M, N, K, d->sm_count, false);
  if (plan.workspace > 0) {
    if (!workspace) return FP8BL_ERR_NULL;
    if (workspace_bytes < plan.workspace) return FP8BL_ERR_WORKSPACE;
    if (overlap(workspace, plan.workspace, y_bf16, ny)) return FP8BL_ERR_OVERLAP;
  }
  return from_cuda(launch_block_linear(q_a, s_a, q_w, s_w, y_bf16, M, N, K, plan, workspace, *d,
                                       as_cuda(stream)));
}

fp8bl_status fp8_block_linear_fused(const void* x_bf16, const void* q_w, const float* s_w,
                                    void* y_bf16, int64_t M, int64_t N, int64_t K, void* workspace,
                                    size_t workspace_bytes, fp8bl_stream_t stream) {
  if (!linear_dims_ok(M, N, K)) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!x_bf16 || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16) || !aligned(s_w, 4) ||
      !aligned(workspace, 16))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (overlap(y_bf16, ny, x_bf16, static_cast<size_t>(M * K) * 2) ||
      overlap(y_bf16, ny, q_w, static_cast<size_t>(N * K)) ||
      overlap(y_bf16, ny, s_w, static_cast<size_t>((N / 128) * (K / 128)) * 4))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  GemmPlan plan = plan_block_linear(M, N, K, d->sm_count, true);
  if (plan.in_kernel_ok && (!workspace || workspace_bytes < plan.workspace)) {
    // prefill sizes without the staging workspace: quantize in the tiles
    plan.kind = 2;
    plan.workspace = 0;
  }
  if (plan.workspace > 0) {
    if (!workspace) return FP8BL_ERR_NULL;
    if (workspace_bytes < plan.workspace) return FP8BL_ERR_WORKSPACE;
    if (overlap(workspace, plan.workspace, y_bf16, ny) ||
        overlap(workspace, plan.workspace, x_bf16, static_cast<size_t>(M * K) * 2) ||
        overlap(workspace, plan.workspace, q_w, static_cast<size_t>(N * K)) ||
        overlap(workspace, plan.workspace, s_w, static_cast<size_t>((N / 128) * (K / 128)) * 4))
      return FP8BL_ERR_OVERLAP;
  }
  return from_cuda(launch_block_linear_fused(x_bf16, q_w, s_w, y_bf16, M, N, K, plan, workspace,
                                             *d, as_cuda(stream)));
}

fp8bl_status fp8_quant_act_ue8m0(const void* x_bf16, int64_t M, int64_t K, void* q_e4m3,
                                 uint8_t* s_ue8m0, fp8bl_stream_t stream) {
  if (!dim_ok(M, true) || !dim_ok(K, false) || K % FP8BL_BLOCK) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!x_bf16 || !q_e4m3 || !s_ue8m0) return FP8BL_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 16)) return FP8BL_ERR_ALIGN;
  const size_t nx = static_cast<size_t>(M * K) * 2, nq = static_cast<size_t>(M * K),
               ns = static_cast<size_t>(M * (K / 128));
  if (overlap(x_bf16, nx, q_e4m3, nq) || overlap(x_bf16, nx, s_ue8m0, ns) ||
      overlap(q_e4m3, nq, s_ue8m0, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(
      launch_act_quant_ue8m0(x_bf16, M, K, q_e4m3, s_ue8m0, d->sm_count, as_cuda(stream)));
}

fp8bl_status fp8_quant_weight_ue8m0(const void* w_bf16, int64_t N, int64_t K, void* q_e4m3,
                                    uint8_t* s_ue8m0, fp8bl_stream_t stream) {
  if (!dim_ok(N, false) || !dim_ok(K, false) || N % FP8BL_BLOCK || K % FP8BL_BLOCK)
    return FP8BL_ERR_SHAPE;
  if (!w_bf16 || !q_e4m3 || !s_ue8m0) return FP8BL_ERR_NULL;
  if (!aligned(w_bf16, 16) || !aligned(q_e4m3, 16)) return FP8BL_ERR_ALIGN;
  const size_t nw = static_cast<size_t>(N * K) * 2, nq = static_cast<size_t>(N * K),
               ns = static_cast<size_t>((N / 128) * (K / 128));
  if (overlap(w_bf16, nw, q_e4m3, nq) || overlap(w_bf16, nw, s_ue8m0, ns) ||
      overlap(q_e4m3, nq, s_ue8m0, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(launch_weight_quant_ue8m0(w_bf16, N, K, q_e4m3, s_ue8m0, as_cuda(stream)));
}

fp8bl_status fp8_block_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                    const uint8_t* s_w, void* y_bf16, int64_t M, int64_t N,
                                    int64_t K, fp8bl_stream_t stream) {
  if (!linear_dims_ok(M, N, K)) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(q_a, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16)) return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (overlap(y_bf16, ny, q_a, static_cast<size_t>(M * K)) ||
      overlap(y_bf16, ny, q_w, static_cast<size_t>(N * K)) ||
      overlap(y_bf16, ny, s_a, static_cast<size_t>(M * (K / 128))) ||
      overlap(y_bf16, ny, s_w, static_cast<size_t>((N / 128) * (K / 128))))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(
      launch_block_linear_ue8m0(q_a, s_a, q_w, s_w, y_bf16, M, N, K, *d, as_cuda(stream)));
}

size_t fp8_block_linear_ue8m0_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (!linear_dims_ok(M, N, K)) return 0;
  return ue8m0_pair_workspace_bytes(M, N, K, 1);
}

fp8bl_status fp8_block_linear_ue8m0_ws(const void* q_a, const uint8_t* s_a, const void* q_w,
                                       const uint8_t* s_w, void* y_bf16, int64_t M, int64_t N,
                                       int64_t K, void* workspace, size_t workspace_bytes,
                                       fp8bl_stream_t stream) {
  if (!linear_dims_ok(M, N, K)) return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(q_a, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16) || !aligned(workspace, 16))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  const size_t na = static_cast<size_t>(M * K), nw = static_cast<size_t>(N * K);
  const size_t nsa = static_cast<size_t>(M * (K / 128)), nsw = static_cast<size_t>((N / 128) * (K / 128));
  if (overlap(y_bf16, ny, q_a, na) || overlap(y_bf16, ny, q_w, nw) || overlap(y_bf16, ny, s_a, nsa) ||
      overlap(y_bf16, ny, s_w, nsw))
    return FP8BL_ERR_OVERLAP;
  const size_t need = ue8m0_pair_workspace_bytes(M, N, K, 1);
  if (need > 0) {
    if (!workspace) return FP8BL_ERR_NULL;
    if (workspace_bytes < need) return FP8BL_ERR_WORKSPACE;
    if (overlap(workspace, need, y_bf16, ny) || overlap(workspace, need, q_a, na) ||
        overlap(workspace, need, q_w, nw) || overlap(workspace, need, s_a, nsa) ||
        overlap(workspace, need, s_w, nsw))
      return FP8BL_ERR_OVERLAP;
  }
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  if (need == 0)
    return from_cuda(
        launch_block_linear_ue8m0(q_a, s_a, q_w, s_w, y_bf16, M, N, K, *d, as_cuda(stream)));
  return from_cuda(launch_linear_ue8m0_pairs(q_a, s_a, q_w, s_w, nullptr, y_bf16, M, N, K, 1,
                                             workspace, *d, as_cuda(stream)));
}

namespace {
// Checks shared by the grouped calls; sets *done when there is no work.
fp8bl_status check_grouped(const void* q_a, const uint8_t* s_a, const void* q_w,
                           const uint8_t* s_w, const int32_t* expert_offsets, void* y_bf16,
                           int64_t M, int64_t N, int64_t K, int64_t E, bool* done) {
  *done = false;
  if (!linear_dims_ok(M, N, K) || E < 1 || E > kMaxExperts || N * E > FP8BL_MAX_DIM)
    return FP8BL_ERR_SHAPE;
  if (M == 0) {
    *done = true;
    return FP8BL_OK;
  }
  if (!q_a || !s_a || !q_w || !s_w || !expert_offsets || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(q_a, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16) || !aligned(expert_offsets, 4))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (overlap(y_bf16, ny, q_a, static_cast<size_t>(M * K)) ||
      overlap(y_bf16, ny, q_w, static_cast<size_t>(E * N * K)) ||
      overlap(y_bf16, ny, s_a, static_cast<size_t>(M * (K / 128))) ||
      overlap(y_bf16, ny, s_w, static_cast<size_t>(E * (N / 128) * (K / 128))) ||
      overlap(y_bf16, ny, expert_offsets, static_cast<size_t>(E + 1) * 4))
    return FP8BL_ERR_OVERLAP;
  return FP8BL_OK;
}
}  // namespace

fp8bl_status fp8_grouped_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                      const uint8_t* s_w, const int32_t* expert_offsets,
                                      void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t E,
                                      fp8bl_stream_t stream) {
  bool done = false;
  fp8bl_status st = check_grouped(q_a, s_a, q_w, s_w, expert_offsets, y_bf16, M, N, K, E, &done);
  if (st != FP8BL_OK || done) return st;
  const DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(launch_grouped_linear_ue8m0(q_a, s_a, q_w, s_w, expert_offsets, y_bf16, M, N,
                                               K, E, *d, as_cuda(stream)));
}

size_t fp8_grouped_linear_ue8m0_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E) {
  if (!linear_dims_ok(M, N, K) || E < 1 || E > kMaxExperts || N * E > FP8BL_MAX_DIM) return 0;
  return ue8m0_pair_workspace_bytes(M, N, K, E);
}

fp8bl_status fp8_grouped_linear_ue8m0_ws(const void* q_a, const uint8_t* s_a, const void* q_w,
                                         const uint8_t* s_w, const int32_t* expert_offsets,
                                         void* y_bf16, int64_t M, int64_t N, int64_t K, int64_t E,
                                         void* workspace, size_t workspace_bytes,
                                         fp8bl_stream_t stream) {
  bool done = false;
  fp8bl_status st = check_grouped(q_a, s_a, q_w, s_w, expert_offsets, y_bf16, M, N, K, E, &done);
  if (st != FP8BL_OK || done) return st;
  if (!aligned(workspace, 16)) return FP8BL_ERR_ALIGN;
  const size_t need = ue8m0_pair_workspace_bytes(M, N, K, E);
  if (need > 0) {
    if (!workspace) return FP8BL_ERR_NULL;
    if (workspace_bytes < need) return FP8BL_ERR_WORKSPACE;
    if (overlap(workspace, need, y_bf16, static_cast<size_t>(M * N) * 2) ||
        overlap(workspace, need, q_a, static_cast<size_t>(M * K)) ||
        overlap(workspace, need, q_w, static_cast<size_t>(E * N * K)) ||
        overlap(workspace, need, s_a, static_cast<size_t>(M * (K / 128))) ||
        overlap(workspace, need, s_w, static_cast<size_t>(E * (N / 128) * (K / 128))) ||
        overlap(workspace, need, expert_offsets, static_cast<size_t>(E + 1) * 4))
      return FP8BL_ERR_OVERLAP;
  }
  const DeviceInfo* d = nullptr;
  st = current_device(&d);
  if (st != FP8BL_OK) return st;
  if (need == 0)
    return from_cuda(launch_grouped_linear_ue8m0(q_a, s_a, q_w, s_w, expert_offsets, y_bf16, M, N,
                                                 K, E, *d, as_cuda(stream)));
  return from_cuda(launch_linear_ue8m0_pairs(q_a, s_a, q_w, s_w, expert_offsets, y_bf16, M, N, K,
                                             E, workspace, *d, as_cuda(stream)));
}

fp8bl_status fp8_quant_rowwise(const void* x_bf16, int64_t R, int64_t K, void* q_e4m3, float* s,
                               fp8bl_stream_t stream) {
  if (!dim_ok(R, true) || !dim_ok(K, false) || K % 16) return FP8BL_ERR_SHAPE;
  if (R == 0) return FP8BL_OK;
  if (!x_bf16 || !q_e4m3 || !s) return FP8BL_ERR_NULL;
  if (!aligned(x_bf16, 16) || !aligned(q_e4m3, 16) || !aligned(s, 4)) return FP8BL_ERR_ALIGN;
  const size_t nx = static_cast<size_t>(R * K) * 2, nq = static_cast<size_t>(R * K),
               ns = static_cast<size_t>(R) * 4;
  if (overlap(x_bf16, nx, q_e4m3, nq) || overlap(x_bf16, nx, s, ns) || overlap(q_e4m3, nq, s, ns))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(launch_rowwise_quant(x_bf16, R, K, q_e4m3, s, as_cuda(stream)));
}

fp8bl_status fp8_linear_rowwise(const void* q_a, const float* s_a, const void* q_w,
                                const float* s_w, void* y_bf16, int64_t M, int64_t N, int64_t K,
                                fp8bl_stream_t stream) {
  if (!dim_ok(M, true) || !dim_ok(N, false) || !dim_ok(K, false) || N % 16 || K % 16)
    return FP8BL_ERR_SHAPE;
  if (M == 0) return FP8BL_OK;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!aligned(q_a, 16) || !aligned(q_w, 16) || !aligned(y_bf16, 16) || !aligned(s_a, 4) ||
      !aligned(s_w, 16))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (overlap(y_bf16, ny, q_a, static_cast<size_t>(M * K)) ||
      overlap(y_bf16, ny, q_w, static_cast<size_t>(N * K)) ||
      overlap(y_bf16, ny, s_a, static_cast<size_t>(M) * 4) ||
      overlap(y_bf16, ny, s_w, static_cast<size_t>(N) * 4))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  return from_cuda(
      launch_linear_rowwise(q_a, s_a, q_w, s_w, y_bf16, M, N, K, *d, as_cuda(stream)));
}

namespace fp8bl {
namespace {
// One thread waits on a freshly initialised mbarrier (phase 0 never
// completes) with the kernels' bounded waits; on expiry it records the
// timeout exactly as the GEMM and quantization kernels do.
__global__ void selftest_wait_kernel(uint64_t limit_cycles, int kind, int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t b = ptx::smem_u32(&bar);
    ptx::mbar_init(b, 1);
    ptx::fence_barrier_init();
    const bool ok = kind == 0 ? ptx::mbar_wait(b, 0, limit_cycles)
                              : ptx::mbar_wait_spin(b, 0, limit_cycles);
    if (!ok) atomicCAS(err, 0, kErrTimeoutSelftest);
  }
}
}  // namespace
}  // namespace fp8bl

fp8bl_status fp8bl_selftest_wait_timeout(uint64_t limit_cycles, int kind, fp8bl_stream_t stream) {
  if (limit_cycles == 0 || limit_cycles > (uint64_t{1} << 32) || (kind != 0 && kind != 1))
    return FP8BL_ERR_SHAPE;
  const DeviceInfo* d = nullptr;
  fp8bl_status st = current_device(&d);
  if (st != FP8BL_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, as_cuda(stream)>>>(limit_cycles, kind, d->error_flag);
  return from_cuda(cudaGetLastError());
}

fp8bl_status fp8bl_check(fp8bl_stream_t stream) {
  if (cudaStreamSynchronize(as_cuda(stream)) != cudaSuccess) return FP8BL_ERR_CUDA;
  const DeviceInfo* d = device_info();
  if (!d) return FP8BL_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, d->error_flag, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
    return FP8BL_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    cudaMemcpy(d->error_flag, &zero, sizeof zero, cudaMemcpyHostToDevice);
    return FP8BL_ERR_TIMEOUT;
  }
  return FP8BL_OK;
}

}  // extern "C"
