// Activation (1 x 128 per token) and weight (128 x 128) e4m3 quantization
// kernels.  "Fine-grained FP8" page, opening bullet list: weights per
// 128 x 128 block, activations per token in groups of 128 input channels.
//
// Activation kernel: with K % 128 == 0 the 1 x 128 groups of a row-major
// [M, K] tensor are consecutive 256-byte chunks of the flat array, and the
// scale of group g sits at s[g] of the row-major [M, K/128] scale tensor.
// The kernel is therefore a flat stream over groups: a half-warp owns one
// group (16 lanes x 16 bytes), reduces amax with four xor-shuffles, and
// writes 8 bytes of codes per lane (the warp writes 256 contiguous bytes)
// plus one scale.  Each warp keeps UNROLL pairs of groups in flight so the
// SM has enough bytes outstanding to run at HBM bandwidth.
//
// The kernels are instantiated per scale mode: kMode 0 writes fp32 scales
// (s = amax / 448); kMode 1 writes UE8M0 codes (the "UE8M0 scale format"
// section of the same page: the scale rounded up to a power of two, one byte
// each) and multiplies by the exact power of two instead of dividing;
// kMode 2 (activations only) is the static scheme of the page's "DeepGEMM
// fast path" section: one given fp32 scale for the whole tensor, no abs-max,
// written into every group's scale slot so the block GEMM applies it.
#include <cstdint>
#include <cuda_runtime.h>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"
#include "quant_math.cuh"

namespace fp8bl {
namespace {

constexpr int kAqThreads = 256;
constexpr int kAqUnroll = 4;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr int kModeFp32 = 0;
constexpr int kModeUe8m0 = 1;
constexpr int kModeStatic = 2;

// Per-group constants of each scale mode, from the group's amax (or, for
// the static mode, from the given scale).
template <int kMode>
struct GroupQuant;

template <>
struct GroupQuant<kModeFp32> {
  float s;
  GroupScale g;
  __device__ __forceinline__ explicit GroupQuant(float amax)
      : s(scale_from_amax(amax)), g(group_scale(s)) {}
  __device__ __forceinline__ uint2 quant(uint4 v) const { return quant8(v, g); }
  __device__ __forceinline__ void store_scale(void* out, int64_t i) const {
    static_cast<float*>(out)[i] = s;
  }
};

template <>
struct GroupQuant<kModeStatic> {
  float s;
  GroupScale g;
  __device__ __forceinline__ explicit GroupQuant(float given) : s(given), g(group_scale(given)) {}
  __device__ __forceinline__ uint2 quant(uint4 v) const { return quant8(v, g); }
  __device__ __forceinline__ void store_scale(void* out, int64_t i) const {
    static_cast<float*>(out)[i] = s;
  }
};

template <>
struct GroupQuant<kModeUe8m0> {
  uint32_t code;
  float2 inv;
  __device__ __forceinline__ explicit GroupQuant(float amax)
      : code(ue8m0_from_amax(amax)), inv(ue8m0_inverse2(code)) {}
  __device__ __forceinline__ uint2 quant(uint4 v) const { return quant8_pow2(v, inv); }
  __device__ __forceinline__ void store_scale(void* out, int64_t i) const {
    static_cast<uint8_t*>(out)[i] = static_cast<uint8_t>(code);
  }
};

// num_groups = M * K / 128.  x: 16 uint4 per group; q: 16 uint2 per group.
template <int kMode>
__global__ void __launch_bounds__(kAqThreads, 4)
act_quant_kernel(const uint4* __restrict__ x, uint2* __restrict__ q, void* __restrict__ s,
                 int64_t num_groups, const float* __restrict__ s_given) {
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();
  const float given = kMode == kModeStatic ? __ldg(s_given) : 0.0f;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kAqThreads + threadIdx.x) >> 5;
  const int64_t num_warps = (static_cast<int64_t>(gridDim.x) * kAqThreads) >> 5;
  const int64_t num_pairs = (num_groups + 1) >> 1;
  // The loop bound depends on the warp only, so every shuffle below runs
  // with all 32 lanes present.
  for (int64_t p0 = warp; p0 < num_pairs; p0 += num_warps * kAqUnroll) {
    uint4 v[kAqUnroll];
#pragma unroll
    for (int u = 0; u < kAqUnroll; ++u) {
      const int64_t g = (p0 + u * num_warps) * 2 + half;
      v[u] = g < num_groups ? ld_stream(x + g * 16 + l16) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kAqUnroll; ++u) {
      const int64_t g = (p0 + u * num_warps) * 2 + half;
      float a = given;
      if (kMode != kModeStatic) {
        uint32_t m = absmax8_bf16x2(v[u]);
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 1));
        a = absmax_halves_f32(m);
      }
      const GroupQuant<kMode> gq(a);
      const uint2 o = gq.quant(v[u]);
      if (g < num_groups) {
        q[g * 16 + l16] = o;
        if (l16 == 0) gq.store_scale(s, g);
      }
    }
  }
}

// 32-byte variant (input 32-byte aligned): a lane loads 32 contiguous bytes
// (16 bf16) with one 256-bit load, 8 lanes own a group and a warp covers 4
// consecutive groups (1 KB) per load instruction.  The per-group work (abs-max
// shuffles, scale, reciprocal) is then spread over twice as many elements,
// and each lane stores 16 codes with one 16-byte store.
constexpr int kAq32Unroll = 2;

__device__ __forceinline__ void ld_stream32(const uint4* p, uint4& a, uint4& b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z),
                 "=r"(b.w)
               : "l"(p));
}

template <int kMode>
__global__ void __launch_bounds__(kAqThreads, 4)
act_quant32_kernel(const uint4* __restrict__ x, uint4* __restrict__ q, void* __restrict__ s,
                   int64_t num_groups, const float* __restrict__ s_given) {
  ptx::grid_dep_wait();
  ptx::grid_dep_launch();
  const float given = kMode == kModeStatic ? __ldg(s_given) : 0.0f;
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 3;      // group within the warp's 4
  const int l8 = lane & 7;        // 32-byte slice within the group
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kAqThreads + threadIdx.x) >> 5;
  const int64_t num_warps = (static_cast<int64_t>(gridDim.x) * kAqThreads) >> 5;
  const int64_t num_quads = (num_groups + 3) >> 2;
  // The loop bound depends on the warp only: every shuffle has all lanes.
  for (int64_t p0 = warp; p0 < num_quads; p0 += num_warps * kAq32Unroll) {
    uint4 va[kAq32Unroll], vb[kAq32Unroll];
#pragma unroll
    for (int u = 0; u < kAq32Unroll; ++u) {
      const int64_t g = (p0 + u * num_warps) * 4 + sub;
      if (g < num_groups) {
        ld_stream32(x + g * 16 + l8 * 2, va[u], vb[u]);
      } else {
        va[u] = make_uint4(0u, 0u, 0u, 0u);
        vb[u] = va[u];
      }
    }
#pragma unroll
    for (int u = 0; u < kAq32Unroll; ++u) {
      const int64_t g = (p0 + u * num_warps) * 4 + sub;
      float a = given;
      if (kMode != kModeStatic) {
        uint32_t m = absmax_bf16x2(absmax8_bf16x2(va[u]), absmax8_bf16x2(vb[u]));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 1));
        a = absmax_halves_f32(m);
      }
      const GroupQuant<kMode> gq(a);
      const uint2 lo = gq.quant(va[u]), hi = gq.quant(vb[u]);
      if (g < num_groups) {
        q[g * 8 + l8] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        if (l8 == 0) gq.store_scale(s, g);
      }
    }
  }
}

// One CTA per 128 x 128 block.  Thread t covers 16-byte chunk (t % 16) of
// rows (t / 16) + 16 i, i = 0..7: every load instruction of a warp reads two
// full 256-byte row segments.
constexpr int kWqThreads = 256;

template <int kMode>
__global__ void __launch_bounds__(kWqThreads)
weight_quant_kernel(const uint4* __restrict__ w, uint2* __restrict__ q, void* __restrict__ s,
                    int64_t K, int64_t KB) {
  __shared__ float warp_amax[kWqThreads / 32];
  const int64_t blk = blockIdx.x;
  const int64_t bi = blk / KB, bj = blk % KB;
  const int c = threadIdx.x & 15;
  const int r0 = threadIdx.x >> 4;
  const int64_t row_stride = K / 8;   // uint4 per row
  const int64_t base = (bi * 128 + r0) * row_stride + bj * 16 + c;
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = ld_stream(w + base + static_cast<int64_t>(16 * i) * row_stride);
  uint32_t m = absmax8_bf16x2(v[0]);
#pragma unroll
  for (int i = 1; i < 8; ++i) m = absmax_bf16x2(m, absmax8_bf16x2(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, o));
  float a = absmax_halves_f32(m);
  if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = a;
  __syncthreads();
  a = warp_amax[0];
#pragma unroll
  for (int i = 1; i < kWqThreads / 32; ++i) a = fmaxf(a, warp_amax[i]);
  const GroupQuant<kMode> gq(a);
  const int64_t qrow_stride = K / 8;  // uint2 per row
  const int64_t qbase = (bi * 128 + r0) * qrow_stride + bj * 16 + c;
#pragma unroll
  for (int i = 0; i < 8; ++i) q[qbase + static_cast<int64_t>(16 * i) * qrow_stride] = gq.quant(v[i]);
  if (threadIdx.x == 0) gq.store_scale(s, bi * KB + bj);
}

}  // namespace

namespace {

// Launch with programmatic stream serialization (the kernels wait for the
// previous kernel before their first global access).
template <class Kernel, class... Args>
cudaError_t launch_pdl(Kernel k, int blocks, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
  cfg.blockDim = dim3(kAqThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  set_programmatic_serialization(at[0]);
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

template <int kMode>
cudaError_t act_quant(const void* x, int64_t M, int64_t K, void* q, void* s, int sm_count,
                      cudaStream_t st, const float* s_given = nullptr) {
  const int64_t groups = M * (K / 128);
  if (groups == 0) return cudaSuccess;
  if ((reinterpret_cast<uintptr_t>(x) & 31) == 0) {
    const int64_t quads = (groups + 3) / 4;
    const int64_t warps_needed = (quads + kAq32Unroll - 1) / kAq32Unroll;
    const int64_t blocks_needed = (warps_needed + (kAqThreads / 32) - 1) / (kAqThreads / 32);
    const int64_t max_blocks = static_cast<int64_t>(sm_count) * 4;
    const int blocks = static_cast<int>(blocks_needed < max_blocks ? blocks_needed : max_blocks);
    return launch_pdl(act_quant32_kernel<kMode>, blocks, st, static_cast<const uint4*>(x),
                      static_cast<uint4*>(q), s, groups, s_given);
  }
  const int64_t pairs = (groups + 1) / 2;
  const int64_t warps_needed = (pairs + kAqUnroll - 1) / kAqUnroll;
  const int64_t blocks_needed = (warps_needed + (kAqThreads / 32) - 1) / (kAqThreads / 32);
  // One pass of resident CTAs (4 per SM at <= 64 registers); larger inputs
  // loop inside the kernel.
  const int64_t max_blocks = static_cast<int64_t>(sm_count) * 4;
  const int blocks = static_cast<int>(blocks_needed < max_blocks ? blocks_needed : max_blocks);
  return launch_pdl(act_quant_kernel<kMode>, blocks, st, static_cast<const uint4*>(x),
                    static_cast<uint2*>(q), s, groups, s_given);
}

template <int kMode>
cudaError_t weight_quant(const void* w, int64_t N, int64_t K, void* q, void* s, cudaStream_t st) {
  const int64_t KB = K / 128;
  const int64_t blocks = (N / 128) * KB;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  weight_quant_kernel<kMode><<<static_cast<unsigned>(blocks), kWqThreads, 0, st>>>(
      static_cast<const uint4*>(w), static_cast<uint2*>(q), s, K, KB);
  return cudaGetLastError();
}

// Row-wise quantization ("BFL (fp8r / nvfp4)" page: one scale per row of
// the weight, and per token row of the activations).  One CTA per row: the
// row's 16-byte vectors are strided over the threads, the first kRowCache
// per thread stay in registers between the abs-max pass and the quantizing
// pass (rows up to 8192 elements are read once), the rest are read again
// (from L2).  The scale and the division are those of the 1 x 128 groups.
constexpr int kRowThreads = 256;
constexpr int kRowCache = 4;

__global__ void __launch_bounds__(kRowThreads)
rowwise_quant_kernel(const uint4* __restrict__ x, uint2* __restrict__ q, float* __restrict__ s,
                     int64_t nvec) {
  __shared__ uint32_t warp_amax[kRowThreads / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * nvec;
  uint2* qr = q + row * nvec;
  uint4 cache[kRowCache];
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < kRowCache; ++i) {
    const int64_t v = threadIdx.x + static_cast<int64_t>(i) * kRowThreads;
    cache[i] = v < nvec ? ld_stream(xr + v) : make_uint4(0u, 0u, 0u, 0u);
    m = absmax_bf16x2(m, absmax8_bf16x2(cache[i]));
  }
  for (int64_t v = threadIdx.x + kRowCache * kRowThreads; v < nvec; v += kRowThreads)
    m = absmax_bf16x2(m, absmax8_bf16x2(__ldg(xr + v)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) warp_amax[threadIdx.x >> 5] = m;
  __syncthreads();
  m = warp_amax[0];
#pragma unroll
  for (int i = 1; i < kRowThreads / 32; ++i) m = absmax_bf16x2(m, warp_amax[i]);
  const GroupQuant<kModeFp32> gq(absmax_halves_f32(m));
#pragma unroll
  for (int i = 0; i < kRowCache; ++i) {
    const int64_t v = threadIdx.x + static_cast<int64_t>(i) * kRowThreads;
    if (v < nvec) qr[v] = gq.quant(cache[i]);
  }
  for (int64_t v = threadIdx.x + kRowCache * kRowThreads; v < nvec; v += kRowThreads)
    qr[v] = gq.quant(__ldg(xr + v));
  if (threadIdx.x == 0) gq.store_scale(s, row);
}

}  // namespace

cudaError_t launch_rowwise_quant(const void* x, int64_t R, int64_t K, void* q, float* s,
                                 cudaStream_t st) {
  if (R == 0) return cudaSuccess;
  if (R > 0x7FFFFFFFll) return cudaErrorInvalidConfiguration;
  rowwise_quant_kernel<<<static_cast<unsigned>(R), kRowThreads, 0, st>>>(
      static_cast<const uint4*>(x), static_cast<uint2*>(q), s, K / 8);
  return cudaGetLastError();
}

cudaError_t launch_act_quant(const void* x, int64_t M, int64_t K, void* q, float* s,
                             int sm_count, cudaStream_t st) {
  return act_quant<kModeFp32>(x, M, K, q, s, sm_count, st);
}

cudaError_t launch_act_quant_ue8m0(const void* x, int64_t M, int64_t K, void* q, uint8_t* s,
                                   int sm_count, cudaStream_t st) {
  return act_quant<kModeUe8m0>(x, M, K, q, s, sm_count, st);
}

cudaError_t launch_act_quant_static(const void* x, int64_t M, int64_t K, const float* s_given,
                                    void* q, float* s, int sm_count, cudaStream_t st) {
  return act_quant<kModeStatic>(x, M, K, q, s, sm_count, st, s_given);
}

cudaError_t launch_weight_quant(const void* w, int64_t N, int64_t K, void* q, float* s,
                                cudaStream_t st) {
  return weight_quant<kModeFp32>(w, N, K, q, s, st);
}

cudaError_t launch_weight_quant_ue8m0(const void* w, int64_t N, int64_t K, void* q, uint8_t* s,
                                      cudaStream_t st) {
  return weight_quant<kModeUe8m0>(w, N, K, q, s, st);
}

}  // namespace fp8bl
