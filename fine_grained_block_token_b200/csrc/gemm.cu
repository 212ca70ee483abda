// Block-scaled FP8 GEMM for sm_100a:  y = bf16( sum_j s_a[:,j] s_w[:,j] (A_j W_j^T) )
//
// "Fine-grained FP8" page: weights carry one scale per 128 x 128 block,
// activations one per (token, 128-group) along the input channel, and the
// FP8 linear applies both per 128-deep K block.  Because the scales change
// every 128 elements of K, the tensor-core accumulator cannot run across K
// blocks: each 128-deep chunk is multiplied into a fresh fp32 partial in
// tensor memory (4 x tcgen05.mma of K = 32), and promotion warps add it,
// times the product of the two scales, into fp32 registers.
//
// Prefill kernel (any M; tuned for large M): one CTA per SM (persistent),
// output tile 128 (M) x 256 (N), tiles visited M-fastest so the CTAs
// running together share the same weight columns.  12 warps:
//   warp 0      TMA producer: A tile 128x128 and W tile 256x128 (e4m3,
//               128-byte swizzle) into a 4-deep shared-memory ring.
//   warp 1      MMA issuer: the whole warp runs the loop and waits (the
//               wait results made warp-uniform by a vote), lane 0 issues
//               4 MMAs per chunk (M=128, N=256, K=32) into one of two
//               256-column TMEM buffers, then commits to release the stage
//               and to mark the buffer full.  (A loop run by lane 0 alone,
//               with a data-dependent exit, measured ~600 cycles per
//               iteration on B200 whatever it waited for.)
//   warp 2      owns the TMEM allocation (512 columns).
//   warps 4-11  promotion: warp w reads TMEM lanes 32 (w % 4) .. +31 (its
//               rows) and column half (w - 4) / 4 (one 128-wide weight
//               block) in 16-column loads, releases the buffer as soon as
//               the last load has landed, and adds partial * s_a[row, j] *
//               s_w[nblk, j] into 128 fp32 registers with packed f32x2
//               FMAs; after the last chunk it converts to bf16 and stores.
// What bounds it (measured on B200): every 128-deep chunk leaves a 128 KB
// fp32 partial in TMEM that must be read into registers before the buffer
// can take the chunk after next.  tcgen05.ld is latency-bound (a 64-column
// load takes ~250 cycles; one warp moves at most ~36 B/cycle), so the read
// rate equals the bytes in flight / ~250 cycles, and with the 128x256 fp32
// accumulator occupying half the register file the promotion warps cannot
// keep the ~64 KB in flight that the tensor core's 512 cycles per chunk
// require.  Variants with two MMA-issuing warps, 64-column loads, 16
// promotion warps, four 128-column TMEM buffers or CTA-pair tiles all land
// at the same ~1.0-1.1 M flop per cycle (about 45% of the tensor core's
// rate); the concurrent TMEM reads, FMAs and the power limit do not slow
// the MMAs themselves.
// Every mbarrier wait is bounded in time; on expiry the kernel records an
// error code in the error word, drains what it started and exits cleanly.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"
#include "quant_math.cuh"

namespace fp8bl {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int STAGES = 4;
constexpr int UMMA_K = 32;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 384;
constexpr int NUM_EPI_WARPS = 8;
constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(BM, BN);

constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * A_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_B_OFF + STAGES * B_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;   // full, empty, tfull[2], tempty[2], drain
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC_OFF + 16 + 1024;  // + slack for 1024-byte alignment

struct GemmArgs {
  const float* s_a;
  const float* s_w;
  __nv_bfloat16* y;
  int M, N, K;
  int* err;
};

__device__ __forceinline__ void record_error(int* err, int code) {
  atomicCAS(err, 0, code);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + SMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_kb = K / BK;
  const int num_tiles = num_m * num_n;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), NUM_EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
      uint32_t c = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % num_m, n_blk = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % STAGES;
          const uint32_t ph = (c / STAGES) & 1u;
          if (!ptx::mbar_wait(empty_bar(s), ph ^ 1u)) {
            record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(full_bar(s), A_BYTES + B_BYTES);
          ptx::tma_load_2d(smem_base + SMEM_A_OFF + s * A_BYTES, &tmap_a, full_bar(s), kb * BK,
                           m_blk * BM);
          ptx::tma_load_2d(smem_base + SMEM_B_OFF + s * B_BYTES, &tmap_b, full_bar(s), kb * BK,
                           n_blk * BN);
          last_phase[s] = static_cast<int>(ph);
        }
      }
      // Every load this thread issued lands before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (last_phase[s] >= 0 && !ptx::mbar_wait(full_bar(s), static_cast<uint32_t>(last_phase[s])))
          record_error(args.err, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    {
      uint32_t c = 0;
      bool ok = true, issued = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % STAGES;
          const uint32_t sph = (c / STAGES) & 1u;
          const int buf = c & 1;
          const uint32_t bph = (c >> 1) & 1u;
          ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(tempty_bar(buf), bph ^ 1u) &&
                                           ptx::mbar_wait_spin(full_bar(s), sph));
          if (!ok) {
            if (lane == 0) record_error(args.err, kErrTimeoutMma);
            break;
          }
          ptx::tc_fence_after();
          if (lane == 0) {
            const uint32_t a_addr = smem_base + SMEM_A_OFF + s * A_BYTES;
            const uint32_t b_addr = smem_base + SMEM_B_OFF + s * B_BYTES;
            const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k) {
              ptx::mma_f8f6f4(d, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                              ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), IDESC, k > 0 ? 1u : 0u);
            }
            ptx::mma_commit(empty_bar(s));
            ptx::mma_commit(tfull_bar(buf));
          }
          __syncwarp();
          issued = true;
        }
      }
      if (issued && lane == 0) {
        // All MMAs finish before the TMEM they write is released.
        ptx::mma_commit(drain_bar);
        if (!ptx::mbar_wait(drain_bar, 0)) record_error(args.err, kErrTimeoutMma);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int nblk_count = N / 128;
    uint32_t c = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const int row = m_blk * BM + quarter * 32 + lane;
      const int nb = n_blk * 2 + half;
      const bool row_ok = row < M;
      const bool col_ok = nb < nblk_count;
      const float* sa_row = args.s_a + static_cast<int64_t>(row_ok ? row : M - 1) * num_kb;
      const float* sw_row = args.s_w + static_cast<int64_t>(col_ok ? nb : nblk_count - 1) * num_kb;
      float2 acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
      float sa1 = __ldg(sa_row), sw1 = __ldg(sw_row);
      float sa2 = num_kb > 1 ? __ldg(sa_row + 1) : 0.0f;
      float sw2 = num_kb > 1 ? __ldg(sw_row + 1) : 0.0f;
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const float scale = sa1 * sw1;
        const float2 sc2 = make_float2(scale, scale);
        sa1 = sa2; sw1 = sw2;
        if (kb + 2 < num_kb) { sa2 = __ldg(sa_row + kb + 2); sw2 = __ldg(sw_row + kb + 2); }
        const int buf = c & 1;
        const uint32_t bph = (c >> 1) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tfull_bar(buf), bph))) {
          record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem_base + lane_off + static_cast<uint32_t>(buf * BN + half * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t v[16];
          ptx::tmem_ld_32x32b_x16(tb + j * 16, v);
          ptx::tmem_ld_wait();
          if (j == 7) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[j * 8 + i] = __ffma2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])), sc2, acc[j * 8 + i]);
        }
      }
      if (!ok) break;
      if (row_ok && col_ok) {
        uint4* dst = reinterpret_cast<uint4*>(args.y + static_cast<int64_t>(row) * N + nb * 128);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          __nv_bfloat162 p0 = __float22bfloat162_rn(acc[4 * j + 0]);
          __nv_bfloat162 p1 = __float22bfloat162_rn(acc[4 * j + 1]);
          __nv_bfloat162 p2 = __float22bfloat162_rn(acc[4 * j + 2]);
          __nv_bfloat162 p3 = __float22bfloat162_rn(acc[4 * j + 3]);
          uint4 o;
          o.x = *reinterpret_cast<uint32_t*>(&p0);
          o.y = *reinterpret_cast<uint32_t*>(&p1);
          o.z = *reinterpret_cast<uint32_t*>(&p2);
          o.w = *reinterpret_cast<uint32_t*>(&p3);
          dst[j] = o;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

cudaError_t ensure_smem_attr() {
  static std::once_flag once[kMaxDevices];
  static cudaError_t st[kMaxDevices];
  return once_per_device(once, st, [](int) {
    return cudaFuncSetAttribute(gemm_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
}

}  // namespace

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a row-major byte matrix [rows, cols] with a (box_rows x
// box_cols) box and the 128-byte swizzle; out-of-range elements read zero.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                  uint32_t box_rows, uint32_t box_cols) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

GemmPlan plan_block_linear(int64_t M, int64_t N, int64_t K, int sm_count, bool fused) {
  GemmPlan p;
  p.kind = 0;
  p.split_k = 1;
  p.workspace = 0;
  if (M <= kDecodeMaxM) {
    // decode sizes: swap-AB stream-K kernel + ordered reduction
    p.kind = 1;
    p.workspace = decode_workspace_bytes(M, N, K, sm_count);
  }
  if (fused && p.kind == 0) {
    // prefill sizes: the activation tile is quantized inside the GEMM
    p.kind = 2;
  } else if (fused) {
    // decode sizes: quantize first (a few KB) into the workspace, after the
    // GEMM's own scratch, then run the decode schedule
    const int64_t qa = M * K;
    const int64_t sa = M * (K / 128) * 4;
    p.workspace = ((p.workspace + 255) / 256) * 256 +
                  static_cast<size_t>(((qa + 255) / 256) * 256 + ((sa + 255) / 256) * 256);
  }
  return p;
}

cudaError_t launch_block_linear(const void* q_a, const float* s_a, const void* q_w,
                                const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                const GemmPlan& plan, void* workspace, const DeviceInfo& dev,
                                cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (plan.kind == 1)
    return launch_block_linear_decode(q_a, s_a, q_w, s_w, y, M, N, K, workspace, dev, st);
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, q_a, M, K, BM, BK) || !make_tmap_u8(&tb, q_w, N, K, BN, BK))
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.err = dev.error_flag;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  gemm_prefill_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ta, tb, a);
  return cudaGetLastError();
}

cudaError_t launch_block_linear_fused(const void* x, const void* q_w, const float* s_w, void* y,
                                      int64_t M, int64_t N, int64_t K, const GemmPlan& plan,
                                      void* workspace, const DeviceInfo& dev, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (plan.kind == 2) return launch_block_linear_fused_tiles(x, q_w, s_w, y, M, N, K, dev, st);
  // staged: quantized activations in the workspace, after the GEMM's own scratch
  const GemmPlan gp = plan_block_linear(M, N, K, dev.sm_count, false);
  uint8_t* qa = static_cast<uint8_t*>(workspace) + ((gp.workspace + 255) / 256) * 256;
  float* sa = reinterpret_cast<float*>(qa + ((M * K + 255) / 256) * 256);
  cudaError_t e = launch_act_quant(x, M, K, qa, sa, dev.sm_count, st);
  if (e != cudaSuccess) return e;
  return launch_block_linear(qa, sa, q_w, s_w, y, M, N, K, gp, workspace, dev, st);
}

}  // namespace fp8bl
