// Row-wise scaled FP8 linear for sm_100a:
//   y[m,n] = bf16( s_a[m] * s_w[n] * sum_k e4m3(q_a[m,k]) e4m3(q_w[n,k]) )
//
// "BFL (fp8r / nvfp4)" page, first bullet of its list and its "Kernels"
// table: an E4M3 weight with one fp32 scale per output row, activations
// quantized per token row, multiplied as a scaled matmul with row-wise
// scales.  With one scale per row and column the scales factor out of the
// K sum, so the tensor core accumulates the whole K extent in fp32 in TMEM
// and the epilogue applies s_a[m] * s_w[n] once.
//
// One CTA per SM (persistent), output tile 128 (M) x 256 (N), tiles visited
// M-fastest.  12 warps:
//   warp 0      TMA producer: A 128x128 and W 256x128 e4m3 tiles (128-byte
//               swizzle; the tail of K past the matrix reads as zero) into a
//               4-deep shared-memory ring.
//   warp 1      MMA issuer (whole warp loops and waits, an elected lane issues): 4
//               MMAs (M=128, N=256, K=32) per stage into the tile's
//               accumulator, one of two 256-column TMEM buffers (tile t uses
//               buffer t % 2, so a tile's epilogue overlaps the next tile's
//               MMAs).
//   warp 2      owns the TMEM allocation (512 columns).
//   warps 4-11  epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 and
//               columns 128 ((w - 4) / 4) .. +127 with two 64-column loads,
//               releases the buffer, multiplies by s_a[row] * s_w[col] and
//               stores bf16.
// Every mbarrier wait is bounded in time; on expiry the kernel records an
// error code in the error word, drains what it started and exits cleanly.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdlib>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"

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
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct LinearArgs {
  const float* s_a;   // [M]
  const float* s_w;   // [N]
  __nv_bfloat16* y;
  int M, N, K;
  int* err;
};

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }

// CTA pairs for M above one 128-row tile (below it the odd CTA would only
// compute padding); FP8BL_ROWWISE_PAIRS=0 in the environment selects the
// single-CTA kernel at every size.
bool rowwise_use_pairs(int64_t M) {
  static const bool enabled = [] {
    const char* v = std::getenv("FP8BL_ROWWISE_PAIRS");
    return v == nullptr || v[0] != '0';
  }();
  return enabled && M > 128;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_rowwise_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b, const LinearArgs args) {
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
  const int num_kb = (K + BK - 1) / BK;
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
    uint32_t c = 0, t_local = 0;
    bool ok = true, issued = false;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t_local) {
      const int buf = t_local & 1;
      const uint32_t bph = (t_local >> 1) & 1u;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(tempty_bar(buf), bph ^ 1u));
      if (!ok) {
        if (lane == 0) record_error(args.err, kErrTimeoutMma);
        break;
      }
      const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const int s = c % STAGES;
        const uint32_t sph = (c / STAGES) & 1u;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(full_bar(s), sph));
        if (!ok) {
          if (lane == 0) record_error(args.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t a_addr = smem_base + SMEM_A_OFF + s * A_BYTES;
          const uint32_t b_addr = smem_base + SMEM_B_OFF + s * B_BYTES;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            ptx::mma_f8f6f4(d, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                            ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), IDESC,
                            (kb | k) != 0 ? 1u : 0u);
          ptx::mma_commit(empty_bar(s));
          if (kb == num_kb - 1) ptx::mma_commit(tfull_bar(buf));
        }
        __syncwarp();
        issued = true;
      }
    }
    if (issued && ptx::elect_one()) {
      // All MMAs finish before the TMEM they write is released.
      ptx::mma_commit(drain_bar);
      if (!ptx::mbar_wait(drain_bar, 0)) record_error(args.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t t_local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t_local) {
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const int row = m_blk * BM + quarter * 32 + lane;
      const int col0 = n_blk * BN + half * 128;
      const int buf = t_local & 1;
      const uint32_t bph = (t_local >> 1) & 1u;
      const float sa = row < M ? __ldg(args.s_a + row) : 0.0f;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tfull_bar(buf), bph))) {
        if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
        break;
      }
      ptx::tc_fence_after();
      uint32_t v0[64], v1[64];
      const uint32_t tb = tmem_base + lane_off + static_cast<uint32_t>(buf * BN + half * 128);
      ptx::tmem_ld_32x32b_x64(tb, v0);
      ptx::tmem_ld_32x32b_x64(tb + 64, v1);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
      if (row < M) {
        __nv_bfloat16* yrow = args.y + static_cast<int64_t>(row) * N;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = col0 + 8 * j;
          if (col < N) {     // N % 16 == 0: an 8-column chunk is all in or all out
            const uint32_t* src = j < 8 ? v0 + 8 * j : v1 + 8 * (j - 8);
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(args.s_w + col));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(args.s_w + col + 4));
            const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = __uint_as_float(src[2 * i]) * (sa * sw[2 * i]);
              const float hi = __uint_as_float(src[2 * i + 1]) * (sa * sw[2 * i + 1]);
              __nv_bfloat162 p = __float22bfloat162_rn(make_float2(lo, hi));
              o[i] = *reinterpret_cast<uint32_t*>(&p);
            }
            *reinterpret_cast<uint4*>(yrow + col) = make_uint4(o[0], o[1], o[2], o[3]);
          }
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

// ------------------------------------------------------------ CTA pairs
//
// Same linear on CTA pairs (clusters of 2): a pair computes a 256 x 256
// tile with tcgen05.mma.cta_group::2 (M = 256).  Each CTA loads its own 128
// rows of A and 128 rows of W per stage (32 KB), so six stages fit and the
// tensor core has five stages of work queued while a stage reloads (the
// single-CTA kernel's four 48 KB stages leave about two and a half).  The
// even CTA (rank 0) issues the MMAs and owns the stage and accumulator
// barriers: both CTAs' TMA loads count their bytes on its full barriers,
// its commits are multicast to the empty / accumulator-full barriers of
// both, and both CTAs' epilogue warps arrive on its accumulator-empty
// barriers (the odd CTA's remotely, release / acquire at cluster scope).
// Accumulator rows 0..127 live in the even CTA's TMEM, 128..255 in the
// odd one's, two 256-column buffers each.
constexpr int PBM = 256;                 // pair tile rows (128 per CTA)
constexpr int PBN = 256;
constexpr int PSTAGES = 6;
constexpr int PA_BYTES = 128 * BK;       // per CTA and stage
constexpr int PB_BYTES = 128 * BK;
constexpr uint32_t PIDESC = ptx::idesc_e4m3_f32(PBM, PBN);
constexpr int PSMEM_A_OFF = 0;
constexpr int PSMEM_B_OFF = PSMEM_A_OFF + PSTAGES * PA_BYTES;
constexpr int PSMEM_BAR_OFF = PSMEM_B_OFF + PSTAGES * PB_BYTES;
constexpr int PNUM_BARS = 2 * PSTAGES + 4 + 1;   // full, empty, tfull[2], tempty[2], drain
constexpr int PSMEM_MISC_OFF = PSMEM_BAR_OFF + PNUM_BARS * 8;
constexpr int PSMEM_BYTES = PSMEM_MISC_OFF + 16 + 1024;
static_assert(PSMEM_BYTES <= 227 * 1024, "shared memory budget");

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_rowwise_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b, const LinearArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + PSMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (PSTAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * PSTAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * PSTAGES + 2 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * PSTAGES + 4);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + PSMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();     // 0 = the pair's MMA issuer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int M = args.M, N = args.N, K = args.K;
  const int num_m = (M + PBM - 1) / PBM;
  const int num_n = (N + PBN - 1) / PBN;
  const int num_kb = (K + BK - 1) / BK;
  const int num_tiles = num_m * num_n;
  constexpr uint16_t kBoth = 0x3;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 2 * NUM_EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
  }
  if (warp == 2) {
    ptx::tmem_alloc_pair(ptx::smem_u32(tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // both CTAs' barriers initialised before any cross-CTA use
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  const bool has_tiles = pair < num_tiles;

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      uint32_t c = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        const int m_blk = tile % num_m, n_blk = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % PSTAGES;
          const uint32_t ph = (c / PSTAGES) & 1u;
          if (!ptx::mbar_wait_cluster(empty_bar(s), ph ^ 1u)) {
            record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          const uint32_t fb = ptx::map_to_cta(full_bar(s), 0);
          if (leader) ptx::mbar_arrive_expect_tx(full_bar(s), 2 * (PA_BYTES + PB_BYTES));
          ptx::tma_load_2d_pair(smem_base + PSMEM_A_OFF + s * PA_BYTES, &tmap_a, fb, kb * BK,
                                m_blk * PBM + 128 * static_cast<int>(rank));
          ptx::tma_load_2d_pair(smem_base + PSMEM_B_OFF + s * PB_BYTES, &tmap_b, fb, kb * BK,
                                n_blk * PBN + 128 * static_cast<int>(rank));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA (even CTA only)
    if (leader) {
      uint32_t c = 0, t_local = 0;
      bool ok = true, issued = false;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++t_local) {
        const int buf = t_local & 1;
        const uint32_t bph = (t_local >> 1) & 1u;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tempty_bar(buf), bph ^ 1u));
        if (!ok) {
          if (lane == 0) record_error(args.err, kErrTimeoutMma);
          break;
        }
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * PBN);
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % PSTAGES;
          const uint32_t sph = (c / PSTAGES) & 1u;
          ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(full_bar(s), sph));
          if (!ok) {
            if (lane == 0) record_error(args.err, kErrTimeoutMma);
            break;
          }
          ptx::tc_fence_after();
          if (ptx::elect_one()) {
            const uint32_t a_addr = smem_base + PSMEM_A_OFF + s * PA_BYTES;
            const uint32_t b_addr = smem_base + PSMEM_B_OFF + s * PB_BYTES;
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              ptx::mma_f8f6f4_pair(d, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                                   ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), PIDESC,
                                   (kb | k) != 0 ? 1u : 0u);
            ptx::mma_commit_pair_multicast(empty_bar(s), kBoth);
            if (kb == num_kb - 1) ptx::mma_commit_pair_multicast(tfull_bar(buf), kBoth);
          }
          __syncwarp();
          issued = true;
        }
      }
      if (issued && ptx::elect_one()) ptx::mma_commit_pair_multicast(drain_bar, kBoth);
      __syncwarp();
    }
    // both CTAs: every MMA into this CTA's TMEM and shared memory is done
    // before the CTA moves on to release them
    if (has_tiles && lane == 0 && !ptx::mbar_wait_cluster(drain_bar, 0))
      record_error(args.err, kErrTimeoutMma);
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t t_local = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++t_local) {
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const int row = m_blk * PBM + 128 * static_cast<int>(rank) + quarter * 32 + lane;
      const int col0 = n_blk * PBN + half * 128;
      const int buf = t_local & 1;
      const uint32_t bph = (t_local >> 1) & 1u;
      const float sa = row < M ? __ldg(args.s_a + row) : 0.0f;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tfull_bar(buf), bph))) {
        if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
        break;
      }
      ptx::tc_fence_after();
      uint32_t v0[64], v1[64];
      const uint32_t tb = tmem_base + lane_off + static_cast<uint32_t>(buf * PBN + half * 128);
      ptx::tmem_ld_32x32b_x64(tb, v0);
      ptx::tmem_ld_32x32b_x64(tb + 64, v1);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) ptx::mbar_arrive(tempty_bar(buf));
        else ptx::mbar_arrive_remote(ptx::map_to_cta(tempty_bar(buf), 0));
      }
      if (row < M) {
        __nv_bfloat16* yrow = args.y + static_cast<int64_t>(row) * N;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = col0 + 8 * j;
          if (col < N) {
            const uint32_t* src = j < 8 ? v0 + 8 * j : v1 + 8 * (j - 8);
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(args.s_w + col));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(args.s_w + col + 4));
            const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float lo = __uint_as_float(src[2 * i]) * (sa * sw[2 * i]);
              const float hi = __uint_as_float(src[2 * i + 1]) * (sa * sw[2 * i + 1]);
              __nv_bfloat162 p = __float22bfloat162_rn(make_float2(lo, hi));
              o[i] = *reinterpret_cast<uint32_t*>(&p);
            }
            *reinterpret_cast<uint4*>(yrow + col) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();   // neither CTA releases TMEM or exits while its peer still uses it
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

cudaError_t ensure_pair_ready(int* max_clusters) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  static int clusters_of[kMaxDevices];
  int dev = 0;
  const cudaError_t r = once_per_device(once, status, [](int d) {
    int& clusters = clusters_of[d];
    cudaError_t st = cudaFuncSetAttribute(gemm_rowwise_pair_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, PSMEM_BYTES);
    if (st != cudaSuccess) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = PSMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    st = cudaOccupancyMaxActiveClusters(&clusters, gemm_rowwise_pair_kernel, &cfg);
    if (st == cudaSuccess && clusters < 1) st = cudaErrorInvalidConfiguration;
    return st;
  }, &dev);
  *max_clusters = r == cudaSuccess ? clusters_of[dev] : 0;
  return r;
}

cudaError_t ensure_smem_attr() {
  static std::once_flag once[kMaxDevices];
  static cudaError_t st[kMaxDevices];
  return once_per_device(once, st, [](int) {
    return cudaFuncSetAttribute(gemm_rowwise_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
}

}  // namespace

cudaError_t launch_linear_rowwise_pairs(const void* q_a, const float* s_a, const void* q_w,
                                        const float* s_w, void* y, int64_t M, int64_t N,
                                        int64_t K, const DeviceInfo& dev, cudaStream_t st) {
  int max_clusters = 0;
  cudaError_t e = ensure_pair_ready(&max_clusters);
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, q_a, M, K, 128, BK) || !make_tmap_u8(&tb, q_w, N, K, 128, BK))
    return cudaErrorInvalidValue;
  LinearArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.err = dev.error_flag;
  const int64_t tiles = ((M + PBM - 1) / PBM) * ((N + PBN - 1) / PBN);
  const int pairs = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = PSMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_rowwise_pair_kernel, ta, tb, a);
}

cudaError_t launch_linear_rowwise(const void* q_a, const float* s_a, const void* q_w,
                                  const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                  const DeviceInfo& dev, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (rowwise_use_pairs(M))
    return launch_linear_rowwise_pairs(q_a, s_a, q_w, s_w, y, M, N, K, dev, st);
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, q_a, M, K, BM, BK) || !make_tmap_u8(&tb, q_w, N, K, BN, BK))
    return cudaErrorInvalidValue;
  LinearArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.err = dev.error_flag;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  gemm_rowwise_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ta, tb, a);
  return cudaGetLastError();
}

}  // namespace fp8bl
