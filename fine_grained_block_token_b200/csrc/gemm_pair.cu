// Block-scaled FP8 GEMM on CTA pairs (tcgen05.mma.cta_group::2) for sm_100a:
//   y = bf16( sum_j s_a[:,j] s_w[:,j] (A_j W_j^T) )
//
// "Fine-grained FP8" page: one scale per 128 x 128 weight block and per
// (token, 128-group) of the activations, both applied per 128-deep K block,
// so every 128-deep chunk is multiplied into a fresh fp32 partial in TMEM
// and promotion warps add partial * s_a * s_w into registers (as in the
// single-CTA kernel, gemm.cu).
//
// Two CTAs of a cluster compute one 256 (M) x 256 (N) tile: CTA r holds
// rows 128 r .. 128 r + 127 of the tile's A block and of its W block (32 KB
// per stage, six stages), the even CTA issues tcgen05.mma.cta_group::2 with
// M = 256, and each CTA's TMEM receives its own 128 rows x 256 columns.  Per
// 128 x 256 x 128 chunk of work an SM then moves 32 KB into shared memory
// and 48 KB out of it to the tensor cores, against 48 + 48 KB for a single
// CTA's 128 x 256 tile; shared-memory traffic is what bounds the single-CTA
// kernel's MMA issue.  No load is multicast: each CTA loads its own halves,
// counted in bytes on the even CTA's full barrier.
//
// Warps (both CTAs):
//   warp 0      TMA producer of this CTA's halves.
//   warp 1      MMA issuer (even CTA): per chunk 4 MMAs (M=256, N=256,
//               K=32) into one of two 256-column TMEM buffers, then commits
//               multicast to both CTAs' stage-empty and buffer-full
//               barriers.
//   warp 2      TMEM allocation for the pair; in the odd CTA it also
//               forwards "buffer read out" to the even CTA: it waits on a
//               local barrier that the odd CTA's eight promotion warps
//               arrive on and makes one remote arrival on the even CTA's
//               buffer-empty barrier per chunk.
//   warp 3      scale products s_a[row, j] * s_w[nblk, j] for this CTA's 128
//               rows and the tile's 2 weight blocks, into a shared ring.
//   warps 4-11  promotion of this CTA's 128 rows, and the bf16 epilogue
//               through staged TMA stores.
// Every wait is bounded; on expiry the kernel records an error code, drains
// what it started and exits cleanly.
#include <cstdint>
#include <cstdlib>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"

namespace fp8bl {
namespace {

constexpr int PBM = 256;                 // pair tile rows (128 per CTA)
constexpr int PBN = 256;
constexpr int BK = 128;
constexpr int STAGES = 6;
constexpr int UMMA_K = 32;
constexpr int HALF_A = 128 * BK;         // per CTA and stage
constexpr int HALF_B = 128 * BK;
constexpr int TMEM_COLS = 512;
constexpr int NUM_THREADS = 384;
constexpr int NUM_EPI_WARPS = 8;
constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(PBM, PBN);
constexpr int STAGE_ROWS = 32;           // epilogue staging: 32 rows x 64 bytes per warp
constexpr int STAGE_COLS = 32;
constexpr int STAGE_WARP_BYTES = STAGE_ROWS * STAGE_COLS * 2;
constexpr int PSLOTS = 8;                // ring of per-chunk scale products
constexpr int PSLOT_FLOATS = 256;        // 128 rows x 2 weight blocks

constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * HALF_A;
constexpr int SMEM_Y_OFF = SMEM_B_OFF + STAGES * HALF_B;
constexpr int SMEM_P_OFF = SMEM_Y_OFF + NUM_EPI_WARPS * STAGE_WARP_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_P_OFF + PSLOTS * PSLOT_FLOATS * 4;
// full, empty, tfull[2], tempty[2], tlocal[2], drain, pfull[PSLOTS], pempty[PSLOTS]
constexpr int NUM_BARS = 2 * STAGES + 6 + 1 + 2 * PSLOTS;
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC_OFF + 16 + 1024;   // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct PairArgs {
  const float* s_a;
  const float* s_w;
  int M, N, K;
  int* err;
};

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_y, const PairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + SMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 2 + b); };
  auto tlocal_bar = [&](int b) { return bar_base + 8u * (2 * STAGES + 4 + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 6);
  auto pfull_bar = [&](int i) { return bar_base + 8u * (2 * STAGES + 7 + i); };
  auto pempty_bar = [&](int i) { return bar_base + 8u * (2 * STAGES + 7 + PSLOTS + i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);
  float* prods = reinterpret_cast<float*>(smem + SMEM_P_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();     // 0 = the pair's MMA issuer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int M = args.M, N = args.N, K = args.K;
  const int num_m = (M + PBM - 1) / PBM;
  const int num_n = (N + PBN - 1) / PBN;
  const int num_kb = K / BK;
  const int num_tiles = num_m * num_n;
  const int nblk_count = N / 128;
  constexpr uint16_t kBoth = 0x3;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      // even CTA: its 8 promotion warps + one forwarded arrival from the odd CTA
      ptx::mbar_init(tempty_bar(b), NUM_EPI_WARPS + 1);
      ptx::mbar_init(tlocal_bar(b), NUM_EPI_WARPS);
    }
    ptx::mbar_init(drain_bar, 1);
    for (int i = 0; i < PSLOTS; ++i) {
      ptx::mbar_init(pfull_bar(i), 32);
      ptx::mbar_init(pempty_bar(i), NUM_EPI_WARPS);
    }
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
    ptx::prefetch_tmap(&tmap_y);
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
          const int s = c % STAGES;
          const uint32_t ph = (c / STAGES) & 1u;
          if (!ptx::mbar_wait_cluster(empty_bar(s), ph ^ 1u)) {
            record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          const uint32_t fb = ptx::map_to_cta(full_bar(s), 0);
          if (leader) ptx::mbar_arrive_expect_tx(full_bar(s), 2 * (HALF_A + HALF_B));
          ptx::tma_load_2d_pair(smem_base + SMEM_A_OFF + s * HALF_A, &tmap_a, fb, kb * BK,
                                m_blk * PBM + 128 * static_cast<int>(rank));
          ptx::tma_load_2d_pair(smem_base + SMEM_B_OFF + s * HALF_B, &tmap_b, fb, kb * BK,
                                n_blk * PBN + 128 * static_cast<int>(rank));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA (even CTA only)
    if (leader) {
      uint32_t c = 0;
      bool ok = true, issued = false;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % STAGES;
          const uint32_t sph = (c / STAGES) & 1u;
          const int buf = c & 1;
          const uint32_t bph = (c >> 1) & 1u;
          ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tempty_bar(buf), bph ^ 1u) &&
                                           ptx::mbar_wait_spin_cluster(full_bar(s), sph));
          if (!ok) {
            if (lane == 0) record_error(args.err, kErrTimeoutMma);
            break;
          }
          ptx::tc_fence_after();
          if (ptx::elect_one()) {
            const uint32_t a_addr = smem_base + SMEM_A_OFF + s * HALF_A;
            const uint32_t b_addr = smem_base + SMEM_B_OFF + s * HALF_B;
            const uint32_t d = tmem_base + static_cast<uint32_t>(buf * PBN);
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              ptx::mma_f8f6f4_pair(d, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                                   ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), IDESC, k > 0 ? 1u : 0u);
            ptx::mma_commit_pair_multicast(empty_bar(s), kBoth);
            ptx::mma_commit_pair_multicast(tfull_bar(buf), kBoth);
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
  } else if (warp == 2) {
    // ------------------- odd CTA: forward "buffer read out" to the even CTA
    if (!leader && lane == 0) {
      const uint32_t remote_empty0 = ptx::map_to_cta(tempty_bar(0), 0);
      const uint32_t remote_empty1 = ptx::map_to_cta(tempty_bar(1), 0);
      uint32_t c = 0;
      for (int tile = pair; tile < num_tiles; tile += num_pairs) {
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int buf = c & 1;
          const uint32_t bph = (c >> 1) & 1u;
          if (!ptx::mbar_wait(tlocal_bar(buf), bph)) {
            record_error(args.err, kErrTimeoutEpilogue);
            ok = false;
            break;
          }
          ptx::mbar_arrive_remote(buf ? remote_empty1 : remote_empty0);
        }
        if (!ok) break;
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------------------ scale products
    // For every chunk of every tile: prods[slot][h * 128 + r] =
    // s_a[row r of this CTA, kb] * s_w[weight block h, kb], up to PSLOTS
    // chunks ahead of the promotion warps.  Lane l covers rows l + 32 i;
    // the scales of a chunk are loaded PF chunks ahead.
    constexpr int PF = 4;
    uint32_t c = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const float* sa_r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = m_blk * PBM + 128 * static_cast<int>(rank) + lane + 32 * i;
        sa_r[i] = args.s_a + static_cast<int64_t>(row < M ? row : M - 1) * num_kb;
      }
      const float* sw_r[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int nb = n_blk * 2 + h;
        sw_r[h] = args.s_w + static_cast<int64_t>(nb < nblk_count ? nb : nblk_count - 1) * num_kb;
      }
      float pa[PF][4], pw[PF][2];
      auto load = [&](int kb, float (&a)[4], float (&w)[2]) {
        if (kb < num_kb) {
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = __ldg(sa_r[i] + kb);
#pragma unroll
          for (int h = 0; h < 2; ++h) w[h] = __ldg(sw_r[h] + kb);
        }
      };
#pragma unroll
      for (int j = 0; j < PF; ++j) load(j, pa[j], pw[j]);
      for (int kb0 = 0; kb0 < num_kb && ok; kb0 += PF) {
#pragma unroll
        for (int j = 0; j < PF; ++j) {
          const int kb = kb0 + j;
          if (kb >= num_kb) break;
          float a[4], w[2];
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] = pa[j][i];
          w[0] = pw[j][0];
          w[1] = pw[j][1];
          load(kb + PF, pa[j], pw[j]);
          const int slot = c % PSLOTS;
          const uint32_t ph = (c / PSLOTS) & 1u;
          ++c;
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(pempty_bar(slot), ph ^ 1u))) {
            if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
            ok = false;
            break;
          }
          float* pr = prods + slot * PSLOT_FLOATS;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int i = 0; i < 4; ++i) pr[h * 128 + lane + 32 * i] = a[i] * w[h];
          ptx::mbar_arrive(pfull_bar(slot));
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------ promotion (both CTAs)
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t stage = smem_base + SMEM_Y_OFF + static_cast<uint32_t>(warp - 4) * STAGE_WARP_BYTES;
    // the even CTA's warps release a buffer on its own barrier; the odd
    // CTA's on a local one that warp 2 forwards
    const uint32_t release0 = leader ? tempty_bar(0) : tlocal_bar(0);
    const uint32_t release1 = leader ? tempty_bar(1) : tlocal_bar(1);
    uint32_t c = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const int row0 = m_blk * PBM + 128 * static_cast<int>(rank) + quarter * 32;
      const int nb = n_blk * 2 + half;
      const bool box_ok = nb < nblk_count && row0 < M;
      float2 acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const int buf = c & 1;
        const uint32_t bph = (c >> 1) & 1u;
        const int slot = c % PSLOTS;
        const uint32_t pph = (c / PSLOTS) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(pfull_bar(slot), pph))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        // s_a[row, kb] * s_w[nb, kb], from the scale-product warp
        const float scale = prods[slot * PSLOT_FLOATS + half * 128 + quarter * 32 + lane];
        const float2 sc2 = make_float2(scale, scale);
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(pempty_bar(slot));
        // the buffer-full barrier is completed by the even CTA's commit
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tfull_bar(buf), bph))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem_base + lane_off + static_cast<uint32_t>(buf * PBN + half * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t v[16];
          ptx::tmem_ld_32x32b_x16(tb + j * 16, v);
          ptx::tmem_ld_wait();
          if (j == 7) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(buf ? release1 : release0);
          }
#pragma unroll
          for (int q = 0; q < 8; ++q)
            acc[j * 8 + q] = __ffma2_rn(make_float2(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1])), sc2, acc[j * 8 + q]);
        }
      }
      if (!ok) break;
      // bf16 out through shared memory: in four passes of 32 columns the
      // warp writes its 32 rows x 64 bytes (row r at r * 64) and one TMA
      // store moves the box to Y (rows past M and columns past N are not
      // written).
#pragma unroll
      for (int pass = 0; pass < 128 / STAGE_COLS; ++pass) {
        if (lane == 0) ptx::bulk_wait_group_read<0>();   // the staging box is free again
        __syncwarp();
#pragma unroll
        for (int j = 0; j < STAGE_COLS / 8; ++j) {
          const int a0 = pass * (STAGE_COLS / 2) + j * 4;
          __nv_bfloat162 p0 = __float22bfloat162_rn(acc[a0 + 0]);
          __nv_bfloat162 p1 = __float22bfloat162_rn(acc[a0 + 1]);
          __nv_bfloat162 p2 = __float22bfloat162_rn(acc[a0 + 2]);
          __nv_bfloat162 p3 = __float22bfloat162_rn(acc[a0 + 3]);
          const uint32_t addr = stage + static_cast<uint32_t>(lane * STAGE_COLS * 2 + j * 16);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                       "r"(*reinterpret_cast<uint32_t*>(&p0)), "r"(*reinterpret_cast<uint32_t*>(&p1)),
                       "r"(*reinterpret_cast<uint32_t*>(&p2)), "r"(*reinterpret_cast<uint32_t*>(&p3))
                       : "memory");
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && box_ok) {
          ptx::tma_store_2d(&tmap_y, stage, (nb * 128 + pass * STAGE_COLS) * 2, row0);
          ptx::bulk_commit_group();
        }
      }
    }
    // every store has left shared memory before the CTA exits
    if (lane == 0) ptx::bulk_wait_group<0>();
    __syncwarp();
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
    cudaError_t st = cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          SMEM_BYTES);
    if (st != cudaSuccess) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int clusters = 0;
    st = cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel, &cfg);
    if (st == cudaSuccess && clusters < 1) st = cudaErrorInvalidConfiguration;
    clusters_of[d] = clusters;
    return st;
  }, &dev);
  *max_clusters = r == cudaSuccess ? clusters_of[dev] : 0;
  return r;
}

}  // namespace

// The pair kernel is opt-in (FP8BL_BLOCK_PAIRS=1 in the environment) for M
// above one 128-row tile.  Measured on B200 it runs at 1.0-1.3 PFLOP/s
// against 1.8-1.95 for the single-CTA kernel: with two 256-column TMEM
// buffers per CTA, the MMA of chunk c + 2 waits until both CTAs have read
// out chunk c, and the odd CTA's "read out" signal has to cross to the
// even CTA's SM every chunk (through a forwarding thread: 1.18-1.28
// PFLOP/s; each warp arriving remotely: 0.77-0.98), which one chunk of MMA
// work cannot cover.
bool block_linear_use_pairs(int64_t M) {
  static const bool enabled = [] {
    const char* v = std::getenv("FP8BL_BLOCK_PAIRS");
    return v != nullptr && v[0] == '1';
  }();
  return enabled && M > 128;
}

cudaError_t launch_block_linear_pairs(const void* q_a, const float* s_a, const void* q_w,
                                      const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                      const DeviceInfo& dev, cudaStream_t st) {
  int max_clusters = 0;
  cudaError_t e = ensure_pair_ready(&max_clusters);
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb, ty;
  if (!make_tmap_u8(&ta, q_a, M, K, 128, BK) || !make_tmap_u8(&tb, q_w, N, K, 128, BK) ||
      !make_tmap_u8(&ty, y, M, 2 * N, STAGE_ROWS, STAGE_COLS * 2, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  PairArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.err = dev.error_flag;
  const int64_t tiles = ((M + PBM - 1) / PBM) * ((N + PBN - 1) / PBN);
  const int pairs = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel, ta, tb, ty, a);
}

}  // namespace fp8bl
