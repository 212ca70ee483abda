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
// running together share the same weight columns (above 32 row blocks in
// groups of 16 row blocks, so that a wave's rows of A stay in L2).  12 warps:
//   warp 0      TMA producer: A tile 128x128 and W tile 256x128 (e4m3,
//               128-byte swizzle) into a 4-deep shared-memory ring.
//   warp 1      MMA issuer: the whole warp runs the loop and waits (the
//               wait results made warp-uniform by a vote), an elected lane issues
//               4 MMAs per chunk (M=128, N=256, K=32) into one of two
//               256-column TMEM buffers, then commits to release the stage
//               and to mark the buffer full.  (A loop run by lane 0 alone,
//               with a data-dependent exit, measured ~600 cycles per
//               iteration on B200 whatever it waited for.)
//   warp 2      owns the TMEM allocation (512 columns).
//   warp 3      scale products: for every chunk the 256 factors
//               s_a[row, j] * s_w[nblk, j] of the tile (128 rows x 2 weight
//               blocks) into a shared ring, up to 8 chunks ahead.
//   warps 4-11  promotion: warp w reads TMEM lanes 32 (w % 4) .. +31 (its
//               rows) and column half (w - 4) / 4 (one 128-wide weight
//               block) in 16-column loads, releases the buffer as soon as
//               the last load has landed, and adds partial * factor into
//               128 fp32 registers with packed f32x2 FMAs; after a tile's
//               last chunk it writes bf16 through a shared staging box and
//               TMA stores (coalesced; rows past M, columns past N clipped).
// Where the time goes (cycle counters in the warps, B200): per 128 x 256 x
// 128 chunk the MMA warp spends ~750 cycles issuing into a busy tensor pipe
// (each chunk moves 48 KB into shared memory by TMA and 48 KB out of it
// into the tensor core, which is about what shared memory delivers in that
// time) and ~150-200 waiting for a free TMEM buffer, ~65 for operands.  The
// read-out of a partial takes ~320 cycles of TMEM loads plus ~275 of the
// FMAs interleaved with them.  Moving the scale loads to warp 3 (they
// stalled the promotion ~110 cycles per chunk) and the bf16 stores to TMA
// (the row-per-thread stores cost ~7,400 cycles per tile) took the chunk
// from ~1,050-1,200 to ~940-1,010 cycles.
// Tail wave: with T tiles on G CTAs, q = T / G full waves leave r = T % G
// tiles; when 2 r <= G each of those is split into two 128 x 128 items
// (MMA N = 128, a 128-row W box, promotion warps 64 columns each) run by
// two CTAs, so the last wave takes about two thirds of a full tile's time
// instead of a whole one.  Every output element is still accumulated in the
// same K order with the same products, so results are bit for bit those of
// the full tiles.  With T <= G / 2 every tile is split.
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
constexpr uint32_t IDESC_HALF = ptx::idesc_e4m3_f32(BM, BN / 2);   // split tail items

constexpr int STAGE_ROWS = 32;     // epilogue staging: 32 rows x 64 bytes per warp
constexpr int STAGE_COLS = 32;     // bf16 columns per staging pass
constexpr int STAGE_WARP_BYTES = STAGE_ROWS * STAGE_COLS * 2;
constexpr int PSLOTS = 8;          // ring of per-chunk scale products
constexpr int PSLOT_FLOATS = 256;  // 128 rows x 2 weight blocks

constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * A_BYTES;
constexpr int SMEM_Y_OFF = SMEM_B_OFF + STAGES * B_BYTES;
constexpr int SMEM_P_OFF = SMEM_Y_OFF + NUM_EPI_WARPS * STAGE_WARP_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_P_OFF + PSLOTS * PSLOT_FLOATS * 4;
// full, empty, tfull[2], tempty[2], drain, pfull[PSLOTS], pempty[PSLOTS]
constexpr int NUM_BARS = 2 * STAGES + 4 + 1 + 2 * PSLOTS;
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC_OFF + 16 + 1024;  // + slack for 1024-byte alignment
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct GemmArgs {
  const float* s_a;
  const float* s_w;
  __nv_bfloat16* y;
  int M, N, K;
  int group_m;   // tile order: groups of group_m row blocks, M-fastest inside (0: no groups)
  int* err;
};

__device__ __forceinline__ void record_error(int* err, int code) {
  atomicCAS(err, 0, code);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_prefill_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_b_half,
                    const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
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
  auto pfull_bar = [&](int i) { return bar_base + 8u * (2 * STAGES + 5 + i); };
  auto pempty_bar = [&](int i) { return bar_base + 8u * (2 * STAGES + 5 + PSLOTS + i); };
  float* prods = reinterpret_cast<float*>(smem + SMEM_P_OFF);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_kb = K / BK;
  const int num_tiles = num_m * num_n;
  // work items: full tiles, then (split tail) two 128-column halves per
  // remaining tile
  const int G = gridDim.x;
  const int q_waves = num_tiles / G, r_tail = num_tiles % G;
  const bool split = r_tail > 0 && 2 * r_tail <= G;
  const int num_items = split ? q_waves * G + 2 * r_tail : num_tiles;
  // item -> (M block, first column, full 256-column tile?)
  auto map_item = [&](int item, int& m_blk, int& col0, bool& full) {
    int tile = item, sub = 0;
    full = true;
    if (split && item >= q_waves * G) {
      const int h = item - q_waves * G;
      tile = q_waves * G + (h >> 1);
      sub = h & 1;
      full = false;
    }
    // tiles in groups of group_m row blocks (M-fastest inside a group, the
    // groups one after another), so that a wave's rows of A stay in L2
    // while W streams past them
    const int gm = args.group_m > 0 && args.group_m < num_m ? args.group_m : num_m;
    const int group = tile / (gm * num_n);
    const int first_m = group * gm;
    const int rows_here = num_m - first_m < gm ? num_m - first_m : gm;
    const int local = tile - group * gm * num_n;
    m_blk = first_m + local % rows_here;
    col0 = (local / rows_here) * BN + sub * (BN / 2);
  };

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
    for (int i = 0; i < PSLOTS; ++i) {
      ptx::mbar_init(pfull_bar(i), 32);
      ptx::mbar_init(pempty_bar(i), NUM_EPI_WARPS);
    }
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
    ptx::prefetch_tmap(&tmap_b_half);
    ptx::prefetch_tmap(&tmap_y);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  // Launched with programmatic stream serialization: the set-up above may
  // overlap the previous kernel's tail; from here on the kernel reads what
  // that kernel may have written (the quantized activations) and writes Y.
  ptx::grid_dep_wait();
  if (threadIdx.x == 0) ptx::grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
      uint32_t c = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x) {
        int m_blk, col0;
        bool full;
        map_item(item, m_blk, col0, full);
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % STAGES;
          const uint32_t ph = (c / STAGES) & 1u;
          if (!ptx::mbar_wait(empty_bar(s), ph ^ 1u)) {
            record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(full_bar(s), A_BYTES + (full ? B_BYTES : B_BYTES / 2));
          ptx::tma_load_2d(smem_base + SMEM_A_OFF + s * A_BYTES, &tmap_a, full_bar(s), kb * BK,
                           m_blk * BM);
          ptx::tma_load_2d(smem_base + SMEM_B_OFF + s * B_BYTES, full ? &tmap_b : &tmap_b_half,
                           full_bar(s), kb * BK, col0);
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
      const uint64_t desc_a = ptx::sdesc_kmajor_sw128(smem_base + SMEM_A_OFF);
      const uint64_t desc_b = ptx::sdesc_kmajor_sw128(smem_base + SMEM_B_OFF);
      uint32_t c = 0;
      bool ok = true, issued = false;
      for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x) {
        int m_blk, col0;
        bool full;
        map_item(item, m_blk, col0, full);
        const uint32_t idesc = full ? IDESC : IDESC_HALF;
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
          const uint64_t da = ptx::sdesc_advance(desc_a, s * A_BYTES);
          const uint64_t db = ptx::sdesc_advance(desc_b, s * B_BYTES);
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
          if (ptx::elect_one()) {
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              ptx::mma_f8f6f4(d, ptx::sdesc_advance(da, k * UMMA_K), ptx::sdesc_advance(db, k * UMMA_K),
                              idesc, k > 0 ? 1u : 0u);
            ptx::mma_commit(empty_bar(s));
            ptx::mma_commit(tfull_bar(buf));
          }
          issued = true;
        }
      }
      if (issued && ptx::elect_one()) {
        // All MMAs finish before the TMEM they write is released.
        ptx::mma_commit(drain_bar);
        if (!ptx::mbar_wait(drain_bar, 0)) record_error(args.err, kErrTimeoutMma);
      }
      __syncwarp();
    }
  } else if (warp == 3) {
    // ------------------------------------------------------ scale products
    // For every chunk of every tile: prods[slot][h * 128 + r] =
    // s_a[row r, kb] * s_w[weight block h, kb], up to PSLOTS chunks ahead
    // of the promotion warps.  Lane l covers rows l + 32 i, i = 0..3; the
    // scales of a chunk are loaded PF chunks ahead into a register slot that
    // is refilled right after its use.
    const int nblk_count = N / 128;
    constexpr int PF = 4;
    uint32_t c = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x) {
      int m_blk, col0;
      bool full;
      map_item(item, m_blk, col0, full);
      const float* sa_r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = m_blk * BM + lane + 32 * i;
        sa_r[i] = args.s_a + static_cast<int64_t>(row < M ? row : M - 1) * num_kb;
      }
      const float* sw_r[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // a full tile's two weight blocks; a split item's one, for both halves
        const int nb = col0 / 128 + (full ? h : 0);
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
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int nblk_count = N / 128;
    const uint32_t stage = smem_base + SMEM_Y_OFF + static_cast<uint32_t>(warp - 4) * STAGE_WARP_BYTES;
    uint32_t c = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < num_items && ok; item += gridDim.x) {
      int m_blk, col0;
      bool full;
      map_item(item, m_blk, col0, full);
      const int row0 = m_blk * BM + quarter * 32;   // this warp's first row
      // this warp's columns: 128 of a full tile, 64 of a split item
      const int ncol = full ? 128 : 64;
      const int wcol0 = col0 + half * ncol;
      const int nj = ncol / 16;                     // 16-column TMEM loads per chunk
      const bool box_ok = wcol0 < nblk_count * 128 && row0 < M;
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
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tfull_bar(buf), bph))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem_base + lane_off + static_cast<uint32_t>(buf * BN + half * ncol);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < nj) {
            uint32_t v[16];
            ptx::tmem_ld_32x32b_x16(tb + j * 16, v);
            ptx::tmem_ld_wait();
            if (j == nj - 1) {
              ptx::tc_fence_before();
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
              acc[j * 8 + q] = __ffma2_rn(make_float2(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1])), sc2, acc[j * 8 + q]);
          }
        }
      }
      if (!ok) break;
      // bf16 out through shared memory: in four passes of 32 columns the
      // warp writes its 32 rows x 64 bytes (row r at r * 64) and one TMA
      // store moves the box to Y (rows past M and columns past N are not
      // written).
#pragma unroll
      for (int pass = 0; pass < 128 / STAGE_COLS; ++pass) {
        if (pass * STAGE_COLS >= ncol) break;
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
          ptx::tma_store_2d(&tmap_y, stage, (wcol0 + pass * STAGE_COLS) * 2, row0);
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
                  uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swizzle) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
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
  if (fused) {
    // Quantize first into the workspace (after the GEMM's own scratch),
    // then run the GEMM on the codes, which stay in L2: measured on B200
    // this is faster at every size than quantizing inside the GEMM's tiles
    // (0.75x at the Llama-3-8B MLP, 0.82-0.97x on the 7168-deep sweep),
    // because the prefill GEMM is bound by shared-memory operand traffic
    // and the per-chunk promotion, which the in-tile quantization adds to.
    // At prefill sizes a call with less workspace than that runs the in-GEMM
    // quantization kernel instead (kind 2), which needs none.
    p.in_kernel_ok = p.kind == 0;
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
  if (block_linear_use_pairs(M))
    return launch_block_linear_pairs(q_a, s_a, q_w, s_w, y, M, N, K, dev, st);
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb, tb2, ty;
  if (!make_tmap_u8(&ta, q_a, M, K, BM, BK) || !make_tmap_u8(&tb, q_w, N, K, BN, BK) ||
      !make_tmap_u8(&tb2, q_w, N, K, BN / 2, BK) ||
      !make_tmap_u8(&ty, y, M, 2 * N, STAGE_ROWS, STAGE_COLS * 2, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  // Above 32 row blocks, tiles go in groups of 16 row blocks: measured on
  // B200 the DeepSeek-V3 MLP GEMMs (64 row blocks) went from 0.573 to 0.593
  // of the fp8 peak, the Llama-3-8B MLP (32) is slightly faster without.
  a.group_m = (M + BM - 1) / BM > 32 ? 16 : 0;
  a.err = dev.error_flag;
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  // one CTA per SM; with at most half as many tiles as SMs, two CTAs per
  // tile (every tile split into two 128-column items)
  int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  if (2 * tiles <= dev.sm_count) grid = static_cast<int>(2 * tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  set_programmatic_serialization(at[0]);
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_prefill_kernel, ta, tb, tb2, ty, a);
}

cudaError_t launch_block_linear_fused(const void* x, const void* q_w, const float* s_w, void* y,
                                      int64_t M, int64_t N, int64_t K, const GemmPlan& plan,
                                      void* workspace, const DeviceInfo& dev, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (plan.kind == 2) return launch_block_linear_fused_tiles(x, q_w, s_w, y, M, N, K, dev, st);
  // staged (plan.kind 0 or 1): quantized activations in the workspace, after
  // the GEMM's own scratch
  const GemmPlan gp = plan_block_linear(M, N, K, dev.sm_count, false);
  uint8_t* qa = static_cast<uint8_t*>(workspace) + ((gp.workspace + 255) / 256) * 256;
  float* sa = reinterpret_cast<float*>(qa + ((M * K + 255) / 256) * 256);
  cudaError_t e = launch_act_quant(x, M, K, qa, sa, dev.sm_count, st);
  if (e != cudaSuccess) return e;
  return launch_block_linear(qa, sa, q_w, s_w, y, M, N, K, gp, workspace, dev, st);
}

}  // namespace fp8bl
