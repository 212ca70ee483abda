// Block-scaled FP8 GEMM with UE8M0 (power-of-two) scales on the hardware
// block-scaled MMA of sm_100a:
//   y = bf16( sum_j 2^(ea[m,j]-127) 2^(ew[n/128,j]-127) (A_j W_j^T) )
//
// "Fine-grained FP8" page, "UE8M0 scale format" section: checkpoints in the
// DeepSeek-V4 style keep their FP8 scales as float8_e8m0fnu, and that is
// the only scale format the Blackwell DeepGEMM expert kernels accept.  The
// reason is this instruction: tcgen05.mma kind::mxf8f6f4.block_scale
// multiplies every 32-deep K slice of A and B by a per-row ue8m0 scale
// factor read from tensor memory, inside the tensor core.  The per-128-K
// scales of the fine-grained scheme become four equal per-32-K factors, so
// the accumulator runs across the whole K extent in TMEM and no promotion
// by CUDA cores is needed (the fp32-scale kernel spends its time there).
//
// One CTA per SM (persistent), output tile 128 (M) x 256 (N), tiles visited
// M-fastest.  12 warps:
//   warp 0      TMA producer: A 128x128 and W 256x128 e4m3 tiles (128-byte
//               swizzle) into a 4-deep shared-memory ring.
//   warp 1      MMA issuer (whole warp loops and waits, an elected lane issues): 4
//               block-scaled MMAs per 128-deep stage (M=128, N=256, K=32,
//               scale-factor id = 32-K slice) into TMEM columns 0..255,
//               reading the stage's scale factors from its own 16 TMEM
//               columns (256 + 16 s ...).
//   warp 2      owns the TMEM allocation (512 columns).
//   warps 4-7   scale-factor writers, then epilogue: warp 4 + q writes lane
//               quarter q of the stage's scale-factor columns with one
//               tcgen05.st -- the tensor core's layout: per lane l, column j
//               (0..3) holds activation row 32 j + l's scale replicated 4x
//               (one byte per 32-K slice), columns 4..7 and 8..11 the two
//               weight blocks' scales -- and arrives on the stage's full
//               barrier.  They stay up to 4 stages ahead of the MMAs; at a
//               tile's end they first fill the next tile's first 4 stages.
//               (Writing from registers keeps the copies off the tensor
//               pipe: three tcgen05.cp per stage cost ~180 cycles of it.)
//   warps 4-11  epilogue: after the tile's last MMA, warp w reads TMEM lanes
//               32 (w % 4) .. +31 and columns 128 ((w - 4) / 4) .. +127 with
//               two 64-column loads, releases the accumulator, and converts
//               to bf16 and stores through a shared staging box, 32 columns
//               at a time, so that each store instruction of the warp writes
//               eight 64-byte row segments instead of 32 scattered 16-byte
//               pieces (rows past the segment end are skipped).
// A single 256-column accumulator is what fits next to the scale-factor
// columns, so the MMAs of the next tile wait for the epilogue's TMEM reads
// (not for its stores).
//
// Grouped (MoE expert) form, same kernel: the rows of A are split into E
// contiguous segments [off[e], off[e+1]) and segment e is multiplied by
// expert e's weights W[e] ([E, N, K] stacked, scales [E, N/128, K/128]).
// Warp 3 turns the offsets into a shared-memory table at start-up (clamped
// to [0, M] and made non-decreasing, so any offsets stay in bounds) with
// each expert's count of 128-row blocks; tiles run expert by expert (each
// expert's blocks times the N tiles, M-fastest), and a tile's rows past its
// segment, like its columns past N, are computed on whatever TMA loads but
// never stored.
// The plain linear is the case E = 1, off = {0, M}.
// Every mbarrier wait is bounded in time; on expiry the kernel records an
// error code in the error word, drains what it started and exits cleanly.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
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
constexpr uint32_t ACC_COL = 0;
constexpr uint32_t SF_COL0 = 256;         // stage s: columns SF_COL0 + 16 s .. + 15
constexpr uint32_t SFA_COL = 0;           // offsets within a stage's columns
constexpr uint32_t SFB_COL = 4;
constexpr int NUM_THREADS = 384;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_SF_WARPS = 4;           // warps 4..7, one per TMEM lane quarter
constexpr uint32_t IDESC = ptx::idesc_mxf8_e4m3_ue8m0(BM, BN);
constexpr uint32_t kUnitScale = 127;      // ue8m0 code of 1.0, for rows past M or N

constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * A_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_B_OFF + STAGES * B_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 3;  // full, empty, tfull, tempty, drain
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_TAB_OFF = SMEM_MISC_OFF + 16;   // expert table: offsets, block prefix
// epilogue staging: 32 rows x 64 bytes (32 bf16 columns) per epilogue warp
constexpr int STAGE_COLS = 32;
constexpr int STAGE_WARP_BYTES = 32 * STAGE_COLS * 2;
constexpr int SMEM_Y_OFF = (SMEM_TAB_OFF + 2 * (kMaxExperts + 1) * 4 + 127) / 128 * 128;
constexpr int SMEM_BYTES = SMEM_Y_OFF + NUM_EPI_WARPS * STAGE_WARP_BYTES + 1024;  // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(SF_COL0 >= ACC_COL + BN && SF_COL0 + 16 * STAGES <= TMEM_COLS, "TMEM columns");

struct GemmArgs {
  const uint8_t* s_a;      // ue8m0 [M, K/128]
  const uint8_t* s_w;      // ue8m0 [E, N/128, K/128]
  const int* offsets;      // [E + 1] segment starts (device), or null for one segment {0, M}
  __nv_bfloat16* y;
  int M, N, K, E;
  int* err;
};

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }

__device__ __forceinline__ uint32_t rep4(uint32_t b) { return b * 0x01010101u; }


__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_ue8m0_kernel(const __grid_constant__ CUtensorMap tmap_a,
                  const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + SMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (STAGES + s); };
  const uint32_t tfull_bar = bar_base + 8u * (2 * STAGES);
  const uint32_t tempty_bar = bar_base + 8u * (2 * STAGES + 1);
  const uint32_t drain_bar = bar_base + 8u * (2 * STAGES + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = args.M, N = args.N, K = args.K, E = args.E;
  const int num_n = (N + BN - 1) / BN;
  const int num_kb = K / BK;
  int* tab_off = reinterpret_cast<int*>(smem + SMEM_TAB_OFF);   // [E + 1]
  int* tab_pre = tab_off + (kMaxExperts + 1);                    // [E + 1] blocks before e

  if (warp == 3) {
    // segment offsets: clamped to [0, M], running max (warp scans, 32 at a time)
    int carry = 0;
    for (int base = 0; base <= E; base += 32) {
      const int i = base + lane;
      int o = 0;
      if (i <= E) {
        o = args.offsets != nullptr ? __ldg(args.offsets + i) : (i == 0 ? 0 : M);
        o = min(max(o, 0), M);
      }
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, o, d);
        if (lane >= d) o = max(o, t);
      }
      o = max(o, carry);
      if (i <= E) tab_off[i] = o;
      carry = __shfl_sync(0xffffffffu, o, 31);
    }
    __syncwarp();
    // 128-row blocks before each expert
    carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int b = e < E ? (tab_off[e + 1] - tab_off[e] + BM - 1) / BM : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, b, d);
        if (lane >= d) b += t;
      }
      b += carry;
      if (e < E) tab_pre[e + 1] = b;
      carry = __shfl_sync(0xffffffffu, b, 31);
    }
    if (lane == 0) tab_pre[0] = 0;
  }

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1 + NUM_SF_WARPS);   // TMA producer + scale-factor writers
      ptx::mbar_init(empty_bar(s), 1);
    }
    ptx::mbar_init(tfull_bar, 1);
    ptx::mbar_init(tempty_bar, NUM_EPI_WARPS);
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
  const int total_m = tab_pre[E];
  const int num_tiles = total_m * num_n;
  // tile -> (expert, first row, end of the expert's rows, N tile).  Tiles
  // are expert-major (all of expert e's tiles, M-fastest, before expert
  // e + 1), so an expert's rows of A and its weights are reused from L2
  // while its tiles run; with one expert this is the plain M-fastest order.
  auto map_tile = [&](int tile, int& e, int& row0, int& row_end, int& n_blk) {
    int lo = 0, hi = E - 1;          // the last expert whose first tile is <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab_pre[mid] * num_n <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;                          // has at least one block (else e + 1 would match)
    const int local = tile - tab_pre[e] * num_n;
    const int blocks = tab_pre[e + 1] - tab_pre[e];
    n_blk = local / blocks;
    row0 = tab_off[e] + (local % blocks) * BM;
    row_end = tab_off[e + 1];
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int last_phase[STAGES];
      for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
      uint32_t c = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int e, row0, row_end, n_blk;
        map_tile(tile, e, row0, row_end, n_blk);
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
                           row0);
          ptx::tma_load_2d(smem_base + SMEM_B_OFF + s * B_BYTES, &tmap_b, full_bar(s), kb * BK,
                           e * N + n_blk * BN);
          last_phase[s] = static_cast<int>(ph);
        }
      }
      // Every load this thread issued lands before the CTA may exit.  The
      // full barrier also needs the scale-factor writers' arrivals, which
      // precede any later phase, so waiting on the phase suffices.
      for (int s = 0; s < STAGES; ++s)
        if (last_phase[s] >= 0 && !ptx::mbar_wait(full_bar(s), static_cast<uint32_t>(last_phase[s])))
          record_error(args.err, kErrTimeoutProducer);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    uint32_t c = 0, t_local = 0;
    bool ok = true, issued = false;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t_local) {
      ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(tempty_bar, (t_local & 1u) ^ 1u));
      if (!ok) {
        if (lane == 0) record_error(args.err, kErrTimeoutMma);
        break;
      }
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
          const uint32_t sf = tmem_base + SF_COL0 + 16u * static_cast<uint32_t>(s);
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            ptx::mma_mxf8f6f4_block_scale(
                tmem_base + ACC_COL, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), IDESC | ptx::idesc_sf_ids(k, k),
                sf + SFA_COL, sf + SFB_COL, (kb | k) != 0 ? 1u : 0u);
          }
          ptx::mma_commit(empty_bar(s));
          if (kb == num_kb - 1) ptx::mma_commit(tfull_bar);
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
    // ------------------------------------ scale-factor writers + epilogue
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const bool sf_writer = warp < 4 + NUM_SF_WARPS;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int nblk_count = N / 128;
    // Chunk c of this CTA = (its (c / num_kb)-th tile, K block c % num_kb),
    // in the producer's order.
    const int my_tiles =
        static_cast<int>(blockIdx.x) < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const uint32_t total = static_cast<uint32_t>(my_tiles) * static_cast<uint32_t>(num_kb);
    uint32_t c_sf = 0;   // next chunk whose scale factors this warp writes
    bool ok = true;
    auto write_sf = [&](uint32_t c) -> bool {
      const int tile = static_cast<int>(blockIdx.x + (c / num_kb) * gridDim.x);
      const int kb = static_cast<int>(c % num_kb);
      int e, row0, row_end, n_blk;
      map_tile(tile, e, row0, row_end, n_blk);
      // loads first: they land while the slot is still in use
      uint32_t v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = row0 + 32 * j + lane;
        v[j] = row < row_end ? __ldg(args.s_a + static_cast<int64_t>(row) * num_kb + kb)
                             : kUnitScale;
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int nb = n_blk * 2 + h;
        v[4 + 4 * h] =
            nb < nblk_count
                ? __ldg(args.s_w + (static_cast<int64_t>(e) * nblk_count + nb) * num_kb + kb)
                : kUnitScale;
      }
      const int s = c % STAGES;
      const uint32_t ph = (c / STAGES) & 1u;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(empty_bar(s), ph ^ 1u))) return false;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = rep4(v[j]);
      const uint32_t b0 = rep4(v[4]), b1 = rep4(v[8]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[4 + j] = b0;
        v[8 + j] = b1;
        v[12 + j] = 0u;
      }
      ptx::tmem_st_32x32b_x16(tmem_base + lane_off + SF_COL0 + 16u * static_cast<uint32_t>(s), v);
      ptx::tmem_st_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(full_bar(s));
      return true;
    };
    uint32_t t_local = 0;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t_local) {
      if (sf_writer) {
        // this tile's stages and the next tile's first STAGES stages (their
        // slots are freed by this tile's MMAs, not by its epilogue)
        const uint32_t upto = (t_local + 1) * static_cast<uint32_t>(num_kb) + STAGES;
        for (; c_sf < total && c_sf < upto; ++c_sf) {
          if (!write_sf(c_sf)) {
            if (lane == 0) record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
        }
        if (!ok) break;
      }
      int e, row0, row_end, n_blk;
      map_tile(tile, e, row0, row_end, n_blk);
      const int nb = n_blk * 2 + half;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tfull_bar, t_local & 1u))) {
        if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
        break;
      }
      ptx::tc_fence_after();
      uint32_t v0[64], v1[64];
      const uint32_t tb = tmem_base + lane_off + ACC_COL + static_cast<uint32_t>(half * 128);
      ptx::tmem_ld_32x32b_x64(tb, v0);
      ptx::tmem_ld_32x32b_x64(tb + 64, v1);
      ptx::tmem_ld_wait();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(tempty_bar);
      if (nb < nblk_count) {
        const int wrow0 = row0 + quarter * 32;   // this warp's first row
        const uint32_t stage =
            smem_base + SMEM_Y_OFF + static_cast<uint32_t>(warp - 4) * STAGE_WARP_BYTES;
        const uint8_t* stage_g = smem + SMEM_Y_OFF + (warp - 4) * STAGE_WARP_BYTES;
#pragma unroll
        for (int pass = 0; pass < 128 / STAGE_COLS; ++pass) {
          // my row's 32 columns -> 64 bytes of the staging box
#pragma unroll
          for (int j = 0; j < STAGE_COLS / 8; ++j) {
            const int col = pass * STAGE_COLS + 8 * j;
            const uint32_t* src = col < 64 ? v0 + col : v1 + (col - 64);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              __nv_bfloat162 p = __float22bfloat162_rn(
                  make_float2(__uint_as_float(src[2 * i]), __uint_as_float(src[2 * i + 1])));
              o[i] = *reinterpret_cast<uint32_t*>(&p);
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                             stage + static_cast<uint32_t>(lane * STAGE_COLS * 2 + 16 * j)),
                         "r"(o[0]), "r"(o[1]), "r"(o[2]), "r"(o[3])
                         : "memory");
          }
          __syncwarp();
          // out: lane l writes 16 bytes of row (8 it + l / 4); the warp's
          // instruction covers eight rows' 64-byte segments
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int r = 8 * it + (lane >> 2);
            const int q = lane & 3;
            const uint4 val = *reinterpret_cast<const uint4*>(stage_g + r * STAGE_COLS * 2 + 16 * q);
            if (wrow0 + r < row_end)
              *reinterpret_cast<uint4*>(args.y + static_cast<int64_t>(wrow0 + r) * N + nb * 128 +
                                        pass * STAGE_COLS + 8 * q) = val;
          }
          __syncwarp();
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
    return cudaFuncSetAttribute(gemm_ue8m0_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SMEM_BYTES);
  });
}

}  // namespace

cudaError_t launch_grouped_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                        const uint8_t* s_w, const int32_t* offsets, void* y,
                                        int64_t M, int64_t N, int64_t K, int64_t E,
                                        const DeviceInfo& dev, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  if (E < 1 || E > kMaxExperts) return cudaErrorInvalidValue;
  cudaError_t e = ensure_smem_attr();
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, q_a, M, K, BM, BK) || !make_tmap_u8(&tb, q_w, E * N, K, BN, BK))
    return cudaErrorInvalidValue;
  GemmArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.offsets = offsets;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.E = static_cast<int>(E);
  a.err = dev.error_flag;
  // tiles: at most ceil(M / 128) + E row blocks (one partial block per segment)
  const int64_t row_blocks = (M + BM - 1) / BM + (offsets != nullptr ? E : 0);
  const int64_t tiles = row_blocks * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < dev.sm_count ? tiles : dev.sm_count);
  gemm_ue8m0_kernel<<<grid, NUM_THREADS, SMEM_BYTES, st>>>(ta, tb, a);
  return cudaGetLastError();
}

cudaError_t launch_block_linear_ue8m0(const void* q_a, const uint8_t* s_a, const void* q_w,
                                      const uint8_t* s_w, void* y, int64_t M, int64_t N,
                                      int64_t K, const DeviceInfo& dev, cudaStream_t st) {
  return launch_grouped_linear_ue8m0(q_a, s_a, q_w, s_w, nullptr, y, M, N, K, 1, dev, st);
}

}  // namespace fp8bl
