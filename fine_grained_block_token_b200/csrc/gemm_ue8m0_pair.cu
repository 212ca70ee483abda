// UE8M0 block-scaled FP8 GEMM on CTA pairs for sm_100a:
//   y = bf16( sum_k (q_a 2^sa) (q_w 2^sw)^T )  with tcgen05.mma.cta_group::2
//   .kind::mxf8f6f4.block_scale.
//
// "UE8M0 scale format" section of the "Fine-grained FP8" page: power-of-two
// scales stored as one byte (float8_e8m0fnu).  The tensor core's block-scaled
// MMA applies them per 32-deep K slice from TMEM, so the accumulator runs
// over all of K (no promotion) and the bound is the MMA pipeline itself.
//
// Two CTAs of a cluster compute one 256 (M) x 256 (N) tile: CTA r loads rows
// 128 r .. +127 of the tile's A block and of its W block (32 KB per stage,
// six stages) and the even CTA issues M = 256 MMAs.  The scale factors reach
// TMEM without any thread arriving across the pair: two small kernels first
// rewrite the scale grids in the order the MMA reads them from TMEM (the
// caller's workspace), the producers TMA-load each stage's factors with its
// operands (counted in bytes on the even CTA's full barrier, like the
// operands), and the MMA issuer copies them into both CTAs' TMEM with
// tcgen05.cp.cta_group::2 ahead of the stage's four MMAs (the tensor pipe
// runs copies and MMAs in issue order, so one factor slot suffices).
// Packed layouts (one 16-byte row per TMEM lane group row r = 0..31):
//   activations: sfa[(kb * MBp + t) * 32 + r] = word j (j = 0..3) holds the
//     code of row 128 t + 32 j + r replicated into its 4 bytes (one byte per
//     32-deep slice of the 128-deep block kb);
//   weights: sfw[(kb * NBp + nb) * 32 + r] = the code of block (nb, kb)
//     replicated into all 16 bytes;
//   rows / blocks past the matrix hold 127, the code of 1.0.
// Grouped (MoE expert) form, same kernel: rows of A split into E contiguous
// segments [off[e], off[e+1]), segment e times expert e's W[e] ([E, N, K],
// scales [E, N/128, K/128]).  Each CTA's warp 3 turns the offsets into a
// shared-memory table at start-up (clamped to [0, M], made non-decreasing)
// with each expert's count of 256-row blocks; tiles run expert by expert.
// The activation factors are packed per expert, each segment padded to 256
// rows (so a tile's 128-row halves start on a packed group), and the weight
// factors per expert.  The plain linear is E = 1, off = {0, M}.
// Warps: 0 producer (both CTAs), 1 MMA issuer (even CTA), 2 TMEM owner,
// 3 expert table, 4-11 epilogue (both CTAs): after a tile's last MMA each warp reads its 32
// TMEM lanes x 128 columns, releases the accumulator (the odd CTA's warps
// arrive on the even CTA's barrier, once per tile) and stores bf16 through a
// shared staging box, 32 columns at a time, in 64-byte row segments.
// Every wait is bounded; on expiry the kernel records an error code, drains
// what it started and exits cleanly.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"

namespace fp8bl {
namespace {

constexpr int BK = 128, UMMA_K = 32;
constexpr int PBM = 256, PBN = 256, PSTAGES = 6;
constexpr int PA_BYTES = 128 * BK, PB_BYTES = 128 * BK;
constexpr int SFA_BYTES = 512, SFB_BYTES = 1024;
constexpr int TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0, SFA_COL = 256, SFB_COL = 264;
constexpr int NUM_THREADS = 384, NUM_EPI_WARPS = 8;
constexpr uint32_t IDESC = ptx::idesc_mxf8_e4m3_ue8m0(PBM, PBN);
constexpr int STAGE_COLS = 32;                       // epilogue staging: 32 rows x 64 bytes
constexpr int STAGE_WARP_BYTES = 32 * STAGE_COLS * 2;
constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + PSTAGES * PA_BYTES;
constexpr int SMEM_SFA_OFF = SMEM_B_OFF + PSTAGES * PB_BYTES;
constexpr int SMEM_SFB_OFF = SMEM_SFA_OFF + PSTAGES * SFA_BYTES;
constexpr int SMEM_Y_OFF = SMEM_SFB_OFF + PSTAGES * SFB_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_Y_OFF + NUM_EPI_WARPS * STAGE_WARP_BYTES;
constexpr int NUM_BARS = 2 * PSTAGES + 3;     // full, empty, tfull, tempty, drain
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_TAB_OFF = SMEM_MISC_OFF + 16;   // expert table: offsets, 256-row block prefix
constexpr int SMEM_BYTES = SMEM_TAB_OFF + 2 * (kMaxExperts + 1) * 4 + 1024;
constexpr uint32_t STAGE_TX = 2u * (PA_BYTES + PB_BYTES + SFA_BYTES + SFB_BYTES);
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(SFB_COL + 8 <= TMEM_COLS && SFA_COL + 4 <= SFB_COL && ACC_COL + PBN <= SFA_COL, "TMEM");

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }
__device__ __forceinline__ uint32_t rep4(uint32_t b) { return b * 0x01010101u; }

// Shared -> tensor memory copy of 32 rows x 128 bits into both CTAs of the
// pair (each from its own shared memory at the same offset), broadcast to
// the four 32-lane quarters.
__device__ __forceinline__ void cp_32x128b_warpx4_pair(uint32_t taddr, uint64_t src_desc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
               : "memory");
}

// D (+)= (A 2^sfa) (B 2^sfb)^T for the pair, e4m3 x e4m3 -> fp32, ue8m0
// factors from TMEM, issued by the even CTA.
__device__ __forceinline__ void mma_block_scale_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                     uint32_t idesc, uint32_t sfa_tmem,
                                                     uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
      "r"(sfb_tmem)
      : "memory");
}

// Expert table, built by one warp: tab_off[0..E] = the segment starts
// clamped to [0, M] and made non-decreasing (running maximum), tab_pre[e] =
// the 256-row blocks of the experts before e.  offsets == nullptr means one
// segment {0, M}.
__device__ void build_expert_table(const int* offsets, int E, int M, int lane, int* tab_off,
                                   int* tab_pre) {
  int carry = 0;
  for (int base = 0; base <= E; base += 32) {
    const int i = base + lane;
    int o = 0;
    if (i <= E) {
      o = offsets != nullptr ? __ldg(offsets + i) : (i == 0 ? 0 : M);
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
  carry = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    int b = e < E ? (tab_off[e + 1] - tab_off[e] + PBM - 1) / PBM : 0;
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
  __syncwarp();
}

// The last expert whose first 256-row block is at or before block `blk`
// (an expert with no rows never matches, since the next one starts at the
// same block).
__device__ __forceinline__ int expert_of_block(const int* tab_pre, int E, int blk) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab_pre[mid] <= blk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Activation factors in MMA order, per expert, every segment padded to a
// multiple of 256 rows: packed 128-row group t holds padded rows 128 t ..;
// padded row p of expert e is row off[e] + (p - 256 tab_pre[e]) of A, or
// padding (127) past the segment.  Grid: KB * MBp * 32 threads.
__global__ void pack_sfa_kernel(const uint8_t* __restrict__ s, int M, int KB, int MBp,
                                const int* offsets, int E, uint4* __restrict__ out) {
  __shared__ int tab_off[kMaxExperts + 1], tab_pre[kMaxExperts + 1];
  if (threadIdx.x < 32) build_expert_table(offsets, E, M, threadIdx.x, tab_off, tab_pre);
  __syncthreads();
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(KB) * MBp * 32;
  if (i >= total) return;
  const int r = static_cast<int>(i & 31);
  const int64_t t = i >> 5;
  const int rb = static_cast<int>(t % MBp);
  const int kb = static_cast<int>(t / MBp);
  const int padded_rows = tab_pre[E] * PBM;
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int p = rb * 128 + 32 * j + r;
    uint32_t code = 127u;
    if (p < padded_rows) {
      const int e = expert_of_block(tab_pre, E, p / PBM);
      const int local = p - tab_pre[e] * PBM;
      if (local < tab_off[e + 1] - tab_off[e])
        code = s[static_cast<int64_t>(tab_off[e] + local) * KB + kb];
    }
    w[j] = rep4(code);
  }
  out[i] = make_uint4(w[0], w[1], w[2], w[3]);
}

// Weight factors in MMA order, per expert: row ((e * KB + kb) * NBp + nb) *
// 32 + r holds block (nb, kb) of expert e replicated into 16 bytes.
__global__ void pack_sfw_kernel(const uint8_t* __restrict__ s, int NB, int KB, int NBp, int E,
                                uint4* __restrict__ out) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = static_cast<int64_t>(E) * KB * NBp * 32;
  if (i >= total) return;
  const int64_t t = i >> 5;
  const int nb = static_cast<int>(t % NBp);
  const int64_t ekb = t / NBp;
  const int kb = static_cast<int>(ekb % KB);
  const int e = static_cast<int>(ekb / KB);
  const uint32_t w =
      rep4(nb < NB ? s[(static_cast<int64_t>(e) * NB + nb) * KB + kb] : 127u);
  out[i] = make_uint4(w, w, w, w);
}

struct PairArgs {
  __nv_bfloat16* y;
  const int* offsets;   // [E + 1] segment starts (device), or null for one segment {0, M}
  int M, N, K, E;
  int MBp, NBp;   // padded 128-row group counts of the packed factor arrays (per expert for W)
  int* err;
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_ue8m0_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                       const __grid_constant__ CUtensorMap tmap_sfa,
                       const __grid_constant__ CUtensorMap tmap_sfb, const PairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + SMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (PSTAGES + s); };
  const uint32_t tfull_bar = bar_base + 8u * (2 * PSTAGES);
  const uint32_t tempty_bar = bar_base + 8u * (2 * PSTAGES + 1);
  const uint32_t drain_bar = bar_base + 8u * (2 * PSTAGES + 2);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();      // 0 = the pair's MMA issuer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  const int M = args.M, N = args.N, K = args.K, E = args.E;
  const int num_n = (N + PBN - 1) / PBN;
  const int num_kb = K / BK;
  const int nblk_count = N / 128;
  constexpr uint16_t kBoth = 0x3;
  int* tab_off = reinterpret_cast<int*>(smem + SMEM_TAB_OFF);   // [E + 1]
  int* tab_pre = tab_off + (kMaxExperts + 1);                    // [E + 1]
  if (warp == 3) build_expert_table(args.offsets, E, M, lane, tab_off, tab_pre);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    ptx::mbar_init(tfull_bar, 1);
    ptx::mbar_init(tempty_bar, 2 * NUM_EPI_WARPS);
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_a);
    ptx::prefetch_tmap(&tmap_b);
    ptx::prefetch_tmap(&tmap_sfa);
    ptx::prefetch_tmap(&tmap_sfb);
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
  const int num_tiles = tab_pre[E] * num_n;
  const bool has_tiles = pair < num_tiles;
  // tile -> (expert, its global 256-row block, first row, end of its rows,
  // N tile); expert-major, M-fastest within an expert.
  auto map_tile = [&](int tile, int& e, int& gblk, int& row0, int& row_end, int& n_blk) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tab_pre[mid] * num_n <= tile) lo = mid; else hi = mid - 1;
    }
    e = lo;
    const int local = tile - tab_pre[e] * num_n;
    const int blocks = tab_pre[e + 1] - tab_pre[e];
    n_blk = local / blocks;
    gblk = tab_pre[e] + local % blocks;
    row0 = tab_off[e] + (local % blocks) * PBM;
    row_end = tab_off[e + 1];
  };

  if (warp == 0) {
    // ------------------------------------------------- producer (both CTAs)
    if (lane == 0) {
      uint32_t c = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int e, gblk, row0, row_end, n_blk;
        map_tile(tile, e, gblk, row0, row_end, n_blk);
        const int mt = gblk * 2 + static_cast<int>(rank);      // this CTA's packed 128-row group
        for (int kb = 0; kb < num_kb; ++kb, ++c) {
          const int s = c % PSTAGES;
          const uint32_t ph = (c / PSTAGES) & 1u;
          if (!ptx::mbar_wait_cluster(empty_bar(s), ph ^ 1u)) {
            record_error(args.err, kErrTimeoutProducer);
            ok = false;
            break;
          }
          const uint32_t fb = ptx::map_to_cta(full_bar(s), 0);
          if (leader) ptx::mbar_arrive_expect_tx(full_bar(s), STAGE_TX);
          ptx::tma_load_2d_pair(smem_base + SMEM_A_OFF + s * PA_BYTES, &tmap_a, fb, kb * BK,
                                row0 + 128 * static_cast<int>(rank));
          ptx::tma_load_2d_pair(smem_base + SMEM_B_OFF + s * PB_BYTES, &tmap_b, fb, kb * BK,
                                e * N + n_blk * PBN + 128 * static_cast<int>(rank));
          ptx::tma_load_2d_pair(smem_base + SMEM_SFA_OFF + s * SFA_BYTES, &tmap_sfa, fb, 0,
                                (kb * args.MBp + mt) * 32);
          ptx::tma_load_2d_pair(smem_base + SMEM_SFB_OFF + s * SFB_BYTES, &tmap_sfb, fb, 0,
                                ((e * num_kb + kb) * args.NBp + n_blk * 2) * 32);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA (even CTA only)
    if (leader) {
      uint32_t c = 0, t_local = 0;
      bool ok = true, issued = false;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++t_local) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tempty_bar, (t_local & 1u) ^ 1u));
        if (!ok) {
          if (lane == 0) record_error(args.err, kErrTimeoutMma);
          break;
        }
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
            const uint32_t a_addr = smem_base + SMEM_A_OFF + s * PA_BYTES;
            const uint32_t b_addr = smem_base + SMEM_B_OFF + s * PB_BYTES;
            const uint32_t sfa_addr = smem_base + SMEM_SFA_OFF + s * SFA_BYTES;
            const uint32_t sfb_addr = smem_base + SMEM_SFB_OFF + s * SFB_BYTES;
            cp_32x128b_warpx4_pair(tmem_base + SFA_COL, ptx::sdesc_rows16_noswizzle(sfa_addr));
            cp_32x128b_warpx4_pair(tmem_base + SFB_COL, ptx::sdesc_rows16_noswizzle(sfb_addr));
            cp_32x128b_warpx4_pair(tmem_base + SFB_COL + 4, ptx::sdesc_rows16_noswizzle(sfb_addr + 512));
#pragma unroll
            for (int k = 0; k < BK / UMMA_K; ++k)
              mma_block_scale_pair(tmem_base + ACC_COL, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                                   ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K),
                                   IDESC | ptx::idesc_sf_ids(k, k), tmem_base + SFA_COL,
                                   tmem_base + SFB_COL, (kb | k) != 0 ? 1u : 0u);
            ptx::mma_commit_pair_multicast(empty_bar(s), kBoth);
            if (kb == num_kb - 1) ptx::mma_commit_pair_multicast(tfull_bar, kBoth);
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
    const uint32_t stage = smem_base + SMEM_Y_OFF + static_cast<uint32_t>(warp - 4) * STAGE_WARP_BYTES;
    const uint8_t* stage_g = smem + SMEM_Y_OFF + (warp - 4) * STAGE_WARP_BYTES;
    uint32_t t_local = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++t_local) {
      int e, gblk, row0, row_end, n_blk;
      map_tile(tile, e, gblk, row0, row_end, n_blk);
      const int wrow0 = row0 + 128 * static_cast<int>(rank) + quarter * 32;
      const int nb = n_blk * 2 + half;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin_cluster(tfull_bar, t_local & 1u))) {
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
      if (lane == 0) {
        if (leader) ptx::mbar_arrive(tempty_bar);
        else ptx::mbar_arrive_remote(ptx::map_to_cta(tempty_bar, 0));
      }
      if (nb < nblk_count) {
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
  ptx::cluster_sync();   // neither CTA releases TMEM or exits while its peer still uses it
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// Packed activation groups: 2 per 256-row block of every expert's segment;
// sum_e ceil(len_e / 256) <= ceil(M / 256) + E bounds the grouped case.
int64_t mbp_of(int64_t M, int64_t E) { return 2 * ((M + PBM - 1) / PBM + (E > 1 ? E : 0)); }
int64_t nbp_of(int64_t N) { return 2 * ((N + PBN - 1) / PBN); }

cudaError_t ensure_ue8m0_pair_ready(int* max_clusters) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  static int clusters_of[kMaxDevices];
  int dev = 0;
  const cudaError_t r = once_per_device(once, status, [](int d) {
    cudaError_t st = cudaFuncSetAttribute(gemm_ue8m0_pair_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
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
    st = cudaOccupancyMaxActiveClusters(&clusters, gemm_ue8m0_pair_kernel, &cfg);
    if (st == cudaSuccess && clusters < 1) st = cudaErrorInvalidConfiguration;
    clusters_of[d] = clusters;
    return st;
  }, &dev);
  *max_clusters = r == cudaSuccess ? clusters_of[dev] : 0;
  return r;
}

}  // namespace

// The pair schedule serves M above one 128-row tile (below it the odd CTA
// would only compute padding); smaller M run on the single-CTA kernel.
bool ue8m0_use_pairs(int64_t M) { return M > 128; }

size_t ue8m0_pair_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E) {
  if (!ue8m0_use_pairs(M)) return 0;
  const int64_t KB = K / 128;
  return static_cast<size_t>(KB * mbp_of(M, E) * 512 + E * KB * nbp_of(N) * 512);
}

cudaError_t launch_linear_ue8m0_pairs(const void* q_a, const uint8_t* s_a, const void* q_w,
                                      const uint8_t* s_w, const int* offsets, void* y, int64_t M,
                                      int64_t N, int64_t K, int64_t E, void* workspace,
                                      const DeviceInfo& dev, cudaStream_t st) {
  if (E < 1 || E > kMaxExperts) return cudaErrorInvalidValue;
  int max_clusters = 0;
  cudaError_t e = ensure_ue8m0_pair_ready(&max_clusters);
  if (e != cudaSuccess) return e;
  const int KB = static_cast<int>(K / 128);
  const int MBp = static_cast<int>(mbp_of(M, E)), NBp = static_cast<int>(nbp_of(N));
  uint8_t* psa = static_cast<uint8_t*>(workspace);
  uint8_t* psw = psa + static_cast<int64_t>(KB) * MBp * 512;
  const int64_t ta = static_cast<int64_t>(KB) * MBp * 32, tw = E * KB * NBp * 32;
  if ((ta + 255) / 256 > 0x7FFFFFFFll || (tw + 255) / 256 > 0x7FFFFFFFll) return cudaErrorInvalidValue;
  pack_sfa_kernel<<<static_cast<unsigned>((ta + 255) / 256), 256, 0, st>>>(
      s_a, static_cast<int>(M), KB, MBp, offsets, static_cast<int>(E), reinterpret_cast<uint4*>(psa));
  pack_sfw_kernel<<<static_cast<unsigned>((tw + 255) / 256), 256, 0, st>>>(
      s_w, static_cast<int>(N / 128), KB, NBp, static_cast<int>(E), reinterpret_cast<uint4*>(psw));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap ta_m, tb_m, tsa, tsb;
  if (!make_tmap_u8(&ta_m, q_a, M, K, 128, BK) || !make_tmap_u8(&tb_m, q_w, E * N, K, 128, BK) ||
      !make_tmap_u8(&tsa, psa, static_cast<uint64_t>(ta), 16, 32, 16, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap_u8(&tsb, psw, static_cast<uint64_t>(tw), 16, 64, 16, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  PairArgs a;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.offsets = offsets;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.E = static_cast<int>(E);
  a.MBp = MBp;
  a.NBp = NBp;
  a.err = dev.error_flag;
  // tiles: at most (ceil(M / 256) + E - 1) 256-row blocks over the experts
  const int64_t mblocks = (M + PBM - 1) / PBM + (E > 1 ? E - 1 : 0);
  const int64_t tiles = mblocks * ((N + PBN - 1) / PBN);
  if (tiles == 0) return cudaSuccess;
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
  return cudaLaunchKernelEx(&cfg, gemm_ue8m0_pair_kernel, ta_m, tb_m, tsa, tsb, a);
}

}  // namespace fp8bl
