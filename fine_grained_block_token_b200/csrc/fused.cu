// Fused activation quantization + block-scaled FP8 GEMM for sm_100a:
//   y = bf16( sum_j s_a[:,j] s_w[:,j] (A_j W_j^T) ),  (A, s_a) = quant(X)
//
// "Fine-grained FP8" page (opening bullet list; "DeepGEMM fast path"
// section: the dynamic activation scheme): activations are quantized per
// token in groups of 128 input channels at run time.  Here that happens
// inside the GEMM, on the bf16 activation tile, with the arithmetic of the
// stand-alone quantizer (quant_math.cuh): codes, scales and therefore Y are
// bit-identical to quantizing first and then multiplying, and the quantized
// activations never reach HBM.
//
// Every 128 x 256 output tile needs the quantized 128 x 128 A chunk, and
// the tiles of one row band share it.  Four CTAs of a thread-block cluster
// compute the four neighbouring N-tiles of one row band; each quantizes a
// quarter of the band (32 rows) and writes the codes and scales into the
// shared memory of all four (distributed shared memory), so each A element
// is quantized once per 1024 output columns instead of once per 256, and
// each CTA loads only 32 rows of bf16 activations.
//
// Per CTA (one per SM, persistent over (row band, group of 4 N-tiles)):
//   warp 0       TMA producer for its 32 bf16 activation rows (two 64-column
//                boxes, 128-byte swizzle) into a 3-slot ring.
//   warp 3       TMA producer for its 256 x 128 e4m3 W tile (4 stages).
//   warps 12-15  quantizers: 4 threads per row, 32 elements each (amax
//                combined with two shuffles).  They write the codes into A
//                stage s of every CTA of the cluster, in the K-major 128-byte
//                swizzled layout the MMA reads, and the scales into a ring,
//                once every CTA's MMA has released stage s (multicast commit).
//   warp 1       MMA issuer (warp-wide loop, one elected lane issues): 4 MMAs per chunk
//                (M=128, N=256, K=32) into one of two 256-column TMEM buffers.
//   warp 2       TMEM owner, then the slice sender: once the quantizers
//                have written their rows, bulk-copies them (and the scales)
//                into the other CTAs' shared memory, completion counted in
//                bytes on the receivers' barriers (no multicast).
//   warps 4-11   promotion as in the unfused kernel, s_a from the ring.
// Registers: the block launches with 512 x 128; warps 0-3 drop to 40, the
// promotion warpgroups take 176 and the quantizers 120 (sum = launch total).
// Every mbarrier wait is bounded in time; on expiry the kernel records an
// error code in the error word, drains what it started and exits cleanly;
// the CTAs of a cluster leave together (cluster barrier) so that no remote
// write or arrival reaches a CTA that has exited.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"
#include "quant_math.cuh"

namespace fp8bl {
namespace {

constexpr int CL = 4;                              // CTAs per cluster (along N)
constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int QROWS = BM / CL;                     // rows each CTA quantizes
constexpr int STAGES = 4;                          // A codes + W tile
constexpr int XSLOTS = 3;                          // bf16 activation slices
constexpr int UMMA_K = 32;
constexpr int A_BYTES = BM * BK;                   // 16 KB of codes
constexpr int B_BYTES = BN * BK;                   // 32 KB of weights
constexpr int X_BOX_BYTES = QROWS * 128;           // 32 rows x 64 bf16
constexpr int X_BYTES = 2 * X_BOX_BYTES;           // 8 KB
constexpr int SA_SLOTS = 8;
constexpr int TMEM_COLS = 512;
constexpr int NUM_EPI_WARPS = 8;
constexpr int FIRST_QUANT_WARP = 12;
constexpr int NUM_QUANT_WARPS = 4;
constexpr int NUM_THREADS = 32 * (FIRST_QUANT_WARP + NUM_QUANT_WARPS);   // 512
constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(BM, BN);
constexpr uint16_t CL_MASK = (1u << CL) - 1;

constexpr int SMEM_A_OFF = 0;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * A_BYTES;
constexpr int SMEM_X_OFF = SMEM_B_OFF + STAGES * B_BYTES;
constexpr int SMEM_SA_OFF = SMEM_X_OFF + XSLOTS * X_BYTES;
constexpr int SMEM_BAR_OFF = SMEM_SA_OFF + SA_SLOTS * BM * 4;
// xfull[X], xempty[X], wfull[S], wempty[S], aempty[S], qdone[S], tfull[2],
// tempty[2], sfull[SA], drain, slice[S]
constexpr int NUM_BARS = 2 * XSLOTS + 5 * STAGES + 4 + SA_SLOTS + 1;
constexpr uint32_t SLICE_BYTES = QROWS * 128;      // one CTA's rows of codes
constexpr uint32_t SCALE_BYTES = QROWS * 4;        // and their scales
constexpr int SMEM_MISC_OFF = SMEM_BAR_OFF + NUM_BARS * 8;
constexpr int SMEM_BYTES = SMEM_MISC_OFF + 16 + 1024;   // + slack for 1024-byte alignment

struct FusedArgs {
  const float* s_w;
  __nv_bfloat16* y;
  int M, N, K;
  int group_m;       // row bands per raster group (see unit_coords)
  int* err;
};

// Unit u -> (row band, group of CL N-tiles).  Row bands are taken in groups
// of group_m; within a group the N-groups are outer and the bands inner, so
// the clusters running together share a few activation bands (which stay in
// L2 while every N-group passes over them) and a few weight groups.
__device__ __forceinline__ void unit_coords(int u, int num_m, int num_g, int group_m, int& m_blk,
                                            int& g) {
  const int per_group = group_m * num_g;
  const int grp = u / per_group;
  const int base = grp * group_m;
  const int gm = min(group_m, num_m - base);
  const int idx = u - grp * per_group;
  g = idx / gm;
  m_blk = base + idx % gm;
}

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_fused_kernel(const __grid_constant__ CUtensorMap tmap_x,
                  const __grid_constant__ CUtensorMap tmap_b, const FusedArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + SMEM_BAR_OFF;
  auto xfull = [&](uint32_t i) { return bar_base + 8u * i; };
  auto xempty = [&](uint32_t i) { return bar_base + 8u * (XSLOTS + i); };
  auto wfull = [&](uint32_t s) { return bar_base + 8u * (2 * XSLOTS + s); };
  auto wempty = [&](uint32_t s) { return bar_base + 8u * (2 * XSLOTS + STAGES + s); };
  auto aempty = [&](uint32_t s) { return bar_base + 8u * (2 * XSLOTS + 2 * STAGES + s); };
  auto qdone = [&](uint32_t s) { return bar_base + 8u * (2 * XSLOTS + 3 * STAGES + s); };
  auto tfull = [&](uint32_t b) { return bar_base + 8u * (2 * XSLOTS + 4 * STAGES + b); };
  auto tempty = [&](uint32_t b) { return bar_base + 8u * (2 * XSLOTS + 4 * STAGES + 2 + b); };
  auto sfull = [&](uint32_t k) { return bar_base + 8u * (2 * XSLOTS + 4 * STAGES + 4 + k); };
  const uint32_t drain_bar = bar_base + 8u * (2 * XSLOTS + 4 * STAGES + 4 + SA_SLOTS);
  auto slice = [&](uint32_t s) { return bar_base + 8u * (2 * XSLOTS + 4 * STAGES + 5 + SA_SLOTS + s); };
  const uint32_t sa_base = smem_base + SMEM_SA_OFF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + SMEM_MISC_OFF);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const int cluster_id = blockIdx.x / CL;
  const int num_clusters = gridDim.x / CL;
  const int M = args.M, N = args.N, K = args.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_g = (num_n + CL - 1) / CL;
  const int num_kb = K / BK;
  const int num_units = num_m * num_g;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < XSLOTS; ++i) {
      ptx::mbar_init(xfull(i), 1);
      ptx::mbar_init(xempty(i), NUM_QUANT_WARPS);
    }
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(wfull(s), 1);
      ptx::mbar_init(wempty(s), 1);
      ptx::mbar_init(aempty(s), CL);                  // one commit per CTA
      ptx::mbar_init(qdone(s), 1);                    // local arrival + remote bytes
      ptx::mbar_init(slice(s), NUM_QUANT_WARPS);      // this CTA's rows written
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(tfull(b), 1);
      ptx::mbar_init(tempty(b), NUM_EPI_WARPS);
    }
    for (int k = 0; k < SA_SLOTS; ++k) ptx::mbar_init(sfull(k), 1);
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_x);
    ptx::prefetch_tmap(&tmap_b);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();   // every CTA's barriers exist before any remote arrival
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);

  if (warp == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    // ------------------------------------------------- activation producer
    int last_phase[XSLOTS];
    for (int i = 0; i < XSLOTS; ++i) last_phase[i] = -1;
    uint32_t c = 0;
    bool ok = true;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      int m_blk, g;
      unit_coords(u, num_m, num_g, args.group_m, m_blk, g);
      const int row0 = m_blk * BM + static_cast<int>(rank) * QROWS;
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const uint32_t xs = c % XSLOTS;
        const uint32_t ph = (c / XSLOTS) & 1u;
        if (c >= XSLOTS) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(xempty(xs), ph ^ 1u));
          if (!ok) {
            if (lane == 0) record_error(args.err, kErrTimeoutProducer);
            break;
          }
        }
        if (lane == 0) {
          const uint32_t dst = smem_base + SMEM_X_OFF + xs * X_BYTES;
          ptx::mbar_arrive_expect_tx(xfull(xs), X_BYTES);
          // X viewed as bytes [M, 2K]: column (bytes) 256 kb + 128 box
          ptx::tma_load_2d(dst, &tmap_x, xfull(xs), kb * 256, row0);
          ptx::tma_load_2d(dst + X_BOX_BYTES, &tmap_x, xfull(xs), kb * 256 + 128, row0);
        }
        __syncwarp();
        last_phase[xs] = static_cast<int>(ph);
      }
    }
    if (lane == 0)
      for (int i = 0; i < XSLOTS; ++i)
        if (last_phase[i] >= 0 && !ptx::mbar_wait(xfull(i), static_cast<uint32_t>(last_phase[i])))
          record_error(args.err, kErrTimeoutProducer);
    __syncwarp();
  } else if (warp == 3) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    // ----------------------------------------------------- weight producer
    int last_phase[STAGES];
    for (int s = 0; s < STAGES; ++s) last_phase[s] = -1;
    uint32_t c = 0;
    bool ok = true;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      int m_blk, g;
      unit_coords(u, num_m, num_g, args.group_m, m_blk, g);
      const int n_blk = g * CL + static_cast<int>(rank);
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const uint32_t s = c % STAGES;
        const uint32_t ph = (c / STAGES) & 1u;
        if (c >= STAGES) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(wempty(s), ph ^ 1u));
          if (!ok) {
            if (lane == 0) record_error(args.err, kErrTimeoutProducer);
            break;
          }
        }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(wfull(s), B_BYTES);
          ptx::tma_load_2d(smem_base + SMEM_B_OFF + s * B_BYTES, &tmap_b, wfull(s), kb * BK, n_blk * BN);
        }
        __syncwarp();
        last_phase[s] = static_cast<int>(ph);
      }
    }
    if (lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (last_phase[s] >= 0 && !ptx::mbar_wait(wfull(s), static_cast<uint32_t>(last_phase[s])))
          record_error(args.err, kErrTimeoutProducer);
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    // ----------------------------------------------------------------- MMA
    uint32_t c = 0;
    bool ok = true, issued = false;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const uint32_t s = c % STAGES;
        const uint32_t sph = (c / STAGES) & 1u;
        const uint32_t buf = c & 1u;
        const uint32_t bph = (c >> 1) & 1u;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(qdone(s), sph) &&
                                         ptx::mbar_wait_spin(wfull(s), sph) &&
                                         ptx::mbar_wait_spin(tempty(buf), bph ^ 1u));
        if (!ok) {
          if (lane == 0) record_error(args.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t a_addr = smem_base + SMEM_A_OFF + s * A_BYTES;
          const uint32_t b_addr = smem_base + SMEM_B_OFF + s * B_BYTES;
          const uint32_t d = tmem_base + buf * BN;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k)
            ptx::mma_f8f6f4(d, ptx::sdesc_kmajor_sw128(a_addr + k * UMMA_K),
                            ptx::sdesc_kmajor_sw128(b_addr + k * UMMA_K), IDESC, k > 0 ? 1u : 0u);
          ptx::mma_commit(wempty(s));
          ptx::mma_commit_multicast(aempty(s), CL_MASK);   // A stage s free in every CTA
          ptx::mma_commit(tfull(buf));
        }
        __syncwarp();
        issued = true;
      }
    }
    if (issued && ptx::elect_one()) {
      // All MMAs (and the arrivals their commits make) finish first.
      ptx::mma_commit(drain_bar);
      if (!ptx::mbar_wait(drain_bar, 0)) record_error(args.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else if (warp == 2) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
    // ----------------------------------------------------- slice sender
    // Once this CTA's quantizers have written their rows of chunk c, send
    // the slice (codes and scales) to the other CTAs, counted in bytes on
    // their barriers, and arrive locally expecting the other three slices.
    uint32_t c = 0;
    bool ok = true;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const uint32_t s = c % STAGES;
        const uint32_t slot = c % SA_SLOTS;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait_spin(slice(s), (c / STAGES) & 1u));
        if (!ok) {
          if (lane == 0) record_error(args.err, kErrTimeoutProducer);
          break;
        }
        if (lane == 0) {
          const uint32_t a_src = smem_base + SMEM_A_OFF + s * A_BYTES + rank * SLICE_BYTES;
          const uint32_t s_src = sa_base + (slot * BM + rank * QROWS) * 4u;
          for (uint32_t k = 1; k < CL; ++k) {
            const uint32_t dst = (rank + k) % CL;
            ptx::bulk_copy_s2s(ptx::map_to_cta(a_src, dst), a_src, SLICE_BYTES,
                               ptx::map_to_cta(qdone(s), dst));
            ptx::bulk_copy_s2s(ptx::map_to_cta(s_src, dst), s_src, SCALE_BYTES,
                               ptx::map_to_cta(sfull(slot), dst));
          }
          ptx::mbar_arrive_expect_tx(qdone(s), (CL - 1) * SLICE_BYTES);
          ptx::mbar_arrive_expect_tx(sfull(slot), (CL - 1) * SCALE_BYTES);
        }
        __syncwarp();
      }
    }
  } else if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
  } else if (warp >= FIRST_QUANT_WARP) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;");
    // ---------------------------------------------------------- quantizers
    const int qw = warp - FIRST_QUANT_WARP;
    const uint32_t rl = static_cast<uint32_t>(qw * 8 + (lane >> 2));   // row in this CTA's slice
    const uint32_t part = static_cast<uint32_t>(lane & 3);               // elements 32 part ..
    const uint32_t rt = rank * QROWS + rl;                               // row in the tile
    const uint32_t sw = rl & 7u;          // 128-byte swizzle phase (same for rt: QROWS % 8 == 0)
    const uint32_t box = part >> 1;
    const uint32_t chunk0 = (part & 1u) * 4u;
    uint32_t c = 0;
    bool ok = true;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const uint32_t xs = c % XSLOTS;
        const uint32_t s = c % STAGES;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(xfull(xs), (c / XSLOTS) & 1u))) {
          if (lane == 0) record_error(args.err, kErrTimeoutProducer);
          ok = false;
          break;
        }
        const uint32_t xsrc = smem_base + SMEM_X_OFF + xs * X_BYTES + box * X_BOX_BYTES + rl * 128u;
        uint4 v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = lds128(xsrc + (((chunk0 + i) ^ sw) << 4));
        uint32_t m = absmax_bf16x2(absmax8_bf16x2(v[0]), absmax8_bf16x2(v[1]));
        m = absmax_bf16x2(m, absmax_bf16x2(absmax8_bf16x2(v[2]), absmax8_bf16x2(v[3])));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, 2));
        // The slot goes back to the producer only once every lane's loads have
        // returned (the shuffled amax depends on all of them).  Arriving right
        // after issuing the loads let the next TMA load overwrite the slot
        // under loads still in flight (measured on B200: wrong codes for
        // whole warps of rows in a few runs out of ten).
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(xempty(xs));
        const float scale = scale_from_amax(absmax_halves_f32(m));
        const GroupScale gs = group_scale(scale);
        // codes of elements 32 part .. +31 = 16-byte code chunks 2 part, 2 part + 1
        uint4 code[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint2 lo = quant8(v[2 * t], gs);
          const uint2 hi = quant8(v[2 * t + 1], gs);
          code[t] = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        // A stage s must be free in every CTA of the cluster (chunk c - STAGES done)
        if (c >= STAGES &&
            !__all_sync(0xffffffffu, ptx::mbar_wait_spin(aempty(s), ((c / STAGES) - 1u) & 1u))) {
          if (lane == 0) record_error(args.err, kErrTimeoutProducer);
          ok = false;
          break;
        }
        const uint32_t astage = smem_base + SMEM_A_OFF + s * A_BYTES;
        const uint32_t slot = c % SA_SLOTS;
#pragma unroll
        for (uint32_t t = 0; t < 2; ++t)
          sts128(astage + rt * 128u + (((2u * part + t) ^ sw) << 4), code[t]);
        if (part == 0) sts32(sa_base + (slot * BM + rt) * 4u, __float_as_uint(scale));
        ptx::fence_proxy_async_smem();   // visible to the tensor core and the bulk copies
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(slice(s));
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 176;");
    // ----------------------------------------------------------- promotion
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int nblk_count = N / 128;
    const int r = quarter * 32 + lane;          // row within the tile
    const float* sa_ring = reinterpret_cast<const float*>(smem + SMEM_SA_OFF);
    uint32_t c = 0;
    bool ok = true;
    for (int u = cluster_id; u < num_units && ok; u += num_clusters) {
      int m_blk, g;
      unit_coords(u, num_m, num_g, args.group_m, m_blk, g);
      const int n_blk = g * CL + static_cast<int>(rank);
      const int row = m_blk * BM + r;
      const int nb = n_blk * 2 + half;
      const bool row_ok = row < M;
      const bool col_ok = nb < nblk_count;
      const float* sw_row = args.s_w + static_cast<int64_t>(col_ok ? nb : nblk_count - 1) * num_kb;
      float2 acc[64];
#pragma unroll
      for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
      float sw1 = __ldg(sw_row);
      float sw2 = num_kb > 1 ? __ldg(sw_row + 1) : 0.0f;
      for (int kb = 0; kb < num_kb; ++kb, ++c) {
        const float swc = sw1;
        sw1 = sw2;
        if (kb + 2 < num_kb) sw2 = __ldg(sw_row + kb + 2);
        const uint32_t buf = c & 1u;
        const uint32_t bph = (c >> 1) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tfull(buf), bph) &&
                                         ptx::mbar_wait_spin(sfull(c % SA_SLOTS), (c / SA_SLOTS) & 1u))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        const float scale = sa_ring[(c % SA_SLOTS) * BM + r] * swc;
        const float2 sc2 = make_float2(scale, scale);
        ptx::tc_fence_after();
        const uint32_t tb = tmem_base + lane_off + buf * BN + static_cast<uint32_t>(half * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint32_t v[16];
          ptx::tmem_ld_32x32b_x16(tb + j * 16, v);
          ptx::tmem_ld_wait();
          if (j == 7) {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(tempty(buf));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            acc[j * 8 + i] = __ffma2_rn(make_float2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1])),
                                        sc2, acc[j * 8 + i]);
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

  // No CTA leaves (or frees TMEM) while another CTA of the cluster may still
  // write into its shared memory or arrive on its barriers.
  ptx::tc_fence_before();
  ptx::cluster_sync();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// One-time set-up: opt in to the dynamic shared memory and find how many
// clusters of CL CTAs fit on the device at once.
cudaError_t ensure_fused_ready(int* max_clusters) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  static int clusters_of[kMaxDevices];
  int dev = 0;
  const cudaError_t r = once_per_device(once, status, [](int d) {
    int& clusters = clusters_of[d];
    cudaError_t st = cudaFuncSetAttribute(gemm_fused_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (st != cudaSuccess) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = CL;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    st = cudaOccupancyMaxActiveClusters(&clusters, gemm_fused_kernel, &cfg);
    if (st == cudaSuccess && clusters < 1) st = cudaErrorInvalidConfiguration;
    return st;
  }, &dev);
  *max_clusters = r == cudaSuccess ? clusters_of[dev] : 0;
  return r;
}

}  // namespace

cudaError_t launch_block_linear_fused_tiles(const void* x, const void* q_w, const float* s_w,
                                            void* y, int64_t M, int64_t N, int64_t K,
                                            const DeviceInfo& dev, cudaStream_t st) {
  if (M == 0) return cudaSuccess;
  int max_clusters = 0;
  cudaError_t e = ensure_fused_ready(&max_clusters);
  if (e != cudaSuccess) return e;
  CUtensorMap tx, tb;
  // X as a byte matrix [M, 2K]: boxes of 128 bytes (64 elements) x 32 rows
  if (!make_tmap_u8(&tx, x, M, 2 * K, QROWS, 128) || !make_tmap_u8(&tb, q_w, N, K, BN, BK))
    return cudaErrorInvalidValue;
  FusedArgs a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  // row bands per raster group: their bf16 activations (128 x K x 2 bytes
  // each) fit in ~40 MB of L2
  const int64_t num_m = (M + BM - 1) / BM;
  const int64_t band_bytes = static_cast<int64_t>(BM) * K * 2;
  int64_t gm = (int64_t{40} << 20) / band_bytes;
  gm = gm < 1 ? 1 : (gm > num_m ? num_m : gm);
  a.group_m = static_cast<int>(gm);
  a.err = dev.error_flag;
  const int64_t units = ((M + BM - 1) / BM) * ((((N + BN - 1) / BN) + CL - 1) / CL);
  const int clusters = static_cast<int>(units < max_clusters ? units : max_clusters);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL * clusters, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = CL;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_fused_kernel, tx, tb, a);
}

}  // namespace fp8bl
