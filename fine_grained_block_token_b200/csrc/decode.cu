// Decode-sized block-scaled FP8 linear (M <= 64 tokens) for sm_100a.
//
// "Fine-grained FP8" page: per-token 1 x 128 activation groups, 128 x 128
// weight blocks, both scale sets applied per 128-deep K block.  At decode
// sizes the work is a stream over the weights (N x K bytes), so the kernel
// is shaped for HBM bandwidth rather than for the tensor cores:
//   - swap-AB: Y^T = W X^T.  A 128-row weight tile is the MMA's A operand
//     (M = 128) and the tokens, padded to a multiple of 16, are N; the fp32
//     partial of one 128-deep chunk lands in TMEM as 128 lanes (weight rows)
//     x Mpad columns (tokens).
//   - stream-K: the flattened (weight block, K chunk) space is cut into
//     equal contiguous ranges, one per CTA (one CTA per SM), so every SM
//     streams the same number of weight bytes.  A CTA's range covers the
//     tail of one weight block, whole blocks and the head of another; for
//     each (CTA, block) segment it writes an fp32 partial [Mpad, 128] to the
//     caller's workspace.
//   - reduce: a block that one CTA covers alone is written as bf16 directly.
//     For a shared block, every contributing CTA writes its partial and
//     bumps the block's counter; the last one to arrive sums the block's
//     partials in increasing CTA order (a fixed order: results are
//     bit-identical run to run) and writes bf16 Y[m, n].  The counters live
//     at the head of the workspace and are zeroed (cudaMemsetAsync) before
//     every launch.
// Warps: 0 TMA producer (W tile 128x128 + X tile Mpad x 128 per stage,
// 8 stages), 1 MMA issuer, 2 TMEM owner, 3 idle, 4-7 promotion (one weight
// row per thread, Mpad fp32 accumulators, scale s_w[blk, j] * s_a[m, j]).
// Every mbarrier wait is bounded; on expiry the kernel records an error
// code, drains what it started and exits cleanly.
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "fp8bl_internal.h"
#include "ptx_sm100.cuh"

namespace fp8bl {
namespace {

constexpr int DBM = 128;          // weight rows per block (MMA M)
constexpr int DBK = 128;          // K per chunk (one scale block)
constexpr int MAX_MPAD = 64;
constexpr int DSTAGES = 8;
constexpr int DTBUFS = 4;
constexpr int DUMMA_K = 32;
constexpr int W_BYTES = DBM * DBK;           // 16 KB
constexpr int X_BYTES = MAX_MPAD * DBK;      // 8 KB (box rows = Mpad <= 64)
constexpr int DTMEM_COLS = 256;              // DTBUFS * MAX_MPAD
constexpr int DNUM_THREADS = 256;

constexpr int DSMEM_W_OFF = 0;
constexpr int DSMEM_X_OFF = DSMEM_W_OFF + DSTAGES * W_BYTES;
constexpr int DSMEM_BAR_OFF = DSMEM_X_OFF + DSTAGES * X_BYTES;
constexpr int DNUM_BARS = 2 * DSTAGES + 2 * DTBUFS + 1;
constexpr int DSMEM_MISC_OFF = DSMEM_BAR_OFF + DNUM_BARS * 8;
constexpr int DSMEM_BYTES = DSMEM_MISC_OFF + 16 + 1024;

struct DecodeArgs {
  const float* s_a;       // [M, KB]
  const float* s_w;       // [NB, KB]
  __nv_bfloat16* y;       // [M, N]
  int* counters;          // [NB], zero on entry
  float* partial;         // [G * maxseg, Mpad, 128]
  int N;
  int M, Mpad, KB;
  int64_t units;          // NB * KB
  int G;                  // CTAs
  int maxseg;
  int* err;
};

__device__ __forceinline__ int64_t range_start(int g, int64_t units, int G) {
  return (static_cast<int64_t>(g) * units) / G;
}

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }

template <int MPAD>
__global__ void __launch_bounds__(DNUM_THREADS, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
              const DecodeArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t smem_base = ptx::smem_u32(smem);
  const uint32_t bar_base = smem_base + DSMEM_BAR_OFF;
  auto full_bar = [&](int s) { return bar_base + 8u * s; };
  auto empty_bar = [&](int s) { return bar_base + 8u * (DSTAGES + s); };
  auto tfull_bar = [&](int b) { return bar_base + 8u * (2 * DSTAGES + b); };
  auto tempty_bar = [&](int b) { return bar_base + 8u * (2 * DSTAGES + DTBUFS + b); };
  const uint32_t drain_bar = bar_base + 8u * (2 * DSTAGES + 2 * DTBUFS);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + DSMEM_MISC_OFF);
  constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(DBM, MPAD);
  constexpr uint32_t STAGE_TX = W_BYTES + MPAD * DBK;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int KB = args.KB;
  const int64_t u_begin = range_start(g, args.units, args.G);
  const int64_t u_end = range_start(g + 1, args.units, args.G);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < DSTAGES; ++s) {
      ptx::mbar_init(full_bar(s), 1);
      ptx::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < DTBUFS; ++b) {
      ptx::mbar_init(tfull_bar(b), 1);
      ptx::mbar_init(tempty_bar(b), 4);
    }
    ptx::mbar_init(drain_bar, 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_holder), DTMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    {
      uint32_t issued_mask = 0, phase_mask = 0;
      uint32_t c = 0;
      int blk = static_cast<int>(u_begin / KB);
      int kb = static_cast<int>(u_begin - static_cast<int64_t>(blk) * KB);
      for (int64_t u = u_begin; u < u_end; ++u, ++c, (++kb == KB ? (kb = 0, ++blk) : 0)) {
        const int s = c % DSTAGES;
        const uint32_t ph = (c / DSTAGES) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(empty_bar(s), ph ^ 1u))) {
          if (lane == 0) record_error(args.err, kErrTimeoutProducer);
          break;
        }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(full_bar(s), STAGE_TX);
          ptx::tma_load_2d(smem_base + DSMEM_W_OFF + s * W_BYTES, &tmap_w, full_bar(s), kb * DBK,
                           blk * DBM);
          ptx::tma_load_2d(smem_base + DSMEM_X_OFF + s * X_BYTES, &tmap_x, full_bar(s), kb * DBK, 0);
        }
        __syncwarp();
        issued_mask |= 1u << s;
        phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
      }
      if (lane == 0)
        for (int s = 0; s < DSTAGES; ++s)
          if (((issued_mask >> s) & 1u) && !ptx::mbar_wait(full_bar(s), (phase_mask >> s) & 1u))
            record_error(args.err, kErrTimeoutProducer);
      __syncwarp();
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // The whole warp runs the loop (the wait results are made warp-uniform
    // with a vote) and lane 0 issues: measured on B200, a loop run by lane 0
    // alone with a data-dependent exit costs ~600 cycles per chunk.
    {
      uint32_t c = 0;
      bool issued = false;
      for (int64_t u = u_begin; u < u_end; ++u, ++c) {
        const int s = c % DSTAGES;
        const uint32_t sph = (c / DSTAGES) & 1u;
        const int buf = c % DTBUFS;
        const uint32_t bph = (c / DTBUFS) & 1u;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(tempty_bar(buf), bph ^ 1u) &&
                                         ptx::mbar_wait_spin(full_bar(s), sph))) {
          if (lane == 0) record_error(args.err, kErrTimeoutMma);
          break;
        }
        ptx::tc_fence_after();
        if (lane == 0) {
          const uint32_t w_addr = smem_base + DSMEM_W_OFF + s * W_BYTES;
          const uint32_t x_addr = smem_base + DSMEM_X_OFF + s * X_BYTES;
          const uint32_t d = tmem_base + static_cast<uint32_t>(buf * MAX_MPAD);
#pragma unroll
          for (int k = 0; k < DBK / DUMMA_K; ++k)
            ptx::mma_f8f6f4(d, ptx::sdesc_kmajor_sw128(w_addr + k * DUMMA_K),
                            ptx::sdesc_kmajor_sw128(x_addr + k * DUMMA_K), IDESC, k > 0 ? 1u : 0u);
          ptx::mma_commit(tfull_bar(buf));
          ptx::mma_commit(empty_bar(s));
        }
        __syncwarp();
        issued = true;
      }
      if (issued && lane == 0) {
        ptx::mma_commit(drain_bar);
        if (!ptx::mbar_wait(drain_bar, 0)) record_error(args.err, kErrTimeoutMma);
      }
      __syncwarp();
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- promotion
    const int quarter = warp & 3;
    const int n_local = quarter * 32 + lane;          // weight row within the block
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int first_blk = static_cast<int>(u_begin / KB);
    float acc[MPAD];
#pragma unroll
    for (int m = 0; m < MPAD; ++m) acc[m] = 0.0f;
    uint32_t c = 0;
    bool ok = true;

    // Scales of chunk u: s_w[blk, kb] and the activation scales of tokens
    // `lane` and `lane + 32`.  They are loaded PF chunks ahead into slot
    // (u - u_begin) % PF; the loop is unrolled PF times so every slot index
    // is a compile-time constant and a slot is refilled right after its use
    // (no register shuffling that would stall on the loads).
    constexpr int PF = 4;
    float pw[PF], plo[PF], phi[PF];
    auto load_scales = [&](int64_t uu, float& w, float& lo, float& hi) {
      if (uu < u_end) {
        const int b = static_cast<int>(uu / KB);
        const int k = static_cast<int>(uu - static_cast<int64_t>(b) * KB);
        w = __ldg(args.s_w + static_cast<int64_t>(b) * KB + k);
        lo = lane < args.M ? __ldg(args.s_a + static_cast<int64_t>(lane) * KB + k) : 0.0f;
        hi = (MPAD > 32 && lane + 32 < args.M)
                 ? __ldg(args.s_a + static_cast<int64_t>(lane + 32) * KB + k)
                 : 0.0f;
      }
    };
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      pw[i] = plo[i] = phi[i] = 0.0f;
      load_scales(u_begin + i, pw[i], plo[i], phi[i]);
    }

    int blk = first_blk;
    int kb = static_cast<int>(u_begin - static_cast<int64_t>(first_blk) * KB) - 1;
    for (int64_t u0 = u_begin; u0 < u_end; u0 += PF) {
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int64_t u = u0 + i;
        if (u >= u_end) break;
        if (++kb == KB) {
          kb = 0;
          ++blk;
        }
        const float sw = pw[i], sa_lo = plo[i], sa_hi = phi[i];
        load_scales(u + PF, pw[i], plo[i], phi[i]);
        const int buf = c % DTBUFS;
        const uint32_t bph = (c / DTBUFS) & 1u;
        ++c;
        // After a timed-out wait this warp stops touching TMEM but keeps
        // walking its range, so that every named barrier below is reached
        // by all four promotion warps.
        if (ok && !ptx::mbar_wait_spin(tfull_bar(buf), bph)) {
          record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
        }
        if (ok) {
          ptx::tc_fence_after();
          uint32_t v[MPAD];
#pragma unroll
          for (int j = 0; j < MPAD / 16; ++j)
            ptx::tmem_ld_32x32b_x16(
                tmem_base + lane_off + static_cast<uint32_t>(buf * MAX_MPAD + j * 16),
                *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
          ptx::tmem_ld_wait();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(tempty_bar(buf));
#pragma unroll
          for (int m = 0; m < MPAD; ++m) {
            const float sa = __shfl_sync(0xffffffffu, m < 32 ? sa_lo : sa_hi, m & 31);
            acc[m] = __fmaf_rn(__uint_as_float(v[m]), sw * sa, acc[m]);
          }
        }
        if (kb == KB - 1 || u + 1 == u_end) {
          // end of this block's segment
          const int64_t blk_u0 = static_cast<int64_t>(blk) * KB;
          const int64_t y_off = static_cast<int64_t>(blk) * 128 + n_local;
          if (blk_u0 >= u_begin && kb == KB - 1) {
            // the whole block was accumulated by this CTA: write bf16 directly
#pragma unroll
            for (int m = 0; m < MPAD; ++m)
              if (m < args.M) args.y[static_cast<int64_t>(m) * args.N + y_off] = __float2bfloat16_rn(acc[m]);
          } else {
            float* dst = args.partial +
                         (static_cast<int64_t>(g) * args.maxseg + (blk - first_blk)) * (MPAD * 128);
#pragma unroll
            for (int m = 0; m < MPAD; ++m) dst[m * 128 + n_local] = acc[m];
            // publish the partial and count this CTA in; the last one reduces.
            // The barrier orders every thread's stores before one thread's
            // fence + atomic (the fence is cumulative), as a grid-wide
            // barrier does; the last CTA fences again before reading.
            ptx::named_barrier_sync(1, 128);
            __shared__ int last_flag;
            const int g_lo = static_cast<int>(((blk_u0 + 1) * args.G - 1) / args.units);
            const int g_hi = static_cast<int>(((blk_u0 + KB) * args.G - 1) / args.units);
            if (threadIdx.x == 128) {
              __threadfence();
              last_flag = atomicAdd(args.counters + blk, 1) == g_hi - g_lo;
              if (last_flag) __threadfence();
            }
            ptx::named_barrier_sync(1, 128);
            if (last_flag) {
              // sum the block's partials in increasing CTA order; the loads
              // of UR partials are in flight together
              constexpr int UR = MPAD <= 16 ? 4 : (MPAD <= 32 ? 2 : 1);
#pragma unroll
              for (int m = 0; m < MPAD; ++m) acc[m] = 0.0f;
              for (int gg = g_lo; gg <= g_hi; gg += UR) {
                float t[UR][MPAD];
#pragma unroll
                for (int r = 0; r < UR; ++r) {
                  const int gi = gg + r <= g_hi ? gg + r : g_hi;
                  const int fb = static_cast<int>(range_start(gi, args.units, args.G) / KB);
                  const float* src = args.partial +
                                     (static_cast<int64_t>(gi) * args.maxseg + (blk - fb)) * (MPAD * 128) +
                                     n_local;
#pragma unroll
                  for (int m = 0; m < MPAD; ++m) t[r][m] = __ldcg(src + m * 128);
                }
#pragma unroll
                for (int r = 0; r < UR; ++r)
                  if (gg + r <= g_hi) {
#pragma unroll
                    for (int m = 0; m < MPAD; ++m) acc[m] += t[r][m];
                  }
              }
#pragma unroll
              for (int m = 0; m < MPAD; ++m)
                if (m < args.M) args.y[static_cast<int64_t>(m) * args.N + y_off] = __float2bfloat16_rn(acc[m]);
            }
          }
#pragma unroll
          for (int m = 0; m < MPAD; ++m) acc[m] = 0.0f;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, DTMEM_COLS);
  }
}

struct DecodeGeometry {
  int Mpad, G, maxseg;
  int64_t units;
};

DecodeGeometry decode_geometry(int64_t M, int64_t N, int64_t K, int sm_count) {
  DecodeGeometry d;
  d.Mpad = static_cast<int>(((M + 15) / 16) * 16);
  const int64_t NB = N / 128, KB = K / 128;
  d.units = NB * KB;
  // at least ceil(KB / 8) chunks per CTA: no block gathers partials from
  // more than about 9 CTAs
  const int64_t min_chunks = (KB + 7) / 8;
  const int64_t g_cap = d.units / min_chunks > 0 ? d.units / min_chunks : 1;
  d.G = static_cast<int>(g_cap < sm_count ? g_cap : sm_count);
  // a range of ceil(units / G) units touches at most this many blocks
  const int64_t span = (d.units + d.G - 1) / d.G;
  d.maxseg = static_cast<int>((span + KB - 1) / KB + 1);
  return d;
}

template <int MPAD>
cudaError_t launch_decode_t(const CUtensorMap& tw, const CUtensorMap& tx, const DecodeArgs& a,
                            cudaStream_t st) {
  static cudaError_t attr = cudaFuncSetAttribute(
      decode_kernel<MPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize, DSMEM_BYTES);
  if (attr != cudaSuccess) return attr;
  decode_kernel<MPAD><<<a.G, DNUM_THREADS, DSMEM_BYTES, st>>>(tw, tx, a);
  return cudaGetLastError();
}

}  // namespace

// Workspace: NB block counters (rounded up to 256 bytes), then the partials.
size_t decode_counter_bytes(int64_t N) { return static_cast<size_t>(((N / 128) * 4 + 255) / 256 * 256); }

size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count) {
  const DecodeGeometry d = decode_geometry(M, N, K, sm_count);
  return decode_counter_bytes(N) + static_cast<size_t>(d.G) * d.maxseg * d.Mpad * 128 * sizeof(float);
}

cudaError_t launch_block_linear_decode(const void* q_a, const float* s_a, const void* q_w,
                                       const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                       void* workspace, const DeviceInfo& dev, cudaStream_t st) {
  const DecodeGeometry d = decode_geometry(M, N, K, dev.sm_count);
  CUtensorMap tw, tx;
  if (!make_tmap_u8(&tw, q_w, N, K, DBM, DBK) ||
      !make_tmap_u8(&tx, q_a, M, K, static_cast<uint32_t>(d.Mpad), DBK))
    return cudaErrorInvalidValue;
  DecodeArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.counters = static_cast<int*>(workspace);
  a.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + decode_counter_bytes(N));
  a.N = static_cast<int>(N);
  a.M = static_cast<int>(M);
  a.Mpad = d.Mpad;
  a.KB = static_cast<int>(K / 128);
  a.units = d.units;
  a.G = d.G;
  a.maxseg = d.maxseg;
  a.err = dev.error_flag;
  cudaError_t e = cudaMemsetAsync(workspace, 0, decode_counter_bytes(N), st);
  if (e != cudaSuccess) return e;
  switch (d.Mpad) {
    case 16: return launch_decode_t<16>(tw, tx, a, st);
    case 32: return launch_decode_t<32>(tw, tx, a, st);
    case 48: return launch_decode_t<48>(tw, tx, a, st);
    case 64: return launch_decode_t<64>(tw, tx, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fp8bl
