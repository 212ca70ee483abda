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
//     counts itself in on the block's counter (one atomic add); the last one
//     to arrive sums the block's partials in increasing CTA order (a fixed
//     order: results are bit-identical run to run) and writes bf16 Y[m, n].
//     The counter is set to zero at the start of the launch by the CTA that
//     holds the block's first chunk, which then stores the launch's 64-bit
//     tag in the block's ready flag; the other contributors wait for that
//     flag before they count in, and the last one clears it.  A flag counts
//     as set only when it holds this launch's tag, so the workspace needs no
//     clearing (leftover bytes, other shapes' partials), and since a
//     completed launch leaves the flags it used cleared, a CUDA graph can
//     replay its launches with the tags they were captured with.
// Warps: 0 TMA producer (W tile 128x128 + X tile Mpad x 128 per stage,
// 8 stages), 1 MMA issuer, 2 TMEM owner and counter set-up, 3 scale
// products (for every chunk the Mpad factors s_w[blk, j] * s_a[m, j], once
// per CTA, into a shared ring), 4-11 promotion: two warps per TMEM lane
// quarter, one weight row per thread, each warp a contiguous part of the
// token columns.  Every warp polls its barriers without suspending
// (mbarrier.test_wait): with suspending waits the weight stream of the large
// linears ran 5-10% slower on B200.
// The kernel is launched with programmatic stream serialization: its set-up
// (barriers, TMEM, tensor-map prefetch) and an L2 prefetch of the weight
// tiles its first ring fill loads overlap the previous kernel's tail, when
// most of that kernel's CTAs have left and HBM would idle; it waits for the
// previous kernel to finish before its first access to anything another
// kernel can write.  Every wait is bounded; on expiry the kernel records an
// error code, drains what it started and exits cleanly.
#include <algorithm>
#include <atomic>
#include <chrono>
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
constexpr int DTBUFS = 4;
constexpr int DUMMA_K = 32;
constexpr int CSLOTS = 16;                   // ring of per-chunk scale products
constexpr int W_BYTES = DBM * DBK;           // 16 KB
constexpr int DTMEM_COLS = 256;              // DTBUFS * MAX_MPAD
constexpr int DNUM_THREADS = 384;
constexpr int PROMO_THREADS = 256;           // warps 4-11
constexpr int kSmemBudget = 227 * 1024;

// Shared-memory layout for Mpad tokens: 8 stages of [W tile 16 KB | X tile
// Mpad x 128 B] (measured on B200: 9-12 stages streamed no faster and
// slightly slower at Mpad 16), then the scale-product ring, the barriers and
// a few words.
template <int MPAD>
struct DLayout {
  static constexpr int SB = W_BYTES + MPAD * DBK;            // stage bytes, multiple of 1024
  static constexpr int FIXED = CSLOTS * MAX_MPAD * 4 + (2 * DTBUFS + 2 * CSLOTS + 1) * 8 + 16 + 1024;
  static constexpr int NS_FIT = (kSmemBudget - FIXED) / (SB + 16);
  static constexpr int NS = NS_FIT < 8 ? NS_FIT : 8;         // stages
  static constexpr int C_OFF = NS * SB;
  static constexpr int BAR_OFF = C_OFF + CSLOTS * MAX_MPAD * 4;
  static constexpr int NUM_BARS = 2 * NS + 2 * DTBUFS + 2 * CSLOTS + 1;
  static constexpr int MISC_OFF = BAR_OFF + NUM_BARS * 8;
  static constexpr int BYTES = MISC_OFF + 16 + 1024;         // + slack for 1024-byte alignment
  static_assert(BYTES <= kSmemBudget, "shared memory budget");
  static_assert(SB % 1024 == 0, "stage alignment");
  // barrier indices
  static __device__ __forceinline__ int full(int s) { return s; }
  static __device__ __forceinline__ int empty(int s) { return NS + s; }
  static __device__ __forceinline__ int tfull(int b) { return 2 * NS + b; }
  static __device__ __forceinline__ int tempty(int b) { return 2 * NS + DTBUFS + b; }
  static __device__ __forceinline__ int cfull(int i) { return 2 * NS + 2 * DTBUFS + i; }
  static __device__ __forceinline__ int cempty(int i) { return 2 * NS + 2 * DTBUFS + CSLOTS + i; }
  static __device__ __forceinline__ int drain() { return 2 * NS + 2 * DTBUFS + 2 * CSLOTS; }
  static __device__ __forceinline__ uint32_t bar(uint32_t smem_base, int i) {
    return smem_base + BAR_OFF + 8u * i;
  }
};

// misc words in shared memory
constexpr int kMiscTmem = 0;       // TMEM base address
constexpr int kMiscLast = 1;       // "this CTA reduces the block" flag
constexpr int kMiscReady = 2;      // first block's counter usable: 0 not yet, 1 yes, 2 gave up
constexpr int kMiscPending = 3;    // the first block, published by warp 2, is left to reduce

struct DecodeArgs {
  const float* s_a;                 // [M, KB]
  const float* s_w;                 // [NB, KB]
  __nv_bfloat16* y;                 // [M, N]
  unsigned long long* flags;        // [NB] ready flags (the launch's tag when set)
  unsigned int* counters;           // [NB] arrival counters
  float* partial;                   // [G * maxseg, Mpad, 128]
  unsigned long long tag;           // this launch's tag, never zero
  int64_t units;                    // NB * KB
  int N, M, KB;
  int G;                            // CTAs
  int maxseg;
  int* err;
};

// a / b for a >= 0, b > 0, by a 32-bit division when a fits in 32 bits
// (always, for the sizes a decode meets; the 64-bit division is a long
// software sequence on the reduction's critical path).
__device__ __forceinline__ int64_t div_nonneg(int64_t a, int64_t b) {
  if ((static_cast<uint64_t>(a) | static_cast<uint64_t>(b)) <= 0xffffffffull)
    return static_cast<uint32_t>(a) / static_cast<uint32_t>(b);
  return a / b;
}

__device__ __forceinline__ int64_t range_start(int g, int64_t units, int G) {
  return div_nonneg(static_cast<int64_t>(g) * units, G);
}

__device__ __forceinline__ void record_error(int* err, int code) { atomicCAS(err, 0, code); }


// Partial of contributor gi for block blk: segment 0 of CTA gi, except for
// the block's first contributor g_lo, whose range may start in an earlier
// block (segment seg_lo).
template <int MPAD>
__device__ __forceinline__ const float* partial_of(const DecodeArgs& args, int gi, int g_lo,
                                                   int seg_lo) {
  return args.partial +
         (static_cast<int64_t>(gi) * args.maxseg + (gi == g_lo ? seg_lo : 0)) * (MPAD * 128);
}

// Contributors of block blk: the CTAs whose ranges hold its chunks.
__device__ __forceinline__ void block_contributors(const DecodeArgs& args, int blk, int& g_lo,
                                                   int& g_hi) {
  const int64_t blk_u0 = static_cast<int64_t>(blk) * args.KB;
  g_lo = static_cast<int>(div_nonneg((blk_u0 + 1) * args.G - 1, args.units));
  g_hi = static_cast<int>(div_nonneg((blk_u0 + args.KB) * args.G - 1, args.units));
}

struct PromoCtx {
  uint32_t smem_base, tmem_base;
  const float* prods;       // shared ring [CSLOTS][MAX_MPAD]
  volatile int* misc;       // shared misc words
  int64_t u_begin, u_end;
  int g, quarter, lane;
  bool async_first;         // warp 2 publishes the first segment (see below)
};


template <int MPAD>
__device__ __forceinline__ void reduce_block_promo(const DecodeArgs& args, int blk, int g_lo, int g_hi);

// End of the range inside a shared block: publish this CTA's partial and
// count it in; the last contributor reduces the block with the 256
// promotion threads.
template <int MPAD>
__device__ __forceinline__ void publish_at_range_end(const DecodeArgs& args, const PromoCtx& cx,
                                                     int blk) {
  // Publish the partial and count this CTA in; the last one reduces.
  // The barrier orders every thread's stores before one thread's
  // acquire-release atomic (a release covers what the barrier ordered
  // before it); the last CTA's acquire makes the other partials
  // visible, and the second barrier orders its threads' reads after it.
  ptx::named_barrier_sync(1, PROMO_THREADS);
  int g_lo, g_hi;
  block_contributors(args, blk, g_lo, g_hi);
  if (threadIdx.x == 128) {
    // the block's counter must have been set up for this launch (by
    // this CTA's warp 2, or by the CTA holding the block's first chunk)
    const uint64_t t0 = clock64();
    while (cx.misc[kMiscReady] == 0 && clock64() - t0 < (1ull << 32)) __nanosleep(32);
    bool last = false;
    if (cx.misc[kMiscReady] == 1) {
      last = ptx::atomic_add_acq_rel_gpu(args.counters + blk, 1u) ==
             static_cast<unsigned>(g_hi - g_lo);
      if (last) {
        // every contributor has counted in: the flag is free again
        // (the launch's end orders this store before the next launch)
        *reinterpret_cast<volatile unsigned long long*>(args.flags + blk) = 0ull;
      }
    } else {
      record_error(args.err, kErrTimeoutEpilogue);
    }
    cx.misc[kMiscLast] = last ? 1 : 0;
  }
  ptx::named_barrier_sync(1, PROMO_THREADS);
  if (cx.misc[kMiscLast]) reduce_block_promo<MPAD>(args, blk, g_lo, g_hi);
}

// Sum block blk's partials in increasing CTA order with the 256 promotion
// threads: thread t sums row t % 128, token columns (t / 128) * MPAD / 2 ..
// + MPAD / 2 - 1; the loads of UR partials (all of them for the usual
// contributor counts) are in flight together.
template <int MPAD>
__device__ __forceinline__ void reduce_block_promo(const DecodeArgs& args, int blk, int g_lo, int g_hi) {
  const int KB = args.KB;
  constexpr int HALF = MPAD / 2;
  constexpr int UR = HALF <= 8 ? 8 : (HALF <= 16 ? 4 : 2);
  const int t = threadIdx.x - 128;
  const int rn = t & 127;
  const int64_t yo = static_cast<int64_t>(blk) * 128 + rn;
  const int seg_lo =
      blk - static_cast<int>(div_nonneg(range_start(g_lo, args.units, args.G), KB));
  auto part = [&](int gi) { return partial_of<MPAD>(args, gi, g_lo, seg_lo); };
  if (args.M <= 2) {
    // one or two tokens: thread t sums row t % 128 of token t / 128,
    // with up to 16 partials' loads in flight (same order, same sums)
    constexpr int URS = 16;
    const int m = t >> 7;
    if (m < args.M) {
      float acc1 = 0.0f;
      for (int gg = g_lo; gg <= g_hi; gg += URS) {
        float tv[URS];
#pragma unroll
        for (int r = 0; r < URS; ++r) {
          const int gi = gg + r <= g_hi ? gg + r : g_hi;
          tv[r] = __ldcg(part(gi) + m * 128 + rn);
        }
#pragma unroll
        for (int r = 0; r < URS; ++r)
          if (gg + r <= g_hi) acc1 += tv[r];
      }
      args.y[static_cast<int64_t>(m) * args.N + yo] = __float2bfloat16_rn(acc1);
    }
  } else {
    const int m0 = (t >> 7) * HALF;
    float sum[HALF];
#pragma unroll
    for (int m = 0; m < HALF; ++m) sum[m] = 0.0f;
    for (int gg = g_lo; gg <= g_hi; gg += UR) {
      float tv[UR][HALF];
#pragma unroll
      for (int r = 0; r < UR; ++r) {
        const int gi = gg + r <= g_hi ? gg + r : g_hi;
        const float* src = part(gi) + m0 * 128 + rn;
#pragma unroll
        for (int m = 0; m < HALF; ++m) tv[r][m] = m0 + m < args.M ? __ldcg(src + m * 128) : 0.0f;
      }
#pragma unroll
      for (int r = 0; r < UR; ++r)
        if (gg + r <= g_hi) {
#pragma unroll
          for (int m = 0; m < HALF; ++m) sum[m] += tv[r][m];
        }
    }
#pragma unroll
    for (int m = 0; m < HALF; ++m)
      if (m0 + m < args.M)
        args.y[static_cast<int64_t>(m0 + m) * args.N + yo] = __float2bfloat16_rn(sum[m]);
  }
}

// Promotion by one warp: token columns COL0 .. COL0 + NC - 1 of its lane
// quarter's 32 weight rows (NC = 0: the warp only takes part in the
// block-end barriers and reductions).  acc[m] += partial[m] * (s_w * s_a[m])
// with the product read from the shared ring.  All eight promotion warps
// walk the same chunks and reach the same named barriers in the same order;
// after a timed-out wait a warp stops touching TMEM and the ring but keeps
// walking.
template <int MPAD, int NC, int COL0>
__device__ __forceinline__ void decode_promote(const DecodeArgs& args, const PromoCtx& cx) {
  using L = DLayout<MPAD>;
  const int lane = cx.lane;
  const int n_local = cx.quarter * 32 + lane;   // weight row within the block
  const uint32_t lane_off = static_cast<uint32_t>(cx.quarter * 32) << 16;
  const int KB = args.KB;
  const int first_blk = static_cast<int>(cx.u_begin / KB);
  constexpr int NA = NC > 0 ? NC : 1;
  float acc[NA];
#pragma unroll
  for (int m = 0; m < NA; ++m) acc[m] = 0.0f;
  uint32_t c = 0;
  bool ok = true;
  int blk = first_blk;
  int kb = static_cast<int>(cx.u_begin - static_cast<int64_t>(first_blk) * KB) - 1;
  for (int64_t u = cx.u_begin; u < cx.u_end; ++u, ++c) {
    if (++kb == KB) {
      kb = 0;
      ++blk;
    }
    const int buf = c % DTBUFS;
    const uint32_t bph = (c / DTBUFS) & 1u;
    const int slot = c % CSLOTS;
    const uint32_t cph = (c / CSLOTS) & 1u;
    if (NC > 0 && ok) {
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(L::bar(cx.smem_base, L::tfull(buf)), bph))) {
        if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
        ok = false;
      } else {
        ptx::tc_fence_after();
        uint32_t v[NA];
#pragma unroll
        for (int j = 0; j < NC / 16; ++j)
          ptx::tmem_ld_32x32b_x16(
              cx.tmem_base + lane_off + static_cast<uint32_t>(buf * MAX_MPAD + COL0 + j * 16),
              *reinterpret_cast<uint32_t(*)[16]>(&v[j * 16]));
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(L::bar(cx.smem_base, L::tempty(buf)));
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(L::bar(cx.smem_base, L::cfull(slot)), cph))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
        } else {
          const float4* cr = reinterpret_cast<const float4*>(cx.prods + slot * MAX_MPAD + COL0);
#pragma unroll
          for (int j = 0; j < NC / 4; ++j) {
            const float4 p = cr[j];
            // packed f32x2 FMAs: each lane an IEEE fma, as fmaf would give
            const float2 lo = __ffma2_rn(
                make_float2(__uint_as_float(v[4 * j + 0]), __uint_as_float(v[4 * j + 1])),
                make_float2(p.x, p.y), make_float2(acc[4 * j + 0], acc[4 * j + 1]));
            const float2 hi = __ffma2_rn(
                make_float2(__uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])),
                make_float2(p.z, p.w), make_float2(acc[4 * j + 2], acc[4 * j + 3]));
            acc[4 * j + 0] = lo.x;
            acc[4 * j + 1] = lo.y;
            acc[4 * j + 2] = hi.x;
            acc[4 * j + 3] = hi.y;
          }
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(L::bar(cx.smem_base, L::cempty(slot)));
        }
      }
    }
    if (kb == KB - 1 || u + 1 == cx.u_end) {
      // end of this block's segment
      const int64_t blk_u0 = static_cast<int64_t>(blk) * KB;
      const int64_t y_off = static_cast<int64_t>(blk) * 128 + n_local;
      if (blk_u0 >= cx.u_begin && kb == KB - 1) {
        // the whole block was accumulated by this CTA: write bf16 directly
#pragma unroll
        for (int m = 0; m < NC; ++m)
          if (COL0 + m < args.M)
            args.y[static_cast<int64_t>(COL0 + m) * args.N + y_off] = __float2bfloat16_rn(acc[m]);
      } else {
        float* dst = args.partial +
                     (static_cast<int64_t>(cx.g) * args.maxseg + (blk - first_blk)) * (MPAD * 128);
#pragma unroll
        for (int m = 0; m < NC; ++m)
          if (COL0 + m < args.M) dst[(COL0 + m) * 128 + n_local] = acc[m];
        if (u + 1 < cx.u_end) {
          // The range goes on into the next block (this is its first
          // segment, the tail of a block): warp 2 publishes the partial and
          // reduces the block if it arrives last, while the promotion warps
          // go on with the next chunks.
          ptx::named_barrier_arrive(2, PROMO_THREADS + 32);
        } else {
          publish_at_range_end<MPAD>(args, cx, blk);
        }
      }
#pragma unroll
      for (int m = 0; m < NA; ++m) acc[m] = 0.0f;
    }
  }
  if (cx.async_first) {
    // Warp 2 published the first segment; if that made this CTA the block's
    // last contributor, the block is reduced here, by all 256 threads.
    ptx::named_barrier_sync(3, PROMO_THREADS + 32);
    if (cx.misc[kMiscPending]) {
      int g_lo, g_hi;
      block_contributors(args, first_blk, g_lo, g_hi);
      reduce_block_promo<MPAD>(args, first_blk, g_lo, g_hi);
    }
  }
}

template <int MPAD>
__global__ void __launch_bounds__(DNUM_THREADS, 1)
decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
              const DecodeArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  using L = DLayout<MPAD>;
  constexpr int NS = L::NS;
  const uint32_t smem_base = ptx::smem_u32(smem);
  auto bar = [&](int i) { return L::bar(smem_base, i); };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* vmisc = reinterpret_cast<volatile int*>(misc);
  float* prods = reinterpret_cast<float*>(smem + L::C_OFF);
  constexpr uint32_t IDESC = ptx::idesc_e4m3_f32(DBM, MPAD);
  constexpr uint32_t STAGE_TX = W_BYTES + MPAD * DBK;
  // token columns per promotion half: half 0 takes NC0, half 1 the rest
  constexpr int NC0 = MPAD <= 32 ? 16 : 32;
  constexpr int NC1 = MPAD - NC0;
  constexpr int LOADERS = NC1 > 0 ? 8 : 4;     // promotion warps that read TMEM

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = blockIdx.x;
  const int KB = args.KB;
  const int64_t u_begin = range_start(g, args.units, args.G);
  const int64_t u_end = range_start(g + 1, args.units, args.G);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(bar(L::full(s)), 1);
      ptx::mbar_init(bar(L::empty(s)), 1);
    }
    for (int b = 0; b < DTBUFS; ++b) {
      ptx::mbar_init(bar(L::tfull(b)), 1);
      ptx::mbar_init(bar(L::tempty(b)), LOADERS);
    }
    for (int i = 0; i < CSLOTS; ++i) {
      ptx::mbar_init(bar(L::cfull(i)), 32);
      ptx::mbar_init(bar(L::cempty(i)), LOADERS);
    }
    ptx::mbar_init(bar(L::drain()), 1);
    ptx::fence_barrier_init();
    ptx::prefetch_tmap(&tmap_w);
    ptx::prefetch_tmap(&tmap_x);
    vmisc[kMiscLast] = 0;
    vmisc[kMiscReady] = 0;
    vmisc[kMiscPending] = 0;
    // Warm the L2 with this CTA's first weight tiles while the previous
    // kernel may still run (a prefetch only; the loads below come after the
    // wait, and a later write by the previous kernel would update L2).
    int blk = static_cast<int>(u_begin / KB);
    int kb = static_cast<int>(u_begin - static_cast<int64_t>(blk) * KB);
    for (int64_t u = u_begin; u < u_end && u < u_begin + NS;
         ++u, (++kb == KB ? (kb = 0, ++blk) : 0))
      ptx::tma_prefetch_2d(&tmap_w, kb * DBK, blk * DBM);
  }
  if (warp == 2) {
    ptx::tmem_alloc(ptx::smem_u32(misc + kMiscTmem), DTMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = vmisc[kMiscTmem];
  // From here on the kernel reads what earlier kernels wrote (activation
  // codes and scales) and writes what they may read (Y, the workspace).
  ptx::grid_dep_wait();
  if (threadIdx.x == 0) ptx::grid_dep_launch();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t issued_mask = 0, phase_mask = 0;
    uint32_t c = 0;
    int blk = static_cast<int>(u_begin / KB);
    int kb = static_cast<int>(u_begin - static_cast<int64_t>(blk) * KB);
    for (int64_t u = u_begin; u < u_end; ++u, ++c, (++kb == KB ? (kb = 0, ++blk) : 0)) {
      const int s = c % NS;
      const uint32_t ph = (c / NS) & 1u;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(bar(L::empty(s)), ph ^ 1u))) {
        if (lane == 0) record_error(args.err, kErrTimeoutProducer);
        break;
      }
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar(L::full(s)), STAGE_TX);
        ptx::tma_load_2d(smem_base + s * L::SB, &tmap_w, bar(L::full(s)), kb * DBK, blk * DBM);
        ptx::tma_load_2d(smem_base + s * L::SB + W_BYTES, &tmap_x, bar(L::full(s)), kb * DBK, 0);
      }
      __syncwarp();
      issued_mask |= 1u << s;
      phase_mask = (phase_mask & ~(1u << s)) | (ph << s);
    }
    // every load issued lands before the CTA may exit
    if (lane == 0)
      for (int s = 0; s < NS; ++s)
        if (((issued_mask >> s) & 1u) && !ptx::mbar_wait(bar(L::full(s)), (phase_mask >> s) & 1u))
          record_error(args.err, kErrTimeoutProducer);
    __syncwarp();
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    // The whole warp runs the loop (the wait results are made warp-uniform
    // with a vote) and an elected lane issues.  Measured on B200 (cycle
    // counters per chunk): a loop run by lane 0 alone with a data-dependent
    // exit cost ~600 cycles; issuing the 4 MMAs from a `lane == 0` branch
    // took ~270 cycles against ~25 from an elect.sync block, which moved the
    // gate+up stream from ~1,050 to ~800 cycles per chunk.
    const uint64_t desc0 = ptx::sdesc_kmajor_sw128(smem_base);
    uint32_t c = 0;
    bool issued = false;
    for (int64_t u = u_begin; u < u_end; ++u, ++c) {
      const int s = c % NS;
      const uint32_t sph = (c / NS) & 1u;
      const int buf = c % DTBUFS;
      const uint32_t bph = (c / DTBUFS) & 1u;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(bar(L::tempty(buf)), bph ^ 1u) &&
                                       ptx::mbar_wait_spin(bar(L::full(s)), sph))) {
        if (lane == 0) record_error(args.err, kErrTimeoutMma);
        break;
      }
      ptx::tc_fence_after();
      const uint64_t dw = ptx::sdesc_advance(desc0, s * L::SB);
      const uint64_t dx = ptx::sdesc_advance(dw, W_BYTES);
      const uint32_t d = tmem_base + static_cast<uint32_t>(buf * MAX_MPAD);
      if (ptx::elect_one()) {
#pragma unroll
        for (int k = 0; k < DBK / DUMMA_K; ++k)
          ptx::mma_f8f6f4(d, ptx::sdesc_advance(dw, k * DUMMA_K), ptx::sdesc_advance(dx, k * DUMMA_K),
                          IDESC, k > 0 ? 1u : 0u);
        ptx::mma_commit(bar(L::tfull(buf)));
        ptx::mma_commit(bar(L::empty(s)));
      }
      issued = true;
    }
    if (issued && ptx::elect_one()) {
      ptx::mma_commit(bar(L::drain()));
      if (!ptx::mbar_wait(bar(L::drain()), 0)) record_error(args.err, kErrTimeoutMma);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------- counter set-up
    // Zero the counters of the shared blocks whose first chunk lies in this
    // CTA's range, then mark them ready with the launch's tag; if this CTA's
    // range starts inside a block, wait until that block's first CTA has
    // done the same for it.
    if (lane == 0) {
      const int64_t b_lo = (u_begin + KB - 1) / KB, b_hi = (u_end - 1) / KB;
      for (int64_t b = b_lo; b <= b_hi; ++b)
        if (((b * KB + KB) * args.G - 1) / args.units > ((b * KB + 1) * args.G - 1) / args.units)
          args.counters[b] = 0u;
      __threadfence();
      for (int64_t b = b_lo; b <= b_hi; ++b)
        if (((b * KB + KB) * args.G - 1) / args.units > ((b * KB + 1) * args.G - 1) / args.units)
          *reinterpret_cast<volatile unsigned long long*>(args.flags + b) = args.tag;
      int ready = 1;
      if (u_begin % KB != 0) {
        const volatile unsigned long long* f =
            reinterpret_cast<const volatile unsigned long long*>(args.flags + u_begin / KB);
        const uint64_t t0 = clock64();
        while (*f != args.tag) {
          if (clock64() - t0 > (1ull << 32)) {
            ready = 2;
            break;
          }
          __nanosleep(64);
        }
        __threadfence();
      }
      vmisc[kMiscReady] = ready;
    }
    __syncwarp();
    const int b0 = static_cast<int>(u_begin / KB);
    if (u_begin % KB != 0 && static_cast<int64_t>(b0 + 1) * KB < u_end) {
      // The range starts inside block b0 and goes on past it: once the
      // promotion warps have stored b0's partial (named barrier 2), count
      // this CTA in and, if it is the last contributor, reduce b0 here.
      ptx::named_barrier_sync(2, PROMO_THREADS + 32);
      int g_lo, g_hi;
      block_contributors(args, b0, g_lo, g_hi);
      if (lane == 0) {
        int last = 0;
        if (vmisc[kMiscReady] == 1) {
          last = ptx::atomic_add_acq_rel_gpu(args.counters + b0, 1u) ==
                 static_cast<unsigned>(g_hi - g_lo);
          if (last) *reinterpret_cast<volatile unsigned long long*>(args.flags + b0) = 0ull;
        } else {
          record_error(args.err, kErrTimeoutEpilogue);
        }
        vmisc[kMiscPending] = last;
      }
      // The promotion warps reduce the block at the end of their range
      // (named barrier 3 orders this acquire and the flag before them).
      __syncwarp();
      ptx::named_barrier_arrive(3, PROMO_THREADS + 32);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------ scale products
    // prods[slot][m] = s_w[blk, kb] * s_a[m, kb] for every chunk of the
    // range, up to CSLOTS chunks ahead of the promotion warps.  Lane l
    // covers tokens l and l + 32.  The scales of a chunk are loaded PF
    // chunks ahead (L2 path: another kernel wrote them) into a register
    // slot that is refilled right after its use.  s_w of unit u is s_w[u]
    // (row-major [NB, KB]).
    constexpr int PF = 4;
    float pw[PF], plo[PF], phi[PF];
    auto load_scales = [&](int64_t uu, float& w, float& lo, float& hi) {
      w = lo = hi = 0.0f;
      if (uu < u_end) {
        const int k = static_cast<int>(uu % KB);
        w = __ldcg(args.s_w + uu);
        if (lane < args.M) lo = __ldcg(args.s_a + static_cast<int64_t>(lane) * KB + k);
        if (MPAD > 32 && lane + 32 < args.M)
          hi = __ldcg(args.s_a + static_cast<int64_t>(lane + 32) * KB + k);
      }
    };
#pragma unroll
    for (int i = 0; i < PF; ++i) load_scales(u_begin + i, pw[i], plo[i], phi[i]);
    uint32_t c = 0;
    bool ok = true;
    for (int64_t u0 = u_begin; u0 < u_end && ok; u0 += PF) {
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int64_t u = u0 + i;
        if (u >= u_end) break;
        const float cw = pw[i], clo = plo[i], chi = phi[i];
        load_scales(u + PF, pw[i], plo[i], phi[i]);
        const int slot = c % CSLOTS;
        const uint32_t ph = (c / CSLOTS) & 1u;
        ++c;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_spin(bar(L::cempty(slot)), ph ^ 1u))) {
          if (lane == 0) record_error(args.err, kErrTimeoutEpilogue);
          ok = false;
          break;
        }
        float* cr = prods + slot * MAX_MPAD;
        cr[lane] = cw * clo;
        if (MPAD > 32) cr[32 + lane] = cw * chi;
        ptx::mbar_arrive(bar(L::cfull(slot)));
      }
    }
  } else if (warp >= 4) {
    // ----------------------------------------------------------- promotion
    PromoCtx cx;
    cx.smem_base = smem_base;
    cx.tmem_base = tmem_base;
    cx.prods = prods;
    cx.misc = vmisc;
    cx.u_begin = u_begin;
    cx.u_end = u_end;
    cx.g = g;
    cx.quarter = warp & 3;
    cx.lane = lane;
    cx.async_first = u_begin % KB != 0 && (u_begin / KB + 1) * KB < u_end;
    if (warp < 8)
      decode_promote<MPAD, NC0, 0>(args, cx);
    else
      decode_promote<MPAD, NC1, NC0>(args, cx);
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
  // Prefer ranges that tile the weight blocks exactly (c chunks per CTA, c
  // a divisor of KB): no range then crosses a block boundary and every
  // block has exactly KB / c contributors.  Taken when it keeps at least
  // 85 % of the CTAs the plain split would use; measured on B200 this cut
  // the 4096 x 4096 decode linear from 18.3 to 13.0 us at 64 tokens (128
  // CTAs of 8 chunks instead of 148 of ~7) and left 4096 x 14336 as fast.
  const int64_t c_min = std::max(min_chunks, (d.units + sm_count - 1) / sm_count);
  for (int64_t c = c_min; c <= KB; ++c) {
    if (KB % c != 0) continue;
    if ((d.units / c) * 100 >= static_cast<int64_t>(d.G) * 85) d.G = static_cast<int>(d.units / c);
    break;
  }
  // a range of ceil(units / G) units touches at most this many blocks
  const int64_t span = (d.units + d.G - 1) / d.G;
  d.maxseg = static_cast<int>((span + KB - 1) / KB + 1);
  return d;
}

// Tag of one launch: a per-process random start advanced by an odd constant
// per launch, never zero (a cleared flag).  A graph replays its launches
// with their tags; that is sound because every launch that completes
// leaves the ready flags it set cleared.
unsigned long long next_launch_tag() {
  static std::atomic<unsigned long long> seq{0};
  static const unsigned long long salt = [] {
    unsigned long long x = static_cast<unsigned long long>(
        std::chrono::high_resolution_clock::now().time_since_epoch().count());
    x ^= reinterpret_cast<uintptr_t>(&seq) * 0x9E3779B97F4A7C15ull;
    x ^= x >> 29;
    x *= 0xBF58476D1CE4E5B9ull;
    x ^= x >> 32;
    return x;
  }();
  const unsigned long long t =
      salt + 0x9E3779B97F4A7C15ull * (seq.fetch_add(1, std::memory_order_relaxed) + 1);
  return t ? t : 1ull;
}

template <int MPAD>
cudaError_t launch_decode_t(const CUtensorMap& tw, const CUtensorMap& tx, const DecodeArgs& a,
                            cudaStream_t st) {
  static std::once_flag once[kMaxDevices];
  static cudaError_t status[kMaxDevices];
  const cudaError_t attr = once_per_device(once, status, [](int) {
    return cudaFuncSetAttribute(decode_kernel<MPAD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                DLayout<MPAD>::BYTES);
  });
  if (attr != cudaSuccess) return attr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.G), 1, 1);
  cfg.blockDim = dim3(DNUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = DLayout<MPAD>::BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  set_programmatic_serialization(at[0]);
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<MPAD>, tw, tx, a);
}

}  // namespace

// Workspace: the ready flags [NB] (64-bit) and the counters [NB] (32-bit),
// rounded up to 256 bytes, then the partials.
namespace {
size_t flag_bytes(int64_t N) { return static_cast<size_t>(((N / 128) * 12 + 255) / 256 * 256); }
}  // namespace

size_t decode_workspace_bytes(int64_t M, int64_t N, int64_t K, int sm_count) {
  const DecodeGeometry d = decode_geometry(M, N, K, sm_count);
  return flag_bytes(N) + static_cast<size_t>(d.G) * d.maxseg * d.Mpad * 128 * sizeof(float);
}

cudaError_t launch_block_linear_decode(const void* q_a, const float* s_a, const void* q_w,
                                       const float* s_w, void* y, int64_t M, int64_t N, int64_t K,
                                       void* workspace, const DeviceInfo& dev, cudaStream_t st) {
  const DecodeGeometry d = decode_geometry(M, N, K, dev.sm_count);
  CUtensorMap tw, tx;
  if (!make_tmap_u8(&tw, q_w, N, K, DBM, DBK) ||
      !make_tmap_u8(&tx, q_a, M, K, static_cast<uint32_t>(d.Mpad), DBK))
    return cudaErrorInvalidValue;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  DecodeArgs a;
  a.s_a = s_a;
  a.s_w = s_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.flags = reinterpret_cast<unsigned long long*>(ws);
  a.counters = reinterpret_cast<unsigned int*>(ws + (N / 128) * 8);
  a.partial = reinterpret_cast<float*>(ws + flag_bytes(N));
  a.tag = next_launch_tag();
  a.units = d.units;
  a.N = static_cast<int>(N);
  a.M = static_cast<int>(M);
  a.KB = static_cast<int>(K / 128);
  a.G = d.G;
  a.maxseg = d.maxseg;
  a.err = dev.error_flag;
  switch (d.Mpad) {
    case 16: return launch_decode_t<16>(tw, tx, a, st);
    case 32: return launch_decode_t<32>(tw, tx, a, st);
    case 48: return launch_decode_t<48>(tw, tx, a, st);
    case 64: return launch_decode_t<64>(tw, tx, a, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fp8bl
