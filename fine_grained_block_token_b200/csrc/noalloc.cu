// fp8_block_linear_noalloc: the decode-sized block-scaled FP8 linear
// (M <= 64) with its scratch memory built into the library, for callers
// that cannot allocate device memory where they run the layer.
//
// The decode schedule needs scratch: per-block counters and fp32 partial
// results of the CTAs that share a weight block.  fp8_block_linear takes
// that scratch from the caller.  This entry point uses a fixed array that
// the library itself defines as a file-scope __device__ variable, so
// neither the caller nor the library allocates anything at call time.
// The array exists on every device that loads the library, from module
// load until the process exits.
//
// Host code must not use the array's name as a device address (on the host
// it names a stand-in object): the device address is fetched with
// cudaGetSymbolAddress on the first call made while a device is current,
// and cached once the lookup has succeeded (a failed lookup is retried by
// the next call).  Because that set-up runs a CUDA runtime query, the first
// call on each device should come before any stream capture.
//
// Every call on a device shares the same array and leaves its contents
// behind.  Nothing needs clearing between calls: the decode schedule's
// hand-over flags count as set only when they hold the launch's own tag,
// and a completed launch leaves the flags it used cleared.  Two calls whose
// GPU
// work overlaps -- on different streams without ordering between them --
// race on the array.
#include <cstdint>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/fp8bl.h"
#include "fp8bl_internal.h"

namespace fp8bl {

// FP8BL_NOALLOC_SCRATCH_BYTES (16 MiB): enough for every decode shape of
// the Llama-3-8B and DeepSeek-V3 linears at up to 64 tokens on a 148-SM
// device.
constexpr size_t kNoAllocScratchBytes = FP8BL_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

void* g_scratch_dev_ptr[kMaxDevices];
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device.  The first
// call per device looks it up; only a successful lookup is cached, so a
// failed one (for instance a call made while a stream capture forbids the
// query) is retried on the next call instead of failing for good.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_dev_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      *out = nullptr;
      return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
    }
    g_scratch_dev_ptr[dev] = p;
  }
  *out = g_scratch_dev_ptr[dev];
  return cudaSuccess;
}

bool is_aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace fp8bl

using namespace fp8bl;

extern "C" fp8bl_status fp8_block_linear_noalloc(const void* q_a, const float* s_a,
                                                 const void* q_w, const float* s_w, void* y_bf16,
                                                 int64_t M, int64_t N, int64_t K,
                                                 fp8bl_stream_t stream) {
  if (M < 1 || M > kDecodeMaxM || N <= 0 || K <= 0 || N > FP8BL_MAX_DIM || K > FP8BL_MAX_DIM ||
      N % FP8BL_BLOCK || K % FP8BL_BLOCK)
    return FP8BL_ERR_SHAPE;
  if (!q_a || !s_a || !q_w || !s_w || !y_bf16) return FP8BL_ERR_NULL;
  if (!is_aligned(q_a, 16) || !is_aligned(q_w, 16) || !is_aligned(y_bf16, 16) ||
      !is_aligned(s_a, 4) || !is_aligned(s_w, 4))
    return FP8BL_ERR_ALIGN;
  const size_t ny = static_cast<size_t>(M * N) * 2;
  if (ranges_overlap(y_bf16, ny, q_a, static_cast<size_t>(M * K)) ||
      ranges_overlap(y_bf16, ny, q_w, static_cast<size_t>(N * K)) ||
      ranges_overlap(y_bf16, ny, s_a, static_cast<size_t>(M * (K / 128)) * 4) ||
      ranges_overlap(y_bf16, ny, s_w, static_cast<size_t>((N / 128) * (K / 128)) * 4))
    return FP8BL_ERR_OVERLAP;
  const DeviceInfo* d = device_info();
  if (!d) return FP8BL_ERR_CUDA;
  if (d->major != 10 || d->minor != 0) return FP8BL_ERR_ARCH;
  if (d->device < 0 || d->device >= kMaxDevices) return FP8BL_ERR_CUDA;
  // the built-in scratch must hold what this shape needs
  if (decode_workspace_bytes(M, N, K, d->sm_count) > kNoAllocScratchBytes)
    return FP8BL_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(d->device, &scratch) != cudaSuccess || !scratch) return FP8BL_ERR_CUDA;
  const cudaError_t e = launch_block_linear_decode(q_a, s_a, q_w, s_w, y_bf16, M, N, K, scratch, *d,
                                                   reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP8BL_OK : FP8BL_ERR_CUDA;
}
