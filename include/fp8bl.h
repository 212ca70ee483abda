/*
 * fp8bl -- fine-grained (block-scaled) FP8 linear layers for NVIDIA B200
 * (sm_100a).  C ABI.
 *
 * The method (transformers docs, "Fine-grained FP8" page, opening bullet
 * list, and its "DeepGEMM fast path" section):
 *   - weights are quantized to 8 bits per two-dimensional 128 x 128 block,
 *     one scale per block;
 *   - activations are quantized dynamically (at run time), per token, in
 *     groups of 128 input channels aligned with the weight blocks, one scale
 *     per (token, group);
 *   - the linear layer multiplies the quantized operands and applies both
 *     scale sets per 128-deep block of the input channel.
 * The pages leave the numerics open; this library implements:
 *   - e4m3 = OCP FP8 E4M3 (torch.float8_e4m3fn): max finite 448, NaN = S.1111.111;
 *   - scale s = fp32(max(amax, FP8BL_AMAX_EPS) / 448), amax = max |x| over
 *     the group or block; scales are fp32;
 *   - q = e4m3(fp32(x / s)) with an IEEE-rounded fp32 quotient, then round to
 *     nearest even and saturate to +-448;
 *   - y[m,n] = bf16( sum_j s_a[m,j] * s_w[n/128,j] *
 *                    sum_{k in block j} e4m3val(q_a[m,k]) * e4m3val(q_w[n,k]) )
 *     accumulated in fp32 (fp32 partial per 128-deep block, promoted with
 *     the product of the two scales), rounded once to bf16 (nearest even).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers to caller-owned memory on the current
 *     CUDA device; the library never allocates, frees or keeps them.
 *   - All tensors are dense and row-major (last index fastest).
 *   - Every pointer must be 16-byte aligned (fp32 scale arrays: 4-byte).
 *   - Outputs must not overlap inputs.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream); the call returns before the GPU finishes.
 *   - Argument errors are detected on the host and returned BEFORE any work
 *     is enqueued.  Launch failures return FP8BL_ERR_CUDA.  Kernels whose
 *     internal waits exceed their time limit record an error that
 *     fp8bl_check() reports as FP8BL_ERR_TIMEOUT.
 *   - Results are bit-identical from run to run for the same arguments.
 *   - The device must be compute capability 10.0 (B200 / sm_100a).
 *   - No exceptions cross this interface; all calls are thread-safe as long
 *     as concurrent calls do not share output buffers or workspaces.
 *   - Several devices per process are supported: each kernel's opt-in to
 *     more than 48 KB of shared memory is made once per device (device
 *     ordinals 0 .. 63), at its first launch on that device.
 */
#ifndef FP8BL_H
#define FP8BL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so that this header
 * does not need the CUDA headers. */
typedef struct CUstream_st *fp8bl_stream_t;

typedef enum {
    FP8BL_OK = 0,
    FP8BL_ERR_NULL = 1,      /* a required pointer is NULL                  */
    FP8BL_ERR_SHAPE = 2,     /* sizes out of range / not multiples of 128   */
    FP8BL_ERR_ALIGN = 3,     /* a pointer is not suitably aligned           */
    FP8BL_ERR_ARCH = 4,      /* current device is not sm_100                */
    FP8BL_ERR_CUDA = 5,      /* a CUDA runtime/driver call failed           */
    FP8BL_ERR_TIMEOUT = 6,   /* a kernel wait ran out (see fp8bl_check)     */
    FP8BL_ERR_WORKSPACE = 7, /* workspace smaller than required             */
    FP8BL_ERR_OVERLAP = 8    /* an output buffer overlaps an input buffer   */
} fp8bl_status;

#define FP8BL_BLOCK 128          /* group / block edge along K and N       */
#define FP8BL_E4M3_MAX 448.0f    /* largest finite e4m3 value              */
#define FP8BL_AMAX_EPS 1e-10f    /* amax floor for all-zero groups/blocks  */

/* Largest sizes accepted (TMA coordinates are 32-bit signed). */
#define FP8BL_MAX_DIM ((int64_t)1 << 30)

/*
 * fp8_quant_act -- dynamic per-token activation quantization.
 * Passage: "Fine-grained FP8" page, second bullet of the opening list
 * (per-token groups whose size matches the weight block along the input
 * channel, 128), dynamic scheme per its "DeepGEMM fast path" section.
 *
 *   x_bf16  in : bf16 [M, K] row-major
 *   q_e4m3  out: e4m3 codes [M, K] row-major (1 byte each)
 *   s       out: fp32 [M, K/128] row-major; s[m,g] scales x[m, 128g .. 128g+127]
 *   M >= 0 (M == 0 enqueues nothing), K > 0, K % 128 == 0, M, K <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_quant_act(const void *x_bf16, int64_t M, int64_t K,
                           void *q_e4m3, float *s, fp8bl_stream_t stream);

/*
 * fp8_quant_act_static -- activation quantization with one given scale
 * (the static scheme).
 * Passage: "Fine-grained FP8" page, "DeepGEMM fast path" section (static
 * activation quantization, next to the dynamic scheme; the page says no more).
 * This library reads it as: one fp32 activation scale per linear, supplied
 * by the caller (calibrated elsewhere), q = e4m3(fp32(x / s)) rounded and
 * saturated as above (|x| > 448 s gives +-448), and the product is the block
 * linear with every activation group scale equal to s.  So the call writes
 * s into every slot of the [M, K/128] scale array, and fp8_block_linear /
 * fp8_block_linear_noalloc take the outputs unchanged.
 *
 *   x_bf16  in : bf16 [M, K]          s_given in : device pointer to one fp32,
 *   q_e4m3  out: e4m3 [M, K]                       finite and > 0 (not checked)
 *   s       out: fp32 [M, K/128], every element = *s_given
 *   M >= 0 (M == 0 enqueues nothing), K > 0, K % 128 == 0, M, K <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_quant_act_static(const void *x_bf16, int64_t M, int64_t K,
                                  const float *s_given, void *q_e4m3, float *s,
                                  fp8bl_stream_t stream);

/*
 * fp8_quant_weight -- 128 x 128 block weight quantization.
 * Passage: "Fine-grained FP8" page, first bullet of the opening list
 * (weight_block_size = (128, 128)).
 *
 *   w_bf16  in : bf16 [N, K] row-major (nn.Linear layout: out x in)
 *   q_e4m3  out: e4m3 codes [N, K]
 *   s       out: fp32 [N/128, K/128] row-major; s[i,j] scales the block of
 *                rows 128i.. and columns 128j..
 *   N, K > 0, multiples of 128, <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_quant_weight(const void *w_bf16, int64_t N, int64_t K,
                              void *q_e4m3, float *s, fp8bl_stream_t stream);

/*
 * fp8_block_linear -- block-scaled FP8 linear, y = x W^T with both scale
 * sets applied per 128-deep K block.
 * Passage: "Fine-grained FP8" page, opening bullet list (the two
 * quantization granularities the product must honour) and "DeepGEMM fast
 * path" section (FP8 linear with weight_block_size (128,128) and dynamic
 * activations).
 *
 *   q_a  in : e4m3 [M, K]          (from fp8_quant_act)
 *   s_a  in : fp32 [M, K/128]
 *   q_w  in : e4m3 [N, K]          (from fp8_quant_weight)
 *   s_w  in : fp32 [N/128, K/128]
 *   y_bf16 out: bf16 [M, N]
 *   workspace: device scratch of at least
 *              fp8_block_linear_workspace_bytes(M, N, K) bytes (16-byte
 *              aligned), or NULL when that size is 0.  It needs no
 *              clearing: it starts with a ready flag and a counter per
 *              128-row weight block, through which the CTAs that share a
 *              block hand over their partial sums; a flag counts as set
 *              only when it holds the launch's own 64-bit tag, so leftover
 *              bytes read as "not set", and every completed call leaves the
 *              flags it set cleared (so a CUDA graph may replay calls on
 *              it).  After FP8BL_ERR_TIMEOUT, zero the workspace before a
 *              graph replays calls on it.
 *   M >= 0, N, K > 0 and multiples of 128, all <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_block_linear(const void *q_a, const float *s_a,
                              const void *q_w, const float *s_w,
                              void *y_bf16, int64_t M, int64_t N, int64_t K,
                              void *workspace, size_t workspace_bytes,
                              fp8bl_stream_t stream);

/*
 * fp8_block_linear_fused -- the same linear from bf16 activations in one
 * call: x_bf16 [M, K] is quantized exactly as fp8_quant_act would
 * (bit-identical codes and scales) and multiplied; y equals
 * fp8_quant_act + fp8_block_linear bit for bit.  Two schedules:
 *   - staged (the faster on B200 at every size measured): the codes and
 *     scales are written into the workspace, where they stay in L2 for the
 *     GEMM that follows; needs fp8_block_linear_fused_workspace_bytes(M, N, K)
 *     bytes (M*K + M*K/128*4 plus the decode scratch, each rounded up to
 *     256 bytes);
 *   - in-GEMM (M > 64 only): the GEMM quantizes each activation tile itself
 *     and the codes never reach memory; taken when workspace is NULL or
 *     smaller than that size.
 *   At M <= 64 the workspace is required.
 */
fp8bl_status fp8_block_linear_fused(const void *x_bf16,
                                    const void *q_w, const float *s_w,
                                    void *y_bf16, int64_t M, int64_t N, int64_t K,
                                    void *workspace, size_t workspace_bytes,
                                    fp8bl_stream_t stream);

/*
 * fp8_block_linear_noalloc -- fp8_block_linear for 1 <= M <= 64 tokens
 * (the decode sizes, whose schedule needs scratch memory) using a scratch
 * array built into the library instead of a caller workspace.  The pages
 * have no counterpart: this is an integration convenience.
 *
 * Some callers cannot allocate device memory at the point where they run
 * the layer -- for example a serving loop whose device memory is fully
 * reserved up front by its own pool, code that must avoid the device-wide
 * synchronisation that cudaMalloc / cudaFree can cause, or a host program
 * that only ever hands over the tensors it already owns.  This call lets
 * them run the decode-sized linear with nothing but its inputs and output.
 *
 *   arguments as fp8_block_linear, without the workspace.
 *   The scratch is a FP8BL_NOALLOC_SCRATCH_BYTES array in device memory that
 *   exists on every GPU that loads the library until the process exits.
 *   Shapes whose decode schedule needs more scratch than that return
 *   FP8BL_ERR_WORKSPACE; M > 64 returns FP8BL_ERR_SHAPE (for M > 64,
 *   fp8_block_linear needs no workspace: pass NULL, 0).
 *   The first call on each device looks up the array's device address (a
 *   CUDA runtime query), so make that first call before any stream capture.
 *   All calls on a device share the array and leave its contents behind;
 *   nothing in it needs clearing between calls (its hand-over flags are
 *   tagged per launch, as in fp8_block_linear's workspace).  Calls
 *   whose GPU work may overlap (different streams with no ordering between
 *   them) race on the array and must not be issued.
 *   Neither this call nor the library allocates or frees device memory.
 */
#define FP8BL_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
fp8bl_status fp8_block_linear_noalloc(const void *q_a, const float *s_a,
                                      const void *q_w, const float *s_w,
                                      void *y_bf16, int64_t M, int64_t N, int64_t K,
                                      fp8bl_stream_t stream);

/*
 * UE8M0 (power-of-two) scale variant.
 * Passage: "Fine-grained FP8" page, "UE8M0 scale format" section
 * (DeepSeek-V4-style checkpoints keep FP8 scales as packed float8_e8m0fnu,
 * scale_fmt="ue8m0"; on Blackwell the DeepGEMM expert kernels accept only
 * that format).  The page fixes neither the rounding to a power of two nor a
 * layout; this library implements:
 *   - the scale of a group or block is the smallest power of two 2^e with
 *     max(amax, FP8BL_AMAX_EPS) <= 448 * 2^e (the fp32 scale rounded up);
 *   - it is stored as one byte, the float8_e8m0fnu code e + 127 (value
 *     2^(code - 127)), in the same row-major grids as the fp32 scales:
 *     [M, K/128] for activations, [N/128, K/128] for weights;
 *   - q = e4m3(x * 2^-e): an exact product, then round to nearest even;
 *   - the linear runs on the tensor core's block-scaled MMA, which applies
 *     the two scales per 32-deep slice of K and accumulates the whole K
 *     extent in fp32; y is rounded once to bf16.
 * Codes stay within 85 .. 247 for finite bf16 inputs.  The scale arrays
 * have no alignment requirement; the other rules are those of the fp32
 * calls above.
 */
fp8bl_status fp8_quant_act_ue8m0(const void *x_bf16, int64_t M, int64_t K,
                                 void *q_e4m3, uint8_t *s_ue8m0,
                                 fp8bl_stream_t stream);
fp8bl_status fp8_quant_weight_ue8m0(const void *w_bf16, int64_t N, int64_t K,
                                    void *q_e4m3, uint8_t *s_ue8m0,
                                    fp8bl_stream_t stream);
/*
 *   q_a  in : e4m3 [M, K]              s_a in : ue8m0 codes [M, K/128]
 *   q_w  in : e4m3 [N, K]              s_w in : ue8m0 codes [N/128, K/128]
 *   y_bf16 out: bf16 [M, N]
 *   M >= 0, N, K > 0 and multiples of 128, all <= FP8BL_MAX_DIM.  Scale
 *   codes must be finite (not 255).  No workspace.
 */
fp8bl_status fp8_block_linear_ue8m0(const void *q_a, const uint8_t *s_a,
                                    const void *q_w, const uint8_t *s_w,
                                    void *y_bf16, int64_t M, int64_t N, int64_t K,
                                    fp8bl_stream_t stream);

/*
 * fp8_block_linear_ue8m0_ws -- the same linear with a caller workspace, which
 * lets M > 128 run on CTA pairs (tcgen05.mma.cta_group::2, 256 x 256 tiles):
 * two small kernels first rewrite s_a and s_w into the workspace in the
 * order the tensor core reads scale factors, so that they travel with the
 * operands.  Same passage, arguments and result as fp8_block_linear_ue8m0
 * (bit for bit: the same MMAs in the same K order), plus
 *   workspace: device scratch of at least
 *              fp8_block_linear_ue8m0_workspace_bytes(M, N, K) bytes
 *              (16-byte aligned), or NULL when that size is 0 (M <= 128:
 *              the single-CTA kernel, no workspace).  Contents on entry are
 *              ignored; it must not overlap any argument.
 */
size_t fp8_block_linear_ue8m0_workspace_bytes(int64_t M, int64_t N, int64_t K);
fp8bl_status fp8_block_linear_ue8m0_ws(const void *q_a, const uint8_t *s_a,
                                       const void *q_w, const uint8_t *s_w,
                                       void *y_bf16, int64_t M, int64_t N, int64_t K,
                                       void *workspace, size_t workspace_bytes,
                                       fp8bl_stream_t stream);

/*
 * fp8_grouped_linear_ue8m0 -- grouped (MoE expert) form of
 * fp8_block_linear_ue8m0.
 * Passage: "Fine-grained FP8" page, "DeepGEMM fast path" section (MoE expert
 * matmuls routed through DeepGEMM, experts_implementation="deepgemm" /
 * "deepgemm_megamoe" on Blackwell) and its "UE8M0 scale format" section
 * (on Blackwell the DeepGEMM expert kernels accept only UE8M0 scales).  The
 * pages give no layout; this library takes the plainest one, a contiguous
 * grouping: the M rows of q_a are sorted by expert, expert e owns rows
 * [expert_offsets[e], expert_offsets[e+1]) and multiplies them by its own
 * weights, y[rows of e] = that expert's fp8_block_linear_ue8m0.
 *
 *   q_a  in : e4m3 [M, K]           s_a in : ue8m0 codes [M, K/128]
 *   q_w  in : e4m3 [E, N, K]        s_w in : ue8m0 codes [E, N/128, K/128]
 *   expert_offsets in: DEVICE int32 [E + 1], 0 = off[0] <= off[1] <= ... <= off[E] = M.
 *            The kernel clamps every value to [0, M] and takes a running maximum,
 *            so malformed offsets cannot make it read or write out of bounds;
 *            rows outside [off[0], off[E]) are not written.
 *   y_bf16 out: bf16 [M, N]
 *   1 <= E <= 1024, M >= 0, N, K > 0 and multiples of 128, E * N <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_grouped_linear_ue8m0(const void *q_a, const uint8_t *s_a,
                                      const void *q_w, const uint8_t *s_w,
                                      const int32_t *expert_offsets, void *y_bf16,
                                      int64_t M, int64_t N, int64_t K, int64_t E,
                                      fp8bl_stream_t stream);

/*
 * fp8_grouped_linear_ue8m0_ws -- the same grouped linear with a caller
 * workspace, which lets M > 128 run on CTA pairs (256-row tiles within each
 * expert's segment, as fp8_block_linear_ue8m0_ws): two small kernels first
 * rewrite s_a (every segment padded to a multiple of 256 rows) and s_w (per
 * expert) into the workspace in the order the tensor core reads scale
 * factors.  Same passage, arguments and result as fp8_grouped_linear_ue8m0
 * (bit for bit), plus
 *   workspace: device scratch of at least
 *              fp8_grouped_linear_ue8m0_workspace_bytes(M, N, K, E) bytes
 *              (16-byte aligned), or NULL when that size is 0 (M <= 128:
 *              the single-CTA kernel).  Contents on entry are ignored; it
 *              must not overlap any argument.  The size bounds the padded
 *              segments for any offsets: K/128 * 2 * (ceil(M/256) + E) * 512
 *              bytes for s_a (E > 1) and E * K/128 * 2 * ceil(N/256) * 512
 *              for s_w.
 */
size_t fp8_grouped_linear_ue8m0_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E);
fp8bl_status fp8_grouped_linear_ue8m0_ws(const void *q_a, const uint8_t *s_a,
                                         const void *q_w, const uint8_t *s_w,
                                         const int32_t *expert_offsets, void *y_bf16,
                                         int64_t M, int64_t N, int64_t K, int64_t E,
                                         void *workspace, size_t workspace_bytes,
                                         fp8bl_stream_t stream);

/*
 * Row-wise FP8 variant (fp8r).
 * Passage: "BFL (fp8r / nvfp4)" page of the diffusers docs, first bullet of
 * its list (an E4M3 weight with one fp32 weight scale per row; activations
 * quantized to E4M3 per row at run time) and its "Kernels" table (a scaled
 * matmul with row-wise scales).  The page gives no formula; this library
 * uses the rule of the calls above with one group per row:
 *   s[r] = fp32(max(amax over row r, FP8BL_AMAX_EPS) / 448),
 *   q = e4m3(fp32(x / s[r])),
 *   y[m,n] = bf16(s_a[m] * s_w[n] * sum_k e4m3val(q_a[m,k]) * e4m3val(q_w[n,k])),
 * the sum accumulated in fp32 on the tensor core, the scales applied once.
 *
 * fp8_quant_rowwise -- bf16 [R, K] -> e4m3 [R, K] + fp32 s [R]; serves both
 *   the activations (R = M tokens) and the weights (R = N output channels).
 *   R >= 0 (0 enqueues nothing), K > 0, K % 16 == 0, both <= FP8BL_MAX_DIM.
 */
fp8bl_status fp8_quant_rowwise(const void *x_bf16, int64_t R, int64_t K,
                               void *q_e4m3, float *s, fp8bl_stream_t stream);
/*
 * fp8_linear_rowwise --
 *   q_a in: e4m3 [M, K]   s_a in: fp32 [M]
 *   q_w in: e4m3 [N, K]   s_w in: fp32 [N] (16-byte aligned)
 *   y_bf16 out: bf16 [M, N]
 *   M >= 0, N > 0, K > 0, N % 16 == 0, K % 16 == 0, all <= FP8BL_MAX_DIM.
 *   No workspace.
 */
fp8bl_status fp8_linear_rowwise(const void *q_a, const float *s_a,
                                const void *q_w, const float *s_w,
                                void *y_bf16, int64_t M, int64_t N, int64_t K,
                                fp8bl_stream_t stream);

/* Workspace sizes (bytes) the two linear calls need for these sizes on the
 * current device; 0 when no scratch is needed.  Never fails: invalid sizes
 * return 0 (the linear call then reports the error). */
size_t fp8_block_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);
size_t fp8_block_linear_fused_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Waits for `stream`, then reports (and clears) a kernel wait that ran out
 * on the current device since the last check: FP8BL_ERR_TIMEOUT, else
 * FP8BL_OK (or FP8BL_ERR_CUDA if the synchronisation itself failed). */
fp8bl_status fp8bl_check(fp8bl_stream_t stream);

/*
 * fp8bl_selftest_wait_timeout -- exercises the kernels' failure detection
 * (no counterpart on the pages).  Enqueues on `stream` a one-thread kernel
 * that waits on an mbarrier nothing ever arrives on, with the bounded wait
 * the library's kernels use, limited to `limit_cycles` SM clock cycles
 * (kind 0: the suspending wait, kind 1: the polling wait).  When the limit
 * runs out the kernel records a timeout in the library's error word and
 * returns, so the next fp8bl_check(stream) returns FP8BL_ERR_TIMEOUT (and
 * clears it) and the device stays usable.  No memory is touched besides
 * the error word.
 *   limit_cycles: 1 .. 2^32;  kind: 0 or 1;  otherwise FP8BL_ERR_SHAPE.
 */
fp8bl_status fp8bl_selftest_wait_timeout(uint64_t limit_cycles, int kind,
                                          fp8bl_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char *fp8bl_status_string(fp8bl_status status);

/* Library version as major*10000 + minor*100 + patch. */
int fp8bl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8BL_H */
