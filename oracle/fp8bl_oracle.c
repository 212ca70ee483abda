/*
 * CPU oracle for fine-grained (block-scaled) FP8 linear layers.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA library; the two meet only in the seeded input
 * generators.
 *
 * What it computes (transformers docs, "Fine-grained FP8" page, opening
 * bullet list):
 *   - weights are quantized to 8 bits per two-dimensional block of
 *     128 x 128 (weight_block_size = (128, 128));
 *   - activations are quantized to 8 bits per token in groups whose size
 *     matches the weight block along the input channel (128).
 * The "DeepGEMM fast path" section of the same page fixes the dynamic
 * activation scheme (scales computed at run time from the activations).
 *
 * The pages do not print the scale formula, rounding, eps or output type.
 * The readings used here (each also listed with its reason in the design
 * notes):
 *   R1  e4m3 is the OCP FP8 E4M3 ("fn") format: bias 7, 3 mantissa bits,
 *       subnormals, no infinities, S.1111.111 is NaN, max finite 448.
 *   R2  encode = round to nearest, ties to the even code, saturating at
 *       +-448 (Inf saturates too), sign kept (negative underflow -> 0x80).
 *   R3  scale s = RN32(max(amax, EPS) / 448) with EPS = 1e-10f; one fp32
 *       scale per (token, 128-group) and per 128 x 128 weight block.
 *   R4  q = encode(RN32(x / s)): IEEE fp32 division, then the e4m3 rounding
 *       (two roundings, the order a GPU computes it in).
 *   R5  GEMM: y[m,n] = sum_j s_a[m,j] * s_w[n/128,j] * B_j[m,n] with
 *       B_j = sum over the 128 k of block j of dec(q_a[m,k]) * dec(q_w[n,k]),
 *       all in fp64.  B_j is exact in fp64: every product is an integer
 *       multiple of 2^-18 below 2^18, so a 128-term sum needs < 44 bits.
 *
 * Parity pins live in the test suite: the e4m3 decode against two library
 * casts, encode against a brute-force nearest-value search over all 2^32
 * fp32 bit patterns, quantization invariants, and the GEMM against
 * exact-rational brute force on tiny shapes.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_BLOCK 128
#define OR_E4M3_MAX 448.0f
#define OR_AMAX_EPS 1e-10f

/* ---------------------------------------------------------------- e4m3 */

/* R1: value of an e4m3 code, from the format definition.
 * exponent field 0 -> subnormal m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7);
 * S.1111.111 -> NaN. */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* R2: e4m3 code of an fp32 value.
 * Inside a binade [2^E, 2^(E+1)) (E >= -6) the e4m3 grid has spacing
 * 2^(E-3); below 2^-6 the subnormal grid keeps the spacing 2^-9.  The value
 * is divided by the spacing (exact: a power of two), rounded to the nearest
 * integer with ties to even, and the integer is turned into exponent and
 * mantissa fields.  An even integer is an even mantissa code, so this is
 * the "ties to the even code" rule. */
uint8_t oracle_e4m3_encode(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, sizeof bits);
    uint8_t sign = (bits >> 31) ? 0x80 : 0x00;
    if (isnan(v))
        return sign | 0x7F;
    double a = fabs((double)v);
    if (a >= 448.0)                 /* saturate, Inf included */
        return sign | 0x7E;
    int E;
    if (a == 0.0) {
        E = -6;
    } else {
        int ex;
        frexp(a, &ex);              /* a = f * 2^ex, f in [0.5, 1) */
        E = ex - 1;                 /* a in [2^E, 2^(E+1)) */
        if (E < -6)
            E = -6;
    }
    double spacing = ldexp(1.0, E - 3);
    double n = a / spacing;         /* exact */
    double fl = floor(n);
    double frac = n - fl;
    if (frac > 0.5 || (frac == 0.5 && fmod(fl, 2.0) != 0.0))
        fl += 1.0;
    int ni = (int)fl;               /* 0 .. 16 */
    if (E == -6 && ni < 8)          /* subnormal (or zero) */
        return sign | (uint8_t)ni;
    if (ni == 16) {                 /* rounded up into the next binade */
        E += 1;
        ni = 8;
    }
    int efield = E + 7;
    int mfield = ni - 8;
    if (efield > 15 || (efield == 15 && mfield == 7))
        return sign | 0x7E;         /* not reachable for a < 448 */
    return sign | (uint8_t)((efield << 3) | mfield);
}

/* bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits. */
static float bf16_to_f32(uint16_t h)
{
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, sizeof f);
    return f;
}

/* R3 + R4 for one group of values with a known amax. */
static float scale_from_amax(float amax)
{
    float a = amax > OR_AMAX_EPS ? amax : OR_AMAX_EPS;
    return a / OR_E4M3_MAX;         /* IEEE fp32 division */
}

/* --------------------------------------------------------- quantizers */

/* Activation quantization (dynamic, per token, 1 x 128 groups).
 * x: bf16 [M, K] row-major; q: e4m3 [M, K]; s: fp32 [M, K/128].
 * Rows m0 .. m1-1 are processed. */
void oracle_quant_act_rows(const uint16_t *x, int64_t M, int64_t K,
                           uint8_t *q, float *s, int64_t m0, int64_t m1)
{
    (void)M;
    int64_t G = K / OR_BLOCK;
    for (int64_t m = m0; m < m1; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *xg = x + m * K + g * OR_BLOCK;
            float amax = 0.0f;
            for (int i = 0; i < OR_BLOCK; ++i) {
                float a = fabsf(bf16_to_f32(xg[i]));
                if (a > amax)
                    amax = a;
            }
            float sc = scale_from_amax(amax);
            s[m * G + g] = sc;
            for (int i = 0; i < OR_BLOCK; ++i)
                q[m * K + g * OR_BLOCK + i] =
                    oracle_e4m3_encode(bf16_to_f32(xg[i]) / sc);
        }
    }
}

/* Weight quantization, one scale per 128 x 128 block.
 * w: bf16 [N, K] row-major; q: e4m3 [N, K]; s: fp32 [N/128, K/128]. */
void oracle_quant_weight(const uint16_t *w, int64_t N, int64_t K,
                         uint8_t *q, float *s)
{
    int64_t NB = N / OR_BLOCK, KB = K / OR_BLOCK;
    for (int64_t bi = 0; bi < NB; ++bi) {
        for (int64_t bj = 0; bj < KB; ++bj) {
            float amax = 0.0f;
            for (int r = 0; r < OR_BLOCK; ++r)
                for (int c = 0; c < OR_BLOCK; ++c) {
                    float a = fabsf(bf16_to_f32(
                        w[(bi * OR_BLOCK + r) * K + bj * OR_BLOCK + c]));
                    if (a > amax)
                        amax = a;
                }
            float sc = scale_from_amax(amax);
            s[bi * KB + bj] = sc;
            for (int r = 0; r < OR_BLOCK; ++r)
                for (int c = 0; c < OR_BLOCK; ++c) {
                    int64_t idx = (bi * OR_BLOCK + r) * K + bj * OR_BLOCK + c;
                    q[idx] = oracle_e4m3_encode(bf16_to_f32(w[idx]) / sc);
                }
        }
    }
}

/* ------------------------------------------------- UE8M0 scale variant
 *
 * "Fine-grained FP8" page, "UE8M0 scale format" section: DeepSeek-V4-style
 * checkpoints keep the FP8 weight scales as packed float8_e8m0fnu values
 * instead of float32 (scale_fmt="ue8m0"), and on Blackwell the DeepGEMM
 * expert kernels accept only these.  The section gives neither how a scale
 * becomes a power of two nor a layout.  Readings used here:
 *   R11  a ue8m0 code c is an unsigned biased exponent: value 2^(c - 127),
 *       c = 255 is NaN (the float8_e8m0fnu format); no sign, no zero.
 *   R12  the scale of a group or block is the smallest power of two
 *       s = 2^e with max(amax, EPS) <= 448 * s, i.e. the fp32 scale of R3
 *       rounded UP to a power of two, so the largest element still maps
 *       inside +-448 and nothing saturates; stored as c = e + 127, one byte
 *       per scale, in the same [M, K/128] and [N/128, K/128] grids.
 *   R13  q = encode(RN32(x * 2^-e)): the product is exact in fp64 and is
 *       rounded once to fp32 (the only rounding besides the e4m3 one; it
 *       matters only when x * 2^-e underflows fp32, where e4m3 gives 0).
 *   The GEMM is R5 with s = 2^(c - 127).
 */

/* R11 */
double oracle_ue8m0_decode(uint8_t c)
{
    if (c == 255)
        return NAN;
    return ldexp(1.0, (int)c - 127);
}

/* R12: the least e with a <= 448 * 2^e, found by exact comparisons
 * (448 * 2^e is exact in fp64, and so is the fp32 amax). */
uint8_t oracle_ue8m0_from_amax(float amax)
{
    double a = amax > OR_AMAX_EPS ? (double)amax : (double)OR_AMAX_EPS;
    int e;
    frexp(a / 448.0, &e);                   /* starting guess */
    while (ldexp(448.0, e - 1) >= a)
        --e;
    while (ldexp(448.0, e) < a)
        ++e;
    return (uint8_t)(e + 127);
}

/* R13 for one value, given the group's code c. */
static uint8_t encode_pow2(float x, uint8_t c)
{
    double v = (double)x * ldexp(1.0, 127 - (int)c);   /* exact */
    return oracle_e4m3_encode((float)v);
}

/* Activation quantization with UE8M0 scales, rows m0 .. m1-1.
 * x: bf16 [M, K]; q: e4m3 [M, K]; s: ue8m0 codes [M, K/128]. */
void oracle_quant_act_ue8m0_rows(const uint16_t *x, int64_t M, int64_t K,
                                 uint8_t *q, uint8_t *s, int64_t m0, int64_t m1)
{
    (void)M;
    int64_t G = K / OR_BLOCK;
    for (int64_t m = m0; m < m1; ++m) {
        for (int64_t g = 0; g < G; ++g) {
            const uint16_t *xg = x + m * K + g * OR_BLOCK;
            float amax = 0.0f;
            for (int i = 0; i < OR_BLOCK; ++i) {
                float a = fabsf(bf16_to_f32(xg[i]));
                if (a > amax)
                    amax = a;
            }
            uint8_t c = oracle_ue8m0_from_amax(amax);
            s[m * G + g] = c;
            for (int i = 0; i < OR_BLOCK; ++i)
                q[m * K + g * OR_BLOCK + i] = encode_pow2(bf16_to_f32(xg[i]), c);
        }
    }
}

/* Weight quantization with UE8M0 scales, one per 128 x 128 block.
 * w: bf16 [N, K]; q: e4m3 [N, K]; s: ue8m0 codes [N/128, K/128]. */
void oracle_quant_weight_ue8m0(const uint16_t *w, int64_t N, int64_t K,
                               uint8_t *q, uint8_t *s)
{
    int64_t NB = N / OR_BLOCK, KB = K / OR_BLOCK;
    for (int64_t bi = 0; bi < NB; ++bi) {
        for (int64_t bj = 0; bj < KB; ++bj) {
            float amax = 0.0f;
            for (int r = 0; r < OR_BLOCK; ++r)
                for (int c = 0; c < OR_BLOCK; ++c) {
                    float a = fabsf(bf16_to_f32(
                        w[(bi * OR_BLOCK + r) * K + bj * OR_BLOCK + c]));
                    if (a > amax)
                        amax = a;
                }
            uint8_t code = oracle_ue8m0_from_amax(amax);
            s[bi * KB + bj] = code;
            for (int r = 0; r < OR_BLOCK; ++r)
                for (int c = 0; c < OR_BLOCK; ++c) {
                    int64_t idx = (bi * OR_BLOCK + r) * K + bj * OR_BLOCK + c;
                    q[idx] = encode_pow2(bf16_to_f32(w[idx]), code);
                }
        }
    }
}

/* ------------------------------------------------- row-wise FP8 (fp8r)
 *
 * "BFL (fp8r / nvfp4)" page, first bullet of its list: each quantized
 * linear keeps an E4M3 weight and one fp32 weight scale per row, and the
 * activations are quantized to E4M3 per row at run time; its "Kernels"
 * table runs the product as a scaled matmul with row-wise scales.  The page
 * gives no scale formula; the readings of R3/R4 carry over with one group
 * per row:
 *   R14  s[r] = RN32(max(amax over row r, EPS) / 448), q = encode(RN32(x / s[r]))
 *        for activation rows (tokens) and weight rows (output channels);
 *   R15  y[m,n] = s_a[m] * s_w[n] * sum over all k of dec(q_a[m,k]) * dec(q_w[n,k]),
 *        in fp64 (the sum is exact: integer multiples of 2^-18 below 2^18,
 *        at most 2^17 terms, < 53 bits).
 */

/* R14 for rows r0 .. r1-1 of a bf16 [R, K] matrix; s: fp32 [R]. */
void oracle_quant_rowwise_rows(const uint16_t *x, int64_t K, uint8_t *q,
                               float *s, int64_t r0, int64_t r1)
{
    for (int64_t r = r0; r < r1; ++r) {
        const uint16_t *xr = x + r * K;
        float amax = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_f32(xr[k]));
            if (a > amax)
                amax = a;
        }
        float sc = scale_from_amax(amax);
        s[r] = sc;
        for (int64_t k = 0; k < K; ++k)
            q[r * K + k] = oracle_e4m3_encode(bf16_to_f32(xr[k]) / sc);
    }
}

/* R15 for the output rows listed in rows[0 .. nrows-1]; y fp64 [nrows, N]. */
int oracle_linear_rowwise_rows(const uint8_t *qa, const float *sa,
                               const uint8_t *qw, const float *sw,
                               int64_t N, int64_t K,
                               const int64_t *rows, int64_t nrows, double *y)
{
    double dec[256];
    for (int c = 0; c < 256; ++c)
        dec[c] = oracle_e4m3_decode((uint8_t)c);
    double *arow = (double *)malloc((size_t)K * sizeof(double));
    if (!arow)
        return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t m = rows[r];
        for (int64_t k = 0; k < K; ++k)
            arow[k] = dec[qa[m * K + k]];
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t *wr = qw + n * K;
            double b = 0.0;
            for (int64_t k = 0; k < K; ++k)
                b += arow[k] * dec[wr[k]];
            y[r * N + n] = (double)sa[m] * (double)sw[n] * b;
        }
    }
    free(arow);
    return 0;
}

/* ------------------------------------------- static activation scale
 *
 * "Fine-grained FP8" page, "DeepGEMM fast path" section: next to the
 * dynamic scheme there is static activation quantization (it always runs on
 * the Triton path); the page says nothing more about it.  Reading:
 *   R16  a static scheme has one given fp32 activation scale s per linear
 *        (calibrated elsewhere): q = encode(RN32(x / s)), saturating by R2
 *        for |x| > 448 s, and the linear is R5 with every s_a[m,j] = s.
 */
void oracle_quant_act_static(const uint16_t *x, int64_t M, int64_t K, float s,
                             uint8_t *q, float *sa)
{
    int64_t G = K / OR_BLOCK;
    for (int64_t i = 0; i < M * K; ++i)
        q[i] = oracle_e4m3_encode(bf16_to_f32(x[i]) / s);
    for (int64_t i = 0; i < M * G; ++i)
        sa[i] = s;
}

/* ----------------------------------------------------------------- GEMM */

/* R5 for the output rows listed in rows[0 .. nrows-1] (all N columns).
 * y: fp64 [nrows, N].  Operands are decoded to fp64 first (exact). */
typedef struct {
    const uint8_t *qa;
    const float *sa;
    const uint8_t *qw;
    const float *sw;
    int64_t N, K;
    const int64_t *rows;
    int64_t r0, r1;
    const double *dec;   /* 256-entry decode table */
    const double *wdec;  /* decoded weights [N, K] */
    double *y;
} gemm_job;

static void *gemm_rows(void *arg)
{
    gemm_job *jb = (gemm_job *)arg;
    int64_t N = jb->N, K = jb->K, KB = K / OR_BLOCK;
    double *arow = (double *)malloc((size_t)K * sizeof(double));
    for (int64_t r = jb->r0; r < jb->r1; ++r) {
        int64_t m = jb->rows[r];
        for (int64_t k = 0; k < K; ++k)
            arow[k] = jb->dec[jb->qa[m * K + k]];
        for (int64_t n = 0; n < N; ++n) {
            const double *wrow = jb->wdec + n * K;
            double acc = 0.0;
            for (int64_t j = 0; j < KB; ++j) {
                double b = 0.0;     /* B_j: exact in fp64 */
                for (int64_t k = j * OR_BLOCK; k < (j + 1) * OR_BLOCK; ++k)
                    b += arow[k] * wrow[k];
                acc += (double)jb->sa[m * KB + j] *
                       (double)jb->sw[(n / OR_BLOCK) * KB + j] * b;
            }
            jb->y[r * N + n] = acc;
        }
    }
    free(arow);
    return NULL;
}

/* Block-scaled FP8 linear, fp64 result R for selected rows.
 * qa e4m3 [M,K], sa fp32 [M,K/128], qw e4m3 [N,K], sw fp32 [N/128,K/128].
 * Rows are split across nthreads worker threads; each output element is
 * computed by one thread in the order written above.  Returns 0 on
 * success, -1 on allocation failure. */
int oracle_block_linear_rows(const uint8_t *qa, const float *sa,
                             const uint8_t *qw, const float *sw,
                             int64_t M, int64_t N, int64_t K,
                             const int64_t *rows, int64_t nrows,
                             double *y, int nthreads)
{
    (void)M;
    double dec[256];
    for (int c = 0; c < 256; ++c)
        dec[c] = oracle_e4m3_decode((uint8_t)c);
    double *wdec = (double *)malloc((size_t)N * (size_t)K * sizeof(double));
    if (!wdec)
        return -1;
    for (int64_t i = 0; i < N * K; ++i)
        wdec[i] = dec[qw[i]];
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > nrows)
        nthreads = nrows > 0 ? (int)nrows : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    gemm_job *jobs = (gemm_job *)malloc(sizeof(gemm_job) * (size_t)nthreads);
    int64_t per = (nrows + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        gemm_job j = {qa, sa, qw, sw, N, K, rows, t * per,
                      (t + 1) * per < nrows ? (t + 1) * per : nrows,
                      dec, wdec, y};
        if (j.r0 > nrows)
            j.r0 = nrows;
        jobs[t] = j;
        pthread_create(&th[t], NULL, gemm_rows, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    free(wdec);
    return 0;
}

/* Parallel activation quantization over rows (the CPU baseline runs this
 * on all host cores). */
typedef struct {
    const uint16_t *x;
    int64_t M, K;
    uint8_t *q;
    float *s;
    uint8_t *s8;        /* UE8M0 codes instead of s when not NULL */
    int64_t m0, m1;
} qa_job;

static void *qa_rows(void *arg)
{
    qa_job *j = (qa_job *)arg;
    if (j->s8)
        oracle_quant_act_ue8m0_rows(j->x, j->M, j->K, j->q, j->s8, j->m0, j->m1);
    else
        oracle_quant_act_rows(j->x, j->M, j->K, j->q, j->s, j->m0, j->m1);
    return NULL;
}

static void quant_act_threads(const uint16_t *x, int64_t M, int64_t K,
                              uint8_t *q, float *s, uint8_t *s8, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > M)
        nthreads = M > 0 ? (int)M : 1;
    pthread_t th[256];
    qa_job jobs[256];
    if (nthreads > 256)
        nthreads = 256;
    int64_t per = (M + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        int64_t m0 = t * per, m1 = (t + 1) * per;
        if (m0 > M) m0 = M;
        if (m1 > M) m1 = M;
        qa_job j = {x, M, K, q, s, s8, m0, m1};
        jobs[t] = j;
        pthread_create(&th[t], NULL, qa_rows, &jobs[t]);
    }
    for (int t = 0; t < nthreads; ++t)
        pthread_join(th[t], NULL);
}

void oracle_quant_act(const uint16_t *x, int64_t M, int64_t K, uint8_t *q,
                      float *s, int nthreads)
{
    quant_act_threads(x, M, K, q, s, NULL, nthreads);
}

void oracle_quant_act_ue8m0(const uint16_t *x, int64_t M, int64_t K,
                            uint8_t *q, uint8_t *s, int nthreads)
{
    quant_act_threads(x, M, K, q, NULL, s, nthreads);
}
