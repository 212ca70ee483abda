/*
 * Exhaustive check of the quotient the CUDA quantizer forms.
 *
 * The kernels compute x / s for a whole 128-group with one correctly
 * rounded reciprocal r = fp32(1/s) and, per element, q0 = fp32(x*r),
 * e = fma(q0, -s, x), q = fma(e, r, q0) (Markstein's correction step).
 * The e4m3 code is then cvt(q) with the sign bit of x OR-ed in: the
 * correction turns x = -0 into +0, and this program also checks that every
 * non-zero q already carries the sign of x, so the OR changes nothing else.
 * The quantization definition wants fp32(x / s), then e4m3 rounding.  This
 * program checks, for EVERY pair the kernels can meet -- amax any
 * non-negative finite bf16 value (s = fp32(max(amax, 1e-10)/448)) and x any
 * bf16 value with |x| <= amax -- that the two quotients give the same e4m3
 * code: either identical fp32 bits, or both at most 2^-10 in magnitude with
 * the same sign (all such values encode to the signed zero).
 * The arithmetic is IEEE binary32 on the host: division, fmaf (correctly
 * rounded) and multiplication, with gradual underflow, exactly as the GPU
 * instructions the kernel uses (div.rn, rcp.rn, mul.rn, fma.rn, no flush).
 *
 * The scale s itself is formed on the GPU with the same correction step
 * against the constant R = fp32(1/448): q0 = fp32(a*R), e = fma(q0,-448,a),
 * s = fma(e, R, q0), a = max(amax, 1e-10).  This program first checks that
 * s equals the IEEE quotient a / 448 for every amax (printing
 * "scales <n> bad <m>"), then uses it for the element check.
 *
 * Usage: div_exhaustive <nthreads>.  Prints "pairs <n> bad <m>".
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static int g_nt;

static float bf(uint32_t h) { uint32_t b = h << 16; float f; memcpy(&f, &b, 4); return f; }
static uint32_t bits(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }

typedef struct { int t; uint64_t pairs, bad, scale_bad; uint32_t bad_a, bad_x; } job;

static void *run(void *arg)
{
    job *j = (job *)arg;
    volatile float eps = 1e-10f, m448 = 448.0f, one = 1.0f;
    const float R = one / m448;
    for (uint32_t a = (uint32_t)j->t; a <= 0x7F7Fu; a += (uint32_t)g_nt) {
        float amax = bf(a);
        float av = fmaxf(amax, eps);
        float sq0 = av * R;
        float se = fmaf(sq0, -m448, av);
        float s = fmaf(se, R, sq0);
        if (bits(s) != bits(av / m448)) {
            j->scale_bad++;
            continue;
        }
        float r = one / s;
        for (uint32_t xm = 0; xm <= a; ++xm) {
            for (uint32_t sg = 0; sg < 2; ++sg) {
                float x = bf(xm | (sg << 15));
                float ref = x / s;
                float q0 = x * r;
                float e = fmaf(q0, -s, x);
                float q = fmaf(e, r, q0);
                j->pairs++;
                if (q != 0.0f && (bits(q) >> 31) != (bits(x) >> 31)) {
                    if (!j->bad) { j->bad_a = a; j->bad_x = xm | (sg << 15); }
                    j->bad++;
                    continue;
                }
                if (q == 0.0f)
                    q = copysignf(0.0f, x);   /* the sign-bit OR on the code */
                if (bits(q) == bits(ref))
                    continue;
                if (fabsf(q) <= 0x1p-10f && fabsf(ref) <= 0x1p-10f &&
                    (bits(q) >> 31) == (bits(ref) >> 31))
                    continue;
                if (!j->bad) { j->bad_a = a; j->bad_x = xm | (sg << 15); }
                j->bad++;
            }
        }
    }
    return NULL;
}

int main(int argc, char **argv)
{
    g_nt = argc > 1 ? atoi(argv[1]) : 8;
    if (g_nt < 1) g_nt = 1;
    if (g_nt > 256) g_nt = 256;
    pthread_t th[256];
    job jobs[256];
    memset(jobs, 0, sizeof jobs);
    for (int t = 0; t < g_nt; ++t) {
        jobs[t].t = t;
        pthread_create(&th[t], 0, run, &jobs[t]);
    }
    uint64_t pairs = 0, bad = 0, scale_bad = 0;
    uint32_t ba = 0, bx = 0;
    for (int t = 0; t < g_nt; ++t) {
        pthread_join(th[t], 0);
        pairs += jobs[t].pairs;
        scale_bad += jobs[t].scale_bad;
        if (jobs[t].bad && !bad) { ba = jobs[t].bad_a; bx = jobs[t].bad_x; }
        bad += jobs[t].bad;
    }
    printf("scales 32640 bad %llu\n", (unsigned long long)scale_bad);
    printf("pairs %llu bad %llu first amax 0x%04x x 0x%04x\n",
           (unsigned long long)pairs, (unsigned long long)bad, ba, bx);
    return (bad || scale_bad) ? 1 : 0;
}
