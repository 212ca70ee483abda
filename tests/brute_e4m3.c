/*
 * Exhaustive pin of the oracle's e4m3 encoder.
 *
 * For every one of the 2^32 fp32 bit patterns, the expected code is found by
 * brute force: the nearest of the 127 non-negative finite e4m3 magnitudes
 * (codes 0x00..0x7E), ties going to the even code, then the sign bit of the
 * input is copied; NaN maps to S.1111.111.  The magnitudes are built here
 * from the OCP E4M3 bit layout in integer units of 2^-9 (value * 512 equals
 * m for exponent field 0, (8 + m) << (e - 1) otherwise), independently of
 * the oracle's decoder.  Nearest-of-finite is the same as "round to nearest
 * even, saturate at 448": every value beyond 448 is nearest to 448.
 *
 * Usage: brute_e4m3 <liboracle.so> <nthreads> [lo_hi16 hi_hi16]
 * Prints "mismatches <count>" and exits 0 when the count is zero.
 */
#include <dlfcn.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

typedef uint8_t (*enc_fn)(float);

static enc_fn g_enc;
static double g_mag[127];
static uint32_t g_lo, g_hi;   /* range of the top 16 bits to cover */
static int g_nthreads;

static uint8_t brute(float v)
{
    uint32_t bits;
    memcpy(&bits, &v, 4);
    uint8_t sign = (bits >> 31) ? 0x80 : 0;
    if (isnan(v))
        return sign | 0x7F;
    double a = fabs((double)v);
    /* binary search: first index with mag >= a */
    int lo = 0, hi = 127;
    while (lo < hi) {
        int mid = (lo + hi) / 2;
        if (g_mag[mid] < a)
            lo = mid + 1;
        else
            hi = mid;
    }
    int best;
    if (lo == 0)
        best = 0;
    else if (lo == 127)
        best = 126;
    else {
        double dlo = a - g_mag[lo - 1], dhi = g_mag[lo] - a;
        if (dlo < dhi)
            best = lo - 1;
        else if (dhi < dlo)
            best = lo;
        else
            best = ((lo - 1) % 2 == 0) ? lo - 1 : lo;
    }
    return sign | (uint8_t)best;
}

typedef struct {
    int t;
    uint64_t mism;
    uint32_t first_bad;
} job;

static void *run(void *arg)
{
    job *j = (job *)arg;
    for (uint32_t top = g_lo + (uint32_t)j->t; top < g_hi; top += (uint32_t)g_nthreads) {
        for (uint32_t low = 0; low < 65536u; ++low) {
            uint32_t bits = (top << 16) | low;
            float v;
            memcpy(&v, &bits, 4);
            uint8_t e = g_enc(v), b = brute(v);
            if (e != b) {
                if (j->mism == 0)
                    j->first_bad = bits;
                j->mism++;
            }
        }
    }
    return NULL;
}

int main(int argc, char **argv)
{
    if (argc < 3) {
        fprintf(stderr, "usage: %s liboracle.so nthreads [lo hi]\n", argv[0]);
        return 2;
    }
    void *h = dlopen(argv[1], RTLD_NOW);
    if (!h) {
        fprintf(stderr, "dlopen: %s\n", dlerror());
        return 2;
    }
    g_enc = (enc_fn)dlsym(h, "oracle_e4m3_encode");
    if (!g_enc)
        return 2;
    g_nthreads = atoi(argv[2]);
    g_lo = argc > 4 ? (uint32_t)strtoul(argv[3], 0, 0) : 0;
    g_hi = argc > 4 ? (uint32_t)strtoul(argv[4], 0, 0) : 65536u;
    for (int c = 0; c < 127; ++c) {
        int e = (c >> 3) & 0xF, m = c & 7;
        long units = e == 0 ? m : ((long)(8 + m) << (e - 1));
        g_mag[c] = (double)units / 512.0;
    }
    pthread_t th[256];
    job jobs[256];
    if (g_nthreads > 256)
        g_nthreads = 256;
    for (int t = 0; t < g_nthreads; ++t) {
        jobs[t].t = t;
        jobs[t].mism = 0;
        jobs[t].first_bad = 0;
        pthread_create(&th[t], 0, run, &jobs[t]);
    }
    uint64_t mism = 0;
    uint32_t first = 0;
    for (int t = 0; t < g_nthreads; ++t) {
        pthread_join(th[t], 0);
        if (jobs[t].mism && !mism)
            first = jobs[t].first_bad;
        mism += jobs[t].mism;
    }
    printf("mismatches %llu first 0x%08x\n", (unsigned long long)mism, first);
    return mism ? 1 : 0;
}
