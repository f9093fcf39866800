/*
 * tw_synth.c — seeded synthetic inputs for tests and benchmarks.
 *
 * Holds no arithmetic of the ternary layer itself: only a counter-based
 * random stream (SplitMix64, Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), the Box–Muller transform
 * (Box & Muller, 1958) and a partial Fisher–Yates shuffle.  The same host
 * arrays feed both the CUDA path and the reference oracle.
 *
 * Stream definition: for a 64-bit key, output i (i = 0, 1, ...) is the
 * SplitMix64 finaliser applied to key + (i + 1) * 0x9E3779B97F4A7C15.
 * Normal sample j uses outputs 2*(j/2) and 2*(j/2)+1 as the uniform pair
 * (u1 in (0,1], u2 in [0,1)); even j takes r*cos(2*pi*u2), odd j r*sin(...),
 * r = sqrt(-2 ln u1).  The fp64 value times sigma is rounded to fp32.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#define TWS_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t tws_fin(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t tws_output(uint64_t key, uint64_t i)
{
    return tws_fin(key + (i + 1) * TWS_GAMMA);
}

/* Derive a stream key from a base seed and up to three small labels. */
uint64_t tws_key(uint64_t base, int64_t a, int64_t b, int64_t c)
{
    uint64_t k = tws_fin(base + TWS_GAMMA);
    k = tws_fin(k ^ ((uint64_t)a + 0x100000001B3ULL));
    k = tws_fin(k ^ ((uint64_t)b + 0x1000193ULL * 7));
    k = tws_fin(k ^ ((uint64_t)c + 0x27D4EB2F165667C5ULL));
    return k;
}

/* out[j] = (float)(sigma * normal_{offset+j}) for j in [0, n). */
void tws_normal_f32(uint64_t key, int64_t offset, int64_t n, double sigma,
                    float *out)
{
    const double two_pi = 6.283185307179586476925286766559;
    const double inv53 = 1.0 / 9007199254740992.0; /* 2^-53 */
    for (int64_t j = 0; j < n; ++j) {
        uint64_t g = (uint64_t)(offset + j);
        uint64_t pair = g >> 1;
        double u1 = (double)((tws_output(key, 2 * pair) >> 11) + 1) * inv53;
        double u2 = (double)(tws_output(key, 2 * pair + 1) >> 11) * inv53;
        double r = sqrt(-2.0 * log(u1));
        double z = (g & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
        out[j] = (float)(sigma * z);
    }
}

/* First `count` entries of a seeded Fisher–Yates shuffle of [0, K). */
void tws_choose(uint64_t key, int64_t K, int64_t count, int64_t *idx_out)
{
    int64_t *perm = (int64_t *)malloc((size_t)K * sizeof(int64_t));
    if (!perm)
        return;
    for (int64_t i = 0; i < K; ++i)
        perm[i] = i;
    for (int64_t i = 0; i < count && i < K; ++i) {
        uint64_t r = tws_output(key, (uint64_t)i);
        int64_t j = i + (int64_t)(r % (uint64_t)(K - i));
        int64_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
        idx_out[i] = perm[i];
    }
    free(perm);
}
