/*
 * Seeded synthetic inputs shared by the tests, the benchmark and the oracle.
 * Holds none of the patcher's or the quantizer's arithmetic: only random
 * numbers, sinusoids and rounding to the stored type.
 *
 * Random numbers come from a counter-based SplitMix64 (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014): the value
 * for (seed, stream, i) is the SplitMix64 output function applied to a state
 * derived from the three, so any element can be drawn on its own, in any
 * order and on any number of threads, with the same result.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Draw number i of stream `stream` under `seed`. */
static uint64_t draw(uint64_t seed, uint64_t stream, uint64_t i)
{
    const uint64_t base = mix64(mix64(seed * GOLDEN_GAMMA + 1) ^ (stream * 0xD1B54A32D192ED03ULL));
    return mix64(base + (i + 1) * GOLDEN_GAMMA);
}

/* Uniform in [0, 1) with 53 random bits. */
static double unit(uint64_t seed, uint64_t stream, uint64_t i)
{
    return (double)(draw(seed, stream, i) >> 11) * 0x1.0p-53;
}

/*
 * Round a double to bfloat16 (nearest, ties to even) from the double's own
 * bits, so the value is rounded once.  Values outside [2^-120, 2^120] in
 * magnitude (never produced here except 0) go through fp32 first.
 */
static uint16_t to_bf16(double v)
{
    if (v != v)
        return 0x7FC0;
    if (v == 0.0 || fabs(v) < 0x1.0p-120 || fabs(v) > 0x1.0p+120) {
        const float f = (float)v;
        uint32_t u;
        memcpy(&u, &f, 4);
        u += 0x7FFFu + ((u >> 16) & 1u);
        return (uint16_t)(u >> 16);
    }
    uint64_t d;
    memcpy(&d, &v, 8);
    /* Keep 8 significant bits (1 implicit + 7), round away the other 45. */
    const uint64_t sign = d >> 63;
    int64_t e = (int64_t)((d >> 52) & 0x7FF) - 1023;
    const uint64_t m = (d & ((1ULL << 52) - 1)) | (1ULL << 52);
    uint64_t keep = m >> 45;
    const uint64_t rest = m & ((1ULL << 45) - 1), halfway = 1ULL << 44;
    if (rest > halfway || (rest == halfway && (keep & 1)))
        keep += 1;
    if (keep == (1ULL << 8)) { /* carried into the next binade */
        keep >>= 1;
        e += 1;
    }
    const uint32_t bits32 = (uint32_t)(sign << 31) | (uint32_t)((e + 127) << 23) | (uint32_t)((keep & 0x7F) << 16);
    return (uint16_t)(bits32 >> 16);
}

/* dtype codes: 0 = fp32, 1 = bf16, 2 = fp64 */
static void store(void *out, int dtype, int64_t i, double v)
{
    if (dtype == 0)
        ((float *)out)[i] = (float)v;
    else if (dtype == 1)
        ((uint16_t *)out)[i] = to_bf16(v);
    else
        ((double *)out)[i] = v;
}

/* out[i] = lo + (hi - lo) * U[0,1) for i < n. */
void synth_uniform(void *out, int dtype, int64_t n, uint64_t seed, uint64_t stream, double lo, double hi)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        store(out, dtype, i, lo + (hi - lo) * unit(seed, stream, (uint64_t)i));
}

/* out[i] = mean + std * N(0,1), Box-Muller on draws 2i and 2i+1. */
void synth_normal(void *out, int dtype, int64_t n, uint64_t seed, uint64_t stream, double mean, double std)
{
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const double u1 = 1.0 - unit(seed, stream, 2 * (uint64_t)i); /* (0, 1] */
        const double u2 = unit(seed, stream, 2 * (uint64_t)i + 1);
        store(out, dtype, i, mean + std * sqrt(-2.0 * log(u1)) * cos(two_pi * u2));
    }
}

/*
 * Smooth random field shaped like natural video, [B][C][T][H][W]:
 * for every (b, c), eight sinusoids with amplitude A ~ U[0.05, 0.25],
 * frequencies f_t ~ U[0, 1/16] cycles per frame and f_y, f_x ~ U[0, 1/64]
 * cycles per pixel, phase ~ U[0, 2pi); each voxel is their sum plus noise
 * U[-noise, noise], clipped to [-1, 1] and rounded once to the stored type.
 * The sinusoids are evaluated separably (rotations per axis), which is the
 * same function up to double rounding.
 */
#define FIELD_TERMS 8
void synth_smooth_field(void *out, int dtype, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W, uint64_t seed,
                        double noise)
{
    const double two_pi = 6.283185307179586476925286766559;
    const uint64_t PARAM_STREAM = 101, NOISE_STREAM = 102;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t frame = 0; frame < B * C * T; ++frame) {
        const int64_t bc = frame / T, t = frame % T;
        double amp[FIELD_TERMS], ft[FIELD_TERMS], fy[FIELD_TERMS], fx[FIELD_TERMS], ph[FIELD_TERMS];
        for (int k = 0; k < FIELD_TERMS; ++k) {
            const uint64_t p = ((uint64_t)bc * FIELD_TERMS + k) * 5;
            amp[k] = 0.05 + 0.20 * unit(seed, PARAM_STREAM, p + 0);
            ft[k] = unit(seed, PARAM_STREAM, p + 1) / 16.0;
            fy[k] = unit(seed, PARAM_STREAM, p + 2) / 64.0;
            fx[k] = unit(seed, PARAM_STREAM, p + 3) / 64.0;
            ph[k] = two_pi * unit(seed, PARAM_STREAM, p + 4);
        }
        double *cx = (double *)malloc(sizeof(double) * FIELD_TERMS * (size_t)W);
        double *sx = (double *)malloc(sizeof(double) * FIELD_TERMS * (size_t)W);
        for (int k = 0; k < FIELD_TERMS; ++k)
            for (int64_t x = 0; x < W; ++x) {
                cx[k * W + x] = cos(two_pi * fx[k] * (double)x);
                sx[k * W + x] = sin(two_pi * fx[k] * (double)x);
            }
        for (int64_t y = 0; y < H; ++y) {
            double re[FIELD_TERMS], im[FIELD_TERMS]; /* A * exp(i(2pi(f_t t + f_y y) + phase)) */
            for (int k = 0; k < FIELD_TERMS; ++k) {
                const double a = two_pi * (ft[k] * (double)t + fy[k] * (double)y) + ph[k];
                re[k] = amp[k] * cos(a);
                im[k] = amp[k] * sin(a);
            }
            const int64_t row = (frame * H + y) * W;
            for (int64_t x = 0; x < W; ++x) {
                double v = 0.0;
                for (int k = 0; k < FIELD_TERMS; ++k) /* Im(A e^{ia} e^{i 2pi f_x x}) */
                    v += re[k] * sx[k * W + x] + im[k] * cx[k * W + x];
                v += noise * (2.0 * unit(seed, NOISE_STREAM, (uint64_t)(row + x)) - 1.0);
                if (v > 1.0)
                    v = 1.0;
                if (v < -1.0)
                    v = -1.0;
                store(out, dtype, row + x, v);
            }
        }
        free(cx);
        free(sx);
    }
}
