/*
 * zsynth.h -- seeded, counter-based synthetic input generator.
 *
 * Input infrastructure shared by the tests and the benchmark: it makes the
 * gradients and initial master weights of the synthetic workloads and holds
 * none of the optimizer's arithmetic. The same source is compiled for the host
 * (oracle inputs, sampled checks) and for the device (full-size inputs), and
 * gives bit-identical binary32 values on both because it uses only integer
 * operations and single IEEE-rounded float operations.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used in counter mode: draw j of element i is
 * mix(key + 8*i + j), key = a hash of (seed, stream, step, rank).
 *
 * Distributions (binary32 results; conversion to fp16 is left to the caller):
 *   ZS_NORMAL       Irwin-Hall(12) approximation of N(0, sigma): the sum of 12
 *                   24-bit uniforms minus 6 * 2^24, converted to float and
 *                   multiplied by c = sigma * 2^-24 (rounded once).
 *   ZS_UNIFORM      a + (b - a) * u, u = u24 * 2^-24 in [0, 1).
 *   ZS_SIGNED_MAG   (a + (b - a) * u) with a random sign.
 *   ZS_NORMAL_TINY  with probability tiny_per_2_24 / 2^24 a value of random sign
 *                   and magnitude tiny_lo + (tiny_hi - tiny_lo) * u, otherwise
 *                   ZS_NORMAL.
 * Every result is finally multiplied by `scale` (a loss scale).
 */
#ifndef ZSYNTH_H
#define ZSYNTH_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ZS_NORMAL = 0, ZS_UNIFORM = 1, ZS_SIGNED_MAG = 2, ZS_NORMAL_TINY = 3 };

typedef struct zsynth_dist {
    int32_t kind;
    int32_t tiny_per_2_24;
    float c;        /* ZS_NORMAL / ZS_NORMAL_TINY: sigma * 2^-24 */
    float a, b;     /* ZS_UNIFORM bounds, ZS_SIGNED_MAG magnitude bounds */
    float tiny_lo;  /* ZS_NORMAL_TINY magnitude bounds */
    float tiny_hi;
    float scale;    /* final multiplier */
} zsynth_dist;

/* ---- host entry points (no GPU needed) ---- */
uint64_t zsynth_key(uint64_t seed, uint64_t stream, uint64_t step, uint64_t rank);
/* out[k] = value of element index0 + k, k < n */
void zsynth_host_f32(float* out, int64_t n, int64_t index0, uint64_t key, const zsynth_dist* d);
/* out[k] = value of element idx[k] */
void zsynth_host_f32_at(float* out, const int64_t* idx, int64_t n, uint64_t key,
                        const zsynth_dist* d);

/* ---- device entry points (stream is a cudaStream_t; 0 on success) ---- */
/* fp16 (round to nearest even) values of elements index0 .. index0 + n - 1 */
int zsynth_fill_f16(uint16_t* out, int64_t n, int64_t index0, uint64_t key,
                    const zsynth_dist* d, void* stream);
int zsynth_fill_f32(float* out, int64_t n, int64_t index0, uint64_t key,
                    const zsynth_dist* d, void* stream);

#ifdef __cplusplus
}
#endif

/* ---- the generator itself, shared by host and device builds ---- */
#ifdef __CUDACC__
#define ZS_HD __host__ __device__ __forceinline__
#else
#define ZS_HD static inline
#endif

ZS_HD uint64_t zs_mix(uint64_t x)
{
    uint64_t z = x + 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

ZS_HD uint64_t zs_draw(uint64_t key, int64_t i, uint32_t j)
{
    return zs_mix(key + ((uint64_t)i << 3) + j);
}

/* single rounded binary32 operations, never contracted into an FMA */
#ifdef __CUDA_ARCH__
#define ZS_MUL(x, y) __fmul_rn((x), (y))
#define ZS_ADD(x, y) __fadd_rn((x), (y))
#define ZS_I2F(x) __int2float_rn((x))
#else
#define ZS_MUL(x, y) ((float)(x) * (float)(y))
#define ZS_ADD(x, y) ((float)(x) + (float)(y))
#define ZS_I2F(x) ((float)(x))
#endif

ZS_HD float zs_u24_unit(uint32_t u24) { return ZS_MUL(ZS_I2F((int32_t)u24), 5.9604644775390625e-8f); }

ZS_HD float zs_normal(uint64_t key, int64_t i, float c)
{
    int32_t acc = 0;
    for (uint32_t j = 0; j < 6; ++j) {
        const uint64_t d = zs_draw(key, i, j);
        acc += (int32_t)(d & 0xFFFFFFu) + (int32_t)((d >> 32) & 0xFFFFFFu);
    }
    acc -= 6 << 24;
    return ZS_MUL(ZS_I2F(acc), c);
}

ZS_HD float zs_value(uint64_t key, int64_t i, const zsynth_dist* d)
{
    float x;
    if (d->kind == ZS_UNIFORM) {
        const uint32_t u = (uint32_t)(zs_draw(key, i, 0) >> 40);
        x = ZS_ADD(d->a, ZS_MUL(ZS_ADD(d->b, -d->a), zs_u24_unit(u)));
    } else if (d->kind == ZS_SIGNED_MAG) {
        const uint64_t r = zs_draw(key, i, 0);
        const float mag = ZS_ADD(d->a, ZS_MUL(ZS_ADD(d->b, -d->a), zs_u24_unit((uint32_t)(r >> 40))));
        x = (r & 1u) ? -mag : mag;
    } else if (d->kind == ZS_NORMAL_TINY) {
        const uint64_t r = zs_draw(key, i, 6);
        if ((int32_t)(r >> 40) < d->tiny_per_2_24) {
            const float mag = ZS_ADD(d->tiny_lo, ZS_MUL(ZS_ADD(d->tiny_hi, -d->tiny_lo),
                                                         zs_u24_unit((uint32_t)(r & 0xFFFFFFu))));
            x = ((r >> 24) & 1u) ? -mag : mag;
        } else {
            x = zs_normal(key, i, d->c);
        }
    } else {
        x = zs_normal(key, i, d->c);
    }
    return ZS_MUL(x, d->scale);
}

#endif
