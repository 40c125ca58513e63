// Host Adam of the offloaded step (see zero_host_adam.h). Built twice:
//   -DZH_AVX2 -mavx2 -mf16c : 8 elements per instruction, vcvtps2ph for fp16
//   (no flags)              : one element at a time, the same operations
// with -ffp-contract=off, so no multiply-add is ever fused.
#include "zero_host_adam.h"

#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef ZH_AVX2
#include <immintrin.h>
#define ZH_ADAM zh_adam_avx2
#define ZH_CAST zh_cast_avx2
#else
#define ZH_ADAM zh_adam_base
#define ZH_CAST zh_cast_base
#endif

namespace {

#ifdef ZH_AVX2
inline uint16_t to_half(float x)
{
    return (uint16_t)_cvtss_sh(x, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC);
}
#else
// binary32 -> binary16, round to nearest, ties to even; overflow to infinity,
// subnormal results kept, NaN kept quiet with the sign.
inline uint16_t to_half(float x)
{
    uint32_t b;
    memcpy(&b, &x, 4);
    const uint32_t sign = (b >> 16) & 0x8000u;
    const uint32_t ax = b & 0x7fffffffu;
    if (ax >= 0x7f800000u)  // inf or NaN
        return (uint16_t)(sign | 0x7c00u | (ax > 0x7f800000u ? 0x200u | ((ax >> 13) & 0x3ffu) : 0u));
    if (ax >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u);  // rounds to >= 2^16: infinity
    const int e = (int)(ax >> 23);                               // biased binary32 exponent
    if (e >= 113) {
        // normal binary16: drop 13 fraction bits with rounding; a carry out of
        // the fraction correctly bumps the exponent
        const uint32_t h = ((uint32_t)(e - 112) << 10) | ((ax >> 13) & 0x3ffu);
        const uint32_t rest = ax & 0x1fffu;
        const uint32_t up = (rest > 0x1000u) || (rest == 0x1000u && (h & 1u));
        return (uint16_t)(sign | (h + up));
    }
    // subnormal binary16 (or zero): value = q * 2^-24, q = round(|x| * 2^24)
    if (e < 102) return (uint16_t)sign;  // |x| < 2^-25: rounds to zero (2^-25 exactly is a tie to 0)
    const uint32_t mant = (ax & 0x7fffffu) | 0x800000u;  // |x| = mant * 2^(e - 150)
    const int shift = 126 - e;                            // |x| * 2^24 = mant >> shift
    const uint32_t q = mant >> shift;
    const uint32_t rest = mant & ((1u << shift) - 1u);
    const uint32_t half = 1u << (shift - 1);
    const uint32_t up = (rest > half) || (rest == half && (q & 1u));
    return (uint16_t)(sign | (q + up));
}
#endif

inline void adam_one(float g, float& w, float& m, float& v, uint16_t& p, const ZhCoef& c, float wd)
{
    const float m1 = c.b1 * m + c.omb1 * g;
    const float v1 = c.b2 * v + c.omb2 * (g * g);
    const float mh = m1 / c.bc1;
    const float vh = v1 / c.bc2;
    const float u = mh / (sqrtf(vh) + c.eps);
    const float w1 = w - c.lr * (u + wd * w);
    m = m1;
    v = v1;
    w = w1;
    p = to_half(w1);
}

}  // namespace

extern "C" void ZH_ADAM(const float* g, float* w, float* m, float* v, uint16_t* p16, int64_t n,
                        const ZhCoef* cp, float wd)
{
    const ZhCoef c = *cp;
    int64_t i = 0;
#ifdef ZH_AVX2
    const __m256 b1 = _mm256_set1_ps(c.b1), b2 = _mm256_set1_ps(c.b2);
    const __m256 omb1 = _mm256_set1_ps(c.omb1), omb2 = _mm256_set1_ps(c.omb2);
    const __m256 bc1 = _mm256_set1_ps(c.bc1), bc2 = _mm256_set1_ps(c.bc2);
    const __m256 eps = _mm256_set1_ps(c.eps), lr = _mm256_set1_ps(c.lr), wdv = _mm256_set1_ps(wd);
    for (; i + 8 <= n; i += 8) {
        const __m256 gg = _mm256_loadu_ps(g + i);
        const __m256 ww = _mm256_loadu_ps(w + i);
        const __m256 m1 = _mm256_add_ps(_mm256_mul_ps(b1, _mm256_loadu_ps(m + i)), _mm256_mul_ps(omb1, gg));
        const __m256 v1 = _mm256_add_ps(_mm256_mul_ps(b2, _mm256_loadu_ps(v + i)),
                                        _mm256_mul_ps(omb2, _mm256_mul_ps(gg, gg)));
        const __m256 mh = _mm256_div_ps(m1, bc1);
        const __m256 vh = _mm256_div_ps(v1, bc2);
        const __m256 u = _mm256_div_ps(mh, _mm256_add_ps(_mm256_sqrt_ps(vh), eps));
        const __m256 w1 = _mm256_sub_ps(ww, _mm256_mul_ps(lr, _mm256_add_ps(u, _mm256_mul_ps(wdv, ww))));
        _mm256_storeu_ps(m + i, m1);
        _mm256_storeu_ps(v + i, v1);
        _mm256_storeu_ps(w + i, w1);
        // the fp16 result goes to page-locked staging that the GPU copies
        // from: a non-temporal store skips reading the line first
        const __m128i h = _mm256_cvtps_ph(w1, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC);
        if ((reinterpret_cast<uintptr_t>(p16 + i) & 15u) == 0)
            _mm_stream_si128(reinterpret_cast<__m128i*>(p16 + i), h);
        else
            _mm_storeu_si128(reinterpret_cast<__m128i*>(p16 + i), h);
    }
    _mm_sfence();  // the streamed stores are visible before the caller hands the slot on
#endif
    for (; i < n; ++i) adam_one(g[i], w[i], m[i], v[i], p16[i], c, wd);
}

extern "C" void ZH_CAST(const float* w, uint16_t* p16, int64_t n)
{
    int64_t i = 0;
#ifdef ZH_AVX2
    for (; i + 8 <= n; i += 8)
        _mm_storeu_si128(reinterpret_cast<__m128i*>(p16 + i),
                         _mm256_cvtps_ph(_mm256_loadu_ps(w + i), _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC));
#endif
    for (; i < n; ++i) p16[i] = to_half(w[i]);
}
