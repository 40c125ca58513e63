/*
 * Oracle for the ZeRO partitioned mixed-precision Adam step.
 *
 * TEST INFRASTRUCTURE. A plain, slow, single-threaded CPU statement of what the
 * step computes, written from the pages' text (page list in zero_ref.h). Only
 * the test suite, the package's smoke check and the benchmark's CPU-baseline
 * leg may load it; the CUDA library never calls it and the two share no code.
 *
 * Build with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math
 * so that every binary32 operation below is one IEEE-rounded operation in the
 * order written (no FMA contraction, no flush-to-zero, SSE arithmetic).
 *
 * Readings where the pages are silent:
 *  - Adam is the Kingma-Ba bias-corrected form, eps outside the square root,
 *    m-hat and v-hat formed by division; weight decay is decoupled and scaled
 *    by lr (AdamW).  [P2] "Where We Were" names Adam/AdamW without equations.
 *  - gradients are summed (not averaged) across ranks, in rank order 0..nd-1,
 *    starting from rank 0's value.
 *  - one global overflow flag for the whole step; on overflow nothing changes
 *    and the step counter t does not advance.
 *  - partitions use the ceil split; trailing ranks may be short or empty.
 */
#include "zero_ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ======================================================================
 * binary16 <-> binary32 / binary64, IEEE 754 interchange format:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * ==================================================================== */

float zr_f32_from_f16(uint16_t h)
{
    const int neg = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1f;
    const int f = h & 0x3ff;
    double mag;
    if (e == 0x1f) {
        if (f != 0) return neg ? -NAN : NAN;
        mag = INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)f, -24);            /* subnormal: f * 2^-24 */
    } else {
        mag = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return (float)(neg ? -mag : mag);           /* exact: fits binary32 */
}

/* Round x to the nearest binary16 value, ties to even, by counting quanta. */
uint16_t zr_f16_from_f64(double x)
{
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return sign | 0x7e00;
    const double a = fabs(x);
    /* 65504 is the largest finite half; its quantum is 32, and the halfway
     * point 65520 rounds to the even neighbour 65536, which overflows. */
    if (a >= 65520.0) return sign | 0x7c00;
    int q_exp; /* quantum 2^q_exp of the binade holding a */
    if (a >= 0x1p-14) {
        int e;
        frexp(a, &e);          /* a = mant * 2^e, mant in [0.5, 1) */
        q_exp = (e - 1) - 10;  /* 10 fraction bits below the leading bit */
    } else {
        q_exp = -24;           /* subnormal spacing */
    }
    const double n = rint(ldexp(a, -q_exp)); /* default mode: nearest, ties even */
    if (n == 0.0) return sign;
    if (q_exp == -24) return sign | (uint16_t)n; /* n = 1024 encodes 2^-14 */
    int biased = q_exp + 10 + 15;
    double sig = n;
    if (sig == 2048.0) { sig = 1024.0; biased += 1; } /* rounded up a binade */
    return sign | (uint16_t)(biased << 10) | (uint16_t)((int)sig - 1024);
}

uint16_t zr_f16_from_f32(float x) { return zr_f16_from_f64((double)x); }

/* ======================================================================
 * bfloat16 <-> binary32: 1 sign bit, 8 exponent bits (bias 127), 7 fraction
 * bits ([P3] "Why parameter count is not training memory": not every BF16
 * setup keeps fp32 master weights).
 * ==================================================================== */

float zr_f32_from_bf16(uint16_t h)
{
    const int neg = (h >> 15) & 1;
    const int e = (h >> 7) & 0xff;
    const int f = h & 0x7f;
    double mag;
    if (e == 0xff) {
        if (f != 0) return neg ? -NAN : NAN;
        mag = INFINITY;
    } else if (e == 0) {
        mag = ldexp((double)f, -133);             /* subnormal: f * 2^-133 */
    } else {
        mag = ldexp((double)(128 + f), e - 134);  /* (1 + f/128) * 2^(e-127) */
    }
    return (float)(neg ? -mag : mag);
}

/* Round x to the nearest bfloat16 value, ties to even, by counting quanta. */
uint16_t zr_bf16_from_f64(double x)
{
    const uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return sign | 0x7fc0;
    const double a = fabs(x);
    /* the largest finite value is (2 - 2^-7) 2^127; from the halfway point
     * (2 - 2^-8) 2^127 on, the nearest even neighbour is 2^128: overflow */
    if (a >= ldexp(2.0 - ldexp(1.0, -8), 127)) return sign | 0x7f80;
    int q_exp;
    if (a >= 0x1p-126) {
        int e;
        frexp(a, &e);
        q_exp = (e - 1) - 7;  /* 7 fraction bits below the leading bit */
    } else {
        q_exp = -133;         /* subnormal spacing */
    }
    const double n = rint(ldexp(a, -q_exp));
    if (n == 0.0) return sign;
    if (q_exp == -133) return sign | (uint16_t)n; /* n = 128 encodes 2^-126 */
    int biased = q_exp + 7 + 127;
    double sig = n;
    if (sig == 256.0) { sig = 128.0; biased += 1; }
    return sign | (uint16_t)(biased << 7) | (uint16_t)((int)sig - 128);
}

uint16_t zr_bf16_from_f32(float x) { return zr_bf16_from_f64((double)x); }

void zr_f32_from_bf16_array(const uint16_t* h, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = zr_f32_from_bf16(h[i]);
}

void zr_bf16_from_f32_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = zr_bf16_from_f32(x[i]);
}

void zr_f32_from_f16_array(const uint16_t* h, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = zr_f32_from_f16(h[i]);
}

void zr_f16_from_f32_array(const float* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = zr_f16_from_f32(x[i]);
}

/* The sum of two binary16 values is exact in binary64 (their exponents differ
 * by at most 39 < 53 - 11), so one rounding to binary16 follows. */
uint16_t zr_direct_f16_update(uint16_t w16, float dw)
{
    const double a = (double)zr_f32_from_f16(w16);
    const double b = (double)zr_f32_from_f16(zr_f16_from_f32(dw));
    return zr_f16_from_f64(a + b);
}

void zr_direct_f16_update_array(const uint16_t* w16, const float* dw, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = zr_direct_f16_update(w16[i], dw[i]);
}

/* ======================================================================
 * Partitions.  [P1] "The replication nobody questioned" and [P2] "The
 * Mathematics": the state is split across the Nd data-parallel ranks.
 * ==================================================================== */

void zr_partition(int64_t psi, int32_t nd, int32_t r, int64_t* begin, int64_t* end)
{
    const int64_t p = (psi + nd - 1) / nd;
    int64_t b = (int64_t)r * p;
    int64_t e = b + p;
    if (b > psi) b = psi;
    if (e > psi) e = psi;
    *begin = b;
    *end = e;
}

void zr_chunk(int64_t n, int32_t nd, int32_t r, int64_t* begin, int64_t* end)
{
    zr_partition(n, nd, r, begin, end);
}

int64_t zr_shard_len(int32_t n_tensors, const int64_t* numel, int32_t nd, int32_t r)
{
    int64_t len = 0;
    for (int32_t t = 0; t < n_tensors; ++t) {
        int64_t b, e;
        zr_chunk(numel[t], nd, r, &b, &e);
        len += e - b;
    }
    return len;
}

/* ======================================================================
 * Step scalars.
 * ==================================================================== */

void zr_bias_corrections(float beta1, float beta2, int64_t t, float* bc1, float* bc2)
{
    double p1 = 1.0, p2 = 1.0;
    for (int64_t k = 0; k < t; ++k) {
        p1 = p1 * (double)beta1;
        p2 = p2 * (double)beta2;
    }
    *bc1 = (float)(1.0 - p1);
    *bc2 = (float)(1.0 - p2);
}

float zr_inv_scale(float loss_scale) { return (float)(1.0 / (double)loss_scale); }

typedef struct {
    float lr, b1, b2, omb1, omb2, bc1, bc2, eps, wd;
} coef_t;

static coef_t make_coef(const zr_hyper* hp, int64_t t_new)
{
    coef_t c;
    c.lr = hp->lr;
    c.b1 = hp->beta1;
    c.b2 = hp->beta2;
    c.omb1 = 1.0f - hp->beta1;
    c.omb2 = 1.0f - hp->beta2;
    c.eps = hp->eps;
    c.wd = hp->weight_decay;
    zr_bias_corrections(hp->beta1, hp->beta2, t_new, &c.bc1, &c.bc2);
    return c;
}

/* One element of mixed-precision Adam, binary32 throughout ([P1] "Why you
 * can't just delete the fp32 copies": the update accumulates into the fp32
 * master and the fp16 copy is derived from it). */
static void adam_element(float g, float* w, float* m, float* v, const coef_t* c)
{
    const float m1 = c->b1 * (*m) + c->omb1 * g;
    const float v1 = c->b2 * (*v) + c->omb2 * (g * g);
    const float mh = m1 / c->bc1;
    const float vh = v1 / c->bc2;
    const float u = mh / (sqrtf(vh) + c->eps);
    const float w1 = *w - c->lr * (u + c->wd * (*w));
    *m = m1;
    *v = v1;
    *w = w1;
}

/* Rank-ordered binary32 sum of the nd fp16 gradients at index i. */
static float reduce_at(const uint16_t* const* grads, int32_t nd, int64_t i)
{
    float s = zr_f32_from_f16(grads[0][i]);
    for (int32_t r = 1; r < nd; ++r) s = s + zr_f32_from_f16(grads[r][i]);
    return s;
}

/* ======================================================================
 * The definition: plain data parallelism ([P1] "The replication nobody
 * questioned": all-reduce, then the identical update on every rank).
 * ==================================================================== */

int zr_dp_step(int64_t n, int32_t nd, const uint16_t* const* grads,
               float* w, float* m, float* v, uint16_t* p16,
               float loss_scale, const zr_hyper* hp, int64_t* t)
{
    return zr_dp_step_masked(n, nd, grads, w, m, v, p16, loss_scale, hp, NULL, t);
}

/* The same with weight decay applied only where decay[i] != 0 (decoupled
 * weight decay, Loshchilov and Hutter; excluding some tensors, such as biases
 * and normalisation gains, is a convention of AdamW setups, not of the pages).
 * An excluded element takes the update with weight decay 0. */
int zr_dp_step_masked(int64_t n, int32_t nd, const uint16_t* const* grads,
                      float* w, float* m, float* v, uint16_t* p16,
                      float loss_scale, const zr_hyper* hp, const uint8_t* decay,
                      int64_t* t)
{
    const float inv = zr_inv_scale(loss_scale);
    float* g = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    int overflow = 0;
    for (int64_t i = 0; i < n; ++i) {
        g[i] = reduce_at(grads, nd, i) * inv;
        if (!isfinite(g[i])) overflow = 1;
    }
    if (overflow) {
        free(g);
        return 1;
    }
    *t = *t + 1;
    const coef_t c = make_coef(hp, *t);
    coef_t c_nodecay = c;
    c_nodecay.wd = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        const coef_t* ci = (decay == NULL || decay[i] != 0) ? &c : &c_nodecay;
        adam_element(g[i], &w[i], &m[i], &v[i], ci);
        p16[i] = zr_f16_from_f32(w[i]);
    }
    free(g);
    return 0;
}

/* The step of a BF16 setup without fp32 master weights ([P3] "Why parameter
 * count is not training memory"): gradients and parameters are bfloat16, the
 * Adam moments binary32. The reduction and the element update are the ones
 * above; the parameter is read from and rounded back to bfloat16 every step,
 * so K = 8 bytes of optimizer state per parameter instead of 12. */
int zr_bf16_step(int64_t n, int32_t nd, const uint16_t* const* grads, uint16_t* w16,
                 float* m, float* v, float loss_scale, const zr_hyper* hp,
                 const uint8_t* decay, int64_t* t)
{
    const float inv = zr_inv_scale(loss_scale);
    float* g = (float*)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    int overflow = 0;
    for (int64_t i = 0; i < n; ++i) {
        float s = zr_f32_from_bf16(grads[0][i]);
        for (int32_t r = 1; r < nd; ++r) s = s + zr_f32_from_bf16(grads[r][i]);
        g[i] = s * inv;
        if (!isfinite(g[i])) overflow = 1;
    }
    if (overflow) {
        free(g);
        return 1;
    }
    *t = *t + 1;
    const coef_t c = make_coef(hp, *t);
    coef_t c_nodecay = c;
    c_nodecay.wd = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float w = zr_f32_from_bf16(w16[i]);
        adam_element(g[i], &w, &m[i], &v[i], (decay == NULL || decay[i] != 0) ? &c : &c_nodecay);
        w16[i] = zr_bf16_from_f32(w);
    }
    free(g);
    return 0;
}

/* ======================================================================
 * ZeRO stage 1/2 ([P1] "The part that sounds too good: communication":
 * reduce-scatter, update only the own slice, all-gather the fp16 params).
 * ==================================================================== */

int zr_zero12_step(int64_t psi, int32_t nd, const uint16_t* const* grads,
                   float* const* w_sh, float* const* m_sh, float* const* v_sh,
                   uint16_t* const* replicas,
                   float loss_scale, const zr_hyper* hp, int64_t* t)
{
    const float inv = zr_inv_scale(loss_scale);
    float** red = (float**)calloc((size_t)nd, sizeof(float*));
    int flag = 0; /* the all-reduced (OR) overflow flag */
    for (int32_t r = 0; r < nd; ++r) {
        int64_t b, e;
        zr_partition(psi, nd, r, &b, &e);
        red[r] = (float*)malloc((size_t)(e - b > 0 ? e - b : 1) * sizeof(float));
        int local = 0;
        for (int64_t i = b; i < e; ++i) { /* reduce-scatter into rank r */
            red[r][i - b] = reduce_at(grads, nd, i) * inv;
            if (!isfinite(red[r][i - b])) local = 1;
        }
        flag = flag | local;
    }
    if (!flag) {
        *t = *t + 1;
        const coef_t c = make_coef(hp, *t);
        for (int32_t r = 0; r < nd; ++r) {
            int64_t b, e;
            zr_partition(psi, nd, r, &b, &e);
            for (int64_t j = 0; j < e - b; ++j) {
                adam_element(red[r][j], &w_sh[r][j], &m_sh[r][j], &v_sh[r][j], &c);
                const uint16_t p = zr_f16_from_f32(w_sh[r][j]);
                for (int32_t k = 0; k < nd; ++k) replicas[k][b + j] = p; /* all-gather */
            }
        }
    }
    for (int32_t r = 0; r < nd; ++r) free(red[r]);
    free(red);
    return flag;
}

/* ======================================================================
 * ZeRO stage 3 ([P1] stage table "Stage 3 (Pos+g+p)"; [P3] "Partitioned
 * parameters still have to participate in computation").
 * ==================================================================== */

int zr_zero3_step(int32_t n_tensors, const int64_t* numel, int32_t nd,
                  const uint16_t* const* grads,
                  float* const* w_sh, float* const* m_sh, float* const* v_sh,
                  uint16_t* const* p_sh,
                  float loss_scale, const zr_hyper* hp, int64_t* t)
{
    const float inv = zr_inv_scale(loss_scale);
    float** red = (float**)calloc((size_t)nd, sizeof(float*));
    int flag = 0;
    for (int32_t r = 0; r < nd; ++r) {
        const int64_t len = zr_shard_len(n_tensors, numel, nd, r);
        red[r] = (float*)malloc((size_t)(len > 0 ? len : 1) * sizeof(float));
        int64_t q = 0, off = 0;
        int local = 0;
        for (int32_t ti = 0; ti < n_tensors; ++ti) {
            int64_t b, e;
            zr_chunk(numel[ti], nd, r, &b, &e);
            for (int64_t i = b; i < e; ++i, ++q) {
                red[r][q] = reduce_at(grads, nd, off + i) * inv;
                if (!isfinite(red[r][q])) local = 1;
            }
            off += numel[ti];
        }
        flag = flag | local;
    }
    if (!flag) {
        *t = *t + 1;
        const coef_t c = make_coef(hp, *t);
        for (int32_t r = 0; r < nd; ++r) {
            const int64_t len = zr_shard_len(n_tensors, numel, nd, r);
            for (int64_t q = 0; q < len; ++q) {
                adam_element(red[r][q], &w_sh[r][q], &m_sh[r][q], &v_sh[r][q], &c);
                p_sh[r][q] = zr_f16_from_f32(w_sh[r][q]);
            }
        }
    }
    for (int32_t r = 0; r < nd; ++r) free(red[r]);
    free(red);
    return flag;
}

int64_t zr_zero3_gather(int32_t n_tensors, const int64_t* numel, const int32_t* unit_of,
                        int32_t nd, int32_t unit, const uint16_t* const* p_sh,
                        uint16_t* out)
{
    int64_t pos = 0;
    for (int32_t ti = 0; ti < n_tensors; ++ti) {
        if (unit_of[ti] != unit) continue;
        for (int32_t r = 0; r < nd; ++r) {
            /* where rank r's chunk of tensor ti sits inside rank r's shard */
            int64_t shard_pos = 0;
            for (int32_t tj = 0; tj < ti; ++tj) {
                int64_t b, e;
                zr_chunk(numel[tj], nd, r, &b, &e);
                shard_pos += e - b;
            }
            int64_t b, e;
            zr_chunk(numel[ti], nd, r, &b, &e);
            for (int64_t i = b; i < e; ++i) out[pos + i] = p_sh[r][shard_pos + (i - b)];
        }
        pos += numel[ti];
    }
    return pos;
}

/* ======================================================================
 * Dynamic loss scaling: multiplicative back-off on overflow, growth after a
 * run of good steps.
 * ==================================================================== */

void zr_scaler_update(float* scale, int32_t* good, int overflow, float growth, float backoff,
                      int32_t interval)
{
    if (overflow) {
        *scale = *scale * backoff;
        *good = 0;
        return;
    }
    *good = *good + 1;
    if (*good >= interval) {
        const float grown = *scale * growth;
        if (isfinite(grown)) *scale = grown;
        *good = 0;
    }
}

/* ======================================================================
 * Ledger.  [P1] "Where 16 bytes per parameter comes from" (2 + 2 + K, K = 12)
 * and the stage table in "The replication nobody questioned"; [P2] "The
 * Mathematics", M_states(p, Nd); [P3] "What each ZeRO stage partitions".
 * ==================================================================== */

void zr_ledger_formula(double psi, double nd, double out[4])
{
    const double K = 12.0;
    out[0] = (2.0 + 2.0 + K) * psi;           /* baseline DP: everything replicated */
    out[1] = 2.0 * psi + 2.0 * psi + K * psi / nd; /* optimizer states partitioned */
    out[2] = 2.0 * psi + (2.0 + K) * psi / nd;     /* + gradients */
    out[3] = (2.0 + 2.0 + K) * psi / nd;           /* + parameters */
}

void zr_ledger_exact(int64_t psi, int32_t nd, int32_t n_tensors, const int64_t* numel,
                     int64_t out[4])
{
    int64_t best[4] = {0, 0, 0, 0};
    for (int32_t r = 0; r < nd; ++r) {
        int64_t b, e;
        zr_partition(psi, nd, r, &b, &e);
        const int64_t pr = e - b;
        const int64_t sr = n_tensors > 0 ? zr_shard_len(n_tensors, numel, nd, r) : pr;
        const int64_t v[4] = {16 * psi, 2 * psi + 2 * psi + 12 * pr, 2 * psi + 14 * pr, 16 * sr};
        for (int k = 0; k < 4; ++k)
            if (v[k] > best[k]) best[k] = v[k];
    }
    for (int k = 0; k < 4; ++k) out[k] = best[k];
}

/* Ring reduce-scatter: in each of nd-1 steps every rank forwards one partial
 * chunk to its neighbour; rank r never sends the chunk it ends up owning, so it
 * sends psi - |that chunk| elements and all ranks together send (nd-1) psi.  The
 * ring all-gather is the mirror image.  ([P1] "The part that sounds too good:
 * communication": a ring all-reduce is a reduce-scatter plus an all-gather.) */
void zr_comm_elements(int64_t psi, int32_t nd, int64_t out[6])
{
    int64_t rs = 0;
    for (int32_t r = 0; r < nd; ++r) {
        int64_t b, e;
        zr_partition(psi, nd, r, &b, &e);
        rs += psi - (e - b);
    }
    const int64_t ag = rs;
    out[0] = rs;
    out[1] = ag;
    out[2] = rs + ag;      /* baseline DP all-reduce */
    out[3] = rs + ag;      /* stage 1: reduce-scatter + all-gather */
    out[4] = rs + ag;      /* stage 2: same traffic */
    out[5] = rs + 2 * ag;  /* stage 3: gathers in forward and again in backward */
}
