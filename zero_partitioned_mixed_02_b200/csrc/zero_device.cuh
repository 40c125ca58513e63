// Device helpers shared by the step kernels (zero_kernels.cu, zero_tma.cu):
// fp16 packing, streaming quad accesses, the step's per-element arithmetic
// and the scalar (head/tail) item body. Internal to libzero.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_internal.h"

namespace zk {
namespace {

__device__ __forceinline__ bool nonfinite(float x)
{
    return (__float_as_uint(x) & 0x7f800000u) == 0x7f800000u;
}

// The bounds-checked build (ZK_BOUNDS_CHECK): an access to elements
// [i, i + n) of a buffer of len elements that is not inside it sets bit 32 of
// the error word and is skipped (the host reports ZERO_ERR_INTERNAL). In the
// normal build the check is the constant true and compiles away.
#ifdef ZK_BOUNDS_CHECK
__device__ __forceinline__ bool in_bounds(long long i, long long n, long long len, unsigned* err)
{
    if (i >= 0 && n >= 0 && i + n <= len) return true;
    atomicOr(err, 32u);
    return false;
}
#else
__device__ __forceinline__ bool in_bounds(long long, long long, long long, unsigned*) { return true; }
#endif

__device__ __forceinline__ float h2f(unsigned short b) { return __half2float(__ushort_as_half(b)); }

__device__ __forceinline__ unsigned short f2h(float x) { return __half_as_ushort(__float2half_rn(x)); }

// ---- quads: 4 fp16 values packed in a uint2, 4 fp32 values ----

__device__ __forceinline__ void unpack(const uint2 q, float* x)
{
    x[0] = h2f((unsigned short)(q.x & 0xffffu));
    x[1] = h2f((unsigned short)(q.x >> 16));
    x[2] = h2f((unsigned short)(q.y & 0xffffu));
    x[3] = h2f((unsigned short)(q.y >> 16));
}

__device__ __forceinline__ unsigned pack2(float lo, float hi)
{
    return (unsigned)f2h(lo) | ((unsigned)f2h(hi) << 16);
}

__device__ __forceinline__ uint2 pack(const float* x) { return make_uint2(pack2(x[0], x[1]), pack2(x[2], x[3])); }

// 4 fp16 values from p (8-byte aligned: quads start on multiples of 4).
__device__ __forceinline__ uint2 ld_hq(const uint16_t* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }

// 4 16-bit values from p with the widest loads p's alignment allows (the
// parameter buffers read back by the step without a master may be out of
// phase with the gradient index).
__device__ __forceinline__ uint2 ld_hq_any(const uint16_t* p)
{
    const unsigned a = (unsigned)reinterpret_cast<uintptr_t>(p);
    if ((a & 7u) == 0) return __ldcs(reinterpret_cast<const uint2*>(p));
    if ((a & 3u) == 0) {
        const unsigned* u = reinterpret_cast<const unsigned*>(p);
        return make_uint2(__ldcs(u), __ldcs(u + 1));
    }
    const unsigned short* h = reinterpret_cast<const unsigned short*>(p);
    return make_uint2((unsigned)__ldcs(h) | ((unsigned)__ldcs(h + 1) << 16),
                      (unsigned)__ldcs(h + 2) | ((unsigned)__ldcs(h + 3) << 16));
}

// ---- element formats of the 16-bit streams ----
// F16: IEEE binary16 gradients and parameters, fp32 master weights.
// BF16: bfloat16 gradients and parameters and no fp32 master: the parameter
// itself is the weight state, read back and rounded to bfloat16 every step.
struct F16 {
    static constexpr bool kMaster = true;
    __device__ static float dec(unsigned short b) { return h2f(b); }
    __device__ static unsigned short enc(float x) { return f2h(x); }
};
struct BF16 {
    static constexpr bool kMaster = false;
    __device__ static float dec(unsigned short b) { return __uint_as_float((unsigned)b << 16); }
    __device__ static unsigned short enc(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
};

template <class C>
__device__ __forceinline__ void unpack_as(const uint2 q, float* x)
{
    x[0] = C::dec((unsigned short)(q.x & 0xffffu));
    x[1] = C::dec((unsigned short)(q.x >> 16));
    x[2] = C::dec((unsigned short)(q.y & 0xffffu));
    x[3] = C::dec((unsigned short)(q.y >> 16));
}

template <class C>
__device__ __forceinline__ uint2 pack_as(const float* x)
{
    return make_uint2((unsigned)C::enc(x[0]) | ((unsigned)C::enc(x[1]) << 16),
                      (unsigned)C::enc(x[2]) | ((unsigned)C::enc(x[3]) << 16));
}

// Store 4 fp16 values with the widest accesses p's alignment allows (the
// branch is uniform over a run).
__device__ __forceinline__ void st_hq(uint16_t* p, const uint2 q)
{
    const unsigned a = (unsigned)reinterpret_cast<uintptr_t>(p);
    if ((a & 7u) == 0) {
        __stcs(reinterpret_cast<uint2*>(p), q);
    } else if ((a & 3u) == 0) {
        unsigned* u = reinterpret_cast<unsigned*>(p);
        __stcs(u, q.x);
        __stcs(u + 1, q.y);
    } else {
        unsigned short* h = reinterpret_cast<unsigned short*>(p);
        __stcs(h, (unsigned short)(q.x & 0xffffu));
        __stcs(h + 1, (unsigned short)(q.x >> 16));
        __stcs(h + 2, (unsigned short)(q.y & 0xffffu));
        __stcs(h + 3, (unsigned short)(q.y >> 16));
    }
}

// 4 fp32 values, widest access the alignment allows.
__device__ __forceinline__ void ldq(const float* p, float* x)
{
    const unsigned a = (unsigned)reinterpret_cast<uintptr_t>(p);
    if ((a & 15u) == 0) {
        const float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        x[0] = t.x;
        x[1] = t.y;
        x[2] = t.z;
        x[3] = t.w;
    } else if ((a & 7u) == 0) {
        const float2 t0 = __ldcs(reinterpret_cast<const float2*>(p));
        const float2 t1 = __ldcs(reinterpret_cast<const float2*>(p) + 1);
        x[0] = t0.x;
        x[1] = t0.y;
        x[2] = t1.x;
        x[3] = t1.y;
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) x[k] = __ldcs(p + k);
    }
}

__device__ __forceinline__ void stq(float* p, const float* x)
{
    const unsigned a = (unsigned)reinterpret_cast<uintptr_t>(p);
    if ((a & 15u) == 0) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
    } else if ((a & 7u) == 0) {
        __stcs(reinterpret_cast<float2*>(p), make_float2(x[0], x[1]));
        __stcs(reinterpret_cast<float2*>(p) + 1, make_float2(x[2], x[3]));
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) __stcs(p + k, x[k]);
    }
}

// A lane's pair of quads: elements [ea, ea + 4) and, if hb, [eb, eb + 4) of
// the run; values 0..3 belong to the first quad, 4..7 to the second.
struct Pair {
    long long ea, eb;
    bool hb;
};

__device__ __forceinline__ void ld_pair(const float* base, long long ia, long long ib, bool hb,
                                        float (&x)[8])
{
    ldq(base + ia, x);
    if (hb)
        ldq(base + ib, x + 4);
    else
        x[4] = x[5] = x[6] = x[7] = 0.0f;
}

__device__ __forceinline__ void st_pair(float* base, long long ia, long long ib, bool hb,
                                        const float (&x)[8])
{
    stq(base + ia, x);
    if (hb) stq(base + ib, x + 4);
}

// ---- the step's arithmetic ----

// Rank-ordered binary32 sum of the Nd 16-bit gradients of a lane's two quads.
// Loads are issued 8 ranks at a time ahead of the additions.
template <class C = F16>
__device__ __forceinline__ void reduce_pair(const uint16_t* const* gp, int nd, long long ga,
                                            long long gb, bool hb, float (&s)[8])
{
    uint2 qa[8], qb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        if (j < nd) {
            qa[j] = ld_hq(gp[j] + ga);
            qb[j] = hb ? ld_hq(gp[j] + gb) : make_uint2(0u, 0u);
        }
    }
    unpack_as<C>(qa[0], s);
    unpack_as<C>(qb[0], s + 4);
#pragma unroll
    for (int j = 1; j < 8; ++j) {
        if (j < nd) {
            float x[8];
            unpack_as<C>(qa[j], x);
            unpack_as<C>(qb[j], x + 4);
#pragma unroll
            for (int i = 0; i < 8; ++i) s[i] = __fadd_rn(s[i], x[i]);
        }
    }
    for (int r0 = 8; r0 < nd; r0 += 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (r0 + j < nd) {
                qa[j] = ld_hq(gp[r0 + j] + ga);
                qb[j] = hb ? ld_hq(gp[r0 + j] + gb) : make_uint2(0u, 0u);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (r0 + j < nd) {
                float x[8];
                unpack_as<C>(qa[j], x);
                unpack_as<C>(qb[j], x + 4);
#pragma unroll
                for (int i = 0; i < 8; ++i) s[i] = __fadd_rn(s[i], x[i]);
            }
        }
    }
}

template <class C = F16>
__device__ __forceinline__ float reduce1(const uint16_t* const* gp, int nd, long long gi)
{
    float s = C::dec(__ldcs(reinterpret_cast<const unsigned short*>(gp[0] + gi)));
    for (int r = 1; r < nd; ++r)
        s = __fadd_rn(s, C::dec(__ldcs(reinterpret_cast<const unsigned short*>(gp[r] + gi))));
    return s;
}

// One element of mixed-precision Adam (bias-corrected, decoupled weight decay
// wd scaled by lr), binary32, in the order of the step's definition. wd is
// c.wd, or 0 for a tensor excluded from weight decay.
__device__ __forceinline__ void adam1(float g, float& w, float& m, float& v, const Coef& c, float wd)
{
    const float m1 = __fadd_rn(__fmul_rn(c.b1, m), __fmul_rn(c.omb1, g));
    const float v1 = __fadd_rn(__fmul_rn(c.b2, v), __fmul_rn(c.omb2, __fmul_rn(g, g)));
    const float mh = __fdiv_rn(m1, c.bc1);
    const float vh = __fdiv_rn(v1, c.bc2);
    const float u = __fdiv_rn(mh, __fadd_rn(__fsqrt_rn(vh), c.eps));
    w = __fsub_rn(w, __fmul_rn(c.lr, __fadd_rn(u, __fmul_rn(wd, w))));
    m = m1;
    v = v1;
}

// What a launch's items use: the state buffers and the step constants. For
// the synchronous step (ASYNC = false: the kernel argument values, which the
// compiler reads straight from the parameter bank) they come from the kernel
// arguments; for the asynchronous step from the control block: the bias corrections for t + 1
// (one more factor on the t-fold products) and 1 / loss scale, with the host
// path's roundings, and the buffers picked by the live index (by selects, so
// nothing is indexed at run time).
struct Live {
    const float* w_in;
    const float* m_in;
    const float* v_in;
    float* w_out;
    float* m_out;
    float* v_out;
    Coef c;
};

template <bool ASYNC>
__device__ __forceinline__ Live live_of(const StepArgs& a)
{
    Live L;
    L.c = a.c;
    if (!ASYNC) {
        L.w_in = a.w_in;
        L.m_in = a.m_in;
        L.v_in = a.v_in;
        L.w_out = a.w_out;
        L.m_out = a.m_out;
        L.v_out = a.v_out;
        return L;
    }
    const Ctrl* c = a.ctrl;
    L.c.bc1 = c->bc1;  // written by zero_async_begin and by the last commit
    L.c.bc2 = c->bc2;
    L.c.inv_scale = c->inv_scale;
    const bool in1 = c->cur != 0;
    const bool out1 = c->fused ? !in1 : in1;
    L.w_in = in1 ? a.st[1][0] : a.st[0][0];
    L.m_in = in1 ? a.st[1][1] : a.st[0][1];
    L.v_in = in1 ? a.st[1][2] : a.st[0][2];
    L.w_out = out1 ? a.st[1][0] : a.st[0][0];
    L.m_out = out1 ? a.st[1][1] : a.st[0][1];
    L.v_out = out1 ? a.st[1][2] : a.st[0][2];
    return L;
}

// live_of with the live buffer known at compile time (PAR, the asynchronous
// step's live index; a fused step writes the other buffer): the state pointers
// are kernel arguments, the constants come from the control block.
template <bool ASYNC, int PAR>
__device__ __forceinline__ Live live_at(const StepArgs& a)
{
    if (!ASYNC) return live_of<false>(a);
    Live L;
    L.c = a.c;
    const Ctrl* c = a.ctrl;
    L.c.bc1 = c->bc1;
    L.c.bc2 = c->bc2;
    L.c.inv_scale = c->inv_scale;
    L.w_in = a.st[PAR][0];
    L.m_in = a.st[PAR][1];
    L.v_in = a.st[PAR][2];
    L.w_out = a.st[1 - PAR][0];
    L.m_out = a.st[1 - PAR][1];
    L.v_out = a.st[1 - PAR][2];
    return L;
}

// C::kMaster false (no fp32 master): K_INIT writes no master, K_UPDATE and
// K_STEP_FUSED read the weight from output a.w_src (the parameter itself)
// and write no master, K_STEP_FUSED leaves the last a.keep_last outputs
// alone; the state buffers hold m and v only.
template <int K, class C = F16>
__device__ __forceinline__ void step_scalar(const StepArgs& a, const Live& L, const uint16_t* const* gp,
                                            uint16_t* const* op, const SegDesc& d, long long e,
                                            bool& bad)
{
    const long long gi = d.grad_begin + e, si = d.state_begin + e, oi = d.out_begin + e;
    if (!(in_bounds(gi, 1, a.grad_len, a.err) & in_bounds(si, 1, a.state_len, a.err) &
          in_bounds(oi, 1, a.out_len, a.err)))
        return;
    float w = 0.0f, m = 0.0f, v = 0.0f, g = 0.0f;
    if (K == K_INIT) {
        w = __ldcs(a.master_init + gi);
        if (C::kMaster) __stcs(L.w_out + si, w);
        __stcs(L.m_out + si, 0.0f);
        __stcs(L.v_out + si, 0.0f);
    } else if (K == K_CAST) {
        w = __ldcs(L.w_in + si);
    } else {
        if (K == K_STEP_FUSED || K == K_UPDATE) {
            if (C::kMaster)
                w = __ldcs(L.w_in + si);
            else
                w = C::dec(__ldcs(reinterpret_cast<const unsigned short*>(op[a.w_src] + oi)));
            m = __ldcs(L.m_in + si);
            v = __ldcs(L.v_in + si);
        }
        if (K == K_STEP_FUSED || K == K_REDUCE) {
            g = __fmul_rn(reduce1<C>(gp, a.nd, gi), L.c.inv_scale);
            bad |= nonfinite(g);
        }
        if (K == K_REDUCE) {
            __stcs(a.red + si, g);
            return;
        }
        if (K == K_UPDATE) g = __ldcs(a.red + si);
        adam1(g, w, m, v, L.c, d.decay ? L.c.wd : 0.0f);
        if (C::kMaster) __stcs(L.w_out + si, w);
        __stcs(L.m_out + si, m);
        __stcs(L.v_out + si, v);
    }
    const unsigned short h = C::enc(w);
    const int n_write = K == K_STEP_FUSED ? a.n_out - a.keep_last : a.n_out;
    for (int k = 0; k < n_write; ++k) __stcs(reinterpret_cast<unsigned short*>(op[k] + oi), h);
}

// Largest run index whose first chunk is <= c.
__device__ __forceinline__ int find_run(const SegDesc* segs, int n, long long c)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (segs[mid].chunk_begin <= c)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

}  // namespace
}  // namespace zk
