// Device kernels of libzero (sm_100a).
//
// All kernels share one work decomposition: a table of runs (SegDesc). A run
// is cut into warp chunks of 256 elements whose vector body starts on a
// 128-byte line of the fp16 gradients, plus scalar chunks for the ragged head
// and tail. A persistent grid walks the chunks warp by warp (warp w takes
// chunks w, w + W, w + 2W, ...), so at any moment the whole GPU streams one
// narrow window of every buffer. Within a chunk lane L owns quads L and L + 32
// (a quad is 4 consecutive elements): every warp load or store is then one
// contiguous, sector-aligned run of 256 bytes (fp16) or 512 bytes (fp32), and
// each lane keeps 8 elements of every stream in flight. fp32 state falls back
// to narrower accesses when a run's state index is out of phase with its
// gradient index. Every access is a streaming (evict-first) load or store:
// each byte is touched once per step.
//
// The path is pure streaming arithmetic (about 20 flops per element against
// at least 56 bytes at Nd = 8), bounded by HBM bandwidth, so no tensor cores.
//
// Arithmetic is written with explicit round-to-nearest intrinsics in the
// order the step defines, so the results do not depend on FMA contraction.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_device.cuh"
#include "zero_internal.h"

// Minimum resident blocks per SM the step kernels are compiled for (caps
// registers per thread at 65536 / (256 * ZK_MIN_BLOCKS)).
#ifndef ZK_MIN_BLOCKS
#define ZK_MIN_BLOCKS 1
#endif

namespace zk {
namespace {

// ---- per-item bodies of the step kernels ----

// C: the 16-bit element format (F16 with an fp32 master; BF16 without one,
// where the weight is read back from the first output and no master is kept).
template <int K, class C>
__device__ __forceinline__ void step_vec(const StepArgs& a, const Live& L, const uint16_t* const* gp,
                                         uint16_t* const* op, const SegDesc& d, const Pair& p,
                                         bool& bad)
{
    const long long ga = d.grad_begin + p.ea, gb = d.grad_begin + p.eb;
    const long long sa = d.state_begin + p.ea, sb = d.state_begin + p.eb;
    const long long oa = d.out_begin + p.ea, ob = d.out_begin + p.eb;
    const bool hb = p.hb;
    if (!(in_bounds(ga, 4, a.grad_len, a.err) & in_bounds(sa, 4, a.state_len, a.err) &
          in_bounds(oa, 4, a.out_len, a.err) &
          (!hb || (in_bounds(gb, 4, a.grad_len, a.err) & in_bounds(sb, 4, a.state_len, a.err) &
                   in_bounds(ob, 4, a.out_len, a.err)))))
        return;
    float w[8], m[8], v[8], g[8];
    if (K == K_INIT) {
        ld_pair(a.master_init, ga, gb, hb, w);
#pragma unroll
        for (int j = 0; j < 8; ++j) m[j] = 0.0f;
        if (C::kMaster) st_pair(L.w_out, sa, sb, hb, w);
        st_pair(L.m_out, sa, sb, hb, m);
        st_pair(L.v_out, sa, sb, hb, m);
    } else if (K == K_CAST) {
        ld_pair(L.w_in, sa, sb, hb, w);
    } else {
        if (K == K_STEP_FUSED || K == K_UPDATE) {
            if (C::kMaster) {
                ld_pair(L.w_in, sa, sb, hb, w);
            } else {
                unpack_as<C>(ld_hq_any(op[a.w_src] + oa), w);
                unpack_as<C>(hb ? ld_hq_any(op[a.w_src] + ob) : make_uint2(0u, 0u), w + 4);
            }
            ld_pair(L.m_in, sa, sb, hb, m);
            ld_pair(L.v_in, sa, sb, hb, v);
        }
        if (K == K_STEP_FUSED || K == K_REDUCE) {
            reduce_pair<C>(gp, a.nd, ga, gb, hb, g);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                g[j] = __fmul_rn(g[j], L.c.inv_scale);
                bad |= nonfinite(g[j]);  // an absent second quad holds zeros
            }
        }
        if (K == K_REDUCE) {
            st_pair(a.red, sa, sb, hb, g);
            return;
        }
        if (K == K_UPDATE) ld_pair(a.red, sa, sb, hb, g);
        const float wd = d.decay ? L.c.wd : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) adam1(g[j], w[j], m[j], v[j], L.c, wd);
        if (C::kMaster) st_pair(L.w_out, sa, sb, hb, w);
        st_pair(L.m_out, sa, sb, hb, m);
        st_pair(L.v_out, sa, sb, hb, v);
    }
    const uint2 h0 = pack_as<C>(w), h1 = pack_as<C>(w + 4);
    const int n_write = K == K_STEP_FUSED ? a.n_out - a.keep_last : a.n_out;
    for (int k = 0; k < n_write; ++k) {
        st_hq(op[k] + oa, h0);
        if (hb) st_hq(op[k] + ob, h1);
    }
}

// Walk the chunks of a run table; call vec(d, pair) for each lane's pair of
// quads and scal(d, e) for each head/tail element (offsets within the run).
template <class Vec, class Scal>
__device__ __forceinline__ void walk(const SegDesc* segs, int n_segs, long long n_chunks, Vec vec,
                                     Scal scal)
{
    const int lane = threadIdx.x & 31;
    const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    SegDesc d;
    long long lo = 0, hi = 0;  // chunk range of the cached run d (empty at start)
    for (long long c = warp; c < n_chunks; c += n_warps) {
        if (c < lo || c >= hi) {
            const int s = find_run(segs, n_segs, c);
            d = segs[s];
            lo = d.chunk_begin;
            hi = (s + 1 < n_segs) ? segs[s + 1].chunk_begin : n_chunks;
        }
        const long long quads = (d.len - d.head - d.tail) / kQuad;
        const long long vec_chunks = (quads + kQuadsPerChunk - 1) / kQuadsPerChunk;
        const long long k = c - d.chunk_begin;
        if (k < vec_chunks) {
            const long long qa = k * kQuadsPerChunk + lane;
            const long long qb = qa + 32;
            if (qa < quads) {
                Pair p;
                p.ea = d.head + qa * kQuad;
                p.hb = qb < quads;
                p.eb = p.hb ? d.head + qb * kQuad : p.ea;
                vec(d, p);
            }
        } else {
            // scalar chunks: head elements first, then the tail
            const long long q = (k - vec_chunks) * 32 + lane;
            long long e = -1;
            if (q < d.head)
                e = q;
            else if (q < d.head + d.tail)
                e = d.len - d.tail + (q - d.head);
            if (e >= 0) scal(d, e);
        }
    }
}

// K_CAST_IF is K_CAST run only when the step overflowed or a kernel gave up.
// ASYNC: the step constants and state buffers come from the control block.
template <int K, bool ASYNC, class C = F16>
__global__ void __launch_bounds__(kThreads, ZK_MIN_BLOCKS) step_kernel(const StepArgs a0)
{
    extern __shared__ uintptr_t s_ptr[];
    if (K == K_UPDATE) {
        // pass 2 of the two-pass variant: the whole step is skipped on overflow
        if (*reinterpret_cast<volatile const unsigned*>(a0.flag) == a0.call_id) return;
    }
    if (K == K_CAST_IF) {
        if (*reinterpret_cast<volatile const unsigned*>(a0.flag) != a0.call_id &&
            *reinterpret_cast<volatile const unsigned*>(a0.err) == 0)
            return;
    }
    const StepArgs& a = a0;
    const Live L = live_of<ASYNC>(a);
    constexpr bool kGrads = (K == K_STEP_FUSED || K == K_REDUCE);
    const int n_g = kGrads ? a.nd : 0;
    const int n_o = (K == K_REDUCE) ? 0 : a.n_out;
    for (int i = threadIdx.x; i < n_g + n_o; i += blockDim.x)
        s_ptr[i] = (i < n_g) ? reinterpret_cast<uintptr_t>(a.grads[i])
                             : reinterpret_cast<uintptr_t>(a.outs[i - n_g]);
    __syncthreads();
    const uint16_t* const* gp = reinterpret_cast<const uint16_t* const*>(s_ptr);
    uint16_t* const* op = reinterpret_cast<uint16_t* const*>(s_ptr + n_g);

    constexpr int KB = (K == K_CAST_IF) ? K_CAST : K;  // the item body
    bool bad = false;
    walk(
        a.segs, a.n_segs, a.n_chunks,
        [&](const SegDesc& d, const Pair& p) { step_vec<KB, C>(a, L, gp, op, d, p, bad); },
        [&](const SegDesc& d, long long e) { step_scalar<KB, C>(a, L, gp, op, d, e, bad); });

    if (kGrads) {
        // one atomic per warp that saw a non-finite unscaled gradient
        if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicMax(a.flag, a.call_id);
    }
}

// The commit pass of the fused step without an fp32 master (the 16-bit
// parameters are the only copy of the weights): the step kernel read the
// weight from the last output and wrote the new one into all the others. On
// overflow, or if a kernel gave up a wait, the last output's (old) values are
// copied back over the others; otherwise output 0's (new) values are copied
// into the last one. 16-bit patterns are copied as they are.
__global__ void __launch_bounds__(kThreads) replica_kernel(const StepArgs a)
{
    const bool roll_back = *reinterpret_cast<volatile const unsigned*>(a.flag) == a.call_id ||
                           *reinterpret_cast<volatile const unsigned*>(a.err) != 0;
    const int last = a.n_out - 1;
    const int src = roll_back ? last : 0;
    const int d0 = roll_back ? 0 : last, d1 = roll_back ? last : a.n_out;
    const uint16_t* sp = a.outs[src];
    walk(
        a.segs, a.n_segs, a.n_chunks,
        [&](const SegDesc& d, const Pair& p) {
            const long long oa = d.out_begin + p.ea, ob = d.out_begin + p.eb;
            if (!(in_bounds(oa, 4, a.out_len, a.err) & (!p.hb || in_bounds(ob, 4, a.out_len, a.err)))) return;
            const uint2 h0 = ld_hq_any(sp + oa);
            const uint2 h1 = p.hb ? ld_hq_any(sp + ob) : make_uint2(0u, 0u);
            for (int k = d0; k < d1; ++k) {
                st_hq(a.outs[k] + oa, h0);
                if (p.hb) st_hq(a.outs[k] + ob, h1);
            }
        },
        [&](const SegDesc& d, long long e) {
            const long long oi = d.out_begin + e;
            if (!in_bounds(oi, 1, a.out_len, a.err)) return;
            const unsigned short h = __ldcs(reinterpret_cast<const unsigned short*>(sp + oi));
            for (int k = d0; k < d1; ++k) __stcs(reinterpret_cast<unsigned short*>(a.outs[k] + oi), h);
        });
}

__global__ void __launch_bounds__(kThreads) gather_kernel(const GatherArgs a)
{
    walk(
        a.segs, a.n_segs, a.n_chunks,
        [&](const SegDesc& d, const Pair& p) {
            if (!(in_bounds(d.grad_begin + p.ea, 4, a.src_len, a.err) &
                  in_bounds(d.out_begin + p.ea, 4, a.dst_len, a.err) &
                  (!p.hb || (in_bounds(d.grad_begin + p.eb, 4, a.src_len, a.err) &
                             in_bounds(d.out_begin + p.eb, 4, a.dst_len, a.err)))))
                return;
            const uint2 qa = ld_hq(a.src + d.grad_begin + p.ea);
            const uint2 qb = p.hb ? ld_hq(a.src + d.grad_begin + p.eb) : make_uint2(0u, 0u);
            st_hq(a.dst + d.out_begin + p.ea, qa);
            if (p.hb) st_hq(a.dst + d.out_begin + p.eb, qb);
        },
        [&](const SegDesc& d, long long e) {
            if (!(in_bounds(d.grad_begin + e, 1, a.src_len, a.err) & in_bounds(d.out_begin + e, 1, a.dst_len, a.err)))
                return;
            __stcs(reinterpret_cast<unsigned short*>(a.dst + d.out_begin + e),
                   __ldcs(reinterpret_cast<const unsigned short*>(a.src + d.grad_begin + e)));
        });
}

__global__ void __launch_bounds__(kThreads) copy_kernel(uint4* dst, const uint4* src, long long n)
{
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        __stcs(dst + i, __ldcs(src + i));
}

// The asynchronous step's commit: skip (back off the loss scale) or commit
// (advance t and the bias-correction products, switch buffers, grow the loss
// scale after a run of good steps), then clear the overflow word.
__global__ void commit_kernel(Ctrl* c, unsigned* flag, const unsigned* err)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const bool skip = (*reinterpret_cast<volatile unsigned*>(flag) != 0) ||
                      (*reinterpret_cast<volatile const unsigned*>(err) != 0);
    if (skip) {
        c->scale = __fmul_rn(c->scale, c->backoff);
        c->good = 0;
        c->skipped += 1;
    } else {
        c->p1 = c->p1 * (double)c->b1;
        c->p2 = c->p2 * (double)c->b2;
        c->t += 1;
        if (c->fused) c->cur = 1 - c->cur;
        c->good += 1;
        if (c->good >= c->interval) {
            const float grown = __fmul_rn(c->scale, c->growth);
            if (!nonfinite(grown)) c->scale = grown;
            c->good = 0;
        }
    }
    ctrl_next_constants(c);
    *flag = 0;
}

const void* kernel_ptr(Kernel k, bool bf16)
{
    if (bf16) {
        switch (k) {
            case K_STEP_FUSED: return reinterpret_cast<const void*>(&step_kernel<K_STEP_FUSED, false, BF16>);
            case K_REPLICA: return reinterpret_cast<const void*>(&replica_kernel);
            case K_REDUCE: return reinterpret_cast<const void*>(&step_kernel<K_REDUCE, false, BF16>);
            case K_UPDATE: return reinterpret_cast<const void*>(&step_kernel<K_UPDATE, false, BF16>);
            case K_CAST: return reinterpret_cast<const void*>(&step_kernel<K_CAST, false, BF16>);
            case K_INIT: return reinterpret_cast<const void*>(&step_kernel<K_INIT, false, BF16>);
            case K_GATHER: return reinterpret_cast<const void*>(&gather_kernel);
            default: return nullptr;
        }
    }
    switch (k) {
        case K_STEP_FUSED: return reinterpret_cast<const void*>(&step_kernel<K_STEP_FUSED, false>);
        case K_REDUCE: return reinterpret_cast<const void*>(&step_kernel<K_REDUCE, false>);
        case K_UPDATE: return reinterpret_cast<const void*>(&step_kernel<K_UPDATE, false>);
        case K_CAST: return reinterpret_cast<const void*>(&step_kernel<K_CAST, false>);
        case K_INIT: return reinterpret_cast<const void*>(&step_kernel<K_INIT, false>);
        case K_GATHER: return reinterpret_cast<const void*>(&gather_kernel);
        case K_CAST_IF: return reinterpret_cast<const void*>(&step_kernel<K_CAST_IF, true>);
        default: return nullptr;
    }
}

}  // namespace

int step_smem_bytes(int nd, int n_out) { return (nd + n_out) * (int)sizeof(uintptr_t); }

cudaError_t occupancy(Kernel k, int smem, int* blocks_per_sm, bool bf16)
{
    const void* f = kernel_ptr(k, bf16);
    if (!f) {
        *blocks_per_sm = 0;
        return cudaSuccess;  // not instantiated for this format
    }
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, f, kThreads, smem);
}

cudaError_t launch_step(Kernel k, const StepArgs& a, int grid, cudaStream_t s, bool bf16)
{
    const int smem = step_smem_bytes(a.nd, a.n_out);
    const bool as = a.ctrl != nullptr;
    if (bf16) {
        // without a master: the two passes, or the fused step with its replica pass
        switch (k) {
            case K_STEP_FUSED:
                if (as) step_kernel<K_STEP_FUSED, true, BF16><<<grid, kThreads, smem, s>>>(a);
                else step_kernel<K_STEP_FUSED, false, BF16><<<grid, kThreads, smem, s>>>(a);
                break;
            case K_REPLICA: replica_kernel<<<grid, kThreads, 0, s>>>(a); break;
            case K_REDUCE:
                if (as) step_kernel<K_REDUCE, true, BF16><<<grid, kThreads, smem, s>>>(a);
                else step_kernel<K_REDUCE, false, BF16><<<grid, kThreads, smem, s>>>(a);
                break;
            case K_UPDATE:
                if (as) step_kernel<K_UPDATE, true, BF16><<<grid, kThreads, smem, s>>>(a);
                else step_kernel<K_UPDATE, false, BF16><<<grid, kThreads, smem, s>>>(a);
                break;
            case K_CAST: step_kernel<K_CAST, false, BF16><<<grid, kThreads, smem, s>>>(a); break;
            case K_INIT: step_kernel<K_INIT, false, BF16><<<grid, kThreads, smem, s>>>(a); break;
            default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    switch (k) {
        case K_STEP_FUSED:
            if (as) step_kernel<K_STEP_FUSED, true><<<grid, kThreads, smem, s>>>(a);
            else step_kernel<K_STEP_FUSED, false><<<grid, kThreads, smem, s>>>(a);
            break;
        case K_REDUCE:
            if (as) step_kernel<K_REDUCE, true><<<grid, kThreads, smem, s>>>(a);
            else step_kernel<K_REDUCE, false><<<grid, kThreads, smem, s>>>(a);
            break;
        case K_UPDATE:
            if (as) step_kernel<K_UPDATE, true><<<grid, kThreads, smem, s>>>(a);
            else step_kernel<K_UPDATE, false><<<grid, kThreads, smem, s>>>(a);
            break;
        case K_CAST: step_kernel<K_CAST, false><<<grid, kThreads, smem, s>>>(a); break;
        case K_INIT: step_kernel<K_INIT, false><<<grid, kThreads, smem, s>>>(a); break;
        case K_CAST_IF:
            if (!as) return cudaErrorInvalidValue;
            step_kernel<K_CAST_IF, true><<<grid, kThreads, smem, s>>>(a);
            break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_commit(Ctrl* ctrl, unsigned* flag, const unsigned* err, cudaStream_t s)
{
    commit_kernel<<<1, 32, 0, s>>>(ctrl, flag, err);
    return cudaGetLastError();
}

cudaError_t launch_gather(const GatherArgs& a, int grid, cudaStream_t s)
{
    gather_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_copy(void* dst, const void* src, size_t bytes, int grid, cudaStream_t s)
{
    copy_kernel<<<grid, kThreads, 0, s>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                                          (long long)(bytes / 16));
    return cudaGetLastError();
}

}  // namespace zk
