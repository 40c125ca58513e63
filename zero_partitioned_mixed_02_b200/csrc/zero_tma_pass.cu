// The two-pass step with TMA staging (sm_100a): the reduce pass and the
// update pass of ZERO_VARIANT_TWO_PASS_TMA, each a persistent producer /
// consumer kernel built like the fused one in zero_tma.cu (the last warp
// produces; its lane 0 stages whole tiles into shared memory with 1D bulk
// asynchronous copies counted on the stage's "full" mbarrier; consumer warps
// wait on their own, read their quads out of shared memory, release the stage
// with one arrival on its "empty" mbarrier before the arithmetic, and write
// results with streaming stores).
//
//   reduce pass: stages the Nd 16-bit gradient slices of a tile; writes the
//                rank-ordered binary32 sum times inv_scale (state order) and
//                raises the overflow word.
//   update pass: returns at once if the step overflowed or the reduce pass
//                gave up a wait; stages the reduced gradient, m, v and the
//                weight (the fp32 master, or without one the 16-bit parameter
//                read back from the first output); runs Adam and writes m, v,
//                the master (if any) in place and the 16-bit parameters.
//
// C is the element format of the gradients and parameters (F16 with an fp32
// master, BF16 without one). Every wait is bounded; a warp that gives up sets
// the error word and leaves its loop; the producer drains its copies in flight.
// The update pass sets its own bits of the error word (kErrUpdate): its writes
// are in place, so the host reports such a failure as a partial update.
// Heads and tails of the runs are scalar items done from global memory. No
// cluster multicast.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_device.cuh"
#include "zero_internal.h"
#include "zero_tma.cuh"

namespace zk {
namespace {

// the error-word bits of a failed wait: the update pass's are shifted into kErrUpdate
template <int MODE>
__device__ __forceinline__ unsigned err_bits(unsigned bit)
{
    return MODE == kPassUpdate ? bit << kErrUpdateShift : bit;
}

// bytes of one element staged by the pass
template <int MODE, class C>
__host__ __device__ constexpr int pass_elem_bytes(int nd)
{
    return MODE == kPassReduce ? 2 * nd : 12 + (C::kMaster ? 4 : 2);
}

template <int MODE, int WARPS, int STAGES, bool ASYNC, class C>
__global__ void __launch_bounds__((WARPS + 1) * 32, 1) pass_tma_kernel(const TmaArgs a)
{
    static_assert(STAGES <= kMaxStages, "too many stages");
    constexpr int kTile = WARPS * 32 * kQuad;
    extern __shared__ __align__(128) char smem[];
    const StepArgs& b = a.b;
    if (MODE == kPassUpdate) {
        if (*reinterpret_cast<volatile const unsigned*>(b.flag) == b.call_id ||
            *reinterpret_cast<volatile const unsigned*>(a.err) != 0)
            return;
    }
    const Live L = live_of<ASYNC>(b);
    const int nd = b.nd;
    const int stage_bytes = pass_elem_bytes<MODE, C>(nd) * kTile;
    const unsigned full0 = smem_u32(smem);
    const unsigned empty0 = full0 + 8 * STAGES;
    TileDesc* desc = reinterpret_cast<TileDesc*>(smem + 16 * STAGES);
    char* stage0 = smem + kHdrBytes;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full0 + 8 * s, 1);       // the producer's expect_tx arrival
            mbar_init(empty0 + 8 * s, WARPS);  // one arrival per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == WARPS) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        int it = 0, r = 0;
        long long lo = 0, hi = 0;
        for (long long t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
            const int st = it % STAGES;
            const unsigned ph = (unsigned)(it / STAGES) & 1u;
            if (it >= STAGES && !mbar_wait(empty0 + 8 * st, ph ^ 1u, a.wait_rounds)) {
                atomicOr(a.err, err_bits<MODE>(1u));
                break;
            }
            if (t < lo || t >= hi) {
                r = find_tma_run<&TmaRun::tile_begin>(a.runs, a.n_runs, t);
                lo = a.runs[r].tile_begin;
                hi = (r + 1 < a.n_runs) ? a.runs[r + 1].tile_begin : a.n_tiles;
            }
            const TmaRun& run = a.runs[r];
            const long long body = run.len - run.head - run.tail;
            const long long e0 = run.head + (t - run.tile_begin) * kTile;
            const long long rem = run.head + body - e0;
            const int n = (int)(rem < kTile ? rem : kTile);
            if (t == a.hold_tile) continue;  // test hook: leave this stage unarmed
            TileDesc& d = desc[st];
            d.gi = run.grad_begin + e0;
            d.si = run.state_begin + e0;
            d.oi = run.out_begin + e0;
            d.n = n;
            d.decay = run.decay;
            char* sp = stage0 + st * stage_bytes;
            const unsigned full = full0 + 8 * st;
            if (!(in_bounds(d.gi, n, b.grad_len, a.err) & in_bounds(d.si, n, b.state_len, a.err) &
                  in_bounds(d.oi, n, b.out_len, a.err))) {
                d.n = 0;  // bounds-checked build: an empty tile, the stage completes at once
                mbar_expect_tx(full, 0u);
                continue;
            }
            mbar_expect_tx(full, (unsigned)n * (unsigned)pass_elem_bytes<MODE, C>(nd));
            if (MODE == kPassReduce) {
                for (int k = 0; k < nd; ++k)
                    bulk_g2s(smem_u32(sp + k * kTile * 2), b.grads[k] + d.gi, 2u * n, full);
            } else {
                bulk_g2s(smem_u32(sp), b.red + d.si, 4u * n, full);
                bulk_g2s(smem_u32(sp + 4 * kTile), L.m_in + d.si, 4u * n, full);
                bulk_g2s(smem_u32(sp + 8 * kTile), L.v_in + d.si, 4u * n, full);
                if (C::kMaster)
                    bulk_g2s(smem_u32(sp + 12 * kTile), L.w_in + d.si, 4u * n, full);
                else
                    bulk_g2s(smem_u32(sp + 12 * kTile), b.outs[0] + d.oi, 2u * n, full);
            }
        }
        // drain: every stage's last armed phase must have landed before exit
        for (int k = 0; k < STAGES && k < it; ++k) {
            const int i = it - 1 - k;
            if (!mbar_wait(full0 + 8 * (i % STAGES), (unsigned)(i / STAGES) & 1u, a.wait_rounds))
                atomicOr(a.err, err_bits<MODE>(2u));
        }
        return;
    }

    // ---------------- consumer warps ----------------
    bool bad = false;
    const int q4 = (warp * 32 + lane) * kQuad;  // this lane's quad in every tile
    int it = 0;
    for (long long t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
        const int st = it % STAGES;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(full0 + 8 * st, (unsigned)(it / STAGES) & 1u, a.wait_rounds));
        if (!ok) {
            if (lane == 0) atomicOr(a.err, err_bits<MODE>(4u));
            break;
        }
        const TileDesc d = desc[st];
        const bool active = q4 < d.n;
        const char* sp = stage0 + st * stage_bytes;
        if (MODE == kPassReduce) {
            float g[4];
            if (active) {
                const uint16_t* sg = reinterpret_cast<const uint16_t*>(sp);
                float x[4];
                unpack_as<C>(*reinterpret_cast<const uint2*>(sg + q4), g);
                for (int k = 1; k < nd; ++k) {
                    unpack_as<C>(*reinterpret_cast<const uint2*>(sg + k * kTile + q4), x);
#pragma unroll
                    for (int j = 0; j < 4; ++j) g[j] = __fadd_rn(g[j], x[j]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * st);  // the warp is done reading the stage
            if (active) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    g[j] = __fmul_rn(g[j], L.c.inv_scale);
                    bad |= nonfinite(g[j]);
                }
                __stcs(reinterpret_cast<float4*>(b.red + d.si + q4), make_float4(g[0], g[1], g[2], g[3]));
            }
        } else {
            float g[4], w[4], m[4], v[4];
            if (active) {
                const float* sf = reinterpret_cast<const float*>(sp);
                const float4 g4 = *reinterpret_cast<const float4*>(sf + q4);
                const float4 m4 = *reinterpret_cast<const float4*>(sf + kTile + q4);
                const float4 v4 = *reinterpret_cast<const float4*>(sf + 2 * kTile + q4);
                g[0] = g4.x; g[1] = g4.y; g[2] = g4.z; g[3] = g4.w;
                m[0] = m4.x; m[1] = m4.y; m[2] = m4.z; m[3] = m4.w;
                v[0] = v4.x; v[1] = v4.y; v[2] = v4.z; v[3] = v4.w;
                if (C::kMaster) {
                    const float4 w4 = *reinterpret_cast<const float4*>(sf + 3 * kTile + q4);
                    w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
                } else {
                    unpack_as<C>(*reinterpret_cast<const uint2*>(sp + 12 * kTile + 2 * q4), w);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * st);
            if (active) {
                const float wd = d.decay ? L.c.wd : 0.0f;
#pragma unroll
                for (int j = 0; j < 4; ++j) adam1(g[j], w[j], m[j], v[j], L.c, wd);
                // state indices are 4-element and output indices 8-element
                // aligned with the gradient index (the host's eligibility rule)
                if (C::kMaster)
                    __stcs(reinterpret_cast<float4*>(L.w_out + d.si + q4), make_float4(w[0], w[1], w[2], w[3]));
                __stcs(reinterpret_cast<float4*>(L.m_out + d.si + q4), make_float4(m[0], m[1], m[2], m[3]));
                __stcs(reinterpret_cast<float4*>(L.v_out + d.si + q4), make_float4(v[0], v[1], v[2], v[3]));
                const uint2 h = pack_as<C>(w);
                for (int k = 0; k < b.n_out; ++k) __stcs(reinterpret_cast<uint2*>(b.outs[k] + d.oi + q4), h);
            }
        }
    }

    // scalar items (heads and tails of the runs), straight from global memory
    constexpr int n_cons_cta = WARPS * 32;
    const long long n_cons = (long long)gridDim.x * n_cons_cta;
    int r = 0;
    long long lo = 0, hi = 0;
    for (long long j = (long long)blockIdx.x * n_cons_cta + tid; j < a.n_scal; j += n_cons) {
        if (j < lo || j >= hi) {
            r = find_tma_run<&TmaRun::scal_begin>(a.runs, a.n_runs, j);
            lo = a.runs[r].scal_begin;
            hi = (r + 1 < a.n_runs) ? a.runs[r + 1].scal_begin : a.n_scal;
        }
        const TmaRun& run = a.runs[r];
        const long long q = j - run.scal_begin;
        SegDesc sd;
        sd.grad_begin = run.grad_begin;
        sd.state_begin = run.state_begin;
        sd.out_begin = run.out_begin;
        sd.len = run.len;
        sd.chunk_begin = 0;
        sd.head = run.head;
        sd.tail = run.tail;
        sd.decay = run.decay;
        const long long e = q < run.head ? q : run.len - run.tail + (q - run.head);
        if (MODE == kPassReduce)
            step_scalar<K_REDUCE, C>(b, L, b.grads, b.outs, sd, e, bad);
        else
            step_scalar<K_UPDATE, C>(b, L, b.grads, b.outs, sd, e, bad);
    }

    if (MODE == kPassReduce) {
        // one atomic per consumer warp that saw a non-finite unscaled gradient
        if (__any_sync(0xffffffffu, bad) && lane == 0) atomicMax(b.flag, b.call_id);
    }
}

template <int MODE, bool ASYNC, class C>
const void* pass_kernel(TmaShape sh)
{
    if (sh.warps == kTmaWide.warps && sh.stages == kTmaWide.stages)
        return reinterpret_cast<const void*>(&pass_tma_kernel<MODE, kTmaWide.warps, kTmaWide.stages, ASYNC, C>);
    if (sh.warps == kTmaDeep.warps && sh.stages == kTmaDeep.stages)
        return reinterpret_cast<const void*>(&pass_tma_kernel<MODE, kTmaDeep.warps, kTmaDeep.stages, ASYNC, C>);
    return nullptr;
}

template <int MODE, class C>
int pass_smem(TmaShape sh, int nd)
{
    return kHdrBytes + sh.stages * pass_elem_bytes<MODE, C>(nd) * sh.tile;
}

template <int MODE, class C>
cudaError_t prepare_mode(TmaShape sh, int nd, int* blocks_per_sm)
{
    const void* f = pass_kernel<MODE, false, C>(sh);
    const void* fa = pass_kernel<MODE, true, C>(sh);
    if (!f || !fa) return cudaErrorInvalidValue;
    const int smem = pass_smem<MODE, C>(sh, nd);
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fa, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int occ = 0, occ_a = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, f, (sh.warps + 1) * 32, smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_a, fa, (sh.warps + 1) * 32, smem);
    *blocks_per_sm = occ < occ_a ? occ : occ_a;
    return e;
}

template <int MODE, class C>
cudaError_t launch_mode(TmaShape sh, const TmaArgs& a, int grid, cudaStream_t s)
{
    // only the two instantiated shapes
    const void* f = a.b.ctrl ? pass_kernel<MODE, true, C>(sh) : pass_kernel<MODE, false, C>(sh);
    if (!f) return cudaErrorInvalidValue;
    const int smem = pass_smem<MODE, C>(sh, a.b.nd);
    const int threads = (sh.warps + 1) * 32;
    if (sh.warps == kTmaWide.warps) {
        if (a.b.ctrl)
            pass_tma_kernel<MODE, kTmaWide.warps, kTmaWide.stages, true, C><<<grid, threads, smem, s>>>(a);
        else
            pass_tma_kernel<MODE, kTmaWide.warps, kTmaWide.stages, false, C><<<grid, threads, smem, s>>>(a);
    } else {
        if (a.b.ctrl)
            pass_tma_kernel<MODE, kTmaDeep.warps, kTmaDeep.stages, true, C><<<grid, threads, smem, s>>>(a);
        else
            pass_tma_kernel<MODE, kTmaDeep.warps, kTmaDeep.stages, false, C><<<grid, threads, smem, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t tma_pass_prepare(int nd, int n_out, bool bf16, int* occ_reduce, int* occ_update)
{
    const TmaShape rs = tma_pass_shape(kPassReduce, n_out), us = tma_pass_shape(kPassUpdate, n_out);
    cudaError_t e;
    if (bf16) {
        e = prepare_mode<kPassReduce, BF16>(rs, nd, occ_reduce);
        if (e == cudaSuccess) e = prepare_mode<kPassUpdate, BF16>(us, nd, occ_update);
    } else {
        e = prepare_mode<kPassReduce, F16>(rs, nd, occ_reduce);
        if (e == cudaSuccess) e = prepare_mode<kPassUpdate, F16>(us, nd, occ_update);
    }
    return e;
}

cudaError_t launch_pass_tma(int mode, const TmaArgs& a, int grid, cudaStream_t s, bool bf16)
{
    const TmaShape sh = tma_pass_shape(mode, a.b.n_out);
    if (mode == kPassReduce)
        return bf16 ? launch_mode<kPassReduce, BF16>(sh, a, grid, s) : launch_mode<kPassReduce, F16>(sh, a, grid, s);
    return bf16 ? launch_mode<kPassUpdate, BF16>(sh, a, grid, s) : launch_mode<kPassUpdate, F16>(sh, a, grid, s);
}

}  // namespace zk
