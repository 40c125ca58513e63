// The fused step with TMA staging (sm_100a).
//
// Persistent CTAs: the last warp is the producer, the others consume. The
// kernel is instantiated for the two shapes of zero_internal.h (consumer
// warps x input stages). The producer's lane 0 stages each tile -- the Nd fp16 gradient
// slices and the fp32 master/m/v of TILE elements -- into one of
// STAGES shared-memory stages with 1D bulk asynchronous copies
// (cp.async.bulk; completion counted in bytes on the stage's "full" mbarrier),
// running up to STAGES tiles ahead of the consumers; a stage is released as
// soon as every consumer warp has read it, before the arithmetic and stores. Each consumer warp
// waits for the tile on its own, reduces, unscales, checks and runs Adam on
// its 32 quads straight out of shared memory, writes the new master/m/v and
// the fp16 parameters to global memory with streaming stores, and releases the
// stage with one arrival on its "empty" mbarrier. Warps never wait on each
// other: there is no CTA-wide barrier after set-up.
//
// Every wait is bounded. A warp that gives up sets the error word and leaves
// its loop (the producer then gives up on that stage too); the producer drains
// its own copies in flight before it returns. No cluster multicast.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_device.cuh"
#include "zero_internal.h"
#include "zero_tma.cuh"

namespace zk {
namespace {

// The kernel body. ASYNC: PAR is the live state buffer, a compile-time
// index, so that every state pointer is a kernel argument as in the
// synchronous form (the kernel branches once, uniformly, on the control
// block's live index).
// C: the element format (F16 with an fp32 master; BF16 without one, whose
// weight is read from output b.w_src and written to all outputs but the last
// b.keep_last, the copy a skipped step is restored from).
template <int WARPS, int STAGES, bool ASYNC, int PAR, class C>
__device__ __forceinline__ void step_tma_body(const TmaArgs& a)
{
    static_assert(STAGES <= kMaxStages, "too many stages");
    constexpr int kTmaConsumerWarps = WARPS;
    constexpr int kTmaStages = STAGES;
    constexpr int kTmaTile = WARPS * 32 * kQuad;
    constexpr int kWBytes = C::kMaster ? 4 : 2;  // bytes of the staged weight
    extern __shared__ __align__(128) char smem[];
    const StepArgs& b = a.b;
    const Live L = live_at<ASYNC, PAR>(b);
    const int nd = b.nd;
    const unsigned full0 = smem_u32(smem);
    const unsigned empty0 = full0 + 8 * kTmaStages;
    TileDesc* desc = reinterpret_cast<TileDesc*>(smem + 16 * kTmaStages);
    const int stage_bytes = nd * kTmaTile * 2 + kTmaTile * (kWBytes + 8);
    char* stage0 = smem + kHdrBytes;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(full0 + 8 * s, 1);                   // the producer's expect_tx arrival
            mbar_init(empty0 + 8 * s, kTmaConsumerWarps);  // one arrival per consumer warp
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    if (warp == kTmaConsumerWarps) {
        // ---------------- producer ----------------
        if (lane != 0) return;
        int it = 0, r = 0;
        long long lo = 0, hi = 0;  // tile range of run r
        for (long long t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
            const int st = it % kTmaStages;
            const unsigned ph = (unsigned)(it / kTmaStages) & 1u;
            if (it >= kTmaStages && !mbar_wait(empty0 + 8 * st, ph ^ 1u, a.wait_rounds)) {
                atomicOr(a.err, 1u);
                break;
            }
            if (t < lo || t >= hi) {
                r = find_tma_run<&TmaRun::tile_begin>(a.runs, a.n_runs, t);
                lo = a.runs[r].tile_begin;
                hi = (r + 1 < a.n_runs) ? a.runs[r + 1].tile_begin : a.n_tiles;
            }
            const TmaRun& run = a.runs[r];
            const long long body = run.len - run.head - run.tail;
            const long long e0 = run.head + (t - run.tile_begin) * kTmaTile;
            const long long rem = run.head + body - e0;
            const int n = (int)(rem < kTmaTile ? rem : kTmaTile);
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
            mbar_expect_tx(full, (unsigned)n * (unsigned)(2 * nd + kWBytes + 8));
            for (int k = 0; k < nd; ++k)
                bulk_g2s(smem_u32(sp + k * kTmaTile * 2), b.grads[k] + d.gi, 2u * n, full);
            char* sw = sp + nd * kTmaTile * 2;
            if (C::kMaster)
                bulk_g2s(smem_u32(sw), L.w_in + d.si, 4u * n, full);
            else
                bulk_g2s(smem_u32(sw), b.outs[b.w_src] + d.oi, 2u * n, full);
            bulk_g2s(smem_u32(sw + kTmaTile * kWBytes), L.m_in + d.si, 4u * n, full);
            bulk_g2s(smem_u32(sw + kTmaTile * kWBytes + kTmaTile * 4), L.v_in + d.si, 4u * n, full);
        }
        // drain: every stage's last armed phase must have landed before exit
        for (int k = 0; k < kTmaStages && k < it; ++k) {
            const int i = it - 1 - k;
            if (!mbar_wait(full0 + 8 * (i % kTmaStages), (unsigned)(i / kTmaStages) & 1u, a.wait_rounds))
                atomicOr(a.err, 2u);
        }
        return;
    }

    // ---------------- consumer warps ----------------
    bool bad = false;
    const int q4 = (warp * 32 + lane) * kQuad;  // this lane's quad in every tile
    int it = 0;
    for (long long t = blockIdx.x; t < a.n_tiles; t += gridDim.x, ++it) {
        const int st = it % kTmaStages;
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait(full0 + 8 * st, (unsigned)(it / kTmaStages) & 1u, a.wait_rounds));
        if (!ok) {
            if (lane == 0) atomicOr(a.err, 4u);
            break;
        }
        const TileDesc d = desc[st];
        const bool active = q4 < d.n;
        float g[4], w[4], m[4], v[4];
        if (active) {
            const char* sp = stage0 + st * stage_bytes;
            const uint16_t* sg = reinterpret_cast<const uint16_t*>(sp);
            const char* sw = sp + nd * kTmaTile * 2;
            const float* smv = reinterpret_cast<const float*>(sw + kTmaTile * kWBytes);
            float x[4];
            unpack_as<C>(*reinterpret_cast<const uint2*>(sg + q4), g);
            for (int k = 1; k < nd; ++k) {
                unpack_as<C>(*reinterpret_cast<const uint2*>(sg + k * kTmaTile + q4), x);
#pragma unroll
                for (int j = 0; j < 4; ++j) g[j] = __fadd_rn(g[j], x[j]);
            }
            if (C::kMaster) {
                const float4 w4 = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(sw) + q4);
                w[0] = w4.x; w[1] = w4.y; w[2] = w4.z; w[3] = w4.w;
            } else {
                unpack_as<C>(*reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(sw) + q4), w);
            }
            const float4 m4 = *reinterpret_cast<const float4*>(smv + q4);
            const float4 v4 = *reinterpret_cast<const float4*>(smv + kTmaTile + q4);
            m[0] = m4.x; m[1] = m4.y; m[2] = m4.z; m[3] = m4.w;
            v[0] = v4.x; v[1] = v4.y; v[2] = v4.z; v[3] = v4.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * st);  // the warp is done reading the stage
        if (active) {
            const float wd = d.decay ? L.c.wd : 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                g[j] = __fmul_rn(g[j], L.c.inv_scale);
                bad |= nonfinite(g[j]);
                adam1(g[j], w[j], m[j], v[j], L.c, wd);
            }
            // state indices are 4-element and output indices 8-element aligned
            // with the gradient index (the host's eligibility rule)
            if (C::kMaster)
                __stcs(reinterpret_cast<float4*>(L.w_out + d.si + q4), make_float4(w[0], w[1], w[2], w[3]));
            __stcs(reinterpret_cast<float4*>(L.m_out + d.si + q4), make_float4(m[0], m[1], m[2], m[3]));
            __stcs(reinterpret_cast<float4*>(L.v_out + d.si + q4), make_float4(v[0], v[1], v[2], v[3]));
            const uint2 h = pack_as<C>(w);
            const int n_write = b.n_out - b.keep_last;
            for (int k = 0; k < n_write; ++k) __stcs(reinterpret_cast<uint2*>(b.outs[k] + d.oi + q4), h);
        }
    }

    // scalar items (heads and tails of the runs), straight from global memory
    constexpr int n_cons_cta = kTmaConsumerWarps * 32;
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
        step_scalar<K_STEP_FUSED, C>(b, L, b.grads, b.outs, sd, e, bad);
    }

    // one atomic per consumer warp that saw a non-finite unscaled gradient
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicMax(b.flag, b.call_id);
}

template <int WARPS, int STAGES, bool ASYNC, class C>
__global__ void __launch_bounds__((WARPS + 1) * 32, 1) step_tma_kernel(const TmaArgs a)
{
    if (!ASYNC)
        step_tma_body<WARPS, STAGES, false, 0, C>(a);
    else if (a.b.ctrl->cur == 0)
        step_tma_body<WARPS, STAGES, true, 0, C>(a);
    else
        step_tma_body<WARPS, STAGES, true, 1, C>(a);
}

int smem_bytes(TmaShape sh, int nd, bool bf16)
{
    return kHdrBytes + sh.stages * (nd * sh.tile * 2 + sh.tile * ((bf16 ? 2 : 4) + 8));
}

template <bool ASYNC, class C>
const void* kernel_for(TmaShape sh)
{
    if (sh.warps == kTmaWide.warps && sh.stages == kTmaWide.stages)
        return reinterpret_cast<const void*>(&step_tma_kernel<kTmaWide.warps, kTmaWide.stages, ASYNC, C>);
    if (sh.warps == kTmaDeep.warps && sh.stages == kTmaDeep.stages)
        return reinterpret_cast<const void*>(&step_tma_kernel<kTmaDeep.warps, kTmaDeep.stages, ASYNC, C>);
    return nullptr;
}

template <int WARPS, int STAGES, class C>
void launch_shape(const TmaArgs& a, int grid, int threads, int smem, cudaStream_t s)
{
    if (a.b.ctrl != nullptr)
        step_tma_kernel<WARPS, STAGES, true, C><<<grid, threads, smem, s>>>(a);
    else
        step_tma_kernel<WARPS, STAGES, false, C><<<grid, threads, smem, s>>>(a);
}

}  // namespace

// Both the synchronous and the asynchronous kernel of the shape get the
// shared-memory attribute; the reported occupancy is the smaller of the two.
cudaError_t tma_prepare(TmaShape sh, int nd, bool bf16, int* blocks_per_sm)
{
    const void* f = bf16 ? kernel_for<false, BF16>(sh) : kernel_for<false, F16>(sh);
    const void* fa = bf16 ? kernel_for<true, BF16>(sh) : kernel_for<true, F16>(sh);
    if (!f || !fa) return cudaErrorInvalidValue;
    const int smem = smem_bytes(sh, nd, bf16);
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(fa, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    int occ = 0, occ_a = 0;
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, f, (sh.warps + 1) * 32, smem);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_a, fa, (sh.warps + 1) * 32, smem);
    *blocks_per_sm = occ < occ_a ? occ : occ_a;
    return e;
}

cudaError_t launch_step_tma(TmaShape sh, const TmaArgs& a, int grid, cudaStream_t s, bool bf16)
{
    const int smem = smem_bytes(sh, a.b.nd, bf16);
    const int threads = (sh.warps + 1) * 32;
    if (sh.warps == kTmaWide.warps && sh.stages == kTmaWide.stages) {
        if (bf16) launch_shape<kTmaWide.warps, kTmaWide.stages, BF16>(a, grid, threads, smem, s);
        else launch_shape<kTmaWide.warps, kTmaWide.stages, F16>(a, grid, threads, smem, s);
    } else if (sh.warps == kTmaDeep.warps && sh.stages == kTmaDeep.stages) {
        if (bf16) launch_shape<kTmaDeep.warps, kTmaDeep.stages, BF16>(a, grid, threads, smem, s);
        else launch_shape<kTmaDeep.warps, kTmaDeep.stages, F16>(a, grid, threads, smem, s);
    } else {
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace zk
