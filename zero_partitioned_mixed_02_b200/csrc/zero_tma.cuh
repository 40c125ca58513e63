// Device helpers of the TMA-staged kernels (zero_tma.cu, zero_tma_pass.cu):
// mbarriers with bounded waits, 1D bulk asynchronous copies global -> shared,
// the per-stage tile descriptor and the run lookup. Internal to libzero.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "zero_internal.h"

namespace zk {
namespace {

constexpr int kHdrBytes = 1024;             // barriers and tile descriptors

struct TileDesc {
    long long gi, si, oi;
    int n;
    int decay;
};
constexpr int kMaxStages = 8;
static_assert(16 * kMaxStages + sizeof(TileDesc) * kMaxStages <= kHdrBytes, "header overflow");

__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(unsigned bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(unsigned bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(unsigned bar, unsigned parity)
{
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000u)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of parity `parity` to complete.
__device__ __forceinline__ bool mbar_wait(unsigned bar, unsigned parity, unsigned rounds)
{
    for (unsigned i = 0; i < rounds; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ void bulk_g2s(unsigned dst, const void* src, unsigned bytes, unsigned bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Largest index whose begin field is <= x.
template <long long TmaRun::*F>
__device__ __forceinline__ int find_tma_run(const TmaRun* runs, int n, long long x)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (runs[mid].*F <= x)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

}  // namespace
}  // namespace zk
