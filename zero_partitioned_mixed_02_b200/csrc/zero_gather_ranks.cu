// The layer gather of a real stage-3 rank (zero_gather_ranks.h): a copy kernel
// bound by memory (and, across GPUs, by NVLink) bandwidth. Each block takes
// tiles of 16 KB in turn; a tile is a piece of one rank's chunk, copied with
// 16-byte loads and stores where source and destination share their offset
// within 16 bytes, element by element otherwise.
#include "zero_gather_ranks.h"

namespace zg {
namespace {

__device__ __forceinline__ void copy_span(const uint16_t* __restrict__ src, uint16_t* __restrict__ dst, int64_t n)
{
    const int bd = blockDim.x;
    const uintptr_t sa = reinterpret_cast<uintptr_t>(src), da = reinterpret_cast<uintptr_t>(dst);
    if (((sa ^ da) & 15) != 0) {
        for (int64_t i = threadIdx.x; i < n; i += bd) dst[i] = src[i];
        return;
    }
    int64_t head = (int64_t)(((16 - (sa & 15)) & 15) >> 1);
    if (head > n) head = n;
    const int64_t body = (n - head) >> 3;
    for (int64_t i = threadIdx.x; i < head; i += bd) dst[i] = src[i];
    const uint4* __restrict__ s4 = reinterpret_cast<const uint4*>(src + head);
    uint4* __restrict__ d4 = reinterpret_cast<uint4*>(dst + head);
    int64_t i = threadIdx.x;
    for (; i + 3 * bd < body; i += 4 * bd) {  // four loads in flight per thread
        const uint4 x0 = s4[i], x1 = s4[i + bd], x2 = s4[i + 2 * bd], x3 = s4[i + 3 * bd];
        d4[i] = x0;
        d4[i + bd] = x1;
        d4[i + 2 * bd] = x2;
        d4[i + 3 * bd] = x3;
    }
    for (; i < body; i += bd) d4[i] = s4[i];
    for (int64_t j = head + body * 8 + threadIdx.x; j < n; j += bd) dst[j] = src[j];
}

__global__ void __launch_bounds__(kThreads) gather_ranks_kernel(const Args a)
{
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
        // the last run whose first tile is at or before this one
        int lo = 0, hi = a.n_runs - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (a.runs[mid].tile_begin <= tile) lo = mid;
            else hi = mid - 1;
        }
        const Run r = a.runs[lo];
        const int64_t e0 = (tile - r.tile_begin) * kTile;
        const int64_t n = r.len - e0 < kTile ? r.len - e0 : kTile;
#ifdef ZK_BOUNDS_CHECK
        if (r.rank < 0 || r.rank >= a.nd || e0 < 0 || n <= 0 || r.src_begin < 0 || r.out_begin < 0 ||
            r.src_begin + e0 + n > a.shard_len[r.rank] || r.out_begin + e0 + n > a.dst_len) {
            if (threadIdx.x == 0) atomicOr(a.err, 32u);
            continue;
        }
#endif
        copy_span(a.shards[r.rank] + r.src_begin + e0, a.dst + r.out_begin + e0, n);
    }
}

}  // namespace

cudaError_t occupancy(int* blocks_per_sm)
{
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, gather_ranks_kernel, kThreads, 0);
}

cudaError_t launch(const Args& a, int grid, cudaStream_t s)
{
    if (a.n_tiles <= 0 || grid <= 0) return cudaSuccess;
    gather_ranks_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace zg
