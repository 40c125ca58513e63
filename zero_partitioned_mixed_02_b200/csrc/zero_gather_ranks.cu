// The stage-3 layer gather (zero_gather_ranks.h), for emulated ranks and for a
// rank of a real job: a copy kernel bound by memory (and, across GPUs, by
// NVLink) bandwidth. Each block takes tiles of 16 KB in turn; a tile is a
// piece of one rank's chunk, copied with 16-byte loads and stores where source
// and destination share their offset within 16 bytes, element by element
// otherwise. Launched as a programmatic dependent (zero_pdl.cuh).
#include "zero_gather_ranks.h"
#include "zero_pdl.cuh"

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
    for (; i + (kUnroll - 1) * bd < body; i += kUnroll * bd) {  // kUnroll loads in flight per thread
        uint4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) x[k] = s4[i + k * bd];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) d4[i + k * bd] = x[k];
    }
    for (; i < body; i += bd) d4[i] = s4[i];
    for (int64_t j = head + body * 8 + threadIdx.x; j < n; j += bd) dst[j] = src[j];
}

// the last run whose first tile is at or before `tile`
__device__ __forceinline__ int find_run(const Run* runs, int n_runs, int64_t tile)
{
    int lo = 0, hi = n_runs - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (runs[mid].tile_begin <= tile) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Tiles go to blocks round robin (tile = block + k * grid), so the whole grid
// copies one narrow, advancing window of the unit at a time. kMinBlocks blocks
// of kThreads per SM with kUnroll 16-byte loads in flight per thread (64 KB
// per SM) measured fastest on the Llama layer walk: more bytes in flight per
// SM (more blocks, or 8 loads per thread), contiguous spans of tiles per block,
// 512-thread blocks, streaming cache hints (on loads, on stores, or both) and
// the read-only load path were all slower; 128-thread blocks (8 per SM) were
// the same within noise.
__global__ void __launch_bounds__(kThreads, kMinBlocks) layer_gather_kernel(const Args a)
{
    // a programmatic dependent launch: wait for the previous kernel on the stream
    zk::pdl_wait();
    zk::pdl_launch_dependents();
    for (int64_t tile = blockIdx.x; tile < a.n_tiles; tile += gridDim.x) {
        const Run r = a.runs[find_run(a.runs, a.n_runs, tile)];
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
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks_per_sm, layer_gather_kernel, kThreads, 0);
}

cudaError_t launch(const Args& a, int grid, cudaStream_t s)
{
    if (a.n_tiles <= 0 || grid <= 0) return cudaSuccess;
    return zk::launch_pdl(layer_gather_kernel, dim3(grid), dim3(kThreads), 0, s, a);
}

}  // namespace zg
