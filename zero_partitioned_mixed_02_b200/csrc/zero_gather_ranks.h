// The stage-3 layer gather ([P1] "The part that sounds too good:
// communication": stage 3 all-gathers each layer's parameters on demand,
// forward and backward; [P2] "ZeRO and the Memory Tricks" -- "The
// Breakthrough"): the fp16 chunks of one layer unit are copied from the Nd
// ranks' shards into one contiguous buffer in tensor order. The shards are
// places in one shard array when the Nd ranks are emulated on one GPU, or a
// real rank's own shard and the other ranks' (peer-mapped). Internal to libzero.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace zg {

// One rank's chunk of one tensor of a unit. Runs are listed in the unit's
// output order; tiles of kTile elements are numbered across the unit's runs.
struct Run {
    int64_t src_begin;   // element offset in the source rank's shard
    int64_t out_begin;   // element offset in the gathered unit
    int64_t len;         // elements, > 0
    int64_t tile_begin;  // the run's first tile
    int32_t rank;        // source rank
    int32_t pad[3];
};
static_assert(sizeof(Run) == 48, "run layout");

#ifndef ZG_TILE
#define ZG_TILE 8192
#endif
#ifndef ZG_UNROLL
#define ZG_UNROLL 4
#endif
#ifndef ZG_MIN_BLOCKS
#define ZG_MIN_BLOCKS 4
#endif
constexpr int64_t kTile = ZG_TILE;  // elements per tile (16 KB of fp16)
constexpr int kThreads = 256;
constexpr int kUnroll = ZG_UNROLL;  // 16-byte loads in flight per thread
constexpr int kMinBlocks = ZG_MIN_BLOCKS;  // resident blocks per SM the registers are capped for

struct Args {
    const Run* runs;
    int n_runs;
    int nd;
    int64_t n_tiles;
    const uint16_t* const* shards;  // device table: Nd shard addresses
    const int64_t* shard_len;       // device table: Nd shard lengths (elements)
    uint16_t* dst;
    int64_t dst_len;
    unsigned* err;                  // kernel-error word (bounds-checked build)
};

// Tiles of `n` elements of a run: ceil(n / kTile).
inline int64_t tiles_of(int64_t n) { return (n + kTile - 1) / kTile; }

cudaError_t occupancy(int* blocks_per_sm);
cudaError_t launch(const Args& a, int grid, cudaStream_t s);

}  // namespace zg
