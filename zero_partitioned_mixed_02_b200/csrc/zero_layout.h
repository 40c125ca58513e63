// Partitions, run tables and workspace layout that follow from a zero_config
// (built in zero_abi.cu), shared by the device-resident handle and the
// host-offload handle. Internal to libzero.
#pragma once

#include <algorithm>
#include <cstdint>
#include <vector>

#include "zero.h"
#include "zero_gather_ranks.h"
#include "zero_internal.h"

namespace zl {

// Ceil split ([P1] "The replication nobody questioned": the state is divided
// across the Nd ranks; trailing ranks may be short or empty).
inline void split(int64_t n, int nd, int r, int64_t* b, int64_t* e)
{
    const int64_t p = (n + nd - 1) / nd;
    *b = std::min<int64_t>((int64_t)r * p, n);
    *e = std::min<int64_t>(*b + p, n);
}

struct Unit {
    int64_t seg0 = 0;     // first gather run of the unit
    int64_t n_segs = 0;
    int64_t n_chunks = 0;
    int64_t flat_begin = 0;
    int64_t numel = 0;
    // the unit's runs from the Nd ranks' shards (the layer gather's table)
    int64_t rank_run0 = 0;
    int64_t rank_n_runs = 0;
    int64_t rank_tiles = 0;
};

// Everything that follows from a configuration: partitions, run tables,
// ledger and workspace layout.
struct Layout {
    int64_t psi = 0;
    int nd = 0, stage = 0, view = -1, variant = 0;
    bool bf16 = false;  // ZERO_PRECISION_BF16: bfloat16 streams, no fp32 master
    std::vector<int64_t> numel;  // tensor sizes (one flat tensor if none given)
    std::vector<int32_t> unit_of;
    std::vector<int> decay_of;   // per tensor: 1 unless flagged ZERO_TENSOR_NO_DECAY
    int64_t P = 0, state_elems = 0, grad_len = 0;
    int n_out = 0, n_units = 0;
    std::vector<int64_t> shard_begin, shard_len;  // per rank, in state elements
    std::vector<zk::SegDesc> step_segs;
    int64_t step_chunks = 0;
    std::vector<zk::SegDesc> gather_segs;  // the offloaded step's layer gather (one shard array)
    std::vector<Unit> units;
    std::vector<zg::Run> rank_gather;  // stage 3: the layer gathers' runs of all units, by source rank
    std::vector<zk::TmaRun> tma_runs;  // TMA variants, when every run is eligible
    bool tma_ok = false;
    zk::TmaShape tma_shape = zk::kTmaDeep;
    int64_t tma_tiles = 0, tma_scal = 0;
    // two-pass TMA variant: the reduce pass's table (its own tile size)
    std::vector<zk::TmaRun> tma_runs_r;
    zk::TmaShape tma_shape_r = zk::kTmaDeep;
    int64_t tma_tiles_r = 0, tma_scal_r = 0;
    int64_t off_flag = 0, off_grad_tab = 0, off_out_tab = 0, off_step_segs = 0,
            off_tma_runs = -1, off_tma_runs_r = -1, off_reduced = -1,
            off_shard16 = -1, off_shard_tab = -1, off_rank_gather = -1,
            total = 0;
    int64_t off_state[2][3] = {{-1, -1, -1}, {-1, -1, -1}};
    int64_t transient_elems = 0;
};

// Validate cfg and fill L; ZERO_OK or ZERO_ERR_ARG.
int build_layout(const zero_config* cfg, Layout* L);

}  // namespace zl
