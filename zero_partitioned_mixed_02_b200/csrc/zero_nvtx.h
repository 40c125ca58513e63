// NVTX ranges around the host calls that enqueue work (header-only NVTX 3:
// no library to link; without a profiler attached a range costs a few
// nanoseconds). Internal to libzero.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace zk {

struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace zk
