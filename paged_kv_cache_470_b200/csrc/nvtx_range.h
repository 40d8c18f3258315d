// A named NVTX range around one call of the C ABI: it shows the call on a
// profiler's timeline (Nsight Systems, ncu's NVTX filters) and costs a few
// nanoseconds when no tool is attached (NVTX 3 is header-only and loads its
// backend only if a tool asks for it).
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace pkv_host {

struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

}  // namespace pkv_host
