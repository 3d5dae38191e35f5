// NVTX ranges for the C entry points: a profiler's timeline shows each library
// call (its host validation and launches) above the kernels it enqueued.  NVTX 3
// is header-only; with no profiler attached a push or pop is one predictable
// branch.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace pa {

struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

}  // namespace pa
