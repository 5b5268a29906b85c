// focus_trace.cuh -- NVTX ranges around the library's entry points.
//
// Every C-ABI call that enqueues work or waits opens a range named after the
// call (nvtxRangePushA / nvtxRangePop from the header-only NVTX 3 API, which
// costs a few nanoseconds and does nothing unless a profiler such as Nsight
// Systems is attached).  Building with -DFOCUS_NO_NVTX removes them.
#pragma once

#ifndef FOCUS_NO_NVTX
#include <nvtx3/nvToolsExt.h>

namespace focus {
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};
}  // namespace focus

#define FOCUS_RANGE() ::focus::NvtxRange focus_nvtx_range_(__func__)
#else
#define FOCUS_RANGE() ((void)0)
#endif
