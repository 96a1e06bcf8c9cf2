// m3_nvtx.h -- NVTX ranges around the host calls of the C ABI.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace m3 {

// An NVTX range around a host call (header-only NVTX 3: a no-op unless a
// profiler is attached).  Every compute entry point of the C ABI opens one
// named after itself, so `ncu --nvtx --nvtx-include "m3_step/"` and the like
// select a call's kernels.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace m3
