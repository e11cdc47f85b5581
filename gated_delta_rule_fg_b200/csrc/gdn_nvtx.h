// gdn_nvtx.h -- one NVTX range per public call (named after the entry point), so that a
// profiler timeline shows each call's kernels under its name.  NVTX v3 is header-only; with no
// tool attached a range costs a few nanoseconds on the host.
#pragma once
#include <nvtx3/nvToolsExt.h>

namespace gdn {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace gdn
