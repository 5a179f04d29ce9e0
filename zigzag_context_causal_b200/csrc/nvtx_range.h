// A named NVTX range around each C-ABI call that enqueues GPU work, so the
// calls show up on Nsight timelines.  NVTX is header-only here; without a
// profiler attached a push/pop costs a branch.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace zz {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace zz

#define ZZ_NVTX(name) ::zz::NvtxRange zz_nvtx_range_(name)
