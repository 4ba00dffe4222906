// NVTX ranges around the library's entry points, so that a profiler's timeline (Nsight
// Systems, or ncu with --nvtx) names the host call each kernel launch came from.  NVTX v3 is
// header-only: with no profiler attached a range costs a check of a function pointer.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace ug {

struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

}  // namespace ug
