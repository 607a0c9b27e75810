// Optional NVTX ranges around the C-ABI entry points, so that a timeline
// profiler shows each rt_* call as a named range.  Compiled in only with
// -DRT_NVTX (the build's RT_NVTX=1 environment switch); otherwise RT_RANGE
// expands to nothing.  NVTX v3 is header-only: without a profiler attached
// the push/pop calls return at once.
#pragma once

#ifdef RT_NVTX
#include <nvtx3/nvToolsExt.h>

namespace rtb {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace rtb
#define RT_RANGE(name) ::rtb::NvtxRange rt_nvtx_range_(name)
#else
#define RT_RANGE(name) ((void)0)
#endif
