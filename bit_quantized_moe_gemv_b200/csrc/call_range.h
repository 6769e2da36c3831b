// One NVTX range per C-ABI call, named after the call, so a profiler's
// timeline groups each call's kernel launches under it. Host code only; with
// no tool attached the push and pop are no-ops.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace moe {

struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

}  // namespace moe
