// NVTX ranges around the ABI calls, so a profiler's timeline shows inject,
// draft and verify as named spans. The NVTX v3 API is header-only: without a
// profiler attached each push/pop is a no-op call.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace dfl {

struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};

}  // namespace dfl
