// NVTX ranges around the C-ABI calls, so that a profiler's timeline names each
// library call (Nsight Systems, or ncu's NVTX filters).  Host side only: with
// no tool attached an NVTX call returns at once, and nothing here touches the
// device or the stream.
#pragma once

#include <nvtx3/nvToolsExt.h>

namespace lcvq {

struct ApiRange {
  explicit ApiRange(const char* name) { nvtxRangePushA(name); }
  ~ApiRange() { nvtxRangePop(); }
  ApiRange(const ApiRange&) = delete;
  ApiRange& operator=(const ApiRange&) = delete;
};

}  // namespace lcvq

// one range per call, named after the entry point, closed on every return path
#define LCVQ_API_RANGE() const ::lcvq::ApiRange lcvq_api_range_(__func__)
