// NVTX ranges around the C-ABI calls (host code).  Built with -DLUTQ_NVTX,
// LUTQ_TRACE_RANGE(name) opens a range named `name` for the rest of the
// enclosing scope, so a timeline (Nsight Systems) shows every library call
// and the kernels it launched beneath it; otherwise it is empty.  The NVTX 3
// headers are header-only: without a tool attached, a range costs a branch.
#pragma once

#ifdef LUTQ_NVTX
#include <nvtx3/nvToolsExt.h>

namespace lutq {
struct TraceRange {
  explicit TraceRange(const char* name) { nvtxRangePushA(name); }
  ~TraceRange() { nvtxRangePop(); }
  TraceRange(const TraceRange&) = delete;
  TraceRange& operator=(const TraceRange&) = delete;
};
}  // namespace lutq
#define LUTQ_TRACE_RANGE(name) ::lutq::TraceRange lutq_trace_range_(name)
#else
#define LUTQ_TRACE_RANGE(name) ((void)0)
#endif
