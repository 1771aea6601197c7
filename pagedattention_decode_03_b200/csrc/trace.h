// Library log and profiler ranges.
//
// Log: the environment variable PA_LOG, read once per process, sets the level
//   0 (unset, empty or not a number)  nothing is written
//   1  every call that returns an error writes "[pa] error: <message>"
//   2  also one "[pa] ..." line per state-changing call (allocation, fork,
//      free, swap, append, decode with its chosen kernel and work split)
// Lines go to stderr, one fprintf each, so lines of concurrent calls do not
// interleave inside a line.
//
// Ranges: built with PA_NVTX defined (python -m pagedattention_decode_03_b200.build
// --nvtx, or PA_NVTX=1 in the build's environment), every C-ABI entry point
// opens an NVTX range named after the call for its duration, so a timeline
// profiler shows host enqueue per call.  NVTX 3 is header-only: with no tool
// attached a range costs one test of a null function pointer.  Without
// PA_NVTX the ranges compile to nothing.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <cstdlib>

#ifdef PA_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

namespace pa {

inline int log_level() {
  static const int level = [] {
    const char* s = std::getenv("PA_LOG");
    if (s == nullptr || *s == '\0') return 0;
    char* end = nullptr;
    const long v = std::strtol(s, &end, 10);
    return (end != s && *end == '\0' && v > 0) ? static_cast<int>(v > 2 ? 2 : v) : 0;
  }();
  return level;
}

#if defined(__GNUC__)
__attribute__((format(printf, 2, 3)))
#endif
inline void logf(int level, const char* fmt, ...) {
  if (log_level() < level) return;
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  std::fprintf(stderr, "[pa] %s\n", buf);
}

#ifdef PA_NVTX
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};
#define PA_RANGE() ::pa::Range pa_call_range_(__func__)
#else
#define PA_RANGE() static_cast<void>(0)
#endif

}  // namespace pa
