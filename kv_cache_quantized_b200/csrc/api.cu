// Status plumbing and small ABI entry points of the axr library.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "axr_common.cuh"

namespace {
thread_local char g_last_error[512] = {0};
}

namespace axr {
axr_status set_error(axr_status st, const char* fmt, ...) {
  if (st == AXR_OK) {
    g_last_error[0] = '\0';
    return st;
  }
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}
}  // namespace axr

extern "C" const char* axr_last_error(void) { return g_last_error; }

extern "C" int axr_version(void) { return 100; }  // 0.1.0
