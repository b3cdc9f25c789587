// Error reporting and version string of the C ABI.
#include "pa_internal.h"

namespace pa {

static thread_local std::string g_last_error;

pa_status fail(pa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

}  // namespace pa

extern "C" const char* pa_last_error(void) { return pa::g_last_error.c_str(); }

extern "C" const char* pa_version(void) { return "paged_kv_cache_356_b200 0.1 (sm_100a)"; }
