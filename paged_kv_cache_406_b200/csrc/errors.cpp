// Per-thread last-error text for the C ABI.
#include "pkv_internal.h"

namespace {
thread_local std::string g_last_error;
}

namespace pkv {

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return PKV_OK;
}

}  // namespace pkv

extern "C" const char* pkv_last_error_string(void) { return g_last_error.c_str(); }

extern "C" const char* pkv_version(void) { return "1.0.0"; }
