// Per-thread last-error text and the version query of the C ABI.
#include <cstdio>

#include "pkv_internal.h"

namespace pkv {

static thread_local std::string g_last_error;

int set_error(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

void clear_error() { g_last_error.clear(); }

}  // namespace pkv

extern "C" const char* pkv_last_error_string(void) { return pkv::g_last_error.c_str(); }

extern "C" int pkv_version(void) { return 10000; }
