// Thread-local error detail shared by the host-side C-ABI entry points.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "pagedkv.h"

namespace pagedkv {

std::string& last_error_slot();

inline pa_status fail(pa_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  last_error_slot() = buf;
  return s;
}

}  // namespace pagedkv
