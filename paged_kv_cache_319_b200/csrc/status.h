// Shared status helpers of libkvp: per-thread last-error message.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "kvp.h"

namespace kvp {

std::string& last_error();

// Records a formatted message for kvp_last_error_message() and returns `code`.
inline int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  last_error() = buf;
  return code;
}

inline int ok() { return KVP_OK; }

}  // namespace kvp
