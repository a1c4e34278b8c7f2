// Host-side helpers shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstddef>
#include <cstdint>
#include <string>

#include "pkv.h"

namespace pkv {

// Record a printf-style message as this thread's last error and return `code`.
int set_error(int code, const char* fmt, ...);
void clear_error();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace pkv
