// Host-side helpers shared by the library's C++ translation units.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "julia_decide.h"

namespace jd {

// Record a thread-local error message and return the status.
jd_status fail(jd_status st, const char *fmt, ...);
void clear_error();

}  // namespace jd
