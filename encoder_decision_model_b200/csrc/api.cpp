// Error reporting and version of the C ABI.
#include <cstring>

#include "host_common.h"

namespace {
thread_local char g_err[512] = "";
}

namespace jd {

jd_status fail(jd_status st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return st;
}

void clear_error() { g_err[0] = 0; }

}  // namespace jd

extern "C" const char *jd_last_error(void) { return g_err; }

extern "C" const char *jd_version(void) { return "julia-decide-b200 0.1 (sm_100a)"; }
