// pkv_diag.cpp -- status strings, the per-thread last-error message and the
// process-wide launch counter.
#include <atomic>
#include <cstdio>
#include <cstring>

#include "pkv.h"
#include "pkv_internal.h"

namespace {
thread_local char g_last_error[256] = "";
std::atomic<uint64_t> g_launches{0};
}  // namespace

namespace pkv {

pkv_status fail(pkv_status status, const char* message) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", pkv_status_string(status),
                  message ? message : "");
    return status;
}

void note_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

}  // namespace pkv

extern "C" uint64_t pkv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" const char* pkv_last_error(void) { return g_last_error; }

extern "C" const char* pkv_status_string(pkv_status status) {
    switch (status) {
        case PKV_OK: return "PKV_OK";
        case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG";
        case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED";
        case PKV_ERR_NO_FREE_BLOCK: return "PKV_ERR_NO_FREE_BLOCK";
        case PKV_ERR_CUDA: return "PKV_ERR_CUDA";
        case PKV_ERR_WORKSPACE_TOO_SMALL: return "PKV_ERR_WORKSPACE_TOO_SMALL";
    }
    return "PKV_ERR_UNKNOWN";
}
