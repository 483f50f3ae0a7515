// pkv_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>

#include "pkv.h"

namespace pkv {

// Record a message for pkv_last_error() and return `status`.
pkv_status fail(pkv_status status, const char* message);

// Count kernel launches for pkv_launch_count().
void note_launches(uint64_t n);

}  // namespace pkv
