// pkv_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "pkv.h"

namespace pkv {

// Record a message for pkv_last_error() and return `status`.
pkv_status fail(pkv_status status, const char* message);

// Count kernel launches for pkv_launch_count().
void note_launches(uint64_t n);

// Launch the prefill kernel's bounded-wait self-test (pkv_selftest_wait_timeout).
cudaError_t prefill_selftest_wait(int32_t* err, cudaStream_t stream);

}  // namespace pkv
