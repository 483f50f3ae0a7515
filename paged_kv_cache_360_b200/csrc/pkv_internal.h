// pkv_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "pkv.h"

namespace pkv {

// Record a message for pkv_last_error() and return `status`.
pkv_status fail(pkv_status status, const char* message);

// Count kernel launches for pkv_launch_count().
void note_launches(uint64_t n);

// Launch the prefill kernel's bounded-wait self-test (pkv_selftest_wait_timeout).
cudaError_t prefill_selftest_wait(int32_t* err, cudaStream_t stream);

// Tensor maps of the tensor-core kernels (pkv_prefill.cu).  Queries [rows]
// [num_heads][D] as 4-D (x = 64 columns, y = head, z = row, w = 64-column
// half), a box of 64 x g x (128 / g) x D/64 landing as the 128-row A operand;
// one pool as 3-D (x = 64 columns, y = pool row, z = half), a box of one
// block's rows of one half.
pkv_status encode_q_map(CUtensorMap* tm, const void* q, int dtype, int num_rows, int num_heads,
                        int D, int g);
pkv_status encode_block_map(CUtensorMap* tm, const void* pool, const pkv_cache_desc* d);

}  // namespace pkv
