// pkv_host.cuh -- host-side helpers shared by the library's CUDA translation
// units: the driver's tensor-map encoder, argument checks, shared-memory opt-in
// and programmatic-dependent launches.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "pkv.h"
#include "pkv_internal.h"

namespace pkv {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline pkv_status check_desc(const pkv_cache_desc* d) {
    if (!d) return fail(PKV_ERR_INVALID_ARG, "cache descriptor is NULL");
    if (d->num_blocks <= 0 || d->num_kv_heads <= 0 || d->block_size <= 0 || d->head_dim <= 0)
        return fail(PKV_ERR_INVALID_ARG, "cache descriptor has a non-positive size");
    if (d->dtype != PKV_F16 && d->dtype != PKV_BF16)
        return fail(PKV_ERR_UNSUPPORTED, "dtype must be PKV_F16 or PKV_BF16");
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (d->block_size != 16 && d->block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 or 32");
    if (static_cast<int64_t>(d->num_blocks) * d->num_kv_heads * d->block_size > INT32_MAX)
        return fail(PKV_ERR_UNSUPPORTED, "num_blocks * num_kv_heads * block_size must be < 2^31");
    return PKV_OK;
}

// Opt a kernel in to the device's maximum dynamic shared memory, once per device
// (the static is per template instantiation of K, and K is per kernel below).
template <typename Tag>
cudaError_t opt_in_smem(const void* kernel) {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    int limit = 0;
    if ((e = cudaDeviceGetAttribute(&limit, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
    // dynamic + static shared memory may not exceed the opt-in limit
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             limit - static_cast<int>(fa.sharedSizeBytes));
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

// Launch `kernel` as a programmatic dependent of the previous work in `stream`:
// it may start while that work finishes, and waits for it in
// griddepcontrol.wait before touching global memory.
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*kernel)(P...), dim3 grid, dim3 block, int smem,
                             cudaStream_t stream, A&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

}  // namespace pkv
