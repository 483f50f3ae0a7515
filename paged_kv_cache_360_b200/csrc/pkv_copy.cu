// pkv_copy.cu -- the two data-movement steps of a decode step: appending the new
// token's keys and values through the slot mapping, and copying shared blocks
// on write.  Both are pure HBM copies done with 16-byte vector loads and stores.
//
// "PagedAttention" ops page, How it works -- The mechanics: each decode step
// writes the new token's key and value into the sequence's current block;
// sequences that share blocks copy a block when they diverge.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kCopyThreads = 256;

// One warp per token (grid-stride over the tokens).  A token's keys are
// num_kv_heads x head_dim contiguous elements of `key` (likewise `value`):
// lane l reads 16-byte chunks l, l + 32, ... of both -- kAppendBatch of each in
// flight before any store -- and writes each chunk into its (block, kv head)
// row of the pool at the slot's offset.  Reads are fully coalesced; every
// 256-byte (D = 128) or 128-byte (D = 64) row lands as whole 16-byte stores.
constexpr int kAppendBatch = 4;

__global__ void __launch_bounds__(kCopyThreads)
append_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
              const uint4* __restrict__ key, const uint4* __restrict__ value,
              const int64_t* __restrict__ slot_mapping, int64_t num_tokens,
              int32_t chunks_per_row, int32_t num_kv_heads, int32_t block_size,
              int64_t num_slots, int32_t* err_flag) {
    // let a decode launched behind this kernel start its set-up now; this kernel
    // is itself launched as a programmatic dependent of the previous work in the
    // stream, so it waits for that work before touching memory
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    const int per_token = chunks_per_row * num_kv_heads;
    for (int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; t < num_tokens;
         t += warps) {
        const int64_t slot = __ldg(slot_mapping + t);
        const uint4* ks = key + t * per_token;
        const uint4* vs = value + t * per_token;
        for (int c0 = 0; c0 < per_token; c0 += 32 * kAppendBatch) {
            uint4 kr[kAppendBatch], vr[kAppendBatch];
#pragma unroll
            for (int j = 0; j < kAppendBatch; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < per_token) {
                    kr[j] = __ldg(ks + c);
                    vr[j] = __ldg(vs + c);
                }
            }
            if (slot < 0) break;  // padding token
            if (slot >= num_slots) {
                if (lane == 0 && c0 == 0 && err_flag) atomicOr(err_flag, PKV_DEVERR_BAD_SLOT);
                break;
            }
            const int64_t block = slot / block_size;
            const int64_t offset = slot - block * block_size;
#pragma unroll
            for (int j = 0; j < kAppendBatch; ++j) {
                const int c = c0 + 32 * j + lane;
                if (c < per_token) {
                    const int head = c / chunks_per_row;
                    const int cc = c - head * chunks_per_row;
                    const int64_t dst = ((block * num_kv_heads + head) * block_size + offset) * chunks_per_row + cc;
                    k_cache[dst] = kr[j];
                    v_cache[dst] = vr[j];
                }
            }
        }
    }
}

// grid = (pair, pool [0 = K, 1 = V], slice).  A block is contiguous in the pool
// ([num_kv_heads][block_size][head_dim] elements), so each copy is one linear
// run of `block_chunks` 16-byte chunks split over gridDim.z CTAs.
__global__ void __launch_bounds__(kCopyThreads)
copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                   const int32_t* __restrict__ block_mapping, int64_t block_chunks,
                   int32_t num_blocks, int32_t* err_flag) {
    const int32_t src = __ldg(block_mapping + 2 * blockIdx.x);
    const int32_t dst = __ldg(block_mapping + 2 * blockIdx.x + 1);
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && err_flag)
            atomicOr(err_flag, PKV_DEVERR_BAD_PAIR);
        return;
    }
    uint4* pool = blockIdx.y == 0 ? k_cache : v_cache;
    const uint4* from = pool + static_cast<int64_t>(src) * block_chunks;
    uint4* to = pool + static_cast<int64_t>(dst) * block_chunks;
    const int64_t stride = static_cast<int64_t>(gridDim.z) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.z) * blockDim.x + threadIdx.x; i < block_chunks;
         i += stride)
        to[i] = from[i];
}

// grid = (list entry i, pool [0 = K, 1 = V], slice): block list[i] of the pool
// and entry i of the page-locked host buffer, copied in the `to_host` direction.
__global__ void __launch_bounds__(kCopyThreads)
swap_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache, uint4* host_k,
                   uint4* host_v, const int32_t* __restrict__ block_list, int64_t block_chunks,
                   int32_t num_blocks, int32_t to_host, int32_t* err_flag) {
    const int32_t blk = __ldg(block_list + blockIdx.x);
    if (blk < 0 || blk >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && err_flag)
            atomicOr(err_flag, PKV_DEVERR_BAD_PAIR);
        return;
    }
    uint4* dev = (blockIdx.y == 0 ? k_cache : v_cache) + static_cast<int64_t>(blk) * block_chunks;
    uint4* host = (blockIdx.y == 0 ? host_k : host_v) + static_cast<int64_t>(blockIdx.x) * block_chunks;
    const int64_t stride = static_cast<int64_t>(gridDim.z) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.z) * blockDim.x + threadIdx.x; i < block_chunks;
         i += stride) {
        if (to_host)
            host[i] = dev[i];
        else
            dev[i] = host[i];
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The device address of page-locked host memory, or NULL for anything else
// (pageable host memory must never reach a kernel).
void* pinned_device_address(void* host) {
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
        cudaGetLastError();  // clear the error of an unknown pointer
        return nullptr;
    }
    if (attr.type != cudaMemoryTypeHost) return nullptr;
    return attr.devicePointer;
}

pkv_status check_desc(const pkv_cache_desc* d, const char* who) {
    if (!d) return fail(PKV_ERR_INVALID_ARG, who);
    if (d->num_blocks <= 0 || d->num_kv_heads <= 0 || d->block_size <= 0 || d->head_dim <= 0)
        return fail(PKV_ERR_INVALID_ARG, "cache descriptor has a non-positive size");
    if (d->dtype != PKV_F16 && d->dtype != PKV_BF16)
        return fail(PKV_ERR_UNSUPPORTED, "dtype must be PKV_F16 or PKV_BF16");
    if (d->head_dim != 64 && d->head_dim != 128)
        return fail(PKV_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (d->block_size != 16 && d->block_size != 32)
        return fail(PKV_ERR_UNSUPPORTED, "block_size must be 16 or 32");
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status paged_kv_append(const pkv_cache_desc* desc, void* k_cache, void* v_cache,
                                      const void* key, const void* value,
                                      const int64_t* slot_mapping, int32_t num_tokens,
                                      int32_t* err_flag, void* stream) {
    pkv_status st = check_desc(desc, "paged_kv_append: desc is NULL");
    if (st != PKV_OK) return st;
    if (num_tokens < 0) return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: num_tokens < 0");
    if (num_tokens == 0) return PKV_OK;
    if (!k_cache || !v_cache || !key || !value || !slot_mapping)
        return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: NULL pointer");
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(key) || !aligned16(value))
        return fail(PKV_ERR_INVALID_ARG, "paged_kv_append: pools, key and value must be 16-byte aligned");
    const int32_t chunks_per_row = desc->head_dim * 2 / 16;
    // one warp per token, at most a full device of warps (148 SMs x 8 CTAs)
    const int64_t want = (static_cast<int64_t>(num_tokens) + kCopyThreads / 32 - 1) / (kCopyThreads / 32);
    const int grid = static_cast<int>(want < 148 * 8 ? want : 148 * 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kCopyThreads);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(
        &cfg, append_kernel, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        static_cast<const uint4*>(key), static_cast<const uint4*>(value), slot_mapping,
        static_cast<int64_t>(num_tokens), chunks_per_row, desc->num_kv_heads, desc->block_size,
        static_cast<int64_t>(desc->num_blocks) * desc->block_size, err_flag);
    note_launches(1);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

extern "C" pkv_status copy_blocks(const pkv_cache_desc* desc, void* k_cache, void* v_cache,
                                  const int32_t* block_mapping, int32_t num_pairs,
                                  int32_t* err_flag, void* stream) {
    pkv_status st = check_desc(desc, "copy_blocks: desc is NULL");
    if (st != PKV_OK) return st;
    if (num_pairs < 0) return fail(PKV_ERR_INVALID_ARG, "copy_blocks: num_pairs < 0");
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !block_mapping)
        return fail(PKV_ERR_INVALID_ARG, "copy_blocks: NULL pointer");
    if (!aligned16(k_cache) || !aligned16(v_cache))
        return fail(PKV_ERR_INVALID_ARG, "copy_blocks: pools must be 16-byte aligned");
    const int64_t block_chunks =
        static_cast<int64_t>(desc->num_kv_heads) * desc->block_size * desc->head_dim * 2 / 16;
    // about 4 chunks (64 B) per thread per CTA
    int64_t slices = (block_chunks + kCopyThreads * 4 - 1) / (kCopyThreads * 4);
    if (slices > 65535) slices = 65535;
    dim3 grid(static_cast<unsigned>(num_pairs), 2, static_cast<unsigned>(slices));
    copy_blocks_kernel<<<grid, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), block_mapping, block_chunks,
        desc->num_blocks, err_flag);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

extern "C" pkv_status swap_blocks(const pkv_cache_desc* desc, void* k_cache, void* v_cache,
                                  void* host_k, void* host_v, const int32_t* block_list, int32_t n,
                                  int32_t to_host, int32_t* err_flag, void* stream) {
    pkv_status st = check_desc(desc, "swap_blocks: desc is NULL");
    if (st != PKV_OK) return st;
    if (n < 0) return fail(PKV_ERR_INVALID_ARG, "swap_blocks: n < 0");
    if (n == 0) return PKV_OK;
    if (!k_cache || !v_cache || !host_k || !host_v || !block_list)
        return fail(PKV_ERR_INVALID_ARG, "swap_blocks: NULL pointer");
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(host_k) || !aligned16(host_v))
        return fail(PKV_ERR_INVALID_ARG, "swap_blocks: pools and host buffers must be 16-byte aligned");
    void* dk = pinned_device_address(host_k);
    void* dv = pinned_device_address(host_v);
    if (!dk || !dv)
        return fail(PKV_ERR_INVALID_ARG, "swap_blocks: host buffers must be page-locked host memory");
    const int64_t block_chunks =
        static_cast<int64_t>(desc->num_kv_heads) * desc->block_size * desc->head_dim * 2 / 16;
    int64_t slices = (block_chunks + kCopyThreads * 4 - 1) / (kCopyThreads * 4);
    if (slices > 65535) slices = 65535;
    dim3 grid(static_cast<unsigned>(n), 2, static_cast<unsigned>(slices));
    swap_blocks_kernel<<<grid, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), static_cast<uint4*>(dk),
        static_cast<uint4*>(dv), block_list, block_chunks, desc->num_blocks, to_host ? 1 : 0, err_flag);
    note_launches(1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}
