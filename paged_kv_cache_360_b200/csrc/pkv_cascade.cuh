// pkv_cascade.cuh -- the table of shared-prefix groups that the shared-prefix
// decode hands to its kernels as a kernel parameter.
//
// "PagedAttention" ops page, At a glance and How it works: sequences that share
// a prompt point their block tables at the same physical blocks.  A group is a
// run of consecutive sequences of the batch whose first `shared_tokens /
// block_size` table entries are the same blocks; the decode attends each
// sequence's own tokens with the balanced decode, every query of the group to
// the shared blocks in one tensor-core pass (prefix_kernel), and merges the
// two into one softmax by log-sum-exp (cascade_finalize_kernel).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

constexpr int kMaxGroups = 64;  // groups per call (the table is a kernel parameter)
constexpr int kPrefixRows = 128;  // query rows of one prefix tile: 128 / g sequences x g heads
constexpr int kPrefixKv = 128;    // kv tokens of one prefix kv tile

struct CascadeGroups {
    int32_t num_groups;
    int32_t tiles_per_item;                 // kv tiles of one prefix work item (1 or 2)
    int32_t grouped_seqs;                   // sequences of the groups that share blocks
    int32_t start[kMaxGroups + 1];          // group i = sequences start[i] .. start[i+1]-1
    int32_t shared_tokens[kMaxGroups];      // tokens of the shared blocks (a multiple of bs)
    int32_t chunks[kMaxGroups];             // prefix partials per (sequence, head)
    int32_t seq_base[kMaxGroups + 1];       // grouped sequences before group i (sharing groups)
    int32_t item_base[kMaxGroups + 1];      // prefix work items before group i
    float* pre_o;                           // [item][kv head][128 rows][D]  un-normalised prefix
    float* pre_ml;                          // [item][kv head][128 rows][2]  partial O and (m, l),
                                            //   m in base-2 units (a row = a prefix tile row)
    float* own_o;                           // [grouped row][D]  the same over each sequence's own
    float* own_ml;                          // [grouped row][2]  tokens (rows: sequence x head)
};

// Prefix partial row of (sequence b of group i, query head h, chunk c): the
// row of the prefix tile (row tile, chunk, kv head) that holds that query.
// Chunk c + 1 of the same query is prefix_chunk_stride rows further.
__host__ __device__ __forceinline__ int64_t prefix_row(const CascadeGroups& cg, int i, int b,
                                                        int log2_group, int num_kv_heads, int h,
                                                        int c) {
    const int spt = kPrefixRows >> log2_group;  // sequences per row tile
    const int rt = (b - cg.start[i]) / spt;
    const int hk = h >> log2_group;
    const int r = (((b - cg.start[i]) - rt * spt) << log2_group) + (h - (hk << log2_group));
    const int64_t item = cg.item_base[i] + static_cast<int64_t>(rt) * cg.chunks[i] + c;
    return (item * num_kv_heads + hk) * kPrefixRows + r;
}

__host__ __device__ __forceinline__ int64_t prefix_chunk_stride(int num_kv_heads) {
    return static_cast<int64_t>(num_kv_heads) * kPrefixRows;
}

// Row of (sequence b of group i, query head h) in own_o / own_ml.
__host__ __device__ __forceinline__ int64_t own_row(const CascadeGroups& cg, int i, int b,
                                                    int num_heads, int h) {
    return (static_cast<int64_t>(cg.seq_base[i]) + (b - cg.start[i])) * num_heads + h;
}

// Index of the group holding sequence b, or -1.
__device__ __forceinline__ int group_of(const CascadeGroups& cg, int b) {
    int lo = 0, hi = cg.num_groups;  // first group whose end is past b
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (cg.start[mid + 1] <= b) lo = mid + 1;
        else hi = mid;
    }
    return lo < cg.num_groups && cg.start[lo] <= b ? lo : -1;
}

// Index of the group holding sequence b if that group shares blocks, else -1.
__device__ __forceinline__ int sharing_group_of(const CascadeGroups& cg, int b) {
    const int i = group_of(cg, b);
    return i >= 0 && cg.shared_tokens[i] > 0 ? i : -1;
}

// Tokens at the start of sequence b that the prefix kernel attends (0 outside
// a group).
__device__ __forceinline__ int shared_begin(const CascadeGroups& cg, int b) {
    const int i = group_of(cg, b);
    return i < 0 ? 0 : cg.shared_tokens[i];
}

// Stand-in for the group table in the plain decode's kernels.
struct NoGroups {
    int32_t unused;
};

// Prefix work items (1 kv tile each) from which an item takes 2 kv tiles.
constexpr int kPrefixTwoTilesFrom = 296;

// Lay out the group table for these shapes from the caller's host arrays
// (group_start [num_groups + 1], group_shared_blocks [num_groups]); *slots =
// prefix partial slots + own-token rows (each D + 2 floats).  Errors are
// recorded for pkv_last_error().
pkv_status plan_groups(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_heads,
                       int32_t max_blocks_per_seq, const int32_t* group_start,
                       const int32_t* group_shared_blocks, int32_t num_groups, CascadeGroups* cg,
                       int64_t* slots);

// The prefix kernel over every work item of `cg` (pkv_cascade.cu); pre_o is
// written through a TMA tensor map, so it must be 16-byte aligned.  It reads
// only inputs of the call, so it does not wait for the kernels launched before
// it in the call (it is launched behind them, when the call's inputs are
// complete); it waits for them before it exits, so that the kernel behind it
// sees all of their results.
pkv_status launch_prefix(const pkv_cache_desc* desc, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                         int32_t num_seqs, int32_t num_heads, float scale, const CascadeGroups& cg,
                         int32_t* err_flag, cudaStream_t stream);

}  // namespace pkv
