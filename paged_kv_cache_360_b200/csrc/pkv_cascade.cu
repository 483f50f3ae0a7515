// pkv_cascade.cu -- the shared-prefix part of the shared-prefix decode: every
// decode query of a group of sequences attends, on the tcgen05 tensor cores,
// to the blocks the group's block tables share.
//
// "PagedAttention" ops page, At a glance and How it works: sequences forked
// from one prompt point their tables at the same physical blocks (reference
// counted, copied only on write).  Read through each sequence's table, those
// blocks are streamed once per sequence, g query rows at a time.  Here the
// queries of 128 / g sequences times the g heads of one kv head form one
// 128-row tile, so Q K^T and P V over the shared blocks are real M = 128
// contractions and every shared K/V row is read once per tile instead of once
// per sequence.
//
// One CTA takes (group, row tile, kv head, chunk of 1 or 2 kv tiles of 128
// tokens) and writes, for every row, the chunk's un-normalised partial
//   m = max_t s_t (base 2),  l = sum_t 2^(s_t - m),  o = sum_t 2^(s_t - m) V_t
// into the workspace; cascade_finalize_kernel (pkv_decode.cu) merges these
// with the partials of each sequence's own tokens by log-sum-exp.
//   warp 4   producer: Q tile (4-D TMA box: x = 64 columns, y = head, z =
//            sequence, w = half), then per kv tile one 3-D box per (block,
//            half) of K and of V, the blocks taken from the group's first
//            table row; rows of blocks past the shared ones are zeroed in V;
//   warp 5   MMA issuer (one thread) and tensor-memory owner: S_j = Q K_j^T
//            into columns 128 j, then O = sum_j (P_hi,j + P_lo,j) V_j into
//            columns 384 .. 384 + D, P read from tensor memory;
//   warps 0-3 softmax, one row per thread (tensor-memory lane = row): the
//            chunk's maximum over both tiles first, then P = 2^(s - m) as a
//            pair of input-type values P_hi = round(P), P_lo = round(P - P_hi)
//            (P_hi over S_j's first 64 columns, P_lo in columns 256 + 64 j),
//            so the weights carry about 16 significant bits as in the decode.
// Every wait is bounded (pkv_wait.cuh); the producer and the MMA thread drain
// their copies and MMAs before the CTA frees its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "pkv.h"
#include "pkv_cascade.cuh"
#include "pkv_host.cuh"
#include "pkv_internal.h"
#include "pkv_ptx.cuh"
#include "pkv_tc.cuh"
#include "pkv_wait.cuh"

namespace pkv {
namespace {

constexpr int kCaThreads = 192;  // softmax warps 0-3, producer 4, MMA 5
constexpr int kCaProducer = 4;
constexpr int kCaMma = 5;
constexpr uint32_t kCaTmemCols = 512;  // S_0, S_1, P_lo (2 x 64), O
constexpr uint32_t kColPlo = 256;
constexpr uint32_t kColO = 384;

enum : int {
    kCbQ = 0,
    kCbK = 1,      // + tile
    kCbV = 3,      // + tile
    kCbS = 5,      // + tile
    kCbP = 7,      // + tile, 128 arrivals
    kCbO = 9,
    kCbDrain = 10,
    kCbCount
};

template <int D>
struct CaLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = kPrefixRows * 128;  // 128 rows x 128 B
    static constexpr int kTile = kHalves * kHalfBytes;
    static constexpr int kQ = 0;
    static constexpr int kK = kTile;          // K_0, K_1
    static constexpr int kV = 3 * kTile;      // V_0, V_1
    static constexpr int kBars = 5 * kTile;
    static constexpr int kMisc = kBars + 8 * kCbCount;  // tmem base, abort word
    static constexpr int kAlloc = kMisc + 16 + 1024;    // + room to align the base
};

struct PrefixArgs {
    const int32_t* tables;
    int32_t* err;
    int32_t num_seqs;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t log2_group;
    int32_t max_blocks;
    int32_t num_blocks;
    float sl2;  // scale * log2(e)
};

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kCaThreads, 1)
    prefix_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                  const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tp,
                  const PrefixArgs a, const __grid_constant__ CascadeGroups cg) {
    using Lay = CaLayout<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescS = f16_idesc(kBf16, kPrefixRows, kPrefixKv, false);
    constexpr uint32_t kIdescO = f16_idesc(kBf16, kPrefixRows, D, true);
    constexpr int kBpt = kPrefixKv / BS;  // blocks per kv tile
    static_assert(kPrefixKv % BS == 0 && kBpt <= 32, "a kv tile holds whole blocks");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sp = smem_raw + (sb - raw);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sp + Lay::kMisc);
    volatile uint32_t* abort_word = misc + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) { return sb + Lay::kBars + 8u * static_cast<uint32_t>(i); };

    // ---- which work item: group, row tile, chunk (blockIdx.x); kv head (y)
    const int item = blockIdx.x;
    int grp = 0;
    while (grp + 1 < cg.num_groups && cg.item_base[grp + 1] <= item) ++grp;
    const int local = item - cg.item_base[grp];
    const int chunks = cg.chunks[grp];
    const int rt = local / chunks, chunk = local - rt * chunks;
    const int hk = blockIdx.y;
    const int g = 1 << a.log2_group;
    const int seqs_per_tile = kPrefixRows >> a.log2_group;
    const int s0 = cg.start[grp] + rt * seqs_per_tile;  // first sequence of the row tile
    const int shared = cg.shared_tokens[grp];
    const int n_tiles = (shared + kPrefixKv - 1) / kPrefixKv;
    const int t0 = chunk * cg.tiles_per_item;
    const int ntl = min(cg.tiles_per_item, n_tiles - t0);  // 1 or 2

    if (threadIdx.x == 0) {
        for (int i = 0; i < kCbCount; ++i) mbar_init(bar(i), i == kCbP || i == kCbP + 1 ? 128 : 1);
        misc[1] = 0u;
        fence_mbar_init();
        prefetch_tensormap(&tq);
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        prefetch_tensormap(&tp);
    }
    if (warp == kCaMma) {
        tmem_alloc(sb + Lay::kMisc, kCaTmemCols);
        tmem_relinquish();
    }
    // Launched behind the call's decode of the sequences' own tokens, as a
    // programmatic dependent: it starts once every CTA before it has passed its
    // own wait for the call's inputs, and reads only those inputs (queries, the
    // pools, the tables) and writes only its own partials, so it runs without
    // waiting; it waits for the kernels before it at the end, so the kernel
    // behind it (launched early here) sees everything complete.
    pdl_launch_dependents();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];

    if (warp < 4) {
        // ---------------------------------------------------------- softmax
        const int r = warp * 32 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        // maximum over the chunk's visible columns (raw scores; sl2 > 0)
        float mraw = -INFINITY;
        bool ok = true;
        for (int j = 0; j < ntl && ok; ++j) {
            if (!(ok = warp_wait(bar(kCbS + j), 0, abort_word, a.err))) break;
            tc_fence_after();
            const int nv = min(kPrefixKv, shared - (t0 + j) * kPrefixKv);
            uint32_t u[32];
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld32(lane_base + 128u * j + 32u * c, u);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (32 * c + i < nv) mraw = fmaxf(mraw, __uint_as_float(u[i]));
            }
        }
        const float m2 = mraw * a.sl2;
        float l = 0.f;
        for (int j = 0; j < ntl && ok; ++j) {
            const int nv = min(kPrefixKv, shared - (t0 + j) * kPrefixKv);
            uint32_t u[128];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                tmem_ld32(lane_base + 128u * j + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * c));
            tmem_wait_ld();
            // all 128 scores are in registers: P_hi may now overwrite S_j's
            // first 64 columns
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c0 = 32 * k + 2 * i;
                    const float p0 = c0 < nv ? exp2_approx(fmaf(__uint_as_float(u[c0]), a.sl2, -m2)) : 0.f;
                    const float p1 =
                        c0 + 1 < nv ? exp2_approx(fmaf(__uint_as_float(u[c0 + 1]), a.sl2, -m2)) : 0.f;
                    l += p0 + p1;
                    float r0, r1, e0, e1;
                    hi[i] = Pack<T>::two(p0, p1, r0, r1);
                    lo[i] = Pack<T>::two(p0 - r0, p1 - r1, e0, e1);
                }
                tmem_st16(lane_base + 128u * j + 16u * k, hi);
                tmem_st16(lane_base + kColPlo + 64u * j + 16u * k, lo);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(kCbP + j));
        }
        if (ok) ok = warp_wait(bar(kCbO), 0, abort_word, a.err);
        // The tile's partial, rows as they stand (rows of other sequences
        // included: the tile's slots are its own).  O goes from tensor memory to
        // shared memory -- the Q and K_0 buffers, no longer read -- as D/32 boxes
        // of [128 rows][128 B], 16-byte chunk c of row r at c ^ (r & 7) (the
        // TMA's 128B swizzle, so that the stores of 8 consecutive rows hit 8 bank
        // groups), then one TMA tensor store per box writes the tile
        // contiguously.  Every softmax warp reaches the barrier, failed or not;
        // the stores go out only if no role raised the abort word.
        const int64_t row0 = (static_cast<int64_t>(item) * a.num_kv_heads + hk) * kPrefixRows;
        const uint32_t stage = sb + Lay::kQ;
        if (ok) {
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(lane_base + kColO + 32u * c, o);
                tmem_wait_ld();
                const uint32_t rowaddr = stage + c * (kPrefixRows * 128) + r * 128;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     rowaddr + ((i ^ (r & 7)) << 4)),
                                 "r"(o[4 * i]), "r"(o[4 * i + 1]), "r"(o[4 * i + 2]), "r"(o[4 * i + 3])
                                 : "memory");
            }
            fence_proxy_async_smem();
            *reinterpret_cast<float2*>(cg.pre_ml + (row0 + r) * 2) = make_float2(m2, l);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0 && *abort_word == 0u) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c)
                tma_store_2d(&tp, stage + c * (kPrefixRows * 128), 32 * c, static_cast<int32_t>(row0));
            bulk_commit_and_wait_all();
        }
    } else if (warp == kCaProducer) {
        // --------------------------------------------------------- producer
        const int32_t* row = a.tables + static_cast<int64_t>(cg.start[grp]) * a.max_blocks;
        const int nblk = shared / BS;  // shared blocks of the group
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(kCbQ), Lay::kTile);
            tma_load_4d(sb + Lay::kQ, &tq, 0, hk * g, s0, 0, bar(kCbQ));
        }
        for (int j = 0; j < ntl; ++j) {
            const int blk = (t0 + j) * kBpt + lane;
            const bool mine = lane < kBpt;
            const bool valid = mine && blk < nblk;
            int id = 0;
            if (valid) {
                id = __ldg(row + blk);
                if (id < 0 || id >= a.num_blocks) {
                    raise_flag(a.err, PKV_DEVERR_BAD_BLOCK_ID);
                    id = 0;
                }
            }
            const uint32_t kdst = sb + Lay::kK + j * Lay::kTile;
            const uint32_t vdst = sb + Lay::kV + j * Lay::kTile;
            if (mine && !valid) {
                // past the shared blocks: P is 0 there, but 0 * NaN is NaN, so
                // the V rows hold zeros instead of whatever the buffer held
#pragma unroll
                for (int h = 0; h < Lay::kHalves; ++h)
                    for (int c = 0; c < BS * 8; ++c)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(
                                         vdst + h * Lay::kHalfBytes + lane * BS * 128 + c * 16),
                                     "r"(0u)
                                     : "memory");
                fence_proxy_async_smem();
            }
            const int nvalid = __popc(__ballot_sync(0xffffffffu, valid));
            __syncwarp();
            if (lane == 0) {
                const uint32_t bytes = static_cast<uint32_t>(nvalid * BS * 128 * Lay::kHalves);
                mbar_arrive_expect_tx(bar(kCbK + j), bytes);
                mbar_arrive_expect_tx(bar(kCbV + j), bytes);
            }
            __syncwarp();
            if (valid) {
                const int y = (id * a.num_kv_heads + hk) * BS;
#pragma unroll
                for (int h = 0; h < Lay::kHalves; ++h) {
                    tma_load_3d(kdst + h * Lay::kHalfBytes + lane * BS * 128, &tk, 0, y, h, bar(kCbK + j));
                    tma_load_3d(vdst + h * Lay::kHalfBytes + lane * BS * 128, &tv, 0, y, h, bar(kCbV + j));
                }
            }
        }
        // every copy in flight lands before the CTA can exit
        if (lane == 0) {
            quiet_wait(bar(kCbQ), 0);
            for (int j = 0; j < ntl; ++j) {
                quiet_wait(bar(kCbK + j), 0);
                quiet_wait(bar(kCbV + j), 0);
            }
        }
    } else if (lane == 0) {
        // ------------------------------------------------------ MMA issuer
        bool ok = one_wait(bar(kCbQ), 0, abort_word, a.err);
        for (int j = 0; j < ntl && ok; ++j) {
            if (!(ok = one_wait(bar(kCbK + j), 0, abort_word, a.err))) break;
            tc_fence_after();
            const uint32_t ks = sb + Lay::kK + j * Lay::kTile;
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t off = (k >> 2) * static_cast<uint32_t>(Lay::kHalfBytes) + (k & 3) * 32u;
                mma_f16_ss(tmem + 128u * j, sw128_desc(sb + Lay::kQ + off, 16, 1024),
                           sw128_desc(ks + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
            }
            mma_commit(bar(kCbS + j));
        }
        // V first: its copies have usually landed while the softmax ran, and a
        // barrier check between P's arrival and the P V MMAs would sit on the
        // softmax -> P V path
        for (int j = 0; j < ntl && ok; ++j) ok = one_wait(bar(kCbV + j), 0, abort_word, a.err);
        for (int j = 0; j < ntl && ok; ++j) {
            if (!(ok = one_wait(bar(kCbP + j), 0, abort_word, a.err))) break;
            tc_fence_after();
            const uint32_t vs = sb + Lay::kV + j * Lay::kTile;
            // O += P_hi V_j, then O += P_lo V_j (16 tokens = 8 columns of P per step)
            for (int part = 0; part < 2; ++part)
#pragma unroll
                for (int k = 0; k < kPrefixKv / 16; ++k)
                    mma_f16_ts(tmem + kColO,
                               tmem + (part ? kColPlo + 64u * j : 128u * j) + 8u * k,
                               sw128_desc(vs + k * 16 * 128, Lay::kHalfBytes, 1024), kIdescO,
                               (j > 0 || part > 0 || k > 0) ? 1u : 0u);
        }
        if (ok) mma_commit(bar(kCbO));
        // every MMA issued above completes before the tensor memory is freed
        mma_commit(bar(kCbDrain));
        quiet_wait(bar(kCbDrain), 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kCaMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kCaTmemCols);
    }
    pdl_wait_primary();
}

template <typename T, int D, int BS>
struct PrefixTag {};

template <typename T, int D, int BS>
cudaError_t launch_prefix_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const CUtensorMap& tp, const PrefixArgs& a, const CascadeGroups& cg,
                            cudaStream_t stream) {
    auto* k = prefix_kernel<T, D, BS>;
    cudaError_t e = opt_in_smem<PrefixTag<T, D, BS>>(reinterpret_cast<const void*>(k));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(cg.item_base[cg.num_groups]),
                    static_cast<unsigned>(a.num_kv_heads));
    return launch_dependent(k, grid, dim3(kCaThreads), CaLayout<D>::kAlloc, stream, tq, tk, tv, tp, a,
                            cg);
}

template <typename T>
cudaError_t launch_prefix_dt(int D, int BS, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, const CUtensorMap& tp, const PrefixArgs& a,
                             const CascadeGroups& cg, cudaStream_t stream) {
    if (D == 128) return BS == 16 ? launch_prefix_t<T, 128, 16>(tq, tk, tv, tp, a, cg, stream)
                                  : launch_prefix_t<T, 128, 32>(tq, tk, tv, tp, a, cg, stream);
    return BS == 16 ? launch_prefix_t<T, 64, 16>(tq, tk, tv, tp, a, cg, stream)
                    : launch_prefix_t<T, 64, 32>(tq, tk, tv, tp, a, cg, stream);
}

// The prefix partials' O as 2-D fp32 (x = head_dim columns, y = tile rows), a
// box of 32 columns (128 B) x 128 rows, 128B swizzle: the layout the prefix
// kernel stages its tiles in.
pkv_status encode_partial_map(CUtensorMap* tm, float* pre_o, int64_t rows, int D) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 4};
    cuuint32_t box[2] = {32, static_cast<cuuint32_t>(kPrefixRows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, pre_o, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (prefix partials)");
    return PKV_OK;
}

}  // namespace

// ------------------------------------------------------------------ host side

pkv_status plan_groups(const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_heads,
                       int32_t max_blocks_per_seq, const int32_t* group_start,
                       const int32_t* group_shared_blocks, int32_t num_groups, CascadeGroups* cg,
                       int64_t* slots) {
    if (num_groups < 0 || num_groups > kMaxGroups)
        return fail(PKV_ERR_UNSUPPORTED, "shared-prefix decode: num_groups must be 0 .. 64");
    if (num_groups > 0 && (!group_start || !group_shared_blocks))
        return fail(PKV_ERR_INVALID_ARG, "shared-prefix decode: NULL group arrays");
    const int g = num_heads / desc->num_kv_heads;
    const int seqs_per_tile = kPrefixRows / g;
    *cg = CascadeGroups{};
    cg->num_groups = num_groups;
    int64_t items1 = 0;  // work items at one kv tile each
    for (int i = 0; i < num_groups; ++i) {
        const int32_t a = group_start[i], b = group_start[i + 1], nb = group_shared_blocks[i];
        if (a < 0 || b <= a || b > num_seqs)
            return fail(PKV_ERR_INVALID_ARG,
                        "shared-prefix decode: group_start must increase strictly within 0 .. num_seqs");
        if (nb < 0 || nb > max_blocks_per_seq)
            return fail(PKV_ERR_INVALID_ARG,
                        "shared-prefix decode: group_shared_blocks must be 0 .. max_blocks_per_seq");
        if (nb > 0 && (g & (g - 1)) != 0)
            return fail(PKV_ERR_UNSUPPORTED,
                        "shared-prefix decode: num_heads / num_kv_heads must be a power of two");
        cg->start[i] = a;
        cg->shared_tokens[i] = nb * desc->block_size;
        const int64_t tiles = (static_cast<int64_t>(nb) * desc->block_size + kPrefixKv - 1) / kPrefixKv;
        items1 += tiles * ((b - a + seqs_per_tile - 1) / seqs_per_tile);
    }
    cg->start[num_groups] = num_groups > 0 ? group_start[num_groups] : 0;
    cg->tiles_per_item = items1 * desc->num_kv_heads >= kPrefixTwoTilesFrom ? 2 : 1;
    int64_t base = 0, items = 0, seqs = 0;
    for (int i = 0; i < num_groups; ++i) {
        const int n = cg->start[i + 1] - cg->start[i];
        const int64_t tiles = (cg->shared_tokens[i] + kPrefixKv - 1) / kPrefixKv;
        cg->chunks[i] = static_cast<int32_t>((tiles + cg->tiles_per_item - 1) / cg->tiles_per_item);
        cg->item_base[i] = static_cast<int32_t>(items);
        cg->seq_base[i] = static_cast<int32_t>(seqs);
        items += static_cast<int64_t>(cg->chunks[i]) * ((n + seqs_per_tile - 1) / seqs_per_tile);
        base = items * desc->num_kv_heads * kPrefixRows;
        if (cg->shared_tokens[i] > 0) seqs += n;
        if (base > INT32_MAX || items > INT32_MAX)
            return fail(PKV_ERR_UNSUPPORTED, "shared-prefix decode: too many prefix partials");
    }
    cg->item_base[num_groups] = static_cast<int32_t>(items);
    cg->seq_base[num_groups] = static_cast<int32_t>(seqs);
    cg->grouped_seqs = static_cast<int32_t>(seqs);
    *slots = base + seqs * num_heads;
    return PKV_OK;
}

// The prefix kernel over every group of `cg` that shares at least one block
// (cg.item_base[num_groups] work items per kv head); the group table, its
// partial slots and work items are laid out by the caller.
pkv_status launch_prefix(const pkv_cache_desc* desc, const void* q, const void* k_cache,
                         const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                         int32_t num_seqs, int32_t num_heads, float scale, const CascadeGroups& cg,
                         int32_t* err_flag, cudaStream_t stream) {
    if (cg.item_base[cg.num_groups] == 0) return PKV_OK;
    const int g = num_heads / desc->num_kv_heads;
    CUtensorMap tq, tk, tv, tp;
    pkv_status st;
    if ((st = encode_q_map(&tq, q, desc->dtype, num_seqs, num_heads, desc->head_dim, g)) != PKV_OK)
        return st;
    if ((st = encode_block_map(&tk, k_cache, desc)) != PKV_OK) return st;
    if ((st = encode_block_map(&tv, v_cache, desc)) != PKV_OK) return st;
    const int64_t rows = static_cast<int64_t>(cg.item_base[cg.num_groups]) * desc->num_kv_heads * kPrefixRows;
    if ((st = encode_partial_map(&tp, cg.pre_o, rows, desc->head_dim)) != PKV_OK) return st;
    PrefixArgs a;
    a.tables = block_tables;
    a.err = err_flag;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = desc->num_kv_heads;
    a.log2_group = __builtin_ctz(static_cast<unsigned>(g));
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = desc->num_blocks;
    a.sl2 = scale * 1.4426950408889634f;
    cudaError_t e = desc->dtype == PKV_BF16
                        ? launch_prefix_dt<__nv_bfloat16>(desc->head_dim, desc->block_size, tq, tk, tv,
                                                          tp, a, cg, stream)
                        : launch_prefix_dt<__half>(desc->head_dim, desc->block_size, tq, tk, tv, tp, a,
                                                   cg, stream);
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

}  // namespace pkv
