// pkv_decode.cu -- paged decode attention for sm_100a.
//
// "PagedAttention" ops page, How it works -- The mechanics: the attention kernel
// reads keys and values through the block table, gathering scattered physical
// blocks, which makes non-contiguous storage transparent to the math.  Concept --
// What it is: a per-sequence block table maps logical positions to physical
// blocks.
//
// Both schedules below share 4 consumer warps + 1 producer warp (the balanced
// kernel adds a merge warp) and the tile arithmetic of pkv_attend.cuh:
//   * the producer issues, per logical block, TMA 2-D tiled loads of the (block,
//     kv head) K and V tiles -- bs rows x 128 B per 64-column half, 128B swizzle
//     -- into a ring of shared-memory stages, completion counted on one mbarrier
//     per stage.  The tensor map spans the whole pool viewed as
//     [num_blocks * num_kv_heads * bs rows][head_dim], so the gather through the
//     block table is just the row coordinate (block * num_kv_heads + hk) * bs;
//   * stage s belongs to consumer warp s % 4; all g = num_heads / num_kv_heads
//     query heads of the kv head share each tile (S = Q K^T and O += P V on
//     mma.sync m16n8k16, fp32 accumulate, online softmax in base 2);
//   * the four warps' (m, l, O) are merged in shared memory in warp order.
//
// Fixed partitions (partition_size > 0): the balanced schedule below with every
// segment cut at partition boundaries (partition_size tokens); each partition's
// un-normalised O and its (m, l) go to a slot of the workspace (a partition
// split across CTAs is first merged by the chain kernel) and reduce_kernel
// merges a row's partitions p = 0, 1, ...  A partition_size of at least the
// table width means no split: decode_kernel, one CTA per (sequence, kv head).
//
// Balanced (partition_size == 0): a persistent grid of G CTAs (the resident
// count).  The work is the list of units (sequence b, kv head hk, logical block)
// in that order, U of them; CTA c takes units [c*U/G, (c+1)*U/G), so every CTA
// streams the same number of blocks (+-1).  Its range is a run of segments (one
// per (b, hk)); the producer walks it, publishing one descriptor per segment --
// with the segment's query rows copied in by a bulk copy -- before the segment's
// tiles.  A segment that covers a whole (b, hk) is written out directly; the at
// most two that do not (the first and the last of the range) leave partials
// that balanced_reduce_kernel chains across neighbouring CTAs in CTA order.
//
// Every reduction order depends only on logical token order and on the shapes,
// never on physical block ids or timing, so results are bit-identical under any
// permutation of physical blocks.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <type_traits>
#include <utility>

#include "pkv.h"
#include "pkv_attend.cuh"
#include "pkv_cascade.cuh"
#include "pkv_host.cuh"
#include "pkv_internal.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int BS>
struct Geom {
    static constexpr int kHalves = D / 64;                   // 128-byte column halves per row
    static constexpr int kHalfBytes = BS * 128;              // one half of one (block, head) tile
    static constexpr int kTileBytes = kHalves * kHalfBytes;  // K (or V) of one (block, head)
    static constexpr int kStageBytes = 2 * kTileBytes;       // K + V
    // Stage s is always consumed by warp s % kConsumerWarps, so a warp waits on
    // the rounds of its stages in order and is never a phase ahead of the
    // barrier it polls (a parity wait cannot tell phase r-1 from phase r+1).
    static constexpr int kStages = kStageBytes <= 8192 ? 8 : 4;
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
    static constexpr int kRingBytes = kStages * kStageBytes;
    static_assert(kHalfBytes % 1024 == 0, "128B-swizzled tiles must start on 1 KB boundaries");
};

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ void flag(int32_t* err, int32_t bit) {
    if (err) atomicOr(err, bit);
}

__device__ __forceinline__ int clamp_len(int L, int max_len) {
    return L < 0 ? 0 : (L > max_len ? max_len : L);
}

// Issue the K and V tiles of (physical block, kv head) into one ring stage.
template <int D, int BS>
__device__ __forceinline__ void load_tile(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                          uint32_t stage_addr, uint32_t full_bar, int phys,
                                          int num_kv_heads, int hk, uint64_t policy) {
    using G = Geom<D, BS>;
    mbar_arrive_expect_tx(full_bar, G::kStageBytes);
    const int y = (phys * num_kv_heads + hk) * BS;
    // one box = every 64-column half of BS rows (see encode_pool_map)
    tma_load_3d(stage_addr, tm_k, 0, y, 0, full_bar, policy);
    tma_load_3d(stage_addr + G::kTileBytes, tm_v, 0, y, 0, full_bar, policy);
}

// =================================================================== fixed partitions

struct DecodeArgs {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;
    float* ws_m;
    float* ws_l;
    int32_t* err_flag;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t group;
    int32_t max_blocks_per_seq;
    int32_t num_blocks;
    int32_t partition_tokens;
    int32_t max_partitions;
    float scale_log2;
};

template <int D, int BS>
struct FixedLayout {
    using G = Geom<D, BS>;
    static constexpr int kMergeBytes = kConsumerWarps * 16 * (D + 2) * 4;
    static constexpr int kBodyBytes = G::kRingBytes > kMergeBytes ? G::kRingBytes : kMergeBytes;
    static constexpr int kBarOffset = kBodyBytes;
    static constexpr int kSmemBytes = kBarOffset + 2 * G::kStages * 8 + 1024;  // + alignment slack
};

// Three CTAs per SM (at most 128 registers a thread: 15 warps leave 4 per SM
// sub-partition): a CTA's start-up -- table entries, then the first copies --
// overlaps the other two CTAs' streaming.
template <typename T, int D, int BS>
__global__ void __launch_bounds__(kThreads, 3)
decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const DecodeArgs a) {
    using G = Geom<D, BS>;
    using Lay = FixedLayout<D, BS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t base = smem_addr(smem);
    const uint32_t bar_full = base + Lay::kBarOffset;        // kStages x 8 B
    const uint32_t bar_empty = bar_full + 8 * G::kStages;    // kStages x 8 B

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x / a.num_kv_heads;
    const int hk = blockIdx.x - b * a.num_kv_heads;
    const int part = blockIdx.y;

    // Launched as a programmatic dependent of the previous kernel in the stream
    // (e.g. the append): nothing global is touched before that kernel is done.
    pdl_wait_primary();

    const int max_len = a.max_blocks_per_seq * BS;
    const int raw_len = __ldg(a.context_lens + b);
    const int L = clamp_len(raw_len, max_len);
    if (raw_len != L && threadIdx.x == 0 && part == 0 && hk == 0)
        flag(a.err_flag, PKV_DEVERR_BAD_CONTEXT_LEN);
    const int t_begin = part * a.partition_tokens;
    const int t_end = min(t_begin + a.partition_tokens, L);
    const int blk_begin = t_begin / BS;
    const int nblk = (t_end - t_begin + BS - 1) / BS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < G::kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
        const uint64_t policy = l2_evict_first_policy();
        const int32_t* row = a.block_tables + static_cast<int64_t>(b) * a.max_blocks_per_seq + blk_begin;
        int ok = 1;
        for (int i0 = 0; i0 < nblk && ok; i0 += 32) {
            int phys = 0;
            if (i0 + lane < nblk) {
                phys = __ldg(row + i0 + lane);
                if (phys < 0 || phys >= a.num_blocks) {
                    flag(a.err_flag, PKV_DEVERR_BAD_BLOCK_ID);
                    phys = 0;
                }
            }
            const int n = min(32, nblk - i0);
            for (int j = 0; j < n; ++j) {
                const int pj = __shfl_sync(0xffffffffu, phys, j);
                if (lane == 0 && ok) {
                    const int it = i0 + j;
                    const int s = it % G::kStages;
                    const int round = it / G::kStages;
                    if (round > 0 && !mbar_wait(bar_empty + 8 * s, (round - 1) & 1)) {
                        flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
                        ok = 0;
                    } else {
                        load_tile<D, BS>(&tm_k, &tm_v, base + s * G::kStageBytes, bar_full + 8 * s,
                                         pj, a.num_kv_heads, hk, policy);
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int group = a.group;
    const T* qbase = static_cast<const T*>(a.q) +
                     (static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group) * D;
    uint32_t qa[D / 16][4];
    load_q_fragments<T, D>(qa, qbase, group, lane);

    SoftmaxState<D> st;
    st.reset();
    for (int it = warp; it < nblk; it += kConsumerWarps) {
        const int s = it % G::kStages;
        const int round = it / G::kStages;
        const bool arrived = __all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, round & 1));
        if (!arrived) {
            if (lane == 0) flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const uint32_t kst = base + s * G::kStageBytes;
        const int tok_blk = (blk_begin + it) * BS;
#pragma unroll
        for (int sub = 0; sub < BS / 16; ++sub) {
            const int tok0 = tok_blk + sub * 16;
            if (tok0 >= t_end) break;
            attend_16<T, D>(st, qa, kst, kst + G::kTileBytes, G::kHalfBytes, sub, tok0, t_end,
                            a.scale_log2, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }

    // ----------------------------------------------- merge the four warps
    finish_row_sums(st);
    consumer_sync();  // every consumer is done with the ring: reuse it
    float* mo = reinterpret_cast<float*>(smem);              // [warp][group][D]
    float* mm = mo + kConsumerWarps * 16 * D;                // [warp][group]
    float* ml = mm + kConsumerWarps * 16;                    // [warp][group]
    store_warp_state(st, mo, mm, ml, warp, group, lane);
    consumer_sync();

    for (int idx = threadIdx.x; idx < group * D; idx += kConsumerWarps * 32) {
        const int r = idx / D;
        const int d = idx - r * D;
        float M, acc, den;
        combine_warps<D>(mo, mm, ml, kConsumerWarps, group, r, d, M, acc, den);
        const int64_t bh = static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group + r;
        static_cast<T*>(a.out)[bh * D + d] = Pack<T>::one(den > 0.f ? acc / den : 0.f);
    }
}

// Merge the partitions of one (sequence, query head) by log-sum-exp:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// With LANES = 1, D threads (one per column) walk p = 0, 1, ... in order.  With
// many partitions (LANES = 4), LANES groups of D threads split them -- group q
// takes p = q, q + LANES, ... in ascending order -- so that many partials are
// read at once, and the groups' sums are added in group order.  Either order
// depends only on the shapes.
template <typename T, int D, int LANES>
__global__ void __launch_bounds__(LANES * D) reduce_kernel(const DecodeArgs a, int32_t max_len) {
    // a kernel launched behind this one may start its set-up now (it waits for
    // this grid before touching memory)
    pdl_launch_dependents();
    pdl_wait_primary();  // the partition kernel's results are visible after this
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / a.num_heads);
    const int tid = threadIdx.x;
    const int L = clamp_len(__ldg(a.context_lens + b), max_len);
    const int n = (L + a.partition_tokens - 1) / a.partition_tokens;
    const float* m = a.ws_m + bh * a.max_partitions;
    const float* l = a.ws_l + bh * a.max_partitions;
    const float* o = a.ws_o + bh * a.max_partitions * D;
    if constexpr (LANES == 1) {
        const int d = tid;
        float M = -INFINITY;
        for (int p = 0; p < n; ++p) M = fmaxf(M, m[p]);
        float acc = 0.f, den = 0.f;
        for (int p = 0; p < n; ++p) {
            const float f = exp2_approx(m[p] - M);
            acc += f * o[static_cast<int64_t>(p) * D + d];
            den += f * l[p];
        }
        static_cast<T*>(a.out)[bh * D + d] = Pack<T>::one(den > 0.f ? acc / den : 0.f);
    } else {
        __shared__ float s_max[LANES * D / 32];
        __shared__ float s_acc[LANES][D];
        __shared__ float s_den[LANES];
        const int q = tid / D;
        const int d = tid - q * D;
        // M over all partitions: one strided pass by every thread, then the block
        float M = -INFINITY;
        for (int p = tid; p < n; p += LANES * D) M = fmaxf(M, m[p]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        if ((tid & 31) == 0) s_max[tid >> 5] = M;
        __syncthreads();
        M = -INFINITY;
#pragma unroll
        for (int w = 0; w < LANES * D / 32; ++w) M = fmaxf(M, s_max[w]);
        float acc = 0.f, den = 0.f;
#pragma unroll 4
        for (int p = q; p < n; p += LANES) {
            const float f = exp2_approx(m[p] - M);
            acc += f * o[static_cast<int64_t>(p) * D + d];
            den += f * l[p];
        }
        s_acc[q][d] = acc;
        if (d == 0) s_den[q] = den;
        __syncthreads();
        if (q == 0) {
            float sum = s_acc[0][d], dsum = s_den[0];
#pragma unroll
            for (int g = 1; g < LANES; ++g) {
                sum += s_acc[g][d];
                dsum += s_den[g];
            }
            static_cast<T*>(a.out)[bh * D + d] = Pack<T>::one(dsum > 0.f ? sum / dsum : 0.f);
        }
    }
}

// Partitions per (sequence, head) from which the merge splits them over four
// thread groups.
constexpr int64_t kWideReduceFrom = 32;

// =========================================================================== balanced

constexpr int kSegSlots = 4;          // segment descriptors in flight
constexpr int kMergeSlots = 2;        // segments handed to the merge warp, in flight
constexpr int kBalancedThreads = (kConsumerWarps + 2) * 32;  // + producer + merge warp
constexpr int kMinUnits = 8;          // fewest units a CTA of the balanced grid takes
constexpr int kMetaValid = 1;         // partial-slot meta flags
constexpr int kMetaBegins = 2;        // the segment starts at the (b, hk)'s first block
constexpr int kMetaEnds = 4;          // the segment ends at the (b, hk)'s last block
constexpr int kSegFirstInCta = 8;     // descriptor-only flags
constexpr int kSegEnd = 16;           // end of the CTA's range

struct BalancedArgs {
    void* out;
    const void* q;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_o;      // [G][2][group][D]   un-normalised partial O
    float* ws_ml;     // [G][2][group][2]   partial (m, l)
    int32_t* ws_meta; // [G][2][4]          (b, hk, flags, 0)
    int32_t* err_flag;
    int32_t num_seqs;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t group;
    int32_t max_blocks_per_seq;
    int32_t num_blocks;
    int32_t max_len;  // max_blocks_per_seq * block_size
    float scale_log2;
    // fixed partitions (part_units > 0): every partition of part_units units
    // leaves its partial in [row][partition] slots for reduce_kernel
    int32_t part_units;
    int32_t max_partitions;
    float* part_o;  // [B][H][P_max][D]
    float* part_m;  // [B][H][P_max]
    float* part_l;  // [B][H][P_max]
};

struct SegDesc {
    int32_t b, hk, first, n;  // CTA-local index of the first unit, unit count
    int32_t blk0, len, flags, beg;  // beg: first token the segment's units count from
    int32_t part, pad[3];           // partition of the segment (fixed partitions)
};

// The balanced kernel streams 16-token units: a block of 32 tokens is two units
// (two TMA boxes of 16 rows), so every block size gets the same 64 KiB ring of
// 8 KiB (head_dim 128) or 4 KiB (head_dim 64) stages, at least two per warp.
template <int D>
struct UnitGeom {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = 16 * 128;               // 16 rows x 128 B, 128B swizzle
    static constexpr int kTileBytes = kHalves * kHalfBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;        // K + V
    static constexpr int kRingBytes = 64 * 1024;
    static constexpr int kStages = kRingBytes / kStageBytes;  // 8 or 16
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
};

// Byte offsets inside the (1 KB aligned) dynamic shared memory of the balanced
// kernel; the part after the ring depends on the group size.
template <int D>
struct BalancedLayout {
    using G = UnitGeom<D>;
    // merge slot: mo [warps][group][D], mm [warps][group], ml [warps][group], 4 ints
    int qslot_bytes, q_off, mslot_bytes, merge_off, desc_off, bar_off, abort_off, total;
    __host__ __device__ explicit BalancedLayout(int group) {
        qslot_bytes = group * D * 2;                                   // multiple of 128
        q_off = G::kRingBytes;
        mslot_bytes = ((kConsumerWarps * group * (D + 2) * 4 + 16) + 15) & ~15;
        merge_off = q_off + kSegSlots * qslot_bytes;
        desc_off = merge_off + kMergeSlots * mslot_bytes;
        bar_off = desc_off + kSegSlots * static_cast<int>(sizeof(SegDesc));
        // full[S], empty[S], seg_full[4], seg_empty[4], mslot_full[2], mslot_empty[2]
        abort_off = bar_off + (2 * G::kStages + 2 * kSegSlots + 2 * kMergeSlots) * 8;
        total = abort_off + 16 + 1024;  // + 1 KB alignment slack
    }
};

// Poll a barrier until the phase with `parity` completes, about kWaitCycles SM
// cycles pass or another warp has aborted; false unless the phase completed.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity,
                                              const volatile int* abort_word) {
    if (mbar_test(bar, parity)) return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_test(bar, parity)) return true;
        if (*abort_word || clock64() - t0 > kWaitCycles) return false;
    }
}

// Diagnostic (pkv_selftest_wait_timeout): one warp waits on an mbarrier that
// nothing ever arrives on -- with the plain bounded wait (which = 0) or the
// abortable one (which = 1) -- and must give up by itself and report it.
__global__ void selftest_wait_kernel(int which, int32_t* err) {
    __shared__ __align__(8) uint64_t bar_word;
    __shared__ int abort_word;
    const uint32_t bar = smem_addr(&bar_word);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        abort_word = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const bool ok = which == 0 ? mbar_wait(bar, 0) : wait_or_abort(bar, 0, &abort_word);
    if (!__all_sync(0xffffffffu, ok) && threadIdx.x == 0) flag(err, PKV_DEVERR_WAIT_TIMEOUT);
}

// Issue the K and V tiles of one 16-token unit: rows [row0, row0 + 16) of the
// pools' 2-D view.
template <int D>
__device__ __forceinline__ void load_unit(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                          uint32_t stage_addr, uint32_t full_bar, int row0,
                                          uint64_t policy) {
    using G = UnitGeom<D>;
    mbar_arrive_expect_tx(full_bar, G::kStageBytes);
    tma_load_3d(stage_addr, tm_k, 0, row0, 0, full_bar, policy);
    tma_load_3d(stage_addr + G::kTileBytes, tm_v, 0, row0, 0, full_bar, policy);
}

// Up to 32 consecutive units of one (b, hk), with the physical block of each
// unit held by lane j of the producer warp (unit j of the chunk).
struct Chunk {
    int b, hk, u0, cnt;   // sequence, kv head, first unit within (b, hk), units
    int len, nu;          // the sequence's length and its units per kv head
    int beg;              // first token of unit 0 (after the shared prefix, if any)
    int pbeg, pend;       // units [pbeg, pend) of (b, hk) form the chunk's partition
                          // (the whole (b, hk) without fixed partitions)
    int seg_start;        // the chunk opens a segment of seg_len units
    int seg_len;
    int phys;             // this lane's physical block
};

// With CASCADE, sequences of a group that shares blocks attend here only to
// their own tokens (from the group's shared_tokens on; units count from
// there), and their results stay un-normalised partials (CascadeGroups
// own_o / own_ml) for cascade_finalize_kernel to merge with the prefix.
template <bool CASCADE>
using GroupsOf = typename std::conditional<CASCADE, CascadeGroups, NoGroups>::type;

template <bool CASCADE>
__device__ __forceinline__ int first_token(const GroupsOf<CASCADE>& cg, int b) {
    if constexpr (CASCADE) return shared_begin(cg, b);
    else return 0;
}

template <typename T, int D, int BS, bool CASCADE>
__global__ void __launch_bounds__(kBalancedThreads, 2)
balanced_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const BalancedArgs a, const __grid_constant__ GroupsOf<CASCADE> cg) {
    using G = UnitGeom<D>;
    constexpr int R = BS / 16;  // units per block
    extern __shared__ uint8_t smem_raw[];
    __shared__ long long s_warp_units[kConsumerWarps + 2];
    __shared__ int s_start[3];

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int group = a.group;
    const BalancedLayout<D> lay(group);
    const uint32_t base = smem_addr(smem);
    const uint32_t bar_full = base + lay.bar_off;
    const uint32_t bar_empty = bar_full + 8 * G::kStages;
    const uint32_t seg_full = bar_empty + 8 * G::kStages;
    const uint32_t seg_empty = seg_full + 8 * kSegSlots;
    const uint32_t mslot_full = seg_empty + 8 * kSegSlots;
    const uint32_t mslot_empty = mslot_full + 8 * kMergeSlots;
    volatile int* abort_word = reinterpret_cast<volatile int*>(smem + lay.abort_off);
    SegDesc* descs = reinterpret_cast<SegDesc*>(smem + lay.desc_off);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int c = blockIdx.x;
    const int grid = gridDim.x;
    const int B = a.num_seqs;
    const int Hkv = a.num_kv_heads;
    const int max_len = a.max_blocks_per_seq * BS;

    // Launched as a programmatic dependent of the previous kernel in the stream
    // (e.g. the append): nothing global is touched before that kernel is done.
    pdl_wait_primary();
    pdl_launch_dependents();
    if (tid < 8) a.ws_meta[static_cast<int64_t>(c) * 8 + tid] = 0;  // both partial slots invalid

    // ---- which units are this CTA's: units per sequence, scanned over the batch
    const int chunk = (B + kBalancedThreads - 1) / kBalancedThreads;
    const int b_lo = min(B, tid * chunk), b_hi = min(B, b_lo + chunk);
    long long mine = 0;
    for (int b = b_lo; b < b_hi; ++b) {
        const int raw = __ldg(a.context_lens + b);
        const int L = clamp_len(raw, max_len);
        const int beg = first_token<CASCADE>(cg, b);
        if ((raw != L || L < beg) && c == 0) flag(a.err_flag, PKV_DEVERR_BAD_CONTEXT_LEN);
        mine += (max(L - beg, 0) + 15) / 16;
    }
    long long incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) s_warp_units[warp] = incl;
    if (tid == 0) s_start[0] = -1;
    __syncthreads();
    long long before = 0, total = 0;
    for (int w = 0; w < kConsumerWarps + 2; ++w) {
        if (w < warp) before += s_warp_units[w];
        total += s_warp_units[w];
    }
    const long long excl = before + incl - mine;          // units (per kv head) before b_lo
    const long long units = total * Hkv;
    // Spread the units over min(G, ceil(U / kMinUnits)) CTAs: every range is
    // non-empty (at least kMinUnits units unless U is smaller), and the CTAs that
    // share one (b, hk) are consecutive.  Small batches thus use fewer CTAs
    // instead of splitting every sequence into one-unit pieces.
    const long long want = (units + kMinUnits - 1) / kMinUnits;
    const long long used = want < grid ? want : grid;
    const long long u0 = c < used ? static_cast<long long>(c) * units / used : 0;
    const long long u1 = c < used ? static_cast<long long>(c + 1) * units / used : 0;
    if (u0 < u1 && mine > 0 && excl * Hkv <= u0 && u0 < (excl + mine) * Hkv) {
        long long p = excl;
        for (int b = b_lo; b < b_hi; ++b) {
            const int nu =
                (max(clamp_len(__ldg(a.context_lens + b), max_len) - first_token<CASCADE>(cg, b), 0) + 15) / 16;
            if (u0 < (p + nu) * Hkv) {
                const long long r = u0 - p * Hkv;
                s_start[0] = b;
                s_start[1] = static_cast<int>(r / nu);
                s_start[2] = static_cast<int>(r % nu);
                break;
            }
            p += nu;
        }
    }
    if (tid == 0) {
        for (int s = 0; s < G::kStages; ++s) {
            mbar_init(bar_full + 8 * s, 1);
            mbar_init(bar_empty + 8 * s, 1);
        }
        for (int k = 0; k < kSegSlots; ++k) {
            mbar_init(seg_full + 8 * k, 1);
            mbar_init(seg_empty + 8 * k, kConsumerWarps);
        }
        for (int k = 0; k < kMergeSlots; ++k) {
            mbar_init(mslot_full + 8 * k, kConsumerWarps);
            mbar_init(mslot_empty + 8 * k, 1);
        }
        *abort_word = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (u0 >= u1 || s_start[0] < 0) return;  // no units for this CTA
    const int n_units = static_cast<int>(u1 - u0);

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        // Walks the range chunk by chunk; the table entries (and the length of
        // the next sequence) are loaded one chunk ahead, before the warp blocks
        // on the ring, so a segment boundary costs no idle DRAM time.
        if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
        }
        const uint64_t policy = l2_evict_first_policy();
        int b = s_start[0], hk = s_start[1], ub = s_start[2];  // walk cursor
        int len = clamp_len(__ldg(a.context_lens + b), max_len);
        int beg = first_token<CASCADE>(cg, b);
        int nu = (max(len - beg, 0) + 15) / 16;
        // raw, clamped only when used, so the load does not stall the warp here
        int len_next_raw = b + 1 < B ? __ldg(a.context_lens + b + 1) : 0;
        int walked = 0;  // units already assigned to chunks

        // Take the next chunk from the cursor and issue its table loads.
        auto take = [&](Chunk& ch) -> bool {
            if (ub == nu) {  // the (b, hk) is done: next kv head, or next sequence with tokens
                ub = 0;
                if (++hk == Hkv) {
                    hk = 0;
                    ++b;
                    len = clamp_len(len_next_raw, max_len);
                    beg = first_token<CASCADE>(cg, b);
                    while (len <= beg && b + 1 < B) {
                        ++b;
                        len = clamp_len(__ldg(a.context_lens + b), max_len);
                        beg = first_token<CASCADE>(cg, b);
                    }
                    nu = (max(len - beg, 0) + 15) / 16;
                    len_next_raw = b + 1 < B ? __ldg(a.context_lens + b + 1) : 0;
                }
            }
            ch.b = b;
            ch.hk = hk;
            ch.u0 = ub;
            ch.len = len;
            ch.nu = nu;
            ch.beg = beg;
            // with fixed partitions a segment never crosses a partition boundary
            const int pu = a.part_units;
            ch.pbeg = pu > 0 ? ub - ub % pu : 0;
            ch.pend = pu > 0 ? min(nu, ch.pbeg + pu) : nu;
            ch.cnt = min(32, min(ch.pend - ub, n_units - walked));
            if (ch.cnt <= 0) return false;  // lengths changed under the kernel
            ch.seg_start = ub == ch.pbeg || walked == 0;
            ch.seg_len = min(ch.pend - ub, n_units - walked);
            // the entries are checked when they are used, so the loads stay in flight
            ch.phys = lane < ch.cnt
                          ? __ldg(a.block_tables + static_cast<int64_t>(b) * a.max_blocks_per_seq +
                                  beg / BS + (ub + lane) / R)
                          : 0;
            ub += ch.cnt;
            walked += ch.cnt;
            return true;
        };

        int ok = 1, i = 0, seg = 0;
        int tiles_issued = 0, queries_issued = 0;  // lane 0's counts of copies issued
        Chunk cur, nxt;
        ok = take(cur);
        while (ok) {
            const bool more = walked < n_units;
            if (more && !take(nxt)) ok = 0;
            if (!ok) break;
            if (cur.seg_start) {
                const int ks = seg % kSegSlots;
                if (lane == 0) {
                    if (seg >= kSegSlots &&
                        !wait_or_abort(seg_empty + 8 * ks, ((seg / kSegSlots) - 1) & 1, abort_word)) {
                        ok = 0;
                    } else {
                        SegDesc& d = descs[ks];
                        d.b = cur.b;
                        d.hk = cur.hk;
                        d.first = i;
                        d.n = cur.seg_len;
                        d.blk0 = cur.u0;
                        d.len = cur.len;
                        d.beg = cur.beg;
                        d.flags = (cur.u0 == cur.pbeg ? kMetaBegins : 0) |
                                  (cur.u0 + cur.seg_len == cur.pend ? kMetaEnds : 0) |
                                  (i == 0 ? kSegFirstInCta : 0);
                        d.part = a.part_units > 0 ? cur.pbeg / a.part_units : 0;
                        // the arrive releases the descriptor's stores to the consumers
                        mbar_arrive_expect_tx(seg_full + 8 * ks, lay.qslot_bytes);
                        const T* qsrc = static_cast<const T*>(a.q) +
                                        (static_cast<int64_t>(cur.b) * a.num_heads +
                                         static_cast<int64_t>(cur.hk) * group) * D;
                        bulk_load(base + lay.q_off + ks * lay.qslot_bytes, qsrc, lay.qslot_bytes,
                                  seg_full + 8 * ks);
                        ++queries_issued;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                ++seg;
                if (!ok) break;
            }
            for (int j = 0; j < cur.cnt; ++j) {
                int pj = __shfl_sync(0xffffffffu, cur.phys, j);
                if (pj < 0 || pj >= a.num_blocks) {
                    if (lane == 0) flag(a.err_flag, PKV_DEVERR_BAD_BLOCK_ID);
                    pj = 0;
                }
                if (lane == 0 && ok) {
                    const int u = i + j;
                    const int s = u % G::kStages;
                    const int round = u / G::kStages;
                    if (round > 0 && !wait_or_abort(bar_empty + 8 * s, (round - 1) & 1, abort_word)) {
                        ok = 0;
                    } else {
                        const int row0 = (pj * Hkv + cur.hk) * BS + ((cur.u0 + j) % R) * 16;
                        load_unit<D>(&tm_k, &tm_v, base + s * G::kStageBytes, bar_full + 8 * s, row0, policy);
                        ++tiles_issued;
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            i += cur.cnt;
            if (!more || !ok) break;
            cur = nxt;
        }
        if (lane == 0) {
            if (ok) {
                const int ks = seg % kSegSlots;
                if (seg >= kSegSlots &&
                    !wait_or_abort(seg_empty + 8 * ks, ((seg / kSegSlots) - 1) & 1, abort_word)) {
                    ok = 0;
                } else {
                    descs[ks].n = 0;
                    descs[ks].flags = kSegEnd;
                    mbar_arrive(seg_full + 8 * ks);
                }
            }
            if (!ok) {
                // Timed out or aborted: flag it, and before leaving wait (bounded)
                // for the copies this warp issued, so none lands after the CTA ends.
                flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
                *abort_word = 1;
                for (int s = 0; s < G::kStages && s < tiles_issued; ++s)
                    mbar_wait(bar_full + 8 * s, ((tiles_issued - 1 - s) / G::kStages) & 1);
                for (int k = 0; k < kSegSlots && k < queries_issued; ++k)
                    mbar_wait(seg_full + 8 * k, ((queries_issued - 1 - k) / kSegSlots) & 1);
            }
        }
        return;
    }

    if (warp == kConsumerWarps + 1) {
        // ---------------------------------------------------------- merge warp
        // Combines the four consumer warps' states of each segment, in segment
        // order, while the consumers already work on the next one.
        for (int seg = 0;; ++seg) {
            const int ms = seg % kMergeSlots;
            if (!__all_sync(0xffffffffu, wait_or_abort(mslot_full + 8 * ms, (seg / kMergeSlots) & 1, abort_word))) {
                if (lane == 0) flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
                *abort_word = 1;
                break;
            }
            const float* mo = reinterpret_cast<const float*>(smem + lay.merge_off + ms * lay.mslot_bytes);
            const float* mm = mo + kConsumerWarps * group * D;
            const float* ml = mm + kConsumerWarps * group;
            const int* smeta = reinterpret_cast<const int*>(ml + kConsumerWarps * group);
            const int flags = smeta[2];
            if (flags & kSegEnd) break;
            const int sb = smeta[0], shk = smeta[1], spart = smeta[3];
            const bool complete = (flags & (kMetaBegins | kMetaEnds)) == (kMetaBegins | kMetaEnds);
            const int64_t pslot = static_cast<int64_t>(c) * 2 + ((flags & kSegFirstInCta) ? 0 : 1);
            // A sequence of a group that shares blocks: its complete result over
            // its own tokens is a partial too (the prefix is folded in later).
            int pgrp = -1;
            if constexpr (CASCADE) pgrp = sharing_group_of(cg, sb);
            // Row by row: the weights 2^(m_w - M) once per row, then four columns
            // per lane (M = max_w m_w; acc = sum_w 2^(m_w - M) o_w; den likewise).
            for (int r = 0; r < group; ++r) {
                float mw[kConsumerWarps], M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    mw[w] = mm[w * group + r];
                    M = fmaxf(M, mw[w]);
                }
                float f[kConsumerWarps], den = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    f[w] = mw[w] == -INFINITY ? 0.f : exp2_approx(mw[w] - M);
                    den += f[w] * ml[w * group + r];
                }
                const int d0 = lane * 4;
                if (d0 < D) {
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        const float4 o = *reinterpret_cast<const float4*>(mo + (w * group + r) * D + d0);
                        acc.x += f[w] * o.x;
                        acc.y += f[w] * o.y;
                        acc.z += f[w] * o.z;
                        acc.w += f[w] * o.w;
                    }
                    if (complete && pgrp >= 0) {
                        if constexpr (CASCADE) {
                            const int64_t row = own_row(cg, pgrp, sb, a.num_heads, shk * group + r);
                            *reinterpret_cast<float4*>(cg.own_o + row * D + d0) = acc;
                            if (lane == 0) *reinterpret_cast<float2*>(cg.own_ml + row * 2) = make_float2(M, den);
                        }
                    } else if (complete && a.part_units > 0) {
                        // a whole partition: its partial goes to its slot
                        const int64_t bh = static_cast<int64_t>(sb) * a.num_heads + static_cast<int64_t>(shk) * group + r;
                        const int64_t slot = bh * a.max_partitions + spart;
                        *reinterpret_cast<float4*>(a.part_o + slot * D + d0) = acc;
                        if (lane == 0) {
                            a.part_m[slot] = M;
                            a.part_l[slot] = den;
                        }
                    } else if (complete) {
                        const float inv = den > 0.f ? 1.f / den : 0.f;
                        float r0, r1;
                        uint2 packed;
                        packed.x = Pack<T>::two(acc.x * inv, acc.y * inv, r0, r1);
                        packed.y = Pack<T>::two(acc.z * inv, acc.w * inv, r0, r1);
                        const int64_t bh = static_cast<int64_t>(sb) * a.num_heads + static_cast<int64_t>(shk) * group + r;
                        *reinterpret_cast<uint2*>(static_cast<T*>(a.out) + bh * D + d0) = packed;
                    } else {
                        *reinterpret_cast<float4*>(a.ws_o + (pslot * group + r) * D + d0) = acc;
                        if (lane == 0) {
                            a.ws_ml[(pslot * group + r) * 2] = M;
                            a.ws_ml[(pslot * group + r) * 2 + 1] = den;
                        }
                    }
                }
            }
            if (!complete && lane == 0) {
                int32_t* meta = a.ws_meta + pslot * 4;
                meta[0] = sb;
                meta[1] = shk;
                meta[2] = kMetaValid | (flags & (kMetaBegins | kMetaEnds));
                meta[3] = spart;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(mslot_empty + 8 * ms);  // the slot may be refilled
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    // Hand this warp's state of segment `seg` (or, with flags = kSegEnd, the end
    // of the range) to the merge warp through merge slot seg % 2.
    auto publish = [&](int seg, const SoftmaxState<D>& state, int b_, int hk_, int flags_,
                       int part_) -> bool {
        const int ms = seg % kMergeSlots;
        if (seg >= kMergeSlots &&
            !__all_sync(0xffffffffu,
                        wait_or_abort(mslot_empty + 8 * ms, ((seg / kMergeSlots) - 1) & 1, abort_word)))
            return false;
        float* mo = reinterpret_cast<float*>(smem + lay.merge_off + ms * lay.mslot_bytes);
        float* mm = mo + kConsumerWarps * group * D;
        float* ml = mm + kConsumerWarps * group;
        int* smeta = reinterpret_cast<int*>(ml + kConsumerWarps * group);
        if (!(flags_ & kSegEnd)) store_warp_state(state, mo, mm, ml, warp, group, lane);
        if (warp == 0 && lane == 0) {
            smeta[0] = b_;
            smeta[1] = hk_;
            smeta[2] = flags_;
            smeta[3] = part_;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(mslot_full + 8 * ms);
        return true;
    };
    SoftmaxState<D> st;
    uint32_t qa[D / 16][4];
    bool ok = true;
    for (int seg = 0; ok; ++seg) {
        const int ks = seg % kSegSlots;
        if (!__all_sync(0xffffffffu, wait_or_abort(seg_full + 8 * ks, (seg / kSegSlots) & 1, abort_word))) {
            ok = false;
            break;
        }
        const SegDesc d = descs[ks];
        if (d.flags & kSegEnd) {
            ok = publish(seg, st, 0, 0, kSegEnd, 0);  // the merge warp stops here
            break;
        }
        load_q_fragments<T, D>(qa, reinterpret_cast<const T*>(smem + lay.q_off + ks * lay.qslot_bytes),
                               group, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(seg_empty + 8 * ks);  // descriptor and queries are in registers

        st.reset();
        for (int u = d.first + ((warp - d.first) & 3); u < d.first + d.n; u += kConsumerWarps) {
            const int s = u % G::kStages;
            const int round = u / G::kStages;
            if (!__all_sync(0xffffffffu, wait_or_abort(bar_full + 8 * s, round & 1, abort_word))) {
                ok = false;
                break;
            }
            const uint32_t kst = base + s * G::kStageBytes;
            attend_16<T, D>(st, qa, kst, kst + G::kTileBytes, G::kHalfBytes, 0,
                            d.beg + (d.blk0 + (u - d.first)) * 16, d.len, a.scale_log2, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_empty + 8 * s);
        }
        if (!ok) break;

        finish_row_sums(st);
        if (!publish(seg, st, d.b, d.hk, d.flags, d.part)) {
            ok = false;
            break;
        }
    }
    if (!ok) {
        if (lane == 0) flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
        *abort_word = 1;
    }
}

// Merge the partials of every (b, hk) that was split across CTAs.  CTA c owns
// the chains that start in it (a partial marked "begins"); a chain continues in
// slot 0 of CTAs c+1, c+2, ... up to the partial marked "ends".  Each chain is
// merged in CTA order: M = max m_p, out = sum 2^(m_p - M) o_p / sum 2^(m_p - M) l_p.
// Sequences with no tokens get zeros here.
constexpr int kReduceThreads = 128;
constexpr int kChainWindow = 32;  // chains up to this many CTAs long are found in one round
constexpr int kShortChain = 4;    // chains up to this long are merged from registers

// With CASCADE, a grouped sequence with no tokens of its own (all of its
// context is the shared prefix) gets the prefix kernel's partials merged here.
template <typename T, int D, bool CASCADE>
__global__ void __launch_bounds__(kReduceThreads)
    balanced_reduce_kernel(const BalancedArgs a, const __grid_constant__ GroupsOf<CASCADE> cg) {
    __shared__ int s_meta[2 + kChainWindow][4];  // own slots 0 and 1, then slot 0 of c+1 ..
    __shared__ int s_len[2];
    const int c = blockIdx.x;
    const int grid = gridDim.x;
    const int group = a.group;
    const int tid = threadIdx.x;
    // a kernel launched behind this one may start its set-up now (it waits for
    // this grid before touching memory)
    pdl_launch_dependents();

    // The lengths are an input of the whole step (ready before the decode
    // started), so they are read before waiting for the decode's results.
    // tokens the balanced kernel attends for sequence b (lengths clamped as there)
    auto own_tokens = [&](int b) {
        const int L = clamp_len(__ldg(a.context_lens + b), a.max_len);
        return L - first_token<CASCADE>(cg, b);
    };
    bool empty_seq[4] = {false, false, false, false};
    {
        int k = 0;
        for (int b = c; b < a.num_seqs && k < 4; b += grid, ++k) empty_seq[k] = own_tokens(b) <= 0;
    }

    pdl_wait_primary();  // the decode's partials and descriptors are visible after this
    if (tid < 2 + kChainWindow) {
        const int cc = tid < 2 ? c : c + tid - 1;
        const int slot = tid == 1 ? 1 : 0;
        int m0 = 0, m1 = 0, m2 = 0, m3 = 0;
        if (cc < grid) {
            const int32_t* m = a.ws_meta + (static_cast<int64_t>(cc) * 2 + slot) * 4;
            m0 = m[0];
            m1 = m[1];
            m2 = m[2];
            m3 = m[3];
        }
        s_meta[tid][0] = m0;
        s_meta[tid][1] = m1;
        s_meta[tid][2] = m2;
        s_meta[tid][3] = m3;
    }
    __syncthreads();
    if (tid < 2) {
        // chain starting in this CTA's slot `tid`: it continues in slot 0 of
        // c+1, c+2, ... up to the partial marked "ends"
        int len = 0;
        const int f = s_meta[tid][2];
        if ((f & kMetaValid) && (f & kMetaBegins)) {
            const int b = s_meta[tid][0], hk = s_meta[tid][1], part = s_meta[tid][3];
            len = 1;
            for (int k = 1;; ++k) {
                int nf, nb, nhk, npart;
                if (k <= kChainWindow) {
                    nb = s_meta[k + 1][0];
                    nhk = s_meta[k + 1][1];
                    nf = s_meta[k + 1][2];
                    npart = s_meta[k + 1][3];
                } else if (c + k < grid) {
                    const int32_t* m = a.ws_meta + static_cast<int64_t>(c + k) * 8;
                    nb = m[0];
                    nhk = m[1];
                    nf = m[2];
                    npart = m[3];
                } else {
                    nf = 0;
                    nb = nhk = npart = -1;
                }
                if (!(nf & kMetaValid) || nb != b || nhk != hk || npart != part) {  // a CTA of the chain is missing
                    flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
                    break;
                }
                ++len;
                if (nf & kMetaEnds) break;
            }
        }
        s_len[tid] = len;
    }
    __syncthreads();

    for (int slot = 0; slot < 2; ++slot) {
        const int n = s_len[slot];
        if (n == 0) continue;
        const int b = s_meta[slot][0], hk = s_meta[slot][1], part = s_meta[slot][3];
        int pgrp = -1;  // a sequence of a sharing group: the chain's result stays a partial
        if constexpr (CASCADE) pgrp = sharing_group_of(cg, b);
        // (row, 4 columns) per thread: M = max m_p, out = sum 2^(m_p - M) o_p / sum 2^(m_p - M) l_p
        for (int item = tid; item < group * (D / 4); item += kReduceThreads) {
            const int r = item / (D / 4);
            const int d0 = (item - r * (D / 4)) * 4;
            float M = -INFINITY;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
            float den = 0.f;
            if (n <= kShortChain) {
                // A short chain's partials are all loaded at once (one round trip
                // after the decode ends), then combined in the order of the loop
                // below.
                float mk[kShortChain], lk[kShortChain];
                float4 ok[kShortChain];
#pragma unroll
                for (int k = 0; k < kShortChain; ++k) {
                    mk[k] = -INFINITY;
                    lk[k] = 0.f;
                    ok[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (k < n) {
                        const int64_t p = static_cast<int64_t>(c + k) * 2 + (k == 0 ? slot : 0);
                        mk[k] = a.ws_ml[(p * group + r) * 2];
                        lk[k] = a.ws_ml[(p * group + r) * 2 + 1];
                        ok[k] = *reinterpret_cast<const float4*>(a.ws_o + (p * group + r) * D + d0);
                    }
                }
#pragma unroll
                for (int k = 0; k < kShortChain; ++k)
                    if (k < n) M = fmaxf(M, mk[k]);
#pragma unroll
                for (int k = 0; k < kShortChain; ++k) {
                    if (k < n) {
                        const float f = exp2_approx(mk[k] - M);
                        acc.x += f * ok[k].x;
                        acc.y += f * ok[k].y;
                        acc.z += f * ok[k].z;
                        acc.w += f * ok[k].w;
                        den += f * lk[k];
                    }
                }
            } else {
                for (int k = 0; k < n; ++k) {
                    const int64_t p = static_cast<int64_t>(c + k) * 2 + (k == 0 ? slot : 0);
                    M = fmaxf(M, a.ws_ml[(p * group + r) * 2]);
                }
                for (int k = 0; k < n; ++k) {
                    const int64_t p = static_cast<int64_t>(c + k) * 2 + (k == 0 ? slot : 0);
                    const float f = exp2_approx(a.ws_ml[(p * group + r) * 2] - M);
                    const float4 o = *reinterpret_cast<const float4*>(a.ws_o + (p * group + r) * D + d0);
                    acc.x += f * o.x;
                    acc.y += f * o.y;
                    acc.z += f * o.z;
                    acc.w += f * o.w;
                    den += f * a.ws_ml[(p * group + r) * 2 + 1];
                }
            }
            if constexpr (CASCADE) {
                if (pgrp >= 0) {
                    const int64_t row = own_row(cg, pgrp, b, a.num_heads, hk * group + r);
                    *reinterpret_cast<float4*>(cg.own_o + row * D + d0) = acc;
                    if (d0 == 0) *reinterpret_cast<float2*>(cg.own_ml + row * 2) = make_float2(M, den);
                    continue;
                }
            }
            if (a.part_units > 0) {  // a partition's partial, to its slot
                const int64_t bh = static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group + r;
                const int64_t pslot = bh * a.max_partitions + part;
                *reinterpret_cast<float4*>(a.part_o + pslot * D + d0) = acc;
                if (d0 == 0) {
                    a.part_m[pslot] = M;
                    a.part_l[pslot] = den;
                }
                continue;
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            float r0, r1;
            uint2 packed;
            packed.x = Pack<T>::two(acc.x * inv, acc.y * inv, r0, r1);
            packed.y = Pack<T>::two(acc.z * inv, acc.w * inv, r0, r1);
            const int64_t bh = static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group + r;
            *reinterpret_cast<uint2*>(static_cast<T*>(a.out) + bh * D + d0) = packed;
        }
    }

    // sequences with no tokens: zeros (context lengths <= 0 count as empty);
    // with CASCADE the sequences of sharing groups are written by
    // cascade_finalize_kernel instead, with fixed partitions every sequence by
    // reduce_kernel
    if (a.part_units > 0) return;
    int k = 0;
    for (int b = c; b < a.num_seqs; b += grid, ++k) {
        const bool empty = k < 4 ? empty_seq[k] : own_tokens(b) <= 0;
        if (!empty) continue;
        if constexpr (CASCADE) {
            if (sharing_group_of(cg, b) >= 0) continue;
        }
        T* o = static_cast<T*>(a.out) + static_cast<int64_t>(b) * a.num_heads * D;
        for (int idx = tid; idx < a.num_heads * D; idx += kReduceThreads) o[idx] = Pack<T>::one(0.f);
    }
}

// The last kernel of the shared-prefix decode: for every sequence of a sharing
// group, the partials of its heads over the shared blocks (one per prefix
// chunk, from prefix_kernel) and over its own tokens (from the kernels above;
// none when all its tokens are shared) merge by log-sum-exp, prefix chunks in
// order, then the own tokens:
//   M = max m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
// One warp per (grouped sequence, head): lane k holds chunk k's (m, l) (32 at
// a time), so the maximum and the weights take shuffles, not round trips;
// every lane then reads four columns of each chunk's O, eight chunks in
// flight.  Launched as a programmatic dependent of the prefix kernel, whose
// completion implies that of every kernel before it in the call.
constexpr int kFinalThreads = 128;
constexpr int kFinalChunks = 8;  // chunks' O rows in flight per lane

template <typename T, int D>
__global__ void __launch_bounds__(kFinalThreads)
    cascade_finalize_kernel(const BalancedArgs a, const __grid_constant__ CascadeGroups cg) {
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t row_all = static_cast<int64_t>(blockIdx.x) * (kFinalThreads / 32) + (threadIdx.x >> 5);
    if (row_all >= static_cast<int64_t>(cg.grouped_seqs) * a.num_heads) return;
    const int j = static_cast<int>(row_all / a.num_heads);  // grouped sequence
    const int h = static_cast<int>(row_all - static_cast<int64_t>(j) * a.num_heads);
    int grp = 0;
    while (grp + 1 < cg.num_groups && cg.seq_base[grp + 1] <= j) ++grp;
    while (grp < cg.num_groups && cg.shared_tokens[grp] == 0) ++grp;  // (seq_base skips them)
    const int b = cg.start[grp] + (j - cg.seq_base[grp]);
    const int L = clamp_len(__ldg(a.context_lens + b), a.max_len);
    const bool has_own = L > cg.shared_tokens[grp];
    const int nchunk = cg.chunks[grp];
    const int log2g = __ffs(a.group) - 1;  // a power of two in sharing groups
    const int64_t p0 = prefix_row(cg, grp, b, log2g, a.num_kv_heads, h, 0);
    const int64_t pstride = prefix_chunk_stride(a.num_kv_heads);
    const int64_t orow = own_row(cg, grp, b, a.num_heads, h);
    const int d0 = lane * 4;
    pdl_wait_primary();

    float M = -INFINITY;
    for (int k0 = 0; k0 < nchunk; k0 += 32)
        if (k0 + lane < nchunk) M = fmaxf(M, cg.pre_ml[(p0 + (k0 + lane) * pstride) * 2]);
    float2 own_ml = make_float2(-INFINITY, 0.f);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (has_own) {
        own_ml = *reinterpret_cast<const float2*>(cg.own_ml + orow * 2);
        M = fmaxf(M, own_ml.x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float den = 0.f;
    for (int k0 = 0; k0 < nchunk; k0 += 32) {
        float f = 0.f, l = 0.f;
        if (k0 + lane < nchunk) {
            const float2 x = *reinterpret_cast<const float2*>(cg.pre_ml + (p0 + (k0 + lane) * pstride) * 2);
            f = x.x == -INFINITY ? 0.f : exp2_approx(x.x - M);
            l = x.y;
        }
        float dl = f * l;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, off);
        den += dl;
        const int n = min(32, nchunk - k0);
        for (int q0 = 0; q0 < n; q0 += kFinalChunks) {
            float4 o[kFinalChunks];
#pragma unroll
            for (int q = 0; q < kFinalChunks; ++q)
                if (q0 + q < n && d0 < D)
                    o[q] = *reinterpret_cast<const float4*>(cg.pre_o + (p0 + (k0 + q0 + q) * pstride) * D + d0);
#pragma unroll
            for (int q = 0; q < kFinalChunks; ++q) {
                if (q0 + q < n) {
                    const float fq = __shfl_sync(0xffffffffu, f, q0 + q);
                    if (d0 < D) {
                        acc.x += fq * o[q].x;
                        acc.y += fq * o[q].y;
                        acc.z += fq * o[q].z;
                        acc.w += fq * o[q].w;
                    }
                }
            }
        }
    }
    if (has_own && own_ml.x != -INFINITY) {
        const float f = exp2_approx(own_ml.x - M);
        if (d0 < D) {
            const float4 o = *reinterpret_cast<const float4*>(cg.own_o + orow * D + d0);
            acc.x += f * o.x;
            acc.y += f * o.y;
            acc.z += f * o.z;
            acc.w += f * o.w;
        }
        den += f * own_ml.y;
    }
    if (d0 < D) {
        const float inv = den > 0.f ? 1.f / den : 0.f;
        float r0, r1;
        uint2 packed;
        packed.x = Pack<T>::two(acc.x * inv, acc.y * inv, r0, r1);
        packed.y = Pack<T>::two(acc.z * inv, acc.w * inv, r0, r1);
        const int64_t bh = static_cast<int64_t>(b) * a.num_heads + h;
        *reinterpret_cast<uint2*>(static_cast<T*>(a.out) + bh * D + d0) = packed;
    }
}

// ------------------------------------------------------------------ host side

// A 3-D view of one pool: x = 64 columns (128 B), y = row (num_blocks *
// num_kv_heads * block_size rows of head_dim elements), z = which 64-column
// half of the row (strides: 2 * head_dim bytes for y, 128 bytes for z).  A box
// of 64 x box_rows x head_dim/64 lands in shared memory as [half][row][128 B],
// 128B-swizzled, so one request fetches a whole (block, kv head) tile.
pkv_status encode_pool_map(CUtensorMap* tm, const void* pool, const pkv_cache_desc* d, int box_rows) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t rows = static_cast<cuuint64_t>(d->num_blocks) * d->num_kv_heads * d->block_size;
    const cuuint32_t halves = static_cast<cuuint32_t>(d->head_dim / 64);
    cuuint64_t dims[3] = {64, rows, halves};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d->head_dim) * 2, 128};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), halves};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(tm,
                        d->dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(pool), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    return PKV_OK;
}

template <typename T, int D, int BS>
struct FixedTag {};
template <typename T, int D, int BS, bool CASCADE>
struct BalancedTag {};

// One CTA per (sequence, kv head): the decode without a split.
template <typename T, int D, int BS>
pkv_status launch_unsplit(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                          int32_t num_seqs, cudaStream_t stream) {
    using Lay = FixedLayout<D, BS>;
    auto k = decode_kernel<T, D, BS>;
    cudaError_t e = opt_in_smem<FixedTag<T, D, BS>>(reinterpret_cast<const void*>(k));
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    e = launch_dependent(k, dim3(static_cast<unsigned>(num_seqs) * a.num_kv_heads), dim3(kThreads),
                         Lay::kSmemBytes, stream, tk, tv, a);
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

// The merge of fixed partitions, behind the kernels that wrote them: one CTA of
// D threads (four groups of D when rows have many partitions) per (sequence,
// query head), a programmatic dependent that waits for their results.
template <typename T, int D>
pkv_status launch_partition_merge(const DecodeArgs& a, int32_t num_seqs, int32_t max_len,
                                  cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_seqs) * a.num_heads);
    const bool wide = a.max_partitions >= kWideReduceFrom;
    cfg.blockDim = dim3((wide ? 4 : 1) * D);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = wide ? cudaLaunchKernelEx(&cfg, reduce_kernel<T, D, 4>, a, max_len)
                         : cudaLaunchKernelEx(&cfg, reduce_kernel<T, D, 1>, a, max_len);
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

// Resident CTAs of the balanced kernel on the current device: its grid size.
template <typename T, int D, int BS>
pkv_status balanced_grid(int group, int* grid_out, int* smem_out) {
    // resident CTAs per (device, group), computed once
    static std::atomic<int> cache[64][17];
    const BalancedLayout<D> lay(group);
    int dev0 = 0;
    if (cudaGetDevice(&dev0) == cudaSuccess && dev0 >= 0 && dev0 < 64 && group >= 1 && group <= 16) {
        const int g = cache[dev0][group].load(std::memory_order_acquire);
        if (g > 0) {
            *grid_out = g;
            *smem_out = lay.total;
            return PKV_OK;
        }
    }
    auto k = balanced_kernel<T, D, BS, false>;
    cudaError_t e = opt_in_smem<BalancedTag<T, D, BS, false>>(reinterpret_cast<const void*>(k));
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kBalancedThreads, lay.total)) != cudaSuccess)
        return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    if (per_sm < 1) return fail(PKV_ERR_UNSUPPORTED, "balanced decode does not fit on an SM");
    *grid_out = sms * per_sm;
    *smem_out = lay.total;
    if (dev >= 0 && dev < 64 && group >= 1 && group <= 16)
        cache[dev][group].store(*grid_out, std::memory_order_release);
    return PKV_OK;
}

// The cascade kernel has the same threads, shared memory and register cap
// (__launch_bounds__(.., 2)) as the plain one, so the same grid (and workspace
// layout) serves both.
template <typename T, int D, int BS, bool CASCADE>
pkv_status launch_balanced(const CUtensorMap& tk, const CUtensorMap& tv, const BalancedArgs& a,
                           const GroupsOf<CASCADE>& cg, int grid, int smem, cudaStream_t stream) {
    cudaError_t e;
    if constexpr (CASCADE) {
        e = opt_in_smem<BalancedTag<T, D, BS, true>>(
            reinterpret_cast<const void*>(balanced_kernel<T, D, BS, true>));
        if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    }
    e = launch_dependent(balanced_kernel<T, D, BS, CASCADE>, dim3(grid), dim3(kBalancedThreads), smem,
                         stream, tk, tv, a, cg);
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kReduceThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, balanced_reduce_kernel<T, D, CASCADE>, a, cg);
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

// Dispatch on (dtype, head_dim, block_size) to F<T, D, BS>::run.
template <template <typename, int, int> class F, typename... Args>
pkv_status dispatch(const pkv_cache_desc* d, Args&&... args) {
    if (d->dtype == PKV_BF16) {
        if (d->head_dim == 128 && d->block_size == 16) return F<__nv_bfloat16, 128, 16>::run(args...);
        if (d->head_dim == 128 && d->block_size == 32) return F<__nv_bfloat16, 128, 32>::run(args...);
        if (d->head_dim == 64 && d->block_size == 16) return F<__nv_bfloat16, 64, 16>::run(args...);
        return F<__nv_bfloat16, 64, 32>::run(args...);
    }
    if (d->head_dim == 128 && d->block_size == 16) return F<__half, 128, 16>::run(args...);
    if (d->head_dim == 128 && d->block_size == 32) return F<__half, 128, 32>::run(args...);
    if (d->head_dim == 64 && d->block_size == 16) return F<__half, 64, 16>::run(args...);
    return F<__half, 64, 32>::run(args...);
}

template <typename T, int D, int BS>
struct GridOf {
    static pkv_status run(int group, int* grid, int* smem) { return balanced_grid<T, D, BS>(group, grid, smem); }
};
template <typename T, int D, int BS>
struct RunUnsplit {
    static pkv_status run(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                          int32_t num_seqs, cudaStream_t st) {
        return launch_unsplit<T, D, BS>(tk, tv, a, num_seqs, st);
    }
};
template <typename T, int D, int BS>
struct RunPartitionMerge {
    static pkv_status run(const DecodeArgs& a, int32_t num_seqs, int32_t max_len, cudaStream_t st) {
        return launch_partition_merge<T, D>(a, num_seqs, max_len, st);
    }
};
template <typename T, int D, int BS>
struct RunBalanced {
    static pkv_status run(const CUtensorMap& tk, const CUtensorMap& tv, const BalancedArgs& a,
                          int grid, int smem, cudaStream_t st) {
        return launch_balanced<T, D, BS, false>(tk, tv, a, NoGroups{0}, grid, smem, st);
    }
};
template <typename T, int D, int BS>
struct RunCascade {
    static pkv_status run(const CUtensorMap& tk, const CUtensorMap& tv, const BalancedArgs& a,
                          const CascadeGroups& cg, int grid, int smem, cudaStream_t st) {
        return launch_balanced<T, D, BS, true>(tk, tv, a, cg, grid, smem, st);
    }
};

// Partition partials of the fixed-partition path (0 when it does not split).
size_t partition_slots_bytes(const pkv_cache_desc* d, int32_t num_seqs, int32_t num_heads,
                             int32_t max_blocks_per_seq, int32_t P) {
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * d->block_size;
    if (P == 0 || P >= max_len) return 0;
    const int64_t pmax = (max_len + P - 1) / P;
    return static_cast<size_t>(num_seqs) * num_heads * pmax * (d->head_dim + 2) * sizeof(float);
}

// Workspace of the balanced path: two partial slots per CTA.
size_t balanced_workspace(int grid, int group, int D) {
    return static_cast<size_t>(grid) * 2 *
           (static_cast<size_t>(group) * (D + 2) * sizeof(float) + 4 * sizeof(int32_t));
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_selftest_wait_timeout(int32_t which, int32_t* err_flag, void* stream) {
    if (which < 0 || which > 2) return fail(PKV_ERR_INVALID_ARG, "which must be 0, 1 or 2");
    if (!err_flag) return fail(PKV_ERR_INVALID_ARG, "err_flag is required");
    cudaError_t e;
    if (which == 2) {
        e = prefill_selftest_wait(err_flag, static_cast<cudaStream_t>(stream));
    } else {
        selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(which, err_flag);
        e = cudaGetLastError();
    }
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

extern "C" size_t paged_attention_workspace_bytes(const pkv_cache_desc* desc, int32_t num_seqs,
                                                  int32_t num_heads, int32_t max_blocks_per_seq,
                                                  int32_t partition_size) {
    if (check_desc(desc) != PKV_OK || num_seqs <= 0 || num_heads <= 0 || max_blocks_per_seq <= 0 ||
        partition_size < 0 || num_heads % desc->num_kv_heads != 0)
        return 0;
    const size_t parts =
        partition_slots_bytes(desc, num_seqs, num_heads, max_blocks_per_seq, partition_size);
    if (partition_size > 0 && parts == 0) return 0;  // fixed partitions, no split
    const int group = num_heads / desc->num_kv_heads;
    if (group > 16) return 0;
    int grid = 0, smem = 0;
    if (dispatch<GridOf>(desc, group, &grid, &smem) != PKV_OK) return 0;
    const size_t balanced = balanced_workspace(grid, group, desc->head_dim);
    return parts ? round256(balanced) + parts : balanced;
}

namespace pkv {
namespace {

// Host checks shared by the decode entry points (nothing is enqueued when they
// fail); num_seqs == 0 passes and means nothing to do.
pkv_status check_decode_args(const pkv_cache_desc* desc, const void* out, const void* q,
                             const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                             int32_t num_seqs, int32_t num_heads, float scale) {
    pkv_status st = check_desc(desc);
    if (st != PKV_OK) return st;
    if (num_seqs < 0 || num_heads <= 0 || max_blocks_per_seq <= 0)
        return fail(PKV_ERR_INVALID_ARG,
                    "paged_attention_decode: bad num_seqs, num_heads or max_blocks_per_seq");
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG,
                    "paged_attention_decode: q, out and pools must be 16-byte aligned");
    if (num_heads % desc->num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_heads must be a multiple of num_kv_heads");
    if (num_heads / desc->num_kv_heads > 16)
        return fail(PKV_ERR_UNSUPPORTED, "num_heads / num_kv_heads must be <= 16");
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
        return fail(PKV_ERR_INVALID_ARG, "scale must be finite");
    if (static_cast<int64_t>(max_blocks_per_seq) * desc->block_size > INT32_MAX / 2)
        return fail(PKV_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size too large");
    if (static_cast<int64_t>(num_seqs) * max_blocks_per_seq * desc->num_kv_heads > INT32_MAX)
        return fail(PKV_ERR_UNSUPPORTED,
                    "num_seqs * max_blocks_per_seq * num_kv_heads must be < 2^31");
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status paged_attention_decode(const pkv_cache_desc* desc, void* out, const void* q,
                                             const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables,
                                             int32_t max_blocks_per_seq,
                                             const int32_t* context_lens, int32_t num_seqs,
                                             int32_t num_heads, float scale,
                                             int32_t partition_size, void* workspace,
                                             size_t workspace_bytes, int32_t* err_flag,
                                             void* stream) {
    pkv_status st = check_decode_args(desc, out, q, k_cache, v_cache, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, num_heads, scale);
    if (st != PKV_OK || num_seqs == 0) return st;
    const int32_t group = num_heads / desc->num_kv_heads;
    if (partition_size < 0 || (partition_size > 0 && partition_size % desc->block_size != 0))
        return fail(PKV_ERR_INVALID_ARG,
                    "partition_size must be 0 or a positive multiple of block_size");

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap tk, tv;

    if (partition_size == 0) {
        int grid = 0, smem = 0;
        if ((st = dispatch<GridOf>(desc, static_cast<int>(group), &grid, &smem)) != PKV_OK) return st;
        const size_t need = balanced_workspace(grid, group, desc->head_dim);
        if (!workspace || workspace_bytes < need)
            return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "paged_attention_decode: workspace too small");
        if (!aligned(workspace, 16))
            return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: workspace must be 16-byte aligned");
        if ((st = encode_pool_map(&tk, k_cache, desc, 16)) != PKV_OK) return st;
        if ((st = encode_pool_map(&tv, v_cache, desc, 16)) != PKV_OK) return st;
        BalancedArgs a = {};
        a.out = out;
        a.q = q;
        a.block_tables = block_tables;
        a.context_lens = context_lens;
        a.ws_o = static_cast<float*>(workspace);
        a.ws_ml = a.ws_o + static_cast<int64_t>(grid) * 2 * group * desc->head_dim;
        a.ws_meta = reinterpret_cast<int32_t*>(a.ws_ml + static_cast<int64_t>(grid) * 2 * group * 2);
        a.err_flag = err_flag;
        a.num_seqs = num_seqs;
        a.num_heads = num_heads;
        a.num_kv_heads = desc->num_kv_heads;
        a.group = group;
        a.max_blocks_per_seq = max_blocks_per_seq;
        a.num_blocks = desc->num_blocks;
        a.max_len = max_blocks_per_seq * desc->block_size;
        a.scale_log2 = scale * kLog2e;
        return dispatch<RunBalanced>(desc, tk, tv, a, grid, smem, s);
    }

    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * desc->block_size;
    const bool split = partition_size < max_len;
    DecodeArgs a = {};
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.err_flag = err_flag;
    a.num_heads = num_heads;
    a.num_kv_heads = desc->num_kv_heads;
    a.group = group;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = desc->num_blocks;
    a.scale_log2 = scale * kLog2e;
    if (split) {
        // Fixed partitions on the balanced schedule: its segments stop at
        // partition boundaries, every partition's partial lands in its slot
        // (whole ones from the decode's merge warp, split ones from the chain
        // merge), and reduce_kernel merges each row's partitions in order.
        const int64_t pmax = (max_len + partition_size - 1) / partition_size;
        if (pmax > 65535) return fail(PKV_ERR_UNSUPPORTED, "too many partitions (> 65535)");
        int grid = 0, smem = 0;
        if ((st = dispatch<GridOf>(desc, static_cast<int>(group), &grid, &smem)) != PKV_OK) return st;
        const size_t balanced = balanced_workspace(grid, group, desc->head_dim);
        const size_t need = round256(balanced) +
                            partition_slots_bytes(desc, num_seqs, num_heads, max_blocks_per_seq,
                                                  partition_size);
        if (!workspace || workspace_bytes < need)
            return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "paged_attention_decode: workspace too small");
        if (!aligned(workspace, 16))
            return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: workspace must be 16-byte aligned");
        const int64_t rows = static_cast<int64_t>(num_seqs) * num_heads * pmax;
        a.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + round256(balanced));
        a.ws_m = a.ws_o + rows * desc->head_dim;
        a.ws_l = a.ws_m + rows;
        a.partition_tokens = partition_size;
        a.max_partitions = static_cast<int32_t>(pmax);
        BalancedArgs ba = {};
        ba.out = out;
        ba.q = q;
        ba.block_tables = block_tables;
        ba.context_lens = context_lens;
        ba.ws_o = static_cast<float*>(workspace);
        ba.ws_ml = ba.ws_o + static_cast<int64_t>(grid) * 2 * group * desc->head_dim;
        ba.ws_meta = reinterpret_cast<int32_t*>(ba.ws_ml + static_cast<int64_t>(grid) * 2 * group * 2);
        ba.err_flag = err_flag;
        ba.num_seqs = num_seqs;
        ba.num_heads = num_heads;
        ba.num_kv_heads = desc->num_kv_heads;
        ba.group = group;
        ba.max_blocks_per_seq = max_blocks_per_seq;
        ba.num_blocks = desc->num_blocks;
        ba.max_len = static_cast<int32_t>(max_len);
        ba.scale_log2 = scale * kLog2e;
        ba.part_units = partition_size / 16;
        ba.max_partitions = static_cast<int32_t>(pmax);
        ba.part_o = a.ws_o;
        ba.part_m = a.ws_m;
        ba.part_l = a.ws_l;
        if ((st = encode_pool_map(&tk, k_cache, desc, 16)) != PKV_OK) return st;
        if ((st = encode_pool_map(&tv, v_cache, desc, 16)) != PKV_OK) return st;
        if ((st = dispatch<RunBalanced>(desc, tk, tv, ba, grid, smem, s)) != PKV_OK) return st;
        return dispatch<RunPartitionMerge>(desc, a, num_seqs, static_cast<int32_t>(max_len), s);
    }
    a.partition_tokens = static_cast<int32_t>(max_len);
    a.max_partitions = 1;
    if ((st = encode_pool_map(&tk, k_cache, desc, desc->block_size)) != PKV_OK) return st;
    if ((st = encode_pool_map(&tv, v_cache, desc, desc->block_size)) != PKV_OK) return st;
    return dispatch<RunUnsplit>(desc, tk, tv, a, num_seqs, s);
}

// ------------------------------------------------------ shared-prefix decode

namespace pkv {
namespace {

size_t align256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

template <typename T, int D>
cudaError_t launch_finalize(const BalancedArgs& a, const CascadeGroups& cg, cudaStream_t stream) {
    const int64_t rows = static_cast<int64_t>(cg.grouped_seqs) * a.num_heads;
    const int64_t per = kFinalThreads / 32;
    return launch_dependent(cascade_finalize_kernel<T, D>, dim3(static_cast<unsigned>((rows + per - 1) / per)),
                            dim3(kFinalThreads), 0, stream, a, cg);
}

}  // namespace
}  // namespace pkv

extern "C" size_t paged_attention_shared_prefix_workspace_bytes(
    const pkv_cache_desc* desc, int32_t num_seqs, int32_t num_heads, int32_t max_blocks_per_seq,
    const int32_t* group_start, const int32_t* group_shared_blocks, int32_t num_groups) {
    const size_t plain = paged_attention_workspace_bytes(desc, num_seqs, num_heads, max_blocks_per_seq, 0);
    if (plain == 0) return 0;
    CascadeGroups cg;
    int64_t slots = 0;
    if (plan_groups(desc, num_seqs, num_heads, max_blocks_per_seq, group_start, group_shared_blocks,
                    num_groups, &cg, &slots) != PKV_OK)
        return 0;
    return align256(plain) + static_cast<size_t>(slots) * (desc->head_dim + 2) * sizeof(float);
}

extern "C" pkv_status paged_attention_decode_shared_prefix(
    const pkv_cache_desc* desc, void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_heads, float scale, const int32_t* group_start,
    const int32_t* group_shared_blocks, int32_t num_groups, void* workspace, size_t workspace_bytes,
    int32_t* err_flag, void* stream) {
    pkv_status st = check_decode_args(desc, out, q, k_cache, v_cache, block_tables,
                                      max_blocks_per_seq, context_lens, num_seqs, num_heads, scale);
    if (st != PKV_OK || num_seqs == 0) return st;
    CascadeGroups cg;
    int64_t slots = 0;
    if ((st = plan_groups(desc, num_seqs, num_heads, max_blocks_per_seq, group_start,
                          group_shared_blocks, num_groups, &cg, &slots)) != PKV_OK)
        return st;
    const int32_t group = num_heads / desc->num_kv_heads;
    int grid = 0, smem = 0;
    if ((st = dispatch<GridOf>(desc, static_cast<int>(group), &grid, &smem)) != PKV_OK) return st;
    const size_t plain = balanced_workspace(grid, group, desc->head_dim);
    const size_t need = align256(plain) + static_cast<size_t>(slots) * (desc->head_dim + 2) * sizeof(float);
    if (!workspace || workspace_bytes < need)
        return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "paged_attention_decode_shared_prefix: workspace too small");
    if (!aligned(workspace, 256))
        return fail(PKV_ERR_INVALID_ARG,
                    "paged_attention_decode_shared_prefix: workspace must be 256-byte aligned");
    if (cg.item_base[cg.num_groups] == 0)  // no group shares a block: the plain decode
        return paged_attention_decode(desc, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                      context_lens, num_seqs, num_heads, scale, 0, workspace,
                                      workspace_bytes, err_flag, stream);
    // workspace: balanced partials | prefix partials (o, then m, l) | own-token
    // partials of the grouped rows (o, then m, l)
    const int64_t own_rows = static_cast<int64_t>(cg.grouped_seqs) * num_heads;
    const int64_t pre_slots = slots - own_rows;
    cg.pre_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(plain));
    cg.pre_ml = cg.pre_o + pre_slots * desc->head_dim;
    cg.own_o = cg.pre_ml + pre_slots * 2;
    cg.own_ml = cg.own_o + own_rows * desc->head_dim;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    CUtensorMap tk, tv;
    if ((st = encode_pool_map(&tk, k_cache, desc, 16)) != PKV_OK) return st;
    if ((st = encode_pool_map(&tv, v_cache, desc, 16)) != PKV_OK) return st;
    BalancedArgs a = {};
    a.out = out;
    a.q = q;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.ws_o = static_cast<float*>(workspace);
    a.ws_ml = a.ws_o + static_cast<int64_t>(grid) * 2 * group * desc->head_dim;
    a.ws_meta = reinterpret_cast<int32_t*>(a.ws_ml + static_cast<int64_t>(grid) * 2 * group * 2);
    a.err_flag = err_flag;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = desc->num_kv_heads;
    a.group = group;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.num_blocks = desc->num_blocks;
    a.max_len = max_blocks_per_seq * desc->block_size;
    a.scale_log2 = scale * kLog2e;
    // 1-2: every sequence's own tokens (balanced decode + chain merge); 3: the
    // shared blocks (prefix kernel, runs as SMs free up); 4: the merge of the two
    if ((st = dispatch<RunCascade>(desc, tk, tv, a, cg, grid, smem, s)) != PKV_OK) return st;
    if ((st = launch_prefix(desc, q, k_cache, v_cache, block_tables, max_blocks_per_seq, num_seqs,
                            num_heads, scale, cg, err_flag, s)) != PKV_OK)
        return st;
    cudaError_t e = desc->head_dim == 128
                        ? (desc->dtype == PKV_BF16 ? launch_finalize<__nv_bfloat16, 128>(a, cg, s)
                                                   : launch_finalize<__half, 128>(a, cg, s))
                        : (desc->dtype == PKV_BF16 ? launch_finalize<__nv_bfloat16, 64>(a, cg, s)
                                                   : launch_finalize<__half, 64>(a, cg, s));
    note_launches(1);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    return PKV_OK;
}

// ------------------------------------------------ decode without allocation
//
// Some callers cannot hand this library a workspace: a plugin running inside a
// serving engine whose allocator has already reserved nearly all device memory
// for its own pools, or a real-time decode loop that may not call cudaMalloc
// (it synchronises the device and can fail under fragmentation).  For them,
// paged_attention_decode_static_scratch keeps the split path's partial results
// in a fixed array compiled into this file instead.
namespace pkv {
namespace {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(PKV_STATIC_SCRATCH_BYTES);

// Every GPU that loads this library holds this array until the process exits.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;

// The array's address is a property of the CUDA context that loaded this
// module: a new context on the same device (after cudaDeviceReset, or a primary
// context released and retained again) may load it elsewhere.  So the address
// looked up for a device is kept together with the id of the context it was
// looked up in (cuCtxGetId: unique for the life of the process), and looked up
// again when the current context is another one.
struct ScratchAddress {
    unsigned long long ctx_id;
    void* addr;
};
std::mutex g_scratch_mu;
ScratchAddress g_scratch_addr[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Id of the current context, or 0 when there is none yet.
pkv_status current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return fail(PKV_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId unavailable");
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuCtxGetCurrent failed");
    *id = 0;
    if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuCtxGetId failed");
    return PKV_OK;
}

// Device address of g_static_scratch in the current context, looked up once
// per (device, context) with that device current.  In host code the array's
// name is only a stand-in, never a device address, so it must not be passed to
// a kernel directly.
pkv_status static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device index >= 64");
    unsigned long long ctx = 0;
    pkv_status st = current_context_id(&ctx);
    if (st != PKV_OK) return st;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (ctx != 0 && g_scratch_addr[dev].ctx_id == ctx && g_scratch_addr[dev].addr) {
        *out = g_scratch_addr[dev].addr;
        return PKV_OK;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // creates the primary context if needed
    if (e != cudaSuccess || !p)
        return fail(PKV_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
    if ((st = current_context_id(&ctx)) != PKV_OK) return st;
    g_scratch_addr[dev] = ScratchAddress{ctx, p};
    *out = p;
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status paged_attention_decode_static_scratch(
    const pkv_cache_desc* desc, void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
    int32_t num_seqs, int32_t num_heads, float scale, int32_t partition_size, int32_t* err_flag,
    void* stream) {
    pkv_status st = check_desc(desc);
    if (st != PKV_OK) return st;
    if (num_seqs < 0 || num_heads <= 0 || max_blocks_per_seq <= 0 || partition_size < 0)
        return fail(PKV_ERR_INVALID_ARG,
                    "paged_attention_decode_static_scratch: bad num_seqs, num_heads, "
                    "max_blocks_per_seq or partition_size");
    const size_t need = paged_attention_workspace_bytes(desc, num_seqs, num_heads,
                                                        max_blocks_per_seq, partition_size);
    if (need > kStaticScratchBytes)
        return fail(PKV_ERR_WORKSPACE_TOO_SMALL,
                    "paged_attention_decode_static_scratch: these shapes need more scratch than "
                    "the 16 MiB static array holds (use paged_attention_decode with a workspace)");
    void* scratch = nullptr;
    if (need > 0 && (st = static_scratch_address(&scratch)) != PKV_OK) return st;
    // No part of the scratch has to start at zero: every partial result the
    // merge reads is written earlier in the same call.
    return paged_attention_decode(desc, out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  context_lens, num_seqs, num_heads, scale, partition_size,
                                  need > 0 ? scratch : nullptr, need > 0 ? kStaticScratchBytes : 0,
                                  err_flag, stream);
}
