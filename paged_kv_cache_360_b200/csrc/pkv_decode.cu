// pkv_decode.cu -- paged decode attention for sm_100a.
//
// "PagedAttention" ops page, How it works -- The mechanics: the attention kernel
// reads keys and values through the block table, gathering scattered physical
// blocks, which makes non-contiguous storage transparent to the math.  Concept --
// What it is: a per-sequence block table maps logical positions to physical
// blocks.
//
// Work item = (sequence b, kv head hk, partition p) = one CTA.  A partition is
// `partition_tokens` consecutive logical tokens (a multiple of the block size),
// or the whole sequence when the call does not split.
//
// CTA = 4 consumer warps + 1 producer warp.
//   * Producer: reads the partition's block-table entries (one coalesced load per
//     32 blocks), and for each logical block issues TMA 2-D tiled loads of the
//     (block, kv head) K and V tiles -- bs rows x 128 B per 64-column half, 128B
//     swizzle -- into a ring of shared-memory stages, completion counted on an
//     mbarrier per stage.  The tensor map spans the whole pool viewed as
//     [num_blocks * num_kv_heads * bs rows][head_dim], so the gather is just the
//     row coordinate (block * num_kv_heads + hk) * bs.
//   * Consumers: warp w takes the partition's logical blocks w, w+4, w+8, ...
//     All g = num_heads / num_kv_heads query heads of the kv head share each K/V
//     tile: S = Q K^T and O += P V run on mma.sync m16n8k16 with the g query
//     heads as the 16-row M side (rows >= g are zero), fp32 accumulators, and an
//     online softmax in base 2 (scale * log2 e folded into the scores).
//   * The four warps' (m, l, O) are merged in shared memory in warp order; the
//     result is either the normalised output or, when split, the partition's
//     un-normalised O with its max m and sum l.
// The reduce kernel merges partitions p = 0, 1, ... in ascending order.  Every
// reduction order depends only on logical token order, never on physical block
// ids or timing, so results are bit-identical under block permutation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pkv.h"
#include "pkv_internal.h"
#include "pkv_ptx.cuh"

namespace pkv {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;

template <int D, int BS>
struct Geom {
    static constexpr int kHalves = D / 64;                // 128-byte column halves per row
    static constexpr int kHalfBytes = BS * 128;           // one half of one (block, head) tile
    static constexpr int kTileBytes = kHalves * kHalfBytes;  // K (or V) of one (block, head)
    static constexpr int kStageBytes = 2 * kTileBytes;    // K + V
    // Stage s is always consumed by warp s % kConsumerWarps, so a warp waits on
    // the rounds of its stages in order and is never a phase ahead of the
    // barrier it polls (a parity wait cannot tell phase r-1 from phase r+1).
    static constexpr int kStages = kStageBytes <= 8192 ? 8 : 4;
    static_assert(kStages % kConsumerWarps == 0, "each stage must belong to one consumer warp");
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kMergeBytes = kConsumerWarps * 16 * (D + 2) * 4;
    static constexpr int kBodyBytes = kRingBytes > kMergeBytes ? kRingBytes : kMergeBytes;
    static constexpr int kBarOffset = kBodyBytes;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8 + 1024;  // + 1 KB alignment slack
    static_assert(kHalfBytes % 1024 == 0, "128B-swizzled tiles must start on 1 KB boundaries");
};

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

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ void flag(int32_t* err, int32_t bit) {
    if (err) atomicOr(err, bit);
}

// Keep the 16-bit halves of `v` whose token index (t for the low half, t + 1
// for the high half) is below `end`; zero the others.
__device__ __forceinline__ uint32_t keep_valid(uint32_t v, int t, int end) {
    if (t >= end) return 0u;
    if (t + 1 >= end) return v & 0xffffu;
    return v;
}

__device__ __forceinline__ int clamp_len(int L, int max_len) {
    return L < 0 ? 0 : (L > max_len ? max_len : L);
}

template <typename T, int D, int BS, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 2)
decode_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const DecodeArgs a) {
    using G = Geom<D, BS>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t base = smem_addr(smem);
    const uint32_t bar_full = base + G::kBarOffset;          // kStages x 8 B
    const uint32_t bar_empty = bar_full + 8 * G::kStages;    // kStages x 8 B

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int b = blockIdx.x / a.num_kv_heads;
    const int hk = blockIdx.x - b * a.num_kv_heads;
    const int part = blockIdx.y;

    if (SPLIT) pdl_launch_dependents();

    const int max_len = a.max_blocks_per_seq * BS;
    const int raw_len = __ldg(a.context_lens + b);
    const int L = clamp_len(raw_len, max_len);
    if (raw_len != L && threadIdx.x == 0 && part == 0 && hk == 0)
        flag(a.err_flag, PKV_DEVERR_BAD_CONTEXT_LEN);
    const int t_begin = part * a.partition_tokens;
    if (SPLIT && t_begin >= L) return;  // this partition holds no tokens
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
                        const uint32_t full = bar_full + 8 * s;
                        mbar_arrive_expect_tx(full, G::kStageBytes);
                        const int y = (pj * a.num_kv_heads + hk) * BS;
                        const uint32_t kdst = base + s * G::kStageBytes;
                        const uint32_t vdst = kdst + G::kTileBytes;
#pragma unroll
                        for (int h = 0; h < G::kHalves; ++h) {
                            tma_load_2d(kdst + h * G::kHalfBytes, &tm_k, 64 * h, y, full, policy);
                            tma_load_2d(vdst + h * G::kHalfBytes, &tm_v, 64 * h, y, full, policy);
                        }
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2;   // fragment row (query head within the group)
    const int t4 = lane & 3;   // fragment column pair
    const int group = a.group;
    const T* qbase = static_cast<const T*>(a.q) +
                     (static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group) * D;

    // Q as the A operand of S = Q K^T, one 16x16 fragment per 16 columns of D.
    uint32_t qa[D / 16][4];
    {
        const bool lo_ok = g < group, hi_ok = g + 8 < group;
        const uint32_t* qlo = reinterpret_cast<const uint32_t*>(qbase + g * D);
        const uint32_t* qhi = reinterpret_cast<const uint32_t*>(qbase + (g + 8) * D);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            qa[kk][0] = lo_ok ? __ldg(qlo + 8 * kk + t4) : 0u;
            qa[kk][1] = hi_ok ? __ldg(qhi + 8 * kk + t4) : 0u;
            qa[kk][2] = lo_ok ? __ldg(qlo + 8 * kk + 4 + t4) : 0u;
            qa[kk][3] = hi_ok ? __ldg(qhi + 8 * kk + 4 + t4) : 0u;
        }
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
    const float sl2 = a.scale_log2;

    for (int it = warp; it < nblk; it += kConsumerWarps) {
        const int s = it % G::kStages;
        const int round = it / G::kStages;
        const bool arrived = __all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, round & 1));
        if (!arrived) {
            if (lane == 0) flag(a.err_flag, PKV_DEVERR_WAIT_TIMEOUT);
            break;
        }
        const uint32_t kst = base + s * G::kStageBytes;
        const uint32_t vst = kst + G::kTileBytes;
        const int tok_blk = (blk_begin + it) * BS;
#pragma unroll
        for (int sub = 0; sub < BS / 16; ++sub) {
            const int tok0 = tok_blk + sub * 16;
            if (tok0 >= t_end) break;

            // S (16 query rows x 16 tokens) = Q K^T
            float sc[2][4];
#pragma unroll
            for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
            {
                const int mi = lane >> 3;
                const int r = sub * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int chunk = 2 * kk + (mi & 1);
                    const uint32_t addr = kst + (chunk >> 3) * G::kHalfBytes + r * 128 +
                                          (((chunk & 7) ^ (r & 7)) << 4);
                    uint32_t kb[4];
                    ldsm_x4(addr, kb);
                    Mma<T>::run(sc[0], qa[kk], kb[0], kb[1]);
                    Mma<T>::run(sc[1], qa[kk], kb[2], kb[3]);
                }
            }

            // scale into base 2, mask tokens past the partition, row maxima
            float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const bool valid = tok0 + nt * 8 + 2 * t4 + j < t_end;
                    sc[nt][j] = valid ? sc[nt][j] * sl2 : -INFINITY;
                    sc[nt][2 + j] = valid ? sc[nt][2 + j] * sl2 : -INFINITY;
                    mx_lo = fmaxf(mx_lo, sc[nt][j]);
                    mx_hi = fmaxf(mx_hi, sc[nt][2 + j]);
                }
            }
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
            mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
            mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
            const float mn_lo = fmaxf(m_lo, mx_lo);
            const float mn_hi = fmaxf(m_hi, mx_hi);
            if (__any_sync(0xffffffffu, mn_lo != m_lo || mn_hi != m_hi)) {
                const float al = exp2_approx(m_lo - mn_lo);
                const float ah = exp2_approx(m_hi - mn_hi);
                l_lo *= al;
                l_hi *= ah;
#pragma unroll
                for (int i = 0; i < D / 8; ++i) {
                    o[i][0] *= al;
                    o[i][1] *= al;
                    o[i][2] *= ah;
                    o[i][3] *= ah;
                }
            }
            m_lo = mn_lo;
            m_hi = mn_hi;

            // P = 2^(S - m), rounded to T: the A operand of O += P V.  The row
            // sums use the rounded values, so the weights that multiply V are
            // exactly the ones that normalise.
            uint32_t pa[4];
            {
                float r0, r1;
                pa[0] = Pack<T>::two(exp2_approx(sc[0][0] - mn_lo), exp2_approx(sc[0][1] - mn_lo), r0, r1);
                l_lo += r0 + r1;
                pa[1] = Pack<T>::two(exp2_approx(sc[0][2] - mn_hi), exp2_approx(sc[0][3] - mn_hi), r0, r1);
                l_hi += r0 + r1;
                pa[2] = Pack<T>::two(exp2_approx(sc[1][0] - mn_lo), exp2_approx(sc[1][1] - mn_lo), r0, r1);
                l_lo += r0 + r1;
                pa[3] = Pack<T>::two(exp2_approx(sc[1][2] - mn_hi), exp2_approx(sc[1][3] - mn_hi), r0, r1);
                l_hi += r0 + r1;
            }

            // O (16 rows x D) += P (16 x 16 tokens) V (16 tokens x D)
            {
                const bool partial = tok0 + 16 > t_end;
                const int mi = lane >> 3;
                const int r = sub * 16 + (mi & 1) * 8 + (lane & 7);
                const int ta = tok0 + 2 * t4, tb = tok0 + 8 + 2 * t4;
#pragma unroll
                for (int nd = 0; nd < D / 16; ++nd) {
                    const int chunk = 2 * nd + (mi >> 1);
                    const uint32_t addr = vst + (chunk >> 3) * G::kHalfBytes + r * 128 +
                                          (((chunk & 7) ^ (r & 7)) << 4);
                    uint32_t vb[4];
                    ldsm_x4_trans(addr, vb);
                    if (partial) {
                        // rows past the end may hold anything (even NaN): zero them
                        vb[0] = keep_valid(vb[0], ta, t_end);
                        vb[2] = keep_valid(vb[2], ta, t_end);
                        vb[1] = keep_valid(vb[1], tb, t_end);
                        vb[3] = keep_valid(vb[3], tb, t_end);
                    }
                    Mma<T>::run(o[2 * nd], pa, vb[0], vb[1]);
                    Mma<T>::run(o[2 * nd + 1], pa, vb[2], vb[3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    }

    // ----------------------------------------------- merge the four warps
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);

    consumer_sync();  // every consumer is done with the ring: reuse it
    float* mo = reinterpret_cast<float*>(smem);              // [warp][16][D]
    float* mm = mo + kConsumerWarps * 16 * D;                // [warp][16]
    float* ml = mm + kConsumerWarps * 16;                    // [warp][16]
    if (t4 == 0) {
        mm[warp * 16 + g] = m_lo;
        mm[warp * 16 + g + 8] = m_hi;
        ml[warp * 16 + g] = l_lo;
        ml[warp * 16 + g + 8] = l_hi;
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        const int col = i * 8 + 2 * t4;
        *reinterpret_cast<float2*>(mo + (warp * 16 + g) * D + col) = make_float2(o[i][0], o[i][1]);
        *reinterpret_cast<float2*>(mo + (warp * 16 + g + 8) * D + col) = make_float2(o[i][2], o[i][3]);
    }
    consumer_sync();

    const int tid = threadIdx.x;  // 0 .. 127 (consumers only)
    for (int idx = tid; idx < group * D; idx += kConsumerWarps * 32) {
        const int r = idx / D;
        const int d = idx - r * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, mm[w * 16 + r]);
        float acc = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = mm[w * 16 + r];
            const float f = mw == -INFINITY ? 0.f : exp2_approx(mw - M);
            acc += f * mo[(w * 16 + r) * D + d];
            den += f * ml[w * 16 + r];
        }
        const int64_t bh = static_cast<int64_t>(b) * a.num_heads + static_cast<int64_t>(hk) * group + r;
        if (SPLIT) {
            const int64_t slot = bh * a.max_partitions + part;
            a.ws_o[slot * D + d] = acc;
            if (d == 0) {
                a.ws_m[slot] = M;
                a.ws_l[slot] = den;
            }
        } else {
            static_cast<T*>(a.out)[bh * D + d] = Pack<T>::one(den > 0.f ? acc / den : 0.f);
        }
    }
}

// Merge the partitions of one (sequence, query head) by log-sum-exp, p ascending:
//   M = max_p m_p,  out = sum_p 2^(m_p - M) o_p / sum_p 2^(m_p - M) l_p.
template <typename T, int D>
__global__ void __launch_bounds__(D) reduce_kernel(const DecodeArgs a, int32_t max_len) {
    pdl_wait_primary();  // the partition kernel's results are visible after this
    const int64_t bh = blockIdx.x;
    const int b = static_cast<int>(bh / a.num_heads);
    const int d = threadIdx.x;
    const int L = clamp_len(__ldg(a.context_lens + b), max_len);
    const int n = (L + a.partition_tokens - 1) / a.partition_tokens;
    const float* m = a.ws_m + bh * a.max_partitions;
    const float* l = a.ws_l + bh * a.max_partitions;
    const float* o = a.ws_o + bh * a.max_partitions * D;
    float M = -INFINITY;
    for (int p = 0; p < n; ++p) M = fmaxf(M, m[p]);
    float acc = 0.f, den = 0.f;
    for (int p = 0; p < n; ++p) {
        const float f = exp2_approx(m[p] - M);
        acc += f * o[static_cast<int64_t>(p) * D + d];
        den += f * l[p];
    }
    static_cast<T*>(a.out)[bh * D + d] = Pack<T>::one(den > 0.f ? acc / den : 0.f);
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// A 2-D view of one pool: rows = num_blocks * num_kv_heads * block_size,
// columns = head_dim; box = 64 columns (128 B) x block_size rows, 128B swizzle.
pkv_status encode_pool_map(CUtensorMap* tm, const void* pool, const pkv_cache_desc* d) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t rows = static_cast<cuuint64_t>(d->num_blocks) * d->num_kv_heads * d->block_size;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d->head_dim), rows};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d->head_dim) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(d->block_size)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(tm,
                        d->dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void*>(pool), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    return PKV_OK;
}

int sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
    return n;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

pkv_status check_desc(const pkv_cache_desc* d) {
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

// Library choice of partition size; 0 = no split.
int32_t choose_partition(const pkv_cache_desc* d, int32_t num_seqs, int32_t max_blocks_per_seq) {
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * d->block_size;
    int32_t P = 512;
    if (max_len <= P) return 0;
    const int64_t target = 4LL * sm_count();  // two resident CTAs per SM, two waves
    const int64_t pairs = static_cast<int64_t>(num_seqs) * d->num_kv_heads;
    while (P > 128 && pairs * ((max_len + P - 1) / P) < target) P /= 2;
    if (P % d->block_size != 0) P = (P / d->block_size) * d->block_size;
    return P;
}

int32_t resolve_partition(const pkv_cache_desc* d, int32_t num_seqs, int32_t max_blocks_per_seq,
                          int32_t requested) {
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * d->block_size;
    const int32_t P = requested == 0 ? choose_partition(d, num_seqs, max_blocks_per_seq) : requested;
    return (P == 0 || P >= max_len) ? 0 : P;
}

size_t workspace_for(const pkv_cache_desc* d, int32_t num_seqs, int32_t num_heads,
                     int32_t max_blocks_per_seq, int32_t P) {
    if (P == 0) return 0;
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * d->block_size;
    const int64_t pmax = (max_len + P - 1) / P;
    return static_cast<size_t>(num_seqs) * num_heads * pmax * (d->head_dim + 2) * sizeof(float);
}

// Opt the kernel in to its dynamic shared memory once per device (the static
// is per template instantiation, i.e. per kernel).
template <typename T, int D, int BS, bool SPLIT>
cudaError_t allow_smem() {
    static std::atomic<uint64_t> done{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const uint64_t bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<T, D, BS, SPLIT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Geom<D, BS>::kSmemBytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_release);
    return e;
}

template <typename T, int D, int BS>
pkv_status launch(const CUtensorMap& tk, const CUtensorMap& tv, const DecodeArgs& a,
                  int32_t num_seqs, bool split, cudaStream_t stream) {
    using G = Geom<D, BS>;
    const dim3 grid(static_cast<unsigned>(num_seqs) * a.num_kv_heads,
                    split ? static_cast<unsigned>(a.max_partitions) : 1u);
    cudaError_t e;
    if (split) {
        if ((e = allow_smem<T, D, BS, true>()) != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
        decode_kernel<T, D, BS, true><<<grid, kThreads, G::kSmemBytes, stream>>>(tk, tv, a);
        note_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
        // The merge launches as a programmatic dependent of the partition
        // kernel: its CTAs may start during the partition kernel's tail and wait
        // in griddepcontrol.wait for the results.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(num_seqs) * a.num_heads);
        cfg.blockDim = dim3(D);
        cfg.dynamicSmemBytes = 0;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const int32_t max_len = a.max_blocks_per_seq * BS;
        e = cudaLaunchKernelEx(&cfg, reduce_kernel<T, D>, a, max_len);
        note_launches(1);
        if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    } else {
        if ((e = allow_smem<T, D, BS, false>()) != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
        decode_kernel<T, D, BS, false><<<grid, kThreads, G::kSmemBytes, stream>>>(tk, tv, a);
        note_launches(1);
        if ((e = cudaGetLastError()) != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    }
    return PKV_OK;
}

template <typename T>
pkv_status dispatch_shape(const pkv_cache_desc* d, const CUtensorMap& tk, const CUtensorMap& tv,
                          const DecodeArgs& a, int32_t num_seqs, bool split, cudaStream_t st) {
    if (d->head_dim == 128 && d->block_size == 16) return launch<T, 128, 16>(tk, tv, a, num_seqs, split, st);
    if (d->head_dim == 128 && d->block_size == 32) return launch<T, 128, 32>(tk, tv, a, num_seqs, split, st);
    if (d->head_dim == 64 && d->block_size == 16) return launch<T, 64, 16>(tk, tv, a, num_seqs, split, st);
    return launch<T, 64, 32>(tk, tv, a, num_seqs, split, st);
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" int32_t paged_attention_partition_size(const pkv_cache_desc* desc, int32_t num_seqs,
                                                  int32_t num_heads, int32_t max_blocks_per_seq) {
    (void)num_heads;
    if (check_desc(desc) != PKV_OK || num_seqs <= 0 || max_blocks_per_seq <= 0) return 0;
    return resolve_partition(desc, num_seqs, max_blocks_per_seq, 0);
}

extern "C" size_t paged_attention_workspace_bytes(const pkv_cache_desc* desc, int32_t num_seqs,
                                                  int32_t num_heads, int32_t max_blocks_per_seq,
                                                  int32_t partition_size) {
    if (check_desc(desc) != PKV_OK || num_seqs <= 0 || num_heads <= 0 || max_blocks_per_seq <= 0 ||
        partition_size < 0)
        return 0;
    const int32_t P = resolve_partition(desc, num_seqs, max_blocks_per_seq, partition_size);
    return workspace_for(desc, num_seqs, num_heads, max_blocks_per_seq, P);
}

extern "C" pkv_status paged_attention_decode(const pkv_cache_desc* desc, void* out, const void* q,
                                             const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables,
                                             int32_t max_blocks_per_seq,
                                             const int32_t* context_lens, int32_t num_seqs,
                                             int32_t num_heads, float scale,
                                             int32_t partition_size, void* workspace,
                                             size_t workspace_bytes, int32_t* err_flag,
                                             void* stream) {
    pkv_status st = check_desc(desc);
    if (st != PKV_OK) return st;
    if (num_seqs < 0 || num_heads <= 0 || max_blocks_per_seq <= 0)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: bad num_seqs, num_heads or max_blocks_per_seq");
    if (num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: q, out and pools must be 16-byte aligned");
    if (num_heads % desc->num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_heads must be a multiple of num_kv_heads");
    const int32_t group = num_heads / desc->num_kv_heads;
    if (group > 16) return fail(PKV_ERR_UNSUPPORTED, "num_heads / num_kv_heads must be <= 16");
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
        return fail(PKV_ERR_INVALID_ARG, "scale must be finite");
    if (static_cast<int64_t>(max_blocks_per_seq) * desc->block_size > INT32_MAX / 2)
        return fail(PKV_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size too large");
    if (static_cast<int64_t>(num_seqs) * desc->num_kv_heads > INT32_MAX)
        return fail(PKV_ERR_UNSUPPORTED, "num_seqs * num_kv_heads too large");
    if (partition_size < 0 || (partition_size > 0 && partition_size % desc->block_size != 0))
        return fail(PKV_ERR_INVALID_ARG, "partition_size must be 0 or a positive multiple of block_size");

    const int32_t P = resolve_partition(desc, num_seqs, max_blocks_per_seq, partition_size);
    const bool split = P != 0;
    const int64_t max_len = static_cast<int64_t>(max_blocks_per_seq) * desc->block_size;
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
        const int64_t pmax = (max_len + P - 1) / P;
        if (pmax > 65535) return fail(PKV_ERR_UNSUPPORTED, "too many partitions (> 65535)");
        const size_t need = workspace_for(desc, num_seqs, num_heads, max_blocks_per_seq, P);
        if (!workspace || workspace_bytes < need)
            return fail(PKV_ERR_WORKSPACE_TOO_SMALL, "paged_attention_decode: workspace too small");
        if (!aligned(workspace, 16))
            return fail(PKV_ERR_INVALID_ARG, "paged_attention_decode: workspace must be 16-byte aligned");
        const int64_t rows = static_cast<int64_t>(num_seqs) * num_heads * pmax;
        a.ws_o = static_cast<float*>(workspace);
        a.ws_m = a.ws_o + rows * desc->head_dim;
        a.ws_l = a.ws_m + rows;
        a.partition_tokens = P;
        a.max_partitions = static_cast<int32_t>(pmax);
    } else {
        a.partition_tokens = static_cast<int32_t>(max_len);
        a.max_partitions = 1;
    }

    CUtensorMap tk, tv;
    if ((st = encode_pool_map(&tk, k_cache, desc)) != PKV_OK) return st;
    if ((st = encode_pool_map(&tv, v_cache, desc)) != PKV_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (desc->dtype == PKV_BF16) return dispatch_shape<__nv_bfloat16>(desc, tk, tv, a, num_seqs, split, s);
    return dispatch_shape<__half>(desc, tk, tv, a, num_seqs, split, s);
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
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of g_static_scratch on the current device, looked up once
// per device.  In host code the array's name is only a stand-in, never a
// device address, so it must not be passed to a kernel directly.
pkv_status static_scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(PKV_ERR_UNSUPPORTED, "device index >= 64");
    void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess || !p)
            return fail(PKV_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
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
