// pkv_prefill.cu -- paged prefill attention on the tcgen05 tensor cores.
//
// The prompt phase of PagedAttention ("PagedAttention" operations page, How it
// works: attention reads keys and values through the block table; Concept:
// prompt processing is the compute-bound phase): the last n_b tokens of every
// sequence attend causally to the sequence's paged context.
//
// One CTA computes one tile of 128 query rows against all the kv tiles it can
// see.  The rows are (token, head) pairs of one kv head: 128 / g consecutive
// query tokens times the g query heads that share the kv head, so every key and
// value row fetched serves g heads.  Per CTA:
//   warp 0      producer: the Q tile once (one 4-D TMA box), then per 128-token
//               kv tile one 3-D TMA box per (block, 64-column half) of K and V
//               into a two-stage ring;
//   warp 1      MMA issuer (one thread) and tensor-memory owner:
//               S_j = Q K_j^T into one of two 128-column TMEM buffers, then
//               O += P_j V_j into a D-column TMEM accumulator;
//   warps 2-5   softmax, one S row per thread (TMEM lane = row): mask, running
//               maximum (rescaling O in TMEM only when the maximum grows by more
//               than 2^8), P_j = 2^(s - m) rounded into a 128x128 shared tile
//               for the next MMA, and at the end O / l to global memory.
// S_{j+1} is computed while the softmax of tile j runs.  In tile 0 the softmax
// also sends the rounding residual of P as a second P V product, so that rows
// with few tokens (the start of every prompt) are accurate to fp32 weights.
//
// Every mbarrier wait is bounded and warp-uniform; a timeout raises a shared
// abort word, records PKV_DEVERR_WAIT_TIMEOUT and every role drains its
// asynchronous work (copies, MMAs) before the CTA frees its tensor memory.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "pkv.h"
#include "pkv_host.cuh"
#include "pkv_internal.h"
#include "pkv_ptx.cuh"
#include "pkv_tc.cuh"

namespace pkv {
namespace {

constexpr int kPfThreads = 192;      // producer warp, MMA warp, 4 softmax warps
constexpr int kPfRows = 128;         // MMA M: query rows per CTA
constexpr int kPfKv = 128;           // kv tokens per tile: N of Q K^T, K of P V
constexpr int kPfStages = 2;         // K/V ring depth
constexpr uint32_t kTmemCols = 512;  // S buffers at columns 0 and 128, O at 256
constexpr uint32_t kTmemO = 256;
constexpr float kRescaleLog2 = 8.f;  // rescale O when the maximum grows by > 2^8

enum : int {
    kBarQ = 0,
    kBarKvFull = 1,
    kBarKvEmpty = kBarKvFull + kPfStages,
    kBarSFull = kBarKvEmpty + kPfStages,  // two
    kBarPFull = kBarSFull + 2,
    kBarODone,
    kBarDrain,
    kNumBars
};

// Shared memory, from a 1 KiB aligned base.  Every operand tile is [half][128
// rows][128 B], 128B-swizzled (the TMA's pattern), halves 16 KiB apart.
template <int D>
struct PfLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = 128 * 128;
    static constexpr int kTile = kHalves * kHalfBytes;          // 128 rows x D
    static constexpr int kQ = 0;
    static constexpr int kStage0 = kTile;                       // stage s: K, then V
    static constexpr int kP = kStage0 + 2 * kPfStages * kTile;  // 128 x 128 probabilities
    static constexpr int kBars = kP + 2 * kHalfBytes;
    static constexpr int kMisc = kBars + 8 * kNumBars;  // tmem base, abort word, work item
    static constexpr int kBytes = kMisc + 32;
    static constexpr int kAlloc = kBytes + 1024;        // room to align the base
};

struct PrefillArgs {
    void* out;
    const int32_t* tables;
    const int32_t* lens;
    const int32_t* qstart;
    int32_t* err;
    int32_t num_seqs;
    int32_t num_tokens;
    int32_t num_heads;
    int32_t num_kv_heads;
    int32_t log2_group;
    int32_t max_blocks;
    int32_t num_blocks;
    float sl2;  // scale * log2(e)
};

__device__ __forceinline__ void flag(int32_t* err, int bit) {
    if (err) atomicOr(err, bit);
}

// Bounded wait that also gives up when another role raised the abort word.
// Warp-uniform: every lane of the calling warp must call it.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity,
                                          volatile uint32_t* abort_word, int32_t* err) {
    bool ok = false;
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_test(bar, parity)) {
            ok = true;
            break;
        }
        if (*abort_word) break;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && *abort_word == 0u) {
        *abort_word = 1u;
        if ((threadIdx.x & 31) == 0) flag(err, PKV_DEVERR_WAIT_TIMEOUT);
    }
    return ok;
}

// Single-thread variant (producer, MMA issuer).
__device__ __forceinline__ bool one_wait(uint32_t bar, uint32_t parity,
                                         volatile uint32_t* abort_word, int32_t* err) {
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_test(bar, parity)) return true;
        if (*abort_word) return false;
    }
    *abort_word = 1u;
    flag(err, PKV_DEVERR_WAIT_TIMEOUT);
    return false;
}

// Sequence lengths as the kernel uses them: out-of-range values are clamped.
__device__ __forceinline__ void seq_shape(const PrefillArgs& a, int cap, int b, int& L, int& n) {
    L = __ldg(a.lens + b);
    n = __ldg(a.qstart + b + 1) - __ldg(a.qstart + b);
    L = L < 0 ? 0 : (L > cap ? cap : L);
    n = n < 0 ? 0 : (n > L ? L : n);
}

// Warp 0: which (sequence, query tile) CTA `i` owns.  Tiles are numbered
// sequence by sequence, the last (most expensive) tile of a sequence first.
__device__ void find_tile(const PrefillArgs& a, int cap, int tok_per_tile, int i, int* work) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int b0 = 0; b0 < a.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        int nt = 0;
        if (b < a.num_seqs) {
            int L, n;
            seq_shape(a, cap, b, L, n);
            nt = (n + tok_per_tile - 1) / tok_per_tile;
        }
        int inc = nt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const int total = __shfl_sync(0xffffffffu, inc, 31);
        if (i < base + total) {
            const unsigned hit = __ballot_sync(0xffffffffu, base + inc > i);
            const int src = __ffs(hit) - 1;
            const int before = __shfl_sync(0xffffffffu, inc - nt, src);
            const int count = __shfl_sync(0xffffffffu, nt, src);
            if (lane == 0) {
                work[0] = b0 + src;
                work[1] = count - 1 - (i - base - before);
            }
            return;
        }
        base += total;
    }
    if (lane == 0) work[0] = -1;
}

// One thread's row of the 128x128 probability tile, K-major and 128B-swizzled:
// element c of row r sits in half c / 64, 16-byte chunk ((c % 64) / 8) ^ (r % 8).
__device__ __forceinline__ void store_p_row(uint32_t p_s, int r, const uint32_t (&pk)[64]) {
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint32_t addr = p_s + (c >> 3) * 16384u + r * 128u + ((((c & 7) ^ (r & 7))) << 4);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * c]),
                     "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                     : "memory");
    }
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const PrefillArgs a) {
    using Lay = PfLayout<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescS = f16_idesc(kBf16, kPfRows, kPfKv, false);
    constexpr uint32_t kIdescO = f16_idesc(kBf16, kPfRows, D, true);
    static_assert(kPfKv % BS == 0, "a kv tile holds whole blocks");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sp = smem_raw + (sb - raw);
    uint32_t* misc = reinterpret_cast<uint32_t*>(sp + Lay::kMisc);
    volatile uint32_t* abort_word = misc + 1;
    int* work = reinterpret_cast<int*>(misc + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto bar = [&](int i) { return sb + Lay::kBars + 8u * static_cast<uint32_t>(i); };

    if (threadIdx.x == 0) {
        mbar_init(bar(kBarQ), 1);
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(bar(kBarKvFull + s), 1);
            mbar_init(bar(kBarKvEmpty + s), 1);
        }
        mbar_init(bar(kBarSFull), 1);
        mbar_init(bar(kBarSFull + 1), 1);
        mbar_init(bar(kBarPFull), 128);
        mbar_init(bar(kBarODone), 1);
        mbar_init(bar(kBarDrain), 1);
        misc[1] = 0u;
        fence_mbar_init();
        prefetch_tensormap(&tq);
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
    }
    if (warp == 1) {
        tmem_alloc(sb + Lay::kMisc, kTmemCols);
        tmem_relinquish();
    }
    pdl_wait_primary();
    const int cap = a.max_blocks * BS;
    const int tok_per_tile = kPfRows >> a.log2_group;
    if (warp == 0) find_tile(a, cap, tok_per_tile, blockIdx.x, work);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int b = work[0];

    if (b >= 0) {
        const int qt = work[1];
        const int hk = blockIdx.y;
        const int g = 1 << a.log2_group;
        int L, n;
        seq_shape(a, cap, b, L, n);
        if (threadIdx.x == 0) {
            const int L_raw = __ldg(a.lens + b);
            const int n_raw = __ldg(a.qstart + b + 1) - __ldg(a.qstart + b);
            if (L_raw != L) flag(a.err, PKV_DEVERR_BAD_CONTEXT_LEN);
            if (n_raw != n) flag(a.err, PKV_DEVERR_BAD_QUERY_COUNT);
        }
        const int q0 = __ldg(a.qstart + b);
        const int t_lo = qt * tok_per_tile;
        const int t_hi = min(n, t_lo + tok_per_tile);
        const int p_hi = L - n + t_hi - 1;  // last query position of the tile
        const int nkv = p_hi / kPfKv + 1;

        if (warp == 0) {
            // ------------------------------------------------------ producer
            // Table entries come 32 at a time (one per lane, one coalesced
            // load), the next 32 prefetched while the current ones are used;
            // lane l issues the copies of block l of each kv tile.
            constexpr int kBlocksPerTile = kPfKv / BS;
            constexpr int kTilesPerChunk = 32 / kBlocksPerTile;
            const int32_t* row = a.tables + static_cast<int64_t>(b) * a.max_blocks;
            auto load_chunk = [&](int c) {
                const int idx = c * 32 + lane;
                int id = 0;  // blocks past the context: any valid block, masked
                if (idx * BS < L) {
                    id = __ldg(row + idx);
                    if (id < 0 || id >= a.num_blocks) {
                        flag(a.err, PKV_DEVERR_BAD_BLOCK_ID);
                        id = 0;
                    }
                }
                return id;
            };
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(kBarQ), Lay::kTile);
                tma_load_4d(sb + Lay::kQ, &tq, 0, hk * g, q0 + t_lo, 0, bar(kBarQ));
            }
            int cur = load_chunk(0), next = 0;
            int issued = 0;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % kPfStages;
                if (j % kTilesPerChunk == 0) {
                    if (j > 0) cur = next;
                    next = load_chunk(j / kTilesPerChunk + 1);
                }
                if (j >= kPfStages &&
                    !warp_wait(bar(kBarKvEmpty + s), ((j / kPfStages) - 1) & 1, abort_word, a.err))
                    break;
                const uint32_t ks = sb + Lay::kStage0 + 2u * s * Lay::kTile;
                const uint32_t vs = ks + Lay::kTile;
                if (lane == 0) mbar_arrive_expect_tx(bar(kBarKvFull + s), 2u * Lay::kTile);
                __syncwarp();
                const int id = __shfl_sync(0xffffffffu, cur,
                                           (j % kTilesPerChunk) * kBlocksPerTile + (lane % kBlocksPerTile));
                if (lane < kBlocksPerTile) {
                    const int y = (id * a.num_kv_heads + hk) * BS;
#pragma unroll
                    for (int h = 0; h < Lay::kHalves; ++h) {
                        const uint32_t off = h * Lay::kHalfBytes + lane * BS * 128;
                        tma_load_3d(ks + off, &tk, 0, y, h, bar(kBarKvFull + s));
                        tma_load_3d(vs + off, &tv, 0, y, h, bar(kBarKvFull + s));
                    }
                }
                issued = j + 1;
            }
            // Let every copy in flight land before the CTA can exit.
            if (lane == 0) {
                for (uint32_t i = 0; i < kWaitLimit && !mbar_test(bar(kBarQ), 0); ++i) {
                }
                for (int j = issued - kPfStages < 0 ? 0 : issued - kPfStages; j < issued; ++j)
                    for (uint32_t i = 0;
                         i < kWaitLimit &&
                         !mbar_test(bar(kBarKvFull + j % kPfStages), (j / kPfStages) & 1);
                         ++i) {
                    }
            }
        } else if (warp == 1) {
            // --------------------------------------------------- MMA issuer
            if (lane == 0) {
                const uint32_t q_s = sb + Lay::kQ, p_s = sb + Lay::kP;
                auto issue_s = [&](int j) {
                    const uint32_t ks = sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile;
                    const uint32_t dst = tmem + (j & 1) * 128u;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k >> 2) * 16384u + (k & 3) * 32u;
                        mma_f16_ss(dst, sw128_desc(q_s + off, 16, 1024),
                                   sw128_desc(ks + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(kBarSFull + (j & 1)));
                };
                bool ok = one_wait(bar(kBarQ), 0, abort_word, a.err);
                if (ok) ok = one_wait(bar(kBarKvFull), 0, abort_word, a.err);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                }
                int ev = 0;
                for (int j = 0; ok && j < nkv; ++j) {
                    if (j + 1 < nkv) {
                        const int s1 = (j + 1) % kPfStages;
                        if (!(ok = one_wait(bar(kBarKvFull + s1), ((j + 1) / kPfStages) & 1,
                                            abort_word, a.err)))
                            break;
                        tc_fence_after();
                        issue_s(j + 1);
                    }
                    const uint32_t vs = sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile +
                                        Lay::kTile;
                    const int parts = j == 0 ? 2 : 1;
                    for (int part = 0; part < parts; ++part, ++ev) {
                        if (!(ok = one_wait(bar(kBarPFull), ev & 1, abort_word, a.err))) break;
                        tc_fence_after();
#pragma unroll
                        for (int k = 0; k < kPfKv / 16; ++k) {
                            const uint64_t ad =
                                sw128_desc(p_s + (k >> 2) * 16384u + (k & 3) * 32u, 16, 1024);
                            const uint64_t bd = sw128_desc(vs + k * 16 * 128, Lay::kHalfBytes, 1024);
                            mma_f16_ss(tmem + kTmemO, ad, bd, kIdescO,
                                       (j > 0 || part > 0 || k > 0) ? 1u : 0u);
                        }
                        if (part == parts - 1) mma_commit(bar(kBarKvEmpty + j % kPfStages));
                        mma_commit(bar(kBarODone));
                    }
                }
                // Every MMA issued above completes before the tensor memory is freed.
                mma_commit(bar(kBarDrain));
                for (uint32_t i = 0; i < kWaitLimit && !mbar_test(bar(kBarDrain), 0); ++i) {
                }
            }
        } else {
            // ------------------------------------------------------ softmax
            const int quarter = warp & 3;  // the TMEM lane quarter this warp may access
            const int r = quarter * 32 + lane;
            const int tok = r >> a.log2_group;
            const int jh = r & (g - 1);
            const bool valid = t_lo + tok < t_hi;
            // rows past the sequence's queries reuse the last valid position
            const int p = L - n + t_lo + min(tok, t_hi - t_lo - 1);
            const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            const uint32_t p_s = sb + Lay::kP;
            const float sl2 = a.sl2;
            float m_used = -INFINITY, l = 0.f;
            int ev = 0;
            bool ok = true;
            for (int j = 0; j < nkv; ++j) {
                if (!(ok = warp_wait(bar(kBarSFull + (j & 1)), (j >> 1) & 1, abort_word, a.err)))
                    break;
                tc_fence_after();
                uint32_t x[128];
                {
                    uint32_t c0[32], c1[32], c2[32], c3[32];
                    const uint32_t src = lane_addr + (j & 1) * 128u;
                    tmem_ld32(src, c0);
                    tmem_ld32(src + 32, c1);
                    tmem_ld32(src + 64, c2);
                    tmem_ld32(src + 96, c3);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        x[i] = c0[i];
                        x[32 + i] = c1[i];
                        x[64 + i] = c2[i];
                        x[96 + i] = c3[i];
                    }
                }
                // S buffer (j & 1) is free once every lane has read it; the
                // arrival on P-full below publishes that to the MMA issuer.
                const int kv0 = j * kPfKv;
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
                if (kv0 + kPfKv - 1 <= p) {  // the whole tile is visible to this row
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const float v = __uint_as_float(x[c]) * sl2;
                        x[c] = __float_as_uint(v);
                        mx[c & 7] = fmaxf(mx[c & 7], v);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const float v = kv0 + c <= p ? __uint_as_float(x[c]) * sl2 : -INFINITY;
                        x[c] = __float_as_uint(v);
                        mx[c & 7] = fmaxf(mx[c & 7], v);
                    }
                }
                const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                       fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const bool rescale = mt > m_used + kRescaleLog2;
                float factor = 1.f;
                if (rescale) {
                    factor = exp2_approx(m_used - mt);
                    m_used = mt;
                    l *= factor;
                }
                uint32_t hi[64], lo[64];
                float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    const float p0 = exp2_approx(__uint_as_float(x[2 * i]) - m_used);
                    const float p1 = exp2_approx(__uint_as_float(x[2 * i + 1]) - m_used);
                    sm[i & 3] += p0 + p1;
                    float r0, r1, q0_, q1_;
                    hi[i] = Pack<T>::two(p0, p1, r0, r1);
                    lo[i] = j == 0 ? Pack<T>::two(p0 - r0, p1 - r1, q0_, q1_) : 0u;
                }
                l += (sm[0] + sm[1]) + (sm[2] + sm[3]);
                // The previous P V must be done: it reads the P tile and writes O.
                if (ev > 0 && !(ok = warp_wait(bar(kBarODone), (ev - 1) & 1, abort_word, a.err)))
                    break;
                tc_fence_after();
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(lane_addr + kTmemO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                        tmem_st32(lane_addr + kTmemO + c * 32, o);
                    }
                    tmem_wait_st();
                }
                if (kv0 + kPfKv > L && kv0 + r >= L) {
                    // Past the context the slots hold whatever a block holds
                    // (possibly NaN or Inf); P is 0 there, but 0 * NaN is NaN, so
                    // the V rows are zeroed.  The copies landed before S_j was
                    // computed, and nothing reads this stage until P V_j.
                    const uint32_t vrow =
                        sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile + Lay::kTile + r * 128u;
#pragma unroll
                    for (int h = 0; h < Lay::kHalves; ++h)
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(
                                             vrow + h * Lay::kHalfBytes + c * 16),
                                         "r"(0u)
                                         : "memory");
                }
                store_p_row(p_s, r, hi);
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(bar(kBarPFull));
                ++ev;
                if (j == 0) {
                    // second product of tile 0: the rounding residual of P
                    if (!(ok = warp_wait(bar(kBarODone), (ev - 1) & 1, abort_word, a.err))) break;
                    store_p_row(p_s, r, lo);
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(bar(kBarPFull));
                    ++ev;
                }
            }
            if (ok && ev > 0) ok = warp_wait(bar(kBarODone), (ev - 1) & 1, abort_word, a.err);
            if (ok) {
                tc_fence_after();
                const int64_t qrow = static_cast<int64_t>(q0) + t_lo + tok;
                const bool store = valid && qrow >= 0 && qrow < a.num_tokens;
                if (valid && !store) flag(a.err, PKV_DEVERR_BAD_QUERY_COUNT);
                const float inv = l > 0.f ? 1.f / l : 0.f;
                T* dst = static_cast<T*>(a.out) +
                         (qrow * a.num_heads + static_cast<int64_t>(hk) * g + jh) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + kTmemO + c * 32, o);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float r0, r1;
                        pk[i] = Pack<T>::two(__uint_as_float(o[2 * i]) * inv,
                                             __uint_as_float(o[2 * i + 1]) * inv, r0, r1);
                    }
                    if (store) {
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

// Q [num_tokens][num_heads][D] as 4-D: x = 64 columns, y = head, z = token,
// w = 64-column half.  A box of 64 x g x (128 / g) x D/64 lands as [half][token]
// [head][128 B] = [half][row][128 B], 128B-swizzled: the A operand of Q K^T.
pkv_status encode_q_map(CUtensorMap* tm, const void* q, int dtype, int num_tokens, int num_heads,
                        int D, int g) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(num_heads), static_cast<cuuint64_t>(num_tokens),
                          static_cast<cuuint64_t>(D / 64)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                             static_cast<cuuint64_t>(num_heads) * D * 2, 128};
    cuuint32_t box[4] = {64, static_cast<cuuint32_t>(g), static_cast<cuuint32_t>(kPfRows / g),
                         static_cast<cuuint32_t>(D / 64)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = encode(tm, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        4, const_cast<void*>(q), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (queries)");
    return PKV_OK;
}

// One pool as 3-D (x = 64 columns, y = row of num_blocks * num_kv_heads *
// block_size, z = 64-column half); a box is one block's rows of one half.
pkv_status encode_block_map(CUtensorMap* tm, const void* pool, const pkv_cache_desc* d) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t rows = static_cast<cuuint64_t>(d->num_blocks) * d->num_kv_heads * d->block_size;
    cuuint64_t dims[3] = {64, rows, static_cast<cuuint64_t>(d->head_dim / 64)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d->head_dim) * 2, 128};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(d->block_size), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(tm, d->dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void*>(pool), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PKV_ERR_CUDA, "cuTensorMapEncodeTiled failed (pool)");
    return PKV_OK;
}

template <typename T, int D, int BS>
struct PrefillTag {};

template <typename T, int D, int BS>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const PrefillArgs& a, cudaStream_t stream) {
    auto* k = prefill_kernel<T, D, BS>;
    cudaError_t e = opt_in_smem<PrefillTag<T, D, BS>>(reinterpret_cast<const void*>(k));
    if (e != cudaSuccess) return e;
    const int tok_per_tile = kPfRows >> a.log2_group;
    dim3 grid(static_cast<unsigned>(a.num_tokens / tok_per_tile + a.num_seqs),
              static_cast<unsigned>(a.num_kv_heads));
    return launch_dependent(k, grid, dim3(kPfThreads), PfLayout<D>::kAlloc, stream, tq, tk, tv, a);
}

template <typename T>
cudaError_t launch_prefill_dt(int D, int BS, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const PrefillArgs& a, cudaStream_t stream) {
    if (D == 128) return BS == 16 ? launch_prefill<T, 128, 16>(tq, tk, tv, a, stream)
                                  : launch_prefill<T, 128, 32>(tq, tk, tv, a, stream);
    return BS == 16 ? launch_prefill<T, 64, 16>(tq, tk, tv, a, stream)
                    : launch_prefill<T, 64, 32>(tq, tk, tv, a, stream);
}

}  // namespace
}  // namespace pkv

using namespace pkv;

extern "C" pkv_status paged_attention_prefill(const pkv_cache_desc* desc, void* out, const void* q,
                                              const void* k_cache, const void* v_cache,
                                              const int32_t* block_tables,
                                              int32_t max_blocks_per_seq,
                                              const int32_t* context_lens,
                                              const int32_t* query_start, int32_t num_seqs,
                                              int32_t num_tokens, int32_t num_heads, float scale,
                                              int32_t* err_flag, void* stream) {
    pkv_status st = check_desc(desc);
    if (st != PKV_OK) return st;
    if (num_seqs < 0 || num_tokens < 0 || num_heads <= 0 || max_blocks_per_seq <= 0)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_prefill: bad sizes");
    if (num_heads % desc->num_kv_heads != 0)
        return fail(PKV_ERR_INVALID_ARG, "num_heads must be a multiple of num_kv_heads");
    const int g = num_heads / desc->num_kv_heads;
    if ((g & (g - 1)) != 0 || g > kPfRows)
        return fail(PKV_ERR_UNSUPPORTED, "num_heads / num_kv_heads must be a power of two <= 128");
    if (!(scale == scale) || scale == INFINITY || scale == -INFINITY)
        return fail(PKV_ERR_INVALID_ARG, "scale must be finite");
    if (static_cast<int64_t>(max_blocks_per_seq) * desc->block_size > INT32_MAX / 2)
        return fail(PKV_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size too large");
    if (num_tokens == 0 || num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_prefill: NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG, "out, q and the pools must be 16-byte aligned");
    if (static_cast<int64_t>(num_tokens) / (kPfRows / g) + num_seqs > INT32_MAX)
        return fail(PKV_ERR_UNSUPPORTED, "too many query tiles");

    CUtensorMap tq, tk, tv;
    if ((st = encode_q_map(&tq, q, desc->dtype, num_tokens, num_heads, desc->head_dim, g)) != PKV_OK)
        return st;
    if ((st = encode_block_map(&tk, k_cache, desc)) != PKV_OK) return st;
    if ((st = encode_block_map(&tv, v_cache, desc)) != PKV_OK) return st;

    PrefillArgs a;
    a.out = out;
    a.tables = block_tables;
    a.lens = context_lens;
    a.qstart = query_start;
    a.err = err_flag;
    a.num_seqs = num_seqs;
    a.num_tokens = num_tokens;
    a.num_heads = num_heads;
    a.num_kv_heads = desc->num_kv_heads;
    a.log2_group = __builtin_ctz(static_cast<unsigned>(g));
    a.max_blocks = max_blocks_per_seq;
    a.num_blocks = desc->num_blocks;
    a.sl2 = scale * 1.4426950408889634f;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = desc->dtype == PKV_BF16
                        ? launch_prefill_dt<__nv_bfloat16>(desc->head_dim, desc->block_size, tq, tk,
                                                           tv, a, s)
                        : launch_prefill_dt<__half>(desc->head_dim, desc->block_size, tq, tk, tv, a, s);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    note_launches(1);
    return PKV_OK;
}
