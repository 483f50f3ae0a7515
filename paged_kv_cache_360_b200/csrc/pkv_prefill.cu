// pkv_prefill.cu -- paged prefill attention on the tcgen05 tensor cores.
//
// The prompt phase of PagedAttention ("PagedAttention" operations page, How it
// works: attention reads keys and values through the block table; Concept:
// prompt processing is the compute-bound phase): the last n_b tokens of every
// sequence attend causally to the sequence's paged context.
//
// A query tile is 128 rows: 128 / g consecutive query tokens times the g query
// heads that share one kv head, so every key and value row fetched serves g
// heads.  One CTA takes two neighbouring query tiles of one (sequence, kv
// head) -- tile 0 the later one, tile 1 the one before it -- against the same
// stream of 128-token kv tiles, so each K/V tile is loaded once for 256 rows and
// the tensor core alternates between the tiles while each tile's softmax runs:
//   warp 8      producer: both Q tiles (4-D TMA boxes), then per kv tile one
//               3-D TMA box per (block, 64-column half) of K and of V into two
//               2-stage rings (K freed by Q K^T, V by P V), K one tile ahead;
//   warp 9      MMA issuer (one thread) and tensor-memory owner.  Per tile t:
//               S_t = Q_t K_j^T (fp32, 128 TMEM columns), then O_t += P_t V_j
//               with P_t read from tensor memory, O_t in its own 128 columns;
//               order: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ...
//   warps 0-3   softmax of tile 0, warps 4-7 of tile 1; one row per thread
//               (TMEM lane = row): causal mask, running maximum, P = 2^(s - m)
//               rounded to the input type and written back over S's first 64
//               columns; for rows that see only the first kv tile the
//               rounding residual goes to columns 64-127 and enters P V as a
//               second product.  O is
//               rescaled in tensor memory only when the maximum grows by more
//               than 2^8.  The MMAs of one thread complete in issue order, so
//               when S_t(j) is complete so is P_t V(j-1): O_t is stable during
//               the softmax and needs no extra wait.  At the end, O / l goes to
//               global memory: a full tile as one bulk tensor store staged in
//               its (by then free) Q buffer, a partial tile row by row.
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
#include "pkv_wait.cuh"

namespace pkv {
namespace {

constexpr int kPfThreads = 384;      // 2 softmax warpgroups, then producer, MMA, 2 idle warps
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// Register split (setmaxnreg): the launch gives 384 threads x 168 registers =
// 64512; the softmax warpgroups take 224 each, the third warpgroup 56:
// 256 x 224 + 128 x 56 = 64512.
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(256 * kSoftmaxRegs + 128 * kOtherRegs <= kPfThreads * 168, "register split");
constexpr int kPfRows = 128;         // MMA M: query rows per tile
constexpr int kPfKv = 128;           // kv tokens per tile: N of Q K^T, K of P V
constexpr int kPfStages = 2;         // K and V ring depth
constexpr uint32_t kTmemCols = 512;  // S_t at 128 t, O_t at 256 + 128 t
constexpr float kRescaleLog2 = 8.f;  // rescale O when the maximum grows by > 2^8
constexpr int kResidualTiles = 1;    // P's rounding residual for rows inside the first kv tile

enum : int {
    kBarQ = 0,
    kBarKFull = 1,
    kBarKEmpty = kBarKFull + kPfStages,
    kBarVFull = kBarKEmpty + kPfStages,
    kBarVEmpty = kBarVFull + kPfStages,
    kBarSFull = kBarVEmpty + kPfStages,  // per query tile
    kBarPFull = kBarSFull + 2,           // per query tile, 128 arrivals
    kBarODone = kBarPFull + 2,           // per query tile
    kBarDrain = kBarODone + 2,
    kNumBars
};

// Shared memory, from a 1 KiB aligned base.  Every operand tile is [half][128
// rows][128 B], 128B-swizzled (the TMA's pattern), halves 16 KiB apart.
template <int D>
struct PfLayout {
    static constexpr int kHalves = D / 64;
    static constexpr int kHalfBytes = 128 * 128;
    static constexpr int kTile = kHalves * kHalfBytes;          // 128 rows x D
    static constexpr int kQ = 0;                                // two Q tiles
    static constexpr int kStage0 = 2 * kTile;                   // stage s: K, then V
    static constexpr int kBars = kStage0 + 2 * kPfStages * kTile;
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

// Paired fp32 arithmetic (two lanes per 64-bit register) and a 3-input max.
__device__ __forceinline__ uint64_t f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_split(uint64_t r, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                     taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
                 "r"(r[7])
                 : "memory");
}

// Two floats rounded to one 32-bit pair of T (first in the low half).
template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi) {
    float r0, r1;
    return Pack<T>::two(lo, hi, r0, r1);
}

__device__ __forceinline__ void flag(int32_t* err, int bit) {
    if (err) atomicOr(err, bit);
}

// Diagnostic (pkv_selftest_wait_timeout, which = 2): one warp waits with the
// prefill kernel's bounded wait on an mbarrier that nothing ever arrives on; the
// wait gives up by itself, raises the abort word and reports the timeout.
__global__ void selftest_wait_kernel(int32_t* err) {
    __shared__ __align__(8) uint64_t bar_word;
    __shared__ uint32_t abort_word;
    const uint32_t bar = smem_addr(&bar_word);
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        abort_word = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    warp_wait(bar, 0, &abort_word, err);
}

// Sequence lengths as the kernel uses them: out-of-range values are clamped.
__device__ __forceinline__ void seq_shape(const PrefillArgs& a, int cap, int b, int& L, int& n) {
    L = __ldg(a.lens + b);
    n = __ldg(a.qstart + b + 1) - __ldg(a.qstart + b);
    L = L < 0 ? 0 : (L > cap ? cap : L);
    n = n < 0 ? 0 : (n > L ? L : n);
}

// Warp 0: which (sequence, pair of query tiles) CTA `i` owns.  A sequence with
// T tiles has ceil(T / 2) items; item k holds tiles T-1-2k and T-2-2k (the last
// item of an odd count holds tile 0 alone), so the most expensive pair of a
// sequence gets its lowest CTA index.  work = {b, upper tile}.
__device__ void find_item(const PrefillArgs& a, int cap, int tok_per_tile, int i, int* work) {
    const int lane = threadIdx.x & 31;
    int base = 0;
    for (int b0 = 0; b0 < a.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        int ni = 0, nt = 0;
        if (b < a.num_seqs) {
            int L, n;
            seq_shape(a, cap, b, L, n);
            nt = (n + tok_per_tile - 1) / tok_per_tile;
            ni = (nt + 1) / 2;
        }
        int inc = ni;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += v;
        }
        const int total = __shfl_sync(0xffffffffu, inc, 31);
        if (i < base + total) {
            const unsigned hit = __ballot_sync(0xffffffffu, base + inc > i);
            const int src = __ffs(hit) - 1;
            const int before = __shfl_sync(0xffffffffu, inc - ni, src);
            const int tiles = __shfl_sync(0xffffffffu, nt, src);
            if (lane == 0) {
                work[0] = b0 + src;
                work[1] = tiles - 1 - 2 * (i - base - before);
            }
            return;
        }
        base += total;
    }
    if (lane == 0) work[0] = -1;
}

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kPfThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                   const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                   const PrefillArgs a) {
    using Lay = PfLayout<D>;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    constexpr uint32_t kIdescS = f16_idesc(kBf16, kPfRows, kPfKv, false);
    constexpr uint32_t kIdescO = f16_idesc(kBf16, kPfRows, D, true);
    static_assert(kPfKv % BS == 0, "a kv tile holds whole blocks");
    static_assert(D <= 128, "O_t has 128 tensor-memory columns");

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
            mbar_init(bar(kBarKFull + s), 1);
            mbar_init(bar(kBarKEmpty + s), 1);
            mbar_init(bar(kBarVFull + s), 1);
            mbar_init(bar(kBarVEmpty + s), 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(kBarSFull + t), 1);
            mbar_init(bar(kBarPFull + t), 128);
            mbar_init(bar(kBarODone + t), 1);
        }
        mbar_init(bar(kBarDrain), 1);
        misc[1] = 0u;
        fence_mbar_init();
        prefetch_tensormap(&tq);
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        prefetch_tensormap(&to);
    }
    if (warp == kMmaWarp) {
        tmem_alloc(sb + Lay::kMisc, kTmemCols);
        tmem_relinquish();
    }
    pdl_wait_primary();
    const int cap = a.max_blocks * BS;
    const int tok_per_tile = kPfRows >> a.log2_group;
    if (warp == kProducerWarp) find_item(a, cap, tok_per_tile, blockIdx.x, work);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    const int b = work[0];
    const int hk = blockIdx.y;
    const int g = 1 << a.log2_group;
    int L = 0, n = 0, q0 = 0, qt0 = 0;
    if (b >= 0) {
        seq_shape(a, cap, b, L, n);
        if (threadIdx.x == 0) {
            const int L_raw = __ldg(a.lens + b);
            const int n_raw = __ldg(a.qstart + b + 1) - __ldg(a.qstart + b);
            if (L_raw != L) flag(a.err, PKV_DEVERR_BAD_CONTEXT_LEN);
            if (n_raw != n) flag(a.err, PKV_DEVERR_BAD_QUERY_COUNT);
        }
        q0 = __ldg(a.qstart + b);
        qt0 = work[1];
    }
    // tile t covers query tokens [lo_t, hi_t) of the sequence and needs kv
    // tiles 0 .. nkv_t - 1 (tile 1 the same tiles or one fewer)
    const int lo0 = qt0 * tok_per_tile, hi0 = min(n, lo0 + tok_per_tile);
    const int lo1 = lo0 - tok_per_tile, hi1 = qt0 > 0 ? lo0 : lo1;
    const int nkv0 = (L - n + hi0 - 1) / kPfKv + 1;
    const int nkv1 = qt0 > 0 ? (L - n + hi1 - 1) / kPfKv + 1 : 0;
    const int nkv = nkv0;
    const int ntiles = qt0 > 0 ? 2 : 1;

    // Each role raises or lowers its register budget first thing in its own
    // branch, so the compiler gives each region the matching limit.
    if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        if (b >= 0) {
            // ------------------------------------------------------ softmax
            const int t = warp >> 2;         // query tile of this warpgroup
            const int quarter = warp & 3;    // the TMEM lane quarter this warp may access
            const int r = quarter * 32 + lane;
            const int tok = r >> a.log2_group;
            const int jh = r & (g - 1);
            const int lo_t = t ? lo1 : lo0, hi_t = t ? hi1 : hi0, my_nkv = t ? nkv1 : nkv0;
            const bool valid = lo_t + tok < hi_t;
            // rows past the sequence's queries reuse the last valid position
            const int p = L - n + lo_t + min(tok, hi_t - lo_t - 1);
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            const uint32_t s_addr = lane_base + 128u * t;
            const uint32_t o_addr = lane_base + 256u + 128u * t;
            const float sl2 = a.sl2;
            float m_used = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j < my_nkv; ++j) {
                if (!(ok = warp_wait(bar(kBarSFull + t), j & 1, abort_word, a.err))) break;
                tc_fence_after();
                uint32_t u[128];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tmem_ld32(s_addr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * c));
                tmem_wait_ld();
                const int kv0 = j * kPfKv;
                const int vis = p - kv0;  // columns 0 .. vis are visible to this row
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                if (__any_sync(0xffffffffu, vis < kPfKv - 1)) {
                    // diagonal tile: masked scores become -inf here (whatever the
                    // slot held), so that 2^(-inf) = 0 below needs no select
#pragma unroll
                    for (int c = 0; c < 128; c += 2) {
                        const float v0 = c <= vis ? __uint_as_float(u[c]) : -INFINITY;
                        const float v1 = c + 1 <= vis ? __uint_as_float(u[c + 1]) : -INFINITY;
                        u[c] = __float_as_uint(v0);
                        u[c + 1] = __float_as_uint(v1);
                        mx[(c >> 1) & 3] = max3(mx[(c >> 1) & 3], v0, v1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 128; c += 2)
                        mx[(c >> 1) & 3] = max3(mx[(c >> 1) & 3], __uint_as_float(u[c]),
                                                __uint_as_float(u[c + 1]));
                }
                // maximum of the raw scores, in base-2 units (sl2 > 0; masked
                // columns never contribute)
                const float mraw = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                const float mt = mraw * sl2;
                const bool rescale = mt > m_used + kRescaleLog2;
                float factor = 1.f;
                if (rescale) {
                    factor = exp2_approx(m_used - mt);
                    m_used = mt;
                    l *= factor;
                }
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O_t is stable: S_t(j) completing means P_t V(j-1) did too
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
                        tmem_st32(o_addr + c * 32, o);
                    }
                }
                // P = 2^(s sl2 - m), 16 columns at a time: the 8 packed pairs go
                // to S_t's columns 8 k .. 8 k + 7 (those scores are already in
                // registers).  Paired fp32 arithmetic for the scaling and sums.
                const uint64_t s2 = f2(sl2, sl2), n2 = f2(-m_used, -m_used);
                uint64_t acc[2] = {0ull, 0ull};
                // Rows that see at most kResidualTiles kv tiles also send the
                // first tile's rounding residual P - round(P) to columns 64 + 8 k
                // (with few visible tokens the 2^-9 relative rounding of each
                // weight does not average out).  Warp-uniform, like the stores.
                if (j == 0 && my_nkv <= kResidualTiles) {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t pk[8], rk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int c0 = 16 * k + 2 * i;
                            float x0, x1;
                            f2_split(ffma2(f2(__uint_as_float(u[c0]), __uint_as_float(u[c0 + 1])), s2,
                                           n2),
                                     x0, x1);
                            const float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
                            acc[i & 1] = fadd2(acc[i & 1], f2(p0, p1));
                            float r0, r1, z0, z1;
                            pk[i] = Pack<T>::two(p0, p1, r0, r1);
                            rk[i] = Pack<T>::two(p0 - r0, p1 - r1, z0, z1);
                        }
                        tmem_st8(s_addr + 8 * k, pk);
                        tmem_st8(s_addr + 64 + 8 * k, rk);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int c0 = 16 * k + 2 * i;
                            float x0, x1;
                            f2_split(ffma2(f2(__uint_as_float(u[c0]), __uint_as_float(u[c0 + 1])), s2,
                                           n2),
                                     x0, x1);
                            const float p0 = exp2_approx(x0), p1 = exp2_approx(x1);
                            acc[i & 1] = fadd2(acc[i & 1], f2(p0, p1));
                            pk[i] = pack_pair<T>(p0, p1);
                        }
                        tmem_st8(s_addr + 8 * k, pk);
                    }
                }
                float sa, sb_, sc, sd;
                f2_split(acc[0], sa, sb_);
                f2_split(acc[1], sc, sd);
                l += (sa + sb_) + (sc + sd);
                if (t == 0 && kv0 + kPfKv > L) {
                    // Past the context the slots hold whatever a block holds
                    // (possibly NaN or Inf); P is 0 there, but 0 * NaN is NaN, so
                    // tile 0's warps zero those V rows once the copy has landed
                    // (tile 0 sees every kv tile tile 1 does, and its P V is
                    // issued first).
                    if (!(ok = warp_wait(bar(kBarVFull + j % kPfStages), (j / kPfStages) & 1,
                                         abort_word, a.err)))
                        break;
                    if (kv0 + r >= L) {
                        const uint32_t vrow = sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile +
                                              Lay::kTile + r * 128u;
#pragma unroll
                        for (int h = 0; h < Lay::kHalves; ++h)
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(
                                                 vrow + h * Lay::kHalfBytes + c * 16),
                                             "r"(0u)
                                             : "memory");
                    }
                    fence_proxy_async_smem();
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(kBarPFull + t));
            }
            if (ok && my_nkv > 0) ok = warp_wait(bar(kBarODone + t), 0, abort_word, a.err);
            // A full tile (every row a query of this sequence) goes out as one
            // bulk tensor store of the tile's rows, staged in its Q buffer (free
            // once the tile's last Q K^T, which completes before its last P V,
            // is done); other tiles store row by row.  Tile-uniform choice, so
            // the tile's four warps all meet the named barrier below.
            const bool full = my_nkv > 0 && hi_t - lo_t == tok_per_tile && q0 + lo_t >= 0 &&
                              static_cast<int64_t>(q0) + lo_t + tok_per_tile <= a.num_tokens;
            const int64_t qrow = static_cast<int64_t>(q0) + lo_t + tok;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if (full) {
                const uint32_t q_t = sb + Lay::kQ + t * Lay::kTile;
                if (ok) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + c * 32, o);
                        tmem_wait_ld();
                        uint32_t pk[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float r0, r1;
                            pk[i] = Pack<T>::two(__uint_as_float(o[2 * i]) * inv,
                                                 __uint_as_float(o[2 * i + 1]) * inv, r0, r1);
                        }
                        // columns 32 c .. 32 c + 31: half c / 2, 16-byte chunks
                        // 4 (c % 2) .. + 3 of the row, 128B-swizzled like the TMA's
                        const uint32_t row = q_t + (c >> 1) * Lay::kHalfBytes + r * 128u;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const uint32_t chunk = (static_cast<uint32_t>((c & 1) * 4 + i) ^ (r & 7u)) * 16u;
                            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + chunk),
                                         "r"(pk[4 * i]), "r"(pk[4 * i + 1]), "r"(pk[4 * i + 2]),
                                         "r"(pk[4 * i + 3])
                                         : "memory");
                        }
                    }
                }
                fence_proxy_async_smem();
                asm volatile("bar.sync %0, 128;" ::"r"(1 + t) : "memory");
                if (r == 0 && ok && *abort_word == 0u) {
                    tma_store_4d(&to, q_t, 0, hk * g, q0 + lo_t, 0);
                    bulk_commit_and_wait_read();
                }
            } else if (ok && my_nkv > 0) {
                tc_fence_after();
                const bool store = valid && qrow >= 0 && qrow < a.num_tokens;
                if (valid && !store) flag(a.err, PKV_DEVERR_BAD_QUERY_COUNT);
                T* dst = static_cast<T*>(a.out) +
                         (qrow * a.num_heads + static_cast<int64_t>(hk) * g + jh) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + c * 32, o);
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
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kOtherRegs));
        if (b >= 0 && warp == kProducerWarp) {
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
                mbar_arrive_expect_tx(bar(kBarQ), ntiles * Lay::kTile);
                for (int t = 0; t < ntiles; ++t)
                    tma_load_4d(sb + Lay::kQ + t * Lay::kTile, &tq, 0, hk * g, q0 + (t ? lo1 : lo0),
                                0, bar(kBarQ));
            }
            auto issue = [&](int j, bool is_v, int id) -> bool {
                const int s = j % kPfStages;
                const int full = (is_v ? kBarVFull : kBarKFull) + s;
                const int empty = (is_v ? kBarVEmpty : kBarKEmpty) + s;
                if (j >= kPfStages &&
                    !warp_wait(bar(empty), ((j / kPfStages) - 1) & 1, abort_word, a.err))
                    return false;
                const uint32_t dst = sb + Lay::kStage0 + 2u * s * Lay::kTile + (is_v ? Lay::kTile : 0u);
                if (lane == 0) mbar_arrive_expect_tx(bar(full), Lay::kTile);
                __syncwarp();
                if (lane < kBlocksPerTile) {
                    const int y = (id * a.num_kv_heads + hk) * BS;
#pragma unroll
                    for (int h = 0; h < Lay::kHalves; ++h)
                        tma_load_3d(dst + h * Lay::kHalfBytes + lane * BS * 128, is_v ? &tv : &tk, 0, y,
                                    h, bar(full));
                }
                return true;
            };
            // K of tile i goes out one step ahead of V of tile i - 1.
            int cur = load_chunk(0), next = 0;
            int k_issued = 0, v_issued = 0, id_prev = 0;
            for (int i = 0; i <= nkv; ++i) {
                int id = 0;
                if (i < nkv) {
                    if (i % kTilesPerChunk == 0) {
                        if (i > 0) cur = next;
                        next = load_chunk(i / kTilesPerChunk + 1);
                    }
                    id = __shfl_sync(0xffffffffu, cur,
                                     (i % kTilesPerChunk) * kBlocksPerTile + (lane % kBlocksPerTile));
                    if (!issue(i, false, id)) break;
                    k_issued = i + 1;
                }
                if (i > 0) {
                    if (!issue(i - 1, true, id_prev)) break;
                    v_issued = i;
                }
                id_prev = id;
            }
            // Let every copy in flight land before the CTA can exit.
            if (lane == 0) {
                quiet_wait(bar(kBarQ), 0);
                for (int j = k_issued - kPfStages < 0 ? 0 : k_issued - kPfStages; j < k_issued; ++j)
                    quiet_wait(bar(kBarKFull + j % kPfStages), (j / kPfStages) & 1);
                for (int j = v_issued - kPfStages < 0 ? 0 : v_issued - kPfStages; j < v_issued; ++j)
                    quiet_wait(bar(kBarVFull + j % kPfStages), (j / kPfStages) & 1);
            }
        } else if (b >= 0 && warp == kMmaWarp) {
            // --------------------------------------------------- MMA issuer
            if (lane == 0) {
                auto issue_s = [&](int t, int j) {
                    const uint32_t q_s = sb + Lay::kQ + t * Lay::kTile;
                    const uint32_t ks = sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile;
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t off = (k >> 2) * 16384u + (k & 3) * 32u;
                        mma_f16_ss(tmem + 128u * t, sw128_desc(q_s + off, 16, 1024),
                                   sw128_desc(ks + off, 16, 1024), kIdescS, k > 0 ? 1u : 0u);
                    }
                    mma_commit(bar(kBarSFull + t));
                };
                bool ok = one_wait(bar(kBarQ), 0, abort_word, a.err);
                if (ok) ok = one_wait(bar(kBarKFull), 0, abort_word, a.err);
                if (ok) {
                    tc_fence_after();
                    for (int t = 0; t < ntiles; ++t) issue_s(t, 0);
                    mma_commit(bar(kBarKEmpty));
                }
                for (int j = 0; ok && j < nkv; ++j) {
                    const uint32_t vs =
                        sb + Lay::kStage0 + 2u * (j % kPfStages) * Lay::kTile + Lay::kTile;
                    // V(j) and K(j + 1) first: they have usually landed by now.  A
                    // barrier check issues nothing for ~100 cycles even on a
                    // completed phase, and between the MMA groups below it would
                    // sit on the softmax -> P V -> S path with the tensor pipe idle.
                    if (!(ok = one_wait(bar(kBarVFull + j % kPfStages), (j / kPfStages) & 1, abort_word,
                                        a.err)))
                        break;
                    if (j + 1 < nkv && !(ok = one_wait(bar(kBarKFull + (j + 1) % kPfStages),
                                                        ((j + 1) / kPfStages) & 1, abort_word, a.err)))
                        break;
                    for (int t = 0; ok && t < 2; ++t) {
                        const int nkv_of_t = t ? nkv1 : nkv0;
                        if (j >= nkv_of_t) continue;
                        if (!(ok = one_wait(bar(kBarPFull + t), j & 1, abort_word, a.err))) break;
                        tc_fence_after();
                        // P V: P in S_t's columns 0-63 (and, in the first kv
                        // tile, its rounding residual in columns 64-127)
                        const int parts = (j == 0 && nkv_of_t <= kResidualTiles) ? 2 : 1;
                        for (int part = 0; part < parts; ++part)
#pragma unroll
                            for (int k = 0; k < kPfKv / 16; ++k)
                                mma_f16_ts(tmem + 256u + 128u * t, tmem + 128u * t + 64u * part + 8u * k,
                                           sw128_desc(vs + k * 16 * 128, Lay::kHalfBytes, 1024), kIdescO,
                                           (j > 0 || part > 0 || k > 0) ? 1u : 0u);
                        if (j + 1 == nkv_of_t) mma_commit(bar(kBarODone + t));
                        if (j + 1 < nkv_of_t) issue_s(t, j + 1);
                    }
                    if (!ok) break;
                    mma_commit(bar(kBarVEmpty + j % kPfStages));
                    if (j + 1 < nkv) mma_commit(bar(kBarKEmpty + (j + 1) % kPfStages));
                }
                // Every MMA issued above completes before the tensor memory is freed.
                mma_commit(bar(kBarDrain));
                quiet_wait(bar(kBarDrain), 0);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

}  // namespace

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

namespace {

template <typename T, int D, int BS>
struct PrefillTag {};

template <typename T, int D, int BS>
cudaError_t launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to,
                           const PrefillArgs& a, cudaStream_t stream) {
    auto* k = prefill_kernel<T, D, BS>;
    cudaError_t e = opt_in_smem<PrefillTag<T, D, BS>>(reinterpret_cast<const void*>(k));
    if (e != cudaSuccess) return e;
    // items per sequence = ceil(ceil(n / tpt) / 2) <= n / (2 tpt) + 1
    const int tok_per_tile = kPfRows >> a.log2_group;
    dim3 grid(static_cast<unsigned>(a.num_tokens / (2 * tok_per_tile) + a.num_seqs),
              static_cast<unsigned>(a.num_kv_heads));
    return launch_dependent(k, grid, dim3(kPfThreads), PfLayout<D>::kAlloc, stream, tq, tk, tv, to, a);
}

template <typename T>
cudaError_t launch_prefill_dt(int D, int BS, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, const CUtensorMap& to, const PrefillArgs& a,
                              cudaStream_t stream) {
    if (D == 128) return BS == 16 ? launch_prefill<T, 128, 16>(tq, tk, tv, to, a, stream)
                                  : launch_prefill<T, 128, 32>(tq, tk, tv, to, a, stream);
    return BS == 16 ? launch_prefill<T, 64, 16>(tq, tk, tv, to, a, stream)
                    : launch_prefill<T, 64, 32>(tq, tk, tv, to, a, stream);
}

}  // namespace
}  // namespace pkv

namespace pkv {
cudaError_t prefill_selftest_wait(int32_t* err, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>(err);
    return cudaGetLastError();
}
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
    if (!(scale > 0.f) || scale == INFINITY)
        return fail(PKV_ERR_INVALID_ARG, "scale must be positive and finite");
    if (static_cast<int64_t>(max_blocks_per_seq) * desc->block_size > INT32_MAX / 2)
        return fail(PKV_ERR_UNSUPPORTED, "max_blocks_per_seq * block_size too large");
    if (num_tokens == 0 || num_seqs == 0) return PKV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
        return fail(PKV_ERR_INVALID_ARG, "paged_attention_prefill: NULL pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(PKV_ERR_INVALID_ARG, "out, q and the pools must be 16-byte aligned");
    {
        const uintptr_t ob = reinterpret_cast<uintptr_t>(out), qb = reinterpret_cast<uintptr_t>(q);
        const uintptr_t bytes = static_cast<uintptr_t>(num_tokens) * num_heads * desc->head_dim * 2u;
        if (ob < qb + bytes && qb < ob + bytes)
            return fail(PKV_ERR_INVALID_ARG, "out must not overlap q");
    }
    if (static_cast<int64_t>(num_tokens) / (kPfRows / g) + num_seqs > INT32_MAX)
        return fail(PKV_ERR_UNSUPPORTED, "too many query tiles");

    CUtensorMap tq, tk, tv, to;
    if ((st = encode_q_map(&tq, q, desc->dtype, num_tokens, num_heads, desc->head_dim, g)) != PKV_OK)
        return st;
    // out has q's shape: the same map describes a tile of output rows
    if ((st = encode_q_map(&to, out, desc->dtype, num_tokens, num_heads, desc->head_dim, g)) != PKV_OK)
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
                                                           tv, to, a, s)
                        : launch_prefill_dt<__half>(desc->head_dim, desc->block_size, tq, tk, tv, to, a,
                                                    s);
    if (e != cudaSuccess) return fail(PKV_ERR_CUDA, cudaGetErrorString(e));
    note_launches(1);
    return PKV_OK;
}
