// pkv_attend.cuh -- the per-tile arithmetic of decode attention, shared by the
// fixed-partition and the balanced schedules.
//
// One warp owns the online-softmax state of the g query heads of one kv head
// (g <= 16 rows of an m16n8k16 tile; rows >= g carry zero queries and are never
// written out).  A K/V tile is `rows` tokens of one (block, kv head), staged in
// shared memory by TMA as 64-column halves of `rows` x 128 B with 128-byte
// swizzle (chunk c of row r sits at chunk c ^ (r & 7)), so every ldmatrix below
// reads 8 distinct bank groups.
#pragma once

#include "pkv_ptx.cuh"

namespace pkv {

template <int D>
struct SoftmaxState {
    float o[D / 8][4];  // O fragment: rows g (o[..][0..1]) and g + 8 (o[..][2..3])
    float m_lo, m_hi;   // running max (base-2 logits) of rows g and g + 8
    float l_lo, l_hi;   // this thread's share of the running sums

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        m_lo = m_hi = -INFINITY;
        l_lo = l_hi = 0.f;
    }
};

// Q rows [g, g+8) of one kv head's group as A fragments of S = Q K^T, read from
// `q` (group rows of D elements, row-major; rows >= group are zero).
template <typename T, int D>
__device__ __forceinline__ void load_q_fragments(uint32_t (&qa)[D / 16][4], const T* q, int group,
                                                 int lane) {
    const int g = lane >> 2, t4 = lane & 3;
    const bool lo_ok = g < group, hi_ok = g + 8 < group;
    const uint32_t* qlo = reinterpret_cast<const uint32_t*>(q + g * D);
    const uint32_t* qhi = reinterpret_cast<const uint32_t*>(q + (g + 8) * D);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        qa[kk][0] = lo_ok ? qlo[8 * kk + t4] : 0u;
        qa[kk][1] = hi_ok ? qhi[8 * kk + t4] : 0u;
        qa[kk][2] = lo_ok ? qlo[8 * kk + 4 + t4] : 0u;
        qa[kk][3] = hi_ok ? qhi[8 * kk + 4 + t4] : 0u;
    }
}

// Keep the 16-bit halves of `v` whose token index (t for the low half, t + 1
// for the high half) is below `end`; zero the others.
__device__ __forceinline__ uint32_t keep_valid(uint32_t v, int t, int end) {
    if (t >= end) return 0u;
    if (t + 1 >= end) return v & 0xffffu;
    return v;
}

// Attend the 16 tokens [tok0, tok0 + 16) held in rows [16*sub, 16*sub + 16) of
// the staged K and V tiles (shared addresses kst, vst; `half_bytes` between the
// 64-column halves).  Tokens at or past t_end are masked: their scores become
// -inf and their V rows are zeroed in registers, so whatever the slots hold
// (even NaN) cannot reach the output.  sl2 = scale * log2(e).
template <typename T, int D>
__device__ __forceinline__ void attend_16(SoftmaxState<D>& st, const uint32_t (&qa)[D / 16][4],
                                          uint32_t kst, uint32_t vst, int half_bytes, int sub,
                                          int tok0, int t_end, float sl2, int lane) {
    const int t4 = lane & 3;
    const int mi = lane >> 3;

    // S (16 query rows x 16 tokens) = Q K^T
    float sc[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
    {
        const int r = sub * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int chunk = 2 * kk + (mi & 1);
            const uint32_t addr =
                kst + (chunk >> 3) * half_bytes + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
            uint32_t kb[4];
            ldsm_x4(addr, kb);
            Mma<T>::run(sc[0], qa[kk], kb[0], kb[1]);
            Mma<T>::run(sc[1], qa[kk], kb[2], kb[3]);
        }
    }

    // scale into base 2, mask tokens past the end, row maxima over the quad
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
    const float mn_lo = fmaxf(st.m_lo, mx_lo);
    const float mn_hi = fmaxf(st.m_hi, mx_hi);
    if (__any_sync(0xffffffffu, mn_lo != st.m_lo || mn_hi != st.m_hi)) {
        const float al = exp2_approx(st.m_lo - mn_lo);
        const float ah = exp2_approx(st.m_hi - mn_hi);
        st.l_lo *= al;
        st.l_hi *= ah;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            st.o[i][0] *= al;
            st.o[i][1] *= al;
            st.o[i][2] *= ah;
            st.o[i][3] *= ah;
        }
    }
    st.m_lo = mn_lo;
    st.m_hi = mn_hi;

    // P = 2^(S - m) as the A operand of O += P V, carried as a pair of T values
    // P = P_hi + P_lo (P_hi = round(P), P_lo = round(P - P_hi)), i.e. about 16
    // significant bits: rounding P to T alone (2^-9 relative for bf16) would
    // put errors of up to 2^-9 * max|V| on outputs whose terms cancel.  The row
    // sums take the fp32 P.
    uint32_t pa[4], pl[4];
    {
        float p[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            p[nt][0] = exp2_approx(sc[nt][0] - mn_lo);
            p[nt][1] = exp2_approx(sc[nt][1] - mn_lo);
            p[nt][2] = exp2_approx(sc[nt][2] - mn_hi);
            p[nt][3] = exp2_approx(sc[nt][3] - mn_hi);
            st.l_lo += p[nt][0] + p[nt][1];
            st.l_hi += p[nt][2] + p[nt][3];
        }
        // A fragment of m16n8k16: a0 = row g, tokens 2t..2t+1; a1 = row g+8, same
        // tokens; a2, a3 = the same rows, tokens 8+2t..8+2t+1 (second n-tile of S).
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float r0, r1, e0, e1;
            pa[2 * nt] = Pack<T>::two(p[nt][0], p[nt][1], r0, r1);
            pl[2 * nt] = Pack<T>::two(p[nt][0] - r0, p[nt][1] - r1, e0, e1);
            pa[2 * nt + 1] = Pack<T>::two(p[nt][2], p[nt][3], r0, r1);
            pl[2 * nt + 1] = Pack<T>::two(p[nt][2] - r0, p[nt][3] - r1, e0, e1);
        }
    }

    // O (16 rows x D) += (P_hi + P_lo) (16 x 16 tokens) V (16 tokens x D)
    {
        const bool partial = tok0 + 16 > t_end;
        const int r = sub * 16 + (mi & 1) * 8 + (lane & 7);
        const int ta = tok0 + 2 * t4, tb = tok0 + 8 + 2 * t4;
#pragma unroll
        for (int nd = 0; nd < D / 16; ++nd) {
            const int chunk = 2 * nd + (mi >> 1);
            const uint32_t addr =
                vst + (chunk >> 3) * half_bytes + r * 128 + (((chunk & 7) ^ (r & 7)) << 4);
            uint32_t vb[4];
            ldsm_x4_trans(addr, vb);
            if (partial) {
                vb[0] = keep_valid(vb[0], ta, t_end);
                vb[2] = keep_valid(vb[2], ta, t_end);
                vb[1] = keep_valid(vb[1], tb, t_end);
                vb[3] = keep_valid(vb[3], tb, t_end);
            }
            Mma<T>::run(st.o[2 * nd], pl, vb[0], vb[1]);
            Mma<T>::run(st.o[2 * nd], pa, vb[0], vb[1]);
            Mma<T>::run(st.o[2 * nd + 1], pl, vb[2], vb[3]);
            Mma<T>::run(st.o[2 * nd + 1], pa, vb[2], vb[3]);
        }
    }
}

// Sum each row's l over the 4 lanes of its quad (call once, before merging).
template <int D>
__device__ __forceinline__ void finish_row_sums(SoftmaxState<D>& st) {
    st.l_lo += __shfl_xor_sync(0xffffffffu, st.l_lo, 1);
    st.l_lo += __shfl_xor_sync(0xffffffffu, st.l_lo, 2);
    st.l_hi += __shfl_xor_sync(0xffffffffu, st.l_hi, 1);
    st.l_hi += __shfl_xor_sync(0xffffffffu, st.l_hi, 2);
}

// Write this warp's rows < group of (m, l, O) into the merge area:
// mo [warps][group][D], mm / ml [warps][group].
template <int D>
__device__ __forceinline__ void store_warp_state(const SoftmaxState<D>& st, float* mo, float* mm,
                                                 float* ml, int warp, int group, int lane) {
    const int g = lane >> 2, t4 = lane & 3;
    if (t4 == 0) {
        if (g < group) {
            mm[warp * group + g] = st.m_lo;
            ml[warp * group + g] = st.l_lo;
        }
        if (g + 8 < group) {
            mm[warp * group + g + 8] = st.m_hi;
            ml[warp * group + g + 8] = st.l_hi;
        }
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        const int col = i * 8 + 2 * t4;
        if (g < group)
            *reinterpret_cast<float2*>(mo + (warp * group + g) * D + col) = make_float2(st.o[i][0], st.o[i][1]);
        if (g + 8 < group)
            *reinterpret_cast<float2*>(mo + (warp * group + g + 8) * D + col) =
                make_float2(st.o[i][2], st.o[i][3]);
    }
}

// Combine `warps` states of row r, column d in warp order:
// M = max m_w, acc = sum 2^(m_w - M) o_w[d], den = sum 2^(m_w - M) l_w.
template <int D>
__device__ __forceinline__ void combine_warps(const float* mo, const float* mm, const float* ml,
                                              int warps, int group, int r, int d, float& M,
                                              float& acc, float& den) {
    M = -INFINITY;
    for (int w = 0; w < warps; ++w) M = fmaxf(M, mm[w * group + r]);
    acc = 0.f;
    den = 0.f;
    for (int w = 0; w < warps; ++w) {
        const float mw = mm[w * group + r];
        const float f = mw == -INFINITY ? 0.f : exp2_approx(mw - M);
        acc += f * mo[(w * group + r) * D + d];
        den += f * ml[w * group + r];
    }
}

}  // namespace pkv
