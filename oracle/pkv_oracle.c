/*
 * pkv_oracle.c -- plain CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library imports, links or calls
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg
 * do.  It shares no code, header or table with the CUDA path.
 *
 * Sources (web pages on PagedAttention):
 *   [ops page]   "PagedAttention" operations page (foundry.adhana.ai), sections
 *                "Concept -- What it is" and "How it works -- The mechanics".
 *   [lesson]     "Paged Attention", lesson 3 of "The KV Cache" (aiacademy.guru),
 *                the method paragraph and the virtual-memory analogy table.
 *   [glossary]   "PagedAttention" glossary entry (aimodelwiki.com).
 *
 * What is computed here is the plain definition, written out with no
 * blocking, fusion or reordering:
 *   - gather: a sequence's logical token t lives in physical block
 *     table[t / bs] at offset t % bs ([ops page] Concept: every sequence has a
 *     table from its logical positions to physical blocks; How it works: the
 *     attention kernel fetches keys and values block by block through that
 *     table, wherever the blocks lie);
 *   - attention of one query over the gathered keys and values, softmax with
 *     the maximum subtracted, in double precision;
 *   - the append and block-copy steps as byte copies ([ops page] How it works:
 *     the new token's key and value go into the sequence's current block; shared
 *     blocks are copied on write).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - block layout [num_blocks][num_kv_heads][block_size][head_dim], K and V in
 *     separate pools;
 *   - query head h reads kv head h / (num_heads / num_kv_heads);
 *   - context_len counts the token appended in the same step; 0 gives zeros;
 *   - a negative slot in the append mapping means the token is skipped;
 *   - fp16 / bf16 storage values are widened exactly to double.
 *
 * Parity status: every exported function is pinned by tests under tests/
 * (brute force against torch's scaled_dot_product_attention in float64, with
 * is_causal for the prefill, closed forms, block-permutation invariance,
 * contiguous-slab equality, the split identity, chunked-prefill consistency,
 * and byte round trips); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };

/* ---------------------------------------------------------------- widening */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double mag;
    if (exp == 0) {
        mag = ldexp((double)frac, -24); /* subnormal: frac * 2^-14 * 2^-10 */
    } else if (exp == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(frac | 0x400), exp - 25); /* (1024 + frac) * 2^(e-15-10) */
    }
    return sign ? -mag : mag;
}

/* bfloat16 is the upper half of an IEEE 754 binary32. */
double oracle_bf16_to_double(uint16_t b) {
    uint32_t bits = (uint32_t)b << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double widen(int dtype, uint16_t w) {
    return dtype == ORACLE_BF16 ? oracle_bf16_to_double(w) : oracle_f16_to_double(w);
}

/* Widen n storage words to double (used by the tests to pin the widening). */
void oracle_widen(int dtype, const uint16_t* src, double* dst, int64_t n) {
    for (int64_t i = 0; i < n; ++i) dst[i] = widen(dtype, src[i]);
}

/* ------------------------------------------------------- dense attention */

/*
 * Softmax attention of one query vector over L contiguous keys/values, the
 * textbook definition:
 *     s_t = scale * sum_d q[d] * K[t][d]
 *     m   = max_t s_t
 *     e_t = exp(s_t - m),  l = sum_t e_t
 *     out = (sum_t e_t * V[t]) / l
 * All sums run in ascending index order.  L = 0 gives out = 0.
 * `scores` is caller scratch of at least L doubles.
 */
void oracle_attend_dense(const double* q, const double* K, const double* V, int64_t L,
                         int32_t D, double scale, double* scores, double* out) {
    for (int32_t d = 0; d < D; ++d) out[d] = 0.0;
    if (L <= 0) return;
    double m = -INFINITY;
    for (int64_t t = 0; t < L; ++t) {
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) dot += q[d] * K[t * D + d];
        scores[t] = scale * dot;
        if (scores[t] > m) m = scores[t];
    }
    double l = 0.0;
    for (int64_t t = 0; t < L; ++t) {
        double e = exp(scores[t] - m);
        scores[t] = e;
        l += e;
    }
    for (int64_t t = 0; t < L; ++t)
        for (int32_t d = 0; d < D; ++d) out[d] += scores[t] * V[t * D + d];
    for (int32_t d = 0; d < D; ++d) out[d] /= l;
}

/* --------------------------------------------------------- paged gather */

/*
 * Copy sequence b's keys and values for kv head hk, tokens [t0, t1), out of
 * the block pool into contiguous double arrays ([ops page] How it works: the
 * kernel reads KV through the block table).  Logical token t sits in physical
 * block block_tables[b][t / bs] at offset t % bs.
 * Returns 0, or -1 if a table entry is outside [0, num_blocks).
 */
static int gather_kv(int dtype, const uint16_t* k_cache, const uint16_t* v_cache,
                     const int32_t* table_row, int32_t num_blocks, int32_t num_kv_heads,
                     int32_t block_size, int32_t D, int32_t hk, int64_t t0, int64_t t1,
                     double* K, double* V) {
    for (int64_t t = t0; t < t1; ++t) {
        int32_t phys = table_row[t / block_size];
        int64_t off = t % block_size;
        if (phys < 0 || phys >= num_blocks) return -1;
        int64_t base = (((int64_t)phys * num_kv_heads + hk) * block_size + off) * D;
        for (int32_t d = 0; d < D; ++d) {
            K[(t - t0) * D + d] = widen(dtype, k_cache[base + d]);
            V[(t - t0) * D + d] = widen(dtype, v_cache[base + d]);
        }
    }
    return 0;
}

/*
 * Paged decode attention, the definition: for every sequence b and query head
 * h, attend q[b][h] over the context_lens[b] tokens gathered through the block
 * table from kv head h / (H / Hkv).
 *   q:        [B][H][D] storage words;  k_cache, v_cache: [NB][Hkv][bs][D]
 *   tables:   int32 [B][max_blocks];    context_lens: int32 [B]
 *   seqs:     optional list of n_seqs sequence indices to compute (NULL = all B)
 *   out:      double [B][H][D]; only the listed sequences are written.
 * Returns 0, -1 on a bad table entry, -2 on bad shapes or a listed index outside
 * 0 .. B-1 (checked before anything of that sequence is read), -3 on allocation
 * failure.
 */
int oracle_paged_decode(int dtype, const uint16_t* q, const uint16_t* k_cache,
                        const uint16_t* v_cache, const int32_t* block_tables,
                        int32_t max_blocks, const int32_t* context_lens, int32_t B, int32_t H,
                        int32_t Hkv, int32_t D, int32_t block_size, int32_t num_blocks,
                        double scale, const int32_t* seqs, int32_t n_seqs, double* out) {
    if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || D <= 0 || block_size <= 0) return -2;
    int32_t group = H / Hkv;
    int64_t max_len = (int64_t)max_blocks * block_size;
    double* K = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * D);
    double* V = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * D);
    double* s = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    double* qd = malloc(sizeof(double) * (size_t)D);
    int rc = (K && V && s && qd) ? 0 : -3;
    int32_t count = seqs ? n_seqs : B;
    for (int32_t i = 0; rc == 0 && i < count; ++i) {
        int32_t b = seqs ? seqs[i] : i;
        if (b < 0 || b >= B) { rc = -2; break; }
        int64_t L = context_lens[b];
        if (L < 0 || L > max_len) { rc = -2; break; }
        for (int32_t hk = 0; rc == 0 && hk < Hkv; ++hk) {
            if (gather_kv(dtype, k_cache, v_cache, block_tables + (int64_t)b * max_blocks,
                          num_blocks, Hkv, block_size, D, hk, 0, L, K, V) != 0) {
                rc = -1;
                break;
            }
            for (int32_t h = hk * group; h < (hk + 1) * group; ++h) {
                const uint16_t* qrow = q + ((int64_t)b * H + h) * D;
                for (int32_t d = 0; d < D; ++d) qd[d] = widen(dtype, qrow[d]);
                oracle_attend_dense(qd, K, V, L, D, scale, s, out + ((int64_t)b * H + h) * D);
            }
        }
    }
    free(K); free(V); free(s); free(qd);
    return rc;
}

/*
 * The same attention split along the sequence into partitions of P tokens,
 * each reduced on its own and then merged by log-sum-exp:
 *     per partition p: m_p = max s_t, l_p = sum e^(s_t - m_p), o_p = sum e^(s_t - m_p) V_t
 *     M = max_p m_p;  out = (sum_p e^(m_p - M) o_p) / (sum_p e^(m_p - M) l_p)
 * This is the identity the GPU's split path relies on; the tests pin it to
 * oracle_paged_decode.  Any P >= 1 is accepted.  Same arguments and return
 * codes as oracle_paged_decode.
 */
int oracle_paged_decode_split(int dtype, const uint16_t* q, const uint16_t* k_cache,
                              const uint16_t* v_cache, const int32_t* block_tables,
                              int32_t max_blocks, const int32_t* context_lens, int32_t B,
                              int32_t H, int32_t Hkv, int32_t D, int32_t block_size,
                              int32_t num_blocks, double scale, int32_t P, double* out) {
    if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || D <= 0 || block_size <= 0 || P <= 0) return -2;
    int32_t group = H / Hkv;
    int64_t max_len = (int64_t)max_blocks * block_size;
    int64_t max_parts = max_len / P + 1;
    double* K = malloc(sizeof(double) * (size_t)P * D);
    double* V = malloc(sizeof(double) * (size_t)P * D);
    double* s = malloc(sizeof(double) * (size_t)P);
    double* qd = malloc(sizeof(double) * (size_t)D);
    double* mp = malloc(sizeof(double) * (size_t)max_parts);
    double* lp = malloc(sizeof(double) * (size_t)max_parts);
    double* op = malloc(sizeof(double) * (size_t)max_parts * D);
    int rc = (K && V && s && qd && mp && lp && op) ? 0 : -3;
    for (int32_t b = 0; rc == 0 && b < B; ++b) {
        int64_t L = context_lens[b];
        if (L < 0 || L > max_len) { rc = -2; break; }
        int64_t n_parts = (L + P - 1) / P;
        for (int32_t h = 0; rc == 0 && h < H; ++h) {
            int32_t hk = h / group;
            const uint16_t* qrow = q + ((int64_t)b * H + h) * D;
            for (int32_t d = 0; d < D; ++d) qd[d] = widen(dtype, qrow[d]);
            for (int64_t p = 0; p < n_parts; ++p) {
                int64_t t0 = p * P, t1 = (p + 1) * P < L ? (p + 1) * P : L;
                if (gather_kv(dtype, k_cache, v_cache, block_tables + (int64_t)b * max_blocks,
                              num_blocks, Hkv, block_size, D, hk, t0, t1, K, V) != 0) {
                    rc = -1;
                    break;
                }
                double m = -INFINITY;
                for (int64_t t = 0; t < t1 - t0; ++t) {
                    double dot = 0.0;
                    for (int32_t d = 0; d < D; ++d) dot += qd[d] * K[t * D + d];
                    s[t] = scale * dot;
                    if (s[t] > m) m = s[t];
                }
                double l = 0.0;
                for (int32_t d = 0; d < D; ++d) op[p * D + d] = 0.0;
                for (int64_t t = 0; t < t1 - t0; ++t) {
                    double e = exp(s[t] - m);
                    l += e;
                    for (int32_t d = 0; d < D; ++d) op[p * D + d] += e * V[t * D + d];
                }
                mp[p] = m;
                lp[p] = l;
            }
            double* o = out + ((int64_t)b * H + h) * D;
            for (int32_t d = 0; d < D; ++d) o[d] = 0.0;
            if (n_parts == 0 || rc != 0) continue;
            double M = -INFINITY;
            for (int64_t p = 0; p < n_parts; ++p) if (mp[p] > M) M = mp[p];
            double denom = 0.0;
            for (int64_t p = 0; p < n_parts; ++p) {
                double w = exp(mp[p] - M);
                denom += w * lp[p];
                for (int32_t d = 0; d < D; ++d) o[d] += w * op[p * D + d];
            }
            for (int32_t d = 0; d < D; ++d) o[d] /= denom;
        }
    }
    free(K); free(V); free(s); free(qd); free(mp); free(lp); free(op);
    return rc;
}

/* ------------------------------------------------------ paged prefill */

/*
 * Paged prefill, the definition: the prompt phase reads keys and values
 * through the same block table as decode ([ops page] How it works: the
 * attention kernel reads KV through the block table; Concept: prompt
 * processing is the compute-heavy phase).  Sequence b holds context_lens[b]
 * tokens in the pool, of which the last n_b = query_start[b + 1] -
 * query_start[b] are this step's query tokens (their keys and values already
 * appended).  Query token i of sequence b sits at position
 * p = context_lens[b] - n_b + i and attends causally to tokens 0 .. p.
 *   q:           [T][H][D] storage words, T = query_start[B], sequence b's
 *                queries in rows query_start[b] .. query_start[b + 1] - 1
 *   query_start: int32 [B + 1], non-decreasing, query_start[0] = 0
 *   out:         double [T][H][D]
 * n_b = 1 is decode of the last token; n_b = context_lens[b] is a whole prompt.
 * Returns 0, -1 on a bad table entry, -2 on bad shapes (n_b < 0 or
 * n_b > context_lens[b], a length past the table), -3 on allocation failure.
 */
int oracle_paged_prefill(int dtype, const uint16_t* q, const uint16_t* k_cache,
                         const uint16_t* v_cache, const int32_t* block_tables,
                         int32_t max_blocks, const int32_t* context_lens,
                         const int32_t* query_start, int32_t B, int32_t H, int32_t Hkv,
                         int32_t D, int32_t block_size, int32_t num_blocks, double scale,
                         double* out) {
    if (H <= 0 || Hkv <= 0 || H % Hkv != 0 || D <= 0 || block_size <= 0) return -2;
    if (query_start[0] != 0) return -2;
    int32_t group = H / Hkv;
    int64_t max_len = (int64_t)max_blocks * block_size;
    double* K = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * D);
    double* V = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1) * D);
    double* s = malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
    double* qd = malloc(sizeof(double) * (size_t)D);
    int rc = (K && V && s && qd) ? 0 : -3;
    for (int32_t b = 0; rc == 0 && b < B; ++b) {
        int64_t L = context_lens[b];
        int64_t n = (int64_t)query_start[b + 1] - query_start[b];
        if (L < 0 || L > max_len || n < 0 || n > L) { rc = -2; break; }
        for (int32_t hk = 0; rc == 0 && hk < Hkv; ++hk) {
            if (gather_kv(dtype, k_cache, v_cache, block_tables + (int64_t)b * max_blocks,
                          num_blocks, Hkv, block_size, D, hk, 0, L, K, V) != 0) {
                rc = -1;
                break;
            }
            for (int64_t i = 0; i < n; ++i) {
                int64_t row = query_start[b] + i;
                int64_t p = L - n + i;
                for (int32_t j = 0; j < group; ++j) {
                    int32_t h = hk * group + j;
                    const uint16_t* qrow = q + (row * H + h) * D;
                    for (int32_t d = 0; d < D; ++d) qd[d] = widen(dtype, qrow[d]);
                    oracle_attend_dense(qd, K, V, p + 1, D, scale, s, out + (row * H + h) * D);
                }
            }
        }
    }
    free(K); free(V); free(s); free(qd);
    return rc;
}

/* ------------------------------------------------------ append and copy */

/*
 * Append: write token i's key and value rows (every kv head) into slot
 * slot_mapping[i] of the pool, i.e. physical block slot / bs at offset
 * slot % bs ([ops page] How it works: each step stores the new token's key and
 * value in the block the sequence is currently filling).  A negative slot skips
 * the token.
 *   key, value: [N][Hkv][D] storage words; caches as above, modified in place.
 * Returns 0, or -1 if a slot is past the pool.
 */
int oracle_append(uint16_t* k_cache, uint16_t* v_cache, const uint16_t* key,
                  const uint16_t* value, const int64_t* slot_mapping, int32_t N, int32_t Hkv,
                  int32_t D, int32_t block_size, int32_t num_blocks) {
    for (int32_t i = 0; i < N; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) return -1;
        int64_t phys = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < Hkv; ++h) {
            int64_t dst = ((phys * Hkv + h) * block_size + off) * D;
            int64_t src = ((int64_t)i * Hkv + h) * D;
            memcpy(k_cache + dst, key + src, sizeof(uint16_t) * (size_t)D);
            memcpy(v_cache + dst, value + src, sizeof(uint16_t) * (size_t)D);
        }
    }
    return 0;
}

/*
 * Copy-on-write: for each pair (src, dst) copy the whole block -- every kv
 * head, every offset -- from src to dst, in K and in V ([ops page] How it
 * works: shared blocks are copied on write when a sequence diverges).  Pairs
 * are applied in list order.  block_mapping: int32 [M][2] (src, dst).
 * Returns 0, or -1 if an id is outside the pool.
 */
int oracle_copy_blocks(uint16_t* k_cache, uint16_t* v_cache, const int32_t* block_mapping,
                       int32_t M, int32_t Hkv, int32_t D, int32_t block_size,
                       int32_t num_blocks) {
    int64_t block_words = (int64_t)Hkv * block_size * D;
    for (int32_t i = 0; i < M; ++i) {
        int32_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return -1;
        memcpy(k_cache + dst * block_words, k_cache + src * block_words,
               sizeof(uint16_t) * (size_t)block_words);
        memcpy(v_cache + dst * block_words, v_cache + src * block_words,
               sizeof(uint16_t) * (size_t)block_words);
    }
    return 0;
}

/*
 * Swap out: host[i] = pool[block_list[i]] for K and V, whole blocks ([ops page]
 * How it works: a preempted sequence's blocks are swapped to host memory).
 * Swap in: pool[block_list[i]] = host[i] (restored later).  host_k, host_v:
 * [n][Hkv][bs][D] words.  Returns 0, or -1 if an id is outside the pool.
 */
int oracle_swap_blocks(uint16_t* k_cache, uint16_t* v_cache, uint16_t* host_k, uint16_t* host_v,
                       const int32_t* block_list, int32_t n, int32_t to_host, int32_t Hkv,
                       int32_t D, int32_t block_size, int32_t num_blocks) {
    int64_t block_words = (int64_t)Hkv * block_size * D;
    for (int32_t i = 0; i < n; ++i) {
        int32_t blk = block_list[i];
        if (blk < 0 || blk >= num_blocks) return -1;
        uint16_t* pk = k_cache + blk * block_words;
        uint16_t* pv = v_cache + blk * block_words;
        uint16_t* hk = host_k + i * block_words;
        uint16_t* hv = host_v + i * block_words;
        if (to_host) {
            memcpy(hk, pk, sizeof(uint16_t) * (size_t)block_words);
            memcpy(hv, pv, sizeof(uint16_t) * (size_t)block_words);
        } else {
            memcpy(pk, hk, sizeof(uint16_t) * (size_t)block_words);
            memcpy(pv, hv, sizeof(uint16_t) * (size_t)block_words);
        }
    }
    return 0;
}
