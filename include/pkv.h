/*
 * pkv.h -- C ABI of libpkv, paged KV-cache decode attention for NVIDIA B200 (sm_100a).
 *
 * The operations follow three web pages on PagedAttention:
 *   [ops page]  "PagedAttention" operations page (foundry.adhana.ai), sections
 *               "Concept -- What it is" and "How it works -- The mechanics";
 *   [lesson]    "Paged Attention", lesson 3 of "The KV Cache" (aiacademy.guru),
 *               the method paragraph and the virtual-memory analogy table;
 *   [glossary]  "PagedAttention" glossary entry (aimodelwiki.com).
 * The pages fix the data structures (fixed-size KV blocks in one pool, a block
 * table per sequence, a free pool, reference-counted sharing with copy on write)
 * and the fact that the attention kernel gathers K/V through the block table.
 * They fix no API, layout or precision; those choices are stated here.
 *
 * Conventions for every call below
 * --------------------------------
 * - Layout.  A cache pool is [num_blocks][num_kv_heads][block_size][head_dim]
 *   elements of `dtype`, row-major; K and V are two pools of the same shape.  A
 *   slot id is `block * block_size + offset`.  q and out are [num_seqs][num_heads]
 *   [head_dim]; query head h reads kv head h / (num_heads / num_kv_heads).
 * - Ownership.  Every device buffer (pools, q, out, tables, lengths, slot and
 *   copy lists, workspace, err_flag) belongs to the caller.  The device calls
 *   allocate no device memory and keep no state between calls.
 * - Pointers.  "device" pointers must be device-accessible CUDA allocations on
 *   the current device; "host" pointers are ordinary host memory.
 * - Streams.  `stream` is a cudaStream_t (passed as void*; NULL = legacy default
 *   stream).  Device calls are asynchronous and stream-ordered: they validate
 *   their host-side arguments, enqueue kernels and return.
 * - Errors.  Host-side validation fails before anything is enqueued and returns
 *   PKV_ERR_INVALID_ARG / PKV_ERR_UNSUPPORTED / PKV_ERR_WORKSPACE_TOO_SMALL.  A
 *   failed launch returns PKV_ERR_CUDA.  Device-side checks (a block id outside
 *   the pool, a context length beyond the table, a slot past the pool) never
 *   trap: the kernel ORs a PKV_DEVERR_* bit into `*err_flag` (device int32,
 *   optional, the caller clears it) and skips or clamps the offending access.
 *   pkv_last_error() gives a message for the last failing call of this thread.
 * - Supported shapes.  head_dim in {64, 128}; block_size in {16, 32}; dtype
 *   fp16 or bf16; 1 <= num_heads / num_kv_heads <= 16; num_blocks * num_kv_heads
 *   * block_size < 2^31.  Others return PKV_ERR_UNSUPPORTED.
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,         /* null / misaligned pointer, bad count or id     */
    PKV_ERR_UNSUPPORTED = 2,         /* shape or dtype outside the supported set       */
    PKV_ERR_NO_FREE_BLOCK = 3,       /* the free pool cannot cover the request         */
    PKV_ERR_CUDA = 4,                /* a CUDA call or kernel launch failed            */
    PKV_ERR_WORKSPACE_TOO_SMALL = 5  /* decode workspace smaller than required         */
} pkv_status;

typedef enum pkv_dtype { PKV_F16 = 0, PKV_BF16 = 1 } pkv_dtype;

/* Bits a kernel ORs into *err_flag. */
#define PKV_DEVERR_BAD_BLOCK_ID 1    /* table entry outside [0, num_blocks): block 0 read instead */
#define PKV_DEVERR_BAD_CONTEXT_LEN 2 /* context length < 0 or > max_blocks_per_seq*block_size: clamped */
#define PKV_DEVERR_BAD_SLOT 4        /* slot >= num_blocks*block_size: token skipped */
#define PKV_DEVERR_WAIT_TIMEOUT 8    /* a pipeline wait ran past its time limit (~0.5 s): work skipped */
#define PKV_DEVERR_BAD_PAIR 16       /* copy pair id outside the pool: pair skipped */
#define PKV_DEVERR_BAD_QUERY_COUNT 32 /* prefill: query count < 0 or > context length, or a query
                                         row past num_tokens: clamped / not written */

/* Shape of one KV pool (shared by the K and V pools). */
typedef struct pkv_cache_desc {
    int32_t num_blocks;   /* physical blocks in the pool                    */
    int32_t block_size;   /* tokens per block (16 or 32)                    */
    int32_t num_kv_heads; /* key/value heads                                */
    int32_t head_dim;     /* elements per head (64 or 128)                  */
    pkv_dtype dtype;      /* element type of q, out, pools, key, value      */
} pkv_cache_desc;

/* ------------------------------------------------------------- device calls */

/*
 * Append: write the keys and values of num_tokens new tokens into the pools
 * through a slot mapping ([ops page] How it works: each decode step writes the
 * new token's key and value into the sequence's current block; [lesson]
 * analogy table, Allocation row).
 *   k_cache, v_cache  device, pools as above, written in place.
 *   key, value        device, [num_tokens][num_kv_heads][head_dim], 16-byte aligned.
 *   slot_mapping      device int64 [num_tokens]; token i goes to slot
 *                     slot_mapping[i]; a negative slot skips the token (padding).
 *                     Slots must be distinct (duplicates: unspecified winner).
 *   err_flag          device int32 or NULL; PKV_DEVERR_BAD_SLOT for a slot past the pool.
 * num_tokens == 0 enqueues nothing.  Bit-exact copy of the input rows.
 */
pkv_status paged_kv_append(const pkv_cache_desc* desc, void* k_cache, void* v_cache,
                           const void* key, const void* value, const int64_t* slot_mapping,
                           int32_t num_tokens, int32_t* err_flag, void* stream);

/*
 * Copy-on-write block copy: for each pair (src, dst) copy block src over block
 * dst -- every kv head and offset -- in both pools ([ops page] How it works:
 * sequences that share blocks get private copies only once their contents
 * differ; At a glance: a shared block is duplicated when one of its sequences
 * writes into it).
 *   block_mapping  device int32 [num_pairs][2] = (src, dst).  Destinations must
 *                  be distinct and no destination may be a source (pairs run
 *                  concurrently); the host block manager's pairs always are.
 *   err_flag       device int32 or NULL; PKV_DEVERR_BAD_PAIR for an id outside the pool.
 * num_pairs == 0 enqueues nothing.  Bit-exact.
 */
pkv_status copy_blocks(const pkv_cache_desc* desc, void* k_cache, void* v_cache,
                       const int32_t* block_mapping, int32_t num_pairs, int32_t* err_flag,
                       void* stream);

/*
 * Swap blocks between the pools and host memory, for preemption by swapping
 * ([ops page] How it works: a preempted sequence's blocks are swapped to host
 * memory and restored later).
 *   block_list  device int32 [n]: physical block ids.
 *   host_k, host_v  page-locked host memory (cudaHostAlloc / cudaMallocHost,
 *               torch pin_memory), [n][num_kv_heads][block_size][head_dim]
 *               elements each; the kernel reads or writes it directly over the
 *               host link.  Pageable memory is refused (PKV_ERR_INVALID_ARG).
 *   to_host     1: host[i] = pool[block_list[i]] (swap out);
 *               0: pool[block_list[i]] = host[i] (swap in).
 *   err_flag    device int32 or NULL; PKV_DEVERR_BAD_PAIR for an id outside the pool.
 * n == 0 enqueues nothing.  Bit-exact.
 */
pkv_status swap_blocks(const pkv_cache_desc* desc, void* k_cache, void* v_cache, void* host_k,
                       void* host_v, const int32_t* block_list, int32_t n, int32_t to_host,
                       int32_t* err_flag, void* stream);

/*
 * Workspace bytes paged_attention_decode needs for these shapes and
 * partition_size.
 *   partition_size 0 (balanced): 2 * G * (group * (head_dim + 2) * 4 + 16) bytes,
 *     G = resident CTAs of the decode on the current device (SM count x CTAs
 *     per SM), group = num_heads / num_kv_heads.  Layout: partial outputs
 *     float [G][2][group][head_dim], partial maxima and sums float
 *     [G][2][group][2], partial descriptors int32 [G][2][4].
 *   partition_size > 0 (fixed): 0 when partition_size >= max_blocks_per_seq *
 *     block_size (no split); else the balanced workspace above rounded up to
 *     256 bytes, then the partitions' float partial outputs
 *     [num_seqs][num_heads][P_max][head_dim], then maxima and sums
 *     [num_seqs][num_heads][P_max] each, P_max = ceil(max_blocks_per_seq *
 *     block_size / partition_size).
 * Returns 0 on invalid arguments, and when a split is asked for but no CUDA
 * device is visible (the balanced part is sized by the current device).
 */
size_t paged_attention_workspace_bytes(const pkv_cache_desc* desc, int32_t num_seqs,
                                       int32_t num_heads, int32_t max_blocks_per_seq,
                                       int32_t partition_size);

/*
 * Paged decode attention: one query token per sequence attends over its
 * context, reading keys and values through the block table ([ops page] How it
 * works: the attention kernel fetches keys and values block by block through
 * the table, wherever the blocks lie; Concept: the block table maps logical
 * positions to physical blocks; [glossary]).
 *   out[b][h][:] = sum_t softmax_t(scale * q[b][h] . K[b][t]) V[b][t],
 *   t < context_lens[b], K/V of logical token t read from physical block
 *   block_tables[b][t / block_size] at offset t % block_size, kv head
 *   h / (num_heads / num_kv_heads).
 * Arithmetic: fp16/bf16 inputs, fp32 scores, softmax and accumulation.  The
 * probabilities enter the probability-value product on the tensor cores as a
 * pair of `dtype` values, p_hi = round(p) and p_lo = round(p - p_hi), each
 * multiplied by V with fp32 accumulation (two products), so they carry about
 * 16 significant bits; output rounded to `dtype`.  The reduction order depends
 * only on logical token order, so the result is bit-identical under any
 * permutation of physical blocks.
 *   out, q          device [num_seqs][num_heads][head_dim], 16-byte aligned.
 *   k_cache, v_cache device pools, 16-byte aligned (read only).
 *   block_tables    device int32 [num_seqs][max_blocks_per_seq]; entries at or
 *                   past ceil(context_len / block_size) are not read.
 *   context_lens    device int32 [num_seqs]; 0 gives an output of zeros.
 *   partition_size  0 = balanced: the whole batch's work -- one unit per
 *                   (sequence, kv head, block) -- is split evenly over the
 *                   GPU's resident CTAs, whatever the length mix; sequences
 *                   that straddle two CTAs are merged by a second kernel
 *                   (log-sum-exp, in CTA order).  Results then depend on the
 *                   device's SM count (not on timing).
 *                   > 0 = fixed partitions of partition_size tokens (a multiple
 *                   of block_size): each partition's un-normalised partial is
 *                   computed on the balanced schedule (its segments stop at
 *                   partition boundaries; a partition split across CTAs is
 *                   merged in CTA order), then each row's partitions are
 *                   merged by log-sum-exp in partition order (three kernels);
 *                   results depend on the SM count as above.  >=
 *                   max_blocks_per_seq * block_size means no split: one CTA per
 *                   (sequence, kv head), independent of the device.
 *   workspace       device, >= paged_attention_workspace_bytes(...), 16-byte
 *                   aligned; may be NULL when that size is 0.
 *   err_flag        device int32 or NULL (PKV_DEVERR_BAD_BLOCK_ID,
 *                   PKV_DEVERR_BAD_CONTEXT_LEN, PKV_DEVERR_WAIT_TIMEOUT).
 */
pkv_status paged_attention_decode(const pkv_cache_desc* desc, void* out, const void* q,
                                  const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t num_seqs,
                                  int32_t num_heads, float scale, int32_t partition_size,
                                  void* workspace, size_t workspace_bytes, int32_t* err_flag,
                                  void* stream);

/*
 * Decode attention for a batch in which groups of sequences share the first
 * blocks of their block tables -- a common prompt prefix whose blocks every
 * sharing table points at ([ops page] At a glance: shared prompt blocks are
 * referenced by every table that uses them; How it works: sharing with
 * reference counts and copy on write; [glossary] prefix caching).  The result
 * is paged_attention_decode's (same definition, same precision rules); only
 * the schedule differs:
 *   - the balanced decode attends every sequence to its own tokens (those past
 *     the shared ones); for the sequences of a group it leaves its results as
 *     un-normalised partials (m, l, O) in the workspace;
 *   - the decode queries of 128 / g sequences of a group times the g heads of
 *     one kv head form one 128-row tile that attends to the group's shared
 *     blocks on the tensor cores (tcgen05), so each shared K/V row is read once
 *     per tile instead of once per sequence; chunks of 128 or 256 shared tokens
 *     leave partials too;
 *   - a last kernel merges each grouped row's partials by log-sum-exp in a
 *     fixed order (prefix chunks, then the own tokens) and writes `out`.
 * The reduction order depends only on the shapes and the groups, so results
 * are bit-identical under any permutation of physical blocks; they differ from
 * paged_attention_decode's by rounding only.
 *   group_start          HOST int32 [num_groups + 1]: group i is sequences
 *                        group_start[i] .. group_start[i+1] - 1 (strictly
 *                        increasing, group_start[num_groups] <= num_seqs);
 *                        sequences outside every group are decoded as usual.
 *   group_shared_blocks  HOST int32 [num_groups]: the first
 *                        group_shared_blocks[i] entries of every table row of
 *                        group i are the same physical blocks, all full
 *                        (0 = nothing shared).  They are read from the row of
 *                        the group's first sequence; each sequence's
 *                        context_len must be at least group_shared_blocks[i] *
 *                        block_size (else PKV_DEVERR_BAD_CONTEXT_LEN and that
 *                        output is undefined).
 *   num_groups           0 .. 64.
 *   num_heads / num_kv_heads must be a power of two <= 16 when a group shares
 *   blocks (PKV_ERR_UNSUPPORTED otherwise).
 *   workspace            device, >= paged_attention_shared_prefix_workspace_bytes
 *                        (...) for the same arguments, 256-byte aligned.
 * Launches four kernels on `stream` (each a programmatic dependent of the one
 * before).
 * Other arguments, layouts and errors as paged_attention_decode (the schedule
 * is always the balanced one).  The host arrays are read during the call only.
 */
pkv_status paged_attention_decode_shared_prefix(const pkv_cache_desc* desc, void* out,
                                                const void* q, const void* k_cache,
                                                const void* v_cache, const int32_t* block_tables,
                                                int32_t max_blocks_per_seq,
                                                const int32_t* context_lens, int32_t num_seqs,
                                                int32_t num_heads, float scale,
                                                const int32_t* group_start,
                                                const int32_t* group_shared_blocks,
                                                int32_t num_groups, void* workspace,
                                                size_t workspace_bytes, int32_t* err_flag,
                                                void* stream);

/*
 * Workspace bytes of paged_attention_decode_shared_prefix: the balanced
 * decode's workspace (paged_attention_workspace_bytes with partition_size 0)
 * rounded up to 256 bytes; then the prefix partials, float O [S][head_dim] and
 * (m, l) [S][2] in whole 128-row tiles, S = 128 x num_kv_heads x (sum over
 * groups that share blocks of ceil(sequences / (128 / g)) x chunks), g =
 * num_heads / num_kv_heads, chunks = ceil(shared tokens / (128 x tiles per
 * chunk)), 1 or 2 tiles per chunk; then the own-token partials of the grouped
 * rows, float O [R][head_dim] and (m, l) [R][2], R = (sequences of groups that
 * share blocks) x num_heads.  0 on invalid arguments.
 */
size_t paged_attention_shared_prefix_workspace_bytes(const pkv_cache_desc* desc, int32_t num_seqs,
                                                     int32_t num_heads, int32_t max_blocks_per_seq,
                                                     const int32_t* group_start,
                                                     const int32_t* group_shared_blocks,
                                                     int32_t num_groups);

/*
 * Paged prefill attention: the prompt phase through the same block table
 * ([ops page] How it works: attention reads keys and values through the block
 * table; Concept: processing the prompt is the compute-bound phase, generation
 * the memory-bound one).  Sequence b holds context_lens[b] tokens in the pool,
 * of which the last n_b = query_start[b + 1] - query_start[b] are this call's
 * query tokens, their keys and values already appended (paged_kv_append).
 * Query token i of sequence b sits at position p = context_lens[b] - n_b + i
 * and attends causally to tokens 0 .. p:
 *   out[query_start[b] + i][h][:] = sum_{t <= p} softmax_t(scale q . K[b][t]) V[b][t]
 * with kv head h / (num_heads / num_kv_heads).  n_b = context_lens[b] is a
 * whole prompt, n_b < context_lens[b] a chunk of one (chunked prefill), n_b = 1
 * a single decode token, n_b = 0 nothing.
 * Arithmetic: fp16/bf16 inputs; Q K^T and P V on the tensor cores with fp32
 * accumulation; softmax in fp32 (base 2, scale * log2 e folded in); the
 * probabilities enter P V rounded to `dtype` (for query rows that see at most
 * 128 tokens their rounding residual is added by a second product); output
 * rounded to `dtype`.  scale must be positive.
 *   out, q          device [num_tokens][num_heads][head_dim], 16-byte aligned,
 *                   not overlapping; rows of a sequence are consecutive,
 *                   sequences in order.  A full 128-row query tile of out is
 *                   written by one bulk tensor store, other rows one by one;
 *                   rows that belong to no sequence are not written.
 *   k_cache, v_cache device pools, 16-byte aligned (read only).
 *   block_tables    device int32 [num_seqs][max_blocks_per_seq]; entries at or
 *                   past ceil(context_len / block_size) are not read.
 *   context_lens    device int32 [num_seqs].
 *   query_start     device int32 [num_seqs + 1], non-decreasing from 0,
 *                   query_start[num_seqs] <= num_tokens.
 *   num_heads / num_kv_heads must be a power of two <= 128.
 *   err_flag        device int32 or NULL (PKV_DEVERR_BAD_BLOCK_ID,
 *                   PKV_DEVERR_BAD_CONTEXT_LEN, PKV_DEVERR_BAD_QUERY_COUNT,
 *                   PKV_DEVERR_WAIT_TIMEOUT).
 * Needs no workspace.  num_tokens == 0 enqueues nothing.
 */
pkv_status paged_attention_prefill(const pkv_cache_desc* desc, void* out, const void* q,
                                   const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, const int32_t* query_start,
                                   int32_t num_seqs, int32_t num_tokens, int32_t num_heads,
                                   float scale, int32_t* err_flag, void* stream);

/*
 * Decode without a caller workspace, for callers that cannot allocate device
 * memory: a plugin inside a serving engine whose allocator already holds nearly
 * all of the GPU's memory, or a latency-critical loop that must never call
 * cudaMalloc (it synchronises the device and can fail when memory is
 * fragmented).  The paper (the pages this library follows) has no
 * counterpart to this call.
 *
 * Same arguments and result as paged_attention_decode without workspace /
 * workspace_bytes: the partial results of split sequences go to a fixed
 * PKV_STATIC_SCRATCH_BYTES array compiled into the library, which every GPU
 * that loads the library holds until the process exits.  Shapes whose
 * paged_attention_workspace_bytes(...) exceeds that size are rejected with
 * PKV_ERR_WORKSPACE_TOO_SMALL and nothing is enqueued.  The call allocates
 * nothing.
 *   - The first call on a device looks up the array's device address with that
 *     device current, and looks it up again only when the current CUDA context
 *     is another one than before (after cudaDeviceReset, say); make the first
 *     call in each context before any stream capture.
 *   - Every call on a device uses the same array, which keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls that can run at the
 *     same time on the GPU (different streams, no ordering) race on the array
 *     and give wrong results: order them on one stream, or use
 *     paged_attention_decode with separate workspaces.
 */
#define PKV_STATIC_SCRATCH_BYTES (16u << 20) /* 16 MiB */
pkv_status paged_attention_decode_static_scratch(const pkv_cache_desc* desc, void* out,
                                                 const void* q, const void* k_cache,
                                                 const void* v_cache,
                                                 const int32_t* block_tables,
                                                 int32_t max_blocks_per_seq,
                                                 const int32_t* context_lens, int32_t num_seqs,
                                                 int32_t num_heads, float scale,
                                                 int32_t partition_size, int32_t* err_flag,
                                                 void* stream);

/* -------------------------------------------------- host block bookkeeping */
/*
 * The block manager of [ops page] Concept and How it works and the [lesson]
 * analogy table: a pool of num_blocks fixed-size blocks, one free pool, a block
 * table per sequence, blocks handed out one at a time when the last one fills,
 * freed blocks returned to the pool, sharing by reference count (fork) and copy
 * on write.  Host memory only; not thread-safe (one pool per thread, or lock).
 * Tie-breaks the pages leave open, fixed so results are reproducible:
 *   - the free pool is a LIFO stack that starts with free_order[0] on top
 *     (free_order NULL = 0, 1, 2, ...);
 *   - pkv_seq_free pushes a sequence's blocks in logical order (its last block
 *     ends on top); shared blocks are only decremented;
 *   - sequence ids count up from 0 and are never reused;
 *   - a request that the free pool cannot cover fails with
 *     PKV_ERR_NO_FREE_BLOCK and changes nothing.
 */
typedef struct pkv_pool pkv_pool;

typedef struct pkv_stats {
    int64_t free_blocks;     /* blocks in the free pool                              */
    int64_t allocated_slots; /* (num_blocks - free_blocks) * block_size              */
    int64_t live_slots;      /* distinct slots holding a token of a live sequence    */
    int64_t live_tokens;     /* sum of live sequence lengths (shared tokens counted per sequence) */
    int64_t shared_blocks;   /* blocks with reference count > 1                      */
    int64_t num_seqs;        /* resident (not swapped-out) sequences                 */
    int64_t swapped_seqs;    /* swapped-out sequences                                */
    int64_t cached_blocks;   /* blocks findable by pkv_seq_new_cached                */
} pkv_stats;

/* free_order: host int32 [num_blocks], a permutation of 0..num_blocks-1, or NULL. */
pkv_status pkv_pool_create(int32_t num_blocks, int32_t block_size, const int32_t* free_order,
                           pkv_pool** out);
void pkv_pool_destroy(pkv_pool* pool);

/* A new, empty sequence. */
pkv_status pkv_seq_new(pkv_pool* pool, int32_t* seq_id);

/* A new sequence sharing every block of `parent` (each block's refcount + 1). */
pkv_status pkv_seq_fork(pkv_pool* pool, int32_t parent, int32_t* child);

/*
 * Make room for n_tokens more tokens of `seq`: slots_out (host int64
 * [n_tokens]) receives their slot ids in order.  A fresh block is taken only
 * when the last block is full.  If the first token lands in a partly filled
 * block that other sequences share, that block is first copied: the pair
 * (src, dst) goes to cow_pair_out (host int32 [2]) and *n_cow_out is 1, else 0.
 * The caller must run copy_blocks on the pair before appending.
 */
pkv_status pkv_seq_reserve(pkv_pool* pool, int32_t seq, int32_t n_tokens, int64_t* slots_out,
                           int32_t* cow_pair_out, int32_t* n_cow_out);

/*
 * One decode step's allocation in one call: for i = 0 .. n_seqs-1, in order,
 * what pkv_seq_reserve(pool, seqs[i], n_tokens[i], ...) does (n_tokens NULL
 * means one token each).  slots_out (host int64, sum of the counts) receives the
 * sequences' slots back to back; copy pairs go to cow_pairs_out (host int32
 * [cow_cap][2]) in order and *n_cow_out counts them (a sequence needs at most
 * one, so cow_cap = n_seqs always suffices).  The first sequence that cannot be
 * served -- free pool exhausted (PKV_ERR_NO_FREE_BLOCK), unknown or swapped out,
 * or needing a copy past cow_cap (PKV_ERR_INVALID_ARG) -- ends the batch with
 * that status; the *n_done sequences before it keep their reservations and
 * their slots and pairs are in the outputs, and nothing of the failing one
 * changed.  n_cow_out and n_done are required.
 */
pkv_status pkv_pool_reserve_batch(pkv_pool* pool, const int32_t* seqs, int32_t n_seqs,
                                  const int32_t* n_tokens, int64_t* slots_out,
                                  int32_t* cow_pairs_out, int32_t cow_cap, int32_t* n_cow_out,
                                  int32_t* n_done);

/*
 * Prefix caching ([glossary], paragraph on prefix caching: requests whose
 * prompts start the same point their block tables at the KV blocks already
 * computed for that start; [ops page] When to use it: a large system prompt
 * shared by many requests).  A full block is named by
 * (the previous block
 * of its sequence, or -1 for the first block; its block_size token ids).
 * pkv_seq_reserve_tokens: pkv_seq_reserve for the token ids `tokens` [n_tokens]
 *   (host int32); every block it fills is registered under its name if its
 *   predecessor is registered (or it is the first block) and the name is free.
 *   A sequence grown by pkv_seq_reserve (ids unknown) registers nothing more.
 * pkv_seq_new_cached: a new sequence that starts on the longest run of
 *   registered blocks matching the prompt's full blocks, each shared (refcount
 *   + 1); *n_cached = the tokens covered (a multiple of block_size).  The caller
 *   appends the rest with pkv_seq_reserve_tokens.
 * An entry lives while its block is in use: when a block's count reaches 0 its
 * entry is dropped, with every entry chained below it.  Copies made on write and
 * blocks returned by swap-in are not registered.
 */
pkv_status pkv_seq_reserve_tokens(pkv_pool* pool, int32_t seq, const int32_t* tokens,
                                  int32_t n_tokens, int64_t* slots_out, int32_t* cow_pair_out,
                                  int32_t* n_cow_out);
pkv_status pkv_seq_new_cached(pkv_pool* pool, const int32_t* prompt, int32_t n, int32_t* seq_id,
                              int32_t* n_cached);

/*
 * Give `seq` a private copy of its logical block `logical_block` if that block
 * is shared: the pair goes to pair_out (host int32 [2]), *n_out = 1; a block
 * already private gives *n_out = 0.
 */
pkv_status pkv_seq_cow(pkv_pool* pool, int32_t seq, int32_t logical_block, int32_t* pair_out,
                       int32_t* n_out);

/* Release the sequence: every block's refcount - 1; blocks reaching 0 return to the pool. */
pkv_status pkv_seq_free(pkv_pool* pool, int32_t seq);

/*
 * Preemption by swapping ([ops page] How it works: when the free pool empties
 * the scheduler preempts a sequence and swaps its blocks to host memory, then
 * restores them later).
 * pkv_seq_swap_out: write the sequence's blocks, logical order, to blocks_out
 * (host int32, capacity cap >= its block count; *n = the count), then release
 * them exactly as pkv_seq_free does.  The sequence keeps its length and id and
 * holds no blocks; reserve, fork, cow and pkv_pool_block_tables refuse it until
 * it is swapped in.  Copy the listed blocks out (swap_blocks, device to host)
 * before anything reuses them.
 * pkv_seq_swap_in: take ceil(len / block_size) fresh blocks, all or nothing
 * (PKV_ERR_NO_FREE_BLOCK and no change if the pool is short), make them the
 * sequence's table and write them, logical order, to blocks_out; then copy the
 * saved contents back into them (swap_blocks, host to device).  Sharing is not
 * restored: every block comes back with reference count 1.
 */
pkv_status pkv_seq_swap_out(pkv_pool* pool, int32_t seq, int32_t* blocks_out, int32_t cap,
                            int32_t* n);
pkv_status pkv_seq_swap_in(pkv_pool* pool, int32_t seq, int32_t* blocks_out, int32_t cap,
                           int32_t* n);

pkv_status pkv_seq_len(const pkv_pool* pool, int32_t seq, int64_t* len);

/* The sequence's block table: *n entries, at most cap of them written to row. */
pkv_status pkv_seq_block_table(const pkv_pool* pool, int32_t seq, int32_t* row, int32_t cap,
                               int32_t* n);

/*
 * Decode-step export: for the n_seqs sequences listed in seqs, write their
 * block tables into tables (host int32 [n_seqs][max_blocks_per_seq], unused
 * entries set to pad) and their lengths into context_lens (host int32 [n_seqs]).
 */
pkv_status pkv_pool_block_tables(const pkv_pool* pool, const int32_t* seqs, int32_t n_seqs,
                                 int32_t* tables, int32_t max_blocks_per_seq,
                                 int32_t* context_lens, int32_t pad);

pkv_status pkv_pool_refcount(const pkv_pool* pool, int32_t block, int32_t* refcount);

/* Free ids from the top of the stack down: *n entries, at most cap written. */
pkv_status pkv_pool_free_list(const pkv_pool* pool, int32_t* out, int32_t cap, int32_t* n);

pkv_status pkv_pool_stats(const pkv_pool* pool, pkv_stats* stats);

/*
 * Shared-prefix groups of a batch for paged_attention_decode_shared_prefix,
 * from host copies of its block tables (int32 [num_seqs][max_blocks_per_seq])
 * and lengths (int32 [num_seqs]).  Sequences that point their tables at the
 * same leading blocks share those blocks' keys and values ([ops page] At a
 * glance and How it works: forked sequences share blocks by reference).
 * Walking the batch in order, a group starts at sequence i and takes i + 1,
 * i + 2, ... while the number of leading entries they all have in common with
 * row i -- counting only blocks that are full in every sequence taken -- stays
 * >= min_shared_blocks; it is kept if it holds >= min_group_seqs sequences,
 * else the walk moves on to i + 1.  A gap between two kept groups is written
 * as a group that shares nothing (group_start must be back to back).  Outputs:
 * group_start [max_groups + 1], group_shared_blocks [max_groups], *num_groups
 * <= max_groups (groups that do not fit are dropped: their sequences are then
 * decoded as usual).  Host memory only; deterministic.
 */
pkv_status pkv_shared_prefix_groups(const int32_t* block_tables, int32_t num_seqs,
                                    int32_t max_blocks_per_seq, const int32_t* context_lens,
                                    int32_t block_size, int32_t min_group_seqs,
                                    int32_t min_shared_blocks, int32_t max_groups,
                                    int32_t* group_start, int32_t* group_shared_blocks,
                                    int32_t* num_groups);

/* --------------------------------------------------------------- diagnostics */

/* Kernels this library has launched in this process (all devices, all threads). */
uint64_t pkv_launch_count(void);

/* Message for the last non-OK status returned to this thread ("" if none). */
const char* pkv_last_error(void);

const char* pkv_status_string(pkv_status status);

/*
 * Self-test of the bounded waits (failure detection without a fault): launches
 * one warp that waits on a shared-memory mbarrier nothing ever arrives on, with
 * the wait the decode kernels use between their producer and consumers
 * (which = 0), the decode kernels' abortable wait (which = 1) or the prefill
 * kernel's wait (which = 2).  The wait gives up by itself -- after about 2^30
 * SM cycles, half a second at full clock, like every wait in the kernels -- and ORs
 * PKV_DEVERR_WAIT_TIMEOUT into *err_flag (device int32, required); the context
 * stays usable.  Stream-ordered; returns PKV_ERR_INVALID_ARG for another `which`
 * or a null err_flag, PKV_ERR_CUDA if the launch fails.
 */
pkv_status pkv_selftest_wait_timeout(int32_t which, int32_t* err_flag, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
