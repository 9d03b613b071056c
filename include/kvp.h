/*
 * kvp.h - C ABI of libkvp: a paged KV cache and its decode-attention path for
 * NVIDIA B200 (sm_100a).
 *
 * The method (sources cited by page title and section):
 *
 *  - The KV cache of each sequence is cut into fixed-size blocks; a
 *    per-sequence block table maps logical block numbers to physical blocks,
 *    which are taken from a shared pool only when the sequence grows into them,
 *    and the attention kernel follows the block table instead of assuming a
 *    contiguous cache. ["Your GPU was mostly empty: how PagedAttention turned
 *    KV cache waste into 2-4x throughput", section "The OS already solved this
 *    in the 1960s"; "vLLM and PagedAttention", section "Architecture, step by
 *    step", steps 1-3]
 *  - Blocks are shared between sequences by reference count; a block is copied
 *    only when a sequence writes into a block that is shared (block-level
 *    copy-on-write, as with fork()). ["Your GPU was mostly empty", section
 *    "Paging's second gift: copy-on-write"]
 *  - A block that no live sequence references returns to the shared pool.
 *    ["PagedAttention: KV cache memory management", sections "How logical
 *    blocks, physical blocks and the block table work" and "A request
 *    lifecycle: allocation, growth, sharing and release"]
 *
 * Conventions for every call:
 *  - Returns KVP_OK (0) or a negative KVP_ERR_* status; no C++ exception
 *    crosses this boundary. kvp_last_error_message() describes the last
 *    failure of the calling thread.
 *  - A failed host call leaves all state unchanged.
 *  - Host metadata (block tables, reference counts, free list) is owned by the
 *    pool handle. A pool is not thread-safe: one thread at a time per pool.
 *  - Device buffers are owned by the caller and passed as raw device pointers;
 *    no call allocates or frees device memory. `stream` is a cudaStream_t
 *    (NULL = the legacy default stream). Device calls are asynchronous with
 *    respect to the host: they validate their arguments, launch, and return.
 *  - Device-side index checks (block ids, slots, context lengths) never fault:
 *    an out-of-range index is skipped and recorded in a device error word that
 *    kvp_check_device_error() reads back.
 *
 * KV cache layout (the pages fix none; this is the library's choice):
 *   k_cache, v_cache : [num_blocks][num_kv_heads][block_size][head_dim],
 *   row-major, separate K and V buffers, elements fp16 or bf16. One
 *   (physical block, KV head) tile is one contiguous block_size*head_dim run.
 *   Token slot s lives in physical block s / block_size at offset
 *   s % block_size.
 */
#ifndef KVP_H_
#define KVP_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVP_API __attribute__((visibility("default")))
#else
#define KVP_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------- */
#define KVP_OK 0
#define KVP_ERR_INVALID (-1)  /* bad argument or unsupported geometry        */
#define KVP_ERR_OOM (-2)      /* the pool has too few free blocks            */
#define KVP_ERR_NO_SEQ (-3)   /* no live sequence with that id               */
#define KVP_ERR_CUDA (-4)     /* a CUDA runtime call failed                  */
#define KVP_ERR_BOUNDS (-5)   /* a device kernel met an out-of-range index   */
#define KVP_ERR_CAPACITY (-6) /* an output buffer is too small              */

/* ---- element types ------------------------------------------------------ */
#define KVP_F16 0
#define KVP_BF16 1
/* E4M3 codes (1 sign, 4 exponent, 3 mantissa bits, bias 7, largest 448, no
 * infinities) with per-KV-head fp32 scales: a pool of this type is written by
 * reshape_and_cache_fp8 and read by paged_attention_decode_fp8. */
#define KVP_FP8_E4M3 2

typedef struct kvp_pool kvp_pool;
typedef void* kvp_stream_t; /* a cudaStream_t */

typedef struct kvp_pool_stats {
  int64_t num_blocks;
  int64_t num_free;         /* blocks on the free list                      */
  int64_t num_used;         /* blocks with reference count > 0              */
  int64_t num_shared;       /* blocks with reference count > 1              */
  int64_t waste_slots;      /* sum over live sequences of unused slots in   */
                            /* their last block                             */
  int64_t cow_copies_total; /* copy-on-write copies queued since creation   */
  int64_t num_seqs;         /* live sequences                               */
} kvp_pool_stats;

/* =========================================================================
 * Host: block pool and sequences (integer bookkeeping)
 * ========================================================================= */

/* Creates a pool of `num_blocks` physical blocks of `block_size` token slots
 * for a layer group with `num_kv_heads` KV heads of `head_dim` elements of
 * `dtype`: the shared pool of fixed-size physical blocks that sequences take
 * blocks from ["vLLM and PagedAttention", section "Architecture, step by
 * step", step 1; "Your GPU was mostly empty", section "The OS already solved
 * this in the 1960s"]. The free list is a stack: the first block handed out is
 * free_order[0], then free_order[1], ... `free_order` must be a permutation of
 * 0..num_blocks-1 (it is copied); NULL means 0, 1, 2, ... Block placement is
 * then fully determined by the call sequence.
 * Errors: KVP_ERR_INVALID (non-positive sizes, not a permutation, bad dtype). */
KVP_API int kv_pool_create(int32_t num_blocks, int32_t block_size, int32_t num_kv_heads,
                   int32_t head_dim, int32_t dtype, const int32_t* free_order,
                   kvp_pool** out);

/* Frees the pool and all its host metadata. NULL is accepted. */
KVP_API int kv_pool_destroy(kvp_pool* pool);

/* Number of free blocks. */
KVP_API int kv_pool_num_free(const kvp_pool* pool, int32_t* n);

/* Free blocks in hand-out order (next block first) into out[0..cap); *n gets
 * the count. KVP_ERR_CAPACITY (with *n set) if cap is too small. */
KVP_API int kv_pool_free_list(const kvp_pool* pool, int32_t* out, int32_t cap, int32_t* n);

/* Reference count of one block. KVP_ERR_INVALID if block is out of range. */
KVP_API int kv_pool_refcount(const kvp_pool* pool, int32_t block, int32_t* rc);

/* Reference counts of all blocks into out[0..num_blocks). */
KVP_API int kv_pool_refcounts(const kvp_pool* pool, int32_t* out, int32_t cap);

/* Counters of the pool (see kvp_pool_stats). */
KVP_API int kv_pool_stats(const kvp_pool* pool, kvp_pool_stats* out);

/* New empty sequence (no blocks). Ids count up from 0 and are never reused;
 * a fork also takes the next id. */
KVP_API int kv_seq_create(kvp_pool* pool, int64_t* seq_id);

/* Appends n_tokens >= 0 tokens to `seq`, one after another, and writes each
 * token's flat slot (physical_block * block_size + offset) to slots_out
 * (may be NULL when n_tokens == 0). Blocks are taken only as the sequence
 * grows into them and mapped through its block table ["vLLM and
 * PagedAttention", section "Architecture, step by step", steps 1-2;
 * "PagedAttention: KV cache memory management", section "A request lifecycle":
 * a full block makes the runtime take another]; a write into a shared block
 * copies it first ["Your GPU was mostly empty", section "Paging's second gift:
 * copy-on-write"]. A token at a block boundary takes a new
 * block from the free list; a token that lands in a partly filled last block
 * that other sequences also reference first takes a private copy: a new block
 * is taken, the pair (old, new) is queued for copy_blocks, the old block loses
 * one reference and the table entry moves to the new block.
 * Errors: KVP_ERR_NO_SEQ, KVP_ERR_INVALID (n_tokens < 0), KVP_ERR_OOM when the
 * free list cannot supply every block the call needs (nothing changes). */
KVP_API int kv_seq_append(kvp_pool* pool, int64_t seq, int32_t n_tokens, int64_t* slots_out);

/* Appends n_each tokens to every sequence of seqs[0..num_seqs), in that order;
 * the result equals num_seqs successive kv_seq_append calls (with prefix
 * caching on, that ends the sequences' registrations: the token-carrying form
 * is kv_seq_append_tokens_batch).
 * slots_out[i*n_each + j] is token j of seqs[i]. All or nothing: on
 * KVP_ERR_OOM / KVP_ERR_NO_SEQ nothing changes. */
KVP_API int kv_seq_append_batch(kvp_pool* pool, const int64_t* seqs, int32_t num_seqs,
                        int32_t n_each, int64_t* slots_out);

/* New sequence sharing every block of `parent` (each block gains one
 * reference); the child has the parent's length. Parallel samples and beams
 * share their common blocks by reference count, as fork() shares pages ["Your
 * GPU was mostly empty", section "Paging's second gift: copy-on-write"]. */
KVP_API int kv_seq_fork(kvp_pool* pool, int64_t parent, int64_t* child);

/* Ends `seq`: each block of its table, in logical order, loses one reference;
 * a block that reaches zero is pushed onto the free list (with prefix caching
 * on, a registered block becomes evictable instead: see below). A finished
 * request's blocks go back to the shared pool ["vLLM and PagedAttention",
 * section "Architecture, step by step", step 4; "PagedAttention: KV cache
 * memory management", section "A request lifecycle": release]. */
KVP_API int kv_seq_release(kvp_pool* pool, int64_t seq);

/* Length (tokens) of `seq`. */
KVP_API int kv_seq_len(const kvp_pool* pool, int64_t seq, int32_t* len);

/* Block table of `seq` into out[0..cap); *n gets its length.
 * KVP_ERR_CAPACITY (with *n set) if cap is too small. */
KVP_API int kv_seq_block_table(const kvp_pool* pool, int64_t seq, int32_t* out, int32_t cap,
                       int32_t* n);

/* Moves the queued copy-on-write pairs, in creation order, into
 * pairs[2*i] = src, pairs[2*i+1] = dst, and clears the queue: the block copies
 * that copy-on-write owes, for copy_blocks to make on the device ["Your GPU
 * was mostly empty", section "Paging's second gift: copy-on-write"]. KVP_ERR_CAPACITY
 * (with *n set, queue kept) if cap (pairs) is too small. */
KVP_API int kv_pool_take_copies(kvp_pool* pool, int32_t* pairs, int32_t cap, int32_t* n);

/* Like kv_pool_take_copies but leaves the queue as it is. */
KVP_API int kv_pool_pending_copies(const kvp_pool* pool, int32_t* pairs, int32_t cap, int32_t* n);

/* ---- prefix caching across requests -------------------------------------
 * Full blocks keep the keys and values of a token prefix, and a later request
 * whose prompt starts with the same tokens reuses them instead of recomputing
 * them ["PagedAttention: KV cache memory management", section "PagedAttention
 * vs KV-cache quantization vs prefix caching"; sharing across requests: "vLLM
 * and PagedAttention", section "Key claims from the paper"]. Off unless
 * turned on. Policy:
 *  - a block that fills during kv_seq_append_tokens is registered under the
 *    key (registration number of the block before it, or -1 for a first
 *    block; its block_size token ids), unless the key is taken (the first
 *    registration stays), the block is registered, or the block before it is
 *    not registered; registration numbers are never reused, so a key names
 *    one exact token prefix. A kv_seq_append (token ids unknown) ends the
 *    sequence's registrations;
 *  - kv_seq_create_prefixed attaches the longest run of leading registered
 *    blocks of a prompt that ends before the prompt's last token;
 *  - a registered block whose reference count reaches zero becomes evictable
 *    (the blocks of one release from the last logical block to the first)
 *    instead of free; a block taken back by a lookup leaves the evictable list;
 *  - a new block comes from the free stack, and when it is empty from evicting
 *    the evictable block released longest ago (its key dropped); appends
 *    check their need against free plus evictable blocks. */

/* Turns prefix caching on (enable != 0; only while no sequence is live) or
 * off (every registration dropped, evictable blocks pushed to the free stack
 * in eviction order, live sequences no longer registered).
 * Errors: KVP_ERR_INVALID (NULL pool, turning it on with live sequences). */
KVP_API int kv_pool_set_prefix_caching(kvp_pool* pool, int32_t enable);

/* Creates a sequence for a prompt of n_tokens token ids: its table starts
 * with the longest run of cached leading blocks of the prompt ending before
 * its last token (each gains a reference), and its length is that run's
 * tokens, returned in *cached_tokens. The caller appends
 * tokens[*cached_tokens:] with kv_seq_append_tokens and writes only their
 * keys and values. Errors: KVP_ERR_INVALID (NULL arguments, n_tokens < 0,
 * prefix caching off), KVP_ERR_OOM (host allocation). */
KVP_API int kv_seq_create_prefixed(kvp_pool* pool, const int32_t* tokens, int32_t n_tokens,
                                   int64_t* seq_id, int32_t* cached_tokens);

/* kv_seq_append with the token ids given (tokens: host int32 [n_tokens]); on a
 * pool with prefix caching, blocks that fill are registered (policy above).
 * Errors: those of kv_seq_append. */
KVP_API int kv_seq_append_tokens(kvp_pool* pool, int64_t seq, const int32_t* tokens,
                                 int32_t n_tokens, int64_t* slots_out);

/* kv_seq_append_batch with token ids: tokens is host int32 [num_seqs][n_each],
 * row i for seqs[i]; the appends run in batch order, as num_seqs calls of
 * kv_seq_append_tokens would, after one check of the whole batch's need. The
 * decode steps of a serving loop use it so that generated blocks are
 * registered too. Errors: those of kv_seq_append_batch. */
KVP_API int kv_seq_append_tokens_batch(kvp_pool* pool, const int64_t* seqs, int32_t num_seqs,
                                       int32_t n_each, const int32_t* tokens, int64_t* slots_out);

/* The evictable blocks, the one evicted next first. Errors: KVP_ERR_INVALID,
 * KVP_ERR_CAPACITY (cap too small; *n is set). */
KVP_API int kv_pool_evictable_list(const kvp_pool* pool, int32_t* out, int32_t cap, int32_t* n);

/* Registered blocks, evictable blocks, and prompt tokens served from the
 * cache so far. Errors: KVP_ERR_INVALID (NULL argument). */
KVP_API int kv_pool_prefix_stats(const kvp_pool* pool, int64_t* registered, int64_t* evictable,
                                 int64_t* hit_tokens);

/* Packs the batch metadata the decode kernels read: block_tables is
 * [num_seqs][max_blocks] (row i = table of seqs[i], padded with -1) and
 * context_lens[i] = length of seqs[i]: the logical-to-physical map the
 * attention kernel follows ["vLLM and PagedAttention", section "Architecture,
 * step by step", steps 2-3; "PagedAttention: KV cache memory management",
 * section "Operational trade-offs and limits": the runtime keeps the block
 * metadata]. Host buffers; copy them to the device.
 * KVP_ERR_CAPACITY if a table is longer than max_blocks. */
KVP_API int kv_build_batch(const kvp_pool* pool, const int64_t* seqs, int32_t num_seqs,
                   int32_t max_blocks, int32_t* block_tables, int32_t* context_lens);

/* Capacity model: KV bytes per token of a model with `hidden` = heads *
 * head_dim and `layers` layers at `elem_bytes` bytes per value, i.e.
 * 2 * hidden * layers * elem_bytes (one key and one value vector per token
 * and layer). ["Your GPU was mostly empty", section "Why the KV cache is an
 * allocator problem", OPT-13B worked example] */
KVP_API int64_t kvp_kv_bytes_per_token(int64_t hidden, int64_t layers, int64_t elem_bytes);

/* =========================================================================
 * Device: sm_100a kernels on caller-owned memory, on the caller's stream
 * ========================================================================= */

/* Writes each new token's keys and values to its slot: for t < num_tokens
 * with s = slot_mapping[t] >= 0,
 *   k_cache[s / block_size][h][s % block_size][:] = k_new[t][h][:]  (all h)
 * and likewise for V. A negative slot marks padding and is skipped; a slot
 * >= num_blocks * block_size is skipped and sets KVP_ERR_BOUNDS in the device
 * error word. If two tokens name one slot, the result is one of them.
 * ["PagedAttention: KV cache memory management", section "A request
 * lifecycle: allocation, growth, sharing and release": decode appends new
 * cache state]
 * k_new, v_new: device [num_tokens][num_kv_heads][head_dim], dtype.
 * slot_mapping: device int64 [num_tokens]. head_dim * 2 bytes must be a
 * multiple of 16. */
KVP_API int reshape_and_cache(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                      const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                      kvp_stream_t stream);

/* Block-level copy-on-write copies: for each i < num_pairs, with
 * src = pairs[2*i], dst = pairs[2*i+1], the whole physical block dst of K and
 * of V (all KV heads, all slots: block_elems = num_kv_heads * block_size *
 * head_dim elements) becomes a copy of block src. Destinations must be
 * distinct and no destination may be a source. Out-of-range ids are skipped
 * and set KVP_ERR_BOUNDS in the device error word. ["Your GPU was mostly
 * empty", section "Paging's second gift: copy-on-write"]
 * pairs: device int32 [num_pairs][2]. block_elems * (bytes per element: 2,
 * or 1 for KVP_FP8_E4M3) must be a multiple of 16. */
KVP_API int copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int32_t num_pairs,
                int32_t num_blocks, int64_t block_elems, int32_t dtype, kvp_stream_t stream);

/* Bytes of device workspace paged_attention_decode needs for this batch
 * shape: 0 when partition_size == 0 or when no sequence can have more than one
 * partition (max_context_len <= partition_size); else room for, per
 * (sequence, query head, partition), a running max, an exponent sum and
 * head_dim fp32 partial outputs, with P = ceil(max_context_len /
 * partition_size) partitions: about num_seqs * num_q_heads * P *
 * (head_dim + 2) * 4 bytes. */
KVP_API size_t kvp_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                  int32_t max_context_len, int32_t partition_size);

/* Decode attention over the paged cache. For sequence s and query head h,
 * with KV head g = h / (num_q_heads / num_kv_heads) and ctx = context_lens[s]:
 *   key j    = k_cache[block_tables[s][j / block_size]][g][j % block_size][:]
 *   value j  = v_cache[...same...]
 *   out[s][h] = sum_j softmax_j(scale * q[s][h] . key j) * value j,  j < ctx.
 * The kernel follows the block table ["vLLM and PagedAttention", section
 * "Architecture, step by step", step 3]; the result is the same as attention
 * over a contiguous cache ["Your GPU was mostly empty", section "The OS
 * already solved this in the 1960s"]. ctx == 0 gives a zero row.
 * Split context: with partition_size > 0 (a multiple of block_size; the
 * grouped-query tensor-core path needs a multiple of 128), each sequence's
 * tokens are cut into partitions of that many tokens; each partition
 * produces its running max, exponent sum and unnormalised output in
 * `workspace`, and a second kernel merges them by the log-sum-exp identity.
 * Sequences with one partition write `out` directly. partition_size == 0
 * processes each (sequence, head) in one pass and needs no workspace.
 * q: device [num_seqs][num_q_heads][head_dim]; out: same shape and dtype.
 * block_tables: device int32 [num_seqs][max_blocks_per_seq];
 * context_lens: device int32 [num_seqs]; every context_lens[s] must be
 * <= max_context_len <= max_blocks_per_seq * block_size (larger values are
 * clamped and set KVP_ERR_BOUNDS). workspace: device, >=
 * kvp_decode_workspace_bytes(...) bytes, 256-byte aligned, contents ignored.
 * Supported: head_dim 64 or 128; block_size 8, 16 or 32; num_q_heads a
 * multiple of num_kv_heads. Grouped-query batches (num_q_heads >
 * num_kv_heads, group <= 16) run on the tensor cores and need head_dim 128
 * and block_size 16 or 32; one query head per KV head runs on the CUDA cores.
 * Accumulation is fp32; out is rounded to nearest even.
 * Errors: KVP_ERR_INVALID (unsupported geometry, misaligned pointers,
 * workspace too small), KVP_ERR_CUDA (launch failure). */
KVP_API int paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                           int32_t partition_size, void* workspace, size_t workspace_bytes,
                           void* out, int32_t dtype, kvp_stream_t stream);

/* Bytes of device workspace paged_attention_decode_grouped needs for this
 * batch shape: 0 when partition_size <= 0 (the call then runs as
 * paged_attention_decode, unsplit); else room for num_seqs * num_q_heads *
 * (P + 1) partial slots of (head_dim + 2) fp32 values, P = ceil(max(
 * max_context_len, 1) / partition_size), plus the grouping plan (about
 * 84 bytes per sequence). Always at least kvp_decode_workspace_bytes(...). */
KVP_API size_t kvp_decode_grouped_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                          int32_t head_dim, int32_t max_context_len,
                                          int32_t partition_size);

/* Decode attention for batches whose sequences share cache blocks: the same
 * arguments and the same result (to fp32 rounding) as paged_attention_decode,
 * but each run of leading blocks that several sequences hold is read from HBM
 * once per subgroup of them instead of once per sequence.
 * Why: sequences forked from one parent (parallel samples of a prompt, beams)
 * share the physical blocks of their common prefix, stored once with a
 * reference count ["Your GPU was mostly empty", section "Paging's second gift:
 * copy-on-write"; "vLLM and PagedAttention", section on parallel sampling and
 * beam search]. The pages' decode kernel still reads a shared block once per
 * sequence that attends to it; this entry point, which the pages do not
 * describe, reads it once per subgroup.
 * How: a grouping plan (the rule is kv_decode_group_plan's) names subgroups of
 * up to M sequences (M = 8 for one query head per KV head, else 16 / G) and
 * each subgroup's shared prefix of c full blocks. The tensor-core kernel
 * attends, per KV head, with all the members' queries of a subgroup as the
 * columns of one contraction over the c shared blocks; each sequence's blocks
 * from c on go to the CUDA-core kernel (one query head per KV head) or to the
 * tensor-core kernel (grouped-query heads). Both ranges are split into
 * partitions of partition_size tokens and a log-sum-exp merge writes every
 * output row.
 * host_plan: NULL, and a one-CTA kernel builds the plan on the GPU; or the
 * plan kv_decode_group_plan built from these same block tables and lengths
 * (host memory, kvp_decode_group_plan_words(num_seqs) words). The kernels read
 * the plan from device memory: device_plan, a copy of host_plan that the
 * caller has placed there (for example uploaded together with its block
 * tables; 4-byte aligned, read-only to the call), or, when device_plan is
 * NULL, a copy the call makes into the workspace by cudaMemcpyAsync on
 * `stream` (pageable host memory may be reused once the call returns;
 * page-locked memory, whose copy runs in stream order, must stay unchanged
 * until the stream has reached this call). A call captured into a CUDA graph
 * needs device_plan, or a host_plan in page-locked memory that stays valid for
 * every replay: a copy from pageable memory cannot be captured.
 * device_plan without host_plan is rejected. A host
 * plan also lets the call give the tensor-core kernel only its share of the
 * SMs and run the CUDA-core kernel beside it. A plan from other tables gives
 * wrong results; one whose header does not fit the batch is rejected.
 * Needs head_dim 128, block_size 16 or 32, a group G = num_q_heads /
 * num_kv_heads with 16 / G >= 2 (G <= 8), partition_size > 0 and a multiple
 * of 128, and num_seqs <= 4096; other batches (and max_context_len == 0) are
 * decoded by paged_attention_decode with the same workspace (host_plan
 * ignored), so the call is valid for every batch paged_attention_decode
 * accepts.
 * workspace: device, >= kvp_decode_grouped_workspace_bytes(...) bytes,
 * 256-byte aligned, contents ignored. Errors: those of paged_attention_decode,
 * and KVP_ERR_INVALID for a host plan that does not fit. */
KVP_API int paged_attention_decode_grouped(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                           int32_t partition_size, const int32_t* host_plan,
                           const int32_t* device_plan, void* workspace, size_t workspace_bytes,
                           void* out, int32_t dtype, kvp_stream_t stream);

/* Words of the grouping plan of a batch of num_seqs sequences (0 if
 * num_seqs <= 0): 8 + num_seqs + (num_seqs / 2 + 1) * 20. */
KVP_API size_t kvp_decode_group_plan_words(int32_t num_seqs);

/* Builds on the host the grouping plan of paged_attention_decode_grouped
 * from host copies of the batch's block tables ([num_seqs][max_blocks_per_seq])
 * and context lengths (clamped to [0, max_context_len]). Rule: a sequence
 * whose context holds a full block and whose first table entry is a valid id
 * is keyed by that id; sorted by (key, sequence index), each run of equal keys
 * is cut in order into subgroups of up to M members (M as above, from
 * num_q_heads / num_kv_heads; a subgroup of one is dropped); a subgroup's
 * shared prefix c is the number of leading entries equal across its members,
 * capped at every member's full blocks. Layout of `plan` (int32 words):
 * [0] subgroups, [1] most partitions of a shared prefix, [2] most partitions
 * of a sequence's own range (from block c on), [3] sum of c over subgroups,
 * [4] blocks of all own ranges, [5..8) zero; [8, 8 + num_seqs) c of each
 * sequence's subgroup (0 if none); then per subgroup 20 words {c, members,
 * 0, 0, member indices [16]}. The GPU plan kernel builds the same words.
 * num_seqs in [1, 4096]; plan_words >= kvp_decode_group_plan_words(num_seqs).
 * Errors: KVP_ERR_INVALID. */
KVP_API int kv_decode_group_plan(const int32_t* block_tables, const int32_t* context_lens,
                         int32_t num_seqs, int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t block_size, int32_t partition_size, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t num_blocks, int32_t* plan,
                         size_t plan_words);

/* ---- packed grouped decode ------------------------------------------------
 * Decode attention for batches whose sequences share cache blocks (forked
 * samples, beams), reading every block once per group of the sequences that
 * hold it ["Your GPU was mostly empty", section "Paging's second gift:
 * copy-on-write": forked sequences share their common blocks]; the pages'
 * decode reads a shared block once per sequence, and this entry point, which
 * the pages do not describe, is an optimisation of the same result. Groups
 * follow kv_decode_group_plan's rule; a sequence in no subgroup is a group of
 * one. Each group's blocks form one stream - the shared prefix, then each
 * member's own blocks - cut into chunks of 512 tokens; one persistent
 * tensor-core kernel takes the chunks (longest first) with the members' query
 * heads as the columns of the contraction, a column counting only the tokens
 * of its member's blocks, and a log-sum-exp merge writes every output row.
 * Unlike paged_attention_decode_grouped (two kernels: shared prefixes on the
 * tensor cores, own ranges on the CUDA cores), short own ranges share key tiles
 * with other members and the shared prefix, so no kernel pays a sequence's
 * dependent loads alone. */

/* Words a packed plan of num_seqs sequences with up to max_blocks_per_seq
 * blocks each may take (an upper bound; 0 for non-positive sizes). */
KVP_API size_t kvp_decode_pack_plan_words(int32_t num_seqs, int32_t max_blocks_per_seq);

/* Builds on the host the packed plan of a batch from host copies of its block
 * tables ([num_seqs][max_blocks_per_seq]) and context lengths (clamped to
 * [0, max_context_len]). Layout (int32 words): [0] groups, [1] units per KV
 * head, [2] entries, [3] most chunks of any group, [4] block size, [5] blocks
 * per chunk (512 / block_size), [6] offset of the unit table, [7] offset of
 * the entries; [8, 8 + S) each sequence's group; per group 20 words {first
 * entry, members, entries, chunks, member sequences [16]}; per unit 4 words
 * {group, first entry, entries, chunk}, longest first; per entry 2 words
 * {block id, column mask << 8 | valid tokens of the block}. Column j of a group
 * is query head g * G + j % G of member j / G.
 * Needs block_size 16 or 32, num_seqs in [1, 4096], at most 16 query heads
 * per KV head, plan_words >= kvp_decode_pack_plan_words(...). Errors:
 * KVP_ERR_INVALID. */
KVP_API int kv_decode_pack_plan(const int32_t* block_tables, const int32_t* context_lens,
                                int32_t num_seqs, int32_t max_blocks_per_seq,
                                int32_t max_context_len, int32_t block_size, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t num_blocks, int32_t* plan,
                                size_t plan_words);

/* Bytes of device workspace paged_attention_decode_packed needs for this
 * host plan: per (sequence, query head) one partial slot of head_dim + 2 fp32
 * values per chunk of the longest group stream, plus room for a copy of the
 * plan. 0 for a NULL plan or non-positive sizes. */
KVP_API size_t kvp_decode_packed_workspace_bytes(const int32_t* host_plan, int32_t num_seqs,
                                                 int32_t num_q_heads, int32_t head_dim);

/* The packed grouped decode: the result of paged_attention_decode (to fp32
 * rounding) for the batch the plan was built from. host_plan (required) is
 * kv_decode_pack_plan's plan of these sequences, checked word by word against
 * the batch (KVP_ERR_INVALID if its shape does not fit); the kernels read it
 * from device_plan, a copy the caller placed in device memory (4-byte aligned,
 * read-only to the call), or, when device_plan is NULL, from a copy the call
 * makes into the workspace by cudaMemcpyAsync on `stream` (see
 * paged_attention_decode_grouped for host memory and graph capture). The block
 * ids are the plan's: the device block tables are not read. context_lens:
 * device int32 [num_seqs]. Needs head_dim 128, block_size 16 or 32, at most 16
 * query heads per KV head. workspace: >= kvp_decode_packed_workspace_bytes(...),
 * 256-byte aligned. Errors: those of paged_attention_decode. */
KVP_API int paged_attention_decode_packed(const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* context_lens, int32_t num_seqs,
                                          int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                          int32_t max_context_len, float scale,
                                          const int32_t* host_plan, const int32_t* device_plan,
                                          void* workspace, size_t workspace_bytes, void* out,
                                          int32_t dtype, kvp_stream_t stream);

/* Bytes of device workspace paged_attention_prefill needs: that of
 * paged_attention_decode for num_seqs * q_len rows (0 if q_len <= 0). */
KVP_API size_t kvp_prefill_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                   int32_t head_dim, int32_t max_context_len,
                                   int32_t partition_size);

/* Attention of a chunk of q_len new tokens per sequence over the paged cache,
 * causal within the chunk: the prefill of a prompt (or of a chunk of it)
 * whose keys and values reshape_and_cache has already written to the
 * sequence's blocks ["PagedAttention: KV cache memory management", section "A
 * request lifecycle": prefill creates the cache state through the block
 * table]. context_lens[s] counts the chunk; query i of sequence s sits at
 * position ctx_s - q_len + i and attends to the tokens j <= ctx_s - q_len + i
 * (a query with none gives a zero row):
 *   out[s][i][h] = sum_j softmax_j(scale * q[s][i][h] . key j) * value j.
 * q, out: device [num_seqs][q_len][num_q_heads][head_dim]; the other arguments
 * as for paged_attention_decode (context_lens[s] <= max_context_len).
 * q_len == 1 is paged_attention_decode. Longer chunks run on the tensor
 * cores, up to 16 / G queries of every sequence per launch (G = num_q_heads /
 * num_kv_heads), each launch reading the sequences' keys and values once, so
 * a whole prompt of T tokens reads them ceil(T * G / 16) times; needs head_dim
 * 128, block_size 16 or 32, G <= 16, partition_size a multiple of 128 (or 0).
 * workspace: >= kvp_prefill_workspace_bytes(...) bytes, 256-byte aligned.
 * Errors: those of paged_attention_decode. */
KVP_API int paged_attention_prefill(const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens,
                            int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int32_t num_blocks, int32_t max_blocks_per_seq,
                            int32_t max_context_len, float scale, int32_t partition_size,
                            void* workspace, size_t workspace_bytes, void* out, int32_t dtype,
                            kvp_stream_t stream);

/* ---- FP8 (E4M3) KV cache ------------------------------------------------
 * Cached keys and values as E4M3 codes, one byte per element, with one fp32
 * scale per KV head for K and one for V: code c of KV head g stands for
 * value(c) * scale[g]. Quantisation keeps the cached state in a
 * lower-precision representation, and it combines with paging, which only
 * decides where the blocks live ["PagedAttention: KV cache memory
 * management", section "PagedAttention vs KV-cache quantization vs prefix
 * caching"]. The pool layout is that of the 16-bit cache with 1-byte
 * elements: [num_blocks][num_kv_heads][block_size][head_dim]. copy_blocks
 * copies its blocks with dtype KVP_FP8_E4M3. */

/* reshape_and_cache into an E4M3 cache: element x of KV head h of token t is
 * stored at slot slot_mapping[t] as the code of x / k_scale[h] (values: of
 * x / v_scale[h]), the division correctly rounded in fp32, the quotient
 * rounded to the nearest E4M3 value (ties to even) and saturated to +-448;
 * a negative slot is skipped, a slot past the pool is skipped and recorded
 * (KVP_ERR_BOUNDS from kvp_check_device_error).
 * k_new, v_new: device [num_tokens][num_kv_heads][head_dim] of dtype
 * (KVP_F16 or KVP_BF16), 16-byte aligned; k_cache, v_cache: device uint8
 * pools; slot_mapping: device int64 [num_tokens]; k_scale, v_scale: device
 * fp32 [num_kv_heads]. head_dim / 16 and block_size must be powers of two.
 * Errors: KVP_ERR_INVALID (sizes, dtype, NULL or misaligned pointers). */
KVP_API int reshape_and_cache_fp8(const void* k_new, const void* v_new, void* k_cache,
                                  void* v_cache, const int64_t* slot_mapping, const float* k_scale,
                                  const float* v_scale, int32_t num_tokens, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  int32_t dtype, kvp_stream_t stream);

/* paged_attention_decode over an E4M3 cache: key j of KV head g is
 * value(code) * k_scale[g] and value j is value(code) * v_scale[g]; the
 * output is the softmax-weighted sum as in paged_attention_decode. q and out
 * are of dtype (KVP_F16 or KVP_BF16); the other arguments, the workspace
 * (kvp_decode_workspace_bytes) and the errors are those of
 * paged_attention_decode. Runs on the CUDA cores for every query head (any
 * num_q_heads / num_kv_heads); needs head_dim 128. */
KVP_API int paged_attention_decode_fp8(const void* q, const void* k_cache, const void* v_cache,
                                       const float* k_scale, const float* v_scale,
                                       const int32_t* block_tables, const int32_t* context_lens,
                                       int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                       int32_t max_blocks_per_seq, int32_t max_context_len,
                                       float scale, int32_t partition_size, void* workspace,
                                       size_t workspace_bytes, void* out, int32_t dtype,
                                       kvp_stream_t stream);

/* ---- virtually contiguous KV cache (CUDA virtual memory management) --------
 * The alternative the pages name to block tables: keep each sequence's cache
 * contiguous in virtual memory and back it with physical pages on demand
 * through CUDA's virtual memory management, so the attention kernel computes
 * addresses instead of dereferencing a block table ["Your GPU was mostly
 * empty", section "The tradeoff: you just wrote a virtual memory subsystem in
 * userspace": translation in the kernel (block tables) or in CUDA's VMM].
 * Here it serves as an A/B of the block table's translation cost: the same
 * decode kernels, tiles and math, with the address of a tile computed from
 * (slot, token) instead of looked up.
 *
 * A cache has num_slots sequence slots of up to max_tokens tokens. Each slot
 * is one reserved virtual range per cache (K, V), token-major:
 *   K of token j of slot s, KV head g = k_base[((s * slot_tokens + j) *
 *   num_kv_heads + g) * head_dim .. + head_dim)
 * (slot_tokens from kv_vcache_layout: >= max_tokens plus a mapped tail, a whole
 * number of physical chunks). Physical chunks (the device's allocation
 * granularity, 2 MiB on B200) are mapped at the end of a slot's range as its
 * capacity grows (kv_vcache_reserve) and unmapped only by kv_vcache_trim; a
 * finished request's slot keeps its chunks for the next request. A slot's
 * capacity is the tokens the kernels may touch; at least 256 more tokens are
 * always mapped past it, so no kernel tile that starts inside the capacity
 * reaches unmapped memory, and the kernels clamp every context length to the
 * capacity of its slot (device copy, updated in stream order). Only head_dim
 * 128 and 16-bit elements; one device (the current one at creation). Host
 * calls are not thread-safe per cache. */
typedef struct kvp_vcache kvp_vcache;

typedef struct kvp_vcache_stats {
  int64_t chunk_bytes;     /* physical mapping granularity                 */
  int64_t mapped_chunks;   /* chunks mapped now, K and V together          */
  int64_t spare_chunks;    /* unmapped chunks kept for reuse               */
  int64_t mapped_bytes;    /* mapped_chunks * chunk_bytes                  */
  int64_t reserved_bytes;  /* virtual bytes reserved, K and V together     */
  int64_t map_calls;       /* chunk mappings made since creation           */
  int64_t create_calls;    /* physical chunks created since creation       */
  int64_t slot_tokens;     /* token stride between slots                   */
} kvp_vcache_stats;

/* Reserves the virtual ranges of a cache of num_slots slots of up to
 * max_tokens tokens of num_kv_heads x head_dim elements of dtype (KVP_F16 or
 * KVP_BF16; head_dim 128) on the current device; no physical memory is mapped
 * yet (every capacity is 0). Errors: KVP_ERR_INVALID (sizes, dtype, more than
 * 2^31 tokens in all), KVP_ERR_CUDA (VMM unavailable, reservation failed),
 * KVP_ERR_OOM. */
KVP_API int kv_vcache_create(int32_t num_slots, int32_t max_tokens, int32_t num_kv_heads,
                             int32_t head_dim, int32_t dtype, kvp_vcache** out);

/* Synchronises the device, unmaps and frees every chunk, releases the
 * reservations. NULL is accepted. */
KVP_API int kv_vcache_destroy(kvp_vcache* vc);

/* Grows the capacity of `slot` to at least `tokens` (<= max_tokens) by mapping
 * chunks at the end of its range; the device copy of the capacity is updated
 * by a one-thread kernel on `stream`, so kernels launched after this call on
 * that stream see it. No-op if the capacity suffices. On failure (KVP_ERR_OOM
 * when the device has no memory for a chunk, KVP_ERR_CUDA) the call's own
 * mappings are undone and nothing changes. */
KVP_API int kv_vcache_reserve(kvp_vcache* vc, int32_t slot, int32_t tokens, kvp_stream_t stream);

/* kv_vcache_reserve for n slots (host int32 arrays slots[n], tokens[n]), in
 * order, as one call: a decode step's growth of the whole batch. All or
 * nothing: if one slot cannot grow, the slots the call grew before it are
 * returned to their earlier capacity (their chunks kept as spares). */
KVP_API int kv_vcache_reserve_batch(kvp_vcache* vc, const int32_t* slots, const int32_t* tokens,
                                    int32_t n, kvp_stream_t stream);

/* Shrinks the capacity of `slot` to what `tokens` needs: the capacity drops on
 * `stream`, the whole device is synchronised (no kernel may still read the
 * chunks), then the chunks past it are unmapped and kept as spares for later
 * reserves. tokens == 0 unmaps the slot entirely. */
KVP_API int kv_vcache_trim(kvp_vcache* vc, int32_t slot, int32_t tokens, kvp_stream_t stream);

/* Returns the spare chunks to the driver. */
KVP_API int kv_vcache_release_spares(kvp_vcache* vc);

/* Capacity (tokens) of `slot`. */
KVP_API int kv_vcache_capacity(const kvp_vcache* vc, int32_t slot, int32_t* tokens);

/* Base device addresses of the K and V ranges and the token stride between
 * slots (see the layout above). Only the mapped part of a slot
 * (kv_vcache_capacity tokens) may be read or written. */
KVP_API int kv_vcache_layout(const kvp_vcache* vc, void** k_base, void** v_base,
                             int32_t* slot_tokens);

/* Counters (see kvp_vcache_stats). */
KVP_API int kv_vcache_stats(const kvp_vcache* vc, kvp_vcache_stats* out);

/* reshape_and_cache into a virtually contiguous cache: for t < num_tokens,
 * token t's keys and values (k_new, v_new: device [num_tokens][num_kv_heads]
 * [head_dim] of the cache's dtype, 16-byte aligned) go to position
 * positions[t] of slot slots[t] (device int32 arrays). A negative slot is
 * padding and skipped; a slot >= num_slots or a position outside [0, capacity)
 * is skipped and recorded (KVP_ERR_BOUNDS from kvp_check_device_error), so no
 * write reaches unmapped memory. Errors: KVP_ERR_INVALID. */
KVP_API int reshape_and_cache_vcache(const void* k_new, const void* v_new, kvp_vcache* vc,
                                     const int32_t* slots, const int32_t* positions,
                                     int32_t num_tokens, kvp_stream_t stream);

/* paged_attention_decode over a virtually contiguous cache: sequence s reads
 * slot seq_slots[s] (device int32 [num_seqs]) through context_lens[s] tokens,
 * each clamped to max_context_len and to the slot's capacity (a length or a
 * slot out of range is recorded; an invalid slot reads nothing). Same result
 * as paged_attention_decode with the block table of the slot's tokens. q, out
 * [num_seqs][num_q_heads][head_dim] of the cache's dtype; num_q_heads a
 * multiple of the cache's num_kv_heads (grouped-query heads, G <= 16, run on
 * the tensor cores and need partition_size % 128 == 0); partition_size and
 * workspace as for paged_attention_decode (kvp_decode_workspace_bytes). One
 * query head per KV head reads 16-token tiles, grouped-query heads 128-token
 * tiles, each one TMA load per tile (per 64-dim half for the keys).
 * Errors: those of paged_attention_decode. */
KVP_API int attention_decode_vcache(const void* q, const kvp_vcache* vc, const int32_t* seq_slots,
                                    const int32_t* context_lens, int32_t num_seqs,
                                    int32_t num_q_heads, int32_t max_context_len, float scale,
                                    int32_t partition_size, void* workspace,
                                    size_t workspace_bytes, void* out, kvp_stream_t stream);

/* Largest split-context scratch, in bytes, that paged_attention_decode_noalloc
 * can serve from its built-in area (40 MiB). */
#define KVP_STATIC_SCRATCH_BYTES (40u * 1024u * 1024u)

/* paged_attention_decode without a workspace argument, for callers that cannot
 * allocate device memory: for example a serving engine whose allocator has
 * already reserved all free device memory for its KV pool, or a latency-
 * critical path that cannot afford cudaMalloc's implicit synchronisation. The
 * paper has no counterpart to this entry point; it is a convenience of this
 * library.
 * The split-context scratch lives in one static device array of
 * KVP_STATIC_SCRATCH_BYTES inside the library; every GPU that loads the
 * library holds that memory until the process exits. The call allocates
 * nothing: inputs and outputs are the caller's, as for
 * paged_attention_decode, and the arguments and results are the same.
 * The first call on a device looks up the array's device address on that
 * device (with it current), and so does the first call after the device's
 * context changes (cudaDeviceReset, or a thread bound to another context);
 * make those calls before any stream capture: a lookup while `stream` is
 * capturing is refused with KVP_ERR_INVALID.
 * All calls share the one array and it keeps the last call's contents;
 * nothing in it needs to start at zero (each call writes every partial it
 * later reads), but calls whose kernels overlap on the GPU (different streams,
 * or several host threads) race on it and must be serialised by the caller.
 * Errors: those of paged_attention_decode, and KVP_ERR_INVALID when the batch
 * needs more scratch than KVP_STATIC_SCRATCH_BYTES (kvp_decode_workspace_bytes
 * gives the need; the message states both sizes). */
KVP_API int paged_attention_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, const int32_t* context_lens,
                           int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           int32_t max_blocks_per_seq, int32_t max_context_len, float scale,
                           int32_t partition_size, void* out, int32_t dtype,
                           kvp_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: KVP_OK, or KVP_ERR_BOUNDS if a kernel skipped an
 * out-of-range index since the last check (the message names the first). */
KVP_API int kvp_check_device_error(kvp_stream_t stream);

/* Diagnostic of the kernels' bounded waits: launches one CTA that waits, with
 * the same bounded-wait code the decode kernels use but a limit of limit_ms
 * (1..2000), for an mbarrier phase that nothing ever completes. The wait runs
 * out, records a timeout in the device error word and the kernel returns; the
 * next kvp_check_device_error() reports KVP_ERR_CUDA ("bounded wait timed
 * out"), and the context stays usable. Asynchronous like the other device
 * calls. */
KVP_API int kvp_selftest_bounded_wait(int32_t limit_ms, kvp_stream_t stream);

/* Description of the calling thread's last failure ("" if none). */
KVP_API const char* kvp_last_error_message(void);

/* Library version string. */
KVP_API const char* kvp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVP_H_ */
