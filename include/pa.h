/*
 * pa.h - C ABI of libpa.so, a B200 (sm_100a) implementation of the PagedAttention
 * decode path: paged decode attention, the slot-mapped KV append, the
 * copy-on-write block copy, and the host block allocator that feeds them.
 *
 * Sources, by page title and section:
 *  [FSAH] "PagedAttention Paper Breakdown: Virtual Memory Allocation for LLM KV
 *         Cache Serving" (fullstackaihub.com).  Section 2 "Virtual Memory Paging &
 *         Block Table Architecture", Address Translation Formula: for logical token
 *         i, b = floor(i/B), o = i mod B, PhysicalAddr(K_i) = T[b]*B + o (a token
 *         slot).  Section 3 "Dynamic Copy-on-Write (CoW) Parallel Sampling".
 *  [INIT] "PagedAttention and vLLM Architecture: Virtual Memory for LLM Serving"
 *         (initnode.dev).  Section 1 "Logical vs Physical Blocks" (fixed pool of
 *         B-token pages allocated at startup, per-request block table kept by the
 *         engine); "Why Internal Fragmentation is Bounded" (a block is taken only
 *         when a token overflows the last one); section 2 "PagedAttention Attention
 *         CUDA Kernel Mechanics" (the kernel takes q and the block table, walks the
 *         physical blocks in table order, dots q with each key, and fuses an online
 *         softmax across blocks with the product by the V blocks); section 3
 *         "Copy-on-Write (CoW) for Parallel Sampling & Beam Search" (shared blocks
 *         carry a reference count; writing into a shared block copies it to a new
 *         block from the free pool, drops the old count and repoints one table).
 *
 * Conventions for every call:
 *  - Tensors are dense and row-major.  Device calls take DEVICE pointers to
 *    caller-owned memory; the library never allocates device memory and keeps no
 *    pointer after a call returns.  pa_alloc_* calls take HOST pointers.
 *  - KV pools: k_cache and v_cache are [num_blocks][num_kv_heads][block_size][head_dim]
 *    of the call's dtype.  Token slot t lives in physical block t / block_size at
 *    offset t % block_size.
 *  - Supported: head_dim in {64, 128}; block_size in {16, 32}; num_heads a multiple
 *    of num_kv_heads with a group of 1, 2, 4 or 8 query heads per kv head;
 *    dtype fp32 or bf16 (q, out and both pools share it).  Other values return
 *    PA_ERR_UNSUPPORTED.  Device pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Device calls are
 *    asynchronous: they validate their host-side arguments, launch, and return.
 *    Launch failures return PA_ERR_CUDA.  Checks that need device data (block
 *    indices, context lengths, slots, copy pairs) are made by the kernels, which
 *    skip the offending access and raise a flag read by pa_device_status().
 *  - Errors never abort or throw; pa_last_error_string() describes the last one
 *    on the calling thread.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

/* Symbols exported from the shared library; everything else stays hidden. */
#if defined(PA_BUILDING_LIBRARY) && defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID = -1,       /* bad argument (null pointer, bad size, misalignment, unknown id) */
    PA_ERR_UNSUPPORTED = -2,   /* shape or dtype outside the supported set above */
    PA_ERR_OOM = -3,           /* allocator: free pool exhausted (allocator state unchanged) */
    PA_ERR_CUDA = -4,          /* a CUDA runtime call failed */
    PA_ERR_DEVICE_CHECK = -5   /* a kernel flagged bad device data (see pa_device_status) */
} pa_status;

typedef enum { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1 } pa_dtype;

/* Bits of the device status word (pa_device_status). */
#define PA_DEV_BAD_BLOCK     1u   /* a block-table entry outside [0, num_blocks) was read */
#define PA_DEV_BAD_CONTEXT   2u   /* a context length < 0, > max_context_len or > max_blocks_per_seq*B */
#define PA_DEV_BAD_SLOT      4u   /* a slot_mapping entry >= num_blocks*block_size */
#define PA_DEV_BAD_PAIR      8u   /* a block_mapping entry outside [0, num_blocks) */
#define PA_DEV_WAIT_TIMEOUT 16u   /* a pipeline wait inside a kernel gave up (bounded wait) */

/* ------------------------------------------------------------------ decode */

/*
 * Context-partition length (tokens) that pa_decode uses for these arguments:
 * `partition_size` itself when > 0 (it must be a multiple of block_size, at most
 * 4096), else the shortest length of the automatic choice (512), which the call may
 * lengthen by doubling, up to 4096, from the batch's size and context lengths (the
 * workspace sized for the shortest length serves every longer one).  A sequence
 * longer than one partition is split into partitions whose softmax states are merged
 * by log-sum-exp in a second kernel.  Returns a negative pa_status on invalid
 * arguments.
 */
PA_API int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                             int max_context_len, int partition_size);

/*
 * Bytes of device workspace pa_decode needs for these arguments (> 0 whenever
 * num_seqs > 0).  The workspace holds the call's work plan (the (sequence,
 * partition) pairs, longest first, and a work counter) and, when a sequence can
 * span more than one partition, per (sequence, query head, partition) the running
 * max, the softmax sum and the unnormalised head_dim-vector of the partition.
 */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_context_len, int partition_size);

/*
 * Paged decode attention ([INIT] section 2; translation per [FSAH] section 2).
 *   out[s][h][:] = sum_i softmax_i(scale * q[s][h] . K_i) V_i
 * over the logical tokens i < context_lens[s] of sequence s, where K_i and V_i are
 * read from physical block block_tables[s][i / block_size], offset
 * i % block_size, kv head h / (num_heads / num_kv_heads).  Accumulation is fp32;
 * out is written in `dtype`.  context_lens[s] == 0 gives a zero row.
 *   out           [num_seqs][num_heads][head_dim]            (device, written)
 *   q             [num_seqs][num_heads][head_dim]            (device)
 *   k_cache/v_cache pools as above                           (device)
 *   block_tables  [num_seqs][max_blocks_per_seq] int32       (device); entries past
 *                 ceil(context_lens[s]/block_size) are never read
 *   context_lens  [num_seqs] int32                           (device), each in
 *                 [0, min(max_context_len, max_blocks_per_seq*block_size)]
 *   max_context_len  host-side upper bound of context_lens (sizes the launch)
 *   partition_size   0 = automatic, else tokens per context partition
 *   workspace     device scratch of at least pa_decode_workspace_size() bytes,
 *                 16-byte aligned; its contents are overwritten (no initial
 *                 contents are needed).  Calls that share a workspace must be
 *                 ordered on one stream.
 */
PA_API pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
                    int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                    int max_context_len, float scale, int partition_size, void* workspace,
                    size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * pa_decode in two parts, for a decode step that runs the attention of many layers
 * over the same sequences (the same block_tables, context_lens and sizes; other q,
 * out and caches per layer).  pa_decode_plan writes the work plan into the workspace
 * (the plan kernel only; no q, out or caches); pa_decode_run then runs the decode
 * from that plan and may be called any number of times: the last CTA of each run to
 * stop taking work (at the end of the work list, or on a wait that gave up) resets
 * the plan's work counter.  A run must use the workspace, block_tables,
 * context_lens and every size argument of its plan (the caller's promise; nothing
 * checks it), and follow it in stream order.  A run on a workspace that holds no plan
 * reads whatever the workspace holds: undefined.  A run that raised a device status
 * bit (pa_device_status) left some outputs unwritten; planning again before the next
 * run is the safe course.  pa_decode is the plan followed by one run.  Errors as for
 * pa_decode.
 */
PA_API pa_status pa_decode_plan(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                                int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                                int num_blocks, int max_context_len, int partition_size, void* workspace,
                                size_t workspace_bytes, pa_dtype dtype, void* stream);
PA_API pa_status pa_decode_run(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads,
                               int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                               int max_context_len, float scale, int partition_size, void* workspace,
                               size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * Fixed size of the library's own decode workspace used by
 * pa_decode_static_workspace: 16 MiB of device memory on every GPU that loads
 * the library, held until the process exits.
 */
#define PA_STATIC_WORKSPACE_BYTES (16u * 1024u * 1024u)

/*
 * pa_decode without a caller workspace, for callers that cannot allocate device
 * memory: for example a plugin or script host that only hands out pointers to
 * tensors it already owns, or a process whose memory pool must not be bypassed.
 * The pages describe no such call (no counterpart there); it exists for these
 * callers only.  Arguments, layouts and results are those of pa_decode; the
 * workspace is a fixed array in the library (PA_STATIC_WORKSPACE_BYTES).
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *  - The first call made on a device resolves that device's array address
 *    (cudaGetSymbolAddress); make that first call before any stream capture.
 *    After a device reset (cudaDeviceReset) the next call resolves it again, so
 *    that call too belongs before any capture.
 *  - Arguments whose pa_decode_workspace_size() exceeds
 *    PA_STATIC_WORKSPACE_BYTES return PA_ERR_UNSUPPORTED before any device work
 *    (a larger partition_size needs less).
 *  - All calls on a device share one array, which keeps the last call's
 *    contents; no part of it needs to start at zero (every call writes what it
 *    later reads).  Calls that may run at the same time on one device (for
 *    example on two unordered streams) race on it: order them on one stream.
 */
PA_API pa_status pa_decode_static_workspace(void* out, const void* q, const void* k_cache, const void* v_cache,
                                            const int32_t* block_tables, const int32_t* context_lens,
                                            int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                            int block_size, int max_blocks_per_seq, int num_blocks,
                                            int max_context_len, float scale, int partition_size,
                                            pa_dtype dtype, void* stream);

/* ------------------------------------------------------------------ KV append */

/*
 * Slot-mapped KV append: for each token t < num_tokens with slot = slot_mapping[t]
 * >= 0, k_cache[slot / block_size][h][slot % block_size][:] = key[t][h][:] and the
 * same for value/v_cache, for every kv head h.  slot = T[b]*B + o is the [FSAH]
 * section 2 address of the token's position.  Negative slots are padding and
 * are skipped.  The copy is bit-exact.  Slots must be distinct (otherwise the
 * surviving row is unspecified).
 *   key, value    [num_tokens][num_kv_heads][head_dim]  (device)
 *   slot_mapping  [num_tokens] int64                    (device)
 */
PA_API pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                               const int64_t* slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                               int block_size, int num_blocks, pa_dtype dtype, void* stream);

/* ------------------------------------------------------------------ CoW copy */

/*
 * Copy-on-write block copy ([INIT] section 3): for each pair i,
 * block block_mapping[2i+1] of both pools becomes a bit-exact copy of block
 * block_mapping[2i] (all kv heads, all block_size slots).  No destination may
 * also be a source or appear twice in one call (pairs run concurrently); the
 * allocator's copy-on-write pairs always satisfy this.
 *   block_mapping [num_pairs][2] int64 (src, dst)   (device)
 */
PA_API pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int num_pairs,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, pa_dtype dtype,
                         void* stream);

/*
 * Optional host-side checks of the two mappings whose misuse the kernels cannot make
 * safe: pairs and slots are handled concurrently, so a repeated destination (or a
 * destination that is also a source) leaves a result that depends on thread order.
 * Both take HOST arrays, touch no device, change nothing and return PA_OK or
 * PA_ERR_INVALID (the first offending index in pa_last_error_string()).
 *   pa_check_block_mapping: block_mapping [num_pairs][2] int64 (src, dst) as for
 *     pa_copy_blocks; invalid if an entry is outside [0, num_blocks), a destination
 *     appears twice, or a destination is also a source.
 *   pa_check_slot_mapping: slot_mapping [num_tokens] int64 as for
 *     pa_reshape_and_cache; invalid if a slot >= 0 appears twice or is past the pool
 *     (num_blocks * block_size); negative slots (padding) are ignored.
 * A null array with a count of 0 is valid.
 */
PA_API pa_status pa_check_block_mapping(const int64_t* block_mapping, int num_pairs, int num_blocks);
PA_API pa_status pa_check_slot_mapping(const int64_t* slot_mapping, int num_tokens, int num_blocks, int block_size);

/* ------------------------------------------------------------------ device status */

/*
 * Waits for `stream`, then returns in *flags the PA_DEV_* bits raised by kernels
 * on the current device since the last call, and clears them.  Returns PA_OK,
 * or PA_ERR_CUDA if the wait or the read failed.
 */
PA_API pa_status pa_device_status(uint32_t* flags, void* stream);

/*
 * Failure-path self-test (no counterpart in the pages; it exercises the library's
 * own failure detection).  Launches one thread that waits, with the kernels' bounded
 * wait and time limit (2 s), on an mbarrier nothing ever arrives at.  The wait gives
 * up, PA_DEV_WAIT_TIMEOUT is raised in the status word (read it with
 * pa_device_status) and the kernel returns; nothing faults or hangs, and the context
 * stays usable.  Blocks until done; *waited_ns (nullable, host) receives how long the
 * wait lasted on the device clock.
 */
PA_API pa_status pa_selftest_bounded_wait(uint64_t* waited_ns, void* stream);

/*
 * Chunked prefill over the paged cache ([INIT] section 3: a prompt's blocks are
 * assigned when it is processed; [FSAH] section 2: token t of a sequence lives at
 * slot T[t / B] * B + t % B), on the tensor cores.  Sequence s holds
 * context_lens[s] tokens in the pools, its new tokens already appended (as for
 * pa_decode); its last n_s = q_start[s+1] - q_start[s] tokens are the queries:
 * q rows q_start[s] .. q_start[s+1]-1 of q [num_query_tokens][num_heads][head_dim],
 * query i at position context_lens[s] - n_s + i.  Each attends causally to tokens
 * 0..its position: out[row][h] = softmax_t(scale * q[row][h] . K_t) . V_t over
 * t <= position, with query head h reading kv head h / (num_heads / num_kv_heads).
 * q_start (device, int32, S+1 entries, non-decreasing, within [0, num_query_tokens])
 * and context_lens are device arrays; max_query_len bounds every n_s (it sizes the
 * grid).  The kernel checks each sequence's device data before any store: a
 * sequence whose rows leave [0, num_query_tokens) or run backwards (q_start[s] < 0,
 * q_start[s+1] > num_query_tokens, q_start[s+1] < q_start[s]), with
 * n_s > max_query_len, n_s > context_lens[s], or a context beyond its table row
 * raises PA_DEV_BAD_CONTEXT and is skipped whole (its output rows untouched).  bf16 only,
 * head_dim 128, num_heads / num_kv_heads in {1, 2, 4, 8} (else PA_ERR_UNSUPPORTED).
 * With every n_s = 1 this is pa_decode.  No workspace: the grid has one CTA per work
 * item (pa_prefill_ws below is the faster form).  Asynchronous on stream.
 */
PA_API pa_status pa_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, const int32_t* context_lens, const int32_t* q_start,
                            int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int num_blocks, int num_query_tokens, int max_query_len,
                            float scale, pa_dtype dtype, void* stream);

/* Bytes of device workspace pa_prefill_ws needs (a fixed size). */
PA_API size_t pa_prefill_workspace_size(void);

/*
 * pa_prefill with a workspace: the same computation, arguments and checks, run by a
 * grid of one CTA per SM that hands out the (sequence, kv head, query-tile pair) work
 * items from a counter in the workspace, longest first, so that a CTA which finishes
 * early takes more and each CTA's next item starts while its last one ends.
 *   workspace  device scratch of at least pa_prefill_workspace_size() bytes, 16-byte
 *              aligned; no initial contents are needed (the call zeroes its counter on
 *              `stream` first).  Calls that share a workspace must be ordered on one
 *              stream.
 * A null or short workspace returns PA_ERR_INVALID.  Asynchronous on stream.
 */
PA_API pa_status pa_prefill_ws(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, const int32_t* context_lens, const int32_t* q_start,
                               int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int num_blocks, int num_query_tokens, int max_query_len,
                               float scale, void* workspace, size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * Whole-block copies from one pool to another ([FSAH] "Engineering Limitations":
 * CPU-GPU block swapping under memory pressure): for each (src, dst) pair in
 * block_mapping[num_pairs][2] (int64), block src of src_k_cache / src_v_cache
 * ([num_src_blocks][Hkv][B][D]) is copied to block dst of dst_k_cache / dst_v_cache
 * ([num_dst_blocks][Hkv][B][D]).  Each pool, and block_mapping, may be device memory
 * or pinned (page-locked) host memory, which the kernel reads or writes over PCIe
 * through its device mapping; pageable host memory is refused (PA_ERR_INVALID).
 * Pairs must not write one destination twice or read a block another pair writes.
 * Out-of-range pairs raise PA_DEV_BAD_PAIR and are skipped.  Asynchronous on stream;
 * the host side must stay allocated (and unread, for a swap-out) until the stream
 * reaches the copy.
 */
PA_API pa_status pa_swap_blocks(void* dst_k_cache, void* dst_v_cache, const void* src_k_cache,
                                const void* src_v_cache, const int64_t* block_mapping, int num_pairs,
                                int num_kv_heads, int head_dim, int block_size, int num_src_blocks,
                                int num_dst_blocks, pa_dtype dtype, void* stream);

/* ------------------------------------------------------------------ block allocator */

/*
 * Host block allocator with reference-counted copy-on-write ([INIT] sections 1
 * and 3, "Why Internal Fragmentation is Bounded"; [FSAH] sections 2 and 3) and a
 * prefix cache ([FSAH] "Paper Methods": shared prefix caching in a radix tree).
 * It owns only host memory.  The free pool is a FIFO queue initialised from
 * free_order (a permutation of 0..num_blocks-1; NULL = ascending); blocks freed
 * later join its tail.  A handle is not thread-safe.  On every error the
 * allocator state is left unchanged.
 *
 * Prefix cache: prompts added with pa_alloc_add_seq_cached build a tree whose
 * nodes are full blocks (edge = the block's B token ids, parent = the block before
 * it).  An unreferenced cached block stays in the tree until a block is needed and
 * the free queue is empty; then the one released longest ago among those with no
 * cached children is evicted and reused.  Every call that takes blocks can evict.
 */
typedef struct pa_allocator pa_allocator;

typedef struct {
    int64_t num_blocks;
    int64_t num_free;
    int64_t num_seqs;
    int64_t shared_blocks;     /* blocks with reference count > 1 */
    int64_t cow_copies;        /* copy-on-write copies made so far */
    int64_t tokens;            /* sum of the sequences' token counts */
    int64_t waste_tokens;      /* unused slots in the sequences' last blocks */
    int64_t cached_blocks;     /* blocks in the prefix tree (referenced or not) */
    int64_t cached_free;       /* unreferenced cached blocks (reusable by eviction) */
    int64_t host_blocks;       /* blocks of the host tier (0 without one) */
    int64_t host_free;         /* free host blocks */
    int64_t swapped_seqs;      /* sequences swapped out to the host tier */
} pa_alloc_stats_t;

/* Returns NULL on bad arguments (see pa_last_error_string). */
PA_API pa_allocator* pa_alloc_create(int num_blocks, int block_size, const int32_t* free_order);
PA_API void pa_alloc_destroy(pa_allocator* a);

/* New sequence of num_tokens tokens (a prompt): takes ceil(num_tokens/B) blocks,
 * each with reference count 1.  slots_out (nullable, num_tokens entries) receives
 * the slot of every token.  PA_ERR_INVALID if seq_id exists. */
PA_API pa_status pa_alloc_add_seq(pa_allocator* a, int64_t seq_id, int num_tokens, int64_t* slots_out);

/*
 * New sequence of num_tokens tokens whose ids are token_ids[num_tokens] (HOST),
 * sharing cached prompt blocks.  The leading full blocks whose token ids (and
 * everything before them) match a cached prefix are reused (count + 1); the other
 * full blocks are taken fresh and cached under their token ids; a partial last
 * block is taken fresh and stays private.  *num_cached_out = tokens covered by the
 * reused blocks (a multiple of B): their K/V are already in the cache, so the
 * caller appends only tokens num_cached .. num_tokens-1 (pa_reshape_and_cache with
 * those slots).  slots_out (nullable) receives the slot of every token.  A fresh
 * cached block must be written before any later call can reuse it, i.e. before the
 * decode of a sequence that shares it, in stream order.
 */
PA_API pa_status pa_alloc_add_seq_cached(pa_allocator* a, int64_t seq_id, const int32_t* token_ids, int num_tokens,
                                         int64_t* slots_out, int* num_cached_out);

/* child shares every block of parent (each reference count + 1) and its token count. */
PA_API pa_status pa_alloc_fork(pa_allocator* a, int64_t parent_id, int64_t child_id);

/*
 * Slot for one new token of seq_id.  A fresh block is taken when the last block is
 * full or absent.  If the last block is partially filled and shared (reference
 * count > 1), it is copied on write: a new block dst is taken, the old count is
 * decremented, the table entry is repointed, and (src, dst) is returned through
 * cow_src_out / cow_dst_out (each -1 when no copy is needed; both nullable).
 * The caller must run pa_copy_blocks for the pair before writing the slot.
 */
PA_API pa_status pa_alloc_append_slot(pa_allocator* a, int64_t seq_id, int64_t* slot_out, int32_t* cow_src_out,
                               int32_t* cow_dst_out);

/*
 * One append per listed sequence, in list order (a decode step).  slots_out[n],
 * cow_pairs_out[2 * n] (src, dst pairs, packed) and *num_cow_out receive the
 * results.  All or nothing: on error no append of the batch remains applied.
 */
PA_API pa_status pa_alloc_append_slots(pa_allocator* a, const int64_t* seq_ids, int n, int64_t* slots_out,
                                int64_t* cow_pairs_out, int* num_cow_out);

/*
 * One beam-search step ([FSAH] section 3 and [INIT] section 3: beams share blocks by
 * copy-on-write until one writes).  The old beams are beam_ids[num_beams]; new beam
 * j continues old beam parents[j] (an index into beam_ids) under id new_ids[j], and
 * gets one new token.  In order: every new beam forks its parent (shares its blocks,
 * counts + 1); the old beams are freed (in list order); then each new beam, in order,
 * takes the slot of its token as pa_alloc_append_slots does.  Freeing before
 * appending means a parent chosen once needs no copy, and a parent chosen k times
 * needs k-1 copies of its partial last block.  slots_out[num_new] receives the
 * slots; cow_pairs_out[2 * num_new] and *num_cow_out the (src, dst) copies, to be
 * run with one pa_copy_blocks before the appends are written.  A new id may reuse
 * an old beam's id; it must not be held by any other sequence.  All or nothing.
 */
PA_API pa_status pa_alloc_beam_step(pa_allocator* a, const int64_t* beam_ids, int num_beams, const int32_t* parents,
                                    const int64_t* new_ids, int num_new, int64_t* slots_out, int64_t* cow_pairs_out,
                                    int* num_cow_out);

/* Drops one reference to each block of seq_id; blocks reaching zero rejoin the free
 * pool, or stay in the prefix tree as unreferenced cached blocks. */
PA_API pa_status pa_alloc_free_seq(pa_allocator* a, int64_t seq_id);

/*
 * Host tier for swapping ([FSAH] "Engineering Limitations": CPU-GPU block swapping
 * under memory pressure).  pa_alloc_add_host_pool gives the allocator
 * num_host_blocks host blocks (ids 0..n-1, a FIFO free queue), once.  The caller
 * owns the host pools themselves: pinned host memory shaped like the device pools
 * ([num_host_blocks][Hkv][B][D] for K and for V), moved with pa_swap_blocks.
 *
 * pa_alloc_swap_out moves a resident sequence to the host: each of its blocks, in
 * table order, gets a host block; (device, host) pairs go to pairs_out[2 * n] and
 * *num_pairs_out = n; each device block loses the sequence's reference (blocks that
 * other sequences share stay with them; cached blocks stay cached).  The caller must
 * run pa_swap_blocks(host pools <- device pools, pairs) before any later write can
 * reach the released device blocks, i.e. before the next append's copy in stream
 * order.  pa_alloc_swap_in brings it back: each host block gets a device block
 * (taken as any other), (host, device) pairs are returned, the host blocks are freed;
 * run pa_swap_blocks(device pools <- host pools, pairs) before the sequence's next
 * decode.  A swapped-out sequence cannot be forked, appended to, reshuffled or put in
 * a dense table (PA_ERR_INVALID); pa_alloc_free_seq frees its host blocks;
 * pa_alloc_block_table returns its host block ids.  Out of host or device blocks:
 * PA_ERR_OOM, nothing changes.
 */
PA_API pa_status pa_alloc_add_host_pool(pa_allocator* a, int num_host_blocks);
PA_API pa_status pa_alloc_swap_out(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int* num_pairs_out);
PA_API pa_status pa_alloc_swap_in(pa_allocator* a, int64_t seq_id, int64_t* pairs_out, int* num_pairs_out);
PA_API int pa_alloc_num_host_free(const pa_allocator* a);
PA_API int pa_alloc_is_swapped(const pa_allocator* a, int64_t seq_id);  /* 1, 0, or -1 if unknown */

/* Copies seq_id's block table into out[capacity]; *n_out = its length.
 * PA_ERR_INVALID if capacity is too small (nothing is written then). */
PA_API pa_status pa_alloc_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int capacity, int* n_out);

/* Dense [n][max_blocks] table of the listed sequences, rows padded with `fill`;
 * *context_lens_out (nullable, n entries) receives their token counts. */
PA_API pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int n, int32_t* out,
                                int max_blocks, int32_t fill, int32_t* context_lens_out);

PA_API int pa_alloc_ref_count(const pa_allocator* a, int32_t block);   /* -1 if out of range */
PA_API int pa_alloc_num_free(const pa_allocator* a);          /* blocks in the free queue */
PA_API int pa_alloc_num_cached_free(const pa_allocator* a);   /* unreferenced cached blocks */
PA_API int pa_alloc_num_tokens(const pa_allocator* a, int64_t seq_id); /* -1 if unknown */
PA_API pa_status pa_alloc_stats(const pa_allocator* a, pa_alloc_stats_t* out);

/* ------------------------------------------------------------------ diagnostics */

/* Message of the last failed call on this thread ("" if none).  Valid until the
 * next failing call on the same thread. */
PA_API const char* pa_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
