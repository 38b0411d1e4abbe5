/*
 * pa.h -- C ABI of the paged KV-cache decode library (libpa.so, sm_100a).
 *
 * The problem these calls solve is stated on three pages:
 *   [P1] "What problem does PagedAttention solve, and what is continuous batching?"
 *   [P2] "PagedAttention & Continuous Batching"
 *   [P3] "Continuous Batching & Paged Attention -- LLM Inference Optimization & Serving"
 * The KV cache is stored in fixed-size physical blocks anywhere in GPU memory; a
 * per-sequence block table maps logical block numbers to physical blocks and the
 * attention kernel follows it when it reads keys and values ([P1] "How
 * PagedAttention works", [P2] "Overview", [P3] "Paged attention borrows a trick
 * from operating systems").  Decode reads the whole cache of each sequence and
 * appends one token's keys and values per step ([P1] "Why the KV cache becomes
 * the problem").
 *
 * Conventions
 *  - Every call returns pa_status; PA_OK is 0.  A failing call leaves the host
 *    state (free list, refcounts, tables, lengths) exactly as it was.  The text
 *    of the last failure on the calling thread is pa_last_error().
 *  - Device memory is owned by the caller: the key and value pools, queries,
 *    outputs, block tables, lengths, slot mappings, copy pairs and workspaces are
 *    raw device pointers the caller allocated.  The opaque pa_pool owns only host
 *    metadata (free stack, refcounts, per-sequence tables and lengths).
 *  - Device work is asynchronous on the given stream (a cudaStream_t passed as
 *    pa_stream; NULL is the legacy default stream).  Launch failures return
 *    PA_ERR_CUDA.  Kernels also record data errors they meet (an out-of-range
 *    block id or slot, a length beyond the table, a bounded wait that ran out)
 *    in a sticky device word read by pa_device_error().
 *  - Not thread-safe: one host thread at a time per pool.
 *
 * Device pool layout (keys and values alike, caller-allocated, 16-byte aligned):
 *   pool[num_layers][num_blocks][num_kv_heads][block_size][head_dim] of `dtype`.
 * One block id names the same block in every layer, as the pages' bytes-per-token
 * figure counts every layer ([P1] "A concrete memory example").  Slot
 * s = block * block_size + offset names one token position inside a block.
 */
#ifndef PA_H
#define PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,    /* a bad pointer, size, id, or combination */
    PA_ERR_OUT_OF_BLOCKS = 2,  /* the free list cannot satisfy the call */
    PA_ERR_DOUBLE_FREE = 3,    /* a block with refcount 0 was freed */
    PA_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed */
    PA_ERR_UNSUPPORTED = 5,    /* a valid shape the kernels are not built for */
    PA_ERR_HOST_MEMORY = 6     /* host memory for the block manager's own records ran out */
} pa_status;

/* PA_FP8_E4M3 is a cache storage type only: see "FP8 cache" below. */
typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2, PA_FP8_E4M3 = 3 } pa_dtype;

typedef struct pa_pool pa_pool;
typedef void *pa_stream;       /* a cudaStream_t */

typedef struct {
    int32_t num_layers;        /* >= 1 */
    int32_t num_blocks;        /* physical blocks in the pool, >= 1 */
    int32_t block_size;        /* tokens per block: 16 or 32 */
    int32_t num_kv_heads;      /* >= 1 */
    int32_t head_dim;          /* 64 or 128 */
    pa_dtype dtype;            /* element type of the K and V pools */
    pa_dtype act_dtype;        /* PA_FP8_E4M3 pools: type of queries, appended rows and
                                  16-bit outputs (PA_F16 or PA_BF16); ignored otherwise
                                  (they are the pool dtype) */
} pa_pool_config;

typedef struct {
    int32_t num_blocks;
    int32_t num_free;          /* blocks on the free list */
    int32_t num_shared;        /* blocks with refcount > 1 */
    int32_t num_seqs;          /* live sequences */
    int64_t num_tokens;        /* sum of live sequence lengths */
    int64_t cow_copies;        /* copy-on-write pairs issued so far */
    int32_t peak_used;         /* most blocks ever in use at once */
    int32_t num_cached;        /* blocks registered for prefix caching */
    int32_t num_evictable;     /* registered blocks with refcount 0 (counted in num_free) */
    int64_t cache_hits;        /* blocks shared through pa_seq_add_cached */
    int64_t cache_evictions;   /* registered blocks reclaimed by allocation */
} pa_pool_stats_t;

/* Message for the last failing call on this thread ("" if none). */
const char *pa_last_error(void);
const char *pa_status_string(pa_status s);

/* ------------------------------------------------------------------ FP8 cache
 *
 * [P1] "Common misconception": paging does not shrink the bytes each token needs;
 * KV-cache quantisation does.  A pool of dtype PA_FP8_E4M3 stores every key and
 * value element as one E4M3 byte (OCP 8-bit floating point, "fn" variant: bias 7,
 * 3 mantissa bits, largest finite 448, 0x7F / 0xFF NaN) and, beside the codes, one
 * scale byte per (token, KV head) row of K and of V in one caller-owned device array
 *   scales [num_layers][num_blocks][num_kv_heads][2][block_size] uint8
 * (index 0 = K, 1 = V), byte e meaning the factor 2^(e - 127).  A row x of head_dim
 * values is written by pa_append_kv as: X = the smallest integer with
 * max|x| <= 448 * 2^X, clamped to [-127, 127] (an all-zero row gets -127);
 * e = X + 127; code_i = x_i * 2^-X (one fp32 multiply) rounded to nearest E4M3,
 * ties to even, saturating at 448.
 * Readers use the value E4M3(code) * 2^(e - 127).  The scales are per row, so an
 * append never re-encodes earlier rows of its block, and copy-on-write, swap and
 * decode carry them with the codes.  Non-finite input rows are outside the
 * contract.  Supported: decode (head_dim 128), append, block copies and swap;
 * pa_prefill_attention returns PA_ERR_UNSUPPORTED for FP8 pools.
 */

/* ------------------------------------------------------------------ pool */

/* Create the host block manager for caller-owned device pools.
 * [P1] "How PagedAttention works": the allocator can take any free block.  The
 * free list is a LIFO stack; `free_order` (num_blocks ids, a permutation, may be
 * NULL for 0..num_blocks-1) fixes which block is handed out first: free_order[0],
 * then free_order[1], ...  k_pool / v_pool may be NULL for host-only use; the
 * device calls then fail with PA_ERR_INVALID_ARG.  *out receives the pool. */
pa_status pa_pool_create(const pa_pool_config *cfg, void *k_pool, void *v_pool,
                         const int32_t *free_order, pa_pool **out);
pa_status pa_pool_destroy(pa_pool *pool);
pa_status pa_pool_stats(const pa_pool *pool, pa_pool_stats_t *out);
/* Attach the scale array of a PA_FP8_E4M3 pool (device, 16-byte aligned,
 * caller-owned, layout above).  Required before any device call on such a pool;
 * PA_ERR_INVALID_ARG for other pools or a null pointer. */
pa_status pa_pool_set_scales(pa_pool *pool, void *scales);

/* ------------------------------------------------------------------ blocks */

/* Pop the top of the free stack into *block with refcount 1.
 * PA_ERR_OUT_OF_BLOCKS when the stack is empty ([P1] "The senior-level nuance":
 * a full pool must queue, preempt or reject; it cannot grow). */
pa_status pa_alloc_block(pa_pool *pool, int32_t *block);
/* Drop one reference; at zero the block goes back on top of the stack and is
 * reused next ([P1] "A concrete memory example": a finished request's blocks
 * return to the pool at once).  PA_ERR_DOUBLE_FREE if the count is already 0. */
pa_status pa_free_block(pa_pool *pool, int32_t block);
/* Add a reference to an allocated block (sharing, [P1] "How PagedAttention
 * works").  PA_ERR_INVALID_ARG for a free block. */
pa_status pa_incref_block(pa_pool *pool, int32_t block);
pa_status pa_block_refcount(const pa_pool *pool, int32_t block, int32_t *rc);
pa_status pa_num_free_blocks(const pa_pool *pool, int32_t *n);
/* Copy the free stack, bottom first (the last entry is handed out next), into
 * out[0..cap); *n receives its length.  For inspection and bit-exact checks. */
pa_status pa_free_list(const pa_pool *pool, int32_t *out, int32_t cap, int32_t *n);
/* Host fault injection: the (n+1)-th block allocation from now fails with
 * PA_ERR_OUT_OF_BLOCKS (n < 0 switches it off). */
pa_status pa_debug_fail_alloc_after(pa_pool *pool, int64_t n);

/* ------------------------------------------------------------------ sequences */

/* New empty sequence; *seq_id receives its handle (handles are never reused). */
pa_status pa_seq_add(pa_pool *pool, int32_t *seq_id);
/* New sequence sharing every block of `parent` (refcount +1 each, logical order):
 * [P1] "How PagedAttention works", beam candidates referencing the same blocks. */
pa_status pa_seq_fork(pa_pool *pool, int32_t parent, int32_t *child);
/* Retire a sequence: drop one reference on each of its blocks, logical order. */
pa_status pa_seq_free(pa_pool *pool, int32_t seq_id);
/* Length and block table of a sequence: *len tokens, *nblk blocks; the first
 * min(cap, nblk) physical ids are written to table (table may be NULL). */
pa_status pa_seq_info(const pa_pool *pool, int32_t seq_id, int32_t *len, int32_t *table,
                      int32_t cap, int32_t *nblk);

/* Reserve cache slots for ntok[i] new tokens of seq_ids[i], i = 0..n-1 in order,
 * one token at a time ([P3] "Paged attention borrows a trick from operating
 * systems": a growing request gets another block; [P1] "How PagedAttention
 * works": a diverging sharer gets a private copy-on-write block).  For a
 * sequence of length L:
 *   L % block_size == 0           -> take a new block from the free stack;
 *   else tail block refcount > 1  -> copy on write: take a new block, record the
 *                                    pair (tail, new), drop one reference on tail,
 *                                    and use the new block as the tail;
 *   slot = table[L / block_size] * block_size + L % block_size;  L += 1.
 * Outputs (host buffers): slot_mapping_out[sum(ntok)] in batch order;
 * cow_pairs_out[2 * k] = (src, dst) for each copy, at most n pairs (one per
 * sequence); *n_cow = k.  seq_ids must be distinct.  On PA_ERR_OUT_OF_BLOCKS
 * nothing changes; a call whose block-boundary crossings alone need more blocks
 * than are free (or evictable) fails that way before anything is taken, whatever
 * the counts.  PA_ERR_HOST_MEMORY (the host could not grow the call's own records)
 * also leaves everything unchanged.  The caller copies the pairs to the device and calls
 * pa_copy_blocks before writing the new tokens with pa_append_kv. */
pa_status pa_reserve_slots(pa_pool *pool, const int32_t *seq_ids, const int32_t *ntok, int32_t n,
                           int64_t *slot_mapping_out, int32_t *cow_pairs_out, int32_t *n_cow);

/* Dense block tables for a batch (host buffers): tables_out[n][max_blocks] holds
 * each sequence's physical ids, padded with -1; lens_out[n] its length.
 * PA_ERR_INVALID_ARG if a sequence has more than max_blocks blocks. */
pa_status pa_build_block_tables(const pa_pool *pool, const int32_t *seq_ids, int32_t n,
                                int32_t max_blocks, int32_t *tables_out, int32_t *lens_out);

/* ------------------------------------------------------------------ prefix caching */

/* [P1] "How PagedAttention works": prefix caching can reuse blocks the way shared
 * beams do; [P2] "If you remember three things": shared prefixes are shared
 * blocks.  The pages define no lookup, so the key of a full block is the caller's:
 * typically a hash chain over the block's token ids and every token before it, so
 * equal keys mean equal key/value contents.
 *  - A registered block keeps its key while it lives.  When its refcount reaches 0
 *    it is not pushed on the free stack: it joins the back of an evictable queue
 *    and can still be found.  Allocation uses the free stack first and only then
 *    evicts the front of the queue (least recently released), forgetting its key.
 *  - pa_num_free_blocks counts free and evictable blocks; pa_free_list lists the
 *    free stack only, pa_prefix_evictable the queue. */

/* Register the first n_blocks blocks of seq_id (they must be full:
 * n_blocks * block_size <= length) under keys[0..n_blocks).  A key that is already
 * registered, or a block that already has a key, is skipped.  *n_new (may be NULL)
 * receives how many blocks were registered. */
pa_status pa_prefix_register(pa_pool *pool, int32_t seq_id, const uint64_t *keys, int32_t n_blocks,
                             int32_t *n_new);
/* New sequence whose leading blocks are the registered blocks of keys[0..n_keys),
 * shared (refcount + 1; an evictable block leaves the queue) up to the first key
 * that is not registered.  *n_hit receives the number shared; the sequence's length
 * is n_hit * block_size, and the caller appends the rest of its prompt with
 * pa_reserve_slots / pa_append_kv as usual. */
pa_status pa_seq_add_cached(pa_pool *pool, const uint64_t *keys, int32_t n_keys, int32_t *seq_id,
                            int32_t *n_hit);
/* Copy the evictable queue, front (next to be evicted) first, into out[0..cap);
 * *n receives its length. */
pa_status pa_prefix_evictable(const pa_pool *pool, int32_t *out, int32_t cap, int32_t *n);

/* ------------------------------------------------------------------ preemption with swap */

/* [P1] "The senior-level nuance" / "What happens when the KV cache is full?": a full
 * pool must queue, preempt, offload cache data or reject.  These calls offload one
 * sequence's cache to host memory and bring it back.
 * Host buffer layout (caller-owned, page-locked so the GPU can reach it, e.g. from
 * cudaHostAlloc): [block i in logical order][layer][K, V][num_kv_heads][block_size]
 * [head_dim] of the pool dtype; for a PA_FP8_E4M3 pool each [block][layer] record
 * is followed by the block's scale bytes [num_kv_heads][2][block_size].
 * pa_swap_bytes gives the size. */
pa_status pa_swap_bytes(const pa_pool *pool, int32_t seq_id, size_t *bytes);
/* Enqueue on `stream` a copy of every block of seq_id (all layers, K and V) into
 * host_buf, then drop one reference on each block (logical order), as a retire does.
 * The sequence keeps its id and length but owns no blocks until pa_swap_in; appends,
 * forks and tables are refused for it meanwhile.  Later device work that reuses the
 * freed blocks must be issued on the same stream (or ordered after it).  A pool
 * without device memory does the bookkeeping only (host_buf may be NULL). */
pa_status pa_swap_out(pa_pool *pool, int32_t seq_id, void *host_buf, size_t buf_bytes, pa_stream stream);
/* Take ceil(length / block_size) blocks (one allocation after the other, as appends
 * would), make them the sequence's table and enqueue on `stream` the copy of host_buf
 * back into them.  PA_ERR_OUT_OF_BLOCKS leaves everything unchanged. */
pa_status pa_swap_in(pa_pool *pool, int32_t seq_id, const void *host_buf, size_t buf_bytes, pa_stream stream);

/* ------------------------------------------------------------------ device work */

/* Copy-on-write block copies: for each pair (src, dst) in pairs_dev[n_pairs][2]
 * (device int32), block dst becomes a bit copy of block src in every layer, keys
 * and values (and their scale bytes in an FP8 pool).  The whole block is copied,
 * so every earlier slot stays valid. */
pa_status pa_copy_blocks(pa_pool *pool, const int32_t *pairs_dev, int32_t n_pairs,
                         pa_stream stream);

/* Append (reshape-and-cache): row i of k_new / v_new (device, [n_tokens]
 * [num_kv_heads][head_dim] of the pool dtype, 16-byte aligned) is bit-copied
 * into slot slot_mapping_dev[i] of `layer`; a negative slot skips the row
 * ([P1] "Why the KV cache becomes the problem": decode appends a small amount
 * of new data each step).  For a PA_FP8_E4M3 pool the rows are of act_dtype and
 * each (token, head) row is quantised as stated under "FP8 cache". */
pa_status pa_append_kv(pa_pool *pool, int32_t layer, const void *k_new, const void *v_new,
                       const int64_t *slot_mapping_dev, int32_t n_tokens, pa_stream stream);

/* Number of splits per sequence the decode kernel uses for a table of width
 * max_blocks when a split holds split_tokens tokens (0 = never split). */
int32_t pa_decode_max_splits(int32_t block_size, int32_t max_blocks, int32_t split_tokens);
/* Workspace bytes for pa_decode_attention with that many splits: the split partials
 * (when max_splits > 1), the longest-first order of the (sequence, split) ranges
 * (int32 [n_seqs * max_splits]) and, with splits, one merge counter per (sequence,
 * query head) at most; each part rounded up to 16 bytes. */
size_t pa_decode_workspace_bytes(int32_t n_seqs, int32_t num_q_heads, int32_t head_dim,
                                 int32_t max_splits);

/* Paged decode attention ([P1] "How PagedAttention works": the kernel follows the
 * block table when it reads keys and values; paging does not change the result,
 * [P1] "Common misconception").  For each sequence s and query head h, with KV
 * head g = h / (num_q_heads / num_kv_heads) and L = seq_lens_dev[s]:
 *   out[s][h] = sum_{j<L} softmax_j(scale * q[s][h] . K_s[j]) V_s[j],
 *   K_s[j] = k_pool[layer][tables[s][j / B]][g][j % B], V_s likewise.
 * q [n_seqs][num_q_heads][head_dim] in the pool dtype (act_dtype for an FP8
 * pool, whose K_s[j] / V_s[j] are the dequantised rows); out the same shape in
 * out_dtype (PA_F32 or the pool dtype / act_dtype); block_tables_dev [n_seqs][max_blocks]
 * int32, seq_lens_dev [n_seqs] int32 >= 1, all device pointers.  Sequences with
 * more than split_tokens tokens (a multiple of block_size; 0 = never) are split
 * into ceil(blocks / (split_tokens / block_size)) ranges of nearly equal length (at
 * most split_tokens tokens each, the first ones one block longer) whose partial
 * results are merged (on the tensor-core paths by the last CTA of each range, on
 * the fp32 path by a second kernel); that needs
 * `workspace` of pa_decode_workspace_bytes(n_seqs, num_q_heads, head_dim,
 * pa_decode_max_splits(...)) bytes (caller-owned device memory, 16-byte aligned,
 * contents need not be initialised).  With a workspace of that size the call first
 * sorts the ranges by length on the device (one small kernel) and starts the longest
 * ranges first, so no long range is left running alone at the end; with a single
 * split the workspace may be NULL, and the ranges then start in batch order.  Supported: head_dim 64/128 (128 for FP8
 * pools), block_size 16/32, num_q_heads / num_kv_heads in {1, 2, 4, 8}. */
pa_status pa_decode_attention(pa_pool *pool, int32_t layer, const void *q, void *out,
                              pa_dtype out_dtype, const int32_t *block_tables_dev,
                              int32_t max_blocks, const int32_t *seq_lens_dev, int32_t n_seqs,
                              int32_t num_q_heads, float scale, int32_t split_tokens,
                              void *workspace, size_t ws_bytes, pa_stream stream);

/* Allocation-free decode attention.  The pages have no counterpart: this entry
 * exists for callers that cannot allocate device memory -- a serving process
 * that has already handed almost all of the GPU to its KV-cache pool, a host
 * whose allocator may not be called on the decode path (cudaMalloc can
 * synchronise the device and stall every stream), or a plain C embedding with no
 * allocator of its own.  It computes exactly what pa_decode_attention computes,
 * with the same arguments minus the workspace: the split-K partials go to a fixed
 * array of PA_STATIC_WORKSPACE_BYTES inside the library, which every GPU that
 * loads the library keeps until the process exits.
 *  - It allocates nothing and frees nothing.  The caller still owns q, out, the
 *    tables, the lengths and the pools.
 *  - A batch whose partials would not fit, i.e. pa_decode_workspace_bytes(n_seqs,
 *    num_q_heads, head_dim, pa_decode_max_splits(block_size, max_blocks,
 *    split_tokens)) > PA_STATIC_WORKSPACE_BYTES, is rejected with
 *    PA_ERR_INVALID_ARG and a message naming both sizes; nothing is launched.
 *  - The first call on a device looks up the array's device address with that
 *    device current and keeps it; make that first call before any stream capture.
 *    The kept address belongs to the device's context: after cudaDeviceReset the
 *    entry must not be called again in the same process.
 *  - All calls on a device share the one array and it keeps the last call's
 *    contents.  Nothing in it needs to start at zero (every partial a call reads
 *    was written earlier in the same call), but calls that overlap on the GPU --
 *    on different streams, or from different host threads -- race on it and must
 *    be serialised by the caller. */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)
pa_status pa_decode_attention_static(pa_pool *pool, int32_t layer, const void *q, void *out,
                                     pa_dtype out_dtype, const int32_t *block_tables_dev,
                                     int32_t max_blocks, const int32_t *seq_lens_dev,
                                     int32_t n_seqs, int32_t num_q_heads, float scale,
                                     int32_t split_tokens, pa_stream stream);

/* Paged chunked-prefill attention (causal) on the tensor cores ([P1] "Why the KV
 * cache becomes the problem": prefill is the compute-heavy pass over the prompt;
 * "The prefill and decode phases need careful scheduling": long prompts are split
 * into chunks).  For sequence s the chunk is its last C_s = q_start_dev[s+1] -
 * q_start_dev[s] tokens, already appended to the cache (seq_lens_dev[s] counts them);
 * query row q_start_dev[s] + i sits at position L_s - C_s + i and attends to keys
 * 0 .. L_s - C_s + i through the block table:
 *   out[r][h] = sum_{j <= pos(r)} softmax_j(scale * q[r][h] . K_s[j]) V_s[j].
 * q [total][num_q_heads][128] in the pool dtype (fp16 or bf16), out the same shape in
 * out_dtype (PA_F32 or the pool dtype), q_start_dev int32 [n_seqs + 1] ascending,
 * max_q_len >= every C_s.  head_dim 128, block_size 16 or 32, num_q_heads /
 * num_kv_heads in {1, 2, 4, 8}; fp32 caches -> PA_ERR_UNSUPPORTED. */
pa_status pa_prefill_attention(pa_pool *pool, int32_t layer, const void *q, void *out, pa_dtype out_dtype,
                               const int32_t *block_tables_dev, int32_t max_blocks,
                               const int32_t *seq_lens_dev, const int32_t *q_start_dev, int32_t n_seqs,
                               int32_t max_q_len, int32_t num_q_heads, float scale, pa_stream stream);

/* ------------------------------------------------------------------ diagnostics */

/* Device error bits recorded by kernels since the last clear (synchronises the
 * device): 1 = block id out of range in a table, 2 = sequence length beyond its
 * table or < 1, 4 = a bounded wait ran out, 8 = slot out of range.  clear != 0
 * resets the word. */
pa_status pa_device_error(int32_t *code, int32_t clear);
/* Kernels this library has launched since it was loaded (all devices). */
uint64_t pa_launch_count(void);

/* Failure-detection test hook (no page counterpart; the pages' failure cases --
 * [P3] "Decisions leaders and practitioners actually face": reject cleanly rather
 * than stall -- only motivate it).  Every device-side wait of the library's kernels
 * is bounded; this sets the bound on the current device to wait_limit_ns
 * (<= 0 restores the default of 2 s) and, when withhold_cta >= 0, makes the
 * producer warp of the CTA with that linear block index issue no copies (every
 * later pa_decode_attention and pa_prefill_attention launch on any device, until
 * called again with -1).  That CTA's other warps then wait for data that never
 * comes: each wait runs out after the bound, records device error bit 4 and
 * returns (the prefill kernel's roles also share an abort flag, and its tensor
 * memory is still freed), no copy is left in flight, and the rest of the launch is
 * unaffected; the withheld CTA's outputs are not meaningful.  Off by default;
 * synchronises the device. */
pa_status pa_debug_wait_test(int64_t wait_limit_ns, int32_t withhold_cta);

#ifdef __cplusplus
}
#endif

#endif /* PA_H */
