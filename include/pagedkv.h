/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged-KV attention for NVIDIA B200 (sm_100a).
 *
 * The method is PagedAttention with iteration-level (continuous) batching as
 * described on the page "LLM 推理引擎 Continuous Batching 与 PagedAttention：
 * 从 vLLM 原理到生产级部署实战" (cited below as [CB-PA]) and in the chapter
 * "动态批处理算法：连续批处理、In-flight 请求管理与 PagedAttention" ([DB]).
 * The KV cache of every request is stored in fixed-size physical blocks of
 * `block_size` tokens taken from one shared pool; a per-request block table
 * maps logical block i to a physical block ([CB-PA] §3.1-§3.2, [DB] §4.3).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every function returns a pa_status; nothing is thrown across the ABI.
 *   On an error the message of the calling thread's last error is available
 *   from pa_last_error().
 * - Device entry points take DEVICE pointers that the caller allocated and
 *   owns; the library never allocates, frees or retains device memory, and
 *   never synchronises.  Kernels are enqueued on `stream` (a cudaStream_t
 *   passed as void*; NULL = the legacy default stream) on the current device.
 *   Argument errors are detected on the host before anything is enqueued.
 *   Pointers themselves are not inspected: one that is not memory of the
 *   current device is the caller's error and faults the kernel that reads it
 *   (the Python binding refuses host tensors and other devices' tensors).
 * - fp16 buffers (pa_half) hold IEEE-754 binary16 values.  Arithmetic inside
 *   the attention kernels is fp32; outputs are rounded to fp16 (nearest even).
 * - The KV cache is two separate tensors, K and V, each laid out
 *   [num_blocks, block_size, num_heads, head_dim] row-major (a token's heads
 *   are contiguous inside its row, as the pointer arithmetic
 *   "+ head_idx * head_dim" of [CB-PA] §3.3 places them).
 * - A slot names one token row of the pool: slot = block * block_size + row.
 * - `err_flag` (nullable, device int32): kernels check every block id, slot
 *   and length they read from device memory; a bad one is skipped (never
 *   dereferenced) and the matching PA_DEVCHK_* bit is OR-ed into *err_flag.
 *   The caller reads the flag after synchronising; pa_check_device_flag()
 *   turns a read-back value into PA_ERR_DEVICE_CHECK.
 * - Supported kernel instances: head_dim 64 or 128; block_size 8 or a
 *   multiple of 16; num_heads a multiple of 4 (or of 2 with head_dim 128).
 *   Anything else returns PA_ERR_UNSUPPORTED.
 * - The block allocator is host-only, single-threaded (one scheduler thread
 *   owns it, as in [CB-PA] §2.2) and owned by the library from
 *   pa_alloc_create to pa_alloc_destroy.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t pa_status;
enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* bad pointer, size, shape or id range            */
    PA_ERR_OOM = 2,           /* not enough free blocks ([CB-PA] §3.2 "return False") */
    PA_ERR_NOT_FOUND = 3,     /* unknown request id                               */
    PA_ERR_EXISTS = 4,        /* request id already has a block table             */
    PA_ERR_UNSUPPORTED = 5,   /* head_dim / block_size / head count not built     */
    PA_ERR_CUDA = 6,          /* a CUDA call failed; see pa_last_error()          */
    PA_ERR_DEVICE_CHECK = 7   /* a device-side check fired (see err_flag)         */
};

/* Bits a kernel ORs into *err_flag. */
enum {
    PA_DEVCHK_BLOCK_ID = 1,   /* block-table entry outside [0, num_blocks)        */
    PA_DEVCHK_SLOT = 2,       /* slot >= num_blocks * block_size                  */
    PA_DEVCHK_SEQ_LEN = 4,    /* seq_len < 0 or > max_blocks * block_size         */
    PA_DEVCHK_QUERY_RANGE = 8, /* q_start not non-decreasing or past num_tokens   */
    PA_DEVCHK_TIMEOUT = 16     /* an internal bounded wait ran out (a library bug) */
};

typedef uint16_t pa_half;
typedef struct pa_alloc pa_alloc;

typedef struct {
    int32_t num_blocks;
    int32_t block_size;
    int32_t num_free;        /* blocks on the free list                             */
    int32_t num_used;        /* blocks with refcount > 0                            */
    int64_t total_refs;      /* sum of refcounts = sum of block-table lengths       */
    int64_t num_requests;    /* requests with a block table                         */
    int64_t oom_count;       /* calls that returned PA_ERR_OOM                      */
    int64_t waste_tokens;    /* sum over requests of blocks*block_size - seq_len    */
} pa_alloc_stats_t;

/* ---- library ------------------------------------------------------------ */

/* ABI version of this header (bumped on any signature change). */
int32_t pa_abi_version(void);
/* Message of the calling thread's last failed call ("" if none). */
const char* pa_last_error(void);
/* Static name of a status code. */
const char* pa_status_string(pa_status s);
/* PA_OK if `flag_value` (a read-back err_flag) is 0, else PA_ERR_DEVICE_CHECK. */
pa_status pa_check_device_flag(int32_t flag_value);

/* Kernels a failure-detection test can stall. */
enum { PA_KERNEL_DECODE = 1, PA_KERNEL_PREFILL = 2 };

/* Test hook for the device-side failure detection.  Every wait inside the
 * attention kernels is bounded (2 s); when one runs out the kernel ORs
 * PA_DEVCHK_TIMEOUT into err_flag, stops its other roles, lets the copies and
 * tensor-core operations it issued complete, frees what it holds and returns,
 * so the CUDA context stays usable.  This call makes the NEXT launch of
 * `kernel` in this process exercise that path: its consumer role (decode:
 * the softmax warps; prefill: the softmax warps) first waits on a barrier
 * that nothing completes, and every pipeline wait of that launch is bounded by
 * wait_limit_ns instead of 2 s (the final drain waits keep 2 s).  The launch
 * then returns with PA_DEVCHK_TIMEOUT set and its output undefined; later
 * launches are normal.  Not for production use.
 * Errors: INVALID_ARG (unknown kernel, wait_limit_ns 0 or above 2e9). */
pa_status pa_debug_inject_stall(int32_t kernel, uint64_t wait_limit_ns);

/* ---- host block allocator ([CB-PA] §3.2 BlockManager, §4.1 shared prefix) --
 *
 * Free list: starts as init_free_order (or 0..num_blocks-1 when NULL); every
 * take pops from its END; blocks whose refcount drops to zero are pushed on
 * the end in block-table order.  A request's block table lists its physical
 * blocks in logical order; its seq_len counts the tokens it stores; it always
 * holds exactly ceil(seq_len / block_size) blocks.  The allocator is not
 * thread-safe. */

/* Create a pool of `num_blocks` blocks of `block_size` tokens.
 * init_free_order: NULL, or a permutation of 0..num_blocks-1 (host, copied).
 * Errors: INVALID_ARG (num_blocks < 0, block_size <= 0, not a permutation, out NULL). */
pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size,
                          const int32_t* init_free_order, pa_alloc** out);
/* Destroy the allocator (NULL is accepted). */
void pa_alloc_destroy(pa_alloc* a);

/* [CB-PA] §3.2 allocate: give `req` a table of ceil(num_tokens / block_size)
 * popped blocks and seq_len = num_tokens.  All-or-nothing.
 * Errors: EXISTS (req has a table), OOM (too few free blocks; nothing changes),
 * INVALID_ARG (num_tokens < 0). */
pa_status pa_alloc_allocate(pa_alloc* a, int64_t req, int32_t num_tokens);

/* [CB-PA] §3.2 append_token: store one more token.  With current_len the
 * tokens stored before the call, a block is popped iff current_len %
 * block_size == 0.  *slot_out (nullable) = slot of position current_len.
 * Errors: NOT_FOUND, OOM (nothing changes). */
pa_status pa_alloc_append_token(pa_alloc* a, int64_t req, int64_t* slot_out);

/* n appends as one all-or-nothing step (same pops, same slots as n calls of
 * pa_alloc_append_token).  slots_out: NULL or host int64[n].
 * Errors: NOT_FOUND, OOM (nothing changes), INVALID_ARG (n < 0). */
pa_status pa_alloc_append_tokens(pa_alloc* a, int64_t req, int32_t n, int64_t* slots_out);

/* [CB-PA] §4.1 shared prefix: `dst` gets the first floor(prefix_tokens /
 * block_size) blocks of `src` (whole blocks only; each refcount + 1) and
 * seq_len = that many full blocks of tokens.  Later appends to either go to
 * private blocks.
 * Errors: NOT_FOUND (src), EXISTS (dst), INVALID_ARG (prefix_tokens < 0 or
 * > seq_len(src)). */
pa_status pa_alloc_fork(pa_alloc* a, int64_t src, int64_t dst, int32_t prefix_tokens);

/* [CB-PA] §3.2 free: decrement the refcount of every block of req's table in
 * order; push the ones reaching zero on the free list in table order (blocks
 * registered by the prefix cache are parked in its LRU instead, see below).
 * Freeing an unknown id is a no-op (PA_OK). */
pa_status pa_alloc_free(pa_alloc* a, int64_t req);

/* Copy req's block table into out[0..cap).  *len_out (nullable) = its length.
 * Errors: NOT_FOUND, INVALID_ARG (cap < length; nothing copied). */
pa_status pa_alloc_get_block_table(const pa_alloc* a, int64_t req, int32_t* out,
                                   int32_t cap, int32_t* len_out);

/* *out = seq_len(req).  Errors: NOT_FOUND, INVALID_ARG (out NULL). */
pa_status pa_alloc_seq_len(const pa_alloc* a, int64_t req, int32_t* out);

/* Slot mapping ([CB-PA] §3.3 address form): slots_out[i] = table[p / block_size]
 * * block_size + p % block_size for p = pos_begin + i, i < n (host int64[n]).
 * Errors: NOT_FOUND, INVALID_ARG (range outside 0..seq_len). */
pa_status pa_alloc_slots(const pa_alloc* a, int64_t req, int32_t pos_begin, int32_t n,
                         int64_t* slots_out);

/* Pack the tables of reqs[0..n) into host int32 tables[n][max_blocks]
 * (padding -1) and seq_lens[n], the form the kernels read.
 * Errors: NOT_FOUND, INVALID_ARG (a table longer than max_blocks; nothing written). */
pa_status pa_alloc_pack(const pa_alloc* a, const int64_t* reqs, int32_t n, int32_t max_blocks,
                        int32_t* tables, int32_t* seq_lens);

/* Counters (see pa_alloc_stats_t). */
pa_status pa_alloc_stats(const pa_alloc* a, pa_alloc_stats_t* out);
/* *out = blocks a take can use now: the free list plus the prefix cache's
 * parked blocks.  O(1).  Errors: INVALID_ARG. */
pa_status pa_alloc_available(const pa_alloc* a, int64_t* out);
/* *out = refcount of physical block `block`.  Errors: INVALID_ARG. */
pa_status pa_alloc_refcount(const pa_alloc* a, int32_t block, int32_t* out);
/* Copy the free list (bottom to top; the next pop takes the last entry).
 * Errors: INVALID_ARG (cap < length; *len_out still set). */
pa_status pa_alloc_free_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* len_out);

/* ---- automatic prefix caching ([CB-PA] §4.1 content-hashed shared blocks,
 * §4.2 Automatic Prefix Caching with an LRU of recently used blocks) ----------
 *
 * A full block's content is identified exactly by its whole token prefix (a
 * prefix-trie node: parent prefix + the block's block_size token ids).  A
 * registered block whose refcount drops to zero is parked in an LRU instead
 * of the free list; any take (allocate, append, allocate_cached) pops the free
 * list first and evicts the least recently parked block when it is empty.
 * Requests are parked last block first, so a prefix outlives its extensions. */

typedef struct {
    int64_t cached_blocks;     /* blocks registered under a prefix node           */
    int64_t evictable_blocks;  /* registered blocks with refcount 0 (the LRU)      */
    int64_t hit_blocks;        /* blocks reused by allocate_cached so far          */
    int64_t evictions;         /* parked blocks taken back for new content         */
    int64_t prefix_nodes;      /* block prefixes in the trie now                   */
} pa_cache_stats_t;

/* Allocate `req` for tokens[0..num_tokens) (host int32 token ids), reusing the
 * cached blocks of the longest cached prefix of whole blocks (refcount + 1,
 * taken out of the LRU) and taking new blocks for the rest; the new full
 * blocks are registered.  *cached_tokens_out (nullable) = reused blocks *
 * block_size: the KV the caller need not recompute or write.  All-or-nothing.
 * Errors: EXISTS, OOM (nothing changes), INVALID_ARG. */
pa_status pa_alloc_allocate_cached(pa_alloc* a, int64_t req, const int32_t* tokens, int32_t num_tokens,
                                   int32_t* cached_tokens_out);
/* The lookup pa_alloc_begin_cached makes, without taking anything: *hit_blocks
 * (nullable) = cached blocks it would reuse for tokens[0..num_tokens), of
 * which *parked_blocks (nullable) now sit in the LRU (a take would remove them
 * from pa_alloc_available's count).  Errors: INVALID_ARG. */
pa_status pa_alloc_cached_prefix(const pa_alloc* a, const int32_t* tokens, int32_t num_tokens,
                                 int32_t* hit_blocks, int32_t* parked_blocks);
/* Start `req` from the prefix cache ([CB-PA] §4.2 inside the §2.2 loop): its
 * table becomes the cached blocks of the longest cached prefix of whole blocks
 * of tokens[0..num_tokens), at most (num_tokens - 1) / block_size of them so
 * that at least one token is left to compute (refcount + 1, taken out of the
 * LRU), and seq_len = those blocks' tokens = *cached_tokens_out (nullable).
 * Nothing new is taken: the caller appends the rest as it computes it.  The
 * request is tracked: every block its appends fill, whose token ids are known
 * (tokens, then pa_alloc_extend_tokens), is registered in the cache under the
 * node of the block before it; tracking ends at the first filled block whose
 * ids are unknown or whose content is already cached in another block.
 * (pa_alloc_allocate_cached also tracks its request, when every full block it
 * holds is its own node's block.)  Errors: EXISTS, INVALID_ARG. */
pa_status pa_alloc_begin_cached(pa_alloc* a, int64_t req, const int32_t* tokens, int32_t num_tokens,
                                int32_t* cached_tokens_out);
/* Append the ids of tokens a tracked request generated to its known ids (a
 * no-op for an untracked request).  Errors: NOT_FOUND, INVALID_ARG. */
pa_status pa_alloc_extend_tokens(pa_alloc* a, int64_t req, const int32_t* ids, int32_t n);
/* Prefix-cache counters.  A cache entry lives as long as its block: when an
 * evicted block's prefix node has no children it is dropped, with every
 * ancestor left without a block and without children, so prefix_nodes stays
 * bounded by the cached blocks and their prefixes. */
pa_status pa_alloc_cache_stats(const pa_alloc* a, pa_cache_stats_t* out);
/* Copy the LRU of parked blocks, least recently parked first (the next
 * eviction takes out[0]).  Errors: INVALID_ARG (cap < length; *len_out set). */
pa_status pa_alloc_evictable_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* len_out);

/* Checkpoint of the allocator's host state (no page describes one; [CB-PA] §4.4's swap moves K/V, not the
 * manager's state): the free-list order, every refcount, each request's block table, length and known
 * token ids, the prefix trie, the cached blocks, the LRU order and the counters, as a versioned
 * little-endian byte string.  Maps are written in key order, so equal states give equal bytes, and the
 * bytes can be compared to diff two allocators.  With buf NULL only *size (the bytes needed) is set and
 * PA_OK returned; otherwise capacity must be >= that size (INVALID_ARG if not, nothing written).  The K/V
 * pool contents are not part of it (they are the caller's device memory).
 * Errors: INVALID_ARG. */
pa_status pa_alloc_serialize(const pa_alloc* a, uint8_t* buf, size_t capacity, size_t* size);

/* Creates an allocator holding a state written by pa_alloc_serialize (resume).  The bytes are checked
 * before use: format and version, every count against the buffer's length, every block id in the pool,
 * no block listed twice in the free list or the LRU, table lengths against request lengths, trie parents
 * present; then the state's consistency: each block's refcount equals the number of request tables
 * holding it, every unreferenced block is either free (unregistered) or parked in the LRU (registered),
 * and each trie node's child count equals the nodes naming it as parent.  On any error nothing is created
 * and *out is NULL.
 * Errors: INVALID_ARG, OOM. */
pa_status pa_alloc_deserialize(const uint8_t* buf, size_t size, pa_alloc** out);

/* ---- swap between the GPU pool and a host pool ([CB-PA] §4.4 Swap: CPU
 * offload, one block manager per pool; §5.4 preemption by swapping) ---------
 *
 * Pools are the K and V pool tensors of two allocators with the same
 * block_size; one block of one pool is `block_bytes` bytes (block_size *
 * num_heads * head_dim * 2 for fp16).  Memory may be device memory or pinned
 * host memory on either side (copies use cudaMemcpyDefault).  Copies are
 * asynchronous on `stream`; the caller keeps the buffers alive until they
 * complete. */

/* Copy K and V blocks: for each pair i, block mapping[2i] of (src_k, src_v)
 * to block mapping[2i+1] of (dst_k, dst_v) (host int64 mapping[num_pairs][2]).
 * Runs of consecutive pairs become one cudaMemcpyAsync each, in list order.
 * num_pairs == 0 or block_bytes == 0 copies nothing.
 * Errors: INVALID_ARG (pair outside [0, src/dst_num_blocks)), CUDA. */
pa_status pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                         const int64_t* mapping, int32_t num_pairs, int64_t block_bytes,
                         int32_t src_num_blocks, int32_t dst_num_blocks, void* stream);

/* Swap `req` out of the GPU pool: allocate it in `cpu` with its seq_len,
 * copy its blocks GPU -> host, free it in `gpu` (its GPU blocks may be
 * reused by work ordered after the copy on `stream`).  Shared blocks are
 * copied and only lose this request's reference.  block_bytes == 0 does the
 * bookkeeping alone.
 * Errors: NOT_FOUND (req not in gpu), EXISTS (req already in cpu), OOM (cpu
 * pool full; nothing changes), INVALID_ARG (block sizes differ), CUDA (the
 * cpu allocation is rolled back). */
pa_status pa_alloc_swap_out(pa_alloc* gpu, pa_alloc* cpu, int64_t req, const void* gpu_k,
                            const void* gpu_v, void* cpu_k, void* cpu_v, int64_t block_bytes,
                            void* stream);
/* The reverse move: allocate `req` in `gpu`, copy host -> GPU, free it in `cpu`.
 * Errors: as pa_alloc_swap_out with the pools exchanged. */
pa_status pa_alloc_swap_in(pa_alloc* gpu, pa_alloc* cpu, int64_t req, void* gpu_k, void* gpu_v,
                           const void* cpu_k, const void* cpu_v, int64_t block_bytes, void* stream);

/* ---- continuous-batching step driver ([CB-PA] §2.2 iteration-level
 * scheduler and mixed prefill/decode batch, §4.3 chunked prefill, §5.3
 * watermark admission, §5.4 preemption by recomputation; [DB] §4.4 loop) -----
 *
 * One step: (1) free requests that produced their last token; (2) while the
 * running decodes need more new blocks than are available, preempt the most
 * recently admitted running request (blocks freed, back to the FRONT of the
 * waiting queue, it will recompute its prompt plus its generated tokens);
 * (3) admit waiting requests in arrival order while fewer than max_num_seqs
 * run and the blocks of the whole prefill + the decodes' needs +
 * watermark_blocks are available; (4) every fully prefilled request decodes
 * one token, then requests still prefilling get chunks, in running order,
 * from a budget of max_num_tokens prefill tokens (whole prompts only when
 * chunked_prefill is 0; a chunk without blocks waits).  The allocator is
 * borrowed (it must outlive the scheduler) and is driven only through its
 * public calls.  Not thread-safe. */

typedef struct pa_sched pa_sched;

typedef struct {
    int32_t max_num_seqs;       /* cap on running requests (= on a step's batch)      */
    int32_t max_num_tokens;     /* prefill-token budget of one step                   */
    int32_t chunked_prefill;    /* 1: split prompts into chunks; 0: whole prompts     */
    int32_t watermark_blocks;   /* blocks admission leaves free                       */
} pa_sched_config_t;

typedef struct {
    int64_t step;               /* index of this step                                 */
    int32_t num_prefill;        /* prefill entries                                    */
    int32_t num_decode;         /* decode entries                                     */
    int32_t num_tokens;         /* rows of the step's slot mapping                    */
    int32_t num_admitted;
    int32_t num_preempted;
    int32_t num_finished;       /* requests freed at the start of this step           */
} pa_step_info_t;

typedef struct {
    int32_t state;              /* 0 waiting, 1 running, 2 finished, 3 swapped out    */
    int32_t prompt_len;
    int32_t max_new_tokens;
    int32_t prefilled;          /* tokens of the current prefill already cached       */
    int32_t to_prefill;         /* prompt (+ generated tokens after a preemption)     */
    int32_t generated;
    int32_t preemptions;
    int32_t pad_;
    int64_t first_token_step;   /* step that emitted its first token, -1 if none      */
    int64_t finish_step;        /* step that emitted its last token, -1 if none       */
} pa_request_info_t;

typedef struct {
    int64_t steps, waiting, running, finished, preemptions, prefill_tokens, decode_tokens;
    int64_t cached_tokens;      /* prompt tokens admission found in the prefix cache  */
    int64_t swapped;            /* requests swapped out now                           */
    int64_t swap_outs, swap_ins;  /* moves so far                                     */
} pa_sched_stats_t;

/* Errors: INVALID_ARG (NULL, non-positive caps, negative watermark). */
pa_status pa_sched_create(pa_alloc* alloc, const pa_sched_config_t* cfg, pa_sched** out);
void pa_sched_destroy(pa_sched* s);
/* Queue a request (arrival order = call order).  Errors: INVALID_ARG
 * (prompt_len or max_new_tokens <= 0), EXISTS (id known to the scheduler or
 * holding blocks in the allocator). */
pa_status pa_sched_add_request(pa_sched* s, int64_t req, int32_t prompt_len, int32_t max_new_tokens);
/* As pa_sched_add_request, with the prompt's token ids (host int32
 * tokens[prompt_len], copied): the request goes through the allocator's
 * prefix cache ([CB-PA] §4.2 in the §2.2 loop).  Admission looks up the
 * longest cached prefix of the ids known so far (pa_alloc_cached_prefix),
 * needs new blocks only for the rest, and starts the request from it
 * (pa_alloc_begin_cached): those tokens are not prefilled again
 * (pa_request_info_t.prefilled starts there).  The blocks its chunks and
 * decodes fill become cacheable, and so do its generated tokens when their
 * ids are reported with pa_sched_complete_tokens.  Errors: as
 * pa_sched_add_request, INVALID_ARG (tokens NULL). */
pa_status pa_sched_add_request_tokens(pa_sched* s, int64_t req, const int32_t* tokens, int32_t prompt_len,
                                      int32_t max_new_tokens);
/* Schedule one step (host buffers, any may be NULL): prefill_reqs /
 * prefill_ctx (tokens already cached) / prefill_len (chunk) and decode_reqs /
 * decode_seq_lens (including the new token) hold up to max_num_seqs entries;
 * slot_mapping up to max_num_tokens + max_num_seqs rows: the prefill chunks'
 * rows in prefill order, then one row per decode.  A request's prefill rows
 * are its positions prefill_ctx .. prefill_ctx + prefill_len - 1.
 * Errors: INVALID_ARG (previous step not completed). */
pa_status pa_sched_step(pa_sched* s, pa_step_info_t* info, int64_t* prefill_reqs, int32_t* prefill_ctx,
                        int32_t* prefill_len, int64_t* decode_reqs, int32_t* decode_seq_lens,
                        int64_t* slot_mapping);
/* Apply the scheduled step after its kernels ran: chunks become cached; a
 * request whose prefill completed, and each decode, emits one token; a request
 * that emitted max_new_tokens finishes (freed at the next step).
 * Errors: INVALID_ARG (no open step). */
pa_status pa_sched_complete(pa_sched* s);
/* pa_sched_complete, reporting the ids of the tokens the step emitted
 * (host int32 ids[n], one per emitted token, in emission order: the requests
 * whose prefill completed, in prefill order, then every decode); the ids of
 * requests added with tokens extend their known ids.
 * Errors: INVALID_ARG (no open step; n differs from the tokens emitted:
 * nothing is applied). */
pa_status pa_sched_complete_tokens(pa_sched* s, const int32_t* ids, int32_t n);

/* Swap preemption ([CB-PA] §5.4 strategy 2 "Swap to CPU", §4.4 SwappingManager).
 * With a CPU-side allocator attached (same block_size; NULL detaches, allowed
 * only while nothing is swapped out), a preempted request is moved to the CPU
 * pool (pa_alloc_swap_out bookkeeping, no data moved by the scheduler) instead
 * of being freed, keeping its progress; if the CPU pool cannot take it, it is
 * recomputed as without swapping.  Each step first brings swapped requests
 * back (most recently preempted first) while seats are free and the blocks of
 * their table, plus one if their next decode opens a block, plus the
 * decodes' needs and the watermark are available, and admits no waiting
 * request while one is still swapped out.  The allocator is borrowed and must
 * outlive the scheduler.  Errors: INVALID_ARG (NULL scheduler, block sizes
 * differ, a step is open, detaching while requests are swapped out). */
pa_status pa_sched_enable_swap(pa_sched* s, pa_alloc* cpu);
/* The block moves of the last scheduled step, which the caller performs before
 * the step's kernels, swap-outs first (e.g. pa_swap_blocks GPU -> CPU pool,
 * then CPU -> GPU): out_pairs[2i], out_pairs[2i+1] = (GPU block, CPU block) of
 * a swap-out; in_pairs likewise (CPU block, GPU block).  Host int64 arrays of
 * capacity out_cap / in_cap pairs (either may be NULL); *n_out / *n_in
 * (nullable) = the pair counts.  Errors: INVALID_ARG (NULL scheduler; a
 * capacity below its count, nothing copied). */
pa_status pa_sched_last_swaps(const pa_sched* s, int64_t* out_pairs, int32_t out_cap, int32_t* n_out,
                              int64_t* in_pairs, int32_t in_cap, int32_t* n_in);
pa_status pa_sched_request_info(const pa_sched* s, int64_t req, pa_request_info_t* out);
pa_status pa_sched_stats(const pa_sched* s, pa_sched_stats_t* out);

/* ---- device kernels -------------------------------------------------------- */

/* reshape_and_cache: write the step's new K/V rows into the pool.
 * For t < num_tokens with s = slot_mapping[t] >= 0:
 *   k_cache[s / block_size][s % block_size][h][d] = k_new[t][h][d]   (same for V)
 * Tokens with a negative slot are padding and skipped.  Bit-exact copy.
 * k_new, v_new: device fp16 [num_tokens][num_heads][head_dim].
 * k_cache, v_cache: device fp16 [num_blocks][block_size][num_heads][head_dim].
 * slot_mapping: device int64 [num_tokens].  Slots >= num_blocks*block_size are
 * skipped and flagged PA_DEVCHK_SLOT.  Rows of k_new/v_new and of the cache
 * must be 16-byte aligned (num_heads*head_dim*2 % 16 == 0).
 * Source: the slots come from append_token ([CB-PA] §3.2) and are the
 * addresses the attention kernel reads ([CB-PA] §3.3).
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
pa_status pa_reshape_and_cache(const pa_half* k_new, const pa_half* v_new,
                               pa_half* k_cache, pa_half* v_cache,
                               const int64_t* slot_mapping, int32_t num_tokens,
                               int32_t num_heads, int32_t head_dim, int32_t block_size,
                               int32_t num_blocks, int32_t* err_flag, void* stream);

/* Bytes of device workspace pa_paged_attention_decode needs for `num_seqs`
 * sequences whose block tables have `max_blocks` columns.  0 on bad arguments. */
size_t pa_decode_workspace_bytes(int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                 int32_t max_blocks, int32_t block_size);

/* Decode attention over the paged cache ([CB-PA] §3.3 paged_attention_kernel,
 * completed with its omitted weighted sum of V; §1.1 decode phase).
 * For every sequence s < num_seqs and head h:
 *   n = seq_lens[s] (including the token decoded in this step, whose K/V must
 *   already be in the cache); position j < n lives in physical block
 *   block_tables[s][j / block_size] at row j % block_size;
 *   out[s][h] = sum_j softmax_j(scale * q[s][h] . K_j[h]) V_j[h].
 * A sequence with n == 0 gets zeros.  Table entries at or beyond
 * ceil(n / block_size) are never read (they may hold anything).
 * out, q: device fp16 [num_seqs][num_heads][head_dim] (16-byte aligned).
 * k_cache, v_cache: as above (16-byte aligned base).
 * block_tables: device int32 [num_seqs][max_blocks]; seq_lens: device int32 [num_seqs].
 * workspace: device, >= pa_decode_workspace_bytes(num_seqs, num_heads, head_dim,
 * max_blocks, block_size) bytes, 256-byte aligned, caller-owned scratch whose
 * contents need no initialisation and are clobbered; two launches in flight
 * at once must not share it.
 * scale: the softmax temperature (1/sqrt(head_dim) for standard attention);
 * it must be finite and > 0, anything else returns INVALID_ARG.
 * The work is split flash-decoding style into partitions of the sequence
 * combined with the exact log-sum-exp rule, so the result does not depend on
 * the physical placement of the blocks (bitwise) and matches a float64
 * reference to about 1e-3.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
pa_status pa_paged_attention_decode(pa_half* out, const pa_half* q,
                                    const pa_half* k_cache, const pa_half* v_cache,
                                    const int32_t* block_tables, const int32_t* seq_lens,
                                    int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                    int32_t block_size, int32_t max_blocks, int32_t num_blocks,
                                    float scale, void* workspace, size_t workspace_bytes,
                                    int32_t* err_flag, void* stream);

/* pa_paged_attention_decode for callers that cannot allocate device memory.
 * The pages describe no counterpart of this entry point; it exists for code
 * that is handed fixed buffers and may not call cudaMalloc (allocator-less
 * embedded loops, plugins whose host forbids allocation after start-up,
 * latency-critical paths that must avoid cudaMalloc's implicit
 * synchronisation).  Same arguments and results as pa_paged_attention_decode
 * minus the workspace: the scratch comes from a fixed 64 MiB (67108864-byte)
 * array that the library keeps in device memory on every GPU that loads it,
 * until the process exits.  A batch whose pa_decode_workspace_bytes exceeds
 * that returns PA_ERR_INVALID_ARG with a message saying so.  The first call on
 * a device looks the array's address up (cudaGetSymbolAddress, with that
 * device current); make that first call before any stream capture.  The
 * address is kept for the life of the process: after cudaDeviceReset (which
 * destroys the device's copy of the array) it is stale, so a process that
 * resets a device must not call this entry point on it again.  Calls on
 * one device share the array: calls whose kernels may overlap on the GPU race
 * and must be serialised by the caller.  Allocates nothing.
 * Errors: as pa_paged_attention_decode. */
pa_status pa_paged_attention_decode_noalloc(pa_half* out, const pa_half* q,
                                            const pa_half* k_cache, const pa_half* v_cache,
                                            const int32_t* block_tables, const int32_t* seq_lens,
                                            int32_t num_seqs, int32_t num_heads, int32_t head_dim,
                                            int32_t block_size, int32_t max_blocks, int32_t num_blocks,
                                            float scale, int32_t* err_flag, void* stream);

/* Chunked-prefill attention over the paged cache ([CB-PA] §4.3 Chunked
 * Prefill; §1.1 prefill phase).  Request b < num_reqs owns query rows
 * q_start[b] .. q_start[b+1]-1 (host-unknown, device int32 [num_reqs+1],
 * q_start[0] = 0, non-decreasing, q_start[num_reqs] <= num_tokens); its row i
 * sits at absolute position p = ctx_before[b] + i and attends causally to
 * positions 0..p of its own sequence through block_tables[b]:
 *   out[row][h] = sum_{j<=p} softmax_j(scale * q[row][h] . K_j[h]) V_j[h].
 * The chunk's own K/V must already be in the cache (pa_reshape_and_cache
 * first).  q, out: device fp16 [num_tokens][num_heads][head_dim];
 * block_tables: device int32 [num_reqs][max_blocks]; ctx_before: device int32
 * [num_reqs].  Rows of out not covered by any request are left unwritten.
 * scale must be finite and > 0 (INVALID_ARG otherwise).
 * QK^T and PV run on the tcgen05 tensor cores (fp16 operands, fp32 TMEM
 * accumulators); the softmax runs in fp32.
 * Errors: INVALID_ARG, UNSUPPORTED, CUDA. */
pa_status pa_paged_attention_prefill_chunk(pa_half* out, const pa_half* q,
                                           const pa_half* k_cache, const pa_half* v_cache,
                                           const int32_t* block_tables, const int32_t* q_start,
                                           const int32_t* ctx_before, int32_t num_reqs,
                                           int32_t num_tokens, int32_t num_heads, int32_t head_dim,
                                           int32_t block_size, int32_t max_blocks,
                                           int32_t num_blocks, float scale,
                                           int32_t* err_flag, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PAGEDKV_H */
