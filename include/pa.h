/*
 * pa.h -- C ABI of the paged decode attention library (libpa370.so).
 *
 * What the library computes is defined by three web pages on vLLM's
 * PagedAttention:
 *   [P1] "大语言模型推理内存管理算法 paged attention"
 *        (https://www.cnblogs.com/wljss/p/20424559)
 *   [P2] "PagedAttention 核心思想解析"
 *        (https://intelliparadigm.com/article/weixin_29574585/2267096)
 *   [P3] "08. PagedAttention：把 KV Cache 分页管理"
 *        (https://niuwancheng.cn/blog/docs/ai/llm-inference/08-paged-attention.html)
 *
 * Conventions shared by every entry point:
 *  - Device operations take raw device pointers owned by the caller and
 *    enqueue work on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream). They never synchronise the host and never
 *    allocate device memory; split-context scratch is the caller's
 *    `workspace`.
 *  - Shapes and dtypes are checked on the host before any launch; a bad
 *    argument returns PA_ERR_INVALID and launches nothing. A failed launch
 *    returns PA_ERR_CUDA.
 *  - Data that only the device sees (block ids, slots, lengths) is checked
 *    by the kernels themselves: an out-of-range value skips the access that
 *    would have used it and sets a bit in a device-side error word, which
 *    pa_device_status() reads. A kernel never faults on such input; its
 *    output is then undefined.
 *  - KV pool layout (the pages fix none; this library's contract): K and V
 *    are separate pools of shape [num_blocks][num_kv_heads][block_size]
 *    [head_dim], row-major, elements fp16 or bf16. One (block, kv head)
 *    tile is block_size * head_dim contiguous elements. The pools must be
 *    16-byte aligned.
 *  - A slot names one token position of the pool: slot = physical_block *
 *    block_size + offset_in_block [P3, section "为什么叫 PagedAttention"].
 *  - Query head h attends with KV head h / (num_q_heads / num_kv_heads)
 *    (grouped-query attention [P1, section 6]).
 */
#ifndef PA370_H
#define PA370_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID = -1,       /* bad argument (shape, dtype, pointer, alignment) */
    PA_ERR_OUT_OF_BLOCKS = -2, /* allocator: not enough free blocks; nothing changed */
    PA_ERR_STATE = -3,         /* allocator: unknown/duplicate sequence, bad reference count */
    PA_ERR_CUDA = -4,          /* a CUDA runtime call failed */
    PA_ERR_UNSUPPORTED = -5    /* valid but not compiled in (e.g. a head_dim/group combination) */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Bits of the device-side error word (see pa_device_status). */
#define PA_DEVERR_BLOCK_ID 1     /* a block table entry was outside [0, num_blocks) */
#define PA_DEVERR_SLOT 2         /* a slot was >= num_blocks * block_size */
#define PA_DEVERR_COPY_PAIR 4    /* a copy pair named a block outside the pool */
#define PA_DEVERR_CONTEXT_LEN 8  /* a context length exceeded the table or max_context_len */
#define PA_DEVERR_TIMEOUT 16     /* a pipeline wait gave up (the kernel returned early) */

/* ------------------------------------------------------------------------------------------
 * pa_reshape_and_cache -- store the K and V of new tokens at their slots.
 * [P3, section "为什么叫 PagedAttention": a new token's K and V are written to
 * the position of the physical block it belongs to; slot = block_table[logical
 * block] * block_size + offset, then a small GPU kernel writes each token's K/V
 * to its slot.]
 *
 *   k_new, v_new   device, [num_tokens][num_kv_heads][head_dim], dtype, contiguous
 *   slot_mapping   device, int64 [num_tokens]; a negative slot marks padding and
 *                  is skipped; slots must be distinct (duplicates: undefined)
 *   k_cache, v_cache  device pools (layout above), updated in place
 * Bit-exact element copy. Returns PA_OK (num_tokens == 0 launches nothing).
 * ------------------------------------------------------------------------------------------ */
pa_status pa_reshape_and_cache(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                               int num_tokens, void *k_cache, void *v_cache, int num_blocks,
                               int num_kv_heads, int block_size, int head_dim, pa_dtype dtype,
                               void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_copy_blocks -- the device half of copy-on-write.
 * [P2, section 2.3: when a sequence must modify a shared block, a new
 * physical block is allocated, the original block's contents are copied
 * into it, the block table is updated and the old block's ref_count drops;
 * P1, section 9.]
 *
 *   block_pairs   device, int64 [num_pairs][2] = (src, dst) physical ids
 * For each pair the whole block -- every KV head, every slot, K and V -- is
 * copied bit-exactly. Destinations must be distinct and no destination may
 * be a source of another pair (undefined otherwise); src == dst is a no-op.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_pairs, int num_pairs,
                         int num_blocks, int num_kv_heads, int block_size, int head_dim,
                         pa_dtype dtype, void *stream);

/* ------------------------------------------------------------------------------------------
 * Host swap space -- blocks moved out of the device pool and back.
 * [P3, section "分页还顺带解决了什么": under memory pressure a request's blocks
 * may be moved to CPU memory and brought back later, which same-size blocks
 * make easy. P2, section 3.1: swap_out of a preempted victim; section 6.1: a
 * CPU swap space of configurable size.]
 *
 * pa_swap_space_create allocates pinned host memory for num_host_blocks
 * blocks of K and of V, laid out like the device pools ([num_host_blocks]
 * [num_kv_heads][block_size][head_dim], the given dtype), and maps it into
 * the current device's address space. This is the library's only
 * allocation, made once, off the hot path; pa_swap_space_destroy frees it.
 * pa_swap_space_pools returns the host addresses of the two pools (for
 * inspection or checkpointing). PA_ERR_CUDA if the pinned allocation fails.
 *
 * pa_swap_out copies, for each pair (device block, host block) of
 * block_pairs, the whole device block (every KV head and slot, K and V) into
 * the host block; pa_swap_in copies pairs (host block, device block) back.
 * One launch moves all pairs; stream-ordered like every device op, so a
 * device block freed by pa_alloc_swap_out may be reused by later work on the
 * same stream. block_pairs: device-accessible int64 [num_pairs][2]. An id
 * outside its pool skips that pair and sets PA_DEVERR_COPY_PAIR. Destinations
 * must be distinct (undefined otherwise). The device pools must have the
 * swap space's block shape.
 * ------------------------------------------------------------------------------------------ */
typedef struct pa_swap_space pa_swap_space;

pa_status pa_swap_space_create(int num_host_blocks, int num_kv_heads, int block_size, int head_dim,
                               pa_dtype dtype, pa_swap_space **out);
void pa_swap_space_destroy(pa_swap_space *space);
pa_status pa_swap_space_pools(const pa_swap_space *space, void **k_host, void **v_host);
pa_status pa_swap_out(const pa_swap_space *space, const void *k_cache, const void *v_cache,
                      int num_blocks, const int64_t *block_pairs, int num_pairs, void *stream);
pa_status pa_swap_in(const pa_swap_space *space, void *k_cache, void *v_cache, int num_blocks,
                     const int64_t *block_pairs, int num_pairs, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_decode -- paged attention for one query token per sequence.
 * [P1, section 5: out = softmax(Q K^T / sqrt(d)) V, where the kernel finds
 * each token's logical block and maps it through the block table to the
 * physical block holding its K/V; section 6: the formula is unchanged by
 * paging. P3, section "它没有解决什么": each decode step reads the whole
 * history. P2, section 2.2: scores are computed per KV block and the partial
 * results merged.]
 *
 *   out            device, [num_seqs][num_q_heads][head_dim], dtype; rounded to
 *                  nearest-even from fp32
 *   q              device, [num_seqs][num_q_heads][head_dim], dtype
 *   block_tables   device, int32 [num_seqs][max_blocks_per_seq]; entries past
 *                  ceil(context_lens[b] / block_size) are never read
 *   context_lens   device, int32 [num_seqs]; tokens of each sequence to attend
 *                  over (including the one just written); 0 yields zeros
 *   max_context_len  host int >= every context_lens[b] (sizes the grid; no
 *                  device-to-host read is made)
 *   scale          softmax scale, normally 1/sqrt(head_dim)
 *   workspace      device scratch of at least pa_decode_workspace_size() bytes
 *                  (same arguments, same current device), 16-byte aligned; may
 *                  be NULL when that size is 0. Zero-fill it once before its
 *                  first use: its first 64 KiB hold counters that every
 *                  completed call leaves at zero (after a call that reported
 *                  PA_DEVERR_TIMEOUT, zero-fill it again). Two calls that share
 *                  a workspace must not overlap on the device
 *   partition_tokens  0 for the library's choice, or a positive multiple of 64
 *                  (at most 8192): about that many tokens of one kv head per
 *                  CTA (smaller values split the work more finely)
 * Supported: head_dim in {64, 128}; num_q_heads / num_kv_heads in {1,2,4,8};
 * any block_size >= 1 with partition_tokens / block_size <= 4094.
 * Kernels: with 2-8 q heads per kv head and a power-of-two block_size >= 8,
 * one persistent wave of CTAs splits all (sequence, kv head) tokens evenly
 * (tensor cores, TMA); a sequence split between CTAs has its partial
 * (max, sum, weighted V) states merged by log-sum-exp by the CTA that
 * finishes last. Otherwise a SIMT kernel processes fixed partitions of
 * partition_tokens tokens (0: pa_decode_default_partition) and a second
 * kernel on the same stream merges them.

 * ------------------------------------------------------------------------------------------ */
size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                int max_context_len, int partition_tokens);

pa_status pa_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                    const int32_t *block_tables, int max_blocks_per_seq,
                    const int32_t *context_lens, int max_context_len, int num_seqs,
                    int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                    int num_blocks, float scale, pa_dtype dtype, void *workspace,
                    size_t workspace_bytes, int partition_tokens, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_decode_static_workspace -- pa_decode for callers that cannot allocate device
 * memory. (The pages have no counterpart: this is a deployment convenience.)
 *
 * Some callers have no way to obtain device scratch: code that runs where a
 * cudaMalloc would break a memory budget or an allocator they do not own (a
 * host framework's pooled allocator, a plug-in restricted to the buffers it is
 * handed), or that must not allocate on a latency-critical path. This entry
 * point takes the same arguments as pa_decode minus the workspace: the
 * split-context scratch is a fixed device array of PA_STATIC_WORKSPACE_BYTES
 * inside the library, which every GPU that loads the library holds until the
 * process exits. The caller still passes q, the pools, the tables, the lengths
 * and the output.
 *  - Calls whose kernel would need more scratch than PA_STATIC_WORKSPACE_BYTES
 *    return PA_ERR_UNSUPPORTED and launch nothing. The need is that of the
 *    kernel the call runs (for the given block_size), which is at most
 *    pa_decode_workspace_size.
 *  - The first call on a device (made with that device current) looks up the
 *    array's device address; make that first call before any stream capture.
 *    Only a successful lookup is kept (a failure returns PA_ERR_CUDA and the
 *    next call tries again).
 *  - No device memory is allocated or freed, by this library or any other.
 *  - All calls share the one array and it keeps the last call's contents. Its
 *    first 64 KiB hold the even-split kernel's counters, which a call expects
 *    at zero and which a call that gave up a wait (PA_DEVERR_TIMEOUT) may leave
 *    non-zero; so every call first clears them on `stream` (a memset, not an
 *    allocation) before its kernels. Calls whose work overlaps on the GPU
 *    (other streams, other host threads) race on the array -- one may clear or
 *    overwrite what the other is using, and both outputs are then undefined:
 *    serialise them.
 * ------------------------------------------------------------------------------------------ */
#define PA_STATIC_WORKSPACE_BYTES (16u << 20)

pa_status pa_decode_static_workspace(void *out, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *block_tables,
                                     int max_blocks_per_seq, const int32_t *context_lens,
                                     int max_context_len, int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, float scale, pa_dtype dtype,
                                     int partition_tokens, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_decode_append -- one decode step: store every sequence's new K/V at its slot,
 * then attend (pa_reshape_and_cache followed by pa_decode, in one call).
 * [P3, section "为什么叫 PagedAttention" (the slot write) and the sources of
 * pa_decode above; the order -- write, then attend over a history that includes
 * the new token -- is this library's reading.]
 *
 *   k_new, v_new   device, [num_seqs][num_kv_heads][head_dim]: the new token of
 *                  sequence b, which is its position context_lens[b] - 1
 *   slot_mapping   device, int64 [num_seqs]: that token's slot; -1 stores nothing
 *                  (pass -1 for sequences with context_lens[b] == 0)
 *   k_cache, v_cache  updated in place; all other arguments as pa_decode
 * Result: identical pools to pa_reshape_and_cache, outputs within the rounding
 * of pa_decode. Where pa_decode runs its even-split kernel (2-8 q heads per kv
 * head, power-of-two block_size >= 8) the write happens inside that kernel: the
 * CTA that reads a sequence's last tile stores the new rows and uses them
 * directly (one launch per step). Otherwise the write kernel runs first.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                           const int64_t *slot_mapping, void *k_cache, void *v_cache,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int max_context_len, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float scale, pa_dtype dtype, void *workspace,
                           size_t workspace_bytes, int partition_tokens, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_decode_window / pa_decode_append_window -- decode over a sliding window.
 * [P2, section 5.2: a sliding window reclaims the blocks that fall out of it.]
 * Each sequence of length len attends only to its last `window` positions,
 * [max(0, len - window), len): softmax over those scores, the same arithmetic
 * as pa_decode otherwise. Block-table entries of blocks wholly before that
 * range are never read, so they may hold anything -- e.g. the -1 that
 * pa_alloc_slide_window leaves. Arguments as pa_decode / pa_decode_append plus
 * `window` (> 0; PA_ERR_INVALID otherwise); pa_decode_workspace_size covers it.
 * Where pa_decode runs its even-split kernel and block_size <= 64, that kernel
 * (one launch) sees each sequence as the part of it from the block holding its
 * first attended position on -- its table read that many blocks further on, its
 * length shorter by as many positions -- and masks that block's positions
 * before the window. pa_decode_append_window writes the new tokens inside that
 * kernel, as pa_decode_append does; pa_decode_append_window_overlapped is the
 * same call with the programmatic early start and contract of
 * pa_decode_append_overlapped (on any other shape it is pa_decode_append_window).
 * Otherwise a window runs in the partition kernel (partitions of the window's
 * positions, then the merge kernel when the longest context has more than one),
 * and pa_decode_append_window writes the new tokens with pa_reshape_and_cache
 * first. pa_decode_window_launches and pa_decode_append_window_launches give
 * the kernels each call launches.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_decode_window(void *out, const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *block_tables, int max_blocks_per_seq,
                           const int32_t *context_lens, int max_context_len, int num_seqs,
                           int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float scale, int window, pa_dtype dtype,
                           void *workspace, size_t workspace_bytes, int partition_tokens,
                           void *stream);
int pa_decode_window_launches(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                              int block_size, int num_blocks, int max_context_len, int window,
                              int partition_tokens);
int pa_decode_append_window_launches(int num_seqs, int num_q_heads, int num_kv_heads,
                                     int head_dim, int block_size, int num_blocks,
                                     int max_context_len, int window, int partition_tokens);
pa_status pa_decode_append_window(void *out, const void *q, const void *k_new, const void *v_new,
                                  const int64_t *slot_mapping, void *k_cache, void *v_cache,
                                  const int32_t *block_tables, int max_blocks_per_seq,
                                  const int32_t *context_lens, int max_context_len, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int num_blocks, float scale, int window, pa_dtype dtype,
                                  void *workspace, size_t workspace_bytes, int partition_tokens,
                                  void *stream);
pa_status pa_decode_append_window_overlapped(
    void *out, const void *q, const void *k_new, const void *v_new, const int64_t *slot_mapping,
    void *k_cache, void *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
    const int32_t *context_lens, int max_context_len, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale, int window,
    pa_dtype dtype, void *workspace, size_t workspace_bytes, int partition_tokens, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_prefill -- paged attention for several query tokens per sequence (a prompt, or one
 * chunk of a chunked prefill).
 * [P2, section 2.2: the rows of Q are cut into blocks, each block is scored against the
 * sequence's K/V blocks found through the block table, and the partial results are merged
 * by position. P3, section "借用操作系统的办法：分页": a request's prefill takes the blocks
 * it needs.]
 *
 *   q             device, [num_tokens][num_q_heads][head_dim]: the query tokens of every
 *                 sequence back to back, sequence b's rows q_start[b] .. q_start[b+1]-1
 *   q_start       device, int32 [num_seqs + 1], q_start[0] = 0, non-decreasing,
 *                 q_start[num_seqs] = num_tokens
 *   context_lens  device, int32 [num_seqs]: positions of each sequence, the query tokens
 *                 included -- they are its last q_start[b+1]-q_start[b] positions, and
 *                 their K/V must already be in the pool (pa_reshape_and_cache)
 *   max_q_len     host: the largest q_start[b+1]-q_start[b] (sizes the grid)
 *   window        0, or > 0: each token attends to its last `window` positions only
 *   out           device, [num_tokens][num_q_heads][head_dim], same dtype as q
 * The token at position p of its sequence attends to positions [lo, p], lo = 0 or
 * p + 1 - window: softmax(scale * q . K^T) V over those positions, fp32 arithmetic.
 * head_dim 64 or 128; block_size a power of two >= 8 (PA_ERR_UNSUPPORTED otherwise).
 * Allocates nothing. Lengths or q_start entries out of range are clamped and reported
 * (PA_DEVERR_CONTEXT_LEN); bad block ids are skipped and reported (PA_DEVERR_BLOCK_ID).
 * Stream work: a one-CTA kernel that writes the device's item order -- the (sequence,
 * query tile) pairs by the number of key tiles they read, most first -- and clears the
 * device's work counter (past 16,384 pairs: a 4-byte clear of the counter only, and
 * items in index order), then one persistent kernel: one CTA per SM takes items from
 * that counter in that order. An item is 128 query tokens of two q heads of one kv head
 * (an even number of q heads per kv head), else 256 query tokens of one q head. The
 * order and the counter are one per device and per library: two pa_prefill calls on one
 * device must not run at the same time (issue them on one stream, or order their
 * streams). The order changes which CTA computes an item and when, never its result.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *context_lens, const int32_t *q_start, int num_seqs,
                     int num_tokens, int max_q_len, int max_context_len, int num_q_heads,
                     int num_kv_heads, int head_dim, int block_size, int num_blocks, float scale,
                     int window, pa_dtype dtype, void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_decode_append_overlapped -- pa_decode_append whose kernel may start before the kernel
 * launched before it on the same stream has finished (programmatic dependent launch), so
 * its start-up -- scanning the lengths, locating its tiles, fetching the first block ids --
 * overlaps the end of that kernel. It reads context_lens, block_tables and slot_mapping
 * before waiting for the preceding kernel, and q, k_new, v_new and the pools after.
 * Contract: those three arrays must not be written by the immediately preceding kernel
 * (e.g. they are uploaded or prepared before it). Same arguments and results as
 * pa_decode_append; without the even-split kernel (block size, GQA group) it is
 * pa_decode_append.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_decode_append_overlapped(void *out, const void *q, const void *k_new,
                                      const void *v_new, const int64_t *slot_mapping,
                                      void *k_cache, void *v_cache, const int32_t *block_tables,
                                      int max_blocks_per_seq, const int32_t *context_lens,
                                      int max_context_len, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, int block_size,
                                      int num_blocks, float scale, pa_dtype dtype,
                                      void *workspace, size_t workspace_bytes,
                                      int partition_tokens, void *stream);

/* Kernels one pa_decode_append call with these arguments launches (0 if none). */
int pa_decode_append_launches(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                              int block_size, int num_blocks, int max_context_len,
                              int partition_tokens);

/* CTAs of the even-split kernel a pa_decode call with these arguments launches (one
 * persistent wave on the current device by default), or 0 when the call runs the
 * partition kernel instead. For accounting (e.g. the split-context scratch bytes). */
int pa_decode_grid_ctas(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int max_context_len,
                        int partition_tokens);

/* Kernels one pa_decode call with these arguments launches (0 if none). */
int pa_decode_launches(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                       int block_size, int num_blocks, int max_context_len, int partition_tokens);

/* The partition size pa_decode uses for partition_tokens == 0. */
int pa_decode_default_partition(int num_seqs, int num_kv_heads, int max_context_len);

/* ------------------------------------------------------------------------------------------
 * pa_device_status -- read and clear the device-side error word (PA_DEVERR_*
 * bits) after the work queued on `stream` has finished. Synchronises
 * `stream`; meant for tests and debugging, not the hot path.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_device_status(void *stream, int32_t *code);

/* ------------------------------------------------------------------------------------------
 * pa_hbm_read -- a measurement utility, not part of the method (the pages have no
 * counterpart): reads `bytes` of device memory at `buf` once, as a read-only stream, so
 * that a caller can time this GPU's read rate beside the kernels that are bound by it.
 *
 *   buf          device, `bytes` bytes, 16-byte aligned; only read
 *   bytes        > 0, a multiple of 16; larger than L2 (126 MB) to measure HBM
 *   sink         device, one uint32: cleared on `stream`, then the XOR of every 32-bit
 *                word of the buffer (written so that the loads cannot be dropped)
 *   ctas_per_sm  1..4: CTAs of 512 threads launched per SM
 * Stream work: a 4-byte clear and one kernel (16-byte evict-first loads, four in flight
 * per thread). Allocates nothing. PA_ERR_INVALID for a null or misaligned pointer, a size
 * that is 0 or not a multiple of 16, or ctas_per_sm outside 1..4.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_hbm_read(const void *buf, size_t bytes, uint32_t *sink, int ctas_per_sm,
                      void *stream);

/* ------------------------------------------------------------------------------------------
 * pa_debug_wait_test -- test hook for the bounded waits of the decode kernels (not for
 * production use; the pages have no counterpart).
 * Every wait of a decode kernel is bounded: a wait that runs out sets PA_DEVERR_TIMEOUT,
 * and the kernel then runs to its end without waiting for data again (so every warp
 * reaches every barrier), issues no further copy, skips the fused KV write, and
 * returns; its outputs are undefined, everything it writes stays in bounds, and the
 * context stays usable. With enable != 0, every later pa_decode* launch runs in a test
 * mode that makes this happen on purpose and safely: its producer warps issue no copy
 * and arrive on no data barrier, and its consumer warps give up each data wait after
 * consumer_wait_ns nanoseconds (0 < consumer_wait_ns <= 2e9). No copy is then in flight
 * when a CTA exits. enable == 0 restores normal launches (waits bounded at 2 s).
 * Process-wide and not thread-safe: set it only while no other thread launches decode
 * work. PA_ERR_INVALID for an out-of-range limit.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_debug_wait_test(int enable, long long consumer_wait_ns);

/* Human-readable name of a status code (static storage). */
const char *pa_status_string(pa_status status);

/* ------------------------------------------------------------------------------------------
 * pa_slot_mapping -- host helper: the slot of every position [0, count) of
 * each sequence, from its block table (for writing a prompt's K/V).
 * [P3, section "为什么叫 PagedAttention", slot formula.]
 *   block_tables  host int32 [num_seqs][max_blocks_per_seq]
 *   counts        host int32 [num_seqs]: positions to map per sequence
 *   slots         host int64 output, sum(counts) entries, sequence-major
 * Returns PA_ERR_INVALID if a count exceeds the table width.
 * ------------------------------------------------------------------------------------------ */
pa_status pa_slot_mapping(const int32_t *block_tables, int max_blocks_per_seq,
                          const int32_t *counts, int num_seqs, int block_size, int64_t *slots);

/* ==========================================================================================
 * Host-side block manager (off the hot path; not thread-safe; one per pool).
 * [P1, sections 7-8: blocks are allocated on demand -- a new one only when the
 * last block is full -- and returned to a free list when the request ends, for
 * immediate reuse. P3, section "借用操作系统的办法：分页": same; section
 * "分页还顺带解决了什么": blocks shared by several tables carry a reference
 * count. P2, section 2.3: copy-on-write. P2, section 5.1: forking sampled
 * sequences from a shared prompt. P2, section 5.2: sliding-window release.]
 * Which free block is handed out is not part of the contract.
 * ========================================================================================== */
typedef struct pa_alloc pa_alloc;

pa_status pa_alloc_create(int num_blocks, int block_size, pa_alloc **out);
void pa_alloc_destroy(pa_alloc *a);

/* New sequence holding num_tokens tokens (a prompt): ceil(num_tokens / block_size)
 * blocks, all or none (PA_ERR_OUT_OF_BLOCKS leaves the state unchanged). */
pa_status pa_alloc_add_seq(pa_alloc *a, int64_t seq_id, int num_tokens);

/* child shares every block of parent (each block's ref_count += 1). */
pa_status pa_alloc_fork(pa_alloc *a, int64_t parent, int64_t child);

/* Reserve the slot of the sequence's next token and advance its length.
 * Takes a new block when the last one is full. If the block to be written is
 * shared (ref_count > 1) it is copied on write: a new block replaces it in
 * this table, the old one loses a reference, and (*cow_src, *cow_dst) name
 * the copy the caller must run (pa_copy_blocks) before writing the slot;
 * otherwise both are -1. On PA_ERR_OUT_OF_BLOCKS nothing changes. */
pa_status pa_alloc_append_slot(pa_alloc *a, int64_t seq_id, int64_t *slot, int64_t *cow_src,
                               int64_t *cow_dst);

/* Slots of existing positions [start, start + count) of a sequence. */
pa_status pa_alloc_seq_slots(const pa_alloc *a, int64_t seq_id, int start, int count,
                             int64_t *slots);

/* Drop the sequence: each block loses a reference; blocks reaching zero go
 * back on the free list. */
pa_status pa_alloc_free_seq(pa_alloc *a, int64_t seq_id);

/* Sliding-window release [P2, section 5.2: blocks that fall out of the window
 * are reclaimed automatically]. Every block wholly before the window
 * [len - window, len) of the sequence's current length loses this sequence's
 * reference (blocks reaching zero go back on the free list) and its table
 * entry becomes -1. Decode with the same or a smaller window never reads those
 * entries (pa_decode_window). *freed (may be NULL) = blocks returned to the
 * free list. window <= 0: PA_ERR_INVALID. Entries already released are skipped,
 * so the call may be repeated every step. Slots of released positions are no
 * longer available (pa_alloc_seq_slots answers PA_ERR_STATE). */
pa_status pa_alloc_slide_window(pa_alloc *a, int64_t seq_id, int window, int *freed);

/* Swapping a group of sequences (the blocks of a preempted request and of the
 * samples forked from it) [P3, section "分页还顺带解决了什么"; P2, section 3.1].
 * pa_alloc_set_host_blocks gives the manager a host swap space of
 * num_host_blocks blocks (once; PA_ERR_STATE if already given).
 * pa_alloc_swap_out moves the n sequences seq_ids (all resident) to the host:
 * each distinct block they use gets one free host block, whose count is the
 * group's references; the device block loses those references (returning to
 * the free list at zero) and the tables then name host blocks. pairs[0 ..
 * *num_pairs) receives (device block, host block) -- the copies pa_swap_out
 * must make. pa_alloc_swap_in is the mirror image for a swapped group:
 * pairs are (host block, device block) for pa_swap_in. A block also used by
 * a sequence outside the group stays in place for it, and the group gets its
 * own copy. All or nothing: PA_ERR_OUT_OF_BLOCKS if the other side lacks free
 * blocks, PA_ERR_STATE if a sequence is unknown or already on the other side,
 * PA_ERR_INVALID if one is listed twice or cap is short. While swapped a
 * sequence can only be swapped in, freed or queried (pa_alloc_block_table
 * then lists host blocks); other calls answer PA_ERR_STATE. */
pa_status pa_alloc_set_host_blocks(pa_alloc *a, int num_host_blocks);
pa_status pa_alloc_swap_out(pa_alloc *a, const int64_t *seq_ids, int n, int64_t *pairs, int cap,
                            int *num_pairs);
pa_status pa_alloc_swap_in(pa_alloc *a, const int64_t *seq_ids, int n, int64_t *pairs, int cap,
                           int *num_pairs);
pa_status pa_alloc_is_swapped(const pa_alloc *a, int64_t seq_id, int *swapped);
pa_status pa_alloc_host_free(const pa_alloc *a, int *free_host_blocks);

/* Copy the sequence's block table into out[0 .. cap); report its block and
 * token counts (either pointer may be NULL). PA_ERR_INVALID if cap is short. */
pa_status pa_alloc_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int cap,
                               int *num_blocks, int *num_tokens);

/* Fill a padded [n][max_blocks_per_seq] table and the lengths for a batch of
 * sequences; unused entries get `pad`. */
pa_status pa_alloc_fill_tables(const pa_alloc *a, const int64_t *seq_ids, int n,
                               int32_t *block_tables, int max_blocks_per_seq, int32_t pad,
                               int32_t *context_lens);

/* Prefix caching of full blocks [P3, section "分页还顺带解决了什么": requests
 * whose prompts begin alike point their first blocks at the same physical
 * blocks; only blocks that are completely filled are shared; P1, section 9:
 * a common prompt prefix's KV is cached].
 *
 * pa_alloc_add_seq_cached adds a sequence holding the prompt tokens[0 ..
 * num_tokens) (token ids; only compared for equality). Its leading full
 * blocks are looked up: logical block i is shared when a cached block holds
 * exactly tokens[0 .. (i+1) * block_size) (the same ids in the same order,
 * from position 0). The lookup covers the full blocks that lie within the
 * first num_tokens - 1 tokens, so at least the last prompt token is always
 * left to compute, and stops at the first block that is not cached. Shared
 * blocks gain a reference; the rest are taken from the free list. Then every
 * full block the prompt fills that is not yet cached under its prefix is
 * registered (a prefix is cached on one block at most). *num_cached_tokens =
 * shared blocks * block_size: the positions whose K/V are already in the
 * pool. The caller writes positions [*num_cached_tokens, num_tokens) (e.g.
 * pa_reshape_and_cache) before any kernel reads them; a request added later
 * in the same step may share these blocks, and stream order makes the write
 * land first. Tokens appended by pa_alloc_append_slot are not registered.
 * All or nothing: PA_ERR_OUT_OF_BLOCKS leaves the state unchanged.
 *
 * A cached block whose last reference is dropped (pa_alloc_free_seq,
 * pa_alloc_slide_window, pa_alloc_swap_out) keeps its contents and stays
 * cached, counted as free. Blocks are taken first from the free blocks that
 * hold no cached prefix; when there are none, the cached free block released
 * longest ago is reused, and only its own prefix is forgotten: a longer
 * prefix still cached on another block is found again once a request caches
 * the shorter one anew.
 *
 * pa_alloc_cached_blocks: blocks holding a cached prefix, and how many of
 * those are free (evictable). pa_alloc_reset_prefix_cache forgets every
 * cached prefix (the blocks themselves are untouched). */
pa_status pa_alloc_add_seq_cached(pa_alloc *a, int64_t seq_id, const int32_t *tokens,
                                  int num_tokens, int *num_cached_tokens);
pa_status pa_alloc_cached_blocks(const pa_alloc *a, int *cached_blocks, int *cached_free_blocks);
pa_status pa_alloc_reset_prefix_cache(pa_alloc *a);

pa_status pa_alloc_ref_count(const pa_alloc *a, int32_t block, int *ref_count);

/* Free blocks; token slots that hold a token; allocated slots that do not
 * (the unfilled tails of last blocks [P1, section 4; P3, section "浪费降到了多少"]). */
pa_status pa_alloc_stats(const pa_alloc *a, int *free_blocks, int64_t *used_tokens,
                         int64_t *wasted_tokens);

#ifdef __cplusplus
}
#endif
#endif /* PA370_H */
