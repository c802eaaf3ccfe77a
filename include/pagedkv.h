/*
 * pagedkv.h — C ABI of libpagedkv.so: paged KV cache append, paged decode
 * attention, block copy, and the host block manager / continuous-batching
 * step loop that produces their indices.
 *
 * Sources the operations are defined by (web pages on PagedAttention):
 *   [A] "大模型推理性能优化：PagedAttention与Continuous Batching原理与实践"
 *       §2.1 (KV cache), §2.2 (PagedAttention: blocks, page table, free list,
 *       shared pages, gather/scatter), §2.3 (continuous batching), §3.4
 *       (--block-size defaults to 16).
 *   [B] "vLLM 原理：PagedAttention 和 Continuous Batching"
 *       "PagedAttention 的思路" (16 tokens per page, ceil arithmetic),
 *       "工作原理" (1. page table, 2. on-demand allocation, 3. immediate release),
 *       "优势 / 3. 支持共享" (shared prefixes, parallel sampling),
 *       "vLLM 的调度 / 调度流程" (the step loop), "Preemption（抢占）".
 *   [C] "如何通过PagedAttention实现LLM高性能推理：实战指南"
 *       §2.2 (allocator: free-block deque, ceil(num_tokens / block_size)).
 *
 * Conventions shared by every call:
 *   - Return value: a pa_status. No call throws, aborts or traps. Arguments
 *     are validated on the host before anything is enqueued; on an error
 *     nothing is launched and no state changes.
 *   - Device calls take caller-owned device pointers and a cudaStream_t
 *     passed as void* (NULL = legacy default stream). They enqueue work and
 *     return without synchronising, and they allocate no device memory.
 *   - Device-side index checks: a block id or slot outside the pool, or a
 *     sequence length outside its bounds, is skipped (never dereferenced) and
 *     recorded in a per-device error word; read it with pa_get_device_error.
 *   - Host objects (pa_bm, pa_sched) are opaque, library-owned, and not
 *     thread-safe: one thread at a time per object.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Tokens per KV block. Fixed: [A] §3.4 gives 16 as the default page size and
 * [B] "PagedAttention 的思路" stores 16 tokens per page. */
#define PA_BLOCK_SIZE 16

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, shape mismatch   */
  PA_ERR_UNSUPPORTED = 2,   /* valid but not built: head_dim, dtype, group   */
  PA_ERR_CUDA = 3,          /* a CUDA runtime call failed (pa_last_error)    */
  PA_ERR_NO_BLOCKS = 4,     /* free list too short; state left unchanged     */
  PA_ERR_UNKNOWN_SEQ = 5,   /* block-manager sequence id not present         */
  PA_ERR_DEVICE_BOUNDS = 6, /* device error word was non-zero                */
  PA_ERR_SEQ_EXISTS = 7,    /* block-manager sequence id already present     */
  PA_ERR_CAPACITY = 8,      /* caller buffer or table width too small        */
  PA_ERR_WORKSPACE = 9      /* decode workspace missing or too small         */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

/* Device error word bits (pa_get_device_error). */
#define PA_DEVERR_SLOT    1u  /* append: slot >= num_blocks * 16             */
#define PA_DEVERR_BLOCK   2u  /* decode/copy: block id outside [0, num_blocks) */
#define PA_DEVERR_SEQLEN  4u  /* decode: seq_len < 0, > max_seq_len, or beyond
                                 max_blocks_per_seq * 16                     */
#define PA_DEVERR_TIMEOUT 8u  /* decode/prefill: a wait for staged data gave
                                 up after 2 s (the kernel returned instead of
                                 hanging)                                    */

/*
 * The KV pool of one attention layer: one contiguous device buffer
 *     kv_pool[num_blocks][2][num_kv_heads][16][head_dim]
 * of `dtype` elements, row-major. Index 0 of the second axis is K, 1 is V.
 * A (block, K|V, kv head) tile is 16 * head_dim contiguous elements, so every
 * gathered unit is one contiguous, 16-byte aligned run ([A] §2.2: a page holds
 * the KV of 16 tokens and may sit anywhere in the pooled buffer). The pages fix
 * only the per-layer [batch, heads, seq, head_dim] view ([A] §2.1); this block
 * layout is this library's choice.
 * Token position p of a sequence with block table T lives in slot
 *     slot = T[p / 16] * 16 + p % 16.
 * Supported: block_size 16; head_dim 64 or 128; dtype PA_F32 or PA_BF16;
 * kv_pool 16-byte aligned.
 */
typedef struct {
  int32_t num_blocks;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;   /* must be PA_BLOCK_SIZE */
  int32_t dtype;        /* pa_dtype */
} pa_pool_desc;

/* ------------------------------------------------------------------------ */
/* Device operations                                                          */
/* ------------------------------------------------------------------------ */

/*
 * Cache append (the "scatter" of [A] §2.2): for every t in [0, num_tokens)
 * with s = slot_mapping[t] >= 0,
 *     kv_pool[s/16][0][h][s%16][:] = k[t][h][:]
 *     kv_pool[s/16][1][h][s%16][:] = v[t][h][:]      for all kv heads h.
 * k, v: device, [num_tokens][num_kv_heads][head_dim] contiguous, pool dtype,
 *       16-byte aligned.
 * slot_mapping: device int64 [num_tokens]. A negative slot is padding and is
 *       skipped. A slot >= num_blocks*16 is skipped and sets PA_DEVERR_SLOT.
 * Two tokens mapped to the same slot race; the caller must not do that.
 * num_tokens == 0 is a no-op returning PA_OK.
 */
pa_status pa_reshape_and_cache(const void* k, const void* v, void* kv_pool,
                               const int64_t* slot_mapping, int32_t num_tokens,
                               pa_pool_desc pool, void* stream);

/*
 * Bytes of device workspace pa_decode needs for this shape (split-KV partial
 * results). 0 means pa_decode needs none and accepts workspace == NULL.
 * Depends on the arguments and on the current device's SM count (read once per
 * device; 148, a B200's, when no device can be queried), so size the
 * workspace with the device current that pa_decode will run on. Returns 0 for
 * invalid arguments too, which pa_decode then rejects.
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads,
                                pa_pool_desc pool, int32_t max_seq_len);

/*
 * Tokens per split-KV partition that pa_decode uses for this shape on the
 * current device (a multiple of 16): 2048, halved down to 128 while the
 * (sequence, KV head, partition) grid would give the device's SMs fewer than
 * four CTAs each. Sequences no longer than this are finished in one pass.
 */
int32_t pa_decode_partition_tokens(int32_t num_seqs, int32_t num_heads,
                                   pa_pool_desc pool, int32_t max_seq_len);

/*
 * Decode-step attention over the paged cache ([A] §2.2: the page table is used
 * to gather the scattered blocks into the sequence's logical KV at attention
 * time; [A] §2 says decode is the bottleneck phase). For every sequence b and
 * query head h, with G = num_heads / num_kv_heads, g = h / G, L = seq_lens[b]
 * and K_t, V_t the key / value of token position t gathered through
 * block_tables[b]:
 *     s_t      = scale * <q[b][h], K_t[g]>                 t in [0, L)
 *     out[b][h] = sum_t softmax(s)_t * V_t[g]
 * computed with fp32 accumulation, as per-partition online softmax (m, l, acc)
 * merged by a log-sum-exp reduce; the final value is rounded once to the pool
 * dtype (round to nearest even for bf16).
 * q, out: device [num_seqs][num_heads][head_dim], pool dtype, 16-byte aligned.
 * block_tables: device int32 [num_seqs][max_blocks_per_seq]; entries past
 *       ceil(L/16) are not read.
 * seq_lens: device int32 [num_seqs], lengths after this step's append.
 *       L == 0 writes zeros. A length that is negative, > max_seq_len or
 *       > max_blocks_per_seq*16 writes zeros and sets PA_DEVERR_SEQLEN.
 * A table entry outside [0, num_blocks) is not read; its tokens count as
 *       zero vectors and PA_DEVERR_BLOCK is set.
 * max_seq_len: host-known upper bound on seq_lens (sets the partition count;
 *       a bound needing more than 65535 partitions is PA_ERR_UNSUPPORTED).
 * workspace: device, >= pa_decode_workspace_size(...) bytes, 256-byte aligned;
 *       contents on entry are ignored; must not be used by another call that
 *       overlaps this one on the GPU.
 * Requires num_heads % num_kv_heads == 0 and num_heads / num_kv_heads <= 16.
 * Must be ordered after the pa_reshape_and_cache that wrote this step's token
 * (same stream, or an event).
 */
pa_status pa_decode(void* out, const void* q, const void* kv_pool,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* seq_lens, int32_t num_seqs, int32_t num_heads,
                    float scale, pa_pool_desc pool, void* workspace,
                    size_t workspace_bytes, int32_t max_seq_len, void* stream);

/*
 * One decode step in one call: the new token of every sequence is appended
 * and attention runs over the updated cache. Same results, pool contents and
 * errors as
 *     pa_reshape_and_cache(k_new, v_new, kv_pool, slot_mapping, num_seqs, ...)
 *     pa_decode(out, q, kv_pool, block_tables, ..., seq_lens, ...)
 * when token b is sequence b's newest token, i.e. slot_mapping[b] is the slot
 * of position seq_lens[b]-1 through block_tables[b] (or negative: not
 * appended). For bf16 pools with head_dim 128 the append is folded into the
 * decode kernel (no separate launch): the CTA that stages the block holding
 * position seq_lens[b]-1 writes the new K/V row into that staged block and
 * stores it to the pool. A token whose slot is not that position's slot is not
 * written and raises PA_DEVERR_SLOT; a sequence of length 0 appends nothing.
 * Other dtypes and head sizes run the two calls in sequence.
 * k_new, v_new: device [num_seqs][num_kv_heads][head_dim], pool dtype, 16-byte
 * aligned; slot_mapping: device int64 [num_seqs]. The remaining arguments are
 * pa_decode's. The append/decode pairing of one step is the same as in the
 * pages' step loop ([B] "vLLM 的调度 / 调度流程": run the step, append the token).
 */
pa_status pa_append_decode(void* out, const void* q, const void* k_new, const void* v_new,
                           void* kv_pool, const int64_t* slot_mapping,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* seq_lens, int32_t num_seqs, int32_t num_heads,
                           float scale, pa_pool_desc pool, void* workspace,
                           size_t workspace_bytes, int32_t max_seq_len, void* stream);

/*
 * Decode without a workspace argument, for callers that cannot allocate
 * device memory. The pages have no counterpart: this is an integration
 * variant of pa_decode, not part of the method.
 * Some callers hand this library only their inputs and outputs and may not
 * allocate on the device themselves: a plugin inside a host engine whose
 * device memory is all owned by that engine's own pool, or a decode loop that
 * must not call cudaMalloc / cudaFree between steps because those calls can
 * synchronise the whole device and stall the other streams. For them the
 * split-KV partial results live in one fixed device array inside the library,
 * PA_DECODE_NOALLOC_SCRATCH_BYTES in size, created on every GPU that loads the
 * library and held until the process exits.
 * Same arguments, results and errors as pa_decode, minus the workspace. This
 * call allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *  - The first call on a device looks up the array's device address (once per
 *    device, with that device current) and keeps it for the life of the
 *    process; make that first call before any stream capture. cudaDeviceReset
 *    on that device ends the context the address belongs to: calling this
 *    entry point after a reset is not supported.
 *  - Arguments are checked exactly as pa_decode checks them, and those errors
 *    come first; then a shape whose partial results need more than
 *    PA_DECODE_NOALLOC_SCRATCH_BYTES (pa_decode_workspace_size) is rejected
 *    with PA_ERR_WORKSPACE before anything is enqueued; use pa_decode then.
 *  - Every call uses the same array and it keeps the last call's contents.
 *    Nothing in it must start at zero (each partial result is written before
 *    it is read), but two calls that overlap on the GPU (different streams,
 *    no ordering between them) race on it and may return wrong results.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)  /* 32 MiB per device */
pa_status pa_decode_noalloc(void* out, const void* q, const void* kv_pool,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* seq_lens, int32_t num_seqs, int32_t num_heads,
                            float scale, pa_pool_desc pool, int32_t max_seq_len,
                            void* stream);

/*
 * Paged prefill / chunked-prefill attention: causal attention of each
 * sequence's new tokens over its paged KV ([A] §2: prefill processes the whole
 * prompt at once; [A] §2.2 / [B] "工作原理": KV is read through the page table).
 * Sequence b holds seq_lens[b] tokens of KV, its n_b = query_start[b+1] -
 * query_start[b] new tokens included as the last n_b positions (their K/V
 * already appended, e.g. by pa_reshape_and_cache with the prompt's slots).
 * Query row query_start[b] + i sits at position p = seq_lens[b] - n_b + i and
 * attends to positions 0..p:
 *     out[r, h, :] = sum_{t<=p} softmax_t(scale * q[r, h, :] . K_t[h / G]) V_t[h / G]
 * A whole prompt is n_b = seq_lens[b]; a later chunk has n_b < seq_lens[b].
 *   out, q: device [num_tokens][num_heads][head_dim] bf16, 16-byte aligned,
 *       row-major; out is written only at the new tokens' rows.
 *   block_tables: device int32 [num_seqs][max_blocks_per_seq];
 *   seq_lens: device int32 [num_seqs]; query_start: device int32 [num_seqs+1]
 *       (normally query_start[0] = 0, non-decreasing, query_start[num_seqs] =
 *       num_tokens).
 *   max_query_len: host bound on n_b (sizes the grid), <= num_tokens; 0
 *       launches nothing.
 * Supported: bf16 pools with head_dim 128, num_heads / num_kv_heads in
 * {1, 2, 4, 8, 16} (else PA_ERR_UNSUPPORTED). Device-side checks: n_b < 0,
 * n_b > max_query_len, query_start[b] < 0, query_start[b+1] > num_tokens,
 * n_b > seq_lens[b] or seq_lens[b] > 16 * max_blocks_per_seq sets
 * PA_DEVERR_SEQLEN and skips sequence b; a block id outside the pool sets
 * PA_DEVERR_BLOCK (that block's contribution is undefined, nothing is read
 * from it). A wait on staged data that exceeds 2 s sets PA_DEVERR_TIMEOUT; while
 * that bit is set (until pa_get_device_error reads it), prefill work units
 * taken later are skipped. Allocates nothing.
 * Kernel: tcgen05 MMAs with tensor-memory accumulators, two 128-row query
 * tiles per work unit, about one persistent CTA per SM taking units in launch
 * order (longest sequences first, up to 128 sequences) by cancelling CTAs of
 * the same launch that have not started. Launches on different streams may
 * run at the same time: each takes only its own units. The call may be
 * captured in a CUDA graph; make one call on the device before the first
 * capture (it sets the kernel's shared-memory limit once per device). There is
 * no run-time kernel choice: the mma.sync kernel exists only in a separate
 * comparison build of this library (compiled with PA_PREFILL_MMA_SYNC; same
 * results within rounding).
 */
pa_status pa_prefill(void* out, const void* q, const void* kv_pool,
                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* seq_lens, const int32_t* query_start,
                     int32_t num_seqs, int32_t num_tokens, int32_t num_heads, float scale,
                     pa_pool_desc pool, int32_t max_query_len, void* stream);

/*
 * Block copy for copy-on-write: for i in [0, n) in order,
 *     kv_pool[dst[i]] = kv_pool[src[i]]    (the whole block: K and V, all heads).
 * src, dst: device int32 [n]. Pairs must not overlap (no block is both a source
 * and a destination, no destination twice). An id outside [0, num_blocks)
 * skips that pair and sets PA_DEVERR_BLOCK. One call covers one layer's pool.
 * Copy-on-write of a shared partial last block is the block manager's rule
 * (pa_bm_append_slot); the pages name shared pages ([A] §2.2,
 * [B] "优势 / 3. 支持共享") but not the copy itself.
 */
pa_status pa_copy_blocks(void* kv_pool, const int32_t* src, const int32_t* dst,
                         int32_t n, pa_pool_desc pool, void* stream);

/*
 * Block copy between two pools of the same block shape (pool's kv heads,
 * head_dim, dtype): for i in [0, n), block src[i] of src_pool is copied to
 * block dst[i] of dst_pool. Either pool may be device memory or pinned host
 * memory mapped into the device's address space (e.g. from cudaHostAlloc),
 * which is how swap-mode preemption moves a preempted sequence's blocks to
 * host memory and back ([A] §3.4 "--swap-space"; [B] "Preemption（抢占）":
 * swap the KV cache out to the CPU). src, dst: int32 [n] the GPU can read.
 * Pointers the GPU cannot address are rejected (PA_ERR_INVALID_ARG) before
 * any launch; an id outside its pool skips the pair and sets PA_DEVERR_BLOCK.
 */
pa_status pa_copy_blocks_between(void* dst_pool, int32_t dst_num_blocks, const void* src_pool,
                                 int32_t src_num_blocks, const int32_t* src, const int32_t* dst,
                                 int32_t n, pa_pool_desc pool, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word (PA_DEVERR_* bits) into *flags. Returns PA_ERR_DEVICE_BOUNDS when the
 * word was non-zero, PA_OK when zero.
 */
pa_status pa_get_device_error(uint32_t* flags, void* stream);

/*
 * Self-test of the timeout path every kernel's waits share: one thread waits
 * on an mbarrier that nothing arrives at, with the same bounded wait as the
 * kernels but a limit of limit_ns nanoseconds (1 .. 10^9), then sets
 * PA_DEVERR_TIMEOUT and returns, leaving the context usable. Enqueued on
 * `stream`; read the bit with pa_get_device_error. A limit outside the range
 * returns PA_ERR_INVALID_ARG.
 */
pa_status pa_selftest_timeout(uint64_t limit_ns, void* stream);

/* Static text for a status code. */
const char* pa_status_string(pa_status s);

/* Detail of the last error raised on the calling thread ("" if none). */
const char* pa_last_error(void);

/* ------------------------------------------------------------------------ */
/* Host block manager ([A] §2.2, [B] "工作原理", [C] §2.2)                     */
/* ------------------------------------------------------------------------ */

typedef struct pa_bm pa_bm;

/*
 * A pool of num_blocks blocks. The free list is a FIFO: allocation takes from
 * its head ([C] §2.2 pops the left end of a deque), freed blocks go to its tail
 * in block-table order. initial_free_order: NULL gives 0..num_blocks-1 ([C]
 * §2.2 starts from range(num_blocks)); otherwise a permutation of
 * 0..num_blocks-1 (host int32 [num_blocks]) that becomes the initial free list
 * (used to place blocks at random pool positions). block_size must be 16.
 */
pa_status pa_bm_create(int32_t num_blocks, int32_t block_size,
                       const int32_t* initial_free_order, pa_bm** out);
void pa_bm_destroy(pa_bm* bm);

/*
 * Admits sequence `seq` with num_tokens tokens of KV: takes
 * ceil(num_tokens / 16) blocks ([C] §2.2; [B] "PagedAttention 的思路": 500
 * tokens -> 32 blocks, 1000 -> 63) from the free-list head, each with
 * refcount 1. All or nothing: PA_ERR_NO_BLOCKS leaves the state unchanged.
 * PA_ERR_SEQ_EXISTS if seq is present. num_tokens == 0 admits an empty table.
 */
pa_status pa_bm_allocate(pa_bm* bm, int64_t seq, int32_t num_tokens);

/*
 * Appends one token to `seq` ([B] "工作原理 / 2. 按需分配"): p = current length.
 *  - p % 16 == 0: takes a fresh block from the free-list head (the 513th token,
 *    p = 512, opens the 33rd block); no copy.
 *  - otherwise, last block L with refcount 1: writes in place.
 *  - otherwise (L shared): copy-on-write — takes a fresh block D, decrements
 *    L's refcount, replaces L by D in this table, and returns cow_src = L,
 *    cow_dst = D; the caller must copy L to D (pa_copy_blocks, every layer)
 *    before the token's K/V is written.
 * *slot = table[p/16]*16 + p%16; *cow_src = *cow_dst = -1 when no copy.
 * PA_ERR_NO_BLOCKS (state unchanged) when a block is needed and none is free.
 */
pa_status pa_bm_append_slot(pa_bm* bm, int64_t seq, int64_t* slot,
                            int32_t* cow_src, int32_t* cow_dst);

/* child gets a copy of parent's table and length; each block's refcount +1
 * ([A] §2.2 and [B] "支持共享": several logical blocks map to one physical
 * block). PA_ERR_UNKNOWN_SEQ / PA_ERR_SEQ_EXISTS. */
pa_status pa_bm_fork(pa_bm* bm, int64_t parent, int64_t child);

/* Releases `seq` ([B] "工作原理 / 3. 及时释放"): each block's refcount -1, in
 * table order; blocks reaching 0 go to the free-list tail. */
pa_status pa_bm_free(pa_bm* bm, int64_t seq);

int32_t pa_bm_num_free(const pa_bm* bm);
int32_t pa_bm_num_blocks(const pa_bm* bm);
pa_status pa_bm_seq_len(const pa_bm* bm, int64_t seq, int32_t* len);
pa_status pa_bm_refcount(const pa_bm* bm, int32_t block, int32_t* refcount);
/* Copies seq's block table into out[0..cap); *n = its length. PA_ERR_CAPACITY
 * (with *n set) when cap is too small. */
pa_status pa_bm_block_table(const pa_bm* bm, int64_t seq, int32_t* out,
                            int32_t cap, int32_t* n);
/* Copies the free list, head first. */
pa_status pa_bm_free_list(const pa_bm* bm, int32_t* out, int32_t cap, int32_t* n);
/* Slots of token positions [start, start+count) of seq into out[count]. */
pa_status pa_bm_slots(const pa_bm* bm, int64_t seq, int32_t start, int32_t count,
                      int64_t* out);
/*
 * Packs a decode batch for pa_decode into host buffers: row i of
 * block_tables[n][max_blocks] is seqs[i]'s table padded with -1, seq_lens[i]
 * its length, last_slots[i] the slot of its last token (-1 if empty; may be
 * NULL). PA_ERR_CAPACITY if a table is wider than max_blocks.
 */
pa_status pa_bm_pack(const pa_bm* bm, const int64_t* seqs, int32_t n,
                     int32_t max_blocks, int32_t* block_tables,
                     int32_t* seq_lens, int64_t* last_slots);

/*
 * Automatic prefix caching ([A] §3.4 "--enable-prefix-caching": requests with
 * a common prompt prefix, e.g. the same system prompt, skip recomputing it;
 * [B] "优势 / 3. 支持共享"). Off by default; switch it on for a fresh block
 * manager. A full block of a prompt is identified by the chained hash
 *     h_i = H(h_{i-1}, tokens[16i .. 16i+15]),   h_{-1} = 0,
 * H(p, t) = x after x = mix(p ^ 0x9E3779B97F4A7C15) and x = mix(x ^ t_j) for
 * each of the 16 token ids t_j (as uint32), mix being SplitMix64's output
 * function. Cached blocks whose refcount drops to 0 stay reusable on an
 * evictable list (least recently released first); a fresh block comes from
 * the free list, else by evicting that list's head. A block's cache entry
 * becomes reusable by others only once pa_bm_mark_written says its KV was
 * written; a request freed before that leaves nothing cached.
 */
pa_status pa_bm_set_prefix_caching(pa_bm* bm, int32_t enable);
/*
 * pa_bm_allocate for a request whose first num_prompt_tokens tokens are
 * prompt_tokens (num_tokens >= num_prompt_tokens tokens of KV in total): the
 * longest run of leading full prompt blocks found in the cache is shared
 * (refcount +1), the rest are fresh blocks; new full prompt blocks enter the
 * cache. *cached_tokens = 16 x the leading shared blocks whose KV is already
 * written (the caller writes KV from that position on). All or nothing
 * (PA_ERR_NO_BLOCKS when the fresh blocks do not fit). Without prefix caching
 * it is pa_bm_allocate with *cached_tokens = 0.
 */
pa_status pa_bm_allocate_prefix(pa_bm* bm, int64_t seq, const int32_t* prompt_tokens,
                                int32_t num_prompt_tokens, int32_t num_tokens,
                                int32_t* cached_tokens);
/* The KV of seq's cached blocks has been written (enqueued): they may be reused. */
pa_status pa_bm_mark_written(pa_bm* bm, int64_t seq);
/* Cached blocks with refcount 0, next to evict first. pa_bm_num_free counts
 * them as free. */
pa_status pa_bm_evictable_list(const pa_bm* bm, int32_t* out, int32_t cap, int32_t* n);
/* Number of blocks currently findable in the prefix cache. */
int32_t pa_bm_num_cached(const pa_bm* bm);

/* ------------------------------------------------------------------------ */
/* Continuous-batching step loop ([A] §2.3, [B] "vLLM 的调度", "Preemption")  */
/* ------------------------------------------------------------------------ */

typedef struct pa_sched pa_sched;

/*
 * Output of one step. Every array is library-owned host memory, valid until
 * the next pa_sched_step or pa_sched_destroy on the same scheduler.
 */
typedef struct {
  int32_t step;                 /* index of this step, from 0                  */
  int32_t done;                 /* 1: every request has finished by its end    */
  int32_t num_running;
  int32_t max_blocks_per_seq;   /* row width of block_tables                   */
  const int64_t* running;       /* [num_running] request ids, admission order  */
  const int32_t* seq_lens;      /* [num_running] KV length after the append    */
  const int32_t* block_tables;  /* [num_running][max_blocks_per_seq], -1 pad   */
  const int64_t* decode_slots;  /* [num_running] slot of the appended token    */
  int32_t num_prompt_seqs;      /* admitted this step and still running        */
  int32_t num_prompt_tokens;
  const int64_t* prompt_seqs;   /* [num_prompt_seqs] request ids               */
  const int32_t* prompt_lens;   /* [num_prompt_seqs] tokens of KV (re)written  */
  const int64_t* prompt_slots;  /* [num_prompt_tokens] positions start..len-1
                                   of each prompt seq, in prompt_seqs order     */
  int32_t num_cow;
  const int32_t* cow_src;       /* [num_cow] copy-on-write pairs, in order     */
  const int32_t* cow_dst;
  int32_t num_admitted;
  const int64_t* admitted;      /* admitted this step (incl. later preempted)  */
  int32_t num_preempted;
  const int64_t* preempted;     /* preempted this step, in preemption order    */
  int32_t num_finished;
  const int64_t* finished;      /* retired at the start of this step           */
  int32_t num_waiting;          /* queue length after the step                 */
  int32_t num_free_blocks;      /* free blocks after the step                  */
  const int32_t* prompt_starts; /* [num_prompt_seqs] first position written:
                                   positions before it are in reused cached
                                   blocks (0 without prefix caching); the
                                   request's prompt_slots cover [start, len)  */
  int32_t num_cached_tokens;    /* sum of prompt_starts this step              */
  /* swap-mode preemption (pa_sched_set_swap); device work order of a step:
     swap-out copies, swap-in copies, copy-on-write copies, prompt appends,
     decode */
  int32_t num_swap_out;
  const int32_t* swap_out_src;  /* [num_swap_out] device blocks to copy ...    */
  const int32_t* swap_out_dst;  /* ... into these host blocks                  */
  int32_t num_swap_in;
  const int32_t* swap_in_src;   /* [num_swap_in] host blocks to copy ...       */
  const int32_t* swap_in_dst;   /* ... into these device blocks                */
  int32_t num_swapped_out;
  const int64_t* swapped_out;   /* preempted this step by swapping out         */
  int32_t num_swapped_in;
  const int64_t* swapped_in;    /* admitted this step by swapping in (not in
                                   prompt_seqs: nothing is recomputed)        */
} pa_step_out;

/*
 * A scheduler over n_requests requests with ids 0..n-1 (used as block-manager
 * sequence ids), driving `bm` (not owned; must outlive the scheduler and not
 * be modified by others meanwhile). Each request i arrives at step
 * arrival_step[i] >= 0 with prompt_len[i] >= 1 tokens and finishes after
 * generating output_len[i] >= 1 tokens. Arrays are copied.
 * Step rules ([B] "调度流程" order, with these readings):
 *  1. retire running requests whose generated count reached output_len,
 *     freeing their blocks;
 *  2. enqueue arrivals (arrival_step <= step) at the waiting tail, by
 *     (arrival_step, id);
 *  3. admit from the waiting head (first come, first served) while the free
 *     list holds ceil((prompt + generated) / 16) blocks for it; stop at the
 *     first that does not fit; admitted requests (re)write positions
 *     0..prompt+generated-1 (recompute);
 *  4. grow: every running request, in admission order, appends one slot; when
 *     no block is free, the most recently admitted running request is
 *     preempted ([B] "Preemption": recompute mode): its blocks are freed and it
 *     goes to the waiting head keeping its generated count; if that request is
 *     the one growing, it is preempted and the grow phase ends;
 *  5. (caller) copy-on-write copies, prompt K/V, decode-token K/V, attention;
 *  6. generated += 1 for every running request.
 * max_blocks_per_seq: width of the packed block tables (must cover
 * ceil((prompt_len + output_len) / 16) for every request).
 */
pa_status pa_sched_create(pa_bm* bm, const int32_t* arrival_step,
                          const int32_t* prompt_len, const int32_t* output_len,
                          int32_t n_requests, int32_t max_blocks_per_seq,
                          pa_sched** out);
/* Runs one step and fills *out. When every request has finished, returns PA_OK
 * with out->done = 1 and nothing running. PA_ERR_NO_BLOCKS if the waiting head
 * cannot fit even with nothing running (the pool is too small for it). */
pa_status pa_sched_step(pa_sched* s, pa_step_out* out);
/*
 * Gives the scheduler the prompt token ids (request i's prompt is
 * tokens[offsets[i] .. offsets[i] + prompt_len[i])), switching admission to
 * pa_bm_allocate_prefix: a (re)admitted request reuses the cached blocks of
 * its prompt's longest cached prefix and only the KV after it is written
 * (prompt_starts). Requires the block manager's prefix caching; call before
 * the first step. Arrays are copied.
 */
pa_status pa_sched_set_prompt_tokens(pa_sched* s, const int32_t* tokens, const int64_t* offsets);
/*
 * Swap-mode preemption ([B] "Preemption（抢占）": the second mode swaps the KV
 * cache to the CPU; [A] §3.4 "--swap-space"). With num_host_blocks > 0 host
 * blocks, a preemption victim whose KV was written before the step and whose
 * blocks are not shared is swapped out: its blocks go to host blocks taken from
 * a FIFO host free list (swap_out pairs) and, when it is admitted again, into
 * fresh device blocks (swap_in pairs; its host blocks return to the host free
 * list at the end of that step) instead of being recomputed. A victim that does
 * not qualify, or finds too few host blocks, is recomputed as before.
 * 0 turns swapping off. Call before the first step.
 */
pa_status pa_sched_set_swap(pa_sched* s, int32_t num_host_blocks);
void pa_sched_destroy(pa_sched* s);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* PAGEDKV_H */
