/*
 * pa_block_manager.h -- C ABI of the host-side block allocator and block tables.
 *
 * Host code (C++), not the hot path: it decides where each token's K/V goes and
 * produces the int32 block tables, the int64 slot mappings and the (src, dst)
 * copy-on-write pairs that pa_cache_write / pa_copy_blocks / pa_decode consume.
 * All pointers here are HOST pointers.  A manager is not thread-safe.  No C++
 * exception crosses this boundary: a failed host allocation inside a call returns
 * PA_ERR_OOM, after which that manager's state is unspecified (destroy it).
 *
 * Sources (page title, section):
 *   devpress.csdn.net/amd vLLM v0.6.x teardown, 关键设计一 (BlockTable,
 *     BlockAllocator with free_blocks = list(range(N)), allocate = pop() from the
 *     end, out-of-memory when empty, free = append; BlockManager.append_slot),
 *     关键设计二 (fork shares the parent's blocks; copy-on-write when the block
 *     to be written is shared).
 *   chenxutan "vLLM 深度拆解" 2.1 (16-token blocks, logical -> physical table,
 *     prefix blocks shared by reference) and 3.3 (append_slot fills the current
 *     block, takes a new one when it is full; free returns all blocks).
 * Readings where the pages are silent or their sketch is wrong:
 *   - free list is a LIFO stack whose initial order the caller may give;
 *   - append allocates a block iff the sequence's token count is a multiple of
 *     block_size, and returns the token's slot (block * block_size + offset);
 *   - fork increments the reference count of every shared block;
 *   - copy-on-write happens only when the token goes into an existing, partly
 *     filled block whose count is > 1; the copy pair is (old, new) and the old
 *     block loses one reference;
 *   - free drops references in logical-block order, pushing each block that
 *     reaches zero onto the free stack;
 *   - an operation that would run out of blocks fails with PA_ERR_OOM and
 *     changes nothing.
 *
 * Automatic prefix caching (chenxutan "vLLM 深度拆解" 5.2: prompts that share a
 * prefix -- a system prompt, RAG context -- reuse its KV instead of computing it
 * again, without the caller naming the prefix).  The pages give no mechanism;
 * the reading taken:
 *   - only sequences created from their prompt's token ids (pa_bm_add_seq_tokens)
 *     take part; a full block of such a prompt is indexed by the key (parent
 *     physical block, the parent's generation, its block_size token ids), where
 *     the parent is the previous block of the same prompt (-1 for the first) and
 *     a block's generation counts how often it has been handed out -- so a key
 *     identifies the whole prefix up to and including the block, and a block that
 *     was reclaimed and reused never matches its old children's keys;
 *   - a new prompt reuses the longest run of leading full blocks found in the
 *     index (counts go up by one) and allocates the rest as appends would; its
 *     own full blocks are indexed;
 *   - an indexed block whose count drops to zero is not freed but becomes
 *     evictable (still indexed, reusable by a later prompt); free_seq puts a
 *     sequence's evictable blocks last-block first; allocation takes the free
 *     stack first, then reclaims the least recently evictable block (removing it
 *     from the index);
 *   - blocks filled by later appends are not indexed (their token ids are not
 *     known here).
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* Create a manager over num_blocks blocks of block_size tokens.  free_order
 * (nullable, num_blocks entries, a permutation of 0..num_blocks-1) is the
 * initial free stack, bottom first: the first allocation takes
 * free_order[num_blocks-1].  NULL means 0..num_blocks-1 (first allocation takes
 * num_blocks-1).  *out receives the handle; free it with pa_bm_destroy. */
PA_API pa_status pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t *free_order,
                       pa_block_manager **out);
PA_API void pa_bm_destroy(pa_block_manager *bm);

/* Register an empty sequence.  PA_ERR_INVALID_ARG if seq_id exists. */
PA_API pa_status pa_bm_add_seq(pa_block_manager *bm, int64_t seq_id);

/* Append n >= 0 tokens to a sequence.  slots_out (nullable, n entries) receives
 * each token's slot.  cow_pairs_out (nullable, room for 2 * cow_capacity int32)
 * receives the (src, dst) copy pairs in order; *num_cow_out (nullable) their
 * count.  PA_ERR_INVALID_ARG if more pairs arise than cow_capacity (nothing is
 * changed); PA_ERR_OOM if the pool lacks the blocks (nothing is changed). */
PA_API pa_status pa_bm_append_slots(pa_block_manager *bm, int64_t seq_id, int32_t n, int64_t *slots_out,
                             int32_t *cow_pairs_out, int32_t cow_capacity, int32_t *num_cow_out);

/* One step for n distinct sequences in one call: appends counts[i] >= 0 tokens
 * (counts NULL: one each) to seq_ids[i], in the order given -- the same result as
 * n pa_bm_append_slots calls in that order.  slots_out (nullable, sum of counts
 * entries) receives the slots sequence by sequence; cow_pairs_out (nullable, room
 * for 2 * cow_capacity int32) the copy pairs in order, *num_cow_out (nullable)
 * their count.  All or nothing: PA_ERR_OOM if the pool lacks the blocks for the
 * whole step, PA_ERR_NOT_FOUND for an unknown id, PA_ERR_INVALID_ARG for a
 * repeated id, a negative count or more pairs than cow_capacity -- and then
 * nothing is changed. */
PA_API pa_status pa_bm_append_step(pa_block_manager *bm, const int64_t *seq_ids, const int32_t *counts,
                                   int32_t n, int64_t *slots_out, int32_t *cow_pairs_out,
                                   int32_t cow_capacity, int32_t *num_cow_out);

/* Child shares all of parent's blocks (their counts go up by one). */
PA_API pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id);

/* Drop a sequence and one reference to each of its blocks. */
PA_API pa_status pa_bm_free_seq(pa_block_manager *bm, int64_t seq_id);

/* Number of tokens / blocks of a sequence (-1 if unknown). */
PA_API int64_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq_id);
PA_API int32_t pa_bm_num_seq_blocks(const pa_block_manager *bm, int64_t seq_id);

/* Longest block table among n sequences: the max_blocks pa_bm_build_tables needs
 * (0 for n == 0; -1 for an unknown id or bad arguments). */
PA_API int32_t pa_bm_max_seq_blocks(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n);

/* Copy a sequence's block table (its first `capacity` entries at most) into out;
 * *len_out (nullable) gets the table length. */
PA_API pa_status pa_bm_block_table(const pa_block_manager *bm, int64_t seq_id, int32_t *out,
                            int32_t capacity, int32_t *len_out);

/* Tables of n sequences as int32 [n][max_blocks], padded with -1, and their
 * int32 lengths (nullable).  PA_ERR_INVALID_ARG if a table is longer than
 * max_blocks; PA_ERR_NOT_FOUND on an unknown id. */
PA_API pa_status pa_bm_build_tables(const pa_block_manager *bm, const int64_t *seq_ids, int32_t n,
                             int32_t max_blocks, int32_t *tables_out, int32_t *lens_out);

/* Reference count of a block (-1 if out of range), free-stack length (evictable
 * blocks are counted by pa_bm_num_evictable), pool size. */
PA_API int32_t pa_bm_refcount(const pa_block_manager *bm, int32_t block);
PA_API int32_t pa_bm_num_free(const pa_block_manager *bm);
PA_API int32_t pa_bm_num_blocks(const pa_block_manager *bm);
PA_API int32_t pa_bm_block_size(const pa_block_manager *bm);   /* tokens per block (-1 for NULL) */

/* Copy the free stack, bottom first (the next allocation takes the last entry);
 * returns its length.  out may be NULL to query the length. */
PA_API int32_t pa_bm_free_stack(const pa_block_manager *bm, int32_t *out, int32_t capacity);

/* Tokens stored over all live sequences (for utilisation statistics). */
PA_API int64_t pa_bm_tokens_stored(const pa_block_manager *bm);

/* Register sequence seq_id holding the n prompt tokens whose ids are tokens[0..n).
 * The longest run of leading full blocks already in the prefix index is reused;
 * *num_cached_out (nullable) receives the number of tokens it covers (a multiple
 * of block_size) -- their K/V are already in the cache.  slots_out (nullable,
 * n - *num_cached_out entries) receives the slots of the remaining tokens, in
 * order, for pa_cache_write.  Full blocks of the prompt are entered in the index.
 * PA_ERR_INVALID_ARG if seq_id exists; PA_ERR_OOM (nothing changed) if too few
 * blocks are free or evictable. */
PA_API pa_status pa_bm_add_seq_tokens(pa_block_manager *bm, int64_t seq_id, const int32_t *tokens,
                                      int32_t n, int64_t *slots_out, int32_t *num_cached_out);

/* Indexed blocks with count zero (reclaimable), and all indexed blocks. */
PA_API int32_t pa_bm_num_evictable(const pa_block_manager *bm);
PA_API int32_t pa_bm_num_cached(const pa_block_manager *bm);

/* Copy the evictable list, next reclaimed first, into out (at most capacity
 * entries); returns its length (-1 if bm is NULL). */
PA_API int32_t pa_bm_evictable(const pa_block_manager *bm, int32_t *out, int32_t capacity);

/* Snapshot of a manager's whole state (free stack, counts, generations, sequences,
 * prefix-cache keys and the evictable order) as bytes, for checkpoints and test
 * reproducibility; a restored manager behaves exactly as the original from then on.
 * pa_bm_snapshot_size: the bytes needed (0 for NULL).  pa_bm_snapshot: writes them
 * into buf; *len_out (nullable) gets the size; PA_ERR_INVALID_ARG if capacity is
 * too small.  pa_bm_restore: a new manager from a snapshot of this format version;
 * PA_ERR_INVALID_ARG for a truncated, foreign or out-of-range buffer (structure and
 * bounds are checked, not that counts match the tables). */
PA_API size_t pa_bm_snapshot_size(const pa_block_manager *bm);
PA_API pa_status pa_bm_snapshot(const pa_block_manager *bm, void *buf, size_t capacity, size_t *len_out);
PA_API pa_status pa_bm_restore(const void *buf, size_t len, pa_block_manager **out);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H_ */
