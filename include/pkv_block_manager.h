/*
 * pkv_block_manager.h - host-side block manager of a paged KV cache (C ABI).
 *
 * Bookkeeping that produces the inputs of the device calls in pkv.h: which
 * physical block holds which tokens of which request.  Sources:
 *   lshu.cn/news/11644 (vLLM architecture analysis)
 *   - "整体架构": one global physical block pool; blocks are handed out on
 *     demand when a request arrives and taken back the moment it finishes.
 *   - "核心创新：PagedAttention 的设计逻辑" / "方案：页式内存管理": one Block
 *     Table per request; a request growing by one token writes into its last
 *     block while it has room, otherwise takes a block from the free pool and
 *     appends it to its table; a finished request returns all its blocks.
 *   - same section, "收益分析" (memory sharing): requests with a common prefix
 *     share its physical blocks read-only; a divergence is copy-on-write.
 *
 * Rules where the pages are silent (fixed here, and followed by the test
 * oracle the manager is checked against):
 *   - The free pool is first-in first-out, initially blocks 0 .. N-1 in
 *     order; a block whose last reference goes away joins its tail (blocks of
 *     one finished request in table order).
 *   - A block's reference count is the number of Block Tables holding it.
 *     Appending to a request whose last block is not full but shared first
 *     copies that block into a fresh one: the pair (old, new) is reported,
 *     the old block loses one reference, the table points at the copy.  The
 *     caller runs the copies (pkv_copy_blocks) before the token writes
 *     (pkv_reshape_and_cache) of the same step.
 *   - A decode step (pkv_bm_append) gives one new token to each listed
 *     request, in list order, and is all-or-nothing: when the pool cannot
 *     supply every block the step needs, it returns PKV_ERR_NO_BLOCKS and
 *     changes nothing.
 *
 * Ownership and threading: a manager is created and destroyed by the caller;
 * all pointers passed in are host memory owned by the caller; calls on one
 * manager are serialised by an internal lock.  Sequence ids are any int64.
 * On an error the manager is unchanged.  A call that runs out of host memory
 * returns PKV_ERR_TOO_LARGE (pkv_bm_blocks_needed: -1), also with the manager
 * unchanged; no C++ exception leaves these calls.  No call touches the GPU.
 */
#ifndef PKV_BLOCK_MANAGER_H_
#define PKV_BLOCK_MANAGER_H_

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;

/* A manager for a pool of num_blocks blocks of block_size tokens; Block
 * Tables hold at most max_blocks_per_seq entries.  PKV_ERR_BAD_SHAPE for a
 * non-positive argument, PKV_ERR_NULL_POINTER when out is NULL. */
PKV_API pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size, int32_t max_blocks_per_seq,
                                 pkv_block_manager **out);
PKV_API void pkv_bm_destroy(pkv_block_manager *bm); /* NULL is a no-op */

PKV_API int32_t pkv_bm_num_free_blocks(const pkv_block_manager *bm);
PKV_API int32_t pkv_bm_num_sequences(const pkv_block_manager *bm);
/* References to one block (0 when free); -1 for a block outside the pool. */
PKV_API int32_t pkv_bm_ref_count(const pkv_block_manager *bm, int32_t block);
/* Tokens of a request; -1 when the id is unknown. */
PKV_API int32_t pkv_bm_context_len(const pkv_block_manager *bm, int64_t seq_id);

/* A new request holding num_tokens >= 0 prompt tokens: ceil(num_tokens / B)
 * blocks from the pool; slot_mapping (may be NULL) receives the num_tokens
 * slots of the prompt tokens (for pkv_reshape_and_cache).  Errors:
 * PKV_ERR_BAD_SEQUENCE (id present), PKV_ERR_TOO_LARGE (table too short),
 * PKV_ERR_NO_BLOCKS. */
PKV_API pkv_status pkv_bm_add_sequence(pkv_block_manager *bm, int64_t seq_id, int32_t num_tokens,
                                       int64_t *slot_mapping);

/* child becomes a request with parent's tokens in parent's blocks (each block
 * gains a reference).  PKV_ERR_BAD_SEQUENCE when parent is unknown or child
 * present. */
PKV_API pkv_status pkv_bm_fork(pkv_block_manager *bm, int64_t parent_id, int64_t child_id);

/* A finished request: each of its blocks loses a reference; blocks left
 * without one return to the pool. */
PKV_API pkv_status pkv_bm_free_sequence(pkv_block_manager *bm, int64_t seq_id);

/* Blocks that pkv_bm_append(seq_ids, n) would take from the pool: one per
 * request whose last block is full (or that has none), one per copy; of k
 * listed holders of one shared block with r references, min(k, r - 1) copy
 * it.  -1 for an unknown or repeated id. */
PKV_API int32_t pkv_bm_blocks_needed(const pkv_block_manager *bm, const int64_t *seq_ids,
                                     int32_t n);

/* One decode step: one new token for each of the n listed requests.
 * slot_mapping[n] receives the new tokens' slots; copy_pairs[copy_capacity][2]
 * receives the (src, dst) block copies of the step, *num_copies their count
 * (copy_capacity >= n always suffices).  Errors: PKV_ERR_BAD_SEQUENCE,
 * PKV_ERR_TOO_LARGE (a table would outgrow max_blocks_per_seq),
 * PKV_ERR_BAD_SHAPE (copy_capacity < n), PKV_ERR_NO_BLOCKS. */
PKV_API pkv_status pkv_bm_append(pkv_block_manager *bm, const int64_t *seq_ids, int32_t n,
                                 int64_t *slot_mapping, int64_t *copy_pairs, int32_t copy_capacity,
                                 int32_t *num_copies);

/* Block Table rows of the listed requests, row r at block_tables + r *
 * row_stride (row_stride >= max_blocks_per_seq), each of its row_stride
 * entries written (unused ones with -1), and their
 * lengths in context_lens[n]: the int32 inputs of
 * pkv_paged_attention_decode. */
PKV_API pkv_status pkv_bm_block_tables(const pkv_block_manager *bm, const int64_t *seq_ids,
                                       int32_t n, int32_t *block_tables, int32_t row_stride,
                                       int32_t *context_lens);

/* The free pool in queue order (first out first): *count = its size, and the
 * first min(count, capacity) ids are written to out. */
PKV_API pkv_status pkv_bm_free_list(const pkv_block_manager *bm, int32_t *out, int32_t capacity,
                                    int32_t *count);

#ifdef __cplusplus
}
#endif

#endif /* PKV_BLOCK_MANAGER_H_ */
