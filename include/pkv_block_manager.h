/*
 * pkv_block_manager.h -- host-side KV-block bookkeeping (C ABI).
 *
 * The memory-management layer of PagedAttention as the pages describe it:
 *  - the KV cache is cut into fixed-size blocks handed out on demand from one
 *    pool; a per-sequence block table maps logical to physical blocks; blocks
 *    return to the pool when a request ends ("vLLM 深读：用 PagedAttention 撑起
 *    高并发 LLM 推理", section "先看浪费在哪里"; ipipp.com vLLM article,
 *    section "二、PagedAttention分页原理深度剖析");
 *  - sequences that share a prefix (parallel samples, beams) point at the same
 *    physical blocks, reference counted, and a write to a shared block first
 *    copies it (copy-on-write) (same sections);
 *  - automatic prefix caching: the prompt is cut into blocks; each full
 *    block's hash is chained from its parent block's hash and its own
 *    contents; cached blocks live in a hash table, are allocated and freed
 *    independently and evicted least-recently-used first; a lookup matches
 *    block by block exactly and reuses only full blocks ("vLLM" wiki entry,
 *    wiki.bytelighting.cn, section "Automatic Prefix Caching（自动前缀缓存）").
 *
 * It produces what the device path consumes: slots for reshape_and_cache,
 * block tables and context lengths for decode, and (src, dst) pairs for
 * copy_blocks.  It never touches device memory.  A manager is not
 * thread-safe: one host thread at a time.
 *
 * Block contents are identified by token ids (int32).  Sequence ids are
 * caller-chosen int64 values.  Slots are block * block_size + offset.
 * Errors: PKV_ERR_NULL, PKV_ERR_SHAPE (bad sizes), PKV_ERR_NOT_FOUND (unknown
 * or duplicate sequence id), PKV_ERR_NO_BLOCKS (pool exhausted; the call
 * leaves the manager unchanged).
 */
#ifndef PKV_BLOCK_MANAGER_H
#define PKV_BLOCK_MANAGER_H

#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;

/* A pool of num_blocks blocks of block_size tokens.  The free list is a
 * permutation of the pool drawn from `seed`, so placement is scattered.
 * prefix_caching != 0 enables automatic prefix caching.  NULL on bad sizes. */
pkv_block_manager *pkv_bm_create(int32_t num_blocks, int32_t block_size, uint64_t seed,
                                 int32_t prefix_caching);
void pkv_bm_destroy(pkv_block_manager *bm);

/* Start sequence `seq_id` with a prompt of n tokens.  With prefix caching,
 * leading full blocks whose hash chain and contents match cached blocks are
 * reused; *cached_tokens (may be NULL) receives how many prompt tokens were
 * found (a multiple of block_size).  Blocks are allocated for the rest; their
 * slots are available through pkv_bm_slots for writing the prompt's K/V. */
pkv_status pkv_bm_add_sequence(pkv_block_manager *bm, int64_t seq_id, const int32_t *tokens,
                               int32_t n, int32_t *cached_tokens);

/* Sequence `child` starts as a copy of `parent`, sharing all its blocks. */
pkv_status pkv_bm_fork(pkv_block_manager *bm, int64_t parent, int64_t child);

/* Append one token to each of n sequences (a decode step).  slots_out[i]
 * receives the slot for seq_ids[i]'s new token.  A sequence whose last block
 * is shared gets a private copy first; the copy is queued for
 * pkv_bm_take_copies.  All or nothing: on PKV_ERR_NO_BLOCKS nothing changed. */
pkv_status pkv_bm_append_tokens(pkv_block_manager *bm, const int64_t *seq_ids,
                                const int32_t *tokens, int32_t n, int64_t *slots_out);

/* Slots of positions [pos_begin, pos_end) of a sequence. */
pkv_status pkv_bm_slots(pkv_block_manager *bm, int64_t seq_id, int32_t pos_begin,
                        int32_t pos_end, int64_t *slots_out);

/* End a sequence: its blocks lose one reference each; blocks nobody holds go
 * back to the pool, or -- full cached blocks -- to the eviction list. */
pkv_status pkv_bm_free_sequence(pkv_block_manager *bm, int64_t seq_id);

/* Move the queued copy-on-write pairs (src, dst) into pairs_out (int64
 * [max_pairs][2]) and return their number; if more than max_pairs are queued,
 * nothing is moved and minus the number queued is returned. */
int32_t pkv_bm_take_copies(pkv_block_manager *bm, int64_t *pairs_out, int32_t max_pairs);

/* Block tables and context lengths of n sequences, for the decode call:
 * tables_out is int32 [n][max_blocks] padded with -1, lens_out int32 [n]. */
pkv_status pkv_bm_block_tables(pkv_block_manager *bm, const int64_t *seq_ids, int32_t n,
                               int32_t max_blocks, int32_t *tables_out, int32_t *lens_out);

/* An order of n sequences (order_out[i] = a position in seq_ids) in which
 * sequences that begin with the same physical blocks are consecutive: the
 * tables' full blocks sorted lexicographically, ties in the given order.
 * Laying out a step's rows (q, out, tables) in this order makes the runs of
 * pkv_bm_shared_prefix_groups as long as the sharing allows. */
pkv_status pkv_bm_prefix_order(pkv_block_manager *bm, const int64_t *seq_ids, int32_t n,
                               int32_t *order_out);

/* Groups for pkv_paged_attention_decode_shared over n sequences taken in the
 * order of seq_ids (the rows of the tables pkv_bm_block_tables exports in the
 * same order): maximal runs of consecutive sequences that hold the same
 * physical blocks at the start of their tables -- what fork gives parallel
 * samples of one prompt, or prefix caching gives requests with one system
 * prompt.  A run starting at sequence i takes the next sequences while they
 * keep at least min_shared_blocks (>= 1) leading blocks in common with
 * sequence i, counting only blocks that are full in both.  For run r:
 * group_start_out[r] .. group_start_out[r+1] - 1 are its positions in seq_ids
 * and shared_blocks_out[r] the leading blocks all its members share (0 for a
 * run of one).  group_start_out needs n + 1 entries, shared_blocks_out n;
 * *num_groups_out receives the number of runs. */
pkv_status pkv_bm_shared_prefix_groups(pkv_block_manager *bm, const int64_t *seq_ids, int32_t n,
                                       int32_t min_shared_blocks, int32_t *group_start_out,
                                       int32_t *shared_blocks_out, int32_t *num_groups_out);

/* Counts: free blocks (never used or returned), cached blocks held by nobody
 * (evictable), blocks referenced by at least one sequence, live sequences. */
pkv_status pkv_bm_stats(const pkv_block_manager *bm, int32_t *free_blocks,
                        int32_t *evictable_blocks, int32_t *used_blocks, int32_t *sequences);

/* Reference count of a physical block (for tests); -1 if out of range. */
int32_t pkv_bm_refcount(const pkv_block_manager *bm, int32_t block);

#ifdef __cplusplus
}
#endif

#endif /* PKV_BLOCK_MANAGER_H */
