/*
 * pa_block_manager.h -- host-side paged KV block manager of libpa_b200.so.
 *
 * It decides where every token's K/V lives in the block pool that the
 * kernels of pa.h read and write, following the block manager the pages
 * describe (cited by title and section):
 *   [A] "vLLM推理引擎深度解析：…" §三 PagedAttention：虚拟内存思想应用于KV Cache
 *       -- PagedAttentionManager: a pool of fixed-size blocks, a free list, one
 *       block table per request, allocate_request, append_token (the token
 *       goes into the last block if it has room, else into a new block),
 *       free_request (reference count down, block back to the free list at
 *       zero), share_prefix (another request's prefix blocks are shared,
 *       reference count up), get_stats.
 *   [B] "vLLM 原理与源码阅读", Block 管理器 -- one block table per request, block
 *       size 16 by default, copy-on-write: a request that writes into a shared
 *       block gets its own copy first.
 *   [C] "vLLM推理引擎深度实战：…" §1.2 -- running out of blocks is an error.
 *   [B] "vLLM 原理与源码阅读", Prefix Caching -- see pa_bm_create_prefix_caching.
 *
 * Readings: the free list is first-in first-out (blocks are taken from its
 * front and returned to its back, as the pages' pop(0) / append do); a write
 * into a block with reference count > 1 always copies it first (the pages'
 * share_prefix + append_token sketch omits this); an operation that cannot
 * get a block returns PA_BM_NO_SPACE and changes nothing.
 *
 * A slot is physical_block * block_size + offset, the same numbering as
 * pa_reshape_and_cache's slot_mapping.  The manager only decides: the caller
 * issues the block copies it returns (pa_copy_blocks) before the token writes
 * (pa_reshape_and_cache or pa_decode_append) and uploads the block tables.
 *
 * All memory here is host memory; no call touches the GPU.  A manager is not
 * thread-safe: calls on one manager must not overlap.
 */
#ifndef PA_B200_BLOCK_MANAGER_H
#define PA_B200_BLOCK_MANAGER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager_t;

typedef enum {
  PA_BM_OK = 0,
  PA_BM_NO_SPACE = 1,     /* not enough free blocks; nothing changed */
  PA_BM_BAD_ARG = 2,      /* negative size, NULL pointer, prefix longer than the source */
  PA_BM_UNKNOWN_SEQ = 3,  /* no such sequence */
  PA_BM_EXISTS = 4,       /* the sequence id is already in use */
  PA_BM_TABLE_FULL = 5,   /* a table does not fit max_blocks_per_seq (pa_bm_block_tables) */
} pa_bm_status_t;

typedef struct {
  int64_t total_blocks;
  int64_t free_blocks;
  int64_t used_blocks;     /* blocks with reference count > 0 */
  int64_t used_tokens;     /* tokens stored in used blocks (a shared block counts once) */
  int64_t logical_tokens;  /* sum of the sequences' context lengths (shared tokens count per sequence) */
  int64_t num_sequences;
} pa_bm_stats_t;

/* A pool of num_blocks blocks of block_size tokens, all free (ids 0..num_blocks-1
 * in the free list in that order).  Returns NULL on bad sizes or no memory. */
pa_block_manager_t *pa_bm_create(int32_t num_blocks, int32_t block_size);
void pa_bm_destroy(pa_block_manager_t *bm);

/* allocate_request: ceil(num_tokens / block_size) blocks from the front of the
 * free list, reference count 1.  slots (may be NULL) receives the slots of the
 * num_tokens prompt tokens, in order. */
pa_bm_status_t pa_bm_allocate(pa_block_manager_t *bm, int64_t seq, int32_t num_tokens, int64_t *slots);

/* share_prefix: new sequence `seq` whose first num_tokens tokens equal those of
 * `src`.  src's blocks are shared (reference count + 1) while the tokens they
 * hold fit in the prefix; the rest of the prefix gets new blocks.  The slots of
 * the tokens not covered by shared blocks go to unshared_slots (capacity
 * num_tokens, may be NULL) and their count to *num_unshared (may be NULL); the
 * caller writes those tokens' K/V. */
pa_bm_status_t pa_bm_share_prefix(pa_block_manager_t *bm, int64_t seq, int64_t src, int32_t num_tokens,
                                  int64_t *unshared_slots, int32_t *num_unshared);

/* append_token: *slot receives the slot of the sequence's next token.  If the
 * last block has room but is shared, a new block replaces it in the table and
 * (*cow_src, *cow_dst) name the copy to issue first; otherwise both are -1. */
pa_bm_status_t pa_bm_append(pa_block_manager_t *bm, int64_t seq, int64_t *slot, int64_t *cow_src,
                            int64_t *cow_dst);

/* One decode step for n sequences, in order: slots[i] as pa_bm_append; the
 * copies go to cow_pairs ([n][2], src, dst) and their count to *num_pairs.
 * Stops at the first sequence that cannot get a block (PA_BM_NO_SPACE; the
 * earlier ones are done) and reports how many were done in *num_done. */
pa_bm_status_t pa_bm_append_batch(pa_block_manager_t *bm, const int64_t *seqs, int32_t n, int64_t *slots,
                                  int64_t *cow_pairs, int32_t *num_pairs, int32_t *num_done);

/* free_request: reference counts down; blocks that reach 0 go to the back of
 * the free list (in table order). */
pa_bm_status_t pa_bm_free(pa_block_manager_t *bm, int64_t seq);

/* The block tables ([n][max_blocks_per_seq] int32, -1 past each table's end)
 * and context lengths ([n] int32, may be NULL) of n sequences, ready to upload
 * for pa_decode. */
pa_bm_status_t pa_bm_block_tables(const pa_block_manager_t *bm, const int64_t *seqs, int32_t n,
                                  int32_t *tables, int32_t max_blocks_per_seq, int32_t *context_lens);

/* Inspection. */
int32_t pa_bm_context_len(const pa_block_manager_t *bm, int64_t seq);   /* -1 if unknown */
int32_t pa_bm_ref_count(const pa_block_manager_t *bm, int32_t block);   /* -1 if out of range */
int32_t pa_bm_free_list(const pa_block_manager_t *bm, int32_t *out, int32_t cap);      /* count; first cap ids */
int32_t pa_bm_sequences(const pa_block_manager_t *bm, int64_t *out, int32_t cap);      /* count; ascending ids */
int32_t pa_bm_table(const pa_block_manager_t *bm, int64_t seq, int32_t *out, int32_t cap); /* length or -1 */
void pa_bm_stats(const pa_block_manager_t *bm, pa_bm_stats_t *out);

/*
 * Prefix caching ([B] Prefix Caching, 自动检测与复用: (1) a cache key from the
 * prompt's content, (2) the longest cached prefix of a new request, (3) only
 * the missed part computed, (4) the hit blocks shared by reference).
 *
 * Readings: the unit is a FULL prompt block (block_size tokens); a block's key
 * is its token ids together with the cache entry of the block before it, so a
 * hit on block i means the whole prefix up to block i is identical (keys are
 * looked up by an FNV-1a hash and then compared exactly: a hash collision
 * cannot share blocks).  Entry numbers are never reused.  Only prompt blocks
 * are cached (decode tokens are not).  A cached block whose reference count
 * drops to 0 keeps its content and becomes evictable; allocation takes the
 * free list first and then evicts the least recently released cached block;
 * a sequence releases its blocks last to first (pa_bm_free), so a cached
 * block's prefix is always cached too.  Every other call of this header works
 * on a prefix-caching manager as described above, taking evictable blocks
 * when the free list is empty.
 */
typedef struct {
  int64_t queried_blocks;    /* full prompt blocks looked up */
  int64_t hit_blocks;        /* of those, found in the cache */
  int64_t cached_blocks;     /* blocks currently in the cache (in use or evictable) */
  int64_t evictable_blocks;  /* cached blocks with reference count 0 */
  int64_t evictions;         /* cached blocks handed out for other content */
} pa_bm_prefix_stats_t;

/* A prefix-caching manager (otherwise as pa_bm_create). */
pa_block_manager_t *pa_bm_create_prefix_caching(int32_t num_blocks, int32_t block_size);

/* allocate_request with prefix caching: the longest run of leading full blocks
 * of token_ids[num_tokens] found in the cache is shared (reference count + 1;
 * an evictable block is taken back), new blocks hold the rest, and the new
 * full blocks are cached.  slots (may be NULL) receives the slots of all
 * num_tokens tokens; *num_cached_tokens (may be NULL) the number of leading
 * tokens whose K/V are already in the cache (a multiple of block_size): the
 * caller computes and writes only the tokens after them.  On a manager made by
 * pa_bm_create it is pa_bm_allocate with *num_cached_tokens = 0. */
pa_bm_status_t pa_bm_allocate_prompt(pa_block_manager_t *bm, int64_t seq, const int32_t *token_ids,
                                     int32_t num_tokens, int64_t *slots, int32_t *num_cached_tokens);

/* Inspection: the evictable blocks, oldest release first (count; first cap ids);
 * whether a block is cached (1, with its entry and parent entry), not (0) or
 * out of range (-1); counters. */
int32_t pa_bm_evictable(const pa_block_manager_t *bm, int32_t *out, int32_t cap);
int32_t pa_bm_cache_entry(const pa_block_manager_t *bm, int32_t block, int64_t *entry, int64_t *parent_entry);
void pa_bm_prefix_stats(const pa_block_manager_t *bm, pa_bm_prefix_stats_t *out);

#ifdef __cplusplus
}
#endif

#endif /* PA_B200_BLOCK_MANAGER_H */
