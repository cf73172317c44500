/*
 * pkv_block_manager.h -- C ABI of the host block manager in libpkv.so: the
 * bookkeeping that produces the block tables, slot mappings and copy-on-write
 * pairs consumed by the device calls of pkv.h.  Host memory only; no call
 * here touches a GPU.
 *
 * Behaviour (from the pages):
 *   - zwxr.cn "PagedAttention 与 Continuous Batching" section 3.1: fixed-size
 *     blocks; a token takes a slot when it is produced; a finished request
 *     gives back whole blocks.  Section 3.2: a per-sequence block table maps
 *     logical block i to any physical block; a new block is taken when the
 *     last one is full.  Section 3.4: blocks shared between sequences carry
 *     reference counts; a sequence about to write into a shared block gets a
 *     copy first (copy-on-write).
 *   - intelliparadigm.com "vLLM 深度解析" section 3.1: free-block list,
 *     reference counting combined with LRU reclamation.
 *   - the prefix-caching section ("4. 前缀缓存") of the article on vLLM's
 *     scheduler: every FULL block has a key = hash(previous block's key, the
 *     block's token ids, extra information); a new request reuses blocks
 *     found under its keys and skips their prefill; blocks of a finished
 *     request are parked, still holding their content, in an LRU queue that
 *     they enter from the request's tail, and are evicted least recently used
 *     first when space is needed; the hash is SHA-256.
 * Readings where the pages are silent:
 *   - key_i = SHA-256(key_{i-1} || token ids as int32 little-endian ||
 *     extras), key_{-1} = 32 zero bytes;
 *   - a new block comes from the never-cached free list (in free_order) first;
 *     a parked block is evicted only when that list is empty;
 *   - a block filled by pkv_bm_append_token is cached under its key unless
 *     another block already holds that key;
 *   - a prompt reuses cached blocks only as a leading run (the first miss
 *     ends the reuse, since every later key depends on the missed block).
 *
 * Errors: PKV_EINVAL for a null pointer, unknown sequence id or bad size;
 * PKV_ENOBLOCKS when the pool cannot supply the blocks a call needs, in
 * which case the call changes nothing.  pkv_last_error_message() (pkv.h)
 * describes the last failure of the calling thread.
 * Thread safety: one manager must not be used by two threads at once.
 */
#ifndef PKV_BLOCK_MANAGER_H
#define PKV_BLOCK_MANAGER_H

#include <stddef.h>
#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;  /* opaque, owned by the library */

typedef struct {
    int64_t num_blocks, block_size;
    int64_t free_blocks;     /* never-cached free blocks */
    int64_t parked_blocks;   /* free blocks that still hold cached content */
    int64_t used_blocks;     /* reference count > 0 */
    int64_t cached_blocks;   /* blocks holding a key (in use or parked) */
    int64_t reserved_slots;  /* used_blocks * block_size */
    int64_t token_slots;     /* slots of used blocks that hold a token (shared blocks once) */
    int64_t hit_blocks;      /* prompt blocks found in the cache, cumulative */
    int64_t evicted_blocks;  /* parked blocks reused for other content, cumulative */
    int64_t cow_copies;      /* copy-on-write pairs issued, cumulative */
    int64_t num_seqs;
} pkv_bm_stats;

/* A pool of num_blocks blocks of block_size tokens.  free_order (host,
 * num_blocks entries, may be NULL for 0..num_blocks-1) is a permutation that
 * fixes the order in which free blocks are first handed out.  prefix_cache
 * != 0 enables the key chain and the parked LRU queue.  *out receives the
 * manager; release it with pkv_bm_destroy. */
pkv_status pkv_bm_create(int64_t num_blocks, int block_size, const int32_t* free_order,
                         int prefix_cache, pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* bm);

/* A new sequence holding the prompt tokens[0..num_tokens) (host array) with
 * the request's extra key bytes (LoRA id, cache salt, ...; may be NULL when
 * extras_len == 0).  Blocks for every prompt token are taken; leading full
 * blocks found in the cache are shared instead.  *seq_id gets the id,
 * *cached_tokens the number of leading tokens whose KV is already cached
 * (a multiple of block_size; may be NULL). */
pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, const int32_t* tokens, int64_t num_tokens,
                               const void* extras, size_t extras_len, int64_t* seq_id,
                               int64_t* cached_tokens);

/* A child sharing every block of parent (parallel sampling, beam search). */
pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t* child);

/* Reserve the slot of the sequence's next token (its id is recorded for the
 * key of the block it completes).  *slot = block * block_size + offset.  If
 * the target block was shared, it is copied first: *cow_src / *cow_dst get
 * the pair for pkv_copy_blocks, else both are set to -1. */
pkv_status pkv_bm_append_token(pkv_block_manager* bm, int64_t seq_id, int32_t token, int64_t* slot,
                               int64_t* cow_src, int64_t* cow_dst);

/* One decode step for a batch: pkv_bm_append_token for seq_ids[i] and
 * tokens[i], i in [0, n), in order.  slots[n] receives the slot mapping,
 * cow_pairs[2 * k + {0, 1}] the k-th copy pair (room for n pairs) and
 * *num_cow their count.  All or nothing: if the pool cannot cover the whole
 * batch, nothing changes and PKV_ENOBLOCKS is returned. */
pkv_status pkv_bm_append_batch(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* tokens,
                               int64_t n, int64_t* slots, int64_t* cow_pairs, int64_t* num_cow);

/* Release the sequence; blocks whose count drops to 0 are parked (cached
 * full blocks, tail first) or returned to the free list. */
pkv_status pkv_bm_free_sequence(pkv_block_manager* bm, int64_t seq_id);

pkv_status pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id, int64_t* len);

/* Copy the sequence's block table into table[0..capacity); *num_blocks gets
 * its length (PKV_EINVAL if capacity is smaller). */
pkv_status pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* table,
                              int64_t capacity, int64_t* num_blocks);

/* Device-call inputs for a batch, in host memory: tables[n, max_blocks_per_seq]
 * (int32, padded with -1) and seq_lens[n] (int32). */
pkv_status pkv_bm_batch_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int64_t n,
                               int32_t* tables, int64_t max_blocks_per_seq, int32_t* seq_lens);

/* Key of the sequence's full block block_index (32 bytes); PKV_EINVAL if
 * that block is not full or caching is off. */
pkv_status pkv_bm_block_key(const pkv_block_manager* bm, int64_t seq_id, int64_t block_index,
                            uint8_t key[32]);

pkv_status pkv_bm_get_stats(const pkv_block_manager* bm, pkv_bm_stats* stats);

/* SHA-256 (FIPS 180-4) of len bytes, the hash of the key chain. */
void pkv_sha256(const void* data, size_t len, uint8_t digest[32]);

#ifdef __cplusplus
}
#endif

#endif /* PKV_BLOCK_MANAGER_H */
