/*
 * pagedkv_blocks.h — C ABI of the KV block manager and the block copies.
 *
 * The bookkeeping that sits in front of the append ("vLLM 推理引擎源码级拆解：
 * PagedAttention 显存虚拟化、Continuous Batching 调度与量化落地全指南",
 * chenxutan.com/d/5333):
 *   - §2.1: the pool is a set of equal, fixed-size blocks; several sequences
 *     may point block-table entries at one physical block, kept correct by a
 *     reference count and copy-on-write;
 *   - §2.2: a new token fills the next slot of the sequence's last block, or,
 *     when that block is full, the first slot of a block taken from the free
 *     pool and appended to the block table;
 *   - §3.1: the scheduler asks can_allocate / allocate for a new request and
 *     can_append / append_slot for each running one;
 *   - §3.2: a preempted request either frees its blocks (to be recomputed) or
 *     has them swapped out to host memory and back;
 *   - §3.3: the manager keeps the ledger only (owners, reference counts, the
 *     free pool) and never touches the cache memory itself;
 *   - §4.2: with prefix caching, each full block is named by a hash of its
 *     token ids and of the hash of the block before it; a new request whose
 *     block hashes are already cached points at those blocks (reference count
 *     + 1) instead of computing them, and cached blocks that no sequence holds
 *     any more are reclaimed least-recently-used first.
 * "vLLM 深度实战" (chenxutan.com/d/3332) §1.2 gives the same block with its
 * reference count and the per-sequence block table, and returns a finished
 * sequence's blocks to the pool at once.
 *
 * The manager is host code. Its outputs (slot mappings, block tables, copy
 * lists) are plain host arrays that the caller moves to the device for
 * paged_kv_append, paged_attention_decode and the block copies below.
 *
 * Conventions:
 *   - A manager is not thread-safe: one thread at a time per manager.
 *   - Sequence ids are caller-chosen int64 values, unique among live sequences.
 *   - Every call checks its arguments and returns a pkv_status (< 0 on error);
 *     a failed call leaves the manager exactly as it was.
 *   - Block ids are int32 in [0, num_blocks) for the device pool and
 *     [0, num_host_blocks) for the host pool.
 */
#ifndef PAGEDKV_BLOCKS_H
#define PAGEDKV_BLOCKS_H

#include <stddef.h>
#include <stdint.h>

#include "pagedkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_block_manager pkv_block_manager;

/* Creates a manager of num_blocks device blocks and num_host_blocks host
 * blocks (swap space; may be 0) of block_size tokens. prefix_caching != 0
 * enables the §4.2 block hashes. Returns NULL on bad sizes or no memory. */
pkv_block_manager* pkv_bm_create(int64_t num_blocks, int64_t num_host_blocks, int block_size,
                                 int prefix_caching);
void pkv_bm_destroy(pkv_block_manager* bm);

/* Device blocks that can be handed out now: free ones plus cached blocks no
 * sequence holds (prefix caching), which are evicted on demand. */
int64_t pkv_bm_num_free(const pkv_block_manager* bm);
int64_t pkv_bm_num_free_host(const pkv_block_manager* bm);

/* 1 if a prompt of num_tokens tokens fits in the free blocks (counting no
 * cache hits), else 0 (§3.1 can_allocate). */
int pkv_bm_can_allocate(const pkv_block_manager* bm, int64_t num_tokens);

/* Admits sequence seq_id with the prompt token_ids[0..num_tokens) (§3.1
 * allocate): one block per block_size tokens, the last one possibly partial.
 * With prefix caching, full blocks whose hash chain and token ids match a
 * cached block share it instead.
 *   slot_mapping  host int64[num_tokens] out: the slot each prompt token's K/V
 *                 must be written to, or -1 for tokens of shared cached blocks
 *                 (already present; paged_kv_append skips negative slots).
 *                 May be NULL.
 *   num_cached    out (may be NULL): the number of leading prompt tokens held
 *                 by cached blocks, whose computation can be skipped.
 * Errors: PKV_ERR_SEQ (id in use), PKV_ERR_NO_BLOCKS, PKV_ERR_NULL (token_ids
 * NULL with num_tokens > 0 and prefix caching on), PKV_ERR_SHAPE. */
int pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, const int32_t* token_ids,
                    int64_t num_tokens, int64_t* slot_mapping, int64_t* num_cached);

/* 1 if append_slot for seq_id would succeed, else 0 (§3.1 can_append). */
int pkv_bm_can_append(const pkv_block_manager* bm, int64_t seq_id);

/* Reserves the slot of the sequence's next token (§2.2 append_slot) and
 * records its id for the block hash. If the last block is full, a new block is
 * taken. If the last block is partial and shared (after pkv_bm_fork), it is
 * copied first (copy-on-write, §2.1): *cow_src / *cow_dst receive the source
 * and the new private block, which the caller copies with paged_kv_copy_blocks
 * before writing the slot; otherwise both are -1.
 * Errors: PKV_ERR_SEQ, PKV_ERR_NO_BLOCKS, PKV_ERR_NULL. */
int pkv_bm_append_slot(pkv_block_manager* bm, int64_t seq_id, int32_t token_id, int64_t* slot,
                       int64_t* cow_src, int64_t* cow_dst);

/* One decode step for a batch: append_slot for each of seq_ids[0..n) (distinct,
 * resident) with token_ids[i], all or nothing.
 *   slot_mapping  host int64[n] out: each sequence's new slot, ready for
 *                 paged_kv_append
 *   cow_pairs     host int64[2 * n] out: the copy-on-write (src, dst) pairs of
 *                 this step, *num_cow of them, to run with paged_kv_copy_blocks
 *                 before the append
 * If the free blocks cannot cover every sequence that needs a new block or a
 * copy, nothing changes and PKV_ERR_NO_BLOCKS is returned. Errors also
 * PKV_ERR_SEQ (unknown, swapped-out or repeated id), PKV_ERR_NULL. */
int pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* token_ids,
                        int n, int64_t* slot_mapping, int64_t* cow_pairs, int64_t* num_cow);

/* Makes child_id a sequence that shares every block of parent_id (parallel
 * sampling, beam search: §2.1 / "pgsm.cn/news/372185" §2.2). Errors:
 * PKV_ERR_SEQ (parent unknown or swapped out, child in use). */
int pkv_bm_fork(pkv_block_manager* bm, int64_t parent_id, int64_t child_id);

/* Releases the sequence's blocks (finished, or preempted for recomputation). */
int pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);

/* Swap-out of a group of sequences (§3.2): each distinct device block they
 * hold gets a host block; blocks held by several of them map to one host
 * block. pairs (host int64[2 * max_pairs], out) receives (device block, host
 * block) per copy and *num_pairs their count; the caller copies them with
 * paged_kv_swap_blocks before the device blocks are reused. The device blocks
 * are released (those other sequences still hold stay). Errors: PKV_ERR_SEQ,
 * PKV_ERR_NO_BLOCKS (host pool), PKV_ERR_SHAPE (max_pairs too small). */
int pkv_bm_swap_out(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int64_t* pairs,
                    int64_t max_pairs, int64_t* num_pairs);
/* Swap-in, the reverse: pairs receive (host block, device block). */
int pkv_bm_swap_in(pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int64_t* pairs,
                   int64_t max_pairs, int64_t* num_pairs);

/* Block tables and lengths of resident sequences, for paged_attention_decode:
 * table (host int32[num_seqs * max_blocks_per_seq], out) row i lists the
 * blocks of seq_ids[i], padded with -1; seq_lens (host int32[num_seqs], out).
 * Errors: PKV_ERR_SEQ, PKV_ERR_SHAPE (a sequence needs more than
 * max_blocks_per_seq blocks). */
int pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs,
                        int max_blocks_per_seq, int32_t* table, int32_t* seq_lens);

/* Length of a live sequence, or PKV_ERR_SEQ. */
int64_t pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id);
/* Reference count of a device block (0 for free or cached-unheld), or
 * PKV_ERR_SHAPE for an id out of range. */
int pkv_bm_refcount(const pkv_block_manager* bm, int32_t block);
/* Pool usage, the ledger's metrics (the pages' KV-pool usage gauge, p4 §6.6):
 * out (host int64[6]) receives num_blocks, blocks held by resident sequences,
 * cached blocks no sequence holds, free blocks, tokens of resident sequences
 * (each sequence counted), and the slots of held blocks that hold a token
 * (a shared block counted once, at its fullest). Fragmentation of the held
 * blocks is 1 - used slots / (held * block_size). */
int pkv_bm_usage(const pkv_block_manager* bm, int64_t* out);

/* Full consistency check of the ledger: every reference count equals the
 * number of table entries that point at the block, and every block is exactly
 * one of held, free, or cached-unheld. PKV_OK or PKV_ERR_SHAPE. */
int pkv_bm_check(const pkv_block_manager* bm);

/*
 * paged_kv_copy_blocks — copy-on-write copies inside one pool (§2.1).
 *
 *   k_cache,
 *   v_cache        device pool [num_blocks, ...] of block_bytes per block
 *   block_mapping  device int64[num_pairs, 2]: (src, dst) block ids
 *   block_bytes    bytes of one block of K (and of V): block_size *
 *                  num_kv_heads * head_dim * element size; a multiple of 16
 * Every pair copies K[src] -> K[dst] and V[src] -> V[dst] byte for byte. Pairs
 * whose ids fall outside [0, num_blocks) copy nothing. No block may be the
 * destination of one pair and the source or destination of another in the
 * same call (the copies run concurrently). Enqueued on `stream`.
 * Errors: PKV_ERR_NULL, PKV_ERR_SHAPE, PKV_ERR_ALIGN, PKV_ERR_CUDA.
 */
int paged_kv_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                         int num_pairs, int64_t block_bytes, int64_t num_blocks, void* stream);

/*
 * paged_kv_swap_blocks — block copies between two pools (§3.2 swap), either of
 * which may be pinned host memory (page-locked, e.g. cudaHostAlloc or a
 * pinned torch tensor) that the kernel reads or writes directly over the
 * host link.
 *
 *   src_k, src_v   pool of src_num_blocks blocks (device or pinned host)
 *   dst_k, dst_v   pool of dst_num_blocks blocks (device or pinned host)
 *   block_mapping  device int64[num_pairs, 2]: (src block, dst block)
 * Pairs with an id out of its pool's range copy nothing; destinations must be
 * distinct. A pool pointer that is neither device memory nor pinned host
 * memory (checked with cudaPointerGetAttributes at both ends of the pool) is
 * rejected with PKV_ERR_MEMORY. Errors otherwise as for paged_kv_copy_blocks.
 */
int paged_kv_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                         const int64_t* block_mapping, int num_pairs, int64_t block_bytes,
                         int64_t src_num_blocks, int64_t dst_num_blocks, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_BLOCKS_H */
