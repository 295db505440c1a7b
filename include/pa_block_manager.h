/*
 * pa_block_manager.h -- the host block manager of libpa.so: the allocator that
 * produces the block_tables and slot_mapping the kernels of pa.h consume, and
 * the (source, destination) block pairs that pa_copy_blocks executes.
 *
 * It is the block manager the pages describe:
 *   [KV量化]          "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置"
 *                     (BlockManager: free_blocks, allocate, append_token)
 *   [深度解析]         "LLM推理优化：vLLM PagedAttention深度解析与工程实践"
 *                     §3.2 (allocation, free), §4.2 (automatic prefix caching)
 *   [KVcache-learning] "KVcache-learning" s05 (copy-on-write), s06 (block manager:
 *                     allocate, copy-on-write, swap_out / swap_in, free), s08
 *                     (prefix cache)
 * with these readings of points they leave open:
 *   - block ids come from the END of the free list and freed ids go back to the
 *     end ([KV量化], s06; [深度解析] §3.2 takes the front instead);
 *   - a sequence of n tokens holds ceil(n / block_size) blocks; appending takes
 *     a new block only when the last one is full;
 *   - copy-on-write on append: a shared, partly filled last block is replaced by a
 *     fresh block, and the caller copies (old, fresh) with pa_copy_blocks
 *     before the token's K/V is written;
 *   - prefix caching (optional) indexes FULL blocks by a 64-bit FNV-1a key over
 *     the previous block's key (8 bytes, little endian) and the block's tokens
 *     (4 bytes each, little endian); the first block's parent is the FNV offset
 *     basis.  A hit also compares the stored parent key and tokens.  A prompt's
 *     last token is never taken from the cache.  A cached block whose last user
 *     leaves stays cached (evictable).  A new block comes from the free list
 *     first, then from the evictable block released longest ago (its key is
 *     dropped);
 *   - swap moves a group of sequences; a block shared inside the group moves once
 *     and stays shared; the returned (source, destination) pairs are for
 *     pa_copy_blocks between the GPU and CPU pools, to run before the freed
 *     blocks are written again.
 *
 * Conventions: everything is host memory; nothing here touches the GPU.  Every
 * call validates first and changes nothing when it fails:
 * PA_ERR_INVALID_ARG for a bad handle, unknown or duplicate sequence id, wrong
 * residency (a swapped-out sequence cannot grow), or an output buffer that is
 * too small; PA_ERR_NO_SPACE when the pool lacks free blocks.  A manager is
 * not thread-safe: calls on one manager must not overlap.
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* A manager over num_gpu_blocks device blocks and num_cpu_blocks host blocks of
 * block_size tokens; prefix_caching != 0 enables the prefix cache.  NULL on
 * bad arguments or out of host memory.  Free it with pa_bm_destroy. */
PA_API pa_block_manager* pa_bm_create(int num_gpu_blocks, int num_cpu_blocks, int block_size,
                                      int prefix_caching);
PA_API void pa_bm_destroy(pa_block_manager* m);

/* Blocks a new allocation can take: free plus evictable (GPU); free (CPU). */
PA_API int pa_bm_free_gpu_blocks(const pa_block_manager* m);
PA_API int pa_bm_free_cpu_blocks(const pa_block_manager* m);

/* Admit a sequence with its prompt tokens[num_tokens] (num_tokens >= 1).
 * slot_mapping[num_tokens] receives each token's slot (block * block_size +
 * offset), or -1 for a token whose K/V is already cached.  *num_cached, if not
 * NULL, receives the cached prefix length (a multiple of block_size). */
PA_API int pa_bm_add_sequence(pa_block_manager* m, int64_t seq_id, const int32_t* tokens,
                              int num_tokens, int64_t* slot_mapping, int* num_cached);

/* Append one token: *slot receives its slot.  If the sequence's last block was
 * shared, *cow_src / *cow_dst (if not NULL) receive the block pair to copy
 * before the write; otherwise -1. */
PA_API int pa_bm_append_token(pa_block_manager* m, int64_t seq_id, int32_t token, int64_t* slot,
                              int64_t* cow_src, int64_t* cow_dst);

/* One decode step for a batch: appends tokens[i] to seq_ids[i] (distinct,
 * resident) and writes slot_mapping[num_seqs].  The copy-on-write pairs go to
 * cow_pairs[*num_cow][2] (room for num_seqs pairs; may be NULL to drop them).
 * The space check counts one block for every sequence whose last block is full
 * or shared before any of the batch's appends. */
PA_API int pa_bm_append_batch(pa_block_manager* m, const int64_t* seq_ids, const int32_t* tokens,
                              int num_seqs, int64_t* slot_mapping, int64_t* cow_pairs,
                              int* num_cow);

/* child_id shares every block of parent_id (parallel sampling, beam search). */
PA_API int pa_bm_fork(pa_block_manager* m, int64_t parent_id, int64_t child_id);

/* Release a sequence (resident or swapped out). */
PA_API int pa_bm_free_sequence(pa_block_manager* m, int64_t seq_id);

/* Move the group seq_ids[num_seqs] to the CPU pool (swap_out) or back (swap_in).
 * mapping[capacity][2] receives *num_pairs (source block, destination block)
 * pairs, in first-seen order: GPU -> CPU for swap_out, CPU -> GPU for swap_in. */
PA_API int pa_bm_swap_out(pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                          int64_t* mapping, int capacity, int* num_pairs);
PA_API int pa_bm_swap_in(pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                         int64_t* mapping, int capacity, int* num_pairs);

/* A sequence's block ids (table[capacity]), block count and token count.  The
 * counts are written even when capacity is too small (then PA_ERR_INVALID_ARG),
 * so a call with capacity 0 asks for the size. */
PA_API int pa_bm_block_table(const pa_block_manager* m, int64_t seq_id, int32_t* table,
                             int capacity, int* num_blocks, int* num_tokens);

/* The decode batch for resident sequences seq_ids[num_seqs]: block_tables
 * int32 [num_seqs][max_blocks] (padding -1) and seq_lens int32 [num_seqs], the
 * arguments of pa_decode_v1 / pa_append_decode_v1. */
PA_API int pa_bm_build_batch(const pa_block_manager* m, const int64_t* seq_ids, int num_seqs,
                             int32_t* block_tables, int max_blocks, int32_t* seq_lens);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H_ */
