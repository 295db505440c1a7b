/*
 * pa.h -- C ABI of libpa.so: paged KV-cache write and paged decode attention
 * for NVIDIA B200 (sm_100a).
 *
 * Pages the operations come from (cited by title and section):
 *   [vllm-musa]  "KV Cache 与 PagedAttention（vllm-musa 实战）" (7yue.com)
 *   [KV量化]      "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置" (yunthe.com)
 *   [深度解析]     "LLM推理优化：vLLM PagedAttention深度解析与工程实践" (jsqmd.com)
 *   [KVcache-learning] "KVcache-learning" (fairy2021.github.io), chapters s00-s13
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *   never allocates or frees memory, never synchronises, and enqueues its work
 *   on `stream` (NULL = the legacy default stream).  Results are visible once
 *   the caller synchronises with that stream.
 * - Tensors are dense and row-major in the layouts given below; the only
 *   explicit stride is the row stride of block_tables (max_blocks_per_seq).
 * - K/V cache layout: [num_blocks, block_size, num_kv_heads, head_dim] for
 *   both K and V ([深度解析] §4.1).  Token t of sequence s is at block
 *   block_tables[s * max_blocks_per_seq + t / block_size], offset
 *   t % block_size ([vllm-musa] §五; [深度解析] §3.1).
 * - Quantised caches (PA_INT8, PA_FP8E4M3) carry one fp32 scale per token per
 *   kv head: k_scale / v_scale [num_blocks, num_kv_heads, block_size]; the
 *   stored value is code * scale.
 * - GQA: query head h reads kv head h / (num_heads / num_kv_heads).
 * - Supported: head_dim 64 or 128; block_size 8, 16 or 32; num_heads /
 *   num_kv_heads <= 8; q / cache dtype pairs (f16,f16) (bf16,bf16)
 *   (f32,f32) and (f16|bf16, int8|fp8).  Others return PA_ERR_UNSUPPORTED.
 * - Return value: a pa_status.  Host-side argument checks come first and
 *   return PA_ERR_INVALID_ARG / PA_ERR_UNSUPPORTED without touching the GPU;
 *   a failed launch returns PA_ERR_CUDA.
 * - err_flag: optional device int.  When non-NULL the kernels also check the
 *   data-dependent bounds (block ids inside [0, num_blocks), seq_len within
 *   the table, slots inside the pool); a violation OR-s a PA_DEVERR_* bit into
 *   *err_flag and the offending access is skipped (never a trap): a bad block
 *   id drops that block's tokens, a bad seq_len drops the whole sequence
 *   (its output is zeros).  When NULL those bounds are the caller's contract
 *   and are not checked.
 * - Every wait inside a kernel has a time limit; a wait that runs out sets
 *   PA_DEVERR_TIMEOUT (in err_flag and in the library's device error word,
 *   see pa_get_device_error) and the kernel returns without hanging.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define PA_API __declspec(dllexport)
#else
#define PA_API __attribute__((visibility("default")))
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* pa_stream_t;

typedef enum {
  PA_F32 = 0,
  PA_F16 = 1,
  PA_BF16 = 2,
  PA_INT8 = 3,
  PA_FP8E4M3 = 4
} pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_CUDA = 3,
  PA_ERR_NO_SPACE = 4     /* block manager: not enough free blocks; nothing changed */
} pa_status;

/* Bits reported through err_flag / pa_get_device_error. */
#define PA_DEVERR_BLOCK_ID 1
#define PA_DEVERR_SEQ_LEN 2
#define PA_DEVERR_SLOT 4
#define PA_DEVERR_TIMEOUT 8

/*
 * pa_reshape_and_cache -- write each new token's K and V row into its slot.
 * The write a block manager performs when a token is appended to a sequence
 * ([KV量化] BlockManager.append_token; [KVcache-learning] s06 allocate_token_block);
 * the INT8 / FP8 modes follow [KVcache-learning] s09 (E4M3, range +-448) and
 * [KV量化] kv_cache_dtype="int8".
 *
 *   key, value     [num_tokens, num_kv_heads, head_dim], dtype src_dtype
 *                  (PA_F32, PA_F16 or PA_BF16).
 *   k_cache/v_cache  cache_dtype; == src_dtype copies the row bit for bit.
 *                  PA_INT8: per (token, head) a = max|x|, s = a / 127 (fp32),
 *                  code = clamp(rne(x / s), -127, 127).  PA_FP8E4M3:
 *                  s = a / 448, code = e4m3(x / s), round to nearest even,
 *                  saturating to +-448.  A row of zeros stores s = 0 and
 *                  codes 0.  All divisions are IEEE fp32, round to nearest.
 *   k_scale/v_scale  fp32 [num_blocks, num_kv_heads, block_size]; required
 *                  for quantised caches, ignored (may be NULL) otherwise.
 *   slot_mapping   int64 [num_tokens]; slot = block * block_size + offset.
 *                  A negative slot skips that token, and so does a slot at or
 *                  past num_blocks * block_size (always; with err_flag it also
 *                  sets PA_DEVERR_SLOT).  Two tokens with the same slot in one
 *                  call race (unspecified winner).
 *   num_tokens may be 0 (nothing is launched).
 */
PA_API int pa_reshape_and_cache(const void* key, const void* value, pa_dtype src_dtype,
                                void* k_cache, void* v_cache, pa_dtype cache_dtype,
                                float* k_scale, float* v_scale, const int64_t* slot_mapping,
                                int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, int* err_flag, pa_stream_t stream);

/*
 * pa_prefill -- multi-token query over the paged cache: each sequence's last
 * q_len tokens (already written to the cache, e.g. by pa_reshape_and_cache)
 * attend causally to every cached token up to and including themselves.  This
 * is the prefill that automatic prefix caching leaves to compute: a request
 * whose prompt starts with cached blocks computes only its new tokens
 * ([深度解析] §4.2; [KVcache-learning] s08).  Row r of sequence s sits at
 * position seq_lens[s] - q_len + r and gets softmax(scale q K^T) V over tokens
 * [0, position].  Runs on the tcgen05 tensor cores.
 *
 *   q, out         [total_q, num_heads, head_dim], rows of sequence s at
 *                  [query_start[s], query_start[s + 1]); dtype q_dtype.
 *   query_start    int32 [num_seqs + 1], query_start[0] = 0, nondecreasing;
 *                  0 <= q_len <= seq_lens[s].
 *   max_query_len  >= every q_len (sets the grid).
 *   Other arguments as pa_decode_v1.  Supported: head_dim 128; q and caches
 *   both PA_F16 or both PA_BF16; num_heads / num_kv_heads dividing 128.
 *   A sequence with a bad q_len or seq_len is skipped (PA_DEVERR_SEQ_LEN when
 *   err_flag is given).  A bad block id is read as zeros and sets
 *   PA_DEVERR_BLOCK_ID in err_flag.
 */
PA_API int pa_prefill(void* out, const void* q, pa_dtype q_dtype, const int32_t* query_start,
                      int total_q, int max_query_len, const void* k_cache, const void* v_cache,
                      pa_dtype cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, float scale, int* err_flag,
                      pa_stream_t stream);

/*
 * pa_decode_cascade -- pa_decode_v1 for a batch whose sequences all begin with
 * the same cached prefix (the same physical blocks: a shared system prompt,
 * copy-on-write sharing, [KVcache-learning] s05; automatic prefix caching,
 * [深度解析] §4.2).  Same result as pa_decode_v1, computed in three launches:
 *   1. the tcgen05 kernel of pa_prefill attends every sequence's query rows to
 *      the shared prefix at once, so the prefix K/V are read once per kv head,
 *      not once per sequence; it leaves (o / l, m, l) partials in `workspace`;
 *   2. the persistent decode of pa_decode_fused covers each sequence's own
 *      tokens [prefix_len, seq_len), every warp an equal share, and leaves one
 *      more partial.  It reads nothing launch 1 writes and never waits for it
 *      (only its last CTA does, so launch 3 runs after both);
 *   3. a merge combines the partials by log-sum-exp and writes out.
 * Placement.  Side by side: launch 1 is split along the prefix over at most
 * half the SMs (up to 4 CTAs per 256 query rows, one CTA per SM), and launch 2
 * gets a grid for exactly the other SMs (three CTAs per SM), so the two run at
 * once.  Split: launch 1 is split over up to 4 CTAs per 256 query rows to fill
 * the GPU, and launch 2 follows on every SM.  Side by side needs PDL on
 * (pa_set_pdl >= 1) and one CTA per 256 query rows of a kv head on at most half
 * the SMs.  The automatic choice (no split count set) takes it when both forms
 * would split the prefix equally; otherwise only when the prefix CTAs fill at
 * least a third of the SMs and the table width (max_blocks_per_seq * block_size
 * - prefix_len) is at least half the prefix, since it pays when the sequences'
 * own tokens keep the suffix busy about as long as the prefix, which the host
 * cannot see.  pa_set_cascade_config(-1, ...) asks for side by side whenever it
 * fits.
 * (pa_set_cascade_config(splits, 1) runs instead, as launch 2, the v1 decode
 * of each sequence's own tokens merging the prefix partials in its epilogue.)
 *
 *   prefix_len     tokens of the shared prefix, a multiple of block_size, <=
 *                  every seq_len; block_tables[s][0 .. prefix_len / block_size)
 *                  must be the same block ids for every s (launch 1 reads row
 *                  0).  0 runs plain pa_decode_v1.
 *   workspace      device memory, 256-byte aligned, at least
 *                  pa_decode_cascade_workspace_bytes(num_seqs, num_heads,
 *                  head_dim) bytes, zero-filled before its first use (every
 *                  complete call leaves its counters at zero again).  Calls that
 *                  share a workspace must not overlap on the GPU.
 *   Supported: head_dim 128; q and caches both PA_F16 or both PA_BF16;
 *   num_heads / num_kv_heads dividing 128.  Other arguments as pa_decode_v1.
 */
PA_API int pa_decode_cascade(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                             const void* v_cache, pa_dtype cache_dtype,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* seq_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                             float scale, int prefix_len, void* workspace,
                             size_t workspace_bytes, int* err_flag, pa_stream_t stream);

/* Workspace bytes of pa_decode_cascade on the current device: the partials of
 * up to 4 prefix splits and of the suffix (5 * num_seqs * num_heads *
 * (head_dim + 2) * 4, rounded up to 256), the persistent decode's workspace
 * (pa_decode_fused_workspace_bytes with num_kv_heads = num_heads and the
 * device's SM count) and 256 bytes of counter. */
PA_API size_t pa_decode_cascade_workspace_bytes(int num_seqs, int num_heads, int head_dim);

/* Knobs of pa_decode_cascade (process-wide): prefix_splits = KV splits of the
 * prefix launch (1..4, the split placement; 0 = automatic, see pa_decode_cascade;
 * -1 = side by side whenever it fits), suffix_form = 0 persistent decode + merge
 * launch (default), 1 the v1 decode merging in its epilogue. */
PA_API int pa_set_cascade_config(int prefix_splits, int suffix_form);

/*
 * pa_copy_blocks -- copy whole KV blocks from one block pool to another, or
 * within one pool.  Copy-on-write of a shared block ([KVcache-learning] s05
 * "写时复制": before a sequence writes into a block that other sequences
 * share, the block is copied to a free id and that sequence's table is
 * repointed) and swap between the GPU pool and a CPU pool ([KVcache-learning]
 * s06 swap_out / swap_in; [KV量化] swap_space) are both this call.
 *
 *   src_*_cache    [src_num_blocks, block_size, num_kv_heads, head_dim],
 *                  dtype cache_dtype; src_*_scale fp32 [src_num_blocks,
 *                  num_kv_heads, block_size] for PA_INT8 / PA_FP8E4M3 caches
 *                  (ignored, may be NULL, otherwise).
 *   dst_*          the same for the destination pool (dst_num_blocks blocks);
 *                  may be the source arrays themselves.
 *   block_mapping  int64 [num_pairs, 2] in device memory: row p = (src id,
 *                  dst id).  Destination block dst becomes a bit-for-bit copy of
 *                  source block src: K, V and, when quantised, both scales.
 *                  Destination ids must be distinct, and within one pool no
 *                  destination may also be a source in the same call.
 *                  Otherwise the result is unspecified.
 *   num_pairs may be 0 (nothing is launched).
 *
 * Every pointer is device memory or pinned host memory mapped into the device
 * address space (cudaHostAlloc / pinned PyTorch tensors).  So a destination in
 * host memory is a swap-out and a source in host memory is a swap-in.  Caches
 * and scale arrays must be 16-byte aligned, block_mapping 8-byte aligned.  A
 * pair with an id outside its pool is always skipped and sets
 * PA_DEVERR_BLOCK_ID (in err_flag when given, and in the library's device
 * error word).  Asynchronous on `stream`; nothing is allocated.
 */
PA_API int pa_copy_blocks(const void* src_k_cache, const void* src_v_cache,
                          const float* src_k_scale, const float* src_v_scale, int src_num_blocks,
                          void* dst_k_cache, void* dst_v_cache, float* dst_k_scale,
                          float* dst_v_scale, int dst_num_blocks, pa_dtype cache_dtype,
                          const int64_t* block_mapping, int num_pairs, int num_kv_heads,
                          int head_dim, int block_size, int* err_flag, pa_stream_t stream);

/*
 * pa_decode_v1 -- single-pass paged decode attention ([深度解析] §4.1
 * paged_attention_v1; kernel arguments as in [vllm-musa] §五):
 *   out[s, h, :] = sum_t softmax_t(scale * q[s,h,:] . K_t) V_t
 * over the seq_lens[s] cached tokens of sequence s, one softmax over all of
 * them ([深度解析] §二; [KVcache-learning] s05).  One CTA per (sequence,
 * kv head) reads each K/V byte once for the whole GQA group.
 *
 *   out            [num_seqs, num_heads, head_dim], dtype q_dtype.  A
 *                  sequence with seq_len 0 gets zeros.
 *   q              [num_seqs, num_heads, head_dim], dtype q_dtype.
 *   block_tables   int32 [num_seqs, max_blocks_per_seq]; entries past
 *                  ceil(seq_len / block_size) are never read.
 *   seq_lens       int32 [num_seqs], 0 <= seq_len <= max_blocks_per_seq * block_size.
 *   scale          softmax scale (typically 1/sqrt(head_dim)).
 */
PA_API int pa_decode_v1(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                        const void* v_cache, pa_dtype cache_dtype, const float* k_scale,
                        const float* v_scale, const int32_t* block_tables,
                        int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                        int num_heads, int num_kv_heads, int head_dim, int block_size,
                        int num_blocks, float scale, int* err_flag, pa_stream_t stream);

/*
 * pa_append_decode_v1 -- one decode step in ONE launch: the cache write of
 * each sequence's new token (pa_reshape_and_cache with num_tokens = num_seqs)
 * followed by pa_decode_v1 over the sequences, the new token included.  The
 * result equals those two calls made in that order.  This is the step the pages
 * describe: append the token to the sequence's last block ([KV量化]
 * BlockManager.append_token), then attend over all cached tokens ([深度解析]
 * §4.1 paged_attention_v1).
 *
 *   key, value     [num_seqs, num_kv_heads, head_dim], dtype q_dtype: the new
 *                  token's K and V rows.
 *   slot_mapping   int64 [num_seqs]: the slot of sequence s's new token.  It must
 *                  be the slot block_tables[s] gives for token seq_lens[s] - 1,
 *                  in a block no other sequence of the call reads.  A block
 *                  manager guarantees this by copy-on-write before appending.  A
 *                  negative slot writes nothing.  A slot past the pool writes
 *                  nothing and sets PA_DEVERR_SLOT.  With err_flag, a slot that
 *                  is not the table's slot for token seq_lens[s] - 1 is also
 *                  not written and sets PA_DEVERR_SLOT (without err_flag that
 *                  contract is not checked: such a write may race with another
 *                  warp's load of the tile it lands in).
 *   k_cache, v_cache, k_scale, v_scale  written (the new rows) and read.
 *   Other arguments as pa_decode_v1.  Inside the kernel, the warp that loads a
 *   sequence's last tile writes the new rows first, then loads the tile.  fp32
 *   caches run the cache write and the pa_decode_v1 kernel as two launches.
 */
PA_API int pa_append_decode_v1(void* out, const void* q, pa_dtype q_dtype, const void* key,
                               const void* value, const int64_t* slot_mapping, void* k_cache,
                               void* v_cache, pa_dtype cache_dtype, float* k_scale,
                               float* v_scale, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                               int num_heads, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, float scale, int* err_flag, pa_stream_t stream);

/*
 * pa_decode_v2_partition -- the split-K half of paged_attention_v2
 * ([深度解析] §4.1 "先 partial accumulate，再 merge").  Partition p of
 * sequence s covers tokens [p*P, min((p+1)*P, seq_len)), P = partition_size
 * (a multiple of max(16, block_size)); one CTA per (sequence, kv head,
 * partition).  For every non-empty partition it writes
 *   max_logits[s, h, p] = m_p = max_t scale * q . K_t            (natural log units)
 *   exp_sums  [s, h, p] = l_p = sum_t exp(scale * q . K_t - m_p)
 *   tmp_out   [s, h, p, :] = sum_t exp(... - m_p) V_t / l_p
 * with max_logits, exp_sums fp32 [num_seqs, num_heads, max_num_partitions] and
 * tmp_out fp32 [num_seqs, num_heads, max_num_partitions, head_dim].  Entries
 * of partitions at or past ceil(seq_len / P) are left untouched.
 * max_num_partitions must be >= ceil(max seq_len / P).  Other arguments as
 * pa_decode_v1.
 */
PA_API int pa_decode_v2_partition(float* tmp_out, float* max_logits, float* exp_sums,
                                  const void* q, pa_dtype q_dtype, const void* k_cache,
                                  const void* v_cache, pa_dtype cache_dtype,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int max_blocks_per_seq,
                                  const int32_t* seq_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  float scale, int partition_size, int max_num_partitions,
                                  int* err_flag, pa_stream_t stream);

/*
 * pa_decode_v2_merge -- the merge half of paged_attention_v2: the
 * log-sum-exp combination of the partitions of each (sequence, head):
 *   M = max_p m_p,  w_p = l_p exp(m_p - M),  out = sum_p w_p o_p / sum_p w_p
 * over the ceil(seq_len / P) partitions of the sequence (partitions with
 * l_p = 0 are skipped; seq_len 0 gives zeros).  out dtype: PA_F32, PA_F16 or
 * PA_BF16, [num_seqs, num_heads, head_dim].
 */
PA_API int pa_decode_v2_merge(void* out, pa_dtype out_dtype, const float* tmp_out,
                              const float* max_logits, const float* exp_sums,
                              const int32_t* seq_lens, int num_seqs, int num_heads, int head_dim,
                              int partition_size, int max_num_partitions, pa_stream_t stream);

/*
 * pa_decode_fused -- the same attention as pa_decode_v1 / v2 in ONE launch,
 * scheduled for B200: a persistent grid (a few CTAs per SM) in which every warp
 * streams an equal contiguous share of the batch's 16-token tiles, in
 * (sequence, kv head) order, through its own TMA pipeline.  A (sequence, kv
 * head) that falls inside one warp's share is written to `out` directly; one
 * split between warps is merged by log-sum-exp by the warp that finishes it
 * last (split-K partitions and merge of [深度解析] §4.1, with partition
 * boundaries set by load balance instead of a fixed size).
 *
 *   workspace      device memory of at least
 *                  pa_decode_fused_workspace_bytes(num_seqs, num_kv_heads,
 *                  head_dim, <SM count of the device>) bytes, 256-byte aligned,
 *                  ZEROED BEFORE ITS FIRST USE.  It holds per-(sequence, kv
 *                  head) arrival counters, which every complete call leaves at
 *                  zero, and the per-warp partial records.  Calls that share a
 *                  workspace must not overlap on the GPU.  After a call that
 *                  reported PA_DEVERR_TIMEOUT, zero it again.
 *   num_seqs <= 8192; other arguments as pa_decode_v1.  fp32 caches run the
 *   pa_decode_v1 kernel (the workspace is then unused).
 *   Returns PA_ERR_INVALID_ARG if the workspace is missing, misaligned or too
 *   small.  Results are deterministic for a given batch.
 */
PA_API int pa_decode_fused(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                           const void* v_cache, pa_dtype cache_dtype, const float* k_scale,
                           const float* v_scale, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float scale, void* workspace, size_t workspace_bytes,
                           int* err_flag, pa_stream_t stream);

/* Workspace bytes pa_decode_fused needs on a device with num_sms SMs. */
PA_API size_t pa_decode_fused_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim,
                                              int num_sms);

/*
 * pa_decode_fused_noalloc -- pa_decode_fused without a caller workspace.  The
 * pages have no counterpart: this exists for callers that cannot allocate
 * device memory where they call (an inference-engine plugin whose enqueue step
 * must not allocate, a library with no allocator of its own because a
 * framework's caching allocator holds the device memory, a server that has
 * given nearly all of HBM to its KV block pool).
 *
 * The scratch is a fixed 24 MiB device array inside this library
 * (pa_decode_fused_noalloc_scratch_bytes()); every GPU that loads the library
 * holds it until the process exits.  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress); make that first call
 * before any stream capture.  The address is kept per device and context: after
 * the device's context is replaced (cudaDeviceReset) the next call looks it up
 * again, so that call too belongs outside a capture.  Host argument checks run
 * before anything touches the GPU.  Every call clears the arrival counters it needs
 * (a cudaMemsetAsync on `stream`) and otherwise reuses the array as it was
 * left, so calls that overlap on the GPU -- on different streams, or from
 * several threads -- race on it and must be serialised by the caller.  It
 * allocates and frees nothing.  Shapes whose scratch would exceed the array
 * (pa_decode_fused_workspace_bytes(...) > 24 MiB) return PA_ERR_UNSUPPORTED.
 * Arguments and results otherwise as pa_decode_fused.
 */
PA_API int pa_decode_fused_noalloc(void* out, const void* q, pa_dtype q_dtype,
                                   const void* k_cache, const void* v_cache, pa_dtype cache_dtype,
                                   const float* k_scale, const float* v_scale,
                                   const int32_t* block_tables, int max_blocks_per_seq,
                                   const int32_t* seq_lens, int num_seqs, int num_heads,
                                   int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                   float scale, int* err_flag, pa_stream_t stream);

/* Size of the fixed scratch array behind pa_decode_fused_noalloc (bytes). */
PA_API size_t pa_decode_fused_noalloc_scratch_bytes(void);

/* Bytes of tmp_out + max_logits + exp_sums for the given shape. */
PA_API size_t pa_decode_v2_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                           int max_num_partitions);

/*
 * A partition size for pa_decode_v2_partition: a multiple of
 * max(16, block_size) chosen so the number of CTAs fills every SM a few times
 * over, bounded so each CTA streams enough KV to amortise its start-up.
 */
PA_API int pa_choose_partition_size(int max_seq_len, int num_seqs, int num_kv_heads, int num_sms,
                                    int block_size);

/* KV bytes one token occupies over all layers: 2 * L * H_kv * D * dtype_bytes
 * ([vllm-musa] §一; [深度解析] §二; [KVcache-learning] s11). */
PA_API double pa_kv_bytes_per_token(int num_layers, int num_kv_heads, int head_dim,
                                    int dtype_bytes);

/* Human-readable name of a pa_status. */
PA_API const char* pa_status_string(int status);

/* The CUDA error behind the calling thread's most recent PA_ERR_CUDA
 * (cudaGetErrorString text; "no error" if there was none). */
PA_API const char* pa_last_cuda_error_string(void);

/*
 * Copy the library's device error word (OR of PA_DEVERR_* bits seen by any
 * kernel on the current device since the last clear) into *value and, if
 * clear != 0, reset it.  Synchronises the device.  Returns a pa_status.
 */
PA_API int pa_get_device_error(int* value, int clear);

/*
 * Tuning knobs of the decode kernels: warps per CTA (1..8) and pipeline stages
 * per warp (1..8); 0 restores the built-in choice.  Built in: 6 warps for a
 * 16-bit v1 CTA and 4 for a 16-bit v2 partition CTA, 8 for 8-bit caches; as
 * many stages as fit a 96 KB ring per CTA (64 KB for 16-bit partitions, so
 * three share an SM), at least 2.  Applies to later calls from any thread.
 */
PA_API int pa_set_decode_config(int warps_per_cta, int stages_per_warp);

/*
 * Tiles per decode warp prefetched into L2 before the PDL wait in mode 2
 * (0..32; 0 = none; -1 restores the default: 4 for 16-bit caches, 2 for 8-bit).
 */
PA_API int pa_set_prefetch_tiles(int tiles_per_warp);

/*
 * Time limit of each pipeline wait inside the decode kernels, in nanoseconds
 * (0 restores the default of 2 s).  A wait that runs out sets
 * PA_DEVERR_TIMEOUT, lets the copies still in flight land (bounded by 4 s),
 * and the warp contributes nothing further.  Tests use a tiny limit to
 * exercise that path without a real hang.
 */
PA_API int pa_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * Fault injection for failure-detection tests (0 = off, the default).  Mode 1:
 * in every decode warp the first pipeline stage is never armed, so the wait
 * on it can only end by running out its time limit (set one with
 * pa_set_wait_limit_ns first).  The kernel then reports PA_DEVERR_TIMEOUT and
 * returns normally; no GPU fault is involved.  Applies to later calls.
 */
PA_API int pa_set_fault_injection(int mode);

/*
 * Programmatic dependent launch (PDL) of the library's kernels.
 *   0: plain launches.
 *   1 (default): kernels are launched so they may start while the previous
 *      kernel in the stream finishes; each waits for that kernel to complete
 *      before reading or writing any tensor.  Same results as 0; the launch
 *      latency between kernels is hidden.
 *   2: as 1, but the decode kernels read seq_lens and block_tables (and derive
 *      their work split and block ids) BEFORE that wait, and ask L2 to fetch
 *      their first KV tiles (a prefetch: nothing is read into the kernel, and
 *      L2 stays coherent with the preceding kernel's writes).  q, the caches,
 *      the scales and every output are read or written only after the wait.
 *      Use only when seq_lens and block_tables are not written by the kernel
 *      that precedes the decode call in the stream (host copies are fine).
 * Applies to later calls from any thread.
 */
PA_API int pa_set_pdl(int mode);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
