// pa_internal.h -- host-side interface between the C ABI (pa_api.cu) and the
// kernel translation units.  Not installed; not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Host checks of pa_decode_fused that do not involve its workspace (pa_api.cu);
// PA_OK or the status pa_decode_fused would return for these arguments.
int fused_host_checks(void* out, const void* q, int q_dtype, const void* k_cache,
                      const void* v_cache, int cache_dtype, const float* k_scale,
                      const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, float scale);

constexpr int kMaxWarps = 8;
constexpr int kDefaultWarps = 6;
constexpr int kMaxStages = 8;
constexpr int kMaxGroup = 8;            // query heads per kv head

struct DecodeArgs {
  void* out;                  // v1: [S, H, D] in q dtype
  float* tmp_out;             // v2: [S, H, maxp, D]
  float* max_logits;          // v2: [S, H, maxp]
  float* exp_sums;            // v2: [S, H, maxp]
  const void* q;              // [S, H, D]
  const void* k_cache;        // [nb, bs, Hkv, D]   (fp32 kernel only; the TC kernel uses TMA)
  const void* v_cache;
  const float* k_scale;       // [nb, Hkv, bs]
  const float* v_scale;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int* err_flag;
  int max_blocks;
  int num_seqs, num_heads, num_kv_heads, num_blocks;
  int partition_size;         // 0: one CTA per (seq, kv head), write `out`
  int max_parts;
  int stages;                 // pipeline stages per warp
  float scale;                // softmax scale
  float scale_log2;           // scale * log2(e)
  unsigned long long timeout_ns;
  int inject;                 // fault injection for tests: 1 = each warp's first tile
                              // never arrives (its bounded wait runs out)
  int pdl;                    // 0 plain launch; 1 PDL, wait first; 2 PDL, read
                              // seq_lens / block_tables before the wait
  int prefetch;               // PDL mode 2: tiles per warp fetched into L2 before the wait
  // Fused cache write of each sequence's new token (null new_k: none).  The warp
  // that owns the sequence's last tile writes the token's K and V rows to slot
  // new_slots[s] before it loads that tile.
  const void* new_k;          // [S, Hkv, D] in q dtype
  const void* new_v;
  const int64_t* new_slots;   // [S]
  void* wk_cache;             // the caches and scales, writable
  void* wv_cache;
  float* wk_scale;
  float* wv_scale;
  // Cascade decode: the v1 pass covers tokens [t_offset, seq_len) and merges a
  // prior partial (o / l, m in the log2 domain, l) per (sequence, head) before
  // writing `out`.  PDL mode 3 waits for the preceding grid only there.
  int t_offset;
  int prior_splits;           // number of prior partials, stacked [split][...]
  const float* prior_o;       // [splits, S, H, D] or null
  const float* prior_m;       // [splits, S, H]
  const float* prior_l;       // [splits, S, H]
};

// Current PDL mode (see pa_set_pdl).
int pdl_mode();

struct DecodeShape {
  int q_dtype, cache_dtype, head_dim, block_size;
  int grid_x;                 // partitions (1 for v1)
  int warps;                  // warps per CTA
};

// Launch the decode kernel for `shape`; returns cudaSuccess or the launch error.
cudaError_t launch_decode(const DecodeArgs& a, const DecodeShape& shape, cudaStream_t stream);

cudaError_t launch_merge(void* out, int out_dtype, const float* tmp_out, const float* max_logits,
                         const float* exp_sums, const int32_t* seq_lens, int num_seqs,
                         int num_heads, int head_dim, int partition_size, int max_parts,
                         cudaStream_t stream);

// Merge `nparts` stacked partials [k][rows][D] (o / l), [k][rows] m (log2 units)
// and l into out [rows][D] (f16 or bf16).
cudaError_t launch_merge_partials(void* out, int out_dtype, const float* part_o,
                                  const float* part_m, const float* part_l, int nparts,
                                  long long rows, int head_dim, cudaStream_t stream);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, int src_dtype,
                                     void* k_cache, void* v_cache, int cache_dtype,
                                     float* k_scale, float* v_scale,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int* err_flag, cudaStream_t stream);

// Persistent single-launch decode (pa_decode_fused): every warp streams an
// equal contiguous range of the batch's 16-token tiles; a (sequence, kv head)
// split between warps is merged by the warp that finishes it last.
constexpr int kFusedWarps = 4;            // warps per CTA
constexpr int kFusedMaxCtasPerSm = 4;     // workspace is sized for this many
constexpr int kFusedMaxSeqs = 8192;       // per-CTA prefix table lives in shared memory

struct FusedArgs {
  void* out;                  // [S, H, D] in q dtype
  const void* q;
  const void* k_cache;        // host side only (tensor maps)
  const void* v_cache;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int* err_flag;
  float* partials;            // [2 * total warps][rec]: o[8][D], m[8], l[8], padding
  int* counters;              // [S * H_kv], zero on entry, left zero
  int max_blocks;
  int num_seqs, num_heads, num_kv_heads, num_blocks;
  int stages;
  float scale_log2;
  unsigned long long timeout_ns;
  int inject;
  int pdl;                      // as DecodeArgs::pdl; 3: never wait for the preceding grid
                                // (it writes nothing read here), the last CTA to finish
                                // waits for it, so this grid ends after it
  int prefetch;                 // PDL mode 2: tiles per warp fetched into L2 before the wait
  // Cascade suffix: each sequence's tokens [t_offset, seq_len) only, and with
  // part_o set, (o / l, m, l) partials instead of `out`: part_o [S, H, D],
  // part_m [S, H] (log2 units of scale * q.k), part_l [S, H]; a sequence with no
  // such token gets o = 0, m = -inf, l = 0.
  int t_offset;
  float* part_o;
  float* part_m;
  float* part_l;
  int* done;                    // PDL mode 3: CTA exit counter, zero on entry, left zero
  int sm_limit;                 // > 0: a grid for this many SMs only (the others are busy
                                // with a launch this one runs beside); 0: every SM
  int ctas_per_sm;              // 3 (16-bit cache, head_dim 128): the build capped at 168
                                // registers, three CTAs per SM; other > 0: at most this
                                // many CTAs per SM; 0: as many as fit
};

// Floats of one partial record (padded to whole 128-byte lines).
inline int fused_record_floats(int head_dim) { return 8 * head_dim + 32; }
size_t fused_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int num_sms);

cudaError_t launch_fused(const FusedArgs& a, int q_dtype, int cache_dtype, int head_dim,
                         int block_size, size_t workspace_bytes, cudaStream_t stream);

// Default stages per warp for a cache dtype / shape: as many as fit `budget_kb` of
// stage ring per CTA (2 to kMaxStages); 96 KB lets two CTAs share an SM, 64 KB three.
int default_stages(int cache_dtype, int head_dim, int block_size, int warps, int budget_kb);

// Block copy (pa_copy_blocks): copy-on-write within one pool, or swap between
// the device pool and a pool in mapped pinned host memory.
struct CopyArgs {
  const void* src_k;
  const void* src_v;
  const float* src_ks;
  const float* src_vs;
  void* dst_k;
  void* dst_v;
  float* dst_ks;
  float* dst_vs;
  const int64_t* block_mapping;   // [num_pairs, 2] = (src id, dst id)
  int* err_flag;
  int64_t block_vecs;             // 16-byte vectors per K (or V) block
  int scale_vecs;                 // 16-byte vectors per block of scales (0: no scales)
  int src_num_blocks;
  int dst_num_blocks;
};

int copy_slices_per_pair(int64_t block_vecs, int scale_vecs);
cudaError_t launch_copy_blocks(const CopyArgs& a, int num_pairs, cudaStream_t stream);

// Multi-token query over the paged cache (pa_prefill), tcgen05 kernel.
struct PrefillArgs {
  void* out;                  // [total_q, H, D] in q dtype
  const void* q;              // [total_q, H, D]
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const int32_t* query_start; // [num_seqs + 1]
  int* err_flag;
  int max_blocks;
  int num_seqs, num_heads, num_kv_heads, num_blocks;
  float scale_log2;
  unsigned long long timeout_ns;
  int inject;
  // Shared-prefix mode (cascade decode): one pseudo-sequence whose cascade_rows
  // query rows (every sequence's decode query) all attend to the first
  // cascade_len tokens of block_tables row 0, with no causal mask, and leave
  // (o / l, m, l) partials instead of `out`.
  int cascade_rows;           // 0: the prefill proper
  int cascade_len;
  int cascade_splits;         // the prefix's KV tiles split over this many CTAs (grid z)
  float* part_o;              // [rows, H, D]
  float* part_m;              // [rows, H], log2 domain (scale folded in)
  float* part_l;              // [rows, H]
};

// allow_pdl = false launches without the programmatic-dependent-launch attribute
// even when it is on: the CTAs are placed on an idle GPU instead of on whichever
// SMs the preceding launch frees first.
cudaError_t launch_prefill(const PrefillArgs& a, int q_dtype, int block_size, int total_q,
                           int max_query_len, cudaStream_t stream, bool allow_pdl = true);

}  // namespace pa
