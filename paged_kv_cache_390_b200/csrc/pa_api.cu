// pa_api.cu -- the C ABI of libpa.so (declared in include/pa.h): host-side
// argument checks, then one asynchronous launch on the caller's stream.
// No allocation, no synchronisation (except pa_get_device_error).
#include <atomic>
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdint>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace {

std::atomic<int> g_warps{0};
std::atomic<int> g_stages{0};
std::atomic<int> g_inject{0};
std::atomic<int> g_pdl{1};
std::atomic<int> g_prefetch{-1};
std::atomic<int> g_cascade_splits{0};     // 0: by the SM count
std::atomic<int> g_cascade_suffix{0};     // 0: persistent decode, 1: one CTA per (seq, kv head)
constexpr int kMaxCascadeSplits = 4;      // prefix splits of pa_decode_cascade (workspace bound)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // default: 2 s per mbarrier wait
std::atomic<unsigned long long> g_wait_limit{0};

unsigned long long wait_limit() {
  const unsigned long long v = g_wait_limit.load(std::memory_order_relaxed);
  return v ? v : kWaitLimitNs;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
bool is_float(int dt) { return dt == PA_F32 || dt == PA_F16 || dt == PA_BF16; }
bool is_quant(int dt) { return dt == PA_INT8 || dt == PA_FP8E4M3; }
int elem_bytes(int dt) { return dt == PA_F32 ? 4 : (dt == PA_F16 || dt == PA_BF16) ? 2 : 1; }
bool block_size_ok(int bs) { return bs == 8 || bs == 16 || bs == 32; }

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return PA_OK;
  t_last_cuda_error = e;
  return PA_ERR_CUDA;
}

// Checks shared by v1 and the v2 partition step.
int check_decode(const void* q, int q_dtype, const void* k_cache, const void* v_cache,
                 int cache_dtype, const float* k_scale, const float* v_scale,
                 const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                 int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                 int num_blocks, float scale) {
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks <= 0 || num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
  if (!block_size_ok(block_size)) return PA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (static_cast<long long>(num_blocks) * block_size > INT_MAX) return PA_ERR_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_heads / num_kv_heads > pa::kMaxGroup) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
  if (q_dtype < PA_F32 || q_dtype > PA_FP8E4M3 || cache_dtype < PA_F32 || cache_dtype > PA_FP8E4M3)
    return PA_ERR_INVALID_ARG;
  const bool pair_ok = (q_dtype == cache_dtype && is_float(q_dtype)) ||
                       ((q_dtype == PA_F16 || q_dtype == PA_BF16) && is_quant(cache_dtype));
  if (!pair_ok) return PA_ERR_UNSUPPORTED;
  if (is_quant(cache_dtype) && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4))
    return PA_ERR_INVALID_ARG;
  if (is_quant(cache_dtype) && (!aligned(k_scale, 16) || !aligned(v_scale, 16)))
    return PA_ERR_INVALID_ARG;
  return PA_OK;
}

pa::DecodeShape make_shape(int q_dtype, int cache_dtype, int head_dim, int block_size, int grid_x) {
  pa::DecodeShape sh;
  sh.q_dtype = q_dtype;
  sh.cache_dtype = cache_dtype;
  sh.head_dim = head_dim;
  sh.block_size = block_size;
  sh.grid_x = grid_x;
  const int w = g_warps.load(std::memory_order_relaxed);
  // 8-bit caches: 8 warps (their kernels are capped at 128 registers, so two such
  // CTAs fit an SM and more warps hide the per-tile dequantisation latency).
  // 16-bit split-K partitions: 4 warps, with a 64 KB stage ring, so three CTAs share
  // an SM and a starting CTA's first copies overlap two others' streams (the
  // 32K-context batch, P = 512, 4096 CTAs: 181.8 us a partition launch against 196.6
  // at 6 warps).
  if (w > 0) sh.warps = w;
  else if (is_quant(cache_dtype)) sh.warps = pa::kMaxWarps;
  else sh.warps = grid_x > 1 ? 4 : pa::kDefaultWarps;
  return sh;
}

int stages_for(const pa::DecodeShape& sh) {
  const int s = g_stages.load(std::memory_order_relaxed);
  const int budget_kb = !is_quant(sh.cache_dtype) && sh.grid_x > 1 ? 64 : 96;
  return s > 0 ? s
               : pa::default_stages(sh.cache_dtype, sh.head_dim, sh.block_size, sh.warps,
                                    budget_kb);
}

// L2 prefetch depth before the PDL wait, measured on the Qwen3-32B-shaped step:
// 16-bit caches 4 tiles per warp (2: 15.95 us, 4: 15.37 us, 6: 17.1 us, 8 or more:
// 18.0 us, the prefetch then competing with the preceding grid's own stream);
// 8-bit caches 2 (INT8 15.20 vs 15.49 us at 4, FP8 14.75 vs 15.07 us).
int prefetch_tiles(int cache_dtype) {
  const int p = g_prefetch.load(std::memory_order_relaxed);
  return p >= 0 ? p : (is_quant(cache_dtype) ? 2 : 4);
}

}  // namespace

namespace pa {
int pdl_mode() { return g_pdl.load(std::memory_order_relaxed); }
}  // namespace pa

extern "C" {

PA_API int pa_set_pdl(int mode) {
  if (mode < 0 || mode > 2) return PA_ERR_INVALID_ARG;
  g_pdl.store(mode, std::memory_order_relaxed);
  return PA_OK;
}

PA_API const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_NO_SPACE: return "PA_ERR_NO_SPACE";
  }
  return "PA_UNKNOWN_STATUS";
}

PA_API const char* pa_last_cuda_error_string(void) {
  return cudaGetErrorString(t_last_cuda_error);
}

PA_API double pa_kv_bytes_per_token(int num_layers, int num_kv_heads, int head_dim,
                                    int dtype_bytes) {
  return 2.0 * num_layers * num_kv_heads * head_dim * dtype_bytes;
}

PA_API size_t pa_decode_v2_workspace_bytes(int num_seqs, int num_heads, int head_dim,
                                           int max_num_partitions) {
  if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_num_partitions <= 0) return 0;
  return static_cast<size_t>(num_seqs) * num_heads * max_num_partitions * (head_dim + 2) *
         sizeof(float);
}

PA_API int pa_choose_partition_size(int max_seq_len, int num_seqs, int num_kv_heads, int num_sms,
                                    int block_size) {
  const int tt = block_size > 16 ? block_size : 16;
  const int min_tiles = 4 * pa::kDefaultWarps;        // >= 4 tiles per warp
  if (max_seq_len <= 0 || num_seqs <= 0 || num_kv_heads <= 0 || num_sms <= 0)
    return min_tiles * tt;
  const long long units = static_cast<long long>(num_seqs) * num_kv_heads;
  const long long target = 4LL * num_sms;              // CTAs wanted in flight overall
  long long parts = (target + units - 1) / units;
  if (parts < 1) parts = 1;
  const long long tiles = (max_seq_len + tt - 1) / tt;
  long long per = (tiles + parts - 1) / parts;
  if (per < min_tiles) per = min_tiles;
  per = (per + pa::kDefaultWarps - 1) / pa::kDefaultWarps * pa::kDefaultWarps;
  long long P = per * tt;
  if (P > (1LL << 20)) P = 1LL << 20;
  return static_cast<int>(P);
}

PA_API int pa_set_decode_config(int warps_per_cta, int stages_per_warp) {
  if (warps_per_cta < 0 || warps_per_cta > pa::kMaxWarps || stages_per_warp < 0 ||
      stages_per_warp > pa::kMaxStages)
    return PA_ERR_INVALID_ARG;
  g_warps.store(warps_per_cta, std::memory_order_relaxed);
  g_stages.store(stages_per_warp, std::memory_order_relaxed);
  return PA_OK;
}

PA_API int pa_set_prefetch_tiles(int tiles_per_warp) {
  if (tiles_per_warp < -1 || tiles_per_warp > 32) return PA_ERR_INVALID_ARG;
  g_prefetch.store(tiles_per_warp, std::memory_order_relaxed);
  return PA_OK;
}

PA_API int pa_set_fault_injection(int mode) {
  if (mode < 0 || mode > 1) return PA_ERR_INVALID_ARG;
  g_inject.store(mode, std::memory_order_relaxed);
  return PA_OK;
}

PA_API int pa_set_wait_limit_ns(unsigned long long limit_ns) {
  g_wait_limit.store(limit_ns, std::memory_order_relaxed);
  return PA_OK;
}

PA_API int pa_get_device_error(int* value, int clear) {
  if (!value) return PA_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return PA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_pa_device_error, sizeof(int)) != cudaSuccess)
    return PA_ERR_CUDA;
  *value = v;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(pa::g_pa_device_error, &zero, sizeof(int)) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  return PA_OK;
}

PA_API int pa_reshape_and_cache(const void* key, const void* value, pa_dtype src_dtype,
                                void* k_cache, void* v_cache, pa_dtype cache_dtype,
                                float* k_scale, float* v_scale, const int64_t* slot_mapping,
                                int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, int* err_flag, pa_stream_t stream) {
  if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PA_ERR_INVALID_ARG;
  if (!block_size_ok(block_size)) return PA_ERR_INVALID_ARG;
  if (!is_float(src_dtype) || cache_dtype < PA_F32 || cache_dtype > PA_FP8E4M3)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (!is_quant(cache_dtype) && cache_dtype != src_dtype) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  if (is_quant(cache_dtype) && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
  const uintptr_t row_align = is_quant(cache_dtype) ? static_cast<uintptr_t>(head_dim / 32) : 16;
  if (!aligned(key, 16) || !aligned(value, 16) || !aligned(k_cache, row_align) ||
      !aligned(v_cache, row_align) || !aligned(slot_mapping, 8))
    return PA_ERR_INVALID_ARG;
  if (is_quant(cache_dtype) && (!aligned(k_scale, 4) || !aligned(v_scale, 4)))
    return PA_ERR_INVALID_ARG;
  (void)elem_bytes;
  cudaError_t e = pa::launch_reshape_and_cache(
      key, value, src_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale, slot_mapping,
      num_tokens, num_kv_heads, head_dim, block_size, num_blocks, err_flag,
      reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

namespace {

// pa_decode_v1, with the fused write of each sequence's new token when new_k is
// not null (pa_append_decode_v1).
int decode_v1_impl(void* out, const void* q, int q_dtype, const void* k_cache,
                   const void* v_cache, int cache_dtype, const float* k_scale,
                   const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                   const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads,
                   int head_dim, int block_size, int num_blocks, float scale, int* err_flag,
                   const void* new_k, const void* new_v, const int64_t* new_slots,
                   cudaStream_t stream, int t_offset = 0, const float* prior = nullptr,
                   int pdl_override = -1, int prior_splits = 1, size_t prior_rows = 0) {
  pa::DecodeShape sh = make_shape(q_dtype, cache_dtype, head_dim, block_size, 1);
  pa::DecodeArgs a{};
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.err_flag = err_flag;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.partition_size = 0;
  a.max_parts = 1;
  a.stages = stages_for(sh);
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = wait_limit();
  a.inject = g_inject.load(std::memory_order_relaxed);
  a.pdl = g_pdl.load(std::memory_order_relaxed);
  a.prefetch = prefetch_tiles(cache_dtype);
  a.new_k = new_k;
  a.new_v = new_v;
  a.new_slots = new_slots;
  a.wk_cache = const_cast<void*>(k_cache);
  a.wv_cache = const_cast<void*>(v_cache);
  a.wk_scale = const_cast<float*>(k_scale);
  a.wv_scale = const_cast<float*>(v_scale);
  a.t_offset = t_offset;
  if (prior) {          // [slots][S,H,D] o, then [slots][S,H] m, then [slots][S,H] l
    a.prior_splits = prior_splits;
    a.prior_o = prior;
    a.prior_m = prior + prior_rows * head_dim;
    a.prior_l = a.prior_m + prior_rows;
  }
  if (pdl_override >= 0) a.pdl = pdl_override;
  return cuda_status(pa::launch_decode(a, sh, stream));
}

int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 148;
  return sms;
}

// Cascade workspace: the stacked partials (prefix splits + the suffix's), then the
// persistent suffix decode's workspace (arrival counters + records), then its CTA
// exit counter.
size_t cascade_partials_bytes(int num_seqs, int num_heads, int head_dim) {
  const size_t b = static_cast<size_t>(kMaxCascadeSplits + 1) * num_seqs * num_heads *
                   (head_dim + 2) * sizeof(float);
  return (b + 255) / 256 * 256;
}

size_t cascade_workspace_bytes(int num_seqs, int num_heads, int head_dim) {
  return cascade_partials_bytes(num_seqs, num_heads, head_dim) +
         pa::fused_workspace_bytes(num_seqs, num_heads, head_dim, device_sms()) + 256;
}

}  // namespace

PA_API int pa_decode_v1(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                        const void* v_cache, pa_dtype cache_dtype, const float* k_scale,
                        const float* v_scale, const int32_t* block_tables,
                        int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                        int num_heads, int num_kv_heads, int head_dim, int block_size,
                        int num_blocks, float scale, int* err_flag, pa_stream_t stream) {
  int rc = check_decode(q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables,
                        max_blocks_per_seq, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (!out || !aligned(out, 16)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  return decode_v1_impl(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                        block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag, nullptr,
                        nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

PA_API int pa_append_decode_v1(void* out, const void* q, pa_dtype q_dtype, const void* key,
                               const void* value, const int64_t* slot_mapping, void* k_cache,
                               void* v_cache, pa_dtype cache_dtype, float* k_scale,
                               float* v_scale, const int32_t* block_tables,
                               int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                               int num_heads, int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, float scale, int* err_flag, pa_stream_t stream) {
  int rc = check_decode(q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables,
                        max_blocks_per_seq, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (!out || !aligned(out, 16)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  if (!key || !value || !slot_mapping || !aligned(key, 16) || !aligned(value, 16) ||
      !aligned(slot_mapping, 8))
    return PA_ERR_INVALID_ARG;
  const uintptr_t row_align = is_quant(cache_dtype) ? static_cast<uintptr_t>(head_dim / 32) : 16;
  if (!aligned(k_cache, row_align) || !aligned(v_cache, row_align)) return PA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cache_dtype == PA_F32) {
    // the fp32 kernel has no fused write: the cache write runs first, then the decode
    cudaError_t e = pa::launch_reshape_and_cache(key, value, q_dtype, k_cache, v_cache, cache_dtype,
                                                 k_scale, v_scale, slot_mapping, num_seqs,
                                                 num_kv_heads, head_dim, block_size, num_blocks,
                                                 err_flag, s);
    if (e != cudaSuccess) return cuda_status(e);
    return decode_v1_impl(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                          block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                          num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag, nullptr,
                          nullptr, nullptr, s);
  }
  return decode_v1_impl(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                        block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag, key, value,
                        slot_mapping, s);
}

PA_API int pa_decode_v2_partition(float* tmp_out, float* max_logits, float* exp_sums,
                                  const void* q, pa_dtype q_dtype, const void* k_cache,
                                  const void* v_cache, pa_dtype cache_dtype,
                                  const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int max_blocks_per_seq,
                                  const int32_t* seq_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                  float scale, int partition_size, int max_num_partitions,
                                  int* err_flag, pa_stream_t stream) {
  int rc = check_decode(q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables,
                        max_blocks_per_seq, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (!tmp_out || !max_logits || !exp_sums || !aligned(tmp_out, 16)) return PA_ERR_INVALID_ARG;
  const int tt = block_size > 16 ? block_size : 16;
  if (partition_size <= 0 || partition_size % tt != 0 || max_num_partitions <= 0)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  pa::DecodeShape sh = make_shape(q_dtype, cache_dtype, head_dim, block_size, max_num_partitions);
  pa::DecodeArgs a{};
  a.tmp_out = tmp_out;
  a.max_logits = max_logits;
  a.exp_sums = exp_sums;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.err_flag = err_flag;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.partition_size = partition_size;
  a.max_parts = max_num_partitions;
  a.stages = stages_for(sh);
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = wait_limit();
  a.inject = g_inject.load(std::memory_order_relaxed);
  a.pdl = g_pdl.load(std::memory_order_relaxed);
  a.prefetch = prefetch_tiles(cache_dtype);
  cudaError_t e = pa::launch_decode(a, sh, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

PA_API size_t pa_decode_fused_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim,
                                              int num_sms) {
  if (num_seqs <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_sms <= 0) return 0;
  return pa::fused_workspace_bytes(num_seqs, num_kv_heads, head_dim, num_sms);
}

}  // extern "C"

namespace pa {
// Host checks of pa_decode_fused up to (not including) its workspace.
int fused_host_checks(void* out, const void* q, int q_dtype, const void* k_cache,
                      const void* v_cache, int cache_dtype, const float* k_scale,
                      const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, float scale) {
  int rc = check_decode(q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale, block_tables,
                        max_blocks_per_seq, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (!out || !aligned(out, 16)) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || cache_dtype == PA_F32) return PA_OK;
  if (num_seqs > kFusedMaxSeqs) return PA_ERR_UNSUPPORTED;
  const long long max_tiles = static_cast<long long>(num_seqs) * num_kv_heads *
                              ((static_cast<long long>(max_blocks_per_seq) * block_size + 15) / 16);
  if (max_tiles >= INT_MAX) return PA_ERR_UNSUPPORTED;
  return PA_OK;
}
}  // namespace pa

extern "C" {

PA_API int pa_decode_fused(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                           const void* v_cache, pa_dtype cache_dtype, const float* k_scale,
                           const float* v_scale, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, float scale, void* workspace, size_t workspace_bytes,
                           int* err_flag, pa_stream_t stream) {
  int rc = pa::fused_host_checks(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                                 block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                                 num_kv_heads, head_dim, block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (num_seqs == 0) return PA_OK;
  if (cache_dtype == PA_F32)             // fp32 caches take the CUDA-core kernel (no workspace)
    return pa_decode_v1(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                        block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                        num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag, stream);
  if (!workspace || !aligned(workspace, 256)) return PA_ERR_INVALID_ARG;
  pa::FusedArgs a{};
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.err_flag = err_flag;
  a.counters = static_cast<int*>(workspace);
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  const int s = g_stages.load(std::memory_order_relaxed);
  a.stages = s > 0 ? s : 2;
  a.prefetch = prefetch_tiles(cache_dtype);
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = wait_limit();
  a.inject = g_inject.load(std::memory_order_relaxed);
  a.pdl = g_pdl.load(std::memory_order_relaxed);
  cudaError_t e = pa::launch_fused(a, q_dtype, cache_dtype, head_dim, block_size, workspace_bytes,
                                   reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue) return PA_ERR_INVALID_ARG;   // workspace too small
  return cuda_status(e);
}

PA_API int pa_decode_v2_merge(void* out, pa_dtype out_dtype, const float* tmp_out,
                              const float* max_logits, const float* exp_sums,
                              const int32_t* seq_lens, int num_seqs, int num_heads, int head_dim,
                              int partition_size, int max_num_partitions, pa_stream_t stream) {
  if (!out || !tmp_out || !max_logits || !exp_sums || !seq_lens) return PA_ERR_INVALID_ARG;
  if (!is_float(out_dtype)) return PA_ERR_INVALID_ARG;
  if (num_seqs < 0 || num_heads <= 0 || partition_size <= 0 || max_num_partitions <= 0)
    return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  cudaError_t e = pa::launch_merge(out, out_dtype, tmp_out, max_logits, exp_sums, seq_lens,
                                   num_seqs, num_heads, head_dim, partition_size,
                                   max_num_partitions, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

PA_API int pa_copy_blocks(const void* src_k_cache, const void* src_v_cache,
                          const float* src_k_scale, const float* src_v_scale, int src_num_blocks,
                          void* dst_k_cache, void* dst_v_cache, float* dst_k_scale,
                          float* dst_v_scale, int dst_num_blocks, pa_dtype cache_dtype,
                          const int64_t* block_mapping, int num_pairs, int num_kv_heads,
                          int head_dim, int block_size, int* err_flag, pa_stream_t stream) {
  if (num_pairs < 0 || num_kv_heads <= 0 || src_num_blocks <= 0 || dst_num_blocks <= 0)
    return PA_ERR_INVALID_ARG;
  if (!block_size_ok(block_size)) return PA_ERR_INVALID_ARG;
  if (cache_dtype < PA_F32 || cache_dtype > PA_FP8E4M3) return PA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_pairs == 0) return PA_OK;
  if (!src_k_cache || !src_v_cache || !dst_k_cache || !dst_v_cache || !block_mapping)
    return PA_ERR_INVALID_ARG;
  const bool quant = is_quant(cache_dtype);
  if (quant && (!src_k_scale || !src_v_scale || !dst_k_scale || !dst_v_scale))
    return PA_ERR_INVALID_ARG;
  if (!aligned(src_k_cache, 16) || !aligned(src_v_cache, 16) || !aligned(dst_k_cache, 16) ||
      !aligned(dst_v_cache, 16) || !aligned(block_mapping, 8))
    return PA_ERR_INVALID_ARG;
  if (quant && (!aligned(src_k_scale, 16) || !aligned(src_v_scale, 16) ||
                !aligned(dst_k_scale, 16) || !aligned(dst_v_scale, 16)))
    return PA_ERR_INVALID_ARG;
  pa::CopyArgs a{};
  a.src_k = src_k_cache;
  a.src_v = src_v_cache;
  a.dst_k = dst_k_cache;
  a.dst_v = dst_v_cache;
  a.src_ks = quant ? src_k_scale : nullptr;
  a.src_vs = quant ? src_v_scale : nullptr;
  a.dst_ks = quant ? dst_k_scale : nullptr;
  a.dst_vs = quant ? dst_v_scale : nullptr;
  a.block_mapping = block_mapping;
  a.err_flag = err_flag;
  // block bytes = block_size * num_kv_heads * head_dim * elem: a multiple of 16
  // for head_dim 64 / 128; scale bytes = num_kv_heads * block_size * 4: also
  a.block_vecs = static_cast<int64_t>(block_size) * num_kv_heads * head_dim *
                 elem_bytes(cache_dtype) / 16;
  a.scale_vecs = quant ? num_kv_heads * block_size / 4 : 0;
  a.src_num_blocks = src_num_blocks;
  a.dst_num_blocks = dst_num_blocks;
  if (pa::copy_slices_per_pair(a.block_vecs, a.scale_vecs) > 65535) return PA_ERR_UNSUPPORTED;
  cudaError_t e = pa::launch_copy_blocks(a, num_pairs, reinterpret_cast<cudaStream_t>(stream));
  return cuda_status(e);
}

PA_API int pa_prefill(void* out, const void* q, pa_dtype q_dtype, const int32_t* query_start,
                      int total_q, int max_query_len, const void* k_cache, const void* v_cache,
                      pa_dtype cache_dtype, const int32_t* block_tables, int max_blocks_per_seq,
                      const int32_t* seq_lens, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int num_blocks, float scale, int* err_flag,
                      pa_stream_t stream) {
  if (!out || !q || !query_start || !k_cache || !v_cache || !block_tables || !seq_lens)
    return PA_ERR_INVALID_ARG;
  if (num_seqs < 0 || total_q < 0 || max_query_len < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0 || num_heads % num_kv_heads != 0)
    return PA_ERR_INVALID_ARG;
  if (!block_size_ok(block_size) || !std::isfinite(scale)) return PA_ERR_INVALID_ARG;
  if (q_dtype != cache_dtype || (q_dtype != PA_F16 && q_dtype != PA_BF16)) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128) return PA_ERR_UNSUPPORTED;
  const int G = num_heads / num_kv_heads;
  if (128 % G != 0) return PA_ERR_UNSUPPORTED;
  if (num_seqs > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
  if (static_cast<long long>(num_blocks) * block_size > INT_MAX) return PA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || total_q == 0 || max_query_len == 0) return PA_OK;
  pa::PrefillArgs a{};
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.query_start = query_start;
  a.err_flag = err_flag;
  a.max_blocks = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_blocks = num_blocks;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.timeout_ns = wait_limit();
  a.inject = g_inject.load(std::memory_order_relaxed);
  return cuda_status(pa::launch_prefill(a, q_dtype, block_size, total_q, max_query_len,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

PA_API size_t pa_decode_cascade_workspace_bytes(int num_seqs, int num_heads, int head_dim) {
  if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0) return 0;
  return cascade_workspace_bytes(num_seqs, num_heads, head_dim);
}

PA_API int pa_decode_cascade(void* out, const void* q, pa_dtype q_dtype, const void* k_cache,
                             const void* v_cache, pa_dtype cache_dtype,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* seq_lens, int num_seqs, int num_heads,
                             int num_kv_heads, int head_dim, int block_size, int num_blocks,
                             float scale, int prefix_len, void* workspace,
                             size_t workspace_bytes, int* err_flag, pa_stream_t stream) {
  int rc = check_decode(q, q_dtype, k_cache, v_cache, cache_dtype, nullptr, nullptr, block_tables,
                        max_blocks_per_seq, seq_lens, num_seqs, num_heads, num_kv_heads, head_dim,
                        block_size, num_blocks, scale);
  if (rc != PA_OK) return rc;
  if (!out || !aligned(out, 16)) return PA_ERR_INVALID_ARG;
  if (q_dtype != cache_dtype || (q_dtype != PA_F16 && q_dtype != PA_BF16)) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128 || 128 % (num_heads / num_kv_heads) != 0) return PA_ERR_UNSUPPORTED;
  if (prefix_len < 0 || prefix_len % block_size != 0 ||
      static_cast<long long>(prefix_len) > static_cast<long long>(max_blocks_per_seq) * block_size)
    return PA_ERR_INVALID_ARG;
  if (num_seqs == 0) return PA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (prefix_len == 0)
    return decode_v1_impl(out, q, q_dtype, k_cache, v_cache, cache_dtype, nullptr, nullptr,
                          block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                          num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag, nullptr,
                          nullptr, nullptr, s);
  if (!workspace || !aligned(workspace, 256) ||
      workspace_bytes < cascade_workspace_bytes(num_seqs, num_heads, head_dim))
    return PA_ERR_INVALID_ARG;
  if (num_seqs > pa::kFusedMaxSeqs) return PA_ERR_UNSUPPORTED;
  float* ws = static_cast<float*>(workspace);
  const size_t sh_rows = static_cast<size_t>(num_seqs) * num_heads;
  pa::PrefillArgs pf{};
  pf.q = q;
  pf.k_cache = k_cache;
  pf.v_cache = v_cache;
  pf.block_tables = block_tables;            // row 0 holds the shared prefix's blocks
  pf.seq_lens = seq_lens;
  pf.err_flag = err_flag;
  pf.max_blocks = max_blocks_per_seq;
  pf.num_seqs = 1;
  pf.num_heads = num_heads;
  pf.num_kv_heads = num_kv_heads;
  pf.num_blocks = num_blocks;
  pf.scale_log2 = scale * 1.4426950408889634f;
  pf.timeout_ns = wait_limit();
  pf.inject = g_inject.load(std::memory_order_relaxed);
  pf.cascade_rows = num_seqs;
  pf.cascade_len = prefix_len;
  // split the prefix over enough CTAs to fill the GPU: each CTA takes 256 query
  // rows (two tiles) of one kv head; keep >= 256 prefix tokens (two KV tiles)
  // per split
  const int G = num_heads / num_kv_heads;
  const long long ctas = static_cast<long long>((num_seqs * G + 255) / 256) * num_kv_heads;
  // Two ways to place the launches.  Side by side: the prefix split over at most
  // half the SMs, one CTA per SM, and the suffix's persistent grid on all the
  // others, both running at once.  Or the prefix split to fill the GPU, then the
  // suffix on every SM.  When both give the prefix the same split count, side by side
  // loses nothing and is taken.  Otherwise it pays only when the suffix on the
  // remaining SMs lasts about as long as the less split prefix, and the host cannot
  // see the sequences' own lengths: the automatic choice then takes it when the
  // prefix CTAs fill at least a third of the SMs and the table width leaves room for
  // own tokens of at least half the prefix (256 sequences after an 8192-token
  // prefix: 231 vs 277 us a step; 192: 230 vs 213, the split form winning).  Split
  // count -1 asks for side by side whenever PDL is on and it fits.
  int splits = g_cascade_splits.load(std::memory_order_relaxed);
  const int pdl_on = g_pdl.load(std::memory_order_relaxed) != 0;
  const int sms = device_sms();
  const int cap = std::max(1, std::min(kMaxCascadeSplits, prefix_len / 256));
  const int s_fill = std::max(1, std::min(cap, static_cast<int>(sms / std::max(1LL, ctas))));
  const int s_side = ctas <= sms / 2 ? std::max(1, std::min(cap, static_cast<int>((sms / 2) / ctas))) : 0;
  const long long own_room = static_cast<long long>(max_blocks_per_seq) * block_size - prefix_len;
  bool beside = false;
  if (pdl_on && s_side > 0) {
    if (splits == -1)
      beside = true;
    else if (splits == 0)
      beside = s_side == s_fill ||
               (ctas * s_side * 3 >= sms && own_room * 2 >= prefix_len);
  }
  if (beside) splits = s_side;
  else if (splits <= 0) splits = s_fill;
  splits = std::max(1, std::min(splits, cap));
  pf.cascade_splits = splits;
  pf.part_o = ws;
  pf.part_m = ws + (kMaxCascadeSplits + 1) * sh_rows * head_dim;
  pf.part_l = pf.part_m + (kMaxCascadeSplits + 1) * sh_rows;
  // beside the suffix, the prefix's CTAs must take distinct SMs spread over the
  // GPU, which a launch on an idle GPU gives and an early (PDL) launch does not:
  // measured on the mixed batch, the early launch cost ~20 us a step
  cudaError_t e = pa::launch_prefill(pf, q_dtype, block_size, num_seqs, num_seqs, s, !beside);
  if (e != cudaSuccess) return cuda_status(e);
  if (g_cascade_suffix.load(std::memory_order_relaxed) == 1) {
    // each sequence's own tokens on one CTA per (sequence, kv head), merging the
    // prefix partials in its epilogue (it waits for the prefix only there)
    return decode_v1_impl(out, q, q_dtype, k_cache, v_cache, cache_dtype, nullptr, nullptr,
                          block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                          num_kv_heads, head_dim, block_size, num_blocks, scale, err_flag,
                          nullptr, nullptr, nullptr, s, prefix_len, ws, pdl_on ? 3 : 0, splits,
                          (kMaxCascadeSplits + 1) * sh_rows);
  }
  // each sequence's own tokens [prefix_len, len) on the persistent decode (every
  // warp an equal share), which leaves one more partial; it never waits for the
  // prefix (it reads nothing the prefix writes), only its last CTA does
  char* wsb = static_cast<char*>(workspace);
  const size_t pbytes = cascade_partials_bytes(num_seqs, num_heads, head_dim);
  const size_t fbytes = pa::fused_workspace_bytes(num_seqs, num_heads, head_dim, device_sms());
  pa::FusedArgs fa{};
  fa.q = q;
  fa.k_cache = k_cache;
  fa.v_cache = v_cache;
  fa.block_tables = block_tables;
  fa.seq_lens = seq_lens;
  fa.err_flag = err_flag;
  fa.counters = reinterpret_cast<int*>(wsb + pbytes);
  fa.max_blocks = max_blocks_per_seq;
  fa.num_seqs = num_seqs;
  fa.num_heads = num_heads;
  fa.num_kv_heads = num_kv_heads;
  fa.num_blocks = num_blocks;
  const int st = g_stages.load(std::memory_order_relaxed);
  fa.stages = st > 0 ? st : 2;
  fa.prefetch = prefetch_tiles(cache_dtype);
  fa.scale_log2 = scale * 1.4426950408889634f;
  fa.timeout_ns = wait_limit();
  fa.inject = g_inject.load(std::memory_order_relaxed);
  fa.pdl = pdl_on ? 3 : 0;
  fa.t_offset = prefix_len;
  fa.part_o = pf.part_o + static_cast<size_t>(splits) * sh_rows * head_dim;
  fa.part_m = pf.part_m + static_cast<size_t>(splits) * sh_rows;
  fa.part_l = pf.part_l + static_cast<size_t>(splits) * sh_rows;
  fa.done = reinterpret_cast<int*>(wsb + pbytes + fbytes);
  // beside the prefix launch: a grid for the SMs it leaves free (its CTAs take a whole
  // SM each), so that no share of the suffix waits for the prefix to finish
  fa.sm_limit = beside ? sms - static_cast<int>(ctas) * splits : 0;
  // on part of the GPU the suffix is bound by warps per SM: three CTAs per SM
  fa.ctas_per_sm = fa.sm_limit > 0 ? 3 : 0;
  e = pa::launch_fused(fa, q_dtype, cache_dtype, head_dim, block_size, fbytes, s);
  if (e != cudaSuccess) return cuda_status(e);
  e = pa::launch_merge_partials(out, q_dtype, pf.part_o, pf.part_m, pf.part_l, splits + 1,
                                static_cast<long long>(sh_rows), head_dim, s);
  return cuda_status(e);
}

PA_API int pa_set_cascade_config(int prefix_splits, int suffix_form) {
  if (prefix_splits < -1 || prefix_splits > kMaxCascadeSplits || suffix_form < 0 || suffix_form > 1)
    return PA_ERR_INVALID_ARG;
  g_cascade_splits.store(prefix_splits, std::memory_order_relaxed);
  g_cascade_suffix.store(suffix_form, std::memory_order_relaxed);
  return PA_OK;
}

}  // extern "C"
