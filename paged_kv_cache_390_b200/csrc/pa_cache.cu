// pa_cache.cu -- the paged KV-cache write (reshape_and_cache) for sm_100a.
//
// Each new token's K and V rows go to slot = block * block_size + offset of the
// cache [num_blocks, block_size, num_kv_heads, head_dim]: the append step of a
// block manager ("大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置",
// BlockManager.append_token; "KVcache-learning" s06).  With an INT8 or FP8 E4M3
// cache each (token, head) row is quantised symmetrically with its own fp32
// scale ("KVcache-learning" s09: E4M3, range +-448; kv_cache_dtype int8 on the
// yunthe.com page): s = max|x| / 127 (or / 448), code = rne(x / s), every
// division IEEE fp32 round-to-nearest, FP8 saturating to +-448.
//
// Plain caches: each warp moves kRowsPerWarp (token, kv head) rows, loading the
// K and V rows of all of them (16-byte vectors, the K row and the V row side by
// side across the lanes) before it stores any, so enough bytes are in flight to
// stream at HBM rate.  Quantised caches: one warp per (token, kv head) loads the
// K and V rows (one vector per lane each), then quantises them with pa_write.cuh:
// a warp-shuffle max and per-lane IEEE-fp32 encodes.
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"
#include "pa_write.cuh"

namespace pa {
namespace {

enum { kCopy = kWriteCopy, kInt8 = kWriteInt8, kFp8 = kWriteFp8 };

constexpr int kRowsPerWarp = 4;

template <typename ST, int D>
__global__ void __launch_bounds__(128)
    cache_copy_kernel(const ST* __restrict__ key, const ST* __restrict__ value,
                      ST* __restrict__ k_cache, ST* __restrict__ v_cache,
                      const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads,
                      int block_size, int num_blocks, int* err_flag) {
  constexpr int NV = D * static_cast<int>(sizeof(ST)) / 16;   // 16-byte vectors per row
  constexpr int VPL = (2 * NV + 31) / 32;                       // per lane: K and V side by side
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const long long w = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long nrows = static_cast<long long>(num_tokens) * num_kv_heads;
  uint4 buf[kRowsPerWarp][VPL];
  long long dst_row[kRowsPerWarp];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const long long row = w * kRowsPerWarp + r;
    dst_row[r] = -1;
    if (row >= nrows) continue;
    const int token = static_cast<int>(row / num_kv_heads);
    const int head = static_cast<int>(row % num_kv_heads);
    const int64_t slot = slots[token];
    if (slot < 0) continue;                                    // no write for this token
    if (slot >= static_cast<int64_t>(num_blocks) * block_size) {   // past the pool: skipped
      if (err_flag && lane == 0) report_error(err_flag, kErrSlot);
      continue;
    }
    dst_row[r] = (slot * num_kv_heads + head) * static_cast<long long>(D);
    const size_t src_row = static_cast<size_t>(row) * D;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int idx = lane + 32 * v;                           // [0, NV): K, [NV, 2 NV): V
      if (idx < 2 * NV)
        buf[r][v] = __ldg(reinterpret_cast<const uint4*>((idx < NV ? key : value) + src_row) +
                          (idx % NV));
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    if (dst_row[r] < 0) continue;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const int idx = lane + 32 * v;
      if (idx < 2 * NV)
        reinterpret_cast<uint4*>((idx < NV ? k_cache : v_cache) + dst_row[r])[idx % NV] = buf[r][v];
    }
  }
}

template <typename ST, int MODE, int D>
__global__ void __launch_bounds__(128)
    cache_kernel(const ST* __restrict__ key, const ST* __restrict__ value, void* k_cache,
                 void* v_cache, float* k_scale, float* v_scale,
                 const int64_t* __restrict__ slots, int num_tokens, int num_kv_heads,
                 int block_size, int num_blocks, int* err_flag) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const long long gw = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int token = static_cast<int>(gw / num_kv_heads);
  const int head = static_cast<int>(gw % num_kv_heads);
  if (token >= num_tokens) return;
  const int64_t slot = slots[token];
  if (slot < 0) return;                                      // no write for this token
  if (slot >= static_cast<int64_t>(num_blocks) * block_size) {   // past the pool: skipped
    if (err_flag && lane == 0) report_error(err_flag, kErrSlot);
    return;
  }
  const int64_t blk = slot / block_size;
  const int off = static_cast<int>(slot % block_size);
  const size_t src_row = (static_cast<size_t>(token) * num_kv_heads + head) * D;
  const size_t dst_row = ((static_cast<size_t>(blk) * block_size + off) * num_kv_heads + head) * D;
  const size_t sidx = (static_cast<size_t>(blk) * num_kv_heads + head) * block_size + off;
  // both rows' loads before either row's arithmetic and stores
  float xk[D / 32], xv[D / 32];
  load_lane<ST, D / 32>(key + src_row + lane * (D / 32), xk);
  load_lane<ST, D / 32>(value + src_row + lane * (D / 32), xv);
  quant_row<MODE, D>(xk, k_cache, dst_row, k_scale + sidx, lane);
  quant_row<MODE, D>(xv, v_cache, dst_row, v_scale + sidx, lane);
}

template <typename ST, int MODE>
cudaError_t launch_t(const void* key, const void* value, void* kc, void* vc, float* ks, float* vs,
                     const int64_t* slots, int num_tokens, int hkv, int D, int bs, int nb,
                     int* err, cudaStream_t s) {
  const ST* k = static_cast<const ST*>(key);
  const ST* v = static_cast<const ST*>(value);
  const bool pdl = pdl_mode() != 0;
  if constexpr (MODE == kCopy) {
    const long long rows = static_cast<long long>(num_tokens) * hkv;
    const unsigned cblocks = static_cast<unsigned>((rows + 4 * kRowsPerWarp - 1) / (4 * kRowsPerWarp));
    ST* kd = static_cast<ST*>(kc);
    ST* vd = static_cast<ST*>(vc);
    if (D == 128)
      return launch_kernel(cache_copy_kernel<ST, 128>, dim3(cblocks), dim3(128), 0, s, pdl, k, v,
                           kd, vd, slots, num_tokens, hkv, bs, nb, err);
    return launch_kernel(cache_copy_kernel<ST, 64>, dim3(cblocks), dim3(128), 0, s, pdl, k, v, kd,
                         vd, slots, num_tokens, hkv, bs, nb, err);
  }
  const long long warps = static_cast<long long>(num_tokens) * hkv;
  const unsigned blocks = static_cast<unsigned>((warps + 3) / 4);
  if (D == 128)
    return launch_kernel(cache_kernel<ST, MODE, 128>, dim3(blocks), dim3(128), 0, s, pdl, k, v, kc,
                         vc, ks, vs, slots, num_tokens, hkv, bs, nb, err);
  return launch_kernel(cache_kernel<ST, MODE, 64>, dim3(blocks), dim3(128), 0, s, pdl, k, v, kc, vc,
                       ks, vs, slots, num_tokens, hkv, bs, nb, err);
}

template <int MODE>
cudaError_t launch_mode(int src_dtype, const void* key, const void* value, void* kc, void* vc,
                        float* ks, float* vs, const int64_t* slots, int n, int hkv, int D, int bs,
                        int nb, int* err, cudaStream_t s) {
  switch (src_dtype) {
    case PA_F32: return launch_t<float, MODE>(key, value, kc, vc, ks, vs, slots, n, hkv, D, bs, nb, err, s);
    case PA_F16: return launch_t<__half, MODE>(key, value, kc, vc, ks, vs, slots, n, hkv, D, bs, nb, err, s);
    case PA_BF16: return launch_t<__nv_bfloat16, MODE>(key, value, kc, vc, ks, vs, slots, n, hkv, D, bs, nb, err, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_reshape_and_cache(const void* key, const void* value, int src_dtype,
                                     void* k_cache, void* v_cache, int cache_dtype,
                                     float* k_scale, float* v_scale,
                                     const int64_t* slot_mapping, int num_tokens,
                                     int num_kv_heads, int head_dim, int block_size,
                                     int num_blocks, int* err_flag, cudaStream_t stream) {
  if (cache_dtype == PA_INT8)
    return launch_mode<kInt8>(src_dtype, key, value, k_cache, v_cache, k_scale, v_scale,
                              slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                              num_blocks, err_flag, stream);
  if (cache_dtype == PA_FP8E4M3)
    return launch_mode<kFp8>(src_dtype, key, value, k_cache, v_cache, k_scale, v_scale,
                             slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                             num_blocks, err_flag, stream);
  return launch_mode<kCopy>(src_dtype, key, value, k_cache, v_cache, k_scale, v_scale,
                            slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                            num_blocks, err_flag, stream);
}

}  // namespace pa
