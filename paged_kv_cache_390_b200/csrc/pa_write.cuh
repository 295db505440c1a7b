// pa_write.cuh -- one warp writes one (token, kv head) row of the paged cache:
// a plain copy, or symmetric per-row quantisation to INT8 / FP8 E4M3 with its
// fp32 scale.  Shared by the cache-write kernel (pa_cache.cu) and the decode
// kernel's fused write of each sequence's new token (pa_decode.cu).
//
// Quantisation as "KVcache-learning" s09 (E4M3, range +-448) and the INT8
// kv_cache_dtype of "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置"
// describe it, per token and head: s = max|x| / 127 (or / 448), code =
// rne(x / s), every division IEEE fp32 round-to-nearest, FP8 saturating to
// +-448; a row of zeros stores s = 0 and codes 0.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace pa {

enum { kWriteCopy = 0, kWriteInt8 = 1, kWriteFp8 = 2 };

template <typename ST>
__device__ __forceinline__ float to_f32(ST v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// One lane's EPL consecutive elements of a row as one vector load (the row start
// is 16-byte aligned and EPL * sizeof(ST) divides 16).
template <typename ST, int EPL>
__device__ __forceinline__ void load_lane(const ST* __restrict__ p, float (&x)[EPL]) {
  struct alignas(EPL * sizeof(ST)) Vec {
    ST v[EPL];
  };
  const Vec w = *reinterpret_cast<const Vec*>(p);
#pragma unroll
  for (int e = 0; e < EPL; ++e) x[e] = to_f32<ST>(w.v[e]);
}

// The code of x / s: the division IEEE binary32, round to nearest even, then INT8
// rounding (nearest even) and clamping to +-127, or E4M3 rounding with saturation.
template <int MODE>
__device__ __forceinline__ uint32_t quant_code(float x, float s) {
  const float y = __fdiv_rn(x, s);
  if constexpr (MODE == kWriteInt8) {
    int k = __float2int_rn(y);
    k = k > 127 ? 127 : (k < -127 ? -127 : k);
    return static_cast<uint32_t>(k) & 0xFFu;
  } else {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3));
  }
}

// Whole warp: quantise one row held as D / 32 values per lane (lane l holds
// elements [l * EPL, (l + 1) * EPL)) into the cache row at element index dst_row,
// and its scale into *scale_slot.
template <int MODE, int D>
__device__ __forceinline__ void quant_row(const float (&x)[D / 32], void* cache, size_t dst_row,
                                          float* scale_slot, int lane) {
  constexpr int EPL = D / 32;
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, MODE == kWriteInt8 ? 127.0f : 448.0f);
  uint32_t packed = 0;
#pragma unroll
  for (int e = 0; e < EPL; ++e)
    if (s != 0.f) packed |= quant_code<MODE>(x[e], s) << (8 * e);
  uint8_t* d = static_cast<uint8_t*>(cache) + dst_row + lane * EPL;
  if constexpr (EPL == 4) *reinterpret_cast<uint32_t*>(d) = packed;
  else *reinterpret_cast<uint16_t*>(d) = static_cast<uint16_t>(packed);
  if (lane == 0) *scale_slot = s;
}

// Whole warp: src = D elements of type ST; dst = the cache row (element index
// dst_row of `cache`); *scale_slot receives s for the quantised modes.
template <typename ST, int MODE, int D>
__device__ __forceinline__ void write_kv_row(const ST* __restrict__ src, void* cache,
                                             size_t dst_row, float* scale_slot, int lane) {
  if constexpr (MODE == kWriteCopy) {
    constexpr int NV = D * static_cast<int>(sizeof(ST)) / 16;   // 16-byte vectors per row
    const uint4* s = reinterpret_cast<const uint4*>(src);
    uint4* d = reinterpret_cast<uint4*>(static_cast<ST*>(cache) + dst_row);
    for (int k = lane; k < NV; k += 32) d[k] = s[k];
  } else {
    float x[D / 32];
    load_lane<ST, D / 32>(src + lane * (D / 32), x);
    quant_row<MODE, D>(x, cache, dst_row, scale_slot, lane);
  }
}

}  // namespace pa
