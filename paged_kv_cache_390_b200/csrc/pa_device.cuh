// pa_device.cuh -- device-side building blocks for the paged decode kernels on
// sm_100a: mbarrier waits with a time limit, TMA tile loads and bulk copies,
// shared-memory swizzle addressing, ldmatrix / movmatrix / mma.sync fragments
// and the 8-bit code conversions.  Everything here is inline PTX or a CUDA
// intrinsic; no library code.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Bits OR-ed into the caller's err_flag (and into the library's device word).
enum : int {
  kErrBlockId = 1,      // a block table entry outside [0, num_blocks)
  kErrSeqLen = 2,       // seq_len < 0 or beyond the table's capacity
  kErrSlot = 4,         // a slot at or past num_blocks * block_size
  kErrTimeout = 8,      // an mbarrier wait gave up after its time limit
};

// Library-wide device error word: set on any device-side error even when the
// caller passed no err_flag.  Read (and cleared) by pa_get_device_error().
extern __device__ int g_pa_device_error;

__device__ __forceinline__ void report_error(int* err_flag, int bits) {
  if (err_flag) atomicOr(err_flag, bits);
  atomicOr(&g_pa_device_error, bits);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- PDL
// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now, and (separately) wait until the previous kernel in the stream
// has completed and its writes are visible.  Both are no-ops for a kernel
// launched without the programmatic-serialization attribute.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for phase `parity` of a barrier, giving up after `limit_ns`.  Returns
// false on time-out; the caller records the error and stops issuing work.
// A limit of at most 1 ns means a single non-blocking test (used to exercise
// the time-out path deterministically).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (limit_ns <= 1) return mbar_test_wait(bar, parity);
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// As mbar_wait_bounded, for kernels whose warps play different roles: a wait
// that runs out sets *abort, and every other wait on the CTA gives up as soon as
// it sees *abort set (so one lost arrival ends all roles within one limit).
__device__ __forceinline__ bool mbar_wait_abortable(uint32_t bar, uint32_t parity,
                                                    uint64_t limit_ns, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      return false;
    }
  }
  return true;
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Orders this thread's earlier generic-proxy global writes before its (or, after
// a barrier, its warp's) later async-proxy reads such as TMA loads.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
// Tiled 3-D tensor load (no multicast) completing on an mbarrier; L2 policy
// `policy` (a createpolicy value) marks streamed KV as evict-first.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1,
                                            int c2, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar), "l"(policy)
      : "memory");
}

// L2 prefetch of one tile of a tensor map (no shared memory, no barrier).
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* map, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// L2 prefetch of `bytes` (a multiple of 16) from a 16-byte aligned address.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a
// multiple of 16), completing on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- swizzle
// Byte offset of 16-byte chunk `chunk` of row `row` in a tile whose rows are
// RB bytes and which TMA filled with the matching swizzle (128B for 128-byte
// rows, 64B for 64-byte rows).  The tile base must be 1024-byte aligned.
template <int RB>
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t chunk) {
  if constexpr (RB == 128) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
  } else {
    static_assert(RB == 64, "rows are 64 or 128 bytes");
    return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
  }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose an 8x8 matrix of 16-bit elements held one row-pair per thread.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

// ---------------------------------------------------------------- mma.sync
template <typename T>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1);

template <>
__device__ __forceinline__ void mma_16816<__half>(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <>
__device__ __forceinline__ void mma_16816<__nv_bfloat16>(float (&d)[4], const uint32_t (&a)[4],
                                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- numerics
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Pack two floats (lo, hi) into a 16-bit pair of type T, round to nearest even.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);

template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t v);

template <>
__device__ __forceinline__ float2 unpack2<__half>(uint32_t v) {
  return __half22float2(*reinterpret_cast<__half2*>(&v));
}

template <>
__device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t v) {
  return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&v));
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Two INT8 codes (bytes 0 and 1 of `w`, already byte-selected) -> exact pair.
// fp16: bias each code by 128 into the mantissa of 1024.0 (0x6400) and
// subtract 1152 = 1024 + 128; every step is exact.
__device__ __forceinline__ uint32_t int8x2_to_f16x2(uint32_t w) {
  const uint32_t biased = __byte_perm(w ^ 0x8080u, 0x6464u, 0x5140);  // {b0^80, 64, b1^80, 64}
  __half2 h = *reinterpret_cast<const __half2*>(&biased);
  h = __hsub2(h, __float2half2_rn(1152.0f));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two INT8 codes of a word already XORed with 0x80808080, picked by a byte_perm
// selector `sel` that interleaves them with the 0x64 exponent bytes
// ({b, 0x64, b', 0x64}), -> exact f16 pair: one permute and one subtract.
template <uint32_t SEL>
__device__ __forceinline__ uint32_t int8x2_biased_to_f16x2(uint32_t wx) {
  const uint32_t biased = __byte_perm(wx, 0x64646464u, SEL);
  __half2 h = *reinterpret_cast<const __half2*>(&biased);
  h = __hsub2(h, __float2half2_rn(1152.0f));
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two E4M3 codes in a 16-bit register -> exact f16 pair.
__device__ __forceinline__ uint32_t e4m3x2h_to_f16x2(uint16_t s) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(s));
  return d;
}

// The two 16-bit halves of a word (a register split, no shifts).
__device__ __forceinline__ void split_halves(uint32_t w, uint16_t& lo, uint16_t& hi) {
  asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(w));
}

__device__ __forceinline__ uint32_t int8x2_to_bf16x2(uint32_t w) {
  const float lo = static_cast<float>(static_cast<int8_t>(w & 0xFFu));
  const float hi = static_cast<float>(static_cast<int8_t>((w >> 8) & 0xFFu));
  return pack2<__nv_bfloat16>(lo, hi);
}

// Two E4M3 codes (low 16 bits of `w`) -> exact f16 pair (E4M3 is a subset of fp16).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t d;
  const uint16_t s = static_cast<uint16_t>(w & 0xFFFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(s));
  return d;
}

__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t w) {
  const float2 f = unpack2<__half>(e4m3x2_to_f16x2(w));   // exact
  return pack2<__nv_bfloat16>(f.x, f.y);                 // exact: E4M3 fits bf16
}

}  // namespace pa
