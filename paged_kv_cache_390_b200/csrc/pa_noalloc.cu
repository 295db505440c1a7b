// pa_noalloc.cu -- pa_decode_fused_noalloc: the single-launch decode of
// pa_decode_fused with its scratch in a fixed device array, for callers that
// cannot allocate device memory at the point of the call (an inference-engine
// plugin whose enqueue step must not allocate, a library that owns no
// allocator because a framework's caching allocator holds the device memory,
// a server that has handed nearly all of HBM to its KV block pool).
//
// The scratch is a file-scope __device__ array: every GPU that loads the
// library holds it until the process exits.  In host code its name is only a
// stand-in for the device symbol, so its device address is fetched with
// cudaGetSymbolAddress, once per device, with that device current (and once more
// if the device's context is replaced, as by cudaDeviceReset).
#include <cuda.h>

#include <cstddef>
#include <mutex>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(24) << 20;   // 24 MiB per device
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
struct ScratchAddr {
  unsigned long long ctx_id = 0;        // the context the address belongs to
  void* ptr = nullptr;
};
ScratchAddr g_noalloc_addr[64];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Identity of the current context (0 if it cannot be had): a device reset
// destroys the context, the next one gets a new id, and the array's address is
// looked up again there.
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of this device's scratch: looked up on the first call per device
// (and again after the device's context has been replaced, e.g. by a reset).
cudaError_t noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const unsigned long long id = current_ctx_id();   // 0 (look up again) if none is current yet
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddr& a = g_noalloc_addr[dev];
  if (!a.ptr || id == 0 || a.ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    a.ptr = p;
    a.ctx_id = id;
  }
  *out = a.ptr;
  return cudaSuccess;
}

}  // namespace
}  // namespace pa

extern "C" {

PA_API size_t pa_decode_fused_noalloc_scratch_bytes(void) { return pa::kNoAllocScratchBytes; }

PA_API int pa_decode_fused_noalloc(void* out, const void* q, pa_dtype q_dtype,
                                   const void* k_cache, const void* v_cache, pa_dtype cache_dtype,
                                   const float* k_scale, const float* v_scale,
                                   const int32_t* block_tables, int max_blocks_per_seq,
                                   const int32_t* seq_lens, int num_seqs, int num_heads,
                                   int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                   float scale, int* err_flag, pa_stream_t stream) {
  // Every host check first: a rejected call touches neither the GPU nor the array.
  const int rc = pa::fused_host_checks(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale,
                                       v_scale, block_tables, max_blocks_per_seq, seq_lens,
                                       num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                       num_blocks, scale);
  if (rc != PA_OK) return rc;
  // Shapes that need no scratch go straight through.
  if (num_seqs == 0 || cache_dtype == PA_F32)
    return pa_decode_fused(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                           block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                           num_kv_heads, head_dim, block_size, num_blocks, scale, nullptr, 0,
                           err_flag, stream);
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return PA_ERR_CUDA;
  const size_t need = pa_decode_fused_workspace_bytes(num_seqs, num_kv_heads, head_dim, sms);
  if (need == 0 || need > pa::kNoAllocScratchBytes) return PA_ERR_UNSUPPORTED;
  void* ws = nullptr;
  if (pa::noalloc_scratch(&ws) != cudaSuccess) return PA_ERR_CUDA;
  // The arrival counters must start at zero; the array keeps the last call's contents.
  const size_t counters = static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int);
  if (cudaMemsetAsync(ws, 0, counters, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PA_ERR_CUDA;
  return pa_decode_fused(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                         block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_heads,
                         num_kv_heads, head_dim, block_size, num_blocks, scale, ws,
                         pa::kNoAllocScratchBytes, err_flag, stream);
}

}  // extern "C"
