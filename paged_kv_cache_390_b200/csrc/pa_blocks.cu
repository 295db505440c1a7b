// pa_blocks.cu -- block copy between KV block pools for sm_100a.
//
// Copy-on-write of a shared block ("KVcache-learning" s05: the sequence that
// writes into a shared block gets its own copy first and its block table is
// repointed) and swap of blocks between the GPU pool and a CPU pool
// ("KVcache-learning" s06 swap_out / swap_in; swap_space on the yunthe.com
// page).  In the cache layout [num_blocks, block_size, num_kv_heads, head_dim]
// a block is one contiguous run of block_size * num_kv_heads * head_dim
// elements, and its scales [num_kv_heads, block_size] are contiguous too, so a
// pair (src, dst) is two (four) contiguous copies.
//
// The copy moves 16-byte vectors.  Each CTA takes a fixed slice of one pair's
// K or V block and keeps kVecPerThread loads per thread in flight before it
// stores them.  The grid is pairs x slices.  Source and destination may live in
// device memory or in mapped pinned host memory (one address space).  The
// kernel does not care which, so the same launch performs copy-on-write,
// swap-out and swap-in.
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"

namespace pa {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kVecPerThread = 4;
constexpr int kVecPerCta = kCopyThreads * kVecPerThread;   // 16 KB per CTA per pass

__global__ void __launch_bounds__(kCopyThreads)
    copy_blocks_kernel(const CopyArgs a) {
  griddep_launch_dependents();
  griddep_wait();
  const int pair = blockIdx.x;
  const int64_t src = a.block_mapping[2 * static_cast<size_t>(pair)];
  const int64_t dst = a.block_mapping[2 * static_cast<size_t>(pair) + 1];
  if (src < 0 || src >= a.src_num_blocks || dst < 0 || dst >= a.dst_num_blocks) {
    if (threadIdx.x == 0 && blockIdx.y == 0) report_error(a.err_flag, kErrBlockId);
    return;                                                  // the pair is skipped
  }
  // slices [0, slices_kv) cover K then V; the last slice of each pair also
  // carries the scales of a quantised cache
  const int64_t nvec = a.block_vecs;                         // 16-byte vectors per block
  const int64_t per_tensor = (nvec + kVecPerCta - 1) / kVecPerCta;
  const int y = blockIdx.y;
  if (y < 2 * per_tensor) {
    const int which = y >= per_tensor;
    const int64_t base = (y - which * per_tensor) * kVecPerCta;
    const uint4* s = reinterpret_cast<const uint4*>(which ? a.src_v : a.src_k) + src * nvec;
    uint4* d = reinterpret_cast<uint4*>(which ? a.dst_v : a.dst_k) + dst * nvec;
    uint4 r[kVecPerThread];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const int64_t i = base + u * kCopyThreads + threadIdx.x;
      if (i < nvec) r[u] = s[i];
    }
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
      const int64_t i = base + u * kCopyThreads + threadIdx.x;
      if (i < nvec) d[i] = r[u];
    }
  } else if (a.scale_vecs > 0) {                             // one extra slice: scales
    for (int i = threadIdx.x; i < 2 * a.scale_vecs; i += kCopyThreads) {
      const int which = i >= a.scale_vecs;
      const int k = i - which * a.scale_vecs;
      const uint4* s = reinterpret_cast<const uint4*>(which ? a.src_vs : a.src_ks) + src * a.scale_vecs;
      uint4* d = reinterpret_cast<uint4*>(which ? a.dst_vs : a.dst_ks) + dst * a.scale_vecs;
      d[k] = s[k];
    }
  }
}

}  // namespace

int copy_slices_per_pair(int64_t block_vecs, int scale_vecs) {
  const int64_t per_tensor = (block_vecs + kVecPerCta - 1) / kVecPerCta;
  return static_cast<int>(2 * per_tensor + (scale_vecs > 0 ? 1 : 0));
}

cudaError_t launch_copy_blocks(const CopyArgs& a, int num_pairs, cudaStream_t stream) {
  const int slices = copy_slices_per_pair(a.block_vecs, a.scale_vecs);
  return launch_kernel(copy_blocks_kernel, dim3(static_cast<unsigned>(num_pairs), slices),
                       dim3(kCopyThreads), 0, stream, pdl_mode() != 0, a);
}

}  // namespace pa
