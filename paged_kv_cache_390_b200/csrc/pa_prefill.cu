// pa_prefill.cu -- multi-token query over the paged KV cache on the 5th-
// generation tensor cores (tcgen05): a chunk of new tokens per sequence
// attends to its cached prefix and, causally, to itself.  This is the prefill
// that automatic prefix caching leaves to compute: the second request sharing
// a cached prompt computes only its new tokens
// ("LLM推理优化：vLLM PagedAttention深度解析与工程实践" §4.2;
// "KVcache-learning" s08), attention as §二 of the former page states it.
//
// One CTA (4 warps) per (128-row query tile, kv head, sequence).  The tile
// packs TQ = 128 / G query tokens x the G query heads of one kv head (row m =
// token m / G, head m % G), so every K/V byte loaded serves the whole GQA
// group.  Per 128-token KV tile:
//   S = Q K^T      tcgen05.mma (M 128, N 128, K = head_dim) into TMEM
//   softmax        each thread owns one row: tcgen05.ld of its S row, causal
//                  mask, online max / sum in the log2 domain, O rescale in TMEM
//                  when the max moves, P (16-bit) into 128-byte swizzled smem
//   O += P V       tcgen05.mma (V read MN-major straight from the TMA tile; bf16
//                  P as a high and a low part, two products)
// In shared-prefix (cascade) mode the rows are every sequence's decode query and
// they all attend, without a causal mask, to the prefix the sequences share: the
// prefix's K/V are read once per kv head instead of once per sequence, and the
// kernel leaves (o / l, m, l) partials that the decode of each sequence's own
// tokens merges (pa_decode_cascade).
// K/V tiles arrive by TMA (one 16-token box per block and 64-column half) into
// two stages; Q arrives once.  Accumulators live in TMEM (256 columns).  Every
// mbarrier wait is bounded; a wait that runs out sets PA_DEVERR_TIMEOUT, lets
// the copies and MMAs in flight finish (bounded), frees TMEM and writes zeros.
#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"
#include "pa_umma.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;                 // query rows per tile (tokens x heads)
constexpr int kKvTile = 128;               // KV tokens per tile
constexpr int kD = 128;                    // head_dim
constexpr int kHalf = 16384;               // one 64-column half of a 128-row tile, bytes
constexpr int kQOff = 0;                   // Q: 2 halves
constexpr int kKvOff = 2 * kHalf;          // stages: K halves then V halves
constexpr int kStageBytes = 4 * kHalf;
constexpr int kPOff = kKvOff + 2 * kStageBytes;     // P (fp16), or P high then P low (bf16)

// bf16 keeps 8 significant bits: P goes in as a high and a low bf16 part (two
// PV products, ~16 bits), fp16's 11 bits need one.
template <typename QT>
__host__ __device__ constexpr int p_parts() { return std::is_same<QT, __nv_bfloat16>::value ? 2 : 1; }
template <typename QT>
__host__ __device__ constexpr int smem_bytes() { return kPOff + p_parts<QT>() * 2 * kHalf + 1024; }   // + alignment slack
constexpr uint32_t kTmemCols = 256;        // S: columns [0,128), O: [128,256)

template <typename QT, int BS>
__global__ void __launch_bounds__(128, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PrefillArgs a) {
  constexpr int BOXH = BS < 16 ? BS : 16;
  constexpr int NBOX = kKvTile / BOXH;     // boxes per 64-column half
  constexpr bool kBf16 = std::is_same<QT, __nv_bfloat16>::value;
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[6];   // q_full, kv_full[2], s_done, o_done, drain
  __shared__ uint32_t tmem_base_slot;

  const int tile = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.num_heads / a.num_kv_heads;
  const int TQ = kRows / G;

  // Wait first, then release the dependent grid: a kernel launched behind this
  // one may then read whatever the kernels before this one wrote.
  griddep_wait();
  griddep_launch_dependents();

  const bool cascade = a.cascade_rows > 0;   // shared-prefix partials, no causal mask
  const int q0 = cascade ? 0 : a.query_start[seq];
  const int q_len = cascade ? a.cascade_rows : a.query_start[seq + 1] - q0;
  const int L = cascade ? a.cascade_len : a.seq_lens[seq];
  const bool bad_len = q_len < 0 || (!cascade && L < q_len) || L < 0 ||
                       static_cast<long long>(L) > static_cast<long long>(a.max_blocks) * BS;
  if (bad_len) {
    if (tid == 0 && a.err_flag) report_error(a.err_flag, kErrSeqLen);
    return;
  }
  if (tile * TQ >= q_len) return;            // this sequence has fewer query tiles
  const int rows_here = min(TQ, q_len - tile * TQ);
  const int pos_last = cascade ? L - 1 : L - q_len + tile * TQ + rows_here - 1;
  const int ntiles = pos_last >= 0 ? pos_last / kKvTile + 1 : 0;

  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  const uint32_t q_s = sbase + kQOff, p_s = sbase + kPOff;
  const uint32_t bar_q = smem_u32(&bars[0]), bar_s = smem_u32(&bars[3]),
                 bar_o = smem_u32(&bars[4]), bar_drain = smem_u32(&bars[5]);
  auto bar_kv = [&](int st) { return smem_u32(&bars[1 + st]); };
  auto kv_s = [&](int st) { return sbase + kKvOff + static_cast<uint32_t>(st * kStageBytes); };
  const int32_t* table = a.block_tables + (cascade ? 0 : static_cast<size_t>(seq) * a.max_blocks);
  const uint64_t pol = policy_evict_first();

  if (tid == 0) {
    for (int i = 0; i < 6; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_barrier_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_slot;
  const uint32_t t_s = tmem, t_o = tmem + 128;
  const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;

  // Warp 0: load KV tile j into stage st (lane b < NBOX finds box b's block).
  int armed_tile[2] = {-1, -1};              // tile in flight into each stage
  auto issue_kv = [&](int j, int st) {
    int row = a.num_blocks * BS;             // past the cache: the box is zero-filled
    if (lane < NBOX) {
      const int t0 = j * kKvTile + lane * BOXH;
      if (t0 < L) {
        const int blk = __ldg(table + t0 / BS);
        if (blk >= 0 && blk < a.num_blocks) row = blk * BS + t0 % BS;
        else if (a.err_flag) report_error(a.err_flag, kErrBlockId);
      }
    }
    if (a.inject == 1 && j == 0) return;     // test hook: this stage never arrives
    armed_tile[st] = j;
    const uint32_t dst = kv_s(st);
#pragma unroll 1
    for (int b = 0; b < NBOX; ++b) {
      const int rb = __shfl_sync(FULL, row, b);
      if (lane == 0) {
        if (b == 0) mbar_arrive_expect_tx(bar_kv(st), 4 * kHalf);
        for (int h = 0; h < 2; ++h) {
          const uint32_t off = static_cast<uint32_t>(h * kHalf + b * BOXH * 128);
          tma_load_3d(dst + off, &tm_k, h * 64, kvh, rb, bar_kv(st), pol);
          tma_load_3d(dst + 2 * kHalf + off, &tm_v, h * 64, kvh, rb, bar_kv(st), pol);
        }
      }
    }
  };

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * kHalf);
      const int qrow = q0 + tile * TQ;
      for (int h = 0; h < 2; ++h)
        tma_load_3d(q_s + h * kHalf, &tm_q, h * 64, kvh * G, qrow, bar_q, pol);
    }
    issue_kv(0, 0);
    if (ntiles > 1) issue_kv(1, 1);
  }

  // This thread's row.
  const int r = tid / G;
  const bool row_valid = tile * TQ + r < q_len;
  const int pos = !row_valid ? -1 : (cascade ? L - 1 : L - q_len + tile * TQ + r);
  float m_run = -INFINITY, l_run = 0.f;

  const uint32_t idesc_s = umma_idesc_f16(kBf16, false, kRows, kKvTile);
  const uint32_t idesc_o = umma_idesc_f16(kBf16, true, kRows, kD);
  bool dead = false;
  int issued_mma = 0;                        // tiles whose PV MMAs were issued

  for (int j = 0; j < ntiles; ++j) {
    const int st = j & 1;
    bool ok = true;
    if (tid == 0) {
      ok = mbar_wait_bounded(bar_q, 0, a.timeout_ns) &&
           mbar_wait_bounded(bar_kv(st), (j >> 1) & 1, a.timeout_ns);
      if (ok) armed_tile[st] = -1;
    }
    if (__syncthreads_or(!ok)) {
      dead = true;
      break;
    }
    if (tid == 0) {                          // S = Q K^T
      tc_fence_after_sync();
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t koff = static_cast<uint32_t>((kk >> 2) * kHalf + (kk & 3) * 32);
        umma_f16_ss(t_s, umma_desc_sw128(q_s + koff, 16, 1024),
                    umma_desc_sw128(kv_s(st) + koff, 16, 1024), idesc_s, kk > 0);
      }
      umma_commit(bar_s);
    }
    ok = mbar_wait_bounded(bar_s, j & 1, a.timeout_ns);
    if (__syncthreads_or(!ok)) {
      dead = true;
      break;
    }
    tc_fence_after_sync();
    float s[kKvTile];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v[32];
      tmem_ld32(t_s + lane_off + 32 * i, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) s[32 * i + e] = v[e];
    }
    tmem_wait_ld();

    if (j > 0) {                             // PV(j-1) done: O, P and stage j-1 are free
      ok = mbar_wait_bounded(bar_o, (j - 1) & 1, a.timeout_ns);
      if (__syncthreads_or(!ok)) {
        dead = true;
        break;
      }
      tc_fence_after_sync();
      if (warp == 0 && j + 1 < ntiles) issue_kv(j + 1, (j + 1) & 1);
    }

    // ---- causal mask + online softmax (log2 domain), one row per thread
    const int t_base = j * kKvTile;
    float tmax = -INFINITY;
#pragma unroll
    for (int c = 0; c < kKvTile; ++c) {
      s[c] = (t_base + c <= pos) ? s[c] * a.scale_log2 : -INFINITY;
      tmax = fmaxf(tmax, s[c]);
    }
    const float m_new = fmaxf(m_run, tmax);
    const float base = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = fast_exp2(m_run - base);
    float psum = 0.f;
#pragma unroll
    for (int c = 0; c < kKvTile; ++c) {
      s[c] = fast_exp2(s[c] - base);
      psum += s[c];
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;

    if (j > 0 && __any_sync(FULL, alpha != 1.f)) {   // rescale this warp's O rows
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float v[32];
        tmem_ld32(t_o + lane_off + 32 * i, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] *= alpha;
        tmem_st32(t_o + lane_off + 32 * i, v);
      }
      tmem_wait_st();
    }

    // ---- P (16-bit; bf16 as high + low parts) into 128-byte swizzled K-major A tiles
    {
      const uint32_t row_addr = p_s + static_cast<uint32_t>(tid * 128);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const float* pp = s + h * 64 + c8 * 8;
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            hw[e] = pack2<QT>(pp[2 * e], pp[2 * e + 1]);
            if constexpr (p_parts<QT>() == 2) {
              const float2 f = unpack2<QT>(hw[e]);
              lw[e] = pack2<QT>(pp[2 * e] - f.x, pp[2 * e + 1] - f.y);
            }
          }
          const uint32_t addr = row_addr + h * kHalf + (static_cast<uint32_t>(c8 ^ (tid & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(hw[0]),
                       "r"(hw[1]), "r"(hw[2]), "r"(hw[3])
                       : "memory");
          if constexpr (p_parts<QT>() == 2)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr + 2 * kHalf),
                         "r"(lw[0]), "r"(lw[1]), "r"(lw[2]), "r"(lw[3])
                         : "memory");
        }
      }
    }
    // V rows of tokens at or past the sequence end: zero them so that poisoned
    // or stale slots cannot turn 0 * x into NaN inside the MMA
    if (t_base + kKvTile > L) {
      const int first = max(0, L - t_base);
      for (int idx = tid; idx < (kKvTile - first) * 16; idx += 128) {
        const int row = first + idx / 16, ch = idx % 16;
        const uint32_t addr = kv_s(st) + 2 * kHalf + (ch >> 3) * kHalf + row * 128 + (ch & 7) * 16;
        asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
      }
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {                          // O += P V
      tc_fence_after_sync();
#pragma unroll
      for (int part = 0; part < p_parts<QT>(); ++part) {
#pragma unroll
        for (int kk = 0; kk < kKvTile / 16; ++kk) {
          const uint32_t poff =
              static_cast<uint32_t>(part * 2 * kHalf + (kk >> 2) * kHalf + (kk & 3) * 32);
          const uint32_t voff = static_cast<uint32_t>(2 * kHalf + kk * 16 * 128);
          umma_f16_ss(t_o, umma_desc_sw128(p_s + poff, 16, 1024),
                      umma_desc_sw128(kv_s(st) + voff, kHalf, 1024), idesc_o,
                      j > 0 || part > 0 || kk > 0);
        }
      }
      umma_commit(bar_o);
    }
    issued_mma = j + 1;
  }

  if (!dead && ntiles > 0) {
    const bool ok = mbar_wait_bounded(bar_o, (ntiles - 1) & 1, a.timeout_ns);
    dead = __syncthreads_or(!ok);
  }
  if (dead) {
    // let every copy and MMA still in flight finish before TMEM and smem go away
    if (tid == 0) {
      report_error(a.err_flag, kErrTimeout);
      for (int st = 0; st < 2; ++st)
        if (armed_tile[st] >= 0)
          mbar_wait_bounded(bar_kv(st), (armed_tile[st] >> 1) & 1, kDrainLimitNs);
      umma_commit(bar_drain);
      mbar_wait_bounded(bar_drain, 0, kDrainLimitNs);
    }
    __syncthreads();
  }
  (void)issued_mma;

  // ---- epilogue: out row = O / l (cascade: the partial o / l, m, l)
  tc_fence_after_sync();
  const float inv = (!dead && l_run > 0.f) ? 1.f / l_run : 0.f;
  const int h = kvh * G + tid % G;
  if (cascade) {
    const size_t pr = static_cast<size_t>(q0 + tile * TQ + r) * a.num_heads + h;
    if (row_valid) {
      a.part_m[pr] = dead ? -INFINITY : m_run;
      a.part_l[pr] = dead ? 0.f : l_run;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v[32];
      tmem_ld32(t_o + lane_off + 32 * i, v);
      tmem_wait_ld();
      if (row_valid) {
        float4* dst = reinterpret_cast<float4*>(a.part_o + pr * kD + 32 * i);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv,
                               v[4 * e + 3] * inv);
      }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
    return;
  }
  QT* orow = reinterpret_cast<QT*>(a.out) +
             (static_cast<size_t>(q0 + tile * TQ + r) * a.num_heads + h) * kD;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v[32];
    tmem_ld32(t_o + lane_off + 32 * i, v);
    tmem_wait_ld();
    if (row_valid) {
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 w;
        w.x = pack2<QT>(v[e] * inv, v[e + 1] * inv);
        w.y = pack2<QT>(v[e + 2] * inv, v[e + 3] * inv);
        w.z = pack2<QT>(v[e + 4] * inv, v[e + 5] * inv);
        w.w = pack2<QT>(v[e + 6] * inv, v[e + 7] * inv);
        *reinterpret_cast<uint4*>(orow + 32 * i + e) = w;
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

cudaError_t make_q_map(CUtensorMap* map, const void* q, int total_q, int num_heads, int G) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(num_heads),
                        static_cast<cuuint64_t>(total_q)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD) * 2,
                           static_cast<cuuint64_t>(num_heads) * kD * 2};
  cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(kRows / G)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult rc = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(q), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename QT, int BS>
cudaError_t launch_t(const PrefillArgs& a, int total_q, int max_query_len, cudaStream_t stream) {
  // cascade: one pseudo-sequence of total_q rows (max_query_len = total_q)
  const int G = a.num_heads / a.num_kv_heads;
  CUtensorMap mq, mk, mv;
  cudaError_t e = make_q_map(&mq, a.q, total_q, a.num_heads, G);
  if (e != cudaSuccess) return e;
  e = make_cache_map<kKind16, kD, BS>(&mk, a.k_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  e = make_cache_map<kKind16, kD, BS>(&mv, a.v_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  auto kern = prefill_kernel<QT, BS>;
  constexpr int kSmemBytes = smem_bytes<QT>();
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int TQ = kRows / G;
  const dim3 grid((max_query_len + TQ - 1) / TQ, a.num_kv_heads, a.cascade_rows > 0 ? 1 : a.num_seqs);
  return launch_kernel(kern, grid, dim3(128), kSmemBytes, stream, pdl_mode() != 0, mq, mk, mv, a);
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, int q_dtype, int block_size, int total_q,
                           int max_query_len, cudaStream_t stream) {
  const bool bf = q_dtype == PA_BF16;
  switch (block_size) {
    case 8: return bf ? launch_t<__nv_bfloat16, 8>(a, total_q, max_query_len, stream)
                      : launch_t<__half, 8>(a, total_q, max_query_len, stream);
    case 16: return bf ? launch_t<__nv_bfloat16, 16>(a, total_q, max_query_len, stream)
                       : launch_t<__half, 16>(a, total_q, max_query_len, stream);
    case 32: return bf ? launch_t<__nv_bfloat16, 32>(a, total_q, max_query_len, stream)
                       : launch_t<__half, 32>(a, total_q, max_query_len, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pa
