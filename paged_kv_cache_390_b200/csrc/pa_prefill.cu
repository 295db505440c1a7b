// pa_prefill.cu -- multi-token query over the paged KV cache on the 5th-
// generation tensor cores (tcgen05): a chunk of new tokens per sequence
// attends to its cached prefix and, causally, to itself.  This is the prefill
// that automatic prefix caching leaves to compute: the second request sharing
// a cached prompt computes only its new tokens
// ("LLM推理优化：vLLM PagedAttention深度解析与工程实践" §4.2;
// "KVcache-learning" s08), attention as §二 of the former page states it.
//
// A query tile packs TQ = 128 / G query tokens x the G query heads of one kv
// head (row m = token m / G, head m % G), so every K/V byte loaded serves the
// whole GQA group.  One CTA holds two such tiles (A and B) and plays four
// roles with its 10 warps:
//   warp 8      TMA: Q once, then 128-token K and V tiles (one box per block
//               and 64-column half) into rings of 3 (K) and 2 (V) stages, K
//               running one tile ahead of V;
//   warp 9      MMA: one thread issues every tcgen05.mma --
//               S_x = Q_x K^T (M 128, N 128, K = head_dim; both operands in
//               shared memory) into TMEM, and O_x += P_x V (N = head_dim, P
//               read from TMEM, V MN-major from the TMA tile), in the order
//               PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the tensor core works
//               on one tile while the other tile's softmax runs;
//   warps 0-3   softmax of tile A, warps 4-7 of tile B: each thread owns one
//               row -- tcgen05.ld of its 128 S columns, causal mask, online sum
//               in the log2 domain against a base that moves only when the row
//               max jumps by more than 8 (then O is rescaled in TMEM), P
//               (16-bit; bf16 as a high and a low part) written back over the
//               S columns it has read, where the PV product takes it from.
//               Its FP32 work runs as packed f32x2 instructions (two results
//               each) and its maxima as 3-input max: the softmax is bound by
//               instruction issue, not by the 16 exponentials per clock of the
//               special-function unit (moving a share of them to a polynomial
//               on the FMA pipe made it slower).
// 128-token tiles keep every MMA at N = 128: a tcgen05.mma of N = 64 costs
// about as long as one of N = 128, so narrower tiles halve the tensor rate.
// P over S needs one order the hardware does not give by itself: S_x(j+1)
// may overwrite P_x(j) only once PV_x(j) has completed, so the MMA thread
// waits for PV_x(j)'s commit before it issues S_x(j+1).
// Hand-offs are mbarriers (TMA transaction counts, tcgen05.commit, thread
// arrivals).  Every wait is bounded: one that runs out sets a CTA-wide abort
// flag that ends every role; the CTA then lets its copies and MMAs finish,
// reports PA_DEVERR_TIMEOUT, writes zeros and frees TMEM.
//
// In shared-prefix (cascade) mode the rows are every sequence's decode query and
// they all attend, without a causal mask, to the prefix the sequences share: the
// prefix's K/V are read once per kv head instead of once per sequence, and the
// kernel leaves (o / l, m, l) partials that the decode of each sequence's own
// tokens merges (pa_decode_cascade).  The prefix's KV tiles may be split over
// blockIdx.z so that a batch of few query tiles still fills the GPU; each split
// leaves its own partial.
#include <cudaTypedefs.h>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"
#include "pa_umma.cuh"

namespace pa {
namespace {

constexpr int kRows = 128;                 // rows per query tile (tokens x heads)
constexpr int kQTiles = 2;                 // query tiles per CTA (A, B)
constexpr int kBN = 128;                   // KV tokens per tile (N of the S product)
constexpr int kD = 128;                    // head_dim
constexpr int kKst = 3, kVst = 2;          // K and V ring stages
constexpr int kQHalf = 16384;              // 128 rows x 128 bytes (one 64-column half)
constexpr int kKvHalf = 16384;             // 128 tokens x 128 bytes
constexpr int kKvTile = 2 * kKvHalf;       // one K or V tile: two 64-column halves
constexpr int kQOff = 0;
constexpr int kKOff = kQTiles * 2 * kQHalf;
constexpr int kVOff = kKOff + kKst * kKvTile;
constexpr int kSmemBytes = kVOff + kVst * kKvTile + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 512;        // S_A, S_B, O_A, O_B: 128 columns each
constexpr int kThreads = 320;
constexpr int kTmaWarp = 8, kMmaWarp = 9;

// bf16 keeps 8 significant bits: P goes in as a high and a low bf16 part (two
// PV products, ~16 bits); fp16's 11 bits need one.  P of 128 tokens takes 64
// TMEM columns per part.
template <typename QT>
__host__ __device__ constexpr int p_parts() { return std::is_same<QT, __nv_bfloat16>::value ? 2 : 1; }

// ---- packed f32x2 arithmetic: two FP32 results per instruction
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t f2splat(float v) { return f2pack(v, v); }
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

enum {
  kBarQ = 0, kBarKFull = 1, kBarKEmpty = kBarKFull + kKst, kBarVFull = kBarKEmpty + kKst,
  kBarVEmpty = kBarVFull + kVst, kBarSFull = kBarVEmpty + kVst, kBarPFull = kBarSFull + 2,
  kBarODone = kBarPFull + 2, kBarDrain = kBarODone + 2, kNumBars
};

template <typename QT, int BS>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PrefillArgs a) {
  constexpr int BOXH = BS < 16 ? BS : 16;
  constexpr int NBOX = kBN / BOXH;         // boxes per 64-column half
  constexpr bool kBf16 = std::is_same<QT, __nv_bfloat16>::value;
  constexpr int PARTS = p_parts<QT>();
  constexpr uint32_t FULL = 0xffffffffu;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;

  const int tile2 = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
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
  const int row0 = tile2 * kQTiles * TQ;     // first query token of tile A
  if (row0 >= q_len) return;                 // this sequence has fewer query tiles
  const int row_end = min(row0 + kQTiles * TQ, q_len);
  const int pos_last = cascade ? L - 1 : L - q_len + row_end - 1;
  int t_lo = 0;                              // first KV tile of this CTA
  int ntiles = pos_last >= 0 ? pos_last / kBN + 1 : 0;
  if (cascade && a.cascade_splits > 1) {     // the prefix split over blockIdx.z
    const int per = (ntiles + a.cascade_splits - 1) / a.cascade_splits;
    t_lo = min(ntiles, seq * per);
    ntiles = min(ntiles - t_lo, per);
  }

  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  auto bar = [&](int i) { return smem_u32(&bars[i]); };
  auto q_s = [&](int x) { return sbase + kQOff + static_cast<uint32_t>(x * 2 * kQHalf); };
  auto k_s = [&](int st) { return sbase + kKOff + static_cast<uint32_t>(st * kKvTile); };
  auto v_s = [&](int st) { return sbase + kVOff + static_cast<uint32_t>(st * kKvTile); };
  const int32_t* table = a.block_tables + (cascade ? 0 : static_cast<size_t>(seq) * a.max_blocks);
  volatile int* abort = &abort_flag;

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) {
      const bool from_threads = i >= kBarPFull && i < kBarPFull + 2;
      mbar_init(bar(i), from_threads ? kRows : 1);
    }
    abort_flag = 0;
    fence_barrier_init();
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&tmem_base_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = tmem_base_slot;
  // S_x (f32) and, over it once read, P_x (16-bit pairs per column; bf16's low
  // part in columns 64..127)
  auto t_s = [&](int x) { return tmem + static_cast<uint32_t>(128 * x); };
  auto t_o = [&](int x) { return tmem + 256u + static_cast<uint32_t>(128 * x); };

  // softmax state (warps 0-7), kept here for the epilogue
  const int x_me = warp < 8 ? warp / 4 : 0;
  const int row_me = tid % kRows;
  const int r_tok = row_me / G;
  const int tok_me = row0 + x_me * TQ + r_tok;          // query token within the chunk
  const bool row_valid = warp < 8 && tok_me < q_len;
  float m_run = -INFINITY, l_run = 0.f;
  int armed_k[kKst], armed_v[kVst];          // TMA warp: last tile issued into each stage
#pragma unroll
  for (int i = 0; i < kKst; ++i) armed_k[i] = -1;
#pragma unroll
  for (int i = 0; i < kVst; ++i) armed_v[i] = -1;

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    const uint64_t pol = policy_evict_first();
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(kBarQ), kQTiles * 2 * kQHalf);
      for (int x = 0; x < kQTiles; ++x)        // rows past the chunk: zero-filled or unused
        for (int h = 0; h < 2; ++h)
          tma_load_3d(q_s(x) + h * kQHalf, &tm_q, h * 64, kvh * G, q0 + row0 + x * TQ,
                      bar(kBarQ), pol);
    }
    // one tile's cache rows, lane b holding box b's (past the cache: the box
    // is zero-filled)
    auto tile_rows = [&](int j) {
      int row = a.num_blocks * BS;
      if (lane < NBOX) {
        const int t0 = (t_lo + j) * kBN + lane * BOXH;
        if (t0 < L) {
          const int blk = __ldg(table + t0 / BS);
          if (blk >= 0 && blk < a.num_blocks) row = blk * BS + t0 % BS;
          else if (a.err_flag) report_error(a.err_flag, kErrBlockId);
        }
      }
      return row;
    };
    auto load_tile = [&](const CUtensorMap* map, uint32_t dst, int row, uint32_t full) {
#pragma unroll 1
      for (int b = 0; b < NBOX; ++b) {
        const int rb = __shfl_sync(FULL, row, b);
        if (lane == 0) {
          if (b == 0) mbar_arrive_expect_tx(full, kKvTile);
          for (int h = 0; h < 2; ++h)
            tma_load_3d(dst + static_cast<uint32_t>(h * kKvHalf + b * BOXH * 128), map, h * 64,
                        kvh, rb, full, pol);
        }
      }
    };
    // K(j), then V(j - 1): the S product of a tile comes one step before its PV
    int row_prev = 0;
    for (int j = 0; j <= ntiles; ++j) {
      int row = 0;
      if (j < ntiles) {
        const int ks = j % kKst;
        if (j >= kKst) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait_abortable(bar(kBarKEmpty + ks), ((j / kKst) - 1) & 1,
                                                  a.timeout_ns, abort);
          if (!__shfl_sync(FULL, ok, 0)) break;
        }
        row = tile_rows(j);
        if (!(a.inject == 1 && j == 0)) {    // test hook: K(0) never arrives
          armed_k[ks] = j;
          load_tile(&tm_k, k_s(ks), row, bar(kBarKFull + ks));
        }
      }
      if (j >= 1) {
        const int jv = j - 1, vs = jv % kVst;
        if (jv >= kVst) {
          bool ok = true;
          if (lane == 0) ok = mbar_wait_abortable(bar(kBarVEmpty + vs), ((jv / kVst) - 1) & 1,
                                                  a.timeout_ns, abort);
          if (!__shfl_sync(FULL, ok, 0)) break;
        }
        armed_v[vs] = jv;
        load_tile(&tm_v, v_s(vs), row_prev, bar(kBarVFull + vs));
      }
      row_prev = row;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc_s = umma_idesc_f16(kBf16, false, kRows, kBN);
    const uint32_t idesc_o = umma_idesc_f16(kBf16, true, kRows, kD);
    auto wait1 = [&](int b, uint32_t parity) {
      bool ok = true;
      if (lane == 0) ok = mbar_wait_abortable(bar(b), parity, a.timeout_ns, abort);
      return __shfl_sync(FULL, ok, 0) != 0;
    };
    // operand descriptors of the first stage / tile; a K slice, stage or tile
    // moves only the start-address field (bytes >> 4), which no offset here
    // carries out of
    const uint64_t dq0 = umma_desc_sw128(q_s(0), 16, 1024);
    const uint64_t dk0 = umma_desc_sw128(k_s(0), 16, 1024);
    const uint64_t dv0 = umma_desc_sw128(v_s(0), kKvHalf, 1024);
    auto issue_s = [&](int x, int j) {       // S_x = Q_x K_j^T
      if (lane == 0) {
        tc_fence_after_sync();
        const uint64_t qd = dq0 + static_cast<uint64_t>(x * (2 * kQHalf >> 4));
        const uint64_t kd = dk0 + static_cast<uint64_t>((j % kKst) * (kKvTile >> 4));
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t qoff = static_cast<uint32_t>(((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4);
          const uint32_t koff = static_cast<uint32_t>(((kk >> 2) * kKvHalf + (kk & 3) * 32) >> 4);
          umma_f16_ss(t_s(x), qd + qoff, kd + koff, idesc_s, kk > 0);
        }
        umma_commit(bar(kBarSFull + x));
      }
      __syncwarp();
    };
    auto issue_pv = [&](int x, int j) {      // O_x += P_x V_j, P from TMEM
      if (lane == 0) {
        tc_fence_after_sync();
        const uint64_t vd = dv0 + static_cast<uint64_t>((j % kVst) * (kKvTile >> 4));
#pragma unroll
        for (int part = 0; part < PARTS; ++part) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk)
            umma_f16_ts(t_o(x), t_s(x) + static_cast<uint32_t>(part * 64 + kk * 8),
                        vd + static_cast<uint32_t>(kk * 16 * 128 >> 4), idesc_o,
                        j > 0 || part > 0 || kk > 0);
        }
        umma_commit(bar(kBarODone + x));
      }
      __syncwarp();
    };
    bool ok = wait1(kBarQ, 0);
    if (ok && ntiles > 0) {
      ok = wait1(kBarKFull, 0);
      if (ok) {
        issue_s(0, 0);
        issue_s(1, 0);
        if (lane == 0) umma_commit(bar(kBarKEmpty));       // K(0) is read by now
      }
    }
    for (int j = 0; ok && j < ntiles; ++j) {
      const int vs = j % kVst;
      if (!(ok = wait1(kBarVFull + vs, (j / kVst) & 1))) break;
      if ((t_lo + j) * kBN + kBN > L) {
        // V rows at or past the sequence end: zero them so that poisoned or
        // stale slots cannot turn 0 * x into NaN inside the MMA
        const int first = max(0, L - (t_lo + j) * kBN);
        for (int idx = lane; idx < (kBN - first) * 16; idx += 32) {
          const int row = first + idx / 16, ch = idx % 16;
          const uint32_t addr = v_s(vs) + (ch >> 3) * kKvHalf + row * 128 + (ch & 7) * 16;
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      if (!(ok = wait1(kBarPFull + 0, j & 1))) break;
      issue_pv(0, j);
      if (j + 1 < ntiles) {
        if (!(ok = wait1(kBarKFull + (j + 1) % kKst, ((j + 1) / kKst) & 1))) break;
        if (!(ok = wait1(kBarODone + 0, j & 1))) break;   // P_A(j) consumed
        issue_s(0, j + 1);
      }
      if (!(ok = wait1(kBarPFull + 1, j & 1))) break;
      issue_pv(1, j);
      if (lane == 0) umma_commit(bar(kBarVEmpty + vs));     // V(j) is read by now
      if (j + 1 < ntiles) {
        if (!(ok = wait1(kBarODone + 1, j & 1))) break;   // P_B(j) consumed
        issue_s(1, j + 1);
        if (lane == 0) umma_commit(bar(kBarKEmpty + (j + 1) % kKst));   // K(j+1) read
      }
    }
  } else {
    // ------------------------------------------------------------ softmax (tile x_me)
    const int x = x_me;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int pos = !row_valid ? -1 : (cascade ? L - 1 : L - q_len + tok_me);
    for (int j = 0; j < ntiles; ++j) {
      // S_x(j) complete also means PV_x(j-1) is: its MMA waited for that
      if (!mbar_wait_abortable(bar(kBarSFull + x), j & 1, a.timeout_ns, abort)) break;
      tc_fence_after_sync();
      float sv[kBN];
#pragma unroll
      for (int i = 0; i < kBN / 32; ++i) {
        float v[32];
        tmem_ld32(t_s(x) + lane_off + 32 * i, v);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[32 * i + e] = v[e];
      }
      tmem_wait_ld();

      // the row max of scale * s (log2 units), taken on the raw dot products:
      // the largest for scale >= 0, the smallest otherwise; four independent
      // chains; no per-element mask on a tile that lies wholly inside this
      // row's causal window
      const int t_base = (t_lo + j) * kBN;
      const bool full = t_base + kBN - 1 <= pos;
      const int nvalid = full ? kBN : max(0, pos - t_base + 1);
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (full && a.scale_log2 >= 0.f) {
#pragma unroll
        for (int c = 0; c < kBN; c += 2)
          mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], sv[c], sv[c + 1]);
      } else if (full) {
#pragma unroll
        for (int c = 0; c < kBN; c += 2)
          mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], -sv[c], -sv[c + 1]);
      } else {
        const float sg = a.scale_log2 >= 0.f ? 1.f : -1.f;
#pragma unroll
        for (int c = 0; c < kBN; ++c) mx[c & 3] = fmaxf(mx[c & 3], c < nvalid ? sg * sv[c] : -INFINITY);
      }
      const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      // the exponent base moves only when the tile's max exceeds it by more
      // than 8 (log2 units): p <= 2^8 stays exact enough in 16 bits, O and l
      // share the base, and O / l is unchanged
      const float tmax = rmax == -INFINITY ? -INFINITY : rmax * fabsf(a.scale_log2);
      const float m_new = tmax > m_run + 8.f ? tmax : m_run;
      const float base = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = m_new == m_run ? 1.f : fast_exp2(m_run - base);
      // P = 2^(scale * s - base) over the S columns just read (masked
      // columns 0), pairs in packed f32x2 arithmetic: 32 tokens per
      // 16-column store
      const uint64_t sc2 = f2splat(a.scale_log2), nb2 = f2splat(-base);
      uint64_t ps2[2] = {f2splat(0.f), f2splat(0.f)};
#pragma unroll
      for (int c32 = 0; c32 < kBN / 32; ++c32) {
        uint32_t hw[16], lw[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 32 * c32 + 2 * e;
          const uint64_t x2 = f2fma(f2pack(sv[c], sv[c + 1]), sc2, nb2);
          const float2 xx = f2unpack(x2);
          float2 p = make_float2(fast_exp2(xx.x), fast_exp2(xx.y));
          if (!full) {
            p.x = c < nvalid ? p.x : 0.f;
            p.y = c + 1 < nvalid ? p.y : 0.f;
          }
          ps2[e & 1] = f2add(ps2[e & 1], f2pack(p.x, p.y));
          hw[e] = pack2<QT>(p.x, p.y);
          if constexpr (PARTS == 2) {
            const float2 f = unpack2<QT>(hw[e]);
            lw[e] = pack2<QT>(p.x - f.x, p.y - f.y);
          }
        }
        tmem_st16(t_s(x) + lane_off + 16 * c32, hw);
        if constexpr (PARTS == 2) tmem_st16(t_s(x) + lane_off + 64 + 16 * c32, lw);
      }
      const float2 s0 = f2unpack(ps2[0]), s1 = f2unpack(ps2[1]);
      l_run = l_run * alpha + ((s0.x + s0.y) + (s1.x + s1.y));
      m_run = m_new;
      if (j > 0 && __any_sync(FULL, alpha != 1.f)) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v[32];
          tmem_ld32(t_o(x) + lane_off + 32 * i, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= alpha;
          tmem_st32(t_o(x) + lane_off + 32 * i, v);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(bar(kBarPFull + x));
    }
    if (ntiles > 0)
      mbar_wait_abortable(bar(kBarODone + x), (ntiles - 1) & 1, a.timeout_ns, abort);
  }

  tc_fence_before_sync();
  __syncthreads();                           // every role is done issuing and waiting
  if (*abort && lane == 0) {
    if (warp == kTmaWarp) {                  // let the copies in flight land
      for (int st = 0; st < kKst; ++st)
        if (armed_k[st] >= 0)
          mbar_wait_bounded(bar(kBarKFull + st), (armed_k[st] / kKst) & 1, kDrainLimitNs);
      for (int st = 0; st < kVst; ++st)
        if (armed_v[st] >= 0)
          mbar_wait_bounded(bar(kBarVFull + st), (armed_v[st] / kVst) & 1, kDrainLimitNs);
    } else if (warp == kMmaWarp) {           // let the MMAs in flight finish
      report_error(a.err_flag, kErrTimeout);
      umma_commit(bar(kBarDrain));
      mbar_wait_bounded(bar(kBarDrain), 0, kDrainLimitNs);
    }
  }
  __syncthreads();                           // drains done
  tc_fence_after_sync();
  const bool dead = *abort;
  const bool empty = ntiles == 0;            // an empty split: m = -inf, l = 0, o = 0
  if (warp < 8) {
    // ---- epilogue: out row = O / l (cascade: the partial o / l, m, l)
    const int x = x_me;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float inv = (!dead && l_run > 0.f) ? 1.f / l_run : 0.f;
    const int h = kvh * G + row_me % G;
    const size_t orow_idx = static_cast<size_t>(q0 + tok_me) * a.num_heads + h;
    const size_t split_rows = cascade ? static_cast<size_t>(seq) * q_len * a.num_heads : 0;
    if (cascade && row_valid) {
      a.part_m[split_rows + orow_idx] = (dead || empty) ? -INFINITY : m_run;
      a.part_l[split_rows + orow_idx] = (dead || empty) ? 0.f : l_run;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v[32];
      tmem_ld32(t_o(x) + lane_off + 32 * i, v);
      tmem_wait_ld();
      if (!row_valid) continue;
      if (dead || empty) {                   // TMEM may hold anything: write plain zeros
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.f;
      }
      if (cascade) {
        float4* dst = reinterpret_cast<float4*>(a.part_o + (split_rows + orow_idx) * kD + 32 * i);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(v[4 * e] * inv, v[4 * e + 1] * inv, v[4 * e + 2] * inv,
                               v[4 * e + 3] * inv);
      } else {
        QT* orow = reinterpret_cast<QT*>(a.out) + orow_idx * kD + 32 * i;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w;
          w.x = pack2<QT>(v[e] * inv, v[e + 1] * inv);
          w.y = pack2<QT>(v[e + 2] * inv, v[e + 3] * inv);
          w.z = pack2<QT>(v[e + 4] * inv, v[e + 5] * inv);
          w.w = pack2<QT>(v[e + 6] * inv, v[e + 7] * inv);
          *reinterpret_cast<uint4*>(orow + e) = w;
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
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
cudaError_t launch_t(const PrefillArgs& a, int total_q, int max_query_len, cudaStream_t stream,
                     bool allow_pdl) {
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
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int rows_per_cta = kQTiles * (kRows / G);
  const dim3 grid((max_query_len + rows_per_cta - 1) / rows_per_cta, a.num_kv_heads,
                  a.cascade_rows > 0 ? max(1, a.cascade_splits) : a.num_seqs);
  return launch_kernel(kern, grid, dim3(kThreads), kSmemBytes, stream,
                       allow_pdl && pdl_mode() != 0, mq, mk, mv, a);
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs& a, int q_dtype, int block_size, int total_q,
                           int max_query_len, cudaStream_t stream, bool allow_pdl) {
  const bool bf = q_dtype == PA_BF16;
  switch (block_size) {
    case 8: return bf ? launch_t<__nv_bfloat16, 8>(a, total_q, max_query_len, stream, allow_pdl)
                      : launch_t<__half, 8>(a, total_q, max_query_len, stream, allow_pdl);
    case 16: return bf ? launch_t<__nv_bfloat16, 16>(a, total_q, max_query_len, stream, allow_pdl)
                       : launch_t<__half, 16>(a, total_q, max_query_len, stream, allow_pdl);
    case 32: return bf ? launch_t<__nv_bfloat16, 32>(a, total_q, max_query_len, stream, allow_pdl)
                       : launch_t<__half, 32>(a, total_q, max_query_len, stream, allow_pdl);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pa
