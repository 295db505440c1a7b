// pa_decode.cu -- paged decode attention kernels for sm_100a: the per-partition
// kernel behind pa_decode_v1 / pa_decode_v2_partition, the fp32 CUDA-core
// kernel, and the v2 merge.
//
// What is computed ([深度解析] = "LLM推理优化：vLLM PagedAttention深度解析与工程实践",
// [vllm-musa] = "KV Cache 与 PagedAttention（vllm-musa 实战）"):
//   out[s,h,:] = sum_t softmax_t(scale * q[s,h,:] . K_t) V_t        ([深度解析] §二)
// over the cached tokens of sequence s, K_t/V_t fetched through the block table
// ([vllm-musa] §五, [深度解析] §3.1), either in one pass per (sequence, kv head)
// (paged_attention_v1) or as split-K partitions merged by log-sum-exp
// (paged_attention_v2, [深度解析] §4.1).
//
// How (B200 design, not the pages' MUSA sketch):
// * one CTA per (partition, kv head, sequence); its warps take the CTA's
//   16-token tiles round-robin, each warp with its own ring of shared-memory
//   stages fed by TMA (3-D tensor maps over the cache, 128B/64B swizzle; a tile
//   is one box of 16 tokens, or two boxes for 8-token blocks) and completed on
//   per-stage mbarriers; block ids come from the table a window of 32 tiles
//   ahead, held in registers.
// * as soon as a stage lands the warp copies its K and V fragments into
//   registers and refills the stage; the tile math (pa_tile.cuh) runs on
//   mma.sync with the GQA group as N, online softmax in the log2 domain.
// * the warps of a CTA merge through shared memory at the end.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"
#include "pa_write.cuh"

namespace pa {

__device__ int g_pa_device_error = 0;

// A v2 partition of a sequence whose seq_len failed the bounds check: written
// as empty (m = -inf, l = 0, o = 0) so the merge skips it and outputs zeros.
__device__ __forceinline__ void write_empty_partial(const DecodeArgs& a, int seq, int kvh,
                                                    int part, int G, int D) {
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, d = idx % D;
    const size_t row =
        (static_cast<size_t>(seq) * a.num_heads + kvh * G + g) * a.max_parts + part;
    a.tmp_out[row * D + d] = 0.f;
    if (d == 0) {
      a.max_logits[row] = -INFINITY;
      a.exp_sums[row] = 0.f;
    }
  }
}

// 8-bit caches: at most 128 registers, so two CTAs of up to 8 warps fit an SM
// (the 8-bit path is issue- and latency-bound: more resident warps help).
template <typename QT, int KIND, int D, int BS>
__global__ void __launch_bounds__(kMaxWarps * 32, KIND == kKind16 ? 0 : 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ DecodeArgs a) {
  using T = Tr<KIND, D, BS>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[kMaxWarps * kMaxStages];
  __shared__ int stage_ok[kMaxWarps * kMaxStages];

  const int part = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int r = lane >> 2, c = lane & 3;
  const int G = a.num_heads / a.num_kv_heads;
  const int S = a.stages;
  const bool check = a.err_flag != nullptr;
  const bool v1 = a.partition_size == 0;
  constexpr uint32_t FULL = 0xffffffffu;

  griddep_launch_dependents();
  // mode 2 first reads lens / tables; mode 3 (cascade suffix) waits only for the
  // prior partial its epilogue merges
  if (a.pdl != 2 && a.pdl != 3) griddep_wait();

  int len = a.seq_lens[seq];
  if (check) {
    const long long cap = static_cast<long long>(a.max_blocks) * BS;
    if (len < 0 || len > cap) {
      if (threadIdx.x == 0) report_error(a.err_flag, kErrSeqLen);
      len = 0;                                    // skip the sequence: its output is zeros
      if (!v1) {
        griddep_wait();
        write_empty_partial(a, seq, kvh, part, G, D);
        return;
      }
    }
  }
  int t_begin = v1 ? min(a.t_offset, len) : 0, t_end = len;
  if (!v1) {
    t_begin = part * a.partition_size;
    t_end = min(len, t_begin + a.partition_size);
    if (t_begin >= t_end) return;                 // empty partition: nothing to write
  }

  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  const uint32_t wbase = sbase + static_cast<uint32_t>(warp * S * T::STAGE);
  const uint32_t bar0 = smem_u32(&bars[warp * kMaxStages]);
  int* ok_slot = &stage_ok[warp * kMaxStages];

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  __syncwarp();

  const int ntok = t_end - t_begin;
  const int ntiles = (ntok + 15) / 16;
  const int nmine = ntiles > warp ? (ntiles - warp + nwarps - 1) / nwarps : 0;
  const int nblk_seq = (len + BS - 1) / BS;
  const int32_t* table = a.block_tables + static_cast<size_t>(seq) * a.max_blocks;
  constexpr int kBeyond = INT_MIN;

  // Block ids of this warp's tiles, 32 tiles per window, one tile per lane.
  int ids_cur[T::NBOX], ids_nxt[T::NBOX];
  auto load_window = [&](int wdx, int (&ids)[T::NBOX]) {
    const int i = wdx * 32 + lane;
    const int t0 = t_begin + 16 * (warp + i * nwarps);
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) {
      const int lb = (t0 + b * T::BOXH) / BS;
      ids[b] = (i < nmine && lb < nblk_seq) ? __ldg(table + lb) : kBeyond;
    }
  };
#pragma unroll
  for (int b = 0; b < T::NBOX; ++b) ids_cur[b] = ids_nxt[b] = kBeyond;
  if (nmine > 0) load_window(0, ids_cur);
  if (nmine > 32) load_window(1, ids_nxt);
  int win_cur = 0;
  uint32_t armed = 0;                             // stages with a completion pending

  // PDL mode 2: fetch this warp's first tiles into L2 while the preceding grid
  // finishes (lane i prefetches tile i of window 0)
  if (a.pdl == 2 && lane < min(a.prefetch, nmine)) {
    const int ob = BS > 16 ? (t_begin + 16 * (warp + lane * nwarps)) % BS : 0;
    prefetch_tile<KIND, D, BS>(&tm_k, &tm_v, a.k_scale, a.v_scale, a.num_kv_heads, a.num_blocks,
                               kvh, ids_cur, ob);
  }

  const uint64_t pol = policy_evict_first();

  // Issue the loads of this warp's i-th tile into stage s (whole warp calls).
  auto issue = [&](int i, int s) {
    const int wdx = i >> 5;
    if (wdx != win_cur) {
#pragma unroll
      for (int b = 0; b < T::NBOX; ++b) ids_cur[b] = ids_nxt[b];
      win_cur = wdx;
      if ((wdx + 1) * 32 < nmine) load_window(wdx + 1, ids_nxt);
    }
    int blk[T::NBOX];
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) blk[b] = __shfl_sync(FULL, ids_cur[b], i & 31);
    if (a.inject == 1 && i == 0) return;          // test hook: this stage never arrives
    armed |= 1u << s;
    if (lane == 0) {
      const uint32_t st = wbase + static_cast<uint32_t>(s * T::STAGE);
      const uint32_t bar = bar0 + 8u * s;
      const int ob = BS > 16 ? (t_begin + 16 * (warp + i * nwarps)) % BS : 0;
      int okm = 0;
#pragma unroll
      for (int b = 0; b < T::NBOX; ++b) {
        if (blk[b] == kBeyond) continue;
        if (check && (blk[b] < 0 || blk[b] >= a.num_blocks)) {
          report_error(a.err_flag, kErrBlockId);
          continue;
        }
        okm |= 1 << b;
      }
      ok_slot[s] = okm;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, tile_bytes<KIND, D, BS>(okm));
      issue_tile_copies<KIND, D, BS>(st, bar, &tm_k, &tm_v, a.k_scale, a.v_scale,
                                     a.num_kv_heads, kvh, blk, okm, ob, pol);
    }
  };

  if (a.pdl == 2) griddep_wait();                 // q and the caches may come from it

  // With a fused cache write, this CTA's range ends at the sequence's last
  // token, and the warp owning that tile writes the token before it loads the
  // tile: its prologue copy of that tile (if any) waits for the write.
  const bool writes = a.new_k != nullptr && t_end == len && ntok > 0;
  const int w_last = writes ? (ntiles - 1) % nwarps : -1;
  const int i_last = writes ? (ntiles - 1) / nwarps : -1;
  const bool writer = warp == w_last;

  const int npro = min(S, nmine);
  for (int i = 0; i < npro; ++i)
    if (!(writer && i == i_last)) issue(i, i);
  if (writer) {
    const int64_t slot = a.new_slots[seq];
    // debug mode: the slot must be where the table puts token len - 1 (a slot in an
    // earlier tile would be written while another warp may be loading that tile)
    bool slot_ok = slot >= 0 && slot < static_cast<int64_t>(a.num_blocks) * BS;
    if (check && slot >= 0) {
      const int64_t want = static_cast<int64_t>(table[(len - 1) / BS]) * BS + (len - 1) % BS;
      slot_ok = slot_ok && slot == want;
    }
    if (slot_ok) {
      constexpr int MODE = KIND == kKind16 ? kWriteCopy : (KIND == kKindI8 ? kWriteInt8 : kWriteFp8);
      const int64_t blk = slot / BS;
      const int off = static_cast<int>(slot % BS);
      const size_t src_row = (static_cast<size_t>(seq) * a.num_kv_heads + kvh) * D;
      const size_t dst_row = ((static_cast<size_t>(blk) * BS + off) * a.num_kv_heads + kvh) * D;
      const size_t sidx = (static_cast<size_t>(blk) * a.num_kv_heads + kvh) * BS + off;
      write_kv_row<QT, MODE, D>(static_cast<const QT*>(a.new_k) + src_row, a.wk_cache, dst_row,
                                MODE ? a.wk_scale + sidx : nullptr, lane);
      write_kv_row<QT, MODE, D>(static_cast<const QT*>(a.new_v) + src_row, a.wv_cache, dst_row,
                                MODE ? a.wv_scale + sidx : nullptr, lane);
      fence_proxy_async_global();
    } else if (slot >= 0 && lane == 0) {
      report_error(a.err_flag, kErrSlot);         // past the pool or off the table: nothing written
    }
    __syncwarp();
    if (i_last < npro) issue(i_last, i_last);
  }

  WarpAttn<QT, KIND, D, BS> wa;
  wa.reset();
  wa.load_q_global(reinterpret_cast<const QT*>(a.q) +
                       (static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G + r) * D,
                   r < G, c);

  int si = 0;
  uint32_t ph = 0;
  bool dead = false;
  for (int i = 0; i < nmine; ++i) {
    const uint32_t st = wbase + static_cast<uint32_t>(si * T::STAGE);
    const bool arrived = __all_sync(FULL, mbar_wait_bounded(bar0 + 8u * si, ph, a.timeout_ns));
    if (!arrived) {
      // Stop consuming; let every copy this warp still has in flight land (each
      // wait again bounded), so none targets shared memory after the CTA exits.
      for (int k = 0; k < S; ++k) {
        const int s2 = (si + k) % S;
        if ((armed >> s2) & 1u)
          mbar_wait_bounded(bar0 + 8u * s2, ph ^ ((si + k) >= S ? 1u : 0u), kDrainLimitNs);
      }
      dead = true;
      break;
    }
    armed &= ~(1u << si);
    const int j = warp + i * nwarps;
    const int nv = min(16, ntok - j * 16);
    const int okm = ok_slot[si];
    TileFrag<KIND, D, BS> fr;
    load_tile<QT, KIND, D, BS>(fr, st, lane);
    __syncwarp();
    if (i + S < nmine) issue(i + S, si);          // refill the stage right away
    tile_compute<QT, KIND, D, BS>(wa, fr, nv, okm, a.scale_log2, lane);
    if (++si == S) {
      si = 0;
      ph ^= 1u;
    }
  }

  if (dead) {
    if (lane == 0) report_error(a.err_flag, kErrTimeout);
    wa.reset();
  } else {
    wa.finish();
  }

  // ---- merge the warps of the CTA through shared memory
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    wa.lsum[0] += __shfl_xor_sync(FULL, wa.lsum[0], off);
    wa.lsum[1] += __shfl_xor_sync(FULL, wa.lsum[1], off);
  }
  __syncthreads();   // every warp is done with its stages
  constexpr int OP = D + 4;
  float* ored = reinterpret_cast<float*>(smem_raw + (sbase - sraw));
  float* mred = ored + nwarps * 8 * OP;
  float* lred = mred + nwarps * 8;
#pragma unroll
  for (int mt = 0; mt < T::NMT; ++mt) {
    const int d0 = out_dim<KIND>(mt, r, 0), d1 = out_dim<KIND>(mt, r, 1);
    float* o0 = ored + (warp * 8 + 2 * c) * OP;
    float* o1 = o0 + OP;
    o0[d0] = wa.oacc[mt][0];
    o1[d0] = wa.oacc[mt][1];
    o0[d1] = wa.oacc[mt][2];
    o1[d1] = wa.oacc[mt][3];
  }
  if (r == 0) {
    mred[warp * 8 + 2 * c] = wa.m2[0];
    mred[warp * 8 + 2 * c + 1] = wa.m2[1];
    lred[warp * 8 + 2 * c] = wa.lsum[0];
    lred[warp * 8 + 2 * c + 1] = wa.lsum[1];
  }
  __syncthreads();

  constexpr int NCH = D / 8;
  if (a.prior_o != nullptr && a.pdl == 3) griddep_wait();   // the prior partial's producer
  for (int idx = threadIdx.x; idx < G * NCH; idx += blockDim.x) {
    const int g = idx / NCH, d0 = (idx % NCH) * 8;
    float M = -INFINITY;
    for (int w = 0; w < nwarps; ++w) M = fmaxf(M, mred[w * 8 + g]);
    float L = 0.f;
    float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (M != -INFINITY) {
      for (int w = 0; w < nwarps; ++w) {
        const float f = fast_exp2(mred[w * 8 + g] - M);
        L += lred[w * 8 + g] * f;
        const float* src = ored + (w * 8 + g) * OP + d0;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] += src[e] * f;
      }
    }
    const int h = kvh * G + g;
    if (v1 && a.prior_o != nullptr) {
      // merge the prior partials (o_p / l_p, m_p, l_p) by log-sum-exp
      const size_t rows = static_cast<size_t>(a.num_seqs) * a.num_heads;
      const size_t pr = static_cast<size_t>(seq) * a.num_heads + h;
      for (int k = 0; k < a.prior_splits; ++k) {
        const float mp = a.prior_m[k * rows + pr], lp = a.prior_l[k * rows + pr];
        if (mp == -INFINITY) continue;         // an empty split
        const float M2 = fmaxf(M, mp);
        const float f1 = M == -INFINITY ? 0.f : fast_exp2(M - M2);
        const float f2 = fast_exp2(mp - M2) * lp;
        const float4* op = reinterpret_cast<const float4*>(a.prior_o + (k * rows + pr) * D + d0);
        const float4 p0 = op[0], p1 = op[1];
        const float pv[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = o[e] * f1 + pv[e] * f2;
        L = L * f1 + f2;
        M = M2;
      }
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    if (v1) {
      uint4 pk;
      pk.x = pack2<QT>(o[0] * inv, o[1] * inv);
      pk.y = pack2<QT>(o[2] * inv, o[3] * inv);
      pk.z = pack2<QT>(o[4] * inv, o[5] * inv);
      pk.w = pack2<QT>(o[6] * inv, o[7] * inv);
      *reinterpret_cast<uint4*>(reinterpret_cast<QT*>(a.out) +
                                (static_cast<size_t>(seq) * a.num_heads + h) * D + d0) = pk;
    } else {
      const size_t row = (static_cast<size_t>(seq) * a.num_heads + h) * a.max_parts + part;
      float4* dst = reinterpret_cast<float4*>(a.tmp_out + row * D + d0);
      dst[0] = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
      dst[1] = make_float4(o[4] * inv, o[5] * inv, o[6] * inv, o[7] * inv);
      if (d0 == 0) {
        a.max_logits[row] = M == -INFINITY ? -INFINITY : M * 0.69314718055994530942f;
        a.exp_sums[row] = L;
      }
    }
  }
}

// --------------------------------------------------------------------------
// fp32 caches: CUDA-core kernel (tensor cores would round to tf32).  One warp
// per token at a time; lanes split head_dim; the same CTA grid and merge as above.
// --------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kMaxWarps * 32)
    decode_f32_kernel(const __grid_constant__ DecodeArgs a, int BS) {
  constexpr int NE = D / 32;
  constexpr uint32_t FULL = 0xffffffffu;
  __shared__ float ored[kMaxWarps * kMaxGroup * D];
  __shared__ float mred[kMaxWarps * kMaxGroup], lred[kMaxWarps * kMaxGroup];

  const int part = blockIdx.x, kvh = blockIdx.y, seq = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int G = a.num_heads / a.num_kv_heads;
  const bool check = a.err_flag != nullptr;
  const bool v1 = a.partition_size == 0;

  griddep_launch_dependents();
  griddep_wait();

  int len = a.seq_lens[seq];
  if (check) {
    const long long cap = static_cast<long long>(a.max_blocks) * BS;
    if (len < 0 || len > cap) {
      if (threadIdx.x == 0) report_error(a.err_flag, kErrSeqLen);
      len = 0;                                    // skip the sequence: its output is zeros
      if (!v1) {
        write_empty_partial(a, seq, kvh, part, G, D);
        return;
      }
    }
  }
  int t_begin = 0, t_end = len;
  if (!v1) {
    t_begin = part * a.partition_size;
    t_end = min(len, t_begin + a.partition_size);
    if (t_begin >= t_end) return;
  }
  const int32_t* table = a.block_tables + static_cast<size_t>(seq) * a.max_blocks;
  const float* kc = reinterpret_cast<const float*>(a.k_cache);
  const float* vc = reinterpret_cast<const float*>(a.v_cache);
  const float* qb = reinterpret_cast<const float*>(a.q) +
                    (static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G) * D;

  float qv[kMaxGroup][NE], acc[kMaxGroup][NE], m2[kMaxGroup], ls[kMaxGroup];
#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) {
    m2[g] = -INFINITY;
    ls[g] = 0.f;
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      qv[g][e] = g < G ? qb[g * D + lane + 32 * e] * a.scale_log2 : 0.f;
      acc[g][e] = 0.f;
    }
  }

  for (int t = t_begin + warp; t < t_end; t += nwarps) {
    const int blk = table[t / BS];
    if (check && (blk < 0 || blk >= a.num_blocks)) {
      if (lane == 0) report_error(a.err_flag, kErrBlockId);
      continue;
    }
    const size_t row = ((static_cast<size_t>(blk) * BS + t % BS) * a.num_kv_heads + kvh) * D;
    float kk[NE], vv[NE];
#pragma unroll
    for (int e = 0; e < NE; ++e) {
      kk[e] = kc[row + lane + 32 * e];
      vv[e] = vc[row + lane + 32 * e];
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
      if (g >= G) break;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < NE; ++e) dot = fmaf(qv[g][e], kk[e], dot);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(FULL, dot, off);
      const float mn = fmaxf(m2[g], dot);
      const float al = fast_exp2(m2[g] - mn);
      const float p = fast_exp2(dot - mn);
      ls[g] = ls[g] * al + p;
#pragma unroll
      for (int e = 0; e < NE; ++e) acc[g][e] = fmaf(p, vv[e], acc[g][e] * al);
      m2[g] = mn;
    }
  }

#pragma unroll
  for (int g = 0; g < kMaxGroup; ++g) {
    if (g >= G) break;
#pragma unroll
    for (int e = 0; e < NE; ++e) ored[(warp * kMaxGroup + g) * D + lane + 32 * e] = acc[g][e];
    if (lane == 0) {
      mred[warp * kMaxGroup + g] = m2[g];
      lred[warp * kMaxGroup + g] = ls[g];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, d = idx % D;
    float M = -INFINITY;
    for (int w = 0; w < nwarps; ++w) M = fmaxf(M, mred[w * kMaxGroup + g]);
    float L = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < nwarps; ++w) {
        const float f = fast_exp2(mred[w * kMaxGroup + g] - M);
        L += lred[w * kMaxGroup + g] * f;
        o += ored[(w * kMaxGroup + g) * D + d] * f;
      }
    }
    const float val = L > 0.f ? o / L : 0.f;
    const int h = kvh * G + g;
    if (v1) {
      reinterpret_cast<float*>(a.out)[(static_cast<size_t>(seq) * a.num_heads + h) * D + d] = val;
    } else {
      const size_t row = (static_cast<size_t>(seq) * a.num_heads + h) * a.max_parts + part;
      a.tmp_out[row * D + d] = val;
      if (d == 0) {
        a.max_logits[row] = M == -INFINITY ? -INFINITY : M * 0.69314718055994530942f;
        a.exp_sums[row] = L;
      }
    }
  }
}

// --------------------------------------------------------------------------
// v2 merge: per (head, sequence), M = max_p m_p, w_p = l_p e^{m_p - M},
// out = sum_p w_p o_p / sum_p w_p over the sequence's partitions (l_p = 0 skipped).
// One CTA (4 warps) per (head, sequence): the CTA reduces M, then each warp streams
// every 4th partition row (one float4 per lane, two rows a step for head_dim 64)
// with four rows in flight, and the warps' sums meet in shared memory.
// --------------------------------------------------------------------------
constexpr int kMergeThreads = 128;

template <typename OT>
__global__ void __launch_bounds__(kMergeThreads)
    merge_kernel(OT* __restrict__ out, const float* __restrict__ tmp,
                 const float* __restrict__ ml, const float* __restrict__ es,
                 const int32_t* __restrict__ seq_lens, int num_heads, int D, int P, int maxp) {
  constexpr uint32_t FULL = 0xffffffffu;
  constexpr float kLog2e = 1.4426950408889634f;
  __shared__ float red[kMergeThreads / 32];
  __shared__ float4 osum[8][32];             // (row group, float4 column)
  __shared__ float wsum[8];
  const int h = blockIdx.x, s = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  griddep_launch_dependents();
  griddep_wait();
  const int len = seq_lens[s];
  int np = len > 0 ? (len + P - 1) / P : 0;
  np = min(np, maxp);
  const size_t base = (static_cast<size_t>(s) * num_heads + h) * maxp;
  float M = -INFINITY;
  for (int p = threadIdx.x; p < np; p += kMergeThreads)
    if (es[base + p] > 0.f) M = fmaxf(M, ml[base + p]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
  if (lane == 0) red[warp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));

  const int L4 = D / 4;                      // float4 columns of a row: 32 or 16
  const int rows = 32 / L4;                  // rows a warp takes per step: 1 or 2
  const int c4 = lane % L4, grp = warp * rows + lane / L4;
  const int ngrp = (kMergeThreads / 32) * rows;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
  if (M != -INFINITY) {
    const float4* t4 = reinterpret_cast<const float4*>(tmp + base * D) + c4;   // row p: t4[p * L4]
    auto add = [&](float l, float m, const float4& v) {
      if (!(l > 0.f)) return;
      const float w = l * fast_exp2((m - M) * kLog2e);
      W += w;
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    };
    int p = grp;
    for (; p + 3 * ngrp < np; p += 4 * ngrp) {
      float l[4], m[4];
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int q = p + u * ngrp;
        l[u] = es[base + q];
        m[u] = ml[base + q];
        v[u] = t4[static_cast<size_t>(q) * L4];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) add(l[u], m[u], v[u]);
    }
    for (; p < np; p += ngrp) add(es[base + p], ml[base + p], t4[static_cast<size_t>(p) * L4]);
  }
  osum[grp][c4] = acc;
  if (c4 == 0) wsum[grp] = W;
  __syncthreads();
  if (threadIdx.x < L4) {
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float Wt = 0.f;
    for (int g = 0; g < ngrp; ++g) {
      const float4 x = osum[g][threadIdx.x];
      o.x += x.x;
      o.y += x.y;
      o.z += x.z;
      o.w += x.w;
      Wt += wsum[g];
    }
    const float v[4] = {Wt > 0.f ? o.x / Wt : 0.f, Wt > 0.f ? o.y / Wt : 0.f,
                        Wt > 0.f ? o.z / Wt : 0.f, Wt > 0.f ? o.w / Wt : 0.f};
    OT* dst = out + (static_cast<size_t>(s) * num_heads + h) * D + 4 * threadIdx.x;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if constexpr (std::is_same<OT, float>::value) dst[e] = v[e];
      else if constexpr (std::is_same<OT, __half>::value) dst[e] = __float2half_rn(v[e]);
      else dst[e] = __float2bfloat16_rn(v[e]);
    }
  }
}

// --------------------------------------------------------------------------
// Merge of stacked partials (the cascade: the shared prefix's splits and the
// sequence's own tokens): per (sequence, head) row, partial k has o_k = O_k / l_k,
// m_k (log2 units) and l_k; out = sum_k l_k 2^{m_k - M} o_k / sum_k l_k 2^{m_k - M},
// M = max_k m_k, partials with l_k = 0 skipped.  One warp per row, 4 dims a lane;
// all of a row's (l, m) and then all its o loads are issued before any is used.
// --------------------------------------------------------------------------
constexpr int kMaxMergeParts = 8;

template <typename OT>
__global__ void __launch_bounds__(128)
    merge_partials_kernel(OT* __restrict__ out, const float* __restrict__ po,
                          const float* __restrict__ pm, const float* __restrict__ pl, int nparts,
                          long long rows, int D) {
  griddep_launch_dependents();
  griddep_wait();
  const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  // every partial's (l, m) first, then every o row: two rounds of loads, not 3 per partial
  float l[kMaxMergeParts], m[kMaxMergeParts];
#pragma unroll
  for (int k = 0; k < kMaxMergeParts; ++k) {
    l[k] = k < nparts ? pl[k * rows + row] : 0.f;
    m[k] = k < nparts ? pm[k * rows + row] : -INFINITY;
  }
  float M = -INFINITY;
#pragma unroll
  for (int k = 0; k < kMaxMergeParts; ++k)
    if (l[k] > 0.f) M = fmaxf(M, m[k]);
  float w[kMaxMergeParts];
#pragma unroll
  for (int k = 0; k < kMaxMergeParts; ++k)
    w[k] = (l[k] > 0.f && M != -INFINITY) ? l[k] * fast_exp2(m[k] - M) : 0.f;
  for (int d = 4 * lane; d < D; d += 128) {
    float4 v[kMaxMergeParts];
#pragma unroll
    for (int k = 0; k < kMaxMergeParts; ++k)
      v[k] = w[k] > 0.f ? *reinterpret_cast<const float4*>(po + (k * rows + row) * D + d)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kMaxMergeParts; ++k) {
      if (!(w[k] > 0.f)) continue;
      W += w[k];
      o.x = fmaf(w[k], v[k].x, o.x);
      o.y = fmaf(w[k], v[k].y, o.y);
      o.z = fmaf(w[k], v[k].z, o.z);
      o.w = fmaf(w[k], v[k].w, o.w);
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    OT* dst = out + row * D + d;
    dst[0] = static_cast<OT>(o.x * inv);
    dst[1] = static_cast<OT>(o.y * inv);
    dst[2] = static_cast<OT>(o.z * inv);
    dst[3] = static_cast<OT>(o.w * inv);
  }
}

// --------------------------------------------------------------------------
// Host side: tensor maps and launches.
// --------------------------------------------------------------------------
namespace {

template <typename QT, int KIND, int D, int BS>
cudaError_t launch_tc(const DecodeArgs& a, const DecodeShape& sh, cudaStream_t stream) {
  using T = Tr<KIND, D, BS>;
  CUtensorMap mk, mv;
  cudaError_t e = make_cache_map<KIND, D, BS>(&mk, a.k_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  e = make_cache_map<KIND, D, BS>(&mv, a.v_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  const int ring = sh.warps * a.stages * T::STAGE;
  const int epi = sh.warps * 8 * (D + 4) * 4 + sh.warps * 16 * 4;   // the warps' merge
  const int smem = (ring > epi ? ring : epi) + 1024;
  auto kern = decode_tc_kernel<QT, KIND, D, BS>;
  static int configured[64] = {0};
  e = opt_in_smem(reinterpret_cast<const void*>(kern), smem, configured);
  if (e != cudaSuccess) return e;
  dim3 grid(sh.grid_x, a.num_kv_heads, a.num_seqs);
  return launch_kernel(kern, grid, dim3(sh.warps * 32), smem, stream, a.pdl != 0, mk, mv, a);
}

template <typename QT, int KIND>
cudaError_t dispatch_shape(const DecodeArgs& a, const DecodeShape& sh, cudaStream_t s) {
  const int D = sh.head_dim, BS = sh.block_size;
#define PA_CASE(DD, BB) \
  if (D == DD && BS == BB) return launch_tc<QT, KIND, DD, BB>(a, sh, s);
  PA_CASE(128, 16)
  PA_CASE(128, 8)
  PA_CASE(128, 32)
  PA_CASE(64, 16)
  PA_CASE(64, 8)
  PA_CASE(64, 32)
#undef PA_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

int default_stages(int cache_dtype, int head_dim, int block_size, int warps, int budget_kb) {
  (void)block_size;
  const int es = (cache_dtype == PA_INT8 || cache_dtype == PA_FP8E4M3) ? 1 : 2;
  const int stage = (2 * 16 * head_dim * es + (es == 1 ? 2 * 16 * 4 : 0) + 1023) / 1024 * 1024;
  int s = (budget_kb * 1024) / (warps * stage);
  if (s < 2) s = 2;
  if (s > kMaxStages) s = kMaxStages;
  return s;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeShape& sh, cudaStream_t s) {
  if (sh.cache_dtype == PA_F32) {
    dim3 grid(sh.grid_x, a.num_kv_heads, a.num_seqs);
    if (sh.head_dim == 128)
      return launch_kernel(decode_f32_kernel<128>, grid, dim3(sh.warps * 32), 0, s, a.pdl != 0, a,
                           sh.block_size);
    return launch_kernel(decode_f32_kernel<64>, grid, dim3(sh.warps * 32), 0, s, a.pdl != 0, a,
                         sh.block_size);
  }
  const bool qh = sh.q_dtype == PA_F16;
  switch (sh.cache_dtype) {
    case PA_F16: return dispatch_shape<__half, kKind16>(a, sh, s);
    case PA_BF16: return dispatch_shape<__nv_bfloat16, kKind16>(a, sh, s);
    case PA_INT8:
      return qh ? dispatch_shape<__half, kKindI8>(a, sh, s)
                : dispatch_shape<__nv_bfloat16, kKindI8>(a, sh, s);
    case PA_FP8E4M3:
      return qh ? dispatch_shape<__half, kKindE4M3>(a, sh, s)
                : dispatch_shape<__nv_bfloat16, kKindE4M3>(a, sh, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge_partials(void* out, int out_dtype, const float* part_o,
                                  const float* part_m, const float* part_l, int nparts,
                                  long long rows, int head_dim, cudaStream_t s) {
  if (nparts < 1 || nparts > kMaxMergeParts) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>((rows + 3) / 4)), block(128);
  const bool pdl = pdl_mode() != 0;
  if (out_dtype == PA_F16)
    return launch_kernel(merge_partials_kernel<__half>, grid, block, 0, s, pdl,
                         static_cast<__half*>(out), part_o, part_m, part_l, nparts, rows, head_dim);
  if (out_dtype == PA_BF16)
    return launch_kernel(merge_partials_kernel<__nv_bfloat16>, grid, block, 0, s, pdl,
                         static_cast<__nv_bfloat16*>(out), part_o, part_m, part_l, nparts, rows,
                         head_dim);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge(void* out, int out_dtype, const float* tmp_out, const float* max_logits,
                         const float* exp_sums, const int32_t* seq_lens, int num_seqs,
                         int num_heads, int head_dim, int partition_size, int max_parts,
                         cudaStream_t s) {
  if (head_dim != 64 && head_dim != 128) return cudaErrorInvalidValue;
  const dim3 grid(num_heads, num_seqs), block(kMergeThreads);
  const bool pdl = pdl_mode() != 0;
  switch (out_dtype) {
    case PA_F32:
      return launch_kernel(merge_kernel<float>, grid, block, 0, s, pdl, static_cast<float*>(out),
                           tmp_out, max_logits, exp_sums, seq_lens, num_heads, head_dim,
                           partition_size, max_parts);
    case PA_F16:
      return launch_kernel(merge_kernel<__half>, grid, block, 0, s, pdl, static_cast<__half*>(out),
                           tmp_out, max_logits, exp_sums, seq_lens, num_heads, head_dim,
                           partition_size, max_parts);
    default:
      return launch_kernel(merge_kernel<__nv_bfloat16>, grid, block, 0, s, pdl,
                           static_cast<__nv_bfloat16*>(out), tmp_out, max_logits, exp_sums,
                           seq_lens, num_heads, head_dim, partition_size, max_parts);
  }
}

}  // namespace pa
