// pa_decode.cu -- paged decode attention kernels for sm_100a.
//
// What is computed ([深度解析] = "LLM推理优化：vLLM PagedAttention深度解析与工程实践",
// [vllm-musa] = "KV Cache 与 PagedAttention（vllm-musa 实战）",
// [KVcache-learning] = "KVcache-learning"):
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
//   registers and refills the stage, so nearly all of shared memory is in
//   flight while the warp computes.
// * the GQA group is the N = 8 side of mma.sync m16n8k16 with tokens as M:
//   S^T = K Q^T (two independent accumulator chains), then P^T is re-laid as
//   the B operand with movmatrix and O^T += V^T P^T, V^T read by ldmatrix.trans.
//   Each K/V byte is read from HBM once for the whole group.
// * P is split into a high and a low half-precision part so the PV product
//   keeps ~16 significant bits; logits, softmax and accumulators are fp32.
// * INT8 / E4M3 caches are widened to the MMA type in registers (exact); the
//   K scale multiplies the logit, the V scale the V values (fp16) or P (bf16).
// * online softmax in the log2 domain with warp-shuffle max reductions; the
//   warps of a CTA merge through shared memory at the end.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

__device__ int g_pa_device_error = 0;

enum { kKind16 = 0, kKindI8 = 1, kKindE4M3 = 2 };

// Limit for the waits that drain in-flight copies after a time-out.
constexpr unsigned long long kDrainLimitNs = 4000000000ull;

template <int KIND, int D, int BS>
struct Tr {
  static constexpr int ES = KIND == kKind16 ? 2 : 1;         // cache element bytes
  static constexpr bool QUANT = KIND != kKind16;
  static constexpr int ROWB = (D * ES >= 128) ? 128 : 64;    // smem row bytes (= swizzle span)
  static constexpr int NDH = D * ES / ROWB;                  // smem rows per token
  static constexpr int NU = ROWB / 64;                       // 64-byte halves per row
  static constexpr int EPC = 16 / ES;                        // elements per 16-byte chunk
  static constexpr int KSPC = EPC / 4;                       // MMA k-steps per chunk
  static constexpr int NKS = D / 16;                         // k-steps of QK^T
  static constexpr int NMT = D / 16;                         // m-tiles of O^T
  static constexpr int BOXH = BS < 16 ? BS : 16;             // tokens per TMA box
  static constexpr int NBOX = 16 / BOXH;                     // boxes (blocks) per 16-token tile
  static constexpr int KTILE = 16 * D * ES;                  // bytes of K (or V) per tile
  static constexpr int SCALES = QUANT ? 2 * 16 * 4 : 0;
  static constexpr int STAGE = (2 * KTILE + SCALES + 1023) / 1024 * 1024;
  static constexpr int BOX_INNER = ROWB / ES;                // TMA box inner extent (elements)
  static constexpr int NKF = NDH * NU;                       // 16-byte K chunks per row per lane
  static constexpr int NVF = ES == 2 ? NMT : NMT / 2;        // ldmatrix.x4 per tile for V
  static_assert(NDH * NU * KSPC == NKS, "k-step bookkeeping");
};

// Token held by MMA row m (0..7) of a 16-token tile.  For 128-byte rows the two
// rows a quarter-warp reads together differ in swizzle phase bit 2, which keeps
// the 16-byte K loads free of bank conflicts.
template <int ROWB>
__device__ __forceinline__ int tau(int m) {
  if constexpr (ROWB == 128) {
    return (m >> 1) | ((m & 1) << 2);
  } else {
    return m;
  }
}

__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// K operand: two 8-bit codes in bits 0..15 -> MMA-type pair.
template <typename QT, int KIND>
__device__ __forceinline__ uint32_t cvt_k_pair(uint32_t w) {
  if constexpr (KIND == kKindI8) {
    if constexpr (std::is_same<QT, __half>::value) return int8x2_to_f16x2(w);
    else return int8x2_to_bf16x2(w);
  } else {
    if constexpr (std::is_same<QT, __half>::value) return e4m3x2_to_f16x2(w);
    else return e4m3x2_to_bf16x2(w);
  }
}

// V operand after ldmatrix.trans of byte pairs: w = {V[ta][d0], V[ta][d1], V[tb][d0], V[tb][d1]};
// which = 0 returns the pair (V[ta][d0], V[tb][d0]), which = 1 the pair for d1.
template <typename QT, int KIND>
__device__ __forceinline__ uint32_t cvt_v_pair(uint32_t w, int which) {
  const uint32_t pair = __byte_perm(w, 0u, which ? 0x0031u : 0x0020u);   // bytes {1,3} or {0,2}
  return cvt_k_pair<QT, KIND>(pair);
}

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

template <typename QT, int KIND, int D, int BS>
__global__ void __launch_bounds__(kMaxWarps * 32)
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
      uint32_t bytes = 0;
#pragma unroll
      for (int b = 0; b < T::NBOX; ++b) {
        if (blk[b] == kBeyond) continue;
        if (check && (blk[b] < 0 || blk[b] >= a.num_blocks)) {
          report_error(a.err_flag, kErrBlockId);
          continue;
        }
        okm |= 1 << b;
        bytes += 2 * T::NDH * T::BOXH * T::ROWB + (T::QUANT ? 2 * T::BOXH * 4 : 0);
      }
      ok_slot[s] = okm;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, bytes);
#pragma unroll
      for (int b = 0; b < T::NBOX; ++b) {
        if (!((okm >> b) & 1)) continue;
        const int row_tok = blk[b] * BS + ob;
#pragma unroll
        for (int dh = 0; dh < T::NDH; ++dh) {
          const uint32_t roff = static_cast<uint32_t>((dh * 16 + b * T::BOXH) * T::ROWB);
          tma_load_3d(st + roff, &tm_k, dh * T::BOX_INNER, kvh, row_tok, bar, pol);
          tma_load_3d(st + T::KTILE + roff, &tm_v, dh * T::BOX_INNER, kvh, row_tok, bar, pol);
        }
        if constexpr (T::QUANT) {
          const size_t so = (static_cast<size_t>(blk[b]) * a.num_kv_heads + kvh) * BS + ob;
          bulk_load(st + 2 * T::KTILE + b * T::BOXH * 4, a.k_scale + so, T::BOXH * 4, bar, pol);
          bulk_load(st + 2 * T::KTILE + 64 + b * T::BOXH * 4, a.v_scale + so, T::BOXH * 4, bar,
                    pol);
        }
      }
    }
  };

  // q of this lane's query head (g = r) as the B operand of S^T = K Q^T, in the
  // k order the K loads below produce.
  uint32_t qf[T::NKS][2];
  {
    const QT* qrow = reinterpret_cast<const QT*>(a.q) +
                     (static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G + r) * D;
#pragma unroll
    for (int ks = 0; ks < T::NKS; ++ks) {
      const int v = ks % T::KSPC, u = (ks / T::KSPC) % T::NU, dh = ks / (T::KSPC * T::NU);
      const int d0 = dh * T::BOX_INNER + (c + 4 * u) * T::EPC + 4 * v;
      uint2 w = make_uint2(0u, 0u);
      if (r < G) w = *reinterpret_cast<const uint2*>(qrow + d0);
      qf[ks][0] = w.x;
      qf[ks][1] = w.y;
    }
  }

  float m2[2] = {-INFINITY, -INFINITY};     // running max, log2 units (g = 2c, 2c+1)
  float lsum[2] = {0.f, 0.f};                // this lane's share of the running sum
  float oacc[T::NMT][4];
#pragma unroll
  for (int mt = 0; mt < T::NMT; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;

  const int npro = min(S, nmine);
  for (int i = 0; i < npro; ++i) issue(i, i);

  // tokens of this lane's rows (QK / softmax) and of its A elements (PV)
  const int tok0 = tau<T::ROWB>(r), tok1 = tok0 + 8;
  const int ta = tau<T::ROWB>(2 * c), tb = tau<T::ROWB>(2 * c + 1);
  const int mi = lane >> 3, jj = lane & 7;
  const int full_ok = (1 << T::NBOX) - 1;

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
    const bool partial = (nv < 16) || (okm != full_ok);

    // ---- stage -> registers
    uint4 kf[T::NKF][2];
#pragma unroll
    for (int dh = 0; dh < T::NDH; ++dh) {
#pragma unroll
      for (int u = 0; u < T::NU; ++u) {
        kf[dh * T::NU + u][0] = lds128(st + swz<T::ROWB>(dh * 16 + tok0, c + 4 * u));
        kf[dh * T::NU + u][1] = lds128(st + swz<T::ROWB>(dh * 16 + tok1, c + 4 * u));
      }
    }
    uint32_t vf[T::NVF][4];
#pragma unroll
    for (int f = 0; f < T::NVF; ++f) {
      if constexpr (KIND == kKind16) {
        const int dh = (f * 16) / T::BOX_INNER;
        const int cl = ((f * 16) % T::BOX_INNER) / 8;
        const int tok = (mi >> 1) * 8 + tau<T::ROWB>(jj);
        ldmatrix_x4_trans(st + T::KTILE + swz<T::ROWB>(dh * 16 + tok, cl + (mi & 1)), vf[f][0],
                          vf[f][1], vf[f][2], vf[f][3]);
      } else {
        const int tok = (mi & 1) * 8 + tau<T::ROWB>(jj);
        ldmatrix_x4_trans(st + T::KTILE + swz<T::ROWB>(tok, 2 * f + (mi >> 1)), vf[f][0],
                          vf[f][1], vf[f][2], vf[f][3]);
      }
    }
    float ks0 = 1.f, ks1 = 1.f, sv0 = 1.f, sv1 = 1.f, sva = 1.f, svb = 1.f, sva8 = 1.f,
          svb8 = 1.f;
    if constexpr (T::QUANT) {
      const uint32_t ksc = st + 2 * T::KTILE, vsc = ksc + 64;
      ks0 = lds_f32(ksc + tok0 * 4);
      ks1 = lds_f32(ksc + tok1 * 4);
      if constexpr (std::is_same<QT, __nv_bfloat16>::value) {
        sv0 = lds_f32(vsc + tok0 * 4);
        sv1 = lds_f32(vsc + tok1 * 4);
      } else {
        sva = lds_f32(vsc + ta * 4);
        svb = lds_f32(vsc + tb * 4);
        sva8 = lds_f32(vsc + (ta + 8) * 4);
        svb8 = lds_f32(vsc + (tb + 8) * 4);
      }
    }
    __syncwarp();
    if (i + S < nmine) issue(i + S, si);          // refill the stage right away

    // ---- S^T = K Q^T
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kc = 0; kc < T::NKF; ++kc) {
      const uint32_t a0[4] = {kf[kc][0].x, kf[kc][0].y, kf[kc][0].z, kf[kc][0].w};
      const uint32_t a1[4] = {kf[kc][1].x, kf[kc][1].y, kf[kc][1].z, kf[kc][1].w};
#pragma unroll
      for (int v = 0; v < T::KSPC; ++v) {
        const int ks = kc * T::KSPC + v;
        uint32_t af[4];
        if constexpr (KIND == kKind16) {
          af[0] = a0[2 * v];
          af[1] = a1[2 * v];
          af[2] = a0[2 * v + 1];
          af[3] = a1[2 * v + 1];
        } else {
          af[0] = cvt_k_pair<QT, KIND>(a0[v]);
          af[1] = cvt_k_pair<QT, KIND>(a1[v]);
          af[2] = cvt_k_pair<QT, KIND>(a0[v] >> 16);
          af[3] = cvt_k_pair<QT, KIND>(a1[v] >> 16);
        }
        if (ks & 1) mma_16816<QT>(acc1, af, qf[ks][0], qf[ks][1]);
        else mma_16816<QT>(acc0, af, qf[ks][0], qf[ks][1]);
      }
    }
    const bool ok0 = tok0 < nv && ((okm >> (tok0 / T::BOXH)) & 1);
    const bool ok1 = tok1 < nv && ((okm >> (tok1 / T::BOXH)) & 1);
    const float s0 = a.scale_log2 * ks0, s1 = a.scale_log2 * ks1;
    float x[4];
    x[0] = ok0 ? (acc0[0] + acc1[0]) * s0 : -INFINITY;
    x[1] = ok0 ? (acc0[1] + acc1[1]) * s0 : -INFINITY;
    x[2] = ok1 ? (acc0[2] + acc1[2]) * s1 : -INFINITY;
    x[3] = ok1 ? (acc0[3] + acc1[3]) * s1 : -INFINITY;

    // ---- online softmax (per query head g = 2c, 2c+1)
    float tm0 = fmaxf(x[0], x[2]), tm1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      tm0 = fmaxf(tm0, __shfl_xor_sync(FULL, tm0, off));
      tm1 = fmaxf(tm1, __shfl_xor_sync(FULL, tm1, off));
    }
    const float mn0 = fmaxf(m2[0], tm0), mn1 = fmaxf(m2[1], tm1);
    const float ms0 = mn0 == -INFINITY ? 0.f : mn0;
    const float ms1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = fast_exp2(m2[0] - ms0), al1 = fast_exp2(m2[1] - ms1);
    m2[0] = mn0;
    m2[1] = mn1;
    float p0 = fast_exp2(x[0] - ms0), p1 = fast_exp2(x[1] - ms1);
    float p2 = fast_exp2(x[2] - ms0), p3 = fast_exp2(x[3] - ms1);
    lsum[0] = lsum[0] * al0 + (p0 + p2);
    lsum[1] = lsum[1] * al1 + (p1 + p3);
    if (__any_sync(FULL, (al0 != 1.f) || (al1 != 1.f))) {
#pragma unroll
      for (int mt = 0; mt < T::NMT; ++mt) {
        oacc[mt][0] *= al0;
        oacc[mt][1] *= al1;
        oacc[mt][2] *= al0;
        oacc[mt][3] *= al1;
      }
    }

    // ---- O^T += V^T P^T
    if constexpr (T::QUANT && std::is_same<QT, __nv_bfloat16>::value) {
      // bf16 keeps fp32's range: fold the V scale into P (fp32) before the split
      p0 = p0 != 0.f ? p0 * sv0 : 0.f;
      p1 = p1 != 0.f ? p1 * sv0 : 0.f;
      p2 = p2 != 0.f ? p2 * sv1 : 0.f;
      p3 = p3 != 0.f ? p3 * sv1 : 0.f;
    }
    const uint32_t h01 = pack2<QT>(p0, p1), h23 = pack2<QT>(p2, p3);
    const float2 f01 = unpack2<QT>(h01), f23 = unpack2<QT>(h23);
    const uint32_t l01 = pack2<QT>(p0 - f01.x, p1 - f01.y);
    const uint32_t l23 = pack2<QT>(p2 - f23.x, p3 - f23.y);
    const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
    const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);

    uint32_t mk01 = ~0u, mk23 = ~0u;
    if (partial) {
      auto valid = [&](int t) { return t < nv && ((okm >> (t / T::BOXH)) & 1); };
      mk01 = (valid(ta) ? 0x0000FFFFu : 0u) | (valid(tb) ? 0xFFFF0000u : 0u);
      mk23 = (valid(ta + 8) ? 0x0000FFFFu : 0u) | (valid(tb + 8) ? 0xFFFF0000u : 0u);
    }
    if constexpr (KIND == kKind16) {
#pragma unroll
      for (int mt = 0; mt < T::NMT; ++mt) {
        uint32_t af[4] = {vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3]};
        if (partial) {
          af[0] &= mk01;
          af[1] &= mk01;
          af[2] &= mk23;
          af[3] &= mk23;
        }
        mma_16816<QT>(oacc[mt], af, bh0, bh1);
        mma_16816<QT>(oacc[mt], af, bl0, bl1);
      }
    } else {
      uint32_t hsA = 0u, hsB = 0u;
      if constexpr (std::is_same<QT, __half>::value) {
        hsA = pack2<__half>(sva, svb);
        hsB = pack2<__half>(sva8, svb8);
      }
#pragma unroll
      for (int f = 0; f < T::NVF; ++f) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int mt = 2 * f + hh;
          uint32_t af[4];
          af[0] = cvt_v_pair<QT, KIND>(vf[f][2 * hh], 0);
          af[1] = cvt_v_pair<QT, KIND>(vf[f][2 * hh], 1);
          af[2] = cvt_v_pair<QT, KIND>(vf[f][2 * hh + 1], 0);
          af[3] = cvt_v_pair<QT, KIND>(vf[f][2 * hh + 1], 1);
          if constexpr (std::is_same<QT, __half>::value) {
            af[0] = hmul2_u32(af[0], hsA);
            af[1] = hmul2_u32(af[1], hsA);
            af[2] = hmul2_u32(af[2], hsB);
            af[3] = hmul2_u32(af[3], hsB);
          }
          if (partial) {
            af[0] &= mk01;
            af[1] &= mk01;
            af[2] &= mk23;
            af[3] &= mk23;
          }
          mma_16816<QT>(oacc[mt], af, bh0, bh1);
          mma_16816<QT>(oacc[mt], af, bl0, bl1);
        }
      }
    }
    if (++si == S) {
      si = 0;
      ph ^= 1u;
    }
  }

  if (dead) {
    if (lane == 0) report_error(a.err_flag, kErrTimeout);
    m2[0] = m2[1] = -INFINITY;
    lsum[0] = lsum[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < T::NMT; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
  }

  // ---- merge the warps of the CTA through shared memory
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    lsum[0] += __shfl_xor_sync(FULL, lsum[0], off);
    lsum[1] += __shfl_xor_sync(FULL, lsum[1], off);
  }
  __syncthreads();   // every warp is done with its stages
  constexpr int OP = D + 4;
  float* ored = reinterpret_cast<float*>(smem_raw + (sbase - sraw));
  float* mred = ored + kMaxWarps * 8 * OP;
  float* lred = mred + kMaxWarps * 8;
#pragma unroll
  for (int mt = 0; mt < T::NMT; ++mt) {
    int d0, d1;
    if constexpr (KIND == kKind16) {
      d0 = mt * 16 + r;
      d1 = d0 + 8;
    } else {
      d0 = mt * 16 + 2 * r;
      d1 = d0 + 1;
    }
    float* o0 = ored + (warp * 8 + 2 * c) * OP;
    float* o1 = o0 + OP;
    o0[d0] = oacc[mt][0];
    o1[d0] = oacc[mt][1];
    o0[d1] = oacc[mt][2];
    o1[d1] = oacc[mt][3];
  }
  if (r == 0) {
    mred[warp * 8 + 2 * c] = m2[0];
    mred[warp * 8 + 2 * c + 1] = m2[1];
    lred[warp * 8 + 2 * c] = lsum[0];
    lred[warp * 8 + 2 * c + 1] = lsum[1];
  }
  __syncthreads();

  constexpr int NCH = D / 8;
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
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int h = kvh * G + g;
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
// out = sum_p w_p o_p / sum_p w_p over the sequence's partitions.
// --------------------------------------------------------------------------
template <typename OT>
__global__ void merge_kernel(OT* __restrict__ out, const float* __restrict__ tmp,
                             const float* __restrict__ ml, const float* __restrict__ es,
                             const int32_t* __restrict__ seq_lens, int num_heads, int D, int P,
                             int maxp) {
  const int h = blockIdx.x, s = blockIdx.y;
  const int len = seq_lens[s];
  int np = len > 0 ? (len + P - 1) / P : 0;
  np = min(np, maxp);
  const size_t base = (static_cast<size_t>(s) * num_heads + h) * maxp;
  float M = -INFINITY;
  for (int p = 0; p < np; ++p)
    if (es[base + p] > 0.f) M = fmaxf(M, ml[base + p]);
  constexpr float kLog2e = 1.4426950408889634f;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float W = 0.f, o = 0.f;
    if (M != -INFINITY) {
      for (int p = 0; p < np; ++p) {
        const float l = es[base + p];
        if (!(l > 0.f)) continue;
        const float w = l * fast_exp2((ml[base + p] - M) * kLog2e);
        W += w;
        o = fmaf(w, tmp[(base + p) * D + d], o);
      }
    }
    const float val = W > 0.f ? o / W : 0.f;
    OT* dst = out + (static_cast<size_t>(s) * num_heads + h) * D + d;
    if constexpr (std::is_same<OT, float>::value) *dst = val;
    else if constexpr (std::is_same<OT, __half>::value) *dst = __float2half_rn(val);
    else *dst = __float2bfloat16_rn(val);
  }
}

// --------------------------------------------------------------------------
// Host side: tensor maps and launches.
// --------------------------------------------------------------------------
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a cache [num_blocks * bs tokens][num_kv_heads][head_dim]:
// dim0 = head_dim (contiguous), dim1 = kv head, dim2 = token slot; the box is
// one kv head's rows of min(bs, 16) consecutive token slots.
template <int KIND, int D, int BS>
cudaError_t make_cache_map(CUtensorMap* map, const void* base, int num_kv_heads, int num_blocks) {
  using T = Tr<KIND, D, BS>;
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(num_kv_heads),
                        static_cast<cuuint64_t>(num_blocks) * BS};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * T::ES,
                           static_cast<cuuint64_t>(num_kv_heads) * D * T::ES};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(T::BOX_INNER), 1u,
                       static_cast<cuuint32_t>(T::BOXH)};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUtensorMapDataType dt =
      T::ES == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const CUtensorMapSwizzle sw =
      T::ROWB == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUresult rc = fn(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename QT, int KIND, int D, int BS>
cudaError_t launch_tc(const DecodeArgs& a, const DecodeShape& sh, cudaStream_t stream) {
  using T = Tr<KIND, D, BS>;
  CUtensorMap mk, mv;
  cudaError_t e = make_cache_map<KIND, D, BS>(&mk, a.k_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  e = make_cache_map<KIND, D, BS>(&mv, a.v_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  const int ring = sh.warps * a.stages * T::STAGE;
  const int epi = kMaxWarps * 8 * (D + 4) * 4 + kMaxWarps * 16 * 4;
  const int smem = (ring > epi ? ring : epi) + 1024;
  auto kern = decode_tc_kernel<QT, KIND, D, BS>;
  // opt in to as much dynamic shared memory as the device allows next to the
  // kernel's static shared memory, once per device (harmless if repeated)
  static int configured[64] = {0};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64 || configured[dev] < smem) {
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    const int avail = optin - static_cast<int>(fa.sharedSizeBytes);
    if (smem > avail) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, avail);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) configured[dev] = avail;
  }
  dim3 grid(sh.grid_x, a.num_kv_heads, a.num_seqs);
  kern<<<grid, sh.warps * 32, smem, stream>>>(mk, mv, a);
  return cudaGetLastError();
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

int default_stages(int cache_dtype, int head_dim, int block_size, int warps) {
  (void)block_size;
  const int es = (cache_dtype == PA_INT8 || cache_dtype == PA_FP8E4M3) ? 1 : 2;
  const int stage = (2 * 16 * head_dim * es + (es == 1 ? 2 * 16 * 4 : 0) + 1023) / 1024 * 1024;
  int s = (96 * 1024) / (warps * stage);
  if (s < 2) s = 2;
  if (s > kMaxStages) s = kMaxStages;
  return s;
}

cudaError_t launch_decode(const DecodeArgs& a, const DecodeShape& sh, cudaStream_t s) {
  if (sh.cache_dtype == PA_F32) {
    dim3 grid(sh.grid_x, a.num_kv_heads, a.num_seqs);
    if (sh.head_dim == 128) decode_f32_kernel<128><<<grid, sh.warps * 32, 0, s>>>(a, sh.block_size);
    else decode_f32_kernel<64><<<grid, sh.warps * 32, 0, s>>>(a, sh.block_size);
    return cudaGetLastError();
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

cudaError_t launch_merge(void* out, int out_dtype, const float* tmp_out, const float* max_logits,
                         const float* exp_sums, const int32_t* seq_lens, int num_seqs,
                         int num_heads, int head_dim, int partition_size, int max_parts,
                         cudaStream_t s) {
  dim3 grid(num_heads, num_seqs);
  const int threads = head_dim;
  switch (out_dtype) {
    case PA_F32:
      merge_kernel<float><<<grid, threads, 0, s>>>(static_cast<float*>(out), tmp_out, max_logits,
                                                   exp_sums, seq_lens, num_heads, head_dim,
                                                   partition_size, max_parts);
      break;
    case PA_F16:
      merge_kernel<__half><<<grid, threads, 0, s>>>(static_cast<__half*>(out), tmp_out,
                                                    max_logits, exp_sums, seq_lens, num_heads,
                                                    head_dim, partition_size, max_parts);
      break;
    default:
      merge_kernel<__nv_bfloat16><<<grid, threads, 0, s>>>(
          static_cast<__nv_bfloat16*>(out), tmp_out, max_logits, exp_sums, seq_lens, num_heads,
          head_dim, partition_size, max_parts);
  }
  return cudaGetLastError();
}

}  // namespace pa
