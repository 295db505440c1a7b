// pa_tile.cuh -- the per-warp math of paged decode attention on one 16-token
// tile of one (sequence, kv head): shared-memory stage -> register fragments,
// S^T = K Q^T on mma.sync, online softmax, O^T += V^T P^T.  Used by the
// per-partition kernel (pa_decode.cu) and the persistent kernel (pa_fused.cu).
//
// Attention as "LLM推理优化：vLLM PagedAttention深度解析与工程实践" §二 states
// it, softmax(q K^T * scale) V, accumulated online over tiles in the log2
// domain (one softmax over all tokens, tile by tile).
#pragma once

#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "pa_device.cuh"

namespace pa {

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
  static constexpr int SCALES = QUANT ? 2 * 16 * 4 : 0;      // K scales then V scales
  static constexpr int KV_BYTES = 2 * KTILE + SCALES;
  static constexpr int STAGE = (KV_BYTES + 1023) / 1024 * 1024;
  static constexpr int BOX_INNER = ROWB / ES;                // TMA box inner extent (elements)
  static constexpr int NKF = NDH * NU;                       // 16-byte K chunks per row per lane
  static constexpr int NVF = ES == 2 ? NMT : NMT / 2;        // ldmatrix.x4 per tile for V
  static_assert(NDH * NU * KSPC == NKS, "k-step bookkeeping");
  // fp16 q over an 8-bit cache: the per-token V scale rides on P, times this power
  // of two (keeps P' in fp16's normal range; removed once per unit)
  static constexpr float VFOLD = KIND == kKindI8 ? 64.f : 256.f;
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

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
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

// Element d of head dimension held by k-step ks, lane quarter c, element e of
// the lane's 4 (the K loads and the q fragments agree on this order).
template <typename T>
__device__ __forceinline__ int qk_dim(int ks, int c) {
  const int v = ks % T::KSPC, u = (ks / T::KSPC) % T::NU, dh = ks / (T::KSPC * T::NU);
  return dh * T::BOX_INNER + (c + 4 * u) * T::EPC + 4 * v;
}

// fp16 q over an 8-bit cache takes the folded-V path (V codes widened without a
// scale multiply, the scale applied to P); bf16 q keeps the scale on P in fp32 and
// splits P into two bf16 parts.
template <typename QT, int KIND>
constexpr bool kFoldV = KIND != kKind16 && std::is_same<QT, __half>::value;

// Per-lane state of one (sequence, kv head) being accumulated by a warp.
template <typename QT, int KIND, int D, int BS>
struct WarpAttn {
  using T = Tr<KIND, D, BS>;
  uint32_t qf[T::NKS][2];           // q as the B operand of S^T = K Q^T (g = lane / 4)
  float m2[2];                      // running max, log2 units (g = 2c, 2c+1)
  float lsum[2];                    // this lane's share of the running sum
  float lv[2];                      // INT8 under fp16 q: this lane's share of sum P'
  float oacc[T::NMT][4];            // O^T accumulator (d rows, g columns)

  __device__ __forceinline__ void reset() {
    m2[0] = m2[1] = -INFINITY;
    lsum[0] = lsum[1] = 0.f;
    lv[0] = lv[1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < T::NMT; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
  }

  // q rows of the group from global memory: qrow points at head (kvh*G + lane/4).
  __device__ __forceinline__ void load_q_global(const QT* qrow, bool valid, int c) {
#pragma unroll
    for (int ks = 0; ks < T::NKS; ++ks) {
      uint2 w = make_uint2(0u, 0u);
      if (valid) w = *reinterpret_cast<const uint2*>(qrow + qk_dim<T>(ks, c));
      qf[ks][0] = w.x;
      qf[ks][1] = w.y;
    }
  }

  // q rows of the group from a shared-memory copy [G][D] of QT at `base`.
  __device__ __forceinline__ void load_q_smem(uint32_t base, int g, bool valid, int c) {
#pragma unroll
    for (int ks = 0; ks < T::NKS; ++ks) {
      uint2 w = make_uint2(0u, 0u);
      if (valid) w = lds64(base + static_cast<uint32_t>((g * D + qk_dim<T>(ks, c)) * 2));
      qf[ks][0] = w.x;
      qf[ks][1] = w.y;
    }
  }

  // End of a unit's tiles (before its lanes' results are combined): fp16 q over an
  // 8-bit cache accumulated sum P' (bias + code) with P' = P * s_v * VFOLD; take
  // the bias term out (INT8 codes enter as 1152 + c) and the fold factor.
  __device__ __forceinline__ void finish() {
    if constexpr (kFoldV<QT, KIND>) {
      constexpr uint32_t FULL = 0xffffffffu;
      constexpr float inv = 1.f / T::VFOLD;
      float b0 = 0.f, b1 = 0.f;
      if constexpr (KIND == kKindI8) {
        float l0 = lv[0], l1 = lv[1];
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          l0 += __shfl_xor_sync(FULL, l0, off);
          l1 += __shfl_xor_sync(FULL, l1, off);
        }
        b0 = -1152.f * inv * l0;
        b1 = -1152.f * inv * l1;
      }
#pragma unroll
      for (int mt = 0; mt < T::NMT; ++mt) {
        oacc[mt][0] = fmaf(oacc[mt][0], inv, b0);
        oacc[mt][1] = fmaf(oacc[mt][1], inv, b1);
        oacc[mt][2] = fmaf(oacc[mt][2], inv, b0);
        oacc[mt][3] = fmaf(oacc[mt][3], inv, b1);
      }
    }
  }
};

// One tile's operands in registers (the stage can be refilled once loaded).
template <int KIND, int D, int BS>
struct TileFrag {
  using T = Tr<KIND, D, BS>;
  uint4 kf[T::NKF][2];
  uint32_t vf[T::NVF][4];
  float ks0, ks1;                   // K scales of this lane's two token rows
  float sv0, sv1;                   // V scales of the same rows (applied to P)
};

template <typename QT, int KIND, int D, int BS>
__device__ __forceinline__ void load_tile(TileFrag<KIND, D, BS>& f, uint32_t st, int lane) {
  using T = Tr<KIND, D, BS>;
  const int r = lane >> 2, c = lane & 3, mi = lane >> 3, jj = lane & 7;
  const int tok0 = tau<T::ROWB>(r), tok1 = tok0 + 8;
#pragma unroll
  for (int dh = 0; dh < T::NDH; ++dh) {
#pragma unroll
    for (int u = 0; u < T::NU; ++u) {
      f.kf[dh * T::NU + u][0] = lds128(st + swz<T::ROWB>(dh * 16 + tok0, c + 4 * u));
      f.kf[dh * T::NU + u][1] = lds128(st + swz<T::ROWB>(dh * 16 + tok1, c + 4 * u));
    }
  }
#pragma unroll
  for (int q = 0; q < T::NVF; ++q) {
    if constexpr (KIND == kKind16) {
      const int dh = (q * 16) / T::BOX_INNER;
      const int cl = ((q * 16) % T::BOX_INNER) / 8;
      const int tok = (mi >> 1) * 8 + tau<T::ROWB>(jj);
      ldmatrix_x4_trans(st + T::KTILE + swz<T::ROWB>(dh * 16 + tok, cl + (mi & 1)), f.vf[q][0],
                        f.vf[q][1], f.vf[q][2], f.vf[q][3]);
    } else {
      const int tok = (mi & 1) * 8 + tau<T::ROWB>(jj);
      ldmatrix_x4_trans(st + T::KTILE + swz<T::ROWB>(tok, 2 * q + (mi >> 1)), f.vf[q][0],
                        f.vf[q][1], f.vf[q][2], f.vf[q][3]);
    }
  }
  f.ks0 = f.ks1 = f.sv0 = f.sv1 = 1.f;
  if constexpr (T::QUANT) {
    const uint32_t ksc = st + 2 * T::KTILE, vsc = ksc + 64;
    f.ks0 = lds_f32(ksc + tok0 * 4);
    f.ks1 = lds_f32(ksc + tok1 * 4);
    f.sv0 = lds_f32(vsc + tok0 * 4);
    f.sv1 = lds_f32(vsc + tok1 * 4);
  }
}

// Accumulate one tile into `w`.  nv = valid tokens of the tile (from its
// start), okm = bit b set if box b was loaded (tokens of other boxes masked).
template <typename QT, int KIND, int D, int BS>
__device__ __forceinline__ void tile_compute(WarpAttn<QT, KIND, D, BS>& w,
                                             const TileFrag<KIND, D, BS>& f, int nv, int okm,
                                             float scale_log2, int lane) {
  using T = Tr<KIND, D, BS>;
  constexpr uint32_t FULL = 0xffffffffu;
  const int r = lane >> 2, c = lane & 3;
  const int tok0 = tau<T::ROWB>(r), tok1 = tok0 + 8;
  const int ta = tau<T::ROWB>(2 * c), tb = tau<T::ROWB>(2 * c + 1);
  const bool partial = (nv < 16) || (okm != (1 << T::NBOX) - 1);

  // ---- S^T = K Q^T, two independent accumulator chains
  float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int kc = 0; kc < T::NKF; ++kc) {
    const uint32_t a0[4] = {f.kf[kc][0].x, f.kf[kc][0].y, f.kf[kc][0].z, f.kf[kc][0].w};
    const uint32_t a1[4] = {f.kf[kc][1].x, f.kf[kc][1].y, f.kf[kc][1].z, f.kf[kc][1].w};
#pragma unroll
    for (int v = 0; v < T::KSPC; ++v) {
      const int ks = kc * T::KSPC + v;
      uint32_t af[4];
      if constexpr (KIND == kKind16) {
        af[0] = a0[2 * v];
        af[1] = a1[2 * v];
        af[2] = a0[2 * v + 1];
        af[3] = a1[2 * v + 1];
      } else if constexpr (KIND == kKindI8 && std::is_same<QT, __half>::value) {
        // one XOR per word, then one permute + one subtract per pair
        const uint32_t x0 = a0[v] ^ 0x80808080u, x1 = a1[v] ^ 0x80808080u;
        af[0] = int8x2_biased_to_f16x2<0x5140u>(x0);
        af[1] = int8x2_biased_to_f16x2<0x5140u>(x1);
        af[2] = int8x2_biased_to_f16x2<0x5342u>(x0);
        af[3] = int8x2_biased_to_f16x2<0x5342u>(x1);
      } else if constexpr (KIND == kKindE4M3 && std::is_same<QT, __half>::value) {
        uint16_t l0, h0, l1, h1;
        split_halves(a0[v], l0, h0);
        split_halves(a1[v], l1, h1);
        af[0] = e4m3x2h_to_f16x2(l0);
        af[1] = e4m3x2h_to_f16x2(l1);
        af[2] = e4m3x2h_to_f16x2(h0);
        af[3] = e4m3x2h_to_f16x2(h1);
      } else {
        af[0] = cvt_k_pair<QT, KIND>(a0[v]);
        af[1] = cvt_k_pair<QT, KIND>(a1[v]);
        af[2] = cvt_k_pair<QT, KIND>(a0[v] >> 16);
        af[3] = cvt_k_pair<QT, KIND>(a1[v] >> 16);
      }
      if (ks & 1) mma_16816<QT>(acc1, af, w.qf[ks][0], w.qf[ks][1]);
      else mma_16816<QT>(acc0, af, w.qf[ks][0], w.qf[ks][1]);
    }
  }
  const bool ok0 = tok0 < nv && ((okm >> (tok0 / T::BOXH)) & 1);
  const bool ok1 = tok1 < nv && ((okm >> (tok1 / T::BOXH)) & 1);
  const float s0 = scale_log2 * f.ks0, s1 = scale_log2 * f.ks1;
  float x0 = ok0 ? (acc0[0] + acc1[0]) * s0 : -INFINITY;
  float x1 = ok0 ? (acc0[1] + acc1[1]) * s0 : -INFINITY;
  float x2 = ok1 ? (acc0[2] + acc1[2]) * s1 : -INFINITY;
  float x3 = ok1 ? (acc0[3] + acc1[3]) * s1 : -INFINITY;

  // ---- online softmax (per query head g = 2c, 2c+1)
  float tm0 = fmaxf(x0, x2), tm1 = fmaxf(x1, x3);
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    tm0 = fmaxf(tm0, __shfl_xor_sync(FULL, tm0, off));
    tm1 = fmaxf(tm1, __shfl_xor_sync(FULL, tm1, off));
  }
  const float mn0 = fmaxf(w.m2[0], tm0), mn1 = fmaxf(w.m2[1], tm1);
  const float ms0 = mn0 == -INFINITY ? 0.f : mn0;
  const float ms1 = mn1 == -INFINITY ? 0.f : mn1;
  const float al0 = fast_exp2(w.m2[0] - ms0), al1 = fast_exp2(w.m2[1] - ms1);
  w.m2[0] = mn0;
  w.m2[1] = mn1;
  float p0 = fast_exp2(x0 - ms0), p1 = fast_exp2(x1 - ms1);
  float p2 = fast_exp2(x2 - ms0), p3 = fast_exp2(x3 - ms1);
  w.lsum[0] = w.lsum[0] * al0 + (p0 + p2);
  w.lsum[1] = w.lsum[1] * al1 + (p1 + p3);
  if constexpr (kFoldV<QT, KIND> && KIND == kKindI8) {
    w.lv[0] *= al0;
    w.lv[1] *= al1;
  }
  if (__any_sync(FULL, (al0 != 1.f) || (al1 != 1.f))) {
#pragma unroll
    for (int mt = 0; mt < T::NMT; ++mt) {
      w.oacc[mt][0] *= al0;
      w.oacc[mt][1] *= al1;
      w.oacc[mt][2] *= al0;
      w.oacc[mt][3] *= al1;
    }
  }

  // ---- O^T += V^T P^T
  if constexpr (T::QUANT) {
    // the V scale of each token rides on its P (fp32; poisoned scales of masked
    // tokens never reach a zero P); fp16 q also multiplies by VFOLD
    const float v0 = kFoldV<QT, KIND> ? f.sv0 * T::VFOLD : f.sv0;
    const float v1 = kFoldV<QT, KIND> ? f.sv1 * T::VFOLD : f.sv1;
    p0 = p0 != 0.f ? p0 * v0 : 0.f;
    p1 = p1 != 0.f ? p1 * v0 : 0.f;
    p2 = p2 != 0.f ? p2 * v1 : 0.f;
    p3 = p3 != 0.f ? p3 * v1 : 0.f;
  }
  // P as the B operand.  bf16 keeps 8 significant bits, so P is split into a
  // high and a low bf16 part (two MMAs, ~16 bits); fp16's 11 bits (P in [0, 1])
  // keep the output within the comparison bound with one MMA.
  constexpr bool kSplitP = std::is_same<QT, __nv_bfloat16>::value;
  const uint32_t h01 = pack2<QT>(p0, p1), h23 = pack2<QT>(p2, p3);
  const float2 f01 = unpack2<QT>(h01), f23 = unpack2<QT>(h23);
  const uint32_t l01 = pack2<QT>(p0 - f01.x, p1 - f01.y);
  const uint32_t l23 = pack2<QT>(p2 - f23.x, p3 - f23.y);
  const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
  const uint32_t bl0 = movmatrix_trans(l01), bl1 = movmatrix_trans(l23);
  if constexpr (kFoldV<QT, KIND> && KIND == kKindI8) {
    // the sum of the P' the MMAs see (fp16-rounded), for the bias of the codes
    w.lv[0] += f01.x + f23.x;
    w.lv[1] += f01.y + f23.y;
  }

  uint32_t mk01 = ~0u, mk23 = ~0u;
  if (partial) {
    auto valid = [&](int t) { return t < nv && ((okm >> (t / T::BOXH)) & 1); };
    mk01 = (valid(ta) ? 0x0000FFFFu : 0u) | (valid(tb) ? 0xFFFF0000u : 0u);
    mk23 = (valid(ta + 8) ? 0x0000FFFFu : 0u) | (valid(tb + 8) ? 0xFFFF0000u : 0u);
  }
  if constexpr (KIND == kKind16) {
#pragma unroll
    for (int mt = 0; mt < T::NMT; ++mt) {
      uint32_t af[4] = {f.vf[mt][0], f.vf[mt][1], f.vf[mt][2], f.vf[mt][3]};
      if (partial) {
        af[0] &= mk01;
        af[1] &= mk01;
        af[2] &= mk23;
        af[3] &= mk23;
      }
      mma_16816<QT>(w.oacc[mt], af, bh0, bh1);
      if constexpr (kSplitP) mma_16816<QT>(w.oacc[mt], af, bl0, bl1);
    }
  } else {
#pragma unroll
    for (int q = 0; q < T::NVF; ++q) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int mt = 2 * q + hh;
        uint32_t af[4];
        if constexpr (KIND == kKindI8 && std::is_same<QT, __half>::value) {
          // pairs {0,2} and {1,3} of each word as fp16 1152 + c (one permute each;
          // the bias comes out once per unit, in finish())
          const uint32_t x0 = f.vf[q][2 * hh] ^ 0x80808080u;
          const uint32_t x1 = f.vf[q][2 * hh + 1] ^ 0x80808080u;
          af[0] = __byte_perm(x0, 0x64646464u, 0x5240u);
          af[1] = __byte_perm(x0, 0x64646464u, 0x5341u);
          af[2] = __byte_perm(x1, 0x64646464u, 0x5240u);
          af[3] = __byte_perm(x1, 0x64646464u, 0x5341u);
        } else {
          af[0] = cvt_v_pair<QT, KIND>(f.vf[q][2 * hh], 0);
          af[1] = cvt_v_pair<QT, KIND>(f.vf[q][2 * hh], 1);
          af[2] = cvt_v_pair<QT, KIND>(f.vf[q][2 * hh + 1], 0);
          af[3] = cvt_v_pair<QT, KIND>(f.vf[q][2 * hh + 1], 1);
        }
        if (partial) {
          af[0] &= mk01;
          af[1] &= mk01;
          af[2] &= mk23;
          af[3] &= mk23;
        }
        mma_16816<QT>(w.oacc[mt], af, bh0, bh1);
        if constexpr (kSplitP) mma_16816<QT>(w.oacc[mt], af, bl0, bl1);
      }
    }
  }
}

// head_dim index of oacc[mt][k] for this lane (k = 0, 1: first row; 2, 3: second).
template <int KIND>
__device__ __forceinline__ int out_dim(int mt, int r, int second) {
  if constexpr (KIND == kKind16) return mt * 16 + r + 8 * second;
  else return mt * 16 + 2 * r + second;
}

// Issue the TMA / bulk copies of one tile (lane 0 only).  blk[b] < 0 entries
// are skipped.  Returns the bytes the stage's barrier must expect.
template <int KIND, int D, int BS>
__device__ __forceinline__ uint32_t tile_bytes(int okm) {
  using T = Tr<KIND, D, BS>;
  return __popc(okm) * (2 * T::NDH * T::BOXH * T::ROWB + (T::QUANT ? 2 * T::BOXH * 4 : 0));
}

template <int KIND, int D, int BS>
__device__ __forceinline__ void issue_tile_copies(uint32_t st, uint32_t bar, const CUtensorMap* mk,
                                                  const CUtensorMap* mv, const float* k_scale,
                                                  const float* v_scale, int num_kv_heads, int kvh,
                                                  const int (&blk)[Tr<KIND, D, BS>::NBOX], int okm,
                                                  int ob, uint64_t pol) {
  using T = Tr<KIND, D, BS>;
#pragma unroll
  for (int b = 0; b < T::NBOX; ++b) {
    if (!((okm >> b) & 1)) continue;
    const int row_tok = blk[b] * BS + ob;
#pragma unroll
    for (int dh = 0; dh < T::NDH; ++dh) {
      const uint32_t roff = static_cast<uint32_t>((dh * 16 + b * T::BOXH) * T::ROWB);
      tma_load_3d(st + roff, mk, dh * T::BOX_INNER, kvh, row_tok, bar, pol);
      tma_load_3d(st + T::KTILE + roff, mv, dh * T::BOX_INNER, kvh, row_tok, bar, pol);
    }
    if constexpr (T::QUANT) {
      const size_t so = (static_cast<size_t>(blk[b]) * num_kv_heads + kvh) * BS + ob;
      bulk_load(st + 2 * T::KTILE + b * T::BOXH * 4, k_scale + so, T::BOXH * 4, bar, pol);
      bulk_load(st + 2 * T::KTILE + 64 + b * T::BOXH * 4, v_scale + so, T::BOXH * 4, bar, pol);
    }
  }
}

// L2 prefetch of the same copies (any thread; ids outside [0, num_blocks) are
// skipped).  Safe before griddepcontrol.wait: L2 is where every SM's writes
// land, so a line fetched early is still current when the TMA load reads it.
template <int KIND, int D, int BS>
__device__ __forceinline__ void prefetch_tile(const CUtensorMap* mk, const CUtensorMap* mv,
                                              const float* k_scale, const float* v_scale,
                                              int num_kv_heads, int num_blocks, int kvh,
                                              const int (&blk)[Tr<KIND, D, BS>::NBOX], int ob) {
  using T = Tr<KIND, D, BS>;
#pragma unroll
  for (int b = 0; b < T::NBOX; ++b) {
    if (blk[b] < 0 || blk[b] >= num_blocks) continue;
    const int row_tok = blk[b] * BS + ob;
#pragma unroll
    for (int dh = 0; dh < T::NDH; ++dh) {
      tma_prefetch_3d(mk, dh * T::BOX_INNER, kvh, row_tok);
      tma_prefetch_3d(mv, dh * T::BOX_INNER, kvh, row_tok);
    }
    if constexpr (T::QUANT) {
      const size_t so = (static_cast<size_t>(blk[b]) * num_kv_heads + kvh) * BS + ob;
      bulk_prefetch_l2(k_scale + so, T::BOXH * 4);
      bulk_prefetch_l2(v_scale + so, T::BOXH * 4);
    }
  }
}

// ---------------------------------------------------------------- host side

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// Launch with or without programmatic dependent launch (PDL).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Opt a kernel in to as much dynamic shared memory as the device allows next
// to its static shared memory, once per device (harmless if repeated).
inline cudaError_t opt_in_smem(const void* kern, int needed, int (&configured)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && configured[dev] >= needed) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  const int avail = optin - static_cast<int>(fa.sharedSizeBytes);
  if (needed > avail) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, avail);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64) configured[dev] = avail;
  return cudaSuccess;
}

}  // namespace pa
