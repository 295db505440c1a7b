// pa_fused.cu -- persistent single-launch paged decode attention (pa_decode_fused).
//
// The same attention as paged_attention_v2 ("LLM推理优化：vLLM PagedAttention深度解析与工程实践"
// §4.1: partial accumulation, then a merge), scheduled for B200 instead of one
// CTA per fixed-size partition:
// * the batch's work is the list of 16-token tiles of every (sequence, kv head)
//   unit, in sequence-major order; every warp of a grid sized to the SMs takes
//   an equal contiguous range of that list, so all SMs stream until the end and
//   no CTA ever starts or drains mid-kernel;
// * a warp streams its range through its own ring of TMA stages without
//   draining at unit boundaries (the next unit's q rows are prefetched into L2
//   when its first tile is issued and read into registers when that tile
//   arrives, so a stage holds K and V only);
// * results leave the accumulator registers by plain stores (no shared-memory
//   transpose), which with the K/V-only stages keeps a CTA at ~66 KB of shared
//   memory.  A second build, capped at 168 registers, fits three CTAs (12 warps)
//   on an SM: the launch that runs beside the cascade's prefix kernel on part of
//   the GPU is bound by warps per SM and takes it.  With the GPU to itself the
//   uncapped build (two CTAs by registers) is faster;
// * a unit that lies wholly inside one warp's range is written straight to
//   `out`; a unit split across warps leaves one (m, l, o) record per warp and
//   the warp that finishes it last (an atomic arrival counter -- nobody waits)
//   merges the records by log-sum-exp, writes `out`, resets the counter and
//   discards the records' L2 lines so they are never written back to HBM.
#include <climits>

#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tile.cuh"

namespace pa {

__device__ __forceinline__ void discard_l2_line(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

__device__ __forceinline__ void put_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void put_elem(__half* p, float v) { *p = __float2half_rn(v); }
__device__ __forceinline__ void put_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <typename QT, int KIND, int D, int BS, int MINB>
__global__ void __launch_bounds__(kFusedWarps * 32, MINB)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ FusedArgs a) {
  using T = Tr<KIND, D, BS>;
  constexpr int NW = kFusedWarps;
  constexpr int STG = T::STAGE;               // K and V of one tile (+ scales)
  constexpr int REC = 8 * D + 32;             // floats per partial record
  constexpr uint32_t FULL = 0xffffffffu;
  constexpr int kBeyond = INT_MIN;
  static_assert(STG % 1024 == 0, "stages stay 1024-byte aligned");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bars[NW * kMaxStages];
  __shared__ int meta[NW * kMaxStages * 4];
  __shared__ int scan_warp[NW];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane >> 2, c = lane & 3;
  const int Hkv = a.num_kv_heads;
  const int G = a.num_heads / Hkv;
  const int S = a.stages;
  const int NS = a.num_seqs;
  const bool check = a.err_flag != nullptr;

  const uint32_t sraw = smem_u32(smem_raw);
  const uint32_t sbase = (sraw + 1023u) & ~1023u;
  const uint32_t wbase = sbase + static_cast<uint32_t>(warp * S * STG);
  int* C = reinterpret_cast<int*>(smem_raw + (sbase - sraw) + static_cast<uint32_t>(NW * S * STG));
  const uint32_t bar0 = smem_u32(&bars[warp * kMaxStages]);
  int* wmeta = &meta[warp * kMaxStages * 4];

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(bar0 + 8u * s, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }

  griddep_launch_dependents();
  // mode 2 first reads lens / tables; mode 3 never waits here
  if (a.pdl != 2 && a.pdl != 3) griddep_wait();
  const int t_off = a.t_offset;

  // ---- tiles per sequence and their prefix C[s] (each CTA keeps its own copy)
  auto tiles_of = [&](int s, bool report) -> int {
    const int len = a.seq_lens[s];
    if (check && (len < 0 || static_cast<long long>(len) > static_cast<long long>(a.max_blocks) * BS)) {
      if (report) report_error(a.err_flag, kErrSeqLen);
      return 0;                                   // skipped: its output is zeros
    }
    return len > t_off ? (len - t_off + 15) / 16 : 0;
  };
  {
    const int per = (NS + blockDim.x - 1) / blockDim.x;
    const int s0 = min(NS, static_cast<int>(threadIdx.x) * per), s1 = min(NS, s0 + per);
    int local = 0;
    for (int s = s0; s < s1; ++s) local += tiles_of(s, blockIdx.x == 0) * Hkv;
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(FULL, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) scan_warp[warp] = incl;
    __syncthreads();
    int wpre = 0;
    for (int w2 = 0; w2 < warp; ++w2) wpre += scan_warp[w2];
    int run = wpre + incl - local;
    for (int s = s0; s < s1; ++s) {
      C[s] = run;
      run += tiles_of(s, false) * Hkv;
    }
    if (threadIdx.x == blockDim.x - 1) C[NS] = wpre + incl;
    __syncthreads();
  }

  // ---- this warp's equal share of the tile list
  const long long Ttot = C[NS];
  const long long W = static_cast<long long>(gridDim.x) * NW;
  const long long wme = static_cast<long long>(blockIdx.x) * NW + warp;
  // warp w gets tiles [w*q + min(w, rem), ...) with q = T / W, rem = T % W: the
  // first rem warps take one extra tile, and no empty range sits between two
  // non-empty ones
  const long long q_per = Ttot / W, rem = Ttot % W;
  auto range_start = [&](long long w2) { return w2 * q_per + (w2 < rem ? w2 : rem); };
  auto warp_of = [&](long long g) {
    return g < (q_per + 1) * rem ? g / (q_per + 1) : rem + (g - (q_per + 1) * rem) / q_per;
  };
  const int t_lo = static_cast<int>(range_start(wme));
  const int nmine = static_cast<int>(range_start(wme + 1) - t_lo);

  // Window: lane l describes tile (32 * window + l) of this warp's range.
  struct Win {
    int ids[T::NBOX];
    int seq, kvh, j, nv;
  };
  auto load_window = [&](int wdx, Win& wn) {
    const int i = wdx * 32 + lane;
    wn.seq = wn.kvh = wn.j = wn.nv = 0;
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) wn.ids[b] = kBeyond;
    if (i >= nmine) return;
    const int g = t_lo + i;
    int lo = 0, hi = NS;                          // C[lo] <= g < C[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (C[mid] <= g) lo = mid;
      else hi = mid;
    }
    const int nt = (C[lo + 1] - C[lo]) / Hkv;
    const int off = g - C[lo];
    wn.seq = lo;
    wn.kvh = off / nt;
    wn.j = off % nt;
    const int len = a.seq_lens[lo];
    wn.nv = min(16, len - t_off - 16 * wn.j);
    const int nblk = (len + BS - 1) / BS;
    const int32_t* table = a.block_tables + static_cast<size_t>(lo) * a.max_blocks;
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) {
      const int lb = (t_off + 16 * wn.j + b * T::BOXH) / BS;
      wn.ids[b] = lb < nblk ? __ldg(table + lb) : kBeyond;
    }
  };
  Win cur, nxt;
  load_window(0, cur);
  if (nmine > 32) load_window(1, nxt);
  // PDL mode 2: fetch this warp's first tiles into L2 while the preceding grid
  // finishes (lane i prefetches tile i of window 0)
  if ((a.pdl == 2 || a.pdl == 3) && lane < min(a.prefetch, nmine)) {
    const int ob = BS > 16 ? (t_off + 16 * cur.j) % BS : 0;
    prefetch_tile<KIND, D, BS>(&tm_k, &tm_v, a.k_scale, a.v_scale, a.num_kv_heads, a.num_blocks,
                               cur.kvh, cur.ids, ob);
  }
  if (a.pdl == 2) griddep_wait();                 // q and the caches may come from it
  // sequences without tiles get zeros (partials: o = 0, m = -inf, l = 0)
  for (int s = blockIdx.x; s < NS; s += gridDim.x) {
    if (C[s + 1] != C[s]) continue;
    if (a.part_o) {
      float* o = a.part_o + static_cast<size_t>(s) * a.num_heads * D;
      for (int e = threadIdx.x * 4; e < a.num_heads * D; e += blockDim.x * 4)
        *reinterpret_cast<float4*>(o + e) = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int h = threadIdx.x; h < a.num_heads; h += blockDim.x) {
        a.part_m[static_cast<size_t>(s) * a.num_heads + h] = -INFINITY;
        a.part_l[static_cast<size_t>(s) * a.num_heads + h] = 0.f;
      }
      continue;
    }
    QT* o = reinterpret_cast<QT*>(a.out) + static_cast<size_t>(s) * a.num_heads * D;
    for (int e = threadIdx.x * 8; e < a.num_heads * D; e += blockDim.x * 8)
      *reinterpret_cast<uint4*>(o + e) = make_uint4(0u, 0u, 0u, 0u);
  }
  int win_cur = 0;
  uint32_t armed = 0;
  const uint64_t pol = policy_evict_first();

  auto issue = [&](int i, int s) {
    const int wdx = i >> 5;
    if (wdx != win_cur) {
      cur = nxt;
      win_cur = wdx;
      if ((wdx + 1) * 32 < nmine) load_window(wdx + 1, nxt);
    }
    const int src = i & 31;
    int blk[T::NBOX];
#pragma unroll
    for (int b = 0; b < T::NBOX; ++b) blk[b] = __shfl_sync(FULL, cur.ids[b], src);
    const int seq = __shfl_sync(FULL, cur.seq, src), kvh = __shfl_sync(FULL, cur.kvh, src);
    const int j = __shfl_sync(FULL, cur.j, src), nv = __shfl_sync(FULL, cur.nv, src);
    if (a.inject == 1 && i == 0) return;          // test hook: this stage never arrives
    armed |= 1u << s;
    if (lane == 0) {
      const uint32_t st = wbase + static_cast<uint32_t>(s * STG);
      const uint32_t bar = bar0 + 8u * s;
      const bool newseg = (i == 0) || (j == 0);
      const int ob = BS > 16 ? (t_off + 16 * j) % BS : 0;
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
      wmeta[s * 4 + 0] = seq;
      wmeta[s * 4 + 1] = kvh;
      wmeta[s * 4 + 2] = j;
      wmeta[s * 4 + 3] = okm | (nv << 8) | (newseg ? (1 << 16) : 0);
      const uint32_t bytes = tile_bytes<KIND, D, BS>(okm);
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(bar, bytes);
      issue_tile_copies<KIND, D, BS>(st, bar, &tm_k, &tm_v, a.k_scale, a.v_scale, Hkv, kvh, blk,
                                     okm, ob, pol);
      // the unit's q rows: into L2 now, read into registers when this tile arrives
      if (newseg)
        bulk_prefetch_l2(reinterpret_cast<const QT*>(a.q) +
                             (static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G) * D,
                         G * D * 2);
    }
  };

  WarpAttn<QT, KIND, D, BS> wa;
  wa.reset();

  // Close the current segment (tiles j0..j1 of unit (seq, kvh)).
  auto finalize = [&](int seq, int kvh, int j0, int j1, bool first) {
    const int nt = (C[seq + 1] - C[seq]) / Hkv;
    wa.finish();
    float l0 = wa.lsum[0], l1 = wa.lsum[1];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(FULL, l0, off);
      l1 += __shfl_xor_sync(FULL, l1, off);
    }
    const bool full = (j0 == 0) && (j1 == nt - 1);
    const float sc0 = full ? (l0 > 0.f ? 1.f / l0 : 0.f) : 1.f;
    const float sc1 = full ? (l1 > 0.f ? 1.f / l1 : 0.f) : 1.f;
    // this lane's accumulator entries are (head 2c, d0), (2c + 1, d0), (2c, d1) and
    // (2c + 1, d1) of every m-tile; heads at or past G are padding
    const bool g0ok = 2 * c < G, g1ok = 2 * c + 1 < G;
    auto emit = [&](auto* base, float s0, float s1) {   // base: head 0's row, pitch D
#pragma unroll
      for (int mt = 0; mt < T::NMT; ++mt) {
        const int d0 = out_dim<KIND>(mt, r, 0), d1 = out_dim<KIND>(mt, r, 1);
        if (g0ok) {
          put_elem(base + (2 * c) * D + d0, wa.oacc[mt][0] * s0);
          put_elem(base + (2 * c) * D + d1, wa.oacc[mt][2] * s0);
        }
        if (g1ok) {
          put_elem(base + (2 * c + 1) * D + d0, wa.oacc[mt][1] * s1);
          put_elem(base + (2 * c + 1) * D + d1, wa.oacc[mt][3] * s1);
        }
      }
    };
    QT* outp = reinterpret_cast<QT*>(a.out) +
               (static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G) * D;
    const size_t prow = static_cast<size_t>(seq) * a.num_heads + static_cast<size_t>(kvh) * G;
    if (full && a.part_o) {                       // the unit's partial: o / l, m, l
      emit(a.part_o + prow * D, sc0, sc1);
      if (r == 0 && g0ok) {
        a.part_m[prow + 2 * c] = wa.m2[0];
        a.part_l[prow + 2 * c] = l0;
      }
      if (r == 0 && g1ok) {
        a.part_m[prow + 2 * c + 1] = wa.m2[1];
        a.part_l[prow + 2 * c + 1] = l1;
      }
      __syncwarp();
      return;
    }
    if (full) {
      emit(outp, sc0, sc1);
      __syncwarp();
      return;
    }
    // split unit: leave this warp's record, the last arriver merges
    float* rec = a.partials + static_cast<size_t>(2 * wme + (first ? 0 : 1)) * REC;
    emit(rec, 1.f, 1.f);
    if (r == 0) {
      rec[8 * D + 2 * c] = wa.m2[0];
      rec[8 * D + 2 * c + 1] = wa.m2[1];
      rec[8 * D + 8 + 2 * c] = l0;
      rec[8 * D + 8 + 2 * c + 1] = l1;
    }
    __threadfence();
    __syncwarp();
    int prev = 0;
    if (lane == 0) prev = atomicAdd(&a.counters[seq * Hkv + kvh], 1);
    prev = __shfl_sync(FULL, prev, 0);
    // contributors: warps wf..wl (every range between them is non-empty)
    const long long start = C[seq] + static_cast<long long>(kvh) * nt;
    const long long wf = warp_of(start), wl = warp_of(start + nt - 1);
    if (prev != static_cast<int>(wl - wf)) {
      __syncwarp();
      return;
    }
    __threadfence();
    const int slot_f = range_start(wf) == start ? 0 : 1;
    auto record = [&](long long w2) {
      return a.partials + static_cast<size_t>(2 * w2 + (w2 == wf ? slot_f : 0)) * REC;
    };
    // Online log-sum-exp merge, 32 contributors at a time: lane t fetches
    // contributor t's (m, l) rows, warp reductions give the weights, then the o
    // rows stream in with independent loads.  Entry k of this lane is
    // (g, d4) = ((lane + 32k) / (D/4), 4 * ((lane + 32k) % (D/4))).
    constexpr int NPL = D / 16;                   // float4 entries per lane (8 rows of D)
    float Mg[8], Lg[8];
    float4 acc[NPL];
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      Mg[g] = -INFINITY;
      Lg[g] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < NPL; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int n = static_cast<int>(wl - wf + 1);
    for (int base = 0; base < n; base += 32) {
      const int t = base + lane;
      float mt[8], lt[8];
      if (t < n) {
        const float4* rm = reinterpret_cast<const float4*>(record(wf + t) + 8 * D);
        const float4 m0 = __ldcg(rm), m1 = __ldcg(rm + 1), l0v = __ldcg(rm + 2), l1v = __ldcg(rm + 3);
        mt[0] = m0.x; mt[1] = m0.y; mt[2] = m0.z; mt[3] = m0.w;
        mt[4] = m1.x; mt[5] = m1.y; mt[6] = m1.z; mt[7] = m1.w;
        lt[0] = l0v.x; lt[1] = l0v.y; lt[2] = l0v.z; lt[3] = l0v.w;
        lt[4] = l1v.x; lt[5] = l1v.y; lt[6] = l1v.z; lt[7] = l1v.w;
      } else {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          mt[g] = -INFINITY;
          lt[g] = 0.f;
        }
      }
      float ft[8], keep[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float cm = mt[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(FULL, cm, off));
        const float nm = fmaxf(Mg[g], cm);
        const float ms = nm == -INFINITY ? 0.f : nm;
        keep[g] = fast_exp2(Mg[g] - ms);
        ft[g] = fast_exp2(mt[g] - ms);
        float ls = lt[g] * ft[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(FULL, ls, off);
        Lg[g] = Lg[g] * keep[g] + ls;
        Mg[g] = nm;
      }
#pragma unroll
      for (int k = 0; k < NPL; ++k) {
        const int g = (lane + 32 * k) / (D / 4);
        float kp = keep[0];
#pragma unroll
        for (int gg = 1; gg < 8; ++gg) kp = g == gg ? keep[gg] : kp;
        acc[k].x *= kp;
        acc[k].y *= kp;
        acc[k].z *= kp;
        acc[k].w *= kp;
      }
      const int cnt = min(32, n - base);
#pragma unroll 2
      for (int u = 0; u < cnt; ++u) {
        const float* ru = record(wf + base + u);
        float fu[8];
#pragma unroll
        for (int g = 0; g < 8; ++g) fu[g] = __shfl_sync(FULL, ft[g], u);
#pragma unroll
        for (int k = 0; k < NPL; ++k) {
          const int idx = lane + 32 * k;
          const int g = idx / (D / 4), d4 = (idx % (D / 4)) * 4;
          float f = fu[0];
#pragma unroll
          for (int gg = 1; gg < 8; ++gg) f = g == gg ? fu[gg] : f;
          if (g < G) {
            const float4 v = __ldcg(reinterpret_cast<const float4*>(ru + g * D + d4));
            acc[k].x += v.x * f;
            acc[k].y += v.y * f;
            acc[k].z += v.z * f;
            acc[k].w += v.w * f;
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < NPL; ++k) {
      const int idx = lane + 32 * k;
      const int g = idx / (D / 4), d4 = (idx % (D / 4)) * 4;
      float L = Lg[0];
#pragma unroll
      for (int gg = 1; gg < 8; ++gg) L = g == gg ? Lg[gg] : L;
      if (g < G) {
        const float inv = L > 0.f ? 1.f / L : 0.f;
        if (a.part_o) {
          *reinterpret_cast<float4*>(a.part_o + (prow + g) * D + d4) =
              make_float4(acc[k].x * inv, acc[k].y * inv, acc[k].z * inv, acc[k].w * inv);
        } else {
          uint2 pk;
          pk.x = pack2<QT>(acc[k].x * inv, acc[k].y * inv);
          pk.y = pack2<QT>(acc[k].z * inv, acc[k].w * inv);
          *reinterpret_cast<uint2*>(outp + g * D + d4) = pk;
        }
      }
    }
    if (a.part_o && lane < G) {
      float M = Mg[0], L = Lg[0];
#pragma unroll
      for (int gg = 1; gg < 8; ++gg) {
        M = lane == gg ? Mg[gg] : M;
        L = lane == gg ? Lg[gg] : L;
      }
      a.part_m[prow + lane] = M;
      a.part_l[prow + lane] = L;
    }
    __syncwarp();
    // the records are dead: drop their L2 lines so they are never written back
    for (long long w2 = wf; w2 <= wl; ++w2) {
      const float* r2 = a.partials + static_cast<size_t>(2 * w2 + (w2 == wf ? slot_f : 0)) * REC;
      for (int ln = lane; ln < REC / 32; ln += 32) discard_l2_line(r2 + ln * 32);
    }
    if (lane == 0) a.counters[seq * Hkv + kvh] = 0;
    __syncwarp();
  };

  const int npro = min(S, nmine);
  for (int i = 0; i < npro; ++i) issue(i, i);

  int si = 0;
  uint32_t ph = 0;
  bool dead = false;
  int cur_seq = 0, cur_kvh = 0, seg_j0 = 0, prev_j = 0;
  bool first_seg = true;
  for (int i = 0; i < nmine; ++i) {
    const uint32_t st = wbase + static_cast<uint32_t>(si * STG);
    const bool arrived = __all_sync(FULL, mbar_wait_bounded(bar0 + 8u * si, ph, a.timeout_ns));
    if (!arrived) {
      for (int k = 0; k < S; ++k) {
        const int s2 = (si + k) % S;
        if ((armed >> s2) & 1u)
          mbar_wait_bounded(bar0 + 8u * s2, ph ^ ((si + k) >= S ? 1u : 0u), kDrainLimitNs);
      }
      dead = true;
      break;
    }
    armed &= ~(1u << si);
    const int seq = wmeta[si * 4 + 0], kvh = wmeta[si * 4 + 1], j = wmeta[si * 4 + 2];
    const int pk = wmeta[si * 4 + 3];
    const int okm = pk & 0xFF, nv = (pk >> 8) & 0xFF;
    if ((pk >> 16) & 1) {                          // a new segment starts with this tile
      if (i > 0) {
        finalize(cur_seq, cur_kvh, seg_j0, prev_j, first_seg);
        first_seg = false;
        wa.reset();
      }
      // its q rows (in L2 since the tile was issued)
      wa.load_q_global(reinterpret_cast<const QT*>(a.q) +
                           (static_cast<size_t>(seq) * a.num_heads +
                            static_cast<size_t>(kvh) * G + r) * D,
                       r < G, c);
      cur_seq = seq;
      cur_kvh = kvh;
      seg_j0 = j;
    }
    TileFrag<KIND, D, BS> fr;
    load_tile<QT, KIND, D, BS>(fr, st, lane);
    __syncwarp();
    if (i + S < nmine) issue(i + S, si);
    tile_compute<QT, KIND, D, BS>(wa, fr, nv, okm, a.scale_log2, lane);
    prev_j = j;
    if (++si == S) {
      si = 0;
      ph ^= 1u;
    }
  }
  if (dead) {
    if (lane == 0) report_error(a.err_flag, kErrTimeout);
  } else if (nmine > 0) {
    finalize(cur_seq, cur_kvh, seg_j0, prev_j, first_seg);
  }
  if (a.pdl == 3) {
    // the CTA that finishes last waits for the preceding grid, so whatever runs
    // after this grid also runs after that one
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      if (atomicAdd(a.done, 1) == static_cast<int>(gridDim.x) - 1) {
        griddep_wait();
        *a.done = 0;
      }
    }
  }
}

// --------------------------------------------------------------------------
// Host side
// --------------------------------------------------------------------------

static size_t fused_counter_bytes(int num_seqs, int num_kv_heads) {
  const size_t b = static_cast<size_t>(num_seqs) * num_kv_heads * sizeof(int);
  return (b + 255) / 256 * 256;
}

size_t fused_workspace_bytes(int num_seqs, int num_kv_heads, int head_dim, int num_sms) {
  const size_t warps = static_cast<size_t>(num_sms) * kFusedMaxCtasPerSm * kFusedWarps;
  return fused_counter_bytes(num_seqs, num_kv_heads) +
         2 * warps * fused_record_floats(head_dim) * sizeof(float);
}

namespace {

template <typename QT, int KIND, int D, int BS>
cudaError_t launch_fused_t(const FusedArgs& a0, size_t ws_bytes, cudaStream_t stream) {
  using T = Tr<KIND, D, BS>;
  FusedArgs a = a0;
  CUtensorMap mk, mv;
  cudaError_t e = make_cache_map<KIND, D, BS>(&mk, a.k_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  e = make_cache_map<KIND, D, BS>(&mv, a.v_cache, a.num_kv_heads, a.num_blocks);
  if (e != cudaSuccess) return e;
  const int smem = 1024 + kFusedWarps * a.stages * T::STAGE + 4 * (a.num_seqs + 1);
  auto kern = decode_fused_kernel<QT, KIND, D, BS, 1>;
  static int configured[64] = {0};
  static int configured3[64] = {0};
  int(*cfg)[64] = &configured;
  if constexpr (KIND == kKind16 && D == 128) {     // the cascade suffix's shapes
    if (a.ctas_per_sm == 3) {
      kern = decode_fused_kernel<QT, KIND, D, BS, 3>;
      cfg = &configured3;
    }
  }
  e = opt_in_smem(reinterpret_cast<const void*>(kern), smem, *cfg);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedWarps * 32, smem)) !=
      cudaSuccess)
    return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  if (per_sm > kFusedMaxCtasPerSm) per_sm = kFusedMaxCtasPerSm;
  if (a.ctas_per_sm > 0 && per_sm > a.ctas_per_sm) per_sm = a.ctas_per_sm;
  if (ws_bytes < fused_workspace_bytes(a.num_seqs, a.num_kv_heads, D, sms))
    return cudaErrorInvalidValue;
  char* ws = reinterpret_cast<char*>(a.counters);
  a.partials = reinterpret_cast<float*>(ws + fused_counter_bytes(a.num_seqs, a.num_kv_heads));
  const int use = a.sm_limit > 0 && a.sm_limit < sms ? a.sm_limit : sms;
  return launch_kernel(kern, dim3(use * per_sm), dim3(kFusedWarps * 32), smem, stream, a.pdl != 0,
                       mk, mv, a);
}

template <typename QT, int KIND>
cudaError_t fused_shape(const FusedArgs& a, int D, int BS, size_t ws, cudaStream_t s) {
#define PA_CASE(DD, BB) \
  if (D == DD && BS == BB) return launch_fused_t<QT, KIND, DD, BB>(a, ws, s);
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

cudaError_t launch_fused(const FusedArgs& a, int q_dtype, int cache_dtype, int head_dim,
                         int block_size, size_t workspace_bytes, cudaStream_t s) {
  const bool qh = q_dtype == PA_F16;
  switch (cache_dtype) {
    case PA_F16: return fused_shape<__half, kKind16>(a, head_dim, block_size, workspace_bytes, s);
    case PA_BF16:
      return fused_shape<__nv_bfloat16, kKind16>(a, head_dim, block_size, workspace_bytes, s);
    case PA_INT8:
      return qh ? fused_shape<__half, kKindI8>(a, head_dim, block_size, workspace_bytes, s)
                : fused_shape<__nv_bfloat16, kKindI8>(a, head_dim, block_size, workspace_bytes, s);
    case PA_FP8E4M3:
      return qh ? fused_shape<__half, kKindE4M3>(a, head_dim, block_size, workspace_bytes, s)
                : fused_shape<__nv_bfloat16, kKindE4M3>(a, head_dim, block_size, workspace_bytes,
                                                        s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace pa
