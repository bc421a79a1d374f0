// pa_decode.cu -- paged decode attention for sm_100a.
//
// Method: one query token per sequence attends over its cached K/V, which live in
// fixed-size physical blocks found through a per-sequence block table ("KV Cache memory
// optimisation and PagedAttention" (yunthe.com), section "PagedAttention注意力计算流程";
// "vLLM source first look: PagedAttention memory design" (trdm.cn), section 三: walk the
// cache block by block so each block's rows are read contiguously).
//
// B200 design (the pages' pseudocode -- one thread per token, one CTA per (head, seq) --
// is prior art only):
//   * Work unit = one physical block x a group of HG heads ("tile").  All tiles of all
//     sequences form one stream ordered (sequence, head group, block); a persistent grid
//     of C CTAs (a small multiple of the SM count) takes equal contiguous slices of it, so
//     ragged context lengths cost no load imbalance.  A slice that ends inside a
//     (sequence, head group) "segment" leaves a partial softmax state (m, l, acc) in the
//     workspace; a second kernel merges the partials of split segments.
//   * Inside a CTA, one producer warp walks the slice, reads block-table entries 32 at a
//     time, and issues one 3-D TMA load per tile for K and one for V ([bs, HG, D] boxes of
//     the [NB*bs, H, D] cache) into an NS-stage shared-memory ring guarded by mbarriers.
//     HG consumer warps (one per head) compute the scores with 16-byte shared loads and
//     warp-shuffle dot products, keep an online softmax (running max / sum, base 2), and
//     accumulate the probability-weighted V rows in fp32.
//   * HBM-bound: ~1 FMA per byte of fp16 K/V, far below the FP32 pipes' limit; tensor cores
//     have nothing dense to do with a single query row per head.
#include <cfloat>
#include <cstdio>
#include <mutex>
#include <type_traits>
#include <vector>

#include "pa_decode_shared.cuh"
#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tmap.h"

namespace pa {

// ---------------------------------------------------------------------------------------
// Partition kernel.
//   IO: q/out type; CT: cache element type; D: head_dim; TT: rows per tile if fixed, 0 = runtime.
// ---------------------------------------------------------------------------------------
// CTAs per SM the register allocation is sized for: 8-bit caches (2 CTAs per SM by shared
// memory) get the registers their widening needs without spilling; for 16-bit caches 3 keeps
// the 72-register allocation that measured fastest (92 registers with 1 ran ~4 % slower).
template <typename CT>
constexpr int partition_min_blocks() {
  return (std::is_same<CT, int8_t>::value || std::is_same<CT, __nv_fp8_e4m3>::value) ? 1 : 3;
}

template <typename IO, typename CT, int D, int TT>
__global__ void __launch_bounds__(kMaxThreads, partition_min_blocks<CT>())
decode_partition_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                        const DecodeParams p) {
  constexpr bool kInt8 = std::is_same<CT, int8_t>::value || std::is_same<CT, __nv_fp8_e4m3>::value;  // scaled 8-bit codes
  constexpr int E = Elem<CT>::kBytes;  // bytes per cache element
  constexpr int EV = Elem<CT>::kEV;    // cache elements per 16-byte vector (dims per lane)
  constexpr int LPR = D / EV;          // lanes covering one token row of one head
  constexpr int RPP = 32 / LPR;        // token rows per warp-wide pass
  constexpr int MAXP = TT > 0 ? (TT + RPP - 1) / RPP : (32 + RPP - 1) / RPP;
  static_assert(LPR >= 1 && LPR <= 32 && 32 % LPR == 0, "lane mapping");

  extern __shared__ __align__(128) uint8_t smem[];

  const int tt = TT > 0 ? TT : p.tt;
  const int HG = p.HG, G = p.G, NS = p.nstage, QW = p.QW;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Programmatic dependent launch: let the merge kernel get resident now, and wait for
  // the previous kernel of the stream (e.g. the cache write) before reading anything.
  grid_dependency_launch_next();
  grid_dependency_wait();

  // ---- 1. Plan: this CTA's slice of the tile stream. ------------------------------------
  __shared__ PlanScratch plan;
  Cursor start;
  long long t0 = 0;
  const long long count = plan_slice(p, plan, &t0, &start);
  if (count == 0) return;  // uniform across the CTA; no barrier in use yet

  // ---- 2. Pipeline barriers. --------------------------------------------------------
  const uint32_t bar_base = smem_u32(smem);
  const uint32_t stage_base = (bar_base + kBarrierBytes + 127u) & ~127u;  // TMA wants 128-B aligned tiles
  auto full_bar = [&](int st) { return bar_base + 8u * st; };
  auto empty_bar = [&](int st) { return bar_base + 8u * (NS + st); };
  if (threadIdx.x == 0) {
    for (int st = 0; st < NS; ++st) {
      mbar_init(full_bar(st), 1);
      mbar_init(empty_bar(st), QW);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int n = static_cast<int>(count);

  if (warp == QW) {
    // ---- 3. Producer warp: block-table lookups + TMA issue. --------------------------
    const uint64_t policy = l2_policy_evict_first();
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      if (kInt8) {
        prefetch_tensormap(&tmKs);
        prefetch_tensormap(&tmVs);
      }
    }
    Cursor c = start;
    int tab_seq = -1, tab_base = 0;
    int32_t tab = 0;
    int issued = 0;
    bool ok = true;
    for (; issued < n; ++issued) {
      const int ti = c.sp.first_t + c.j;  // tile index within the sequence
      const int lb = ti / p.tpb;          // logical block index
      if (c.s != tab_seq || lb - tab_base >= 32 || lb < tab_base) {
        tab_seq = c.s;
        tab_base = lb;
        const int idx = tab_base + lane;
        const int lb_end = (c.sp.first_t + c.sp.nb - 1) / p.tpb + 1;
        tab = idx < lb_end ? __ldg(p.block_tables + static_cast<size_t>(c.s) * p.MB + idx) : 0;
      }
      int pb = __shfl_sync(0xffffffffu, tab, lb - tab_base);
      if (pb < 0 || pb >= p.NB) {
        if (lane == 0) decode_error(PA_DEVERR_TABLE);
        pb = 0;
      }
      const int st = issued % NS;
      if (lane == 0) {
        if (issued >= NS && !mbar_wait_bounded(empty_bar(st), ((issued / NS) - 1) & 1)) {
          decode_error(PA_DEVERR_TIMEOUT);
          ok = false;
        }
        if (ok) {
          const uint32_t dst = stage_base + st * p.stage_bytes;
          const int head0 = c.g * HG, row0 = pb * p.bs + (ti % p.tpb) * tt;
          mbar_arrive_expect_tx(full_bar(st), p.tx_bytes);
          tma_load_3d(dst, &tmK, full_bar(st), 0, head0, row0, policy);
          tma_load_3d(dst + p.v_off, &tmV, full_bar(st), 0, head0, row0, policy);
          if (kInt8) {
            const int hx = head0 & ~7;  // 16-byte aligned x for the fp16 scale rows
            tma_load_2d(dst + p.ks_off, &tmKs, full_bar(st), hx, row0, policy);
            tma_load_2d(dst + p.vs_off, &tmVs, full_bar(st), hx, row0, policy);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      advance(c, p);
    }
    // Never leave the CTA with copies in flight: wait (bounded) for the last stages.
    if (lane == 0) {
      for (int k = issued - NS < 0 ? 0 : issued - NS; k < issued; ++k)
        if (!mbar_wait_bounded(full_bar(k % NS), (k / NS) & 1)) decode_error(PA_DEVERR_TIMEOUT);
    }
    return;
  }

  // ---- 4. Consumer warps: warp w owns query head g*QW + w of every tile, which reads ------
  //         cached head g*HG + w/GQ (grouped-query; GQ = 1 is multi-head attention).
  const int w = warp;
  const int kw = w / p.GQ;  // cached head of this warp within the tile
  const int r = lane / LPR;  // token row within a pass
  const int v = lane % LPR;  // 16-byte vector within the row: dims [v*EV, v*EV + EV)
  Cursor c = start;
  bool seg_from_start = (c.j == 0);
  // INT8 weighted sums of V: code + 128 spliced under the exponent of 1024 is the f16 value
  // 1152 + c, exactly, two codes per byte-permute; one f16 x f16 -> f32 FMA per code adds
  // w * (1152 + c) with the weight w = p * v_scale rounded to f16, and the bias 1152 * sum(w)
  // is removed once when the segment ends (the cancellation costs ~7 of fp32's 24 bits of the
  // biased sum; typical error ~1e-5 of the output scale against the 1e-2 tolerance).
  constexpr bool kBiasV = std::is_same<CT, int8_t>::value;
  // INT8 scores are integer dot products: q is held as 16-bit fixed point per row (row
  // maximum in [2^14, 2^15) steps), split into a signed high byte and an unsigned low byte;
  // each byte plane is dotted with four codes per dp4a instruction and the two sums are
  // combined as hi * 256 + lo, exactly, in int32 (|sum| < 2^27 for a lane's 16 dims, < 2^30
  // after the reduction over the row's 8 lanes).  The one rounding is that of q, to 2^-15
  // of its row maximum (finer than the f16 q of the FP8 path).
  constexpr bool kDp4a = std::is_same<CT, int8_t>::value;
  // FP8 scores and weighted sums run on f16 x f16 -> f32 fused multiply-adds: pairs of E4M3
  // codes convert exactly to f16 pairs, q is held in f16 after an exact power-of-two
  // rescaling of its row (row maximum in [2^14, 2^15)), the softmax weight p * v_scale is
  // rounded to f16 (relative 2^-11), and every product is exact in the fp32 accumulator.
  constexpr bool kMixed = std::is_same<CT, __nv_fp8_e4m3>::value;
  float qf[EV], acc[EV];
  float wsum = 0.f;        // INT8: sum of the f16 weights, for the bias of the V sum
  uint32_t qb[2][EV / 4];  // byte planes of the fixed-point q: [1] signed high, [0] unsigned low
  uint32_t qh2[EV / 2];    // f16 pairs of the rescaled q (FP8 cache)
  float q_unit = 1.f;      // factor from the raw dot product to the base-2 score (before the K scale)
  float m = -FLT_MAX, l = 0.f;  // running max (base 2) and sum; -FLT_MAX keeps exp2 finite
  auto load_q = [&](const Cursor& cc) {
    const int h = cc.g * QW + w;
    const IO* qrow = reinterpret_cast<const IO*>(p.q) + (static_cast<size_t>(cc.s) * p.Hq + h) * D + v * EV;
    load_floats<IO, EV>(qrow, qf);
    if constexpr (kMixed) {
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < EV; ++e) amax = fmaxf(amax, fabsf(qf[e]));
#pragma unroll
      for (int off = LPR / 2; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      int ex = 0;
      frexpf(amax, &ex);                          // amax < 2^ex
      const int E = max(-100, min(100, 15 - ex));  // amax * 2^E < 2^15: finite in f16
      const float up = ldexpf(1.f, E);
      q_unit = p.qscale * ldexpf(1.f, -E);
#pragma unroll
      for (int j = 0; j < EV / 2; ++j) {
        const __half2 h2 = __floats2half2_rn(qf[2 * j] * up, qf[2 * j + 1] * up);
        qh2[j] = *reinterpret_cast<const uint32_t*>(&h2);
      }
    } else {
#pragma unroll
      for (int e = 0; e < EV; ++e) qf[e] *= p.qscale;
    }
    if constexpr (kDp4a) {
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < EV; ++e) amax = fmaxf(amax, fabsf(qf[e]));
#pragma unroll
      for (int off = LPR / 2; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      int ex = 0;
      frexpf(amax, &ex);                           // amax < 2^ex
      const int E = max(-100, min(100, 15 - ex));  // amax * 2^E < 2^15
      const float up = ldexpf(1.f, E);
      q_unit = ldexpf(1.f, -E);
#pragma unroll
      for (int j = 0; j < EV / 4; ++j) {
        uint32_t w1 = 0, w0 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int qi = max(-32767, min(32767, __float2int_rn(qf[4 * j + k] * up)));
          w1 |= (static_cast<uint32_t>(qi >> 8) & 0xffu) << (8 * k);
          w0 |= (static_cast<uint32_t>(qi) & 0xffu) << (8 * k);
        }
        qb[1][j] = w1;
        qb[0][j] = w0;
      }
    }
  };
  load_q(c);
#pragma unroll
  for (int e = 0; e < EV; ++e) acc[e] = 0.f;

  for (int it = 0; it < n; ++it) {
    const int st = it % NS;
    if (!mbar_wait_bounded(full_bar(st), (it / NS) & 1)) {
      if (lane == 0) decode_error(PA_DEVERR_TIMEOUT);
      break;
    }
    const uint32_t kt = stage_base + st * p.stage_bytes;
    const uint32_t vt = kt + p.v_off;
    const int tok0 = (c.sp.first_t + c.j) * tt;  // logical index of the tile's first row
    const int hs = c.g * HG - ((c.g * HG) & ~7) + kw;  // head column in the 8-bit scale tile

    // Scores of this lane's rows (tokens pi*RPP + r), base-2 scaled.
    float sc[MAXP];
    float tile_max = -FLT_MAX;
#pragma unroll
    for (int pi = 0; pi < MAXP; ++pi) {
      sc[pi] = -INFINITY;
      if (TT > 0 || pi * RPP < tt) {  // warp-uniform
        const int t = pi * RPP + r;
        float part = 0.f;
        int ipart = 0;  // INT8: the exact integer dot product
        if (t < tt) {
          const uint4 kv = ld_shared_v4(kt + ((t * HG + kw) * D + v * EV) * E);
          if constexpr (kDp4a) {
            const uint32_t words[4] = {kv.x, kv.y, kv.z, kv.w};
            int a1 = 0, a0 = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              a1 = dp4a_ss(words[j], qb[1][j], a1);
              a0 = dp4a_su(words[j], qb[0][j], a0);
            }
            ipart = a1 * 256 + a0;
          } else if constexpr (kMixed) {
            const uint32_t words[4] = {kv.x, kv.y, kv.z, kv.w};
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t lo, hi;
              e4m3x4_to_f16x2x2(words[j], lo, hi);
              a0 = fma2_f16_f32(qh2[2 * j], lo, a0);
              a1 = fma2_f16_f32(qh2[2 * j + 1], hi, a1);
            }
            part = a0 + a1;
          } else {
            float kf[EV];
            Elem<CT>::to_float(kv, kf);
#pragma unroll
            for (int e = 0; e < EV; ++e) part = fmaf(qf[e], kf[e], part);
          }
        }
        if constexpr (kDp4a) {
#pragma unroll
          for (int off = LPR / 2; off >= 1; off >>= 1) ipart += __shfl_xor_sync(0xffffffffu, ipart, off);
          part = static_cast<float>(ipart);
        } else {
#pragma unroll
          for (int off = LPR / 2; off >= 1; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        }
        const int tok = tok0 + t;
        if (t < tt && tok >= c.sp.lo && tok < c.sp.ctx) {
          if (kInt8) part *= __half2float(__ushort_as_half(ld_shared_u16(kt + p.ks_off + (t * 8 + hs) * 2))) * q_unit;
          sc[pi] = part;
          tile_max = fmaxf(tile_max, part);
        }
      }
    }
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) tile_max = fmaxf(tile_max, __shfl_xor_sync(0xffffffffu, tile_max, off));

    // Online softmax update, then the probability-weighted V rows.
    const float m_new = fmaxf(m, tile_max);
    const float alpha = exp2f(m - m_new);
    m = m_new;
    l *= alpha;
#pragma unroll
    for (int e = 0; e < EV; ++e) acc[e] *= alpha;
    if (kBiasV) wsum *= alpha;
#pragma unroll
    for (int pi = 0; pi < MAXP; ++pi) {
      if (TT > 0 || pi * RPP < tt) {
        const int t = pi * RPP + r;
        if (sc[pi] != -INFINITY) {  // attended row (rows outside [lo, ctx) may hold garbage)
          const float pr = exp2f(sc[pi] - m);
          l += pr;
          const uint4 vv = ld_shared_v4(vt + ((t * HG + kw) * D + v * EV) * E);
          float pv = pr;
          if (kInt8) pv *= __half2float(__ushort_as_half(ld_shared_u16(kt + p.vs_off + (t * 8 + hs) * 2)));
          if constexpr (kBiasV) {
            const __half2 w2 = __float2half2_rn(pv);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(&w2);
            wsum += __low2float(w2);
            const uint32_t words[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t u = words[j] ^ 0x80808080u;
              fma_f16x2_f32x2(wb, __byte_perm(u, 0x6464u, 0x4140u), acc[4 * j], acc[4 * j + 1]);
              fma_f16x2_f32x2(wb, __byte_perm(u, 0x6464u, 0x4342u), acc[4 * j + 2], acc[4 * j + 3]);
            }
          } else if constexpr (kMixed) {
            const uint32_t words[4] = {vv.x, vv.y, vv.z, vv.w};
            const __half2 w2 = __float2half2_rn(pv);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(&w2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t lo, hi;
              e4m3x4_to_f16x2x2(words[j], lo, hi);
              fma_f16x2_f32x2(wb, lo, acc[4 * j], acc[4 * j + 1]);
              fma_f16x2_f32x2(wb, hi, acc[4 * j + 2], acc[4 * j + 3]);
            }
          } else {
            float vf[EV];
            Elem<CT>::to_float(vv, vf);
#pragma unroll
            for (int e = 0; e < EV; ++e) acc[e] = fmaf(pv, vf[e], acc[e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(st));

    const bool seg_last = (c.j == c.sp.nb - 1);
    if (seg_last || it == n - 1) {
      if constexpr (kBiasV)
#pragma unroll
        for (int e = 0; e < EV; ++e) acc[e] = fmaf(-1152.f, wsum, acc[e]);
      // Combine the RPP row groups of the warp.
      float lt = l;
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
        lt += __shfl_xor_sync(0xffffffffu, lt, off);
#pragma unroll
        for (int e = 0; e < EV; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
      }
      const int h = c.g * QW + w;
      if (seg_from_start && seg_last) {  // whole segment in this CTA: final output
        if (r == 0) {
          const float inv = 1.f / lt;
          float o[EV];
#pragma unroll
          for (int e = 0; e < EV; ++e) o[e] = acc[e] * inv;
          IO* orow = reinterpret_cast<IO*>(p.out) + (static_cast<size_t>(c.s) * p.Hq + h) * D + v * EV;
          store_floats<IO, EV>(orow, o);
        }
      } else {  // partial state for the merge kernel
        const long long slot = blockIdx.x + static_cast<long long>(c.s) * G + c.g;
        if (r == 0) {
          float4* dst = reinterpret_cast<float4*>(p.ws_acc + (slot * QW + w) * D + v * EV);
#pragma unroll
          for (int i = 0; i < EV / 4; ++i) dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
        }
        if (lane == 0) {
          p.ws_ml[(slot * QW + w) * 2 + 0] = m;
          p.ws_ml[(slot * QW + w) * 2 + 1] = lt;
        }
      }
      m = -FLT_MAX;
      l = 0.f;
      wsum = 0.f;
#pragma unroll
      for (int e = 0; e < EV; ++e) acc[e] = 0.f;
    }
    if (it + 1 < n) {
      advance(c, p);
      if (c.j == 0) {  // a new segment starts
        seg_from_start = true;
        load_q(c);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------
// Merge kernel: one warp per (sequence, head) combines the partial states of a segment that
// was split across CTAs:  M = max_k m_k,  out = sum_k 2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k.
// Sequences with nothing to attend get zeros; segments held by one CTA were written by it.
// Launched as a programmatic dependent of the partition kernel: the grid is resident while
// the partition kernel runs and proceeds the moment its results are visible.
// ---------------------------------------------------------------------------------------
constexpr int kMergeWarps = 8;

template <typename IO, int D>
__global__ void __launch_bounds__(32 * kMergeWarps) decode_merge_kernel(const DecodeParams p) {
  constexpr int DL = D / 32;  // dims per lane
  grid_dependency_wait();
  const int lane = threadIdx.x & 31;
  const long long item = static_cast<long long>(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  if (item >= static_cast<long long>(p.S) * p.Hq) return;
  const int s = static_cast<int>(item / p.Hq), h = static_cast<int>(item % p.Hq);
  // The plan's unit stream (tiles plus seg_units per segment; see plan_slice).
  const long long per_group = p.ws_prefix[p.S];
  const long long pre = p.ws_prefix[s];
  const long long su = p.ws_prefix[s + 1] - pre;  // units of one head group of this sequence
  const long long nb = su > 0 ? su - p.seg_units : 0;
  IO* orow = reinterpret_cast<IO*>(p.out) + (static_cast<size_t>(s) * p.Hq + h) * D + lane * DL;
  float o[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = 0.f;
  if (nb == 0) {
#pragma unroll
    for (int e = 0; e < DL; ++e) orow[e] = float_to<IO>(0.f);
    return;
  }
  const long long U = per_group * p.G;
  const int g = h / p.QW, w = h % p.QW;
  const long long a = p.G * pre + g * su + p.seg_units;  // unit of the segment's first tile
  const int c0 = cta_of(a, U, p.num_ctas), c1 = cta_of(a + nb - 1, U, p.num_ctas);
  if (c0 == c1) return;
  const long long seg = static_cast<long long>(s) * p.G + g;
  const float2* ml = reinterpret_cast<const float2*>(p.ws_ml);
  // Global max over the partials, 32 partials per round (one per lane).
  float M = -FLT_MAX;
  for (int k = c0 + lane; k <= c1; k += 32) M = fmaxf(M, ml[(k + seg) * p.QW + w].x);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
#pragma unroll 4
  for (int k = c0; k <= c1; ++k) {
    const long long row = (k + seg) * p.QW + w;
    const float2 st = ml[row];
    const float f = exp2f(st.x - M);
    L = fmaf(f, st.y, L);
    const float* src = p.ws_acc + row * D + lane * DL;
#pragma unroll
    for (int e = 0; e < DL; ++e) o[e] = fmaf(f, src[e], o[e]);
  }
  const float inv = 1.f / L;
#pragma unroll
  for (int e = 0; e < DL; ++e) orow[e] = float_to<IO>(o[e] * inv);
}

// ---------------------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------------------
namespace {

cudaError_t read_decode_error(uint32_t* flags, int clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_decode_error, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (clear && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_decode_error, &z, sizeof z);
  }
  return e;
}

struct RegisterDecode {
  RegisterDecode() { register_device_error_reader(read_decode_error); }
} g_register_decode;

size_t elem_bytes(pa_dtype t) { return t == PA_F32 ? 4 : ((t == PA_I8 || t == PA_FP8_E4M3) ? 1 : 2); }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout for `rows` = (partial slots x heads per slot) rows.
struct WsLayout {
  size_t prefix_off, ml_off, acc_off, total;
};
WsLayout ws_layout(int S, int D, long long rows) {
  WsLayout l;
  l.prefix_off = 0;
  l.ml_off = align256(sizeof(long long) * (static_cast<size_t>(S) + 1));
  l.acc_off = l.ml_off + align256(sizeof(float) * 2 * static_cast<size_t>(rows));
  l.total = l.acc_off + align256(sizeof(float) * static_cast<size_t>(D) * rows);
  return l;
}

// Cached heads per CTA: the largest power of two <= cap dividing H with K+V tiles of one
// stage <= 32 KiB.
int pick_head_group(int H, int tt, int D, size_t e, int cap) {
  int hg = cap;
  while (hg > 1 && (H % hg != 0 || 2 * static_cast<size_t>(tt) * hg * D * e > 32768)) hg >>= 1;
  return hg;
}

struct KernelInfo {
  const void* fn = nullptr;
  int smem_configured = 0;
};

template <typename IO, typename CT, int D>
const void* partition_kernel_for(int tt) {
  switch (tt) {
    case 8: return reinterpret_cast<const void*>(&decode_partition_kernel<IO, CT, D, 8>);
    case 16: return reinterpret_cast<const void*>(&decode_partition_kernel<IO, CT, D, 16>);
    default: return reinterpret_cast<const void*>(&decode_partition_kernel<IO, CT, D, 0>);
  }
}

template <typename IO, typename CT>
const void* partition_kernel_for(int D, int bs) {
  return D == 64 ? partition_kernel_for<IO, CT, 64>(bs) : partition_kernel_for<IO, CT, 128>(bs);
}

const void* select_partition(pa_dtype io, pa_dtype cache, int D, int bs) {
  if (cache == PA_I8) {
    return io == PA_F16 ? partition_kernel_for<__half, int8_t>(D, bs)
                        : partition_kernel_for<__nv_bfloat16, int8_t>(D, bs);
  }
  if (cache == PA_FP8_E4M3) {
    return io == PA_F16 ? partition_kernel_for<__half, __nv_fp8_e4m3>(D, bs)
                        : partition_kernel_for<__nv_bfloat16, __nv_fp8_e4m3>(D, bs);
  }
  switch (io) {
    case PA_F32: return partition_kernel_for<float, float>(D, bs);
    case PA_F16: return partition_kernel_for<__half, __half>(D, bs);
    default: return partition_kernel_for<__nv_bfloat16, __nv_bfloat16>(D, bs);
  }
}

const void* select_merge(pa_dtype io, int D) {
  switch (io) {
    case PA_F32: return D == 64 ? reinterpret_cast<const void*>(&decode_merge_kernel<float, 64>)
                                : reinterpret_cast<const void*>(&decode_merge_kernel<float, 128>);
    case PA_F16: return D == 64 ? reinterpret_cast<const void*>(&decode_merge_kernel<__half, 64>)
                                : reinterpret_cast<const void*>(&decode_merge_kernel<__half, 128>);
    default: return D == 64 ? reinterpret_cast<const void*>(&decode_merge_kernel<__nv_bfloat16, 64>)
                            : reinterpret_cast<const void*>(&decode_merge_kernel<__nv_bfloat16, 128>);
  }
}

// Make `fn` launchable with `smem` bytes of dynamic shared memory and return its occupancy.
// The per-kernel dynamic-smem limit is a global attribute of the function: it is only ever
// raised (lowering it for a small ring would break a later launch with a larger one).  The
// occupancy answers are cached per (kernel, block size, smem).  Thread-safe.
pa_status occupancy(const void* fn, int threads, size_t smem, int* occ) {
  struct Entry { const void* fn; int threads; size_t smem; int occ; };
  struct Limit { const void* fn; size_t smem; };
  static std::mutex m;
  static std::vector<Entry> cache;
  static std::vector<Limit> limits;
  std::lock_guard<std::mutex> lock(m);
  for (const Entry& en : cache)
    if (en.fn == fn && en.threads == threads && en.smem == smem) {
      *occ = en.occ;
      return PA_OK;
    }
  Limit* lim = nullptr;
  for (Limit& l : limits)
    if (l.fn == fn) lim = &l;
  if (!lim || lim->smem < smem) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(MaxDynamicSharedMemorySize)");
    if (lim) lim->smem = smem;
    else limits.push_back(Limit{fn, smem});
  }
  int o = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, fn, threads, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveBlocksPerMultiprocessor");
  cache.push_back(Entry{fn, threads, smem, o});
  *occ = o;
  return PA_OK;
}

bool valid_pair(pa_dtype io, pa_dtype cache) {
  if (io == PA_F32) return cache == PA_F32;
  if (io == PA_F16) return cache == PA_F16 || cache == PA_I8 || cache == PA_FP8_E4M3;
  if (io == PA_BF16) return cache == PA_BF16 || cache == PA_I8 || cache == PA_FP8_E4M3;
  return false;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim) {
  if (num_seqs < 0 || num_heads <= 0 || (head_dim != 64 && head_dim != 128)) return 0;
  int dev = 0, sms = 0;
  if (current_device(&dev, &sms) != PA_OK) return 0;
  const long long rows = static_cast<long long>(sms) * kMaxCtasPerSm * kMaxHeadGroup +
                         static_cast<long long>(num_seqs) * num_heads;
  return ws_layout(num_seqs, head_dim, rows).total;
}

namespace pa {
namespace {

bool g_tensor_cores = true;  // pa_decode_use_tensor_cores()

// Grouped-query decode on the tensor cores: one CTA per SM (two for 8-bit caches with up to
// 8 query heads per cached head), 128-token tiles of one cached head (pa_decode_tc.cu,
// pa_decode_tc8.cu), then the shared merge kernel.
pa_status decode_launch_tc(void* out, const void* q, const void* k_cache, const void* v_cache, const void* k_scale,
                           const void* v_scale, const int32_t* block_tables, const int32_t* context_lens,
                           int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                           int num_blocks, int max_blocks_per_seq, float scale, int window, pa_dtype io_dtype,
                           pa_dtype cache_dtype, void* workspace, int sms, cudaStream_t s) {
  const int SG = tc_decode_subgroup(num_q_heads / num_kv_heads);  // query heads per head group
  const int NSUB = num_q_heads / num_kv_heads / SG;               // head groups per cached head
  const int GQ = SG;
  const bool eight_bit = cache_dtype != io_dtype;  // INT8 or FP8 codes with per-token scales
  const int C = sms * (eight_bit ? tc8_ctas_per_sm(GQ) : 1);
  const long long rows = static_cast<long long>(C) * GQ + static_cast<long long>(num_seqs) * num_q_heads;
  const WsLayout lay = ws_layout(num_seqs, head_dim, rows);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  EncodeTiledFn enc = nullptr;
  pa_status st = get_encoder(&enc);
  if (st != PA_OK) return st;
  const CUtensorMapDataType ttype = io_dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tmK, tmV, tmQ, tmKs, tmVs;
  if (!eight_bit) {
    // [NB*bs rows][Hkv][head_dim]: boxes of one block's rows x one head x 64 dims, 128-byte swizzle
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * 2,
                                   static_cast<cuuint64_t>(num_kv_heads) * head_dim * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(block_size)};
    if ((st = encode(enc, &tmK, ttype, 3, k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    if ((st = encode(enc, &tmV, ttype, 3, v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    tmKs = tmK;
    tmVs = tmV;
  } else {
    // 8-bit codes [NB*bs rows][Hkv][128 B]: one block's rows x one head x all 128 dims,
    // 128-byte swizzle; scales [NB*bs rows][Hkv] fp16: one block's rows x 8 heads (16 B)
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(num_kv_heads) * 128};
    const cuuint32_t box[3] = {128, 1, static_cast<cuuint32_t>(block_size)};
    const CUtensorMapDataType ctype = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if ((st = encode(enc, &tmK, ctype, 3, k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    if ((st = encode(enc, &tmV, ctype, 3, v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    const cuuint64_t sdims[2] = {static_cast<cuuint64_t>(num_kv_heads), static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t sstrides[1] = {static_cast<cuuint64_t>(num_kv_heads) * 2};
    const cuuint32_t sbox[2] = {8, static_cast<cuuint32_t>(block_size)};
    if ((st = encode(enc, &tmKs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, k_scale, sdims, sstrides, sbox)) != PA_OK) return st;
    if ((st = encode(enc, &tmVs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, v_scale, sdims, sstrides, sbox)) != PA_OK) return st;
  }
  {
    // q as [S*Hq rows][head_dim]: the GQ rows of one head group x 64 dims
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_seqs) * num_q_heads};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(head_dim) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(GQ)};
    if ((st = encode(enc, &tmQ, ttype, 2, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
  }
  DecodeParams prm = {};
  prm.out = out;
  prm.q = q;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.ws_prefix = reinterpret_cast<long long*>(ws + lay.prefix_off);
  prm.ws_ml = reinterpret_cast<float*>(ws + lay.ml_off);
  prm.ws_acc = reinterpret_cast<float*>(ws + lay.acc_off);
  prm.S = num_seqs;
  prm.H = num_kv_heads;
  prm.bs = block_size;
  prm.MB = max_blocks_per_seq;
  prm.NB = num_blocks;
  prm.window = window;
  prm.tt = tc_decode_tile_tokens();
  prm.tpb = 1;
  prm.HG = 1;
  prm.G = num_kv_heads * NSUB;
  prm.num_ctas = C;
  prm.nstage = 0;
  prm.Hq = num_q_heads;
  prm.GQ = GQ;
  prm.QW = GQ;
  prm.sub = NSUB;
  prm.dim = head_dim;
  // A segment's end (denominators, output or partial written, the pipeline refilled) costs
  // about one tile on the tensor-core kernels: CTAs whose shares hold many short segments
  // finished last when the stream was split by tiles alone.
  prm.seg_units = 1;
  prm.qscale = scale * 1.4426950408889634f;

  cudaEvent_t ev[3];
  profiling_next_events(ev);
  if (ev[0]) cudaEventRecord(ev[0], s);
  if ((st = tc_decode_launch(tmK, tmV, tmQ, tmKs, tmVs, prm, io_dtype, cache_dtype, C, s)) != PA_OK) return st;
  if (ev[1]) cudaEventRecord(ev[1], s);
  {
    void* args[] = {&prm};
    const long long items = static_cast<long long>(num_seqs) * num_q_heads;
    const unsigned grid = static_cast<unsigned>((items + kMergeWarps - 1) / kMergeWarps);
    cudaError_t err = launch_dependent(select_merge(io_dtype, head_dim), dim3(grid), dim3(32 * kMergeWarps), 0, s, args);
    if (err != cudaSuccess) return cuda_fail(err, "launching the decode merge kernel");
  }
  if (ev[2]) cudaEventRecord(ev[2], s);
  return PA_OK;
}

pa_status decode_launch(void* out, const void* q, const void* k_cache, const void* v_cache,
                                            const void* k_scale, const void* v_scale, const int32_t* block_tables,
                                            const int32_t* context_lens, int num_seqs, int num_q_heads, int num_heads, int head_dim,
                                            int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                                            int window, pa_dtype io_dtype, pa_dtype cache_dtype, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  // ---- host validation (no CUDA call before this block passes) ----
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "num_seqs < 0");
  if (num_heads <= 0 || num_heads > 4096 || num_q_heads <= 0 || num_q_heads > 4096)
    return fail(PA_ERR_INVALID_ARG, "head counts must be in [1, 4096]");
  if (num_q_heads % num_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "num_q_heads (%d) must be a multiple of num_kv_heads (%d)", num_q_heads, num_heads);
  const int GQ = num_q_heads / num_heads;  // query heads per cached head
  const bool use_tc = g_tensor_cores && tc_decode_eligible(io_dtype, cache_dtype, head_dim, block_size, GQ);
  if (GQ > kMaxHeadGroup && !use_tc)
    return fail(PA_ERR_UNSUPPORTED,
                "%d query heads per cached head: up to %d on the CUDA-core kernel; more need the tensor-core "
                "kernel (fp16/bf16 io, head_dim 128, block_size a multiple of 8 dividing 128, and a group "
                "of up to 16 or with a divisor in [4, 16])",
                GQ, kMaxHeadGroup);
  if (head_dim != 64 && head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", head_dim);
  if (block_size < 1 || block_size > 32) return fail(PA_ERR_UNSUPPORTED, "block_size %d (supported: 1..32)", block_size);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0) return fail(PA_ERR_INVALID_ARG, "num_blocks and max_blocks_per_seq must be positive");
  if (static_cast<long long>(num_blocks) * block_size > 0x7fffffffLL ||
      static_cast<long long>(max_blocks_per_seq) * block_size > 0x7fffffffLL)
    return fail(PA_ERR_INVALID_ARG, "num_blocks*block_size and max_blocks_per_seq*block_size must fit in int32");
  if (window < 0) return fail(PA_ERR_INVALID_ARG, "window must be >= 0 (0 = full attention)");
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return fail(PA_ERR_INVALID_ARG, "scale is not finite");
  if (!valid_pair(io_dtype, cache_dtype))
    return fail(PA_ERR_INVALID_ARG, "dtype pair (io %d, cache %d) not supported: cache must equal io, or be PA_I8 / PA_FP8_E4M3 with fp16/bf16 io",
                static_cast<int>(io_dtype), static_cast<int>(cache_dtype));
  const bool int8 = cache_dtype == PA_I8 || cache_dtype == PA_FP8_E4M3;  // scaled 8-bit cache
  if (int8 && (num_heads % 8 != 0)) return fail(PA_ERR_UNSUPPORTED, "an INT8 or FP8 cache needs num_heads to be a multiple of 8");
  if (num_seqs == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
    return fail(PA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (int8 && (!k_scale || !v_scale)) return fail(PA_ERR_INVALID_ARG, "INT8 and FP8 caches need k_scale and v_scale");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (int8 && (!aligned16(k_scale) || !aligned16(v_scale))) || !aligned16(workspace))
    return fail(PA_ERR_INVALID_ARG, "tensor base addresses must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(block_tables) % 4 || reinterpret_cast<uintptr_t>(context_lens) % 4)
    return fail(PA_ERR_INVALID_ARG, "block_tables / context_lens must be 4-byte aligned");

  // ---- launch configuration ----
  int dev = 0, sms = 0;
  pa_status st = current_device(&dev, &sms);
  if (st != PA_OK) return st;
  const size_t need = pa_decode_workspace_bytes(num_seqs, num_q_heads, head_dim);
  if (workspace_bytes < need)
    return fail(PA_ERR_INVALID_ARG, "workspace too small: %zu bytes given, %zu needed", workspace_bytes, need);
  if (use_tc)
    return decode_launch_tc(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_seqs,
                            num_q_heads, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                            window, io_dtype, cache_dtype, workspace, sms, static_cast<cudaStream_t>(stream));

  // Rows per tile: the largest divisor of block_size in [8, 16] (the whole block if none),
  // so 32-token blocks stream as two 16-row tiles and keep four heads per CTA.
  int tt = block_size;
  for (int d = 16; d >= 8; --d)
    if (block_size % d == 0) {
      tt = d;
      break;
    }
  const size_t e = elem_bytes(cache_dtype);
  const int HG = pick_head_group(num_heads, tt, head_dim, e, kMaxHeadGroup / GQ);
  const int QW = HG * GQ;  // consumer warps: one per query head of the tile
  const int G = num_heads / HG;
  const uint32_t kv_tile = static_cast<uint32_t>(tt) * HG * head_dim * e;
  const uint32_t kv_tile_al = (kv_tile + 127u) & ~127u;
  const uint32_t sc_tile = int8 ? static_cast<uint32_t>(tt) * 8 * 2 : 0;
  const uint32_t sc_tile_al = (sc_tile + 127u) & ~127u;
  const uint32_t stage_bytes = 2 * kv_tile_al + 2 * sc_tile_al;
  int nstage = static_cast<int>((96 * 1024) / stage_bytes);
  nstage = nstage < 2 ? 2 : (nstage > 8 ? 8 : nstage);
  const size_t smem = kBarrierBytes + 128 + static_cast<size_t>(nstage) * stage_bytes;
  const int threads = 32 * (QW + 1);

  const void* part_fn = select_partition(io_dtype, cache_dtype, head_dim, tt);
  const void* merge_fn = select_merge(io_dtype, head_dim);
  int occ = 0;
  st = occupancy(part_fn, threads, smem, &occ);
  if (st != PA_OK) return st;
  if (occ <= 0) return fail(PA_ERR_CUDA, "partition kernel cannot be resident (smem %zu)", smem);
  const int C = sms * (occ < kMaxCtasPerSm ? occ : kMaxCtasPerSm);

  const long long rows = static_cast<long long>(C) * QW + static_cast<long long>(num_seqs) * num_q_heads;
  const WsLayout lay = ws_layout(num_seqs, head_dim, rows);
  uint8_t* ws = static_cast<uint8_t*>(workspace);

  // ---- tensor maps ----
  EncodeTiledFn enc = nullptr;
  st = get_encoder(&enc);
  if (st != PA_OK) return st;
  const CUtensorMapDataType ttype = cache_dtype == PA_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : cache_dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                  : cache_dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap tmK, tmV, tmKs, tmVs;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_heads),
                                static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(head_dim) * e, static_cast<cuuint64_t>(num_heads) * head_dim * e};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(head_dim), static_cast<cuuint32_t>(HG),
                               static_cast<cuuint32_t>(tt)};
    if ((st = encode(enc, &tmK, ttype, 3, k_cache, dims, strides, box)) != PA_OK) return st;
    if ((st = encode(enc, &tmV, ttype, 3, v_cache, dims, strides, box)) != PA_OK) return st;
  }
  if (int8) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(num_heads), static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(num_heads) * 2};
    const cuuint32_t box[2] = {8, static_cast<cuuint32_t>(tt)};
    if ((st = encode(enc, &tmKs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, k_scale, dims, strides, box)) != PA_OK) return st;
    if ((st = encode(enc, &tmVs, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, v_scale, dims, strides, box)) != PA_OK) return st;
  } else {
    tmKs = tmK;
    tmVs = tmV;
  }

  DecodeParams prm = {};
  prm.out = out;
  prm.q = q;
  prm.block_tables = block_tables;
  prm.context_lens = context_lens;
  prm.ws_prefix = reinterpret_cast<long long*>(ws + lay.prefix_off);
  prm.ws_ml = reinterpret_cast<float*>(ws + lay.ml_off);
  prm.ws_acc = reinterpret_cast<float*>(ws + lay.acc_off);
  prm.S = num_seqs;
  prm.H = num_heads;
  prm.bs = block_size;
  prm.tt = tt;
  prm.tpb = block_size / tt;
  prm.MB = max_blocks_per_seq;
  prm.NB = num_blocks;
  prm.window = window;
  prm.HG = HG;
  prm.Hq = num_q_heads;
  prm.GQ = GQ;
  prm.QW = QW;
  prm.G = G;
  prm.sub = 1;
  prm.dim = head_dim;
  prm.seg_units = 0;  // the stream is split by tiles alone
  prm.num_ctas = C;
  prm.nstage = nstage;
  prm.qscale = scale * 1.4426950408889634f;  // log2(e): exp(x) = 2^(x log2 e)
  prm.stage_bytes = stage_bytes;
  prm.v_off = kv_tile_al;
  prm.ks_off = 2 * kv_tile_al;
  prm.vs_off = 2 * kv_tile_al + sc_tile_al;
  prm.tx_bytes = 2 * kv_tile + 2 * sc_tile;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev[3];
  profiling_next_events(ev);
  if (ev[0]) cudaEventRecord(ev[0], s);

  {
    void* args[] = {&tmK, &tmV, &tmKs, &tmVs, &prm};
    cudaError_t err = launch_dependent(part_fn, dim3(C), dim3(threads), smem, s, args);
    if (err != cudaSuccess) return cuda_fail(err, "launching the decode partition kernel");
  }
  if (ev[1]) cudaEventRecord(ev[1], s);
  {
    void* args[] = {&prm};
    const long long items = static_cast<long long>(num_seqs) * num_q_heads;
    const unsigned grid = static_cast<unsigned>((items + kMergeWarps - 1) / kMergeWarps);
    cudaError_t err = launch_dependent(merge_fn, dim3(grid), dim3(32 * kMergeWarps), 0, s, args);
    if (err != cudaSuccess) return cuda_fail(err, "launching the decode merge kernel");
  }
  if (ev[2]) cudaEventRecord(ev[2], s);
  return PA_OK;
}
}  // namespace
}  // namespace pa

extern "C" pa_status paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                                            const void* k_scale, const void* v_scale, const int32_t* block_tables,
                                            const int32_t* context_lens, int num_seqs, int num_heads, int head_dim,
                                            int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                                            int window, pa_dtype io_dtype, pa_dtype cache_dtype, void* workspace,
                                            size_t workspace_bytes, void* stream) {
  return decode_launch(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_seqs, num_heads,
                       num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, scale, window, io_dtype,
                       cache_dtype, workspace, workspace_bytes, stream);
}

extern "C" pa_status paged_attention_decode_gqa(void* out, const void* q, const void* k_cache, const void* v_cache,
                                                const void* k_scale, const void* v_scale, const int32_t* block_tables,
                                                const int32_t* context_lens, int num_seqs, int num_q_heads,
                                                int num_kv_heads, int head_dim, int block_size, int num_blocks,
                                                int max_blocks_per_seq, float scale, int window, pa_dtype io_dtype,
                                                pa_dtype cache_dtype, void* workspace, size_t workspace_bytes,
                                                void* stream) {
  return decode_launch(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_seqs,
                       num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, scale, window,
                       io_dtype, cache_dtype, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc: a plugin living inside a host framework that owns
// every byte of device memory and hands out nothing but the tensors of the op, or a
// latency-critical loop where cudaMalloc's implicit device synchronisation is not
// acceptable.  For them the split-softmax scratch lives in a fixed array in the library's
// own device memory (kStaticScratchBytes on every GPU that loads the library, held until
// the process exits).  The array's host-side name is only a stand-in for it, so its device
// address is looked up once per device with cudaGetSymbolAddress (on the first call on
// that device, which must therefore come before any stream capture) and that address is
// handed to paged_attention_decode.
// ---------------------------------------------------------------------------------------
namespace pa {
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

pa_status static_scratch_address(void** out) {
  static std::mutex m;
  static void* addr[256] = {nullptr};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 256) return fail(PA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(m);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static decode scratch)");
    addr[dev] = p;
  }
  *out = addr[dev];
  return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" pa_status paged_attention_decode_static_scratch(
    void* out, const void* q, const void* k_cache, const void* v_cache, const void* k_scale, const void* v_scale,
    const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_heads, int head_dim,
    int block_size, int num_blocks, int max_blocks_per_seq, float scale, int window, pa_dtype io_dtype,
    pa_dtype cache_dtype, void* stream) {
  if (num_seqs == 0) return PA_OK;
  const size_t need = pa_decode_workspace_bytes(num_seqs, num_heads, head_dim);
  if (need == 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_decode_static_scratch: invalid sizes or no CUDA device");
  if (need > kStaticScratchBytes)
    return fail(PA_ERR_INVALID_ARG,
                "paged_attention_decode_static_scratch: %d sequences x %d heads x %d dims need %zu bytes of "
                "scratch, above the built-in %zu; use paged_attention_decode with a workspace",
                num_seqs, num_heads, head_dim, need, kStaticScratchBytes);
  void* scratch = nullptr;
  pa_status st = static_scratch_address(&scratch);
  if (st != PA_OK) return st;
  return paged_attention_decode(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, context_lens, num_seqs,
                                num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, scale, window,
                                io_dtype, cache_dtype, scratch, kStaticScratchBytes, stream);
}

extern "C" pa_status pa_decode_use_tensor_cores(int enable) {
  g_tensor_cores = enable != 0;
  return PA_OK;
}
