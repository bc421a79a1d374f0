// pa_decode_tc.cu -- grouped-query paged decode on the 5th-generation tensor cores (sm_100a).
//
// With GQ query heads sharing one cached head, every cached K/V byte feeds GQ dot products
// and GQ weighted sums.  At 8 query heads per cached head that is more FP32 FMA work per
// HBM byte than the CUDA cores can retire at full bandwidth, so here the two contractions
// of a 128-token tile run as tcgen05 MMAs with fp32 accumulators in tensor memory (TMEM):
//
//   S^T[128 tok x 16]  = K[128 tok x 128 d] . Q^T[128 d x 16 heads]     (K-major A, K-major B)
//   O^T[128 d   x 16]  = V^T[128 d x 128 tok] . P^T[128 tok x 16 heads] (MN-major A and B)
//
// (query heads padded to N = 16; M = 128 puts one token, then one head dim, on each TMEM lane).
// A cached head with more than 16 query heads (multi-query attention) is split into query
// sub-groups of at most 16 that form head groups of their own and read the same cached
// head; consecutive sub-groups are neighbouring segments of the tile stream, so their
// copies of the same tiles mostly meet in L2.
// The pages fix only the cache layout and the block-table walk ("KV Cache memory
// optimisation and PagedAttention" (yunthe.com), section "PagedAttention注意力计算流程";
// "vLLM source first look: PagedAttention memory design" (trdm.cn), section 三); the
// grouped-query tile is this library's design.
//
// Roles (one CTA per SM, 14 warps):
//   warps 0,6-8 TMA producers, one per part of a tile (K or V, 64-dim half, 128-byte
//               swizzle): each issues its part of every attended block into a 3-stage ring
//               (warp 0 also the q rows of the head group); block-table entries are loaded
//               by the lanes in parallel.
//   warp 1      TMEM owner and MMA issuer (one lane); with up to 8 query heads per cached
//               head warp 9 issues the value MMAs and warp 1 only the score MMAs.
//   warps 2..5, 10..13  softmax (thread = token row of S^T) and accumulation (thread = head
//               dim row of O^T), two warps per TMEM lane quarter, each with half of the
//               row's query heads: online softmax in base 2, probabilities written as the B
//               operand of the value MMA, V rows of unattended tokens zeroed, running output
//               rescaled in registers.  Segment ends write the output or a partial (m, l,
//               acc) exactly like the CUDA-core kernel, so the same merge kernel finishes
//               split segments.
// 8-bit caches run on the kernel of pa_decode_tc8.cu, which feeds the codes to the tensor
// cores as they are.
// Every wait is bounded; a wait that gives up sets an abort flag that ends all the others.
#include <algorithm>
#include <cfloat>
#include <mutex>
#include <type_traits>
#include <vector>

#include "pa_decode_shared.cuh"
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {
namespace {

constexpr int kTokens = 128;                    // tile rows (MMA M of the score product)
constexpr int kDim = 128;                       // head_dim (64: the hi halves stay unused)
constexpr int kHeadsN = 16;                     // query heads per cached head, padded (MMA N)
constexpr int kHalf = kTokens * 128;            // one 64-dim half of a tile: 128 rows x 128 B
constexpr int kQHalf = kHeadsN * 128;           // one 64-dim half of the q rows: 16 rows x 128 B
// Stage: K lo, K hi, V lo, V hi, Q lo, Q hi.
constexpr int kStageBytes = 4 * kHalf + 2 * kQHalf;
constexpr int kStages = 3;
constexpr int kPBytes = kTokens * kHeadsN * 2;  // one probability operand, 128 tokens x 16 heads
// Threads of the kernel tracking NH query heads per row: TMA warps 0 and 6..8, MMA warps
// 1 and 9, softmax warps 2..5 (and 10..13 when NH = 16: two warps per TMEM lane quarter,
// 8 heads each).
constexpr int base_threads(int) { return 448; }
static_assert(base_threads(16) <= kMaxPlanThreads, "plan_slice keeps one scratch entry per thread");
constexpr uint32_t kTmemCols = 64;              // S0 [0,16)  S1 [16,32)  O0 [32,48)  O1 [48,64)
// Probability operands: 2 tiles in flight x (hi, lo) parts for a bf16 cache, x 1 part otherwise.
// The plan scratch shares their space (the plan is done before the first one is written).
constexpr int p_parts(bool split) { return split ? 2 : 1; }
constexpr size_t smem_bytes(bool split) {
  return 1024 + static_cast<size_t>(kStages) * kStageBytes + 2 * p_parts(split) * kPBytes;
}
static_assert(sizeof(PlanScratch) <= 2 * kPBytes, "plan scratch fits the probability buffers");

struct TcShared {
  uint64_t full[kStages], empty[kStages];       // TMA ring
  uint64_t s_full[2], s_empty[2];               // score accumulators in TMEM
  uint64_t p_full[2], o_full[2];                // probabilities written / value MMA done
  uint64_t mma_done;                            // both MMA warps' last MMAs finished
  uint32_t tmem_base;
  int abort;
  float red[2][4][kHeadsN];                     // per-tile maxima across the softmax warps (by tile parity)
  float red_l[4][kHeadsN];                      // softmax denominators at segment ends
  int stop[2];                                  // abort flag as seen before a tile's exchange barrier
};

__device__ __forceinline__ uint32_t bits16(__half x) { return __half_as_ushort(x); }
__device__ __forceinline__ uint32_t bits16(__nv_bfloat16 x) { return __bfloat16_as_ushort(x); }

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
  }
  *abort = 1;
  decode_error(PA_DEVERR_TIMEOUT);
  return false;
}

// Rows of a probability operand P^T (MN-major, 32-byte swizzle): 16 heads = 32 B, the two
// 16-byte chunks trade places on rows 4..7 of every 8.
// Heads 4 * hh .. 4 * hh + 3 of row r only (8 bytes of the first 16-byte chunk).
__device__ __forceinline__ void store_p_quarter_row(uint32_t buf, int r, int hh, const uint32_t* w) {
  const uint32_t sw = (r >> 2) & 1;
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(buf + r * 32 + 16 * sw + 8 * hh), "r"(w[0]), "r"(w[1])
               : "memory");
}
// Heads 8 * hh .. 8 * hh + 7 of row r only (the other 16-byte chunk belongs to another warp).
__device__ __forceinline__ void store_p_half_row(uint32_t buf, int r, int hh, const uint32_t* w) {
  const uint32_t sw = (r >> 2) & 1;
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(buf + r * 32 + 16 * (hh ^ sw)), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]) : "memory");
}

// IO: fp16 or bf16 queries and cache.  NH: query heads of a row (8 or 16 >= GQ); a softmax
// thread tracks NH / 2 of them.  bf16 probabilities are split into hi + lo bf16 parts and the
// value MMA runs on both, so the weights keep ~16 significant bits (one bf16 part alone
// keeps 8).
template <typename IO, int NH>
__global__ void __launch_bounds__(base_threads(NH), 1)
decode_gqa_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, const DecodeParams p) {
  constexpr bool kSplit = std::is_same<IO, __nv_bfloat16>::value;
  constexpr int kParts = p_parts(kSplit);
  constexpr uint32_t kFmt = std::is_same<IO, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t kIdescS = mma_idesc_f16(kFmt, 0, 0, kTokens, kHeadsN);  // K-major A and B
  constexpr uint32_t kIdescO = mma_idesc_f16(kFmt, 1, 1, kDim, kHeadsN);  // MN-major A and B

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ TcShared sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int GQ = p.GQ;

  grid_dependency_launch_next();
  grid_dependency_wait();

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // swizzle atoms are 1024-B aligned
  const uint32_t pbase = base + kStages * kStageBytes;
  auto stage = [&](int st) { return base + st * kStageBytes; };
  auto pbuf = [&](int b, int part) { return pbase + (kParts * b + part) * kPBytes; };

  Cursor start;
  long long t0 = 0;
  PlanScratch& plan = *reinterpret_cast<PlanScratch*>(smem_raw + (pbase - smem_u32(smem_raw)));
  const long long count = plan_slice(p, plan, &t0, &start);
  if (count == 0) return;
  const int n = static_cast<int>(count);
  __syncthreads();  // every thread is done with the plan scratch before its space is reused

  const uint32_t full0 = smem_u32(&sh.full[0]), empty0 = smem_u32(&sh.empty[0]);
  const uint32_t s_full0 = smem_u32(&sh.s_full[0]), s_empty0 = smem_u32(&sh.s_empty[0]);
  const uint32_t p_full0 = smem_u32(&sh.p_full[0]), o_full0 = smem_u32(&sh.o_full[0]);
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full0 + 8 * st, 4);  // one arrival per TMA warp
      mbar_init(empty0 + 8 * st, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full0 + 8 * b, 1);
      mbar_init(s_empty0 + 8 * b, 256);  // every softmax thread
      mbar_init(p_full0 + 8 * b, 256);
      mbar_init(o_full0 + 8 * b, 1);
    }
    mbar_init(smem_u32(&sh.mma_done), 2);
    sh.abort = 0;
    fence_barrier_init();
  }
  // The probability operands start as zeros (they held the plan scratch): with up to 8 query
  // heads per row the padding heads 8..15 are never written again.
  for (int i = threadIdx.x; i < 2 * kParts * kPBytes / 16; i += blockDim.x) {
    uint8_t* ptr = smem_raw + (pbase - smem_u32(smem_raw)) + 16 * i;
    *reinterpret_cast<uint4*>(ptr) = make_uint4(0, 0, 0, 0);
  }
  // The q rows of a head group fill rows 0..GQ-1 of each stage's 16-row q block; rows
  // GQ..15 stay zero (padding of the MMA N dimension).
  for (int i = threadIdx.x; i < kStages * 2 * kQHalf / 16; i += blockDim.x) {
    const int st = i / (2 * kQHalf / 16), off = (i % (2 * kQHalf / 16)) * 16;
    uint8_t* ptr = smem_raw + (stage(st) - smem_u32(smem_raw)) + 4 * kHalf + off;
    *reinterpret_cast<uint4*>(ptr) = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_shared();
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0 || (warp >= 6 && warp <= 8)) {
    // ------------------------------------------------------------------ TMA producers --
    // Four warps, one per (K or V) x (64-dim half) part of a tile: a warp issues its copies
    // one after another, so four warps issue a tile four times as fast as one.  Warp 0
    // also loads the q rows.  Every warp walks the same tile stream and block table.
    const int part = warp == 0 ? 0 : warp - 5;  // 0: K lo, 1: K hi, 2: V lo, 3: V hi
    const CUtensorMap* map = part < 2 ? &tmK : &tmV;
    const uint64_t policy = l2_policy_evict_first();
    if (lane == 0) {
      prefetch_tensormap(map);
      if (part == 0) prefetch_tensormap(&tmQ);
    }
    const int bs = p.bs;
    const int bpt = kTokens / bs;  // blocks per tile
    // Block-table entries travel in 32-entry windows held one per lane, starting at a tile
    // boundary.  The window after the current one is loaded in the background, and the
    // first window of the sequence is kept for its other head groups, so the TMA issue
    // rarely waits for a table load.
    auto fetch = [&](int s, int from, int lim) -> int {
      const int idx = from + lane;
      return idx < lim ? __ldg(p.block_tables + static_cast<size_t>(s) * p.MB + idx) : 0;
    };
    int win_seq = -1, win_base = 0, win = 0;     // window in use
    int pre_seq = -1, pre_base = 0, pre = 0;     // next window, in flight
    int fst_seq = -1, fst_base = 0, fst = 0;     // first window of the sequence
    Cursor c = start;
    int issued = 0;
    // Issue the copies of tile `issued` (waiting, bounded, for its stage to be free).
    auto issue_next = [&]() -> bool {
      const int st = issued % kStages;
      const int kh = c.g / p.sub;  // cached head of this head group
      const int tok0 = (c.sp.first_t + c.j) * kTokens;
      const int lb_first = tok0 / bs;
      const int lb_lo = max(lb_first, c.sp.lo / bs), lb_hi = min(lb_first + bpt - 1, (c.sp.ctx - 1) / bs);
      const int nload = lb_hi - lb_lo + 1;
      const int lim = (c.sp.ctx - 1) / bs + 1;  // blocks of this sequence
      if (!(c.s == win_seq && lb_lo >= win_base && lb_hi < win_base + 32)) {
        if (c.s == pre_seq && lb_lo >= pre_base && lb_hi < pre_base + 32) {
          win_seq = pre_seq, win_base = pre_base, win = pre;
        } else if (c.s == fst_seq && lb_lo >= fst_base && lb_hi < fst_base + 32) {
          win_seq = fst_seq, win_base = fst_base, win = fst;
        } else {
          win_seq = c.s, win_base = lb_first, win = fetch(c.s, lb_first, lim);
        }
        if (c.s != fst_seq && c.j == 0) fst_seq = win_seq, fst_base = win_base, fst = win;
        pre_seq = c.s, pre_base = win_base + 32;
        pre = pre_base < lim ? fetch(c.s, pre_base, lim) : 0;
      }
      int pb = __shfl_sync(0xffffffffu, win, (lb_lo - win_base + lane) & 31);
      if (lane < nload && (pb < 0 || pb >= p.NB)) {
        if (part == 0) decode_error(PA_DEVERR_TABLE);
        pb = 0;
      }
      bool ok = true;
      if (lane == 0) {
        if (issued >= kStages) ok = wait_or_abort(empty0 + 8 * st, ((issued / kStages) - 1) & 1, abort);
        if (ok) {
          const uint32_t bar = full0 + 8 * st;
          const uint32_t halves = p.dim / 64;  // 64-dim halves of q (and of K, V) to copy
          const int nblk = ((part & 1) && halves == 1) ? 0 : nload;  // head_dim 64: no hi halves
          mbar_arrive_expect_tx(bar, (part == 0 ? halves * GQ * 128u : 0u) + static_cast<uint32_t>(nblk) * bs * 128u);
          if (part == 0) {
            const uint32_t sb = stage(st);
            const int qrow = c.s * p.Hq + c.g * GQ;
            tma_load_2d(sb + 4 * kHalf, &tmQ, bar, 0, qrow, policy);
            if (halves == 2) tma_load_2d(sb + 4 * kHalf + kQHalf, &tmQ, bar, 64, qrow, policy);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);  // also orders lane 0's expect_tx before any copy
      if (!ok) return false;
      const bool copies = !(part & 1) || p.dim == 128;  // head_dim 64: the hi-half warps only arrive
      if (copies && lane < nload) {  // this warp's part of each attended block, one copy per lane
        const uint32_t row0 = static_cast<uint32_t>(lb_lo + lane - lb_first) * bs;  // first row in the tile
        tma_load_3d(stage(st) + part * kHalf + row0 * 128u, map, full0 + 8 * st, (part & 1) * 64, kh, pb * bs, policy);
      }
      advance(c, p);
      ++issued;
      return true;
    };
    while (issued < n)
      if (!issue_next()) break;
    if (lane == 0)  // never leave with copies in flight
      for (int k = issued - kStages < 0 ? 0 : issued - kStages; k < issued; ++k)
        wait_or_abort(full0 + 8 * (k % kStages), (k / kStages) & 1, abort);
  } else if (warp == 1 || warp == 9) {
    // ------------------------------------------------------------------ MMA issuers --
    // Score MMAs: S^T[b] = K . Q^T, 16 dims per MMA.  Value MMAs: O^T[b] = V^T . P^T, 16
    // tokens per MMA.  A stage is released by the value MMA that last reads it (its score
    // MMA finished before the probabilities were written).
    auto issue_scores = [&](int i) {
      const int st = i % kStages, b = i % 2;
      const uint32_t sb = stage(st);
#pragma unroll
      for (int kk = 0; kk < kDim / 16; ++kk) {
        if (kk * 16 >= p.dim) break;  // head_dim 64: the lo halves only
        const uint32_t koff = (kk / 4) * kHalf + (kk % 4) * 32;  // 32 B steps inside a swizzled row
        const uint32_t qoff = 4 * kHalf + (kk / 4) * kQHalf + (kk % 4) * 32;
        tc_mma_f16(tmem + b * kHeadsN, smem_desc(sb + koff, 16, 1024, kSwizzle128B),
                   smem_desc(sb + qoff, 16, 1024, kSwizzle128B), kIdescS, kk > 0);
      }
      tc_commit(s_full0 + 8 * b);
    };
    auto issue_values = [&](int i) {
      const int b = i % 2;
      const uint32_t sb = stage(i % kStages);
      const uint32_t o_tmem = tmem + 2 * kHeadsN + b * kHeadsN;
#pragma unroll
      for (int part = 0; part < kParts; ++part) {
#pragma unroll
        for (int kk = 0; kk < kTokens / 16; ++kk) {
          tc_mma_f16(o_tmem, smem_desc(sb + 2 * kHalf + kk * 2048, kHalf, 1024, kSwizzle128B),
                     smem_desc(pbuf(b, part) + kk * 512, kPBytes, 256, kSwizzle32B), kIdescO, part > 0 || kk > 0);
        }
      }
      tc_commit(o_full0 + 8 * b);
      tc_commit(empty0 + 8 * (i % kStages));
    };
    // With up to 8 query heads per cached head the MMAs are small enough that issuing them
    // is the cost, so warp 1 issues the score MMAs and warp 9 the value MMAs.  With 16 the
    // softmax work per tile is larger and one lane of warp 1 polling for either kind of
    // ready work measured faster (3.98 vs 3.08 TB/s at 4 cached heads); warp 9 then idles.
    constexpr bool kTwoIssuers = NH <= 8;
    const uint32_t ready0 = full0;  // a stage's operands are complete
    if (lane == 0 && kTwoIssuers) {
      if (warp == 1) {
        for (int i = 0; i < n; ++i) {
          if (!wait_or_abort(ready0 + 8 * (i % kStages), (i / kStages) & 1, abort)) break;
          if (i >= 2 && !wait_or_abort(s_empty0 + 8 * (i % 2), ((i / 2) - 1) & 1, abort)) break;
          tc_fence_after_sync();
          issue_scores(i);
        }
      } else {
        for (int i = 0; i < n; ++i) {
          if (!wait_or_abort(p_full0 + 8 * (i % 2), (i / 2) & 1, abort)) break;
          tc_fence_after_sync();
          issue_values(i);
        }
      }
    }
    if (lane == 0 && !kTwoIssuers && warp == 1) {
      int s_next = 0, o_next = 0;
      uint32_t idle = 0;
      while (o_next < n) {
        bool progressed = false;
        if (s_next < n && mbar_test_wait(ready0 + 8 * (s_next % kStages), (s_next / kStages) & 1) &&
            (s_next < 2 || mbar_test_wait(s_empty0 + 8 * (s_next % 2), ((s_next / 2) - 1) & 1))) {
          tc_fence_after_sync();
          issue_scores(s_next++);
          progressed = true;
        }
        if (o_next < s_next && mbar_test_wait(p_full0 + 8 * (o_next % 2), (o_next / 2) & 1)) {
          tc_fence_after_sync();
          issue_values(o_next++);
          progressed = true;
        }
        if (progressed) {
          idle = 0;
        } else if (*abort || ++idle > 16 * kWaitLimit) {
          if (!*abort) decode_error(PA_DEVERR_TIMEOUT);
          *abort = 1;
          break;
        }
      }
    }
    if (lane == 0) {  // every MMA this warp issued has finished before TMEM is released
      tc_commit(smem_u32(&sh.mma_done));
      mbar_wait_bounded(smem_u32(&sh.mma_done), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------- softmax + accumulation warps --
    // Warps 2..5 and 10..13: two per TMEM lane quarter, each with half of the row's heads.
    constexpr int HPW = NH / 2;           // query heads a thread tracks
    constexpr int kSoftmax = 256;
    const int q4 = warp & 3;              // TMEM lane quarter this warp may access
    const int hh = warp >= 10 ? 1 : 0;    // which half of the row's heads
    const int h_base = HPW * hh;
    const int r = 32 * q4 + lane;         // token row (softmax) and head-dim row (accumulate)
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    float m[HPW], l[HPW], acc[HPW], alpha_prev[HPW];
#pragma unroll
    for (int h = 0; h < HPW; ++h) {
      m[h] = -FLT_MAX;
      l[h] = 0.f;
      acc[h] = 0.f;
      alpha_prev[h] = 1.f;
    }
    // No softmax thread leaves the loop on its own: a wait that gives up only stops the
    // thread's arrivals, and all of them leave together after a tile's exchange barrier once
    // the abort flag, as one thread saw it before that barrier, is set.  So no thread is ever
    // left at a named barrier.  (The TMEM loads run in every lane either way: the allocation
    // is held until the end, and values read after a failed wait are never written out.)
    // Fold the value product of tile t into the running output (thread = head dim r).
    auto accumulate = [&](int t, const float* alpha) {
      wait_or_abort(o_full0 + 8 * (t % 2), (t / 2) & 1, abort);
      tc_fence_after_sync();
      float o[HPW];
      tmem_load<HPW>(tmem + lane_addr + 2 * kHeadsN + (t % 2) * kHeadsN + h_base, o);
      tc_fence_before_sync();
#pragma unroll
      for (int h = 0; h < HPW; ++h) acc[h] = acc[h] * alpha[h] + o[h];
    };
    Cursor c = start;
    bool seg_from_start = (c.j == 0);
    bool pending = false;  // the value product of the previous tile is not folded in yet
    for (int i = 0; i < n; ++i) {
      const int b = i % 2, st = i % kStages;
      const bool got = wait_or_abort(s_full0 + 8 * b, (i / 2) & 1, abort);
      tc_fence_after_sync();
      float sc[HPW];
      tmem_load<HPW>(tmem + lane_addr + b * kHeadsN + h_base, sc);
      tc_fence_before_sync();
      if (got) mbar_arrive(s_empty0 + 8 * b);

      const int tok = (c.sp.first_t + c.j) * kTokens + r;
      const bool valid = tok >= c.sp.lo && tok < c.sp.ctx;
      const float sfac = p.qscale;
      {
        float mv[HPW];
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          sc[h] = (valid && h_base + h < GQ) ? sc[h] * sfac : -INFINITY;
          mv[h] = sc[h];
        }
        int hm;
        const float x = warp_reduce_transposed<HPW, true>(mv, lane, &hm);
        if ((lane & (32 / HPW - 1)) == 0) sh.red[b][q4][h_base + hm] = x;
      }
      if (threadIdx.x == 64) sh.stop[b] = *abort;  // the first softmax thread
      named_barrier_sync(1, kSoftmax);
      if (sh.stop[b]) break;  // every softmax thread, at the same tile
      float alpha[HPW];
      uint32_t w_hi[8], w_lo[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) w_hi[k] = w_lo[k] = 0;
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        const int hg = h_base + h;
        const float t = fmaxf(fmaxf(sh.red[b][0][hg], sh.red[b][1][hg]), fmaxf(sh.red[b][2][hg], sh.red[b][3][hg]));
        const float m_new = fmaxf(m[h], t);
        alpha[h] = ex2_ftz(m[h] - m_new);
        m[h] = m_new;
        const float pr = sc[h] == -INFINITY ? 0.f : ex2_ftz(sc[h] - m_new);
        const IO hi = float_to<IO>(pr);
        w_hi[h / 2] |= bits16(hi) << (16 * (h & 1));
        if (kSplit) {
          const IO lo = float_to<IO>(pr - static_cast<float>(hi));
          w_lo[h / 2] |= bits16(lo) << (16 * (h & 1));
          l[h] = l[h] * alpha[h] + pr;
        } else {
          l[h] = l[h] * alpha[h] + static_cast<float>(hi);  // the rounded weight the MMA uses
        }
      }
      if (NH > 8) {  // this warp's 16-byte chunk of the 32-byte row
        store_p_half_row(pbuf(b, 0), r, hh, w_hi);
        if (kSplit) store_p_half_row(pbuf(b, 1), r, hh, w_lo);
      } else {       // heads 4 hh .. 4 hh + 3: 8 bytes of the first chunk (heads 8..15 stay zero)
        store_p_quarter_row(pbuf(b, 0), r, hh, w_hi);
        if (kSplit) store_p_quarter_row(pbuf(b, 1), r, hh, w_lo);
      }
      if (!valid && hh == 0) {  // unattended rows may hold anything (NaN): give the value MMA zeros
        // Chunk k ^ (r & 7) at step k: neighbouring rows (128 B apart, the same banks)
        // write different 16-byte chunks at each step, so a warp's stores do not conflict.
        const uint32_t v0 = stage(st) + 2 * kHalf + r * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t c = 16 * (k ^ (r & 7));
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(v0 + c), "r"(0) : "memory");
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(v0 + kHalf + c), "r"(0) : "memory");
        }
      }
      fence_proxy_async_shared();
      mbar_arrive(p_full0 + 8 * b);

      // Overlap: the value MMA of tile i runs while the previous tile is folded in.
      if (pending) accumulate(i - 1, alpha_prev);
      pending = false;
      const bool seg_last = (c.j == c.sp.nb - 1);
      if (!(seg_last || i == n - 1)) {
        pending = true;
#pragma unroll
        for (int h = 0; h < HPW; ++h) alpha_prev[h] = alpha[h];
      } else {
        accumulate(i, alpha);
        // Softmax denominators: every thread holds the sums of its own token rows.
        float lt[HPW];
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          float x = l[h];
#pragma unroll
          for (int off = 16; off >= 1; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
          lt[h] = x;
        }
        if (lane == 0)
#pragma unroll
          for (int h = 0; h < HPW; ++h) sh.red_l[q4][h_base + h] = lt[h];
        named_barrier_sync(1, kSoftmax);
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          const int hg = h_base + h;
          lt[h] = sh.red_l[0][hg] + sh.red_l[1][hg] + sh.red_l[2][hg] + sh.red_l[3][hg];
        }
        named_barrier_sync(1, kSoftmax);  // sh.red_l is free again
        const int h0 = c.g * GQ + h_base;
        if (seg_from_start && seg_last) {
          IO* orow = reinterpret_cast<IO*>(p.out) + (static_cast<size_t>(c.s) * p.Hq + h0) * p.dim + r;
          if (r < p.dim)  // (head_dim 64: rows 64..127 of O^T come from the unused V hi half)
#pragma unroll
            for (int h = 0; h < HPW; ++h)
              if (h_base + h < GQ) orow[static_cast<size_t>(h) * p.dim] = float_to<IO>(acc[h] / lt[h]);
        } else {
          const long long slot = blockIdx.x + static_cast<long long>(c.s) * p.G + c.g;
#pragma unroll
          for (int h = 0; h < HPW; ++h) {
            const int hg = h_base + h;
            if (hg >= GQ) continue;
            if (r < p.dim) p.ws_acc[(slot * GQ + hg) * p.dim + r] = acc[h];
            if (r == 0) {
              p.ws_ml[(slot * GQ + hg) * 2 + 0] = m[h];
              p.ws_ml[(slot * GQ + hg) * 2 + 1] = lt[h];
            }
          }
        }
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          m[h] = -FLT_MAX;
          l[h] = 0.f;
          acc[h] = 0.f;
        }
      }
      if (i + 1 < n) {
        advance(c, p);
        if (c.j == 0) seg_from_start = true;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t read_tc_error(uint32_t* flags, int clear) {
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

struct RegisterTc {
  RegisterTc() { register_device_error_reader(read_tc_error); }
} g_register_tc;

}  // namespace

int tc_decode_subgroup(int group) {
  if (group <= kHeadsN) return group;
  for (int sg = kHeadsN; sg >= 4; --sg)
    if (group % sg == 0) return sg;
  return 0;
}

bool tc_decode_eligible(pa_dtype io, pa_dtype cache, int head_dim, int block_size, int group) {
  const bool eight_bit = cache == PA_I8 || cache == PA_FP8_E4M3;
  return (io == PA_F16 || io == PA_BF16) && (cache == io || eight_bit) &&
         (head_dim == kDim || (head_dim == 64 && !eight_bit)) && block_size >= 8 &&
         block_size <= kTokens && block_size % 8 == 0 && kTokens % block_size == 0 && group >= 4 &&
         tc_decode_subgroup(group) >= 4;
}

int tc_decode_tile_tokens() { return kTokens; }

namespace {
template <typename IO, int NH>
const void* tc_fn() {
  return reinterpret_cast<const void*>(&decode_gqa_tc_kernel<IO, NH>);
}
}  // namespace

pa_status tc_decode_launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                           const CUtensorMap& tmKs, const CUtensorMap& tmVs, const DecodeParams& prm, pa_dtype io,
                           pa_dtype cache, int grid, cudaStream_t stream) {
  if (cache != io) return tc8_decode_launch(tmK, tmV, tmKs, tmVs, prm, io, cache, grid, stream);
  const bool small = prm.GQ <= 8;
  const void* fn = io == PA_BF16 ? (small ? tc_fn<__nv_bfloat16, 8>() : tc_fn<__nv_bfloat16, 16>())
                                 : (small ? tc_fn<__half, 8>() : tc_fn<__half, 16>());
  const size_t smem = smem_bytes(io == PA_BF16);
  // The dynamic shared-memory limit is a per-kernel attribute: set once per kernel.
  static std::mutex m;
  static std::vector<const void*> ready;
  {
    std::lock_guard<std::mutex> lock(m);
    if (std::find(ready.begin(), ready.end(), fn) == ready.end()) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tensor-core decode)");
      ready.push_back(fn);
    }
  }
  CUtensorMap k = tmK, v = tmV, q = tmQ;
  DecodeParams p = prm;
  void* args[] = {&k, &v, &q, &p};
  cudaError_t err = launch_dependent(fn, dim3(grid), dim3(base_threads(small ? 8 : 16)), smem, stream, args);
  if (err != cudaSuccess) return cuda_fail(err, "launching the tensor-core decode kernel");
  return PA_OK;
}

}  // namespace pa
