// pa_decode_tc8.cu -- grouped-query paged decode over an 8-bit cache on the 5th-generation
// tensor cores (sm_100a), the codes multiplied as they are.
//
// An INT8 or FP8 E4M3 cache holds one code per element and one fp16 scale per (token, cached
// head) ("KV Cache optimisation strategies in deployment" (yunthe.com), section
// "量化压缩KV Cache的INT8与FP8方案"); the block-table walk and cache layout are those of the
// 16-bit kernel ("KV Cache memory optimisation and PagedAttention" (yunthe.com), section
// "PagedAttention注意力计算流程").  Per 128-token tile of one cached head:
//
//   S^T[128 tok x N]  = Kc[128 tok x 128 d] . Qd^T[128 d x N]    (K-major A and B)
//   O^T[128 d x N]    = Vc^T[128 d x 128 tok] . Wd^T[128 tok x N] (MN-major A and B)
//
// Kc, Vc are the codes straight from the cache (tcgen05 kind::i8 for INT8, kind::f8f6f4 for
// E4M3, so a tile's operands are its 32 KiB of codes and no 16-bit copy is made).  The other
// operand of each product must have the same 8-bit kind, so q and the softmax weights enter
// as digits:
//   INT8: q = 2^-E (256 hi + lo) with hi, lo signed bytes (16-bit fixed point per head, E
//         chosen per head from max |q|); a weight w = p v_scale / v_max in [0, 1] enters as
//         round(65535 w) = 256 hi + lo with unsigned bytes.  Products and sums are exact
//         integers (s32 accumulators); S = 256 S_hi + S_lo, O = 256 O_hi + O_lo.
//   FP8:  q 2^E (|.| < 256) and 256 w are split into three E4M3 digits x ~ d1 + d2/16 + d3/256
//         (each digit the rounded remainder of the previous step, scaled by 16), which keeps
//         ~12 significant bits; S and O sum their three digit products the same way.
// Each group of 8 query heads takes N = 32 columns (8 heads x up to 3 digits, padded), so
// N = 32 for up to 8 query heads per cached head and 64 for up to 16.  The softmax applies
// each token's K scale and the head's q unit 2^-E to its score row; the V scales are folded
// into the weights relative to the tile's largest V scale v_max, and O is scaled back by
// v_max / 65535 (INT8) or v_max / 256 (FP8) when it is folded into the running output.
//
// Roles (14 warps; two CTAs per SM with up to 8 query heads per cached head, one with 16):
//   warps 0,6-8 TMA producers (K codes, V codes, K scales, V scales), each into a 2-stage
//               (two CTAs per SM) or 4-stage ring; their 128 lanes also hold the head group's q digits (loaded
//               and split once per segment, the next segment's q rows prefetched) and store
//               them into each stage with the copies.
//   warp 1      TMEM owner and MMA issuer; with up to 8 query heads per cached head warp 9
//               issues the value MMAs and warp 1 the score MMAs.
//   warps 2..5, 10..13  softmax (thread = token row of S^T) and accumulation (thread = head
//               dim row of O^T) with the digit products combined, two warps per TMEM lane
//               quarter, each with half of the row's query heads (a timeline of one CTA showed
//               the softmax, not the copies or the MMAs, setting the tile period); per-head
//               tile maxima are reduced by a transposing shuffle (9 shuffles for 8 heads
//               instead of 40).  FP8 V rows of unattended tokens are zeroed (an E4M3 code may
//               be NaN; INT8 codes are finite and meet a zero weight).
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

constexpr int kTokens = 128;                 // tile rows (MMA M of the score product)
constexpr int kDim = 128;                    // head_dim: one 128-byte code row per token and head
constexpr int kHeadsN = 16;                  // query heads per cached head, at most
constexpr int kNBlock = 32;                  // MMA N per 8 query heads (8 heads x 2 or 3 digits, padded)
constexpr int kCodeBytes = kTokens * kDim;   // one tile of one cached head's K (or V) codes: 16 KiB
constexpr int kScaleBytes = kTokens * 16;    // fp16 scales of a tile for an 8-head column group
constexpr int kUnitBytes = 128;              // q units 2^-E of the head group (16 floats)
constexpr int q_digit_bytes(int nh) { return (nh / 8) * kNBlock * kDim; }  // q digit operand
// Stage: K codes, V codes, q digits, K scales, V scales, q units.
constexpr int stage_bytes(int nh) {
  return (2 * kCodeBytes + q_digit_bytes(nh) + 2 * kScaleBytes + kUnitBytes + 1023) / 1024 * 1024;
}
// Up to 8 query heads per cached head two CTAs share an SM (72 registers a thread): each
// CTA's per-tile softmax chain is latency-bound, and a second chain per SM runs in its gaps.
// Two stages each then fit the SM's shared memory.
constexpr int ctas_per_sm(int nh) { return nh > 8 ? 1 : 2; }
constexpr int stages_for(int nh) { return nh > 8 ? 4 : 2; }
constexpr int p_bytes(int nh) { return kTokens * kNBlock * (nh / 8); }  // one weight-digit operand W^T
constexpr size_t smem_bytes(int nh) {
  return 1024 + static_cast<size_t>(stages_for(nh)) * stage_bytes(nh) + 2 * p_bytes(nh);
}
constexpr int kMaxStages = 5;
static_assert(smem_bytes(8) <= 232448 && smem_bytes(16) <= 232448, "shared memory per CTA");
static_assert(sizeof(PlanScratch) <= 2 * p_bytes(8), "plan scratch fits the weight operands");
constexpr int base_threads(int) { return 448; }
static_assert(base_threads(16) <= kMaxPlanThreads, "plan_slice keeps one scratch entry per thread");

struct Tc8Shared {
  uint64_t full[kMaxStages], empty[kMaxStages];  // TMA ring
  uint64_t s_full[2], s_empty[2];                // score accumulators in TMEM
  uint64_t p_full[2], o_full[2];                 // weights written / value MMA done
  uint64_t mma_done;                             // both MMA warps' last MMAs finished
  uint32_t tmem_base;
  int abort;
  float red[2][4][kHeadsN + 1];                  // per-tile maxima across the softmax warps (+ v_max)
  float red_l[4][kHeadsN];                       // softmax denominators at segment ends
  int stop[2];                                   // abort flag as seen before a tile's exchange barrier
};

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
  }
  *abort = 1;
  decode_error(PA_DEVERR_TIMEOUT);
  return false;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Low bytes of four integers, a in the lowest.
__device__ __forceinline__ uint32_t pack_bytes(int a, int b, int c, int d) {
  return __byte_perm(__byte_perm(a, b, 0x0040u), __byte_perm(c, d, 0x0040u), 0x5410u);
}

// x in [0, 256] (an f16 pair) -> three E4M3 digit pairs with x ~ d1 + d2 / 16 + d3 / 256.
// Each remainder x - d is exact in f16 (d is within a factor of two of x, or 0 when x is
// below half the smallest E4M3 step) and so is its scaling by 16.
__device__ __forceinline__ void f16_digits(uint32_t x, uint32_t& d1, uint32_t& d2, uint32_t& d3) {
  const uint32_t sixteen = 0x4C004C00u;  // 16.0, 16.0
  d1 = f16x2_to_e4m3x2(x);
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(e4m3x2_to_f16x2(d1)));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(sixteen));
  d2 = f16x2_to_e4m3x2(r);
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(e4m3x2_to_f16x2(d2)));
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(sixteen));
  d3 = f16x2_to_e4m3x2(r);
}

// tcgen05.ld of the D digit columns of H consecutive heads (digit k of head j at column
// col + 8 k + j), one wait for all: out[k * H + j].  The wait sits in the same statement as
// the loads, so no use of a destination register can be scheduled before the data arrives.
template <int H, int D> __device__ __forceinline__ void tmem_load_digits(uint32_t col, float* out);
template <> __device__ __forceinline__ void tmem_load_digits<4, 2>(uint32_t col, float* out) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%8];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [%9];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(col), "r"(col + 8)
      : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) out[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_load_digits<4, 3>(uint32_t col, float* out) {
  uint32_t r[12];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%12];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%4, %5, %6, %7}, [%13];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%8, %9, %10, %11}, [%14];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11])
      : "r"(col), "r"(col + 8), "r"(col + 16)
      : "memory");
#pragma unroll
  for (int i = 0; i < 12; ++i) out[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_load_digits<8, 2>(uint32_t col, float* out) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(col)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) out[i] = __uint_as_float(r[i]);
}
template <> __device__ __forceinline__ void tmem_load_digits<8, 3>(uint32_t col, float* out) {
  uint32_t r[24];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%24];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%16, %17, %18, %19, %20, %21, %22, %23}, [%25];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23])
      : "r"(col), "r"(col + 16)
      : "memory");
#pragma unroll
  for (int i = 0; i < 24; ++i) out[i] = __uint_as_float(r[i]);
}

// IO: fp16 or bf16 queries and output; CT: int8_t or __nv_fp8_e4m3 codes; NH: query heads of
// a row (8 or 16 >= GQ); a softmax thread tracks NH / 2 of them.
template <typename IO, typename CT, int NH>
__global__ void __launch_bounds__(base_threads(NH), ctas_per_sm(NH))
decode_gqa_tc8_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmKs, const __grid_constant__ CUtensorMap tmVs,
                      const DecodeParams p) {
  constexpr bool kInt = std::is_same<CT, int8_t>::value;
  constexpr int kDigits = kInt ? 2 : 3;        // digits of q and of the weights
  constexpr int kStages = stages_for(NH);
  constexpr int kStage = stage_bytes(NH);
  constexpr int NC = kNBlock * (NH / 8);       // S and O columns per buffer (MMA N)
  constexpr int kPBytes = p_bytes(NH);
  constexpr uint32_t kOffV = kCodeBytes, kOffQ = 2 * kCodeBytes, kOffKs = kOffQ + q_digit_bytes(NH),
                     kOffVs = kOffKs + kScaleBytes, kOffU = kOffVs + kScaleBytes;
  // Scores: signed K codes x signed q bytes (INT8); values: signed V codes x unsigned weight
  // bytes.  E4M3 everywhere for FP8.
  constexpr uint32_t kIdescS = kInt ? mma_idesc_i8(1, 1, 0, 0, kTokens, NC) : mma_idesc_e4m3(0, 0, kTokens, NC);
  constexpr uint32_t kIdescO = kInt ? mma_idesc_i8(1, 0, 1, 1, kDim, NC) : mma_idesc_e4m3(1, 1, kDim, NC);
  constexpr uint32_t kTmemCols = 4 * NC;       // S0 S1 O0 O1
  static_assert(kOffU + kUnitBytes <= kStage, "stage layout");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ Tc8Shared sh;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int GQ = p.GQ;

  grid_dependency_launch_next();
  grid_dependency_wait();

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // swizzle atoms are 1024-B aligned
  const uint32_t pbase = base + kStages * kStage;
  auto stage = [&](int st) { return base + st * kStage; };
  auto pbuf = [&](int b) { return pbase + b * kPBytes; };
  auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    if constexpr (kInt) tc_mma_i8(d, a, b, idesc, acc);
    else tc_mma_f8(d, a, b, idesc, acc);
  };

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
  // The q digit operands of every stage and both weight operands start as zeros: their
  // padding rows (columns) are never written again.
  for (int i = threadIdx.x; i < kStages * q_digit_bytes(NH) / 16; i += blockDim.x)
    st_shared_v4(stage(i / (q_digit_bytes(NH) / 16)) + kOffQ + 16 * (i % (q_digit_bytes(NH) / 16)), 0, 0, 0, 0);
  for (int i = threadIdx.x; i < 2 * kPBytes / 16; i += blockDim.x) st_shared_v4(pbase + 16 * i, 0, 0, 0, 0);
  fence_proxy_async_shared();
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0 || (warp >= 6 && warp <= 8)) {
    // ------------------------------------------------------------------ TMA producers --
    const int part = warp == 0 ? 0 : warp - 5;  // 0: K codes, 1: V codes, 2: K scales, 3: V scales
    const CUtensorMap* map = part == 0 ? &tmK : part == 1 ? &tmV : part == 2 ? &tmKs : &tmVs;
    // Codes are read once (evict first); a scale row holds 8 cached heads and serves the
    // tiles of all 8, which follow one another in the stream (evict last).
    const uint64_t policy = part < 2 ? l2_policy_evict_first() : l2_policy_evict_last();
    if (lane == 0) prefetch_tensormap(map);
    const int bs = p.bs;
    const int bpt = kTokens / bs;  // blocks per tile
    // q digits: lane l of producer `part` holds dims 16 * (qt & 7) .. + 15 of query head
    // qt >> 3 of the head group (qt = 32 * part + l), as kDigits 16-byte rows.
    const int qt = 32 * part + lane, qh = qt >> 3, qseg = qt & 7;
    uint32_t qd[kDigits][4];
    float qunit = 0.f;
    int q_s = -1, q_g = -1;    // segment whose digits qd holds
    int nx_s = -1, nx_g = -1;  // segment whose q rows qn holds (loads in flight)
    uint4 qn0 = make_uint4(0, 0, 0, 0), qn1 = qn0;
    auto fetch_q = [&](int s, int g) {
      qn0 = qn1 = make_uint4(0, 0, 0, 0);
      if (qh < GQ && qh < NH) {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const IO*>(p.q) +
                                                          (static_cast<size_t>(s) * p.Hq + g * GQ + qh) * kDim +
                                                          16 * qseg);
        qn0 = __ldg(src);
        qn1 = __ldg(src + 1);
      }
      nx_s = s;
      nx_g = g;
    };
    // Split the q rows in qn into digits; the 8 lanes of a head agree on its exponent.
    auto split_q = [&]() {
      float f[16];
      Elem<IO>::to_float(qn0, f);
      Elem<IO>::to_float(qn1, f + 8);
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(f[i]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      // max |q| * 2^E in [2^top, 2^(top + 1)): 16-bit fixed point (INT8), below 256 (E4M3)
      constexpr int kTop = kInt ? 14 : 7;
      const int ex = max(static_cast<int>((__float_as_uint(mx) >> 23) & 0xFF) - 127, -100);
      const float up = __uint_as_float(static_cast<uint32_t>(127 + kTop - ex) << 23);
      qunit = __uint_as_float(static_cast<uint32_t>(127 + ex - kTop) << 23);
      if constexpr (kInt) {
        int hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int x = min(max(__float2int_rn(f[i] * up), -32640), 32639);
          hi[i] = (x + 128) >> 8;  // x = 256 hi + lo, both in [-128, 127]
          lo[i] = x - (hi[i] << 8);
        }
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          qd[0][w] = pack_bytes(hi[4 * w], hi[4 * w + 1], hi[4 * w + 2], hi[4 * w + 3]);
          qd[1][w] = pack_bytes(lo[4 * w], lo[4 * w + 1], lo[4 * w + 2], lo[4 * w + 3]);
        }
      } else {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t c[3][2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            float x0 = f[4 * w + 2 * j] * up, x1 = f[4 * w + 2 * j + 1] * up;  // exact
#pragma unroll
            for (int k = 0; k < 3; ++k) {
              c[k][j] = f32x2_to_e4m3x2(x0, x1);
              const uint32_t hb = e4m3x2_to_f16x2(c[k][j]);
              const float2 y = __half22float2(*reinterpret_cast<const __half2*>(&hb));
              x0 = (x0 - y.x) * 16.f;  // exact remainders
              x1 = (x1 - y.y) * 16.f;
            }
          }
#pragma unroll
          for (int k = 0; k < kDigits; ++k) qd[k][w] = c[k][0] | (c[k][1] << 16);
        }
      }
    };
    int win_seq = -1, win_base = 0, win = 0;  // block-table window in use
    int pre_seq = -1, pre_base = 0, pre = 0;  // next window, in flight
    int fst_seq = -1, fst_base = 0, fst = 0;  // first window of the sequence
    auto fetch = [&](int s, int from, int lim) -> int {
      const int idx = from + lane;
      return idx < lim ? __ldg(p.block_tables + static_cast<size_t>(s) * p.MB + idx) : 0;
    };
    Cursor c = start;
    int issued = 0;
    auto issue_next = [&]() -> bool {
      const int st = issued % kStages;
      const int kh = c.g / p.sub;  // cached head of this head group
      if (c.s != q_s || c.g != q_g) {  // a new segment: its q digits, then the next segment's q rows
        if (c.s != nx_s || c.g != nx_g) fetch_q(c.s, c.g);
        split_q();
        q_s = c.s;
        q_g = c.g;
        Cursor nx = c;
        nx.j = nx.sp.nb - 1;
        advance(nx, p);
        if (nx.s < p.S) fetch_q(nx.s, nx.g);
      }
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
      if (lane == 0 && issued >= kStages) ok = wait_or_abort(empty0 + 8 * st, ((issued / kStages) - 1) & 1, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      // The stage is free: this thread's q digits and its head's unit, then the copies.
      if (qh < NH) {
        const int blk = qh >> 3, hl = qh & 7;
#pragma unroll
        for (int k = 0; k < kDigits; ++k) {
          const int row = kNBlock * blk + 8 * k + hl;  // (row & 7) == hl: the 128-byte swizzle
          st_shared_v4(stage(st) + kOffQ + row * 128 + 16 * (qseg ^ hl), qd[k][0], qd[k][1], qd[k][2], qd[k][3]);
        }
        if (qseg == 0) asm volatile("st.shared.f32 [%0], %1;" ::"r"(stage(st) + kOffU + 4 * qh), "f"(qunit) : "memory");
      }
      fence_proxy_async_shared();
      __syncwarp();
      const uint32_t bar = full0 + 8 * st;
      if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nload) * bs * (part < 2 ? 128u : 16u));
      __syncwarp();  // the expected bytes are posted before any copy
      if (lane < nload) {  // this warp's part of each attended block, one copy per lane
        const uint32_t row0 = static_cast<uint32_t>(lb_lo + lane - lb_first) * bs;  // first row in the tile
        if (part < 2)
          tma_load_3d(stage(st) + (part == 0 ? 0u : kOffV) + row0 * 128u, map, bar, 0, kh, pb * bs, policy);
        else  // scale rows: x rounded down to a 16-byte boundary (8 heads)
          tma_load_2d(stage(st) + (part == 2 ? kOffKs : kOffVs) + row0 * 16u, map, bar, kh & ~7, pb * bs, policy);
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
    // Score MMAs: S^T[b] = Kc . Qd^T, 32 dims per MMA.  Value MMAs: O^T[b] = Vc^T . Wd^T, 32
    // tokens per MMA.  A stage is released by the value MMA that last reads it.
    auto issue_scores = [&](int i) {
      const int b = i % 2;
      const uint32_t sb = stage(i % kStages);
#pragma unroll
      for (int kk = 0; kk < kDim / 32; ++kk)  // 32-byte steps inside the swizzled rows
        mma(tmem + b * NC, smem_desc(sb + kk * 32, 16, 1024, kSwizzle128B),
            smem_desc(sb + kOffQ + kk * 32, 16, 1024, kSwizzle128B), kIdescS, kk > 0);
      tc_commit(s_full0 + 8 * b);
    };
    auto issue_values = [&](int i) {
      const int b = i % 2;
      const uint32_t sb = stage(i % kStages);
#pragma unroll
      for (int kk = 0; kk < kTokens / 32; ++kk)  // 32 token rows per step; 8-head column blocks kTokens * 32 B apart
        mma(tmem + 2 * NC + b * NC, smem_desc(sb + kOffV + kk * 4096, kCodeBytes, 1024, kSwizzle128B),
            smem_desc(pbuf(b) + kk * 1024, kTokens * kNBlock, 256, kSwizzle32B), kIdescO, kk > 0);
      tc_commit(o_full0 + 8 * b);
      tc_commit(empty0 + 8 * (i % kStages));
    };
    constexpr bool kTwoIssuers = NH <= 8;
    if (lane == 0 && kTwoIssuers) {
      if (warp == 1) {
        for (int i = 0; i < n; ++i) {
          if (!wait_or_abort(full0 + 8 * (i % kStages), (i / kStages) & 1, abort)) break;
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
        if (s_next < n && mbar_test_wait(full0 + 8 * (s_next % kStages), (s_next / kStages) & 1) &&
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
    // Digit k of head h sits in column 32 (h / 8) + 8 k + h % 8 of an S or O buffer.
    const uint32_t dcol = static_cast<uint32_t>(kNBlock * (h_base >> 3) + (h_base & 7));
    float m[HPW], l[HPW], acc[HPW], alpha_prev[HPW];
    float unit_prev = 0.f;
#pragma unroll
    for (int h = 0; h < HPW; ++h) {
      m[h] = -FLT_MAX;
      l[h] = 0.f;
      acc[h] = 0.f;
      alpha_prev[h] = 1.f;
    }
    // The digit products of this thread's heads combined.
    auto combine = [&](uint32_t col, float* out) {
      float d[kDigits * HPW];
      tmem_load_digits<HPW, kDigits>(col, d);
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        if constexpr (kInt)
          out[h] = static_cast<float>(__float_as_int(d[h]) * 256 + __float_as_int(d[HPW + h]));
        else
          out[h] = fmaf(d[2 * HPW + h], 1.f / 256.f, fmaf(d[HPW + h], 1.f / 16.f, d[h]));
      }
    };
    // No softmax thread leaves the loop on its own: a wait that gives up only stops the
    // thread's arrivals, and all of them leave together after a tile's exchange barrier once
    // the abort flag, as one thread saw it before that barrier, is set.  So no thread is ever
    // left at a named barrier.  (The TMEM loads run in every lane either way: the allocation
    // is held until the end, and values read after a failed wait are never written out.)
    // Fold the value product of tile t into the running output (thread = head dim r).
    auto accumulate = [&](int t, const float* alpha, float unit) {
      wait_or_abort(o_full0 + 8 * (t % 2), (t / 2) & 1, abort);
      tc_fence_after_sync();
      float o[HPW];
      combine(tmem + lane_addr + 2 * NC + (t % 2) * NC + dcol, o);
      tc_fence_before_sync();
#pragma unroll
      for (int h = 0; h < HPW; ++h) acc[h] = fmaf(acc[h], alpha[h], o[h] * unit);
    };
    Cursor c = start;
    bool seg_from_start = (c.j == 0);
    bool pending = false;  // the value product of the previous tile is not folded in yet
    for (int i = 0; i < n; ++i) {
      const int b = i % 2, st = i % kStages;
      const bool got = wait_or_abort(s_full0 + 8 * b, (i / 2) & 1, abort);
      tc_fence_after_sync();
      float sc[HPW];
      combine(tmem + lane_addr + b * NC + dcol, sc);
      tc_fence_before_sync();
      if (got) mbar_arrive(s_empty0 + 8 * b);

      const int tok = (c.sp.first_t + c.j) * kTokens + r;
      const bool valid = tok >= c.sp.lo && tok < c.sp.ctx;
      float kscale = 0.f, vscale = 0.f;  // this token's scales
      if (valid) {
        const uint32_t sa = stage(st) + kOffKs + r * 16 + 2 * ((c.g / p.sub) & 7);
        kscale = __half2float(__ushort_as_half(ld_shared_u16(sa)));
        vscale = __half2float(__ushort_as_half(ld_shared_u16(sa + kScaleBytes)));
      }
      float qu[HPW];
#pragma unroll
      for (int k = 0; k < HPW / 4; ++k) {
        const uint4 u = ld_shared_v4(stage(st) + kOffU + 4 * h_base + 16 * k);
        qu[4 * k] = __uint_as_float(u.x), qu[4 * k + 1] = __uint_as_float(u.y);
        qu[4 * k + 2] = __uint_as_float(u.z), qu[4 * k + 3] = __uint_as_float(u.w);
      }
      const float sfac = p.qscale * kscale;
      {
        float mv[HPW];
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          sc[h] = (valid && h_base + h < GQ) ? sc[h] * qu[h] * sfac : -INFINITY;
          mv[h] = sc[h];
        }
        int hm;
        const float x = warp_reduce_transposed<HPW, true>(mv, lane, &hm);
        if ((lane & (32 / HPW - 1)) == 0) sh.red[b][q4][h_base + hm] = x;
      }
      {
        float x = vscale;  // the tile's largest V scale (0 for unattended rows)
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
        if (lane == 0 && hh == 0) sh.red[b][q4][kHeadsN] = x;
      }
      if (threadIdx.x == 64) sh.stop[b] = *abort;  // the first softmax thread
      named_barrier_sync(1, kSoftmax);
      if (sh.stop[b]) break;  // every softmax thread, at the same tile
      const float vmax = fmaxf(fmaxf(sh.red[b][0][kHeadsN], sh.red[b][1][kHeadsN]),
                               fmaxf(sh.red[b][2][kHeadsN], sh.red[b][3][kHeadsN]));
      const float vrel = vmax > 0.f ? vscale / vmax : 0.f;  // in [0, 1]
      const float unit = kInt ? vmax * (1.f / 65535.f) : vmax * (1.f / 256.f);
      float alpha[HPW], w[HPW];
#pragma unroll
      for (int h = 0; h < HPW; ++h) {
        const int hg = h_base + h;
        const float t = fmaxf(fmaxf(sh.red[b][0][hg], sh.red[b][1][hg]), fmaxf(sh.red[b][2][hg], sh.red[b][3][hg]));
        const float m_new = fmaxf(m[h], t);
        alpha[h] = ex2_ftz(m[h] - m_new);
        m[h] = m_new;
        const float pr = sc[h] == -INFINITY ? 0.f : ex2_ftz(sc[h] - m_new);
        l[h] = l[h] * alpha[h] + pr;
        w[h] = fminf(pr * vrel, 1.f);
      }
      // Digit k of head h goes to byte 8 k + h % 8 of the 32-byte row of its 8-head block.
      const uint32_t prow = pbuf(b) + (h_base >> 3) * (kTokens * kNBlock) + r * 32;
      const uint32_t sw = (r >> 2) & 1;  // 32-byte swizzle: the row's 16-byte chunks trade places on rows 4..7 of 8
      const uint32_t c0 = prow + 16 * sw, c1 = prow + 16 * (sw ^ 1);
      uint32_t dw[kDigits][HPW / 4];  // digit k of heads 4 i .. 4 i + 3 in word [k][i]
      if constexpr (kInt) {
#pragma unroll
        for (int i = 0; i < HPW / 4; ++i) {
          uint32_t wb[4];  // low 16 bits: round(65535 w)
#pragma unroll
          for (int j = 0; j < 4; ++j) wb[j] = __float_as_uint(fmaf(w[4 * i + j], 65535.f, 8388608.f));
          const uint32_t t0 = __byte_perm(wb[0], wb[1], 0x5140u), t1 = __byte_perm(wb[2], wb[3], 0x5140u);
          dw[0][i] = __byte_perm(t0, t1, 0x7632u);  // high bytes
          dw[1][i] = __byte_perm(t0, t1, 0x5410u);  // low bytes
        }
      } else {
#pragma unroll
        for (int i = 0; i < HPW / 4; ++i) {
          uint32_t d[3][2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const __half2 x = __floats2half2_rn(256.f * w[4 * i + 2 * j], 256.f * w[4 * i + 2 * j + 1]);
            f16_digits(*reinterpret_cast<const uint32_t*>(&x), d[0][j], d[1][j], d[2][j]);
          }
#pragma unroll
          for (int k = 0; k < 3; ++k) dw[k][i] = d[k][0] | (d[k][1] << 16);
        }
      }
      if constexpr (HPW == 8) {  // the whole block: bytes 0..15 in one chunk, 16..23 in the other
        st_shared_v4(c0, dw[0][0], dw[0][1], dw[1][0], dw[1][1]);
        if constexpr (!kInt) st_shared_v4(c1, dw[2][0], dw[2][1], 0, 0);
      } else {                          // heads h0 .. h0 + 3 of the block: 4 bytes per digit
        const uint32_t h0 = h_base & 7;
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(c0 + h0), "r"(dw[0][0]) : "memory");
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(c0 + 8 + h0), "r"(dw[1][0]) : "memory");
        if constexpr (!kInt) asm volatile("st.shared.b32 [%0], %1;" ::"r"(c1 + h0), "r"(dw[kDigits - 1][0]) : "memory");
      }
      if (!kInt && !valid && hh == 0) {  // an unattended row may hold NaN codes: give the value MMA zeros
        const uint32_t v0 = stage(st) + kOffV + r * 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) st_shared_v4(v0 + 16 * (k ^ (r & 7)), 0, 0, 0, 0);
      }
      fence_proxy_async_shared();
      mbar_arrive(p_full0 + 8 * b);

      // Overlap: the value MMA of tile i runs while the previous tile is folded in.
      if (pending) accumulate(i - 1, alpha_prev, unit_prev);
      pending = false;
      const bool seg_last = (c.j == c.sp.nb - 1);
      if (!(seg_last || i == n - 1)) {
        pending = true;
        unit_prev = unit;
#pragma unroll
        for (int h = 0; h < HPW; ++h) alpha_prev[h] = alpha[h];
      } else {
        accumulate(i, alpha, unit);
        // Softmax denominators: every thread holds the sums of its own token rows.
        float lt[HPW];
        {
          float ls[HPW];
#pragma unroll
          for (int h = 0; h < HPW; ++h) ls[h] = l[h];
          int hl;
          const float x = warp_reduce_transposed<HPW, false>(ls, lane, &hl);
          if ((lane & (32 / HPW - 1)) == 0) sh.red_l[q4][h_base + hl] = x;
        }
        named_barrier_sync(1, kSoftmax);
#pragma unroll
        for (int h = 0; h < HPW; ++h) {
          const int hg = h_base + h;
          lt[h] = sh.red_l[0][hg] + sh.red_l[1][hg] + sh.red_l[2][hg] + sh.red_l[3][hg];
        }
        named_barrier_sync(1, kSoftmax);  // sh.red_l is free again
        const int h0 = c.g * GQ + h_base;
        if (seg_from_start && seg_last) {
          IO* orow = reinterpret_cast<IO*>(p.out) + (static_cast<size_t>(c.s) * p.Hq + h0) * kDim + r;
#pragma unroll
          for (int h = 0; h < HPW; ++h)
            if (h_base + h < GQ) orow[static_cast<size_t>(h) * kDim] = float_to<IO>(acc[h] / lt[h]);
        } else {
          const long long slot = blockIdx.x + static_cast<long long>(c.s) * p.G + c.g;
#pragma unroll
          for (int h = 0; h < HPW; ++h) {
            const int hg = h_base + h;
            if (hg >= GQ) continue;
            p.ws_acc[(slot * GQ + hg) * kDim + r] = acc[h];
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

template <typename IO, typename CT, int NH>
const void* tc8_fn() {
  return reinterpret_cast<const void*>(&decode_gqa_tc8_kernel<IO, CT, NH>);
}
template <typename IO, int NH>
const void* tc8_fn_for(pa_dtype cache) {
  return cache == PA_I8 ? tc8_fn<IO, int8_t, NH>() : tc8_fn<IO, __nv_fp8_e4m3, NH>();
}

}  // namespace

int tc8_ctas_per_sm(int group) { return ctas_per_sm(group <= 8 ? 8 : 16); }

pa_status tc8_decode_launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKs,
                            const CUtensorMap& tmVs, const DecodeParams& prm, pa_dtype io, pa_dtype cache, int grid,
                            cudaStream_t stream) {
  if ((cache != PA_I8 && cache != PA_FP8_E4M3) || (io != PA_F16 && io != PA_BF16) || prm.dim != kDim)
    return fail(PA_ERR_UNSUPPORTED, "tensor-core decode: 8-bit caches need fp16/bf16 I/O and head_dim 128");
  const bool small = prm.GQ <= 8;
  const void* fn = io == PA_BF16 ? (small ? tc8_fn_for<__nv_bfloat16, 8>(cache) : tc8_fn_for<__nv_bfloat16, 16>(cache))
                                 : (small ? tc8_fn_for<__half, 8>(cache) : tc8_fn_for<__half, 16>(cache));
  const size_t smem = smem_bytes(small ? 8 : 16);
  static std::mutex m;
  static std::vector<const void*> ready;
  {
    std::lock_guard<std::mutex> lock(m);
    if (std::find(ready.begin(), ready.end(), fn) == ready.end()) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(8-bit tensor-core decode)");
      ready.push_back(fn);
    }
  }
  CUtensorMap k = tmK, v = tmV, ks = tmKs, vs = tmVs;
  DecodeParams p = prm;
  void* args[] = {&k, &v, &ks, &vs, &p};
  cudaError_t err = launch_dependent(fn, dim3(grid), dim3(base_threads(small ? 8 : 16)), smem, stream, args);
  if (err != cudaSuccess) return cuda_fail(err, "launching the 8-bit tensor-core decode kernel");
  return PA_OK;
}

}  // namespace pa
