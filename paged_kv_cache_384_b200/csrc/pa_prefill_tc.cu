// pa_prefill_tc.cu -- paged prefill / chunked-prefill attention on the 5th-generation tensor
// cores (sm_100a).
//
// Each sequence brings q_len new query tokens whose K/V rows are already in the paged cache
// (written by reshape_and_cache).  Query i of the chunk sits at position ctx - q_len + i
// and attends causally: tokens [lo, pos] with lo = pos - window + 1 (clamped at 0) when a
// window is set.  The pages motivate the operation (a prompt stage that writes many tokens'
// K/V at once: "vLLM source first look: PagedAttention memory design" (trdm.cn), section
// 四; long single-sequence contexts: "KV Cache memory optimisation and PagedAttention"
// (yunthe.com), section "PagedAttention在不同推理场景下的适用性") and fix the cache layout
// and block-table walk (the same page, section "PagedAttention注意力计算流程"); the causal
// rule is the usual definition and the tiling below is this library's design.
//
// A persistent grid (one CTA per SM) works through units of 128 query rows of one cached
// head: tq = 128 / GQ consecutive query tokens times the GQ query heads that share the
// cached head (row = token * GQ + head; GQ a power of two up to 128, so multi-query
// attention with up to 128 query heads per cached head fits one unit's rows).  Per 128-token KV tile of a unit:
//
//   S[128 rows x 128 kv]  = Q[128 x 128 d] . K^T          (K-major A and B in shared memory)
//   O_h[128 rows x 128 d] += P[:, 64h..] . V[64h.., :]   (A = P in TMEM over S, MN-major V)
//
// with fp32 accumulators in TMEM.  Keeping P in tensor memory leaves shared memory to the
// q rows and 3-deep K and V rings.
//
// Roles (one CTA per SM, 16 warps in four warpgroups; registers are moved with setmaxnreg
// from the copy and MMA warpgroups, 64 each, to the softmax warpgroups, 192 each):
//   warp 0       TMEM owner and MMA issuer (one lane), polling: score MMA of the next tile
//                whose K landed, value MMA of the tile whose probabilities are written.
//   warps 1..3   TMA producers: K (both 64-dim halves, warp 1) into a 3-deep ring, V and
//                each unit's q rows (lo half warp 2, hi half warp 3) into another (128-byte
//                swizzle, one copy per lane); block ids are fetched in prefetched windows.
//                (warps 4..7 idle)
//   warps 8..15  softmax, two warps per query row (TMEM lane), each with its own half of
//                every tile's kv tokens and its own accumulator O_h: scale, causal/window
//                mask, online softmax in base 2 with a lazily moved reference maximum (O_h
//                is rescaled only when the half's maximum grows by more than 2^8),
//                probabilities into TMEM as the A operand; the halves are merged when the
//                unit's rows are written, which happens after the next unit's first tile.
// bf16 probabilities are split into hi + lo bf16 parts (two value MMAs) so the weights keep
// ~16 significant bits.
// 8-bit caches (INT8 or FP8 E4M3 codes with one fp16 scale per token and cached head, "KV
// Cache optimisation strategies in deployment" (yunthe.com), section
// "量化压缩KV Cache的INT8与FP8方案"): the copy warps bring each tile's codes (one 128-byte row
// per token) into the lo half of its ring slot, and warps 4..7, one thread per kv row, turn
// them in place into the 16-bit operand -- code times the row's scale, rounded once: K to
// the I/O type (relative error 2^-11 for fp16, 2^-8 for bf16), V to fp16 (2^-11) -- with
// zeros in rows no query attends; the MMA warp then sees an ordinary 16-bit tile, and the
// value MMA runs in fp16 with fp16 weights whatever the I/O type (no hi + lo split).
// head_dim 64 (16-bit caches): q, K and V use only the lo 64-dim halves of their slots, the
// score MMAs take 4 K-steps instead of 8 and the value MMA has N = 64; each softmax warp
// writes 32 of a row's 64 output dims.
// Every wait is bounded; one that gives up raises PA_DEVERR_TIMEOUT and an abort flag that
// ends the others.
#include <cfloat>
#include <mutex>
#include <type_traits>
#include <vector>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tmap.h"

namespace pa {

static __device__ unsigned int g_prefill_error;

__device__ __forceinline__ void prefill_error(unsigned int bits) { atomicOr(&g_prefill_error, bits); }

namespace {

constexpr int kRows = 128;                // query rows per CTA (MMA M)
constexpr int kKv = 128;                  // kv tokens per tile
constexpr int kDim = 128;                 // largest head_dim (64 uses the lo halves only)
constexpr int kHalf = 128 * 128;          // one 64-element half of a 128-row operand: 16 KiB
constexpr int kOpBytes = 2 * kHalf;       // a whole 128 x 128 operand (Q, K, V or P)
constexpr int kRing = 3;                  // depth of the K ring and of the V ring
constexpr int kSoftmaxThreads = 256;      // 8 warps: two per TMEM lane quarter, 64 columns each
constexpr int kThreads = 256 + kSoftmaxThreads;  // + 4 copy warps, MMA warpgroup
// Registers: the launch gives every thread 128 (65536 / 512); the copy and MMA warpgroups
// hand back down to kRegsLow, the softmax warpgroups take kRegsHigh.  The split must add up
// to the launch's 65536 exactly or less, else the increase waits for ever.
constexpr int kRegsLaunch = 128, kRegsLow = 64, kRegsHigh = 192;
static_assert(256 * kRegsLow + 256 * kRegsHigh <= kThreads * kRegsLaunch, "register split exceeds the launch's");
static_assert(kRegsLow % 8 == 0 && kRegsHigh % 8 == 0, "setmaxnreg counts are multiples of 8");
constexpr uint32_t kTmemCols = 512;       // S0 [0,128)  S1 [128,256)  O_0 [256,384)  O_1 [384,512)
// Each softmax half h owns the 64 score columns [64h, 64h+64) of an S buffer and writes its
// probabilities over them: hi weights in the first 32 columns (two 16-bit weights per
// column), the lo parts of bf16 weights in the next 32.  Half h accumulates O_h over its
// own kv tokens with its own running maximum; the halves are combined once at the end.
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.f;  // log2 units: probabilities stay below 2^8

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(1 + 2 * kRing) * kOpBytes;  // Q, K ring, V ring

struct PrefillParams {
  void* out;
  const uint16_t* k_scale;  // [NB*bs][Hkv] fp16 bits (8-bit cache only)
  const uint16_t* v_scale;
  const int32_t* block_tables;
  const int32_t* cu_q;
  const int32_t* context_lens;
  int S, T, Hq, Hkv, GQ, gq_shift, tq, bs, MB, NB, window, max_q_len;
  int dim;       // head_dim: 128, or 64 (16-bit cache; the hi 64-dim halves stay unused)
  int qtiles;    // query tiles of the longest sequence: ceil(max_q_len / tq)
  int units;     // S * Hkv * qtiles work units, walked by a persistent grid
  float qscale;  // scale * log2(e)
};

struct PfShared {
  uint64_t q_full, q_empty, o_free;  // q rows landed / read by the last score MMA; O read out
  uint64_t k_full[kRing], k_empty[kRing], v_full[kRing], v_empty[kRing];
  uint64_t k_conv[kRing], v_conv[kRing];  // 8-bit codes of a slot widened into the operand
  uint64_t s_full[2];
  uint64_t p_full[2], o_full[2];  // by tile parity: probabilities written / value MMA done
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  float xch[2][kRows];  // the two softmax halves of a row combine (m, l) through here
};

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int* abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
  }
  *abort = 1;
  prefill_error(PA_DEVERR_TIMEOUT);
  return false;
}

// Two weights rounded to IO by one packed conversion, with their values back in fp32.
template <typename IO> struct Pair;
template <> struct Pair<__half> {
  __half2 v;
  uint32_t bits;
  __device__ __forceinline__ Pair(float a, float b) : v(__floats2half2_rn(a, b)) {
    bits = *reinterpret_cast<const uint32_t*>(&v);
  }
  __device__ __forceinline__ float lo_f() const { return __low2float(v); }
  __device__ __forceinline__ float hi_f() const { return __high2float(v); }
};
template <> struct Pair<__nv_bfloat16> {
  __nv_bfloat162 v;
  uint32_t bits;
  __device__ __forceinline__ Pair(float a, float b) : v(__floats2bfloat162_rn(a, b)) {
    bits = *reinterpret_cast<const uint32_t*>(&v);
  }
  __device__ __forceinline__ float lo_f() const { return __uint_as_float(bits << 16); }
  __device__ __forceinline__ float hi_f() const { return __uint_as_float(bits & 0xFFFF0000u); }
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Logical blocks of KV tile j that hold tokens some row of this CTA attends.
struct TileBlocks {
  int first, lo, hi;
};
__device__ __forceinline__ TileBlocks tile_blocks(int jt, int bs, int kv_lo, int p_max) {
  TileBlocks t;
  t.first = jt * kKv / bs;
  t.lo = max(t.first, kv_lo / bs);
  t.hi = min(t.first + kKv / bs - 1, p_max / bs);
  return t;
}

// One unit of work: 128 query rows (query tile qt of sequence s, cached head kh).  Units
// are numbered with the query tile fastest (heaviest first), so the CTAs working at the
// same time share the K/V tiles of a few (sequence, head) pairs in L2.  The persistent
// grid deals them out in rounds of gridDim.x, in alternate directions (CTA c takes the
// c-th unit of even rounds and the c-th from the end of odd ones), which evens out the
// causal tiles' unequal costs.
__device__ __forceinline__ int unit_of(int k) {  // k-th unit of this CTA
  const int G = gridDim.x;
  return k * G + ((k & 1) ? G - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x));
}
struct Unit {
  int s, kh, q_start, i0, ntok, ctx, p_min, p_max, kv_lo, j_lo, n;
};
// Unit u from its sequence's bounds q_start, q_end (cu_q_lens) and ctx (context_lens);
// false if the unit holds no query rows.
__device__ __forceinline__ bool unit_at(const PrefillParams& p, int u, int q_start, int q_end, int ctx, Unit* w) {
  const int qt = p.qtiles - 1 - u % p.qtiles;
  const int g = u / p.qtiles;
  w->kh = g % p.Hkv;
  w->s = g / p.Hkv;
  const int q_len = q_end - q_start;
  if (q_start < 0 || q_len < 0 || q_start + q_len > p.T || q_len > ctx || ctx > p.MB * p.bs || q_len > p.max_q_len) {
    if (threadIdx.x == 0) prefill_error(PA_DEVERR_CONTEXT);
    return false;
  }
  w->i0 = qt * p.tq;
  if (w->i0 >= q_len) return false;
  w->q_start = q_start;
  w->ctx = ctx;
  w->ntok = min(p.tq, q_len - w->i0);
  w->p_min = ctx - q_len + w->i0;  // positions of the unit's first and last query
  w->p_max = w->p_min + w->ntok - 1;
  w->kv_lo = p.window > 0 ? max(0, w->p_min - p.window + 1) : 0;
  w->j_lo = w->kv_lo / kKv;
  w->n = w->p_max / kKv - w->j_lo + 1;  // KV tiles
  return true;
}

// Walks this CTA's units in order.  The sequence bounds of the next candidate are loaded
// while the current unit is worked on, so moving on rarely waits for memory.
struct UnitCursor {
  int k, u, q0, q1, ctx;
  __device__ __forceinline__ void fetch(const PrefillParams& p) {
    u = unit_of(k);
    if (u < p.units) {
      const int s = u / p.qtiles / p.Hkv;
      q0 = __ldg(p.cu_q + s);
      q1 = __ldg(p.cu_q + s + 1);
      ctx = __ldg(p.context_lens + s);
    }
  }
  __device__ __forceinline__ void start(const PrefillParams& p) {
    k = 0;
    fetch(p);
  }
  // The next unit holding query rows; false once the list is done.
  __device__ __forceinline__ bool next(const PrefillParams& p, Unit* w) {
    while (u < p.units) {
      const bool has = unit_at(p, u, q0, q1, ctx, w);
      ++k;
      fetch(p);
      if (has) return true;
    }
    return false;
  }
};

// Block-table entries of one sequence, 32 at a time, one per lane: the window in use and
// the next one, whose load is in flight while the current one serves.
struct TableWindow {
  const int32_t* table;
  int lim, base, cur, next;
  __device__ __forceinline__ int fetch(int from, int lane) const {
    return from + lane < lim ? __ldg(table + from + lane) : 0;
  }
  __device__ __forceinline__ void init(const int32_t* t, int limit, int first, int lane) {
    table = t;
    lim = limit;
    base = first;
    cur = fetch(first, lane);
    next = fetch(first + 32, lane);
  }
  // Lane l (< count <= 16) gets the entry of block lo + l; lo never decreases.
  __device__ __forceinline__ int get(int lo, int count, int lane) {
    while (lo >= base + 32) {
      base += 32;
      cur = next;
      next = fetch(base + 32, lane);
    }
    const int idx = lo - base + lane;
    const int a = __shfl_sync(0xffffffffu, cur, idx & 31);
    if (lo - base + count <= 32) return a;  // uniform: the tile lies in the current window
    const int b = __shfl_sync(0xffffffffu, next, idx & 31);
    return idx < 32 ? a : b;
  }
};

// Warps 0..7 (the copy and MMA warpgroups) hold the MMA warp and the copy warps.  A copy
// warp's role is 4 * tensor + halves (tensor 0 = K, 1 = V; halves: bit 0 the lo 64-dim half,
// bit 1 the hi half); -1 = none.  Every SM sub-partition (warp % 4) also runs two softmax
// warps, and those measured ~0.45 us per tile slower when two busy warps (two copy warps,
// or a copy warp and the MMA warp) shared their sub-partition; the softmax warps gate the
// value MMA, so the busy warps sit on different sub-partitions: the MMA warp on 0, K (both
// halves) on 1, V lo on 2, V hi on 3.  Warps 4..7 are idle.
constexpr int kMmaWarp = 0;
constexpr int kCopyWarpsK = 1, kCopyWarpsV = 2;  // copy warps per tensor
constexpr int kConvWarp0 = 4, kConvThreads = 128;  // warps 4..7 widen 8-bit codes, one kv row each
__device__ __forceinline__ int copy_role(int warp) {
  switch (warp) {
    case 1: return 3;      // K, both halves
    case 2: return 4 + 1;  // V, lo half
    case 3: return 4 + 2;  // V, hi half
    default: return -1;
  }
}

// 16 8-bit codes (one 16-byte chunk) times a scale, rounded to IO: out[0..3] hold codes 0..7,
// out[4..7] codes 8..15, two per word, the lower code in the lower half.  fp16: the codes
// widen exactly to f16 pairs, then one f16x2 multiply rounds each product once.  bf16: the
// codes widen exactly to fp32, the product is rounded to fp32 and then to bf16.
template <typename IO, typename CT>
__device__ __forceinline__ void widen_scaled16(const uint4& in, float scale, uint32_t* out) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  if constexpr (std::is_same<IO, __half>::value) {
    const __half2 s2 = __float2half2_rn(scale);  // the stored fp16 scale: exact
    const uint32_t sb = *reinterpret_cast<const uint32_t*>(&s2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t lo, hi;
      if constexpr (std::is_same<CT, int8_t>::value) {
        // c + 128 spliced under the exponent of 1024, minus 1152: exact f16 codes
        const uint32_t u = w[i] ^ 0x80808080u;
        const uint32_t bias = 0x64806480u;
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(lo) : "r"(__byte_perm(u, 0x6464u, 0x4140u)), "r"(bias));
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(hi) : "r"(__byte_perm(u, 0x6464u, 0x4342u)), "r"(bias));
      } else {
        e4m3x4_to_f16x2x2(w[i], lo, hi);
      }
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[2 * i]) : "r"(lo), "r"(sb));
      asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(out[2 * i + 1]) : "r"(hi), "r"(sb));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float f[4];
      if constexpr (std::is_same<CT, int8_t>::value) {
        const uint32_t u = w[i] ^ 0x80808080u;
#pragma unroll
        for (int b = 0; b < 4; ++b) f[b] = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7440u | b)) - 8388736.0f;
      } else {
        uint32_t lo, hi;
        e4m3x4_to_f16x2x2(w[i], lo, hi);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&lo));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hi));
        f[0] = a.x, f[1] = a.y, f[2] = b.x, f[3] = b.y;
      }
      const __nv_bfloat162 p0 = __floats2bfloat162_rn(f[0] * scale, f[1] * scale);
      const __nv_bfloat162 p1 = __floats2bfloat162_rn(f[2] * scale, f[3] * scale);
      out[2 * i] = *reinterpret_cast<const uint32_t*>(&p0);
      out[2 * i + 1] = *reinterpret_cast<const uint32_t*>(&p1);
    }
  }
}

template <int N> __device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N> __device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

template <typename IO, typename CT>
__global__ void __launch_bounds__(kThreads, 1)  // 16 warps, 128 registers each at launch
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const PrefillParams p) {
  constexpr bool kQuant = !std::is_same<CT, IO>::value;  // 8-bit codes + per-token scales
  constexpr bool kSplit = std::is_same<IO, __nv_bfloat16>::value && !kQuant;
  constexpr uint32_t kFmt = std::is_same<IO, __nv_bfloat16>::value ? 1u : 0u;
  constexpr uint32_t kIdescS = mma_idesc_f16(kFmt, 0, 0, kRows, kKv);  // K-major Q and K
  // With an 8-bit cache the value MMA runs in fp16 whatever q's type: V rows (code x scale)
  // and the weights then keep 11 significant bits (8 in bf16).
  using PW = typename std::conditional<kQuant, __half, IO>::type;  // probability / V operand type
  constexpr uint32_t kIdescO = mma_idesc_f16(kQuant ? 0u : kFmt, 0, 1, kRows, kDim);  // K-major P, MN-major V
  constexpr uint32_t kIdescO64 = mma_idesc_f16(kQuant ? 0u : kFmt, 0, 1, kRows, 64);  // head_dim 64
  const int nhalf = p.dim / 64;  // 64-dim halves of q, K, V and O in use (1 or 2)

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ PfShared sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_launch_next();
  grid_dependency_wait();
  const int bs = p.bs;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // swizzle atoms are 1024-B aligned
  const uint32_t sQ = base;
  auto sK = [&](int st) { return base + kOpBytes + st * kOpBytes; };
  auto sV = [&](int st) { return base + (1 + kRing) * kOpBytes + st * kOpBytes; };
  const uint32_t q_full = smem_u32(&sh.q_full), q_empty = smem_u32(&sh.q_empty), o_free = smem_u32(&sh.o_free);
  const uint32_t k_full0 = smem_u32(&sh.k_full[0]), k_empty0 = smem_u32(&sh.k_empty[0]);
  const uint32_t v_full0 = smem_u32(&sh.v_full[0]), v_empty0 = smem_u32(&sh.v_empty[0]);
  const uint32_t k_conv0 = smem_u32(&sh.k_conv[0]), v_conv0 = smem_u32(&sh.v_conv[0]);
  // The MMA warp's operands are complete once the copies landed (16-bit cache) or once the
  // codes were widened (8-bit cache).
  const uint32_t k_ready0 = kQuant ? k_conv0 : k_full0, v_ready0 = kQuant ? v_conv0 : v_full0;
  const uint32_t s_full0 = smem_u32(&sh.s_full[0]);
  const uint32_t p_full0 = smem_u32(&sh.p_full[0]), o_full0 = smem_u32(&sh.o_full[0]);
  const uint32_t mma_done = smem_u32(&sh.mma_done);
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    mbar_init(q_full, kCopyWarpsV);  // the V copy warps bring the q rows' halves
    mbar_init(q_empty, 1);
    mbar_init(o_free, kSoftmaxThreads);
    for (int st = 0; st < kRing; ++st) {
      mbar_init(k_full0 + 8 * st, kCopyWarpsK);  // one arrival per copy warp of the tensor
      mbar_init(k_empty0 + 8 * st, 1);
      mbar_init(v_full0 + 8 * st, kCopyWarpsV);
      mbar_init(v_empty0 + 8 * st, 1);
      mbar_init(k_conv0 + 8 * st, kConvThreads);
      mbar_init(v_conv0 + 8 * st, kConvThreads);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full0 + 8 * b, 1);
      mbar_init(p_full0 + 8 * b, kSoftmaxThreads);
      mbar_init(o_full0 + 8 * b, 1);
    }
    mbar_init(mma_done, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;
  // Each role ends with the CTA-wide barrier of its own (bar.sync 0 from every warp), after
  // which the MMA warp releases TMEM.  setmaxnreg sits at the top of each role's branch.
  auto end_barrier = [&]() {
    tc_fence_before_sync();
    __syncthreads();
  };

  // Every role walks the same units in the same order; tile counters (ring slots and
  // barrier parities) and unit counters run on across units.
  if (warp < 8) {
    regs_decrease<kRegsLow>();
    const int cr = copy_role(warp);
    if (cr >= 0) {
      // ------------------------------------------------------------------ TMA producers --
      // The K warps load their 64-dim halves of K, the V warps those of V and of each unit's
      // q rows (once the last score MMA of the previous unit has read them), each tensor
      // into its own ring, one copy (a half of one block) per lane.  A warp's copies go out
      // one after another (~60 ns each).  Each warp walks the block table through its own
      // prefetched window.
      const bool is_v = cr >= 4;
      const int nh = (cr & 3) == 3 ? 2 : 1;    // halves this warp copies
      const int h0 = (cr & 3) == 2 ? 1 : 0;    // its first half
      const uint64_t keep = l2_policy_evict_last();    // K/V tiles are shared by the sequence's q tiles
      const uint64_t once = l2_policy_evict_first();   // q rows are read once
      const CUtensorMap* map = is_v ? &tmV : &tmK;
      if (lane == 0) {
        prefetch_tensormap(map);
        if (is_v) prefetch_tensormap(&tmQ);
      }
      const uint32_t full0 = is_v ? v_full0 : k_full0, empty0 = is_v ? v_empty0 : k_empty0;
      int gt = 0, uq = 0;
      bool ok = true;
      UnitCursor cur;
      cur.start(p);
      Unit w;
      while (ok && cur.next(p, &w)) {
        if (is_v) {
          if (lane == 0) {
            ok = uq == 0 || wait_or_abort(q_empty, (uq - 1) & 1, abort);
            if (ok) {
              const int nq = max(0, min(h0 + nh, nhalf) - h0);  // halves of q this warp brings
              mbar_arrive_expect_tx(q_full, nq * kHalf);
              for (int dh = h0; dh < h0 + nq; ++dh)
                tma_load_3d(sQ + dh * kHalf, &tmQ, q_full, dh * 64, w.kh * p.GQ, w.q_start + w.i0, once);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
        }
        TableWindow win;
        win.init(p.block_tables + static_cast<size_t>(w.s) * p.MB, w.p_max / bs + 1,
                 tile_blocks(w.j_lo, bs, w.kv_lo, w.p_max).lo, lane);
        for (int j = 0; j < w.n; ++j, ++gt) {
          const int st = gt % kRing;
          bool ready = true;
          if (lane == 0 && gt >= kRing) ready = wait_or_abort(empty0 + 8 * st, ((gt / kRing) - 1) & 1, abort);
          if (!__shfl_sync(0xffffffffu, ready, 0)) {
            ok = false;
            break;
          }
          const TileBlocks tb = tile_blocks(w.j_lo + j, bs, w.kv_lo, w.p_max);
          const int nload = tb.hi - tb.lo + 1;
          int pb = win.get(tb.lo, nload, lane);
          if (lane < nload && (pb < 0 || pb >= p.NB)) {
            if (!is_v && h0 == 0) prefill_error(PA_DEVERR_TABLE);
            pb = 0;
          }
          // 8-bit cache: one copy per block (a token's 128 codes are one 128-byte row) into
          // the slot's lo half, by the K warp and the V lo warp; the V hi warp only arrives.
          // head_dim 64: the lo halves only.
          const int ncopy = kQuant ? (is_v && h0 == 1 ? 0 : 1) : max(0, min(h0 + nh, nhalf) - h0);  // per block
          if (lane == 0) mbar_arrive_expect_tx(full0 + 8 * st, static_cast<uint32_t>(ncopy * nload) * bs * 128u);
          __syncwarp();
          const int bi = ncopy == 2 ? lane >> 1 : lane;  // block of this lane's copy
          const int dh = ncopy == 2 ? lane & 1 : (kQuant ? 0 : h0);  // and its 64-dim half
          const int blk = __shfl_sync(0xffffffffu, pb, bi & 31);
          if (lane < ncopy * nload) {  // ncopy * nload <= 32 copies, one per lane
            const uint32_t row = static_cast<uint32_t>(tb.lo + bi - tb.first) * bs * 128u;
            const uint32_t dst = (is_v ? sV(st) : sK(st)) + dh * kHalf + row;
            tma_load_3d(dst, map, full0 + 8 * st, kQuant ? 0 : dh * 64, w.kh, blk * bs, keep);
          }
        }
        ++uq;
      }
      if (lane == 0) {  // never leave with copies in flight
        if (is_v && uq > 0) mbar_wait_bounded(q_full, (uq - 1) & 1);
        for (int k = gt - kRing < 0 ? 0 : gt - kRing; k < gt; ++k)
          mbar_wait_bounded(full0 + 8 * (k % kRing), (k / kRing) & 1);
      }
      __syncwarp();
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------------------- MMA issuer --
      // Polls without blocking (a nap when idle measured slower).  Score MMAs run ahead through
      // the unit list (the next unit's first scores overlap the current unit's last
      // softmax); the value MMA goes first when both are ready, since the softmax warps wait
      // on it and the next score MMA reuses its probabilities' columns.
      if (lane == 0) {
        struct Side {
          UnitCursor cur;
          bool live;
          int uq, base, n, idx;
        };
        auto next_unit = [&](Side& sd) {  // advance to the next unit holding query rows
          Unit w;
          sd.live = sd.cur.next(p, &w);
          if (sd.live) {
            sd.base += sd.n;
            sd.n = w.n;
            sd.idx = 0;
            ++sd.uq;
          }
        };
        Side S;
        S.cur.start(p);
        S.uq = -1;
        S.base = S.n = S.idx = 0;
        next_unit(S);
        Side P = S;
        bool q_ready = false;
        uint32_t idle = 0;
        while (P.live) {
          bool progressed = false;
          if (P.idx < P.n && P.base + P.idx < S.base + S.idx) {
            const int t = P.base + P.idx;
            const int st = t % kRing, b = t % 2;
            if (mbar_test_wait(p_full0 + 8 * b, (t / 2) & 1) && mbar_test_wait(v_ready0 + 8 * st, (t / kRing) & 1) &&
                (P.idx > 0 || P.uq == 0 || mbar_test_wait(o_free, (P.uq - 1) & 1))) {
              tc_fence_after_sync();
              const uint32_t idesc_o = nhalf == 2 ? kIdescO : kIdescO64;
  #pragma unroll
              for (int part = 0; part < (kSplit ? 2 : 1); ++part) {
  #pragma unroll
                for (int kk = 0; kk < kKv / 16; ++kk) {  // O_h += P_h . V_h, 16 kv tokens per MMA
                  const int h = kk / 4;                    // softmax half owning these tokens
                  tc_mma_f16_ts(tmem + kColO + 128 * h, tmem + b * kKv + 64 * h + 32 * part + (kk % 4) * 8,
                                smem_desc(sV(st) + kk * 2048, kHalf, 1024, kSwizzle128B), idesc_o,
                                P.idx > 0 || part > 0 || (kk % 4) > 0);
                }
              }
              tc_commit(o_full0 + 8 * b);
              tc_commit(v_empty0 + 8 * st);
              if (++P.idx == P.n) next_unit(P);
              progressed = true;
            }
          }
          if (S.live) {
            const int t = S.base + S.idx;
            const int st = t % kRing, b = t % 2;
            if (!q_ready) q_ready = mbar_test_wait(q_full, S.uq & 1);
            // S(t) lands on P(t - 2): the value MMA that reads it must be issued first.
            if (q_ready && t - 1 <= P.base + P.idx && mbar_test_wait(k_ready0 + 8 * st, (t / kRing) & 1)) {
              tc_fence_after_sync();
  #pragma unroll
              for (int kk = 0; kk < kDim / 16; ++kk) {  // S[b] = Q . K^T, 16 dims per MMA
                if (kk >= 4 * nhalf) break;
                const uint32_t off = (kk / 4) * kHalf + (kk % 4) * 32;
                tc_mma_f16(tmem + b * kKv, smem_desc(sQ + off, 16, 1024, kSwizzle128B),
                           smem_desc(sK(st) + off, 16, 1024, kSwizzle128B), kIdescS, kk > 0);
              }
              tc_commit(s_full0 + 8 * b);
              tc_commit(k_empty0 + 8 * st);
              if (++S.idx == S.n) {
                tc_commit(q_empty);  // the q rows may be replaced once these MMAs are done
                q_ready = false;
                next_unit(S);
              }
              progressed = true;
            }
          }
          if (progressed) {
            idle = 0;
          } else if (*abort || ++idle > kWaitLimit) {
            if (!*abort) prefill_error(PA_DEVERR_TIMEOUT);
            *abort = 1;
            break;
          }
        }
        tc_commit(mma_done);  // every MMA issued above has finished before TMEM is released
        mbar_wait_bounded(mma_done, 0);
      }
      __syncwarp();
    } else if (kQuant && warp >= kConvWarp0) {
      // --------------------------------------------------------------- 8-bit widening --
      // Thread r owns kv row r of every tile.  It looks up its token's block and scales
      // while the copies are in flight, then rewrites its row of the slot: dims 64..127
      // into the hi half first, then dims 0..63 over the codes' own 128 bytes (both in the
      // 128-byte-swizzled operand layout; chunk c of row r sits at c ^ (r & 7)).  Rows of
      // tokens outside the loaded blocks or past the context become zeros (their codes may
      // be anything, NaN included).
      const int r = 32 * (warp - kConvWarp0) + lane;
      const uint32_t sw = r & 7;
      // Code chunk c (codes 16c .. 16c + 15) becomes operand chunks 2c and 2c + 1 of the lo
      // half (c < 4) or, less 4, of the hi half.  Two chunks at a time (two independent
      // chains in flight within the 64 registers of this warpgroup), in the order (4, 5),
      // (6, 7) -- the hi half -- then (3, 2), (1, 0), so every lo chunk written over the
      // codes' own bytes was read already.  The loop stays rolled (fully unrolled code starved
      // the warps of instructions).
      auto widen_row = [&](uint32_t row, bool live, float sc, bool to_half) {
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
          const int c0 = i < 2 ? 4 + 2 * i : 7 - 2 * i, c1 = i < 2 ? c0 + 1 : c0 - 1;
          const uint4 raw0 = ld_shared_v4(row + 16 * (c0 ^ sw)), raw1 = ld_shared_v4(row + 16 * (c1 ^ sw));
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int c = k ? c1 : c0;
            uint32_t o[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (live) {
              if (to_half) widen_scaled16<__half, CT>(k ? raw1 : raw0, sc, o);
              else widen_scaled16<IO, CT>(k ? raw1 : raw0, sc, o);
            }
            const uint32_t dst = row + (c >= 4 ? kHalf : 0);
            const int m = 2 * (c & 3);
            st_shared_v4(dst + 16 * (m ^ sw), o[0], o[1], o[2], o[3]);
            st_shared_v4(dst + 16 * ((m + 1) ^ sw), o[4], o[5], o[6], o[7]);
          }
        }
        fence_proxy_async_shared();  // the operand is read by the tensor cores
      };
      // The tiles of this CTA in order, with this thread's row of each: whether it is live,
      // its block-table entry and its scales.  Loads run two tiles ahead: while a tile is
      // widened, the block-table entry of the tile after next and the scales of the next tile
      // (from the entry loaded one tile earlier) are in flight, so neither dependent global
      // load sits on the critical path.
      struct RowRef {
        bool ok, live;
        int kv, s, kh, pb;
        uint16_t ks, vs;  // fp16 bits of the scales (live rows)
      };
      UnitCursor cur;
      cur.start(p);
      Unit w;
      int j = 0;
      bool more = cur.next(p, &w);
      auto take = [&](RowRef& t) {  // the next tile's row: table entry loaded, scales not yet
        t.ok = more;
        if (!more) return;
        const int kv0 = (w.j_lo + j) * kKv;
        const TileBlocks tb = tile_blocks(w.j_lo + j, bs, w.kv_lo, w.p_max);
        t.live = r >= tb.lo * bs - kv0 && r < min(w.ctx, (tb.hi + 1) * bs) - kv0;
        t.kv = kv0 + r;
        t.s = w.s;
        t.kh = w.kh;
        t.ks = t.vs = 0;
        t.pb = t.live ? __ldg(p.block_tables + static_cast<size_t>(w.s) * p.MB + t.kv / bs) : 0;
        if (++j == w.n) {
          j = 0;
          more = cur.next(p, &w);
        }
      };
      auto scales = [&](RowRef& t) {
        if (!t.ok || !t.live) return;
        const int pb = (t.pb < 0 || t.pb >= p.NB) ? 0 : t.pb;  // reported by the K copy warp
        const size_t srow = (static_cast<size_t>(pb) * bs + t.kv % bs) * p.Hkv + t.kh;
        t.ks = __ldg(p.k_scale + srow);
        t.vs = __ldg(p.v_scale + srow);
      };
      RowRef now, nxt, after;
      take(now);
      scales(now);
      take(nxt);
      for (int gt = 0; now.ok; ++gt) {
        take(after);   // block-table entry of the tile after next: in flight
        scales(nxt);   // scales of the next tile: in flight while this tile is widened
        const int st = gt % kRing;
        if (!__all_sync(0xffffffffu, wait_or_abort(k_full0 + 8 * st, (gt / kRing) & 1, abort))) break;
        widen_row(sK(st) + r * 128, now.live, __half2float(__ushort_as_half(now.ks)), false);
        mbar_arrive(k_conv0 + 8 * st);
        if (!__all_sync(0xffffffffu, wait_or_abort(v_full0 + 8 * st, (gt / kRing) & 1, abort))) break;
        widen_row(sV(st) + r * 128, now.live, __half2float(__ushort_as_half(now.vs)), true);
        mbar_arrive(v_conv0 + 8 * st);
        now = nxt;
        nxt = after;
      }
    }
    end_barrier();
    if (warp == kMmaWarp) {
      tc_fence_after_sync();
      tmem_dealloc(tmem, kTmemCols);
    }
  } else {
    regs_increase<kRegsHigh>();
    // ------------------------------------------------------------- softmax warps --
    // Warps 8..15.  A warp may only touch the TMEM lane quarter (warp % 4); the two warps of
    // a quarter share its 32 query rows and split each tile's kv tokens: half h takes
    // tokens [64h, 64h + 64).  Each half runs its own online softmax (maximum, sum and
    // output accumulator O_h), so the halves never wait for each other within a unit;
    // they combine when the unit is finished.  A unit is finished (its rows written out)
    // after the probabilities of the next unit's first tile: that tile never touches O, its
    // scores are ready early, and by then the unit's last value MMA is long done, so the
    // softmax warps do not sit idle at unit boundaries.  Both halves finish every unit, with
    // both exchange barriers, even after a failed wait (then doing no other work), so
    // neither can leave the other waiting at a barrier.
    const int q4 = warp & 3;
    const int half = (warp - 8) >> 2;
    const int r = 32 * q4 + lane;  // query row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const uint32_t o_col = tmem + lane_addr + kColO + 128 * half;
    const uint32_t pair_bar = 1 + q4;
    const int tl = r >> p.gq_shift, g = r & (p.GQ - 1);
    // Bounded wait for the value MMA of tile t, agreed by the whole warp.
    auto wait_pv = [&](int t) {
      return __all_sync(0xffffffffu, wait_or_abort(o_full0 + 8 * (t % 2), (t / 2) & 1, abort));
    };
    // The unit whose rows are still to be written (its last tile is gt - 1): this thread's
    // maximum and sum, and its output row (token * Hq + head; -1: no query row here).
    // pend_row == -2: none.
    float pend_m = 0.f, pend_l = 0.f;
    int pend_row = -2;
    bool ok = true;
    int gt = 0;
    auto finish = [&]() {
      const bool fin = ok && wait_pv(gt - 1);
      if (half == 1) {
        sh.xch[0][r] = pend_m;
        sh.xch[1][r] = pend_l;
      }
      named_barrier_sync(pair_bar, 64);
      float w_me, w_other;  // weights of O_half and O_(1-half) in the output
      if (half == 0) {
        const float m1 = sh.xch[0][r], l1 = sh.xch[1][r];
        const float m_all = fmaxf(pend_m, m1);
        const float a0 = ex2_ftz(pend_m - m_all), a1 = ex2_ftz(m1 - m_all);
        const float l_all = pend_l * a0 + l1 * a1;
        const float inv = pend_row >= 0 && l_all > 0.f ? 1.f / l_all : 0.f;
        w_me = a0 * inv;
        w_other = a1 * inv;
        sh.xch[0][r] = w_other;  // half 1's own weight
        sh.xch[1][r] = w_me;     // half 1's weight for O_0
      }
      named_barrier_sync(pair_bar, 64);
      if (half == 1) {
        w_me = sh.xch[0][r];
        w_other = sh.xch[1][r];
      }
      if (fin) {
        tc_fence_after_sync();
        const float w0 = half == 0 ? w_me : w_other, w1 = half == 0 ? w_other : w_me;
        const int hd = 32 * nhalf;  // head dims this warp writes: 64, or 32 at head_dim 64
        IO* orow = reinterpret_cast<IO*>(p.out) + static_cast<size_t>(pend_row) * p.dim + hd * half;
#pragma unroll
        for (int c4 = 0; c4 < 2; ++c4) {  // this warp's head dims, 32 at a time
          if (c4 >= nhalf) break;
          float o0[32], o1[32];
          tmem_load32(tmem + lane_addr + kColO + hd * half + 32 * c4, o0);
          tmem_load32(tmem + lane_addr + kColO + 128 + hd * half + 32 * c4, o1);
          if (pend_row >= 0) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t wd[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = 8 * v + 2 * e;
                wd[e] = Pair<IO>(o0[c] * w0 + o1[c] * w1, o0[c + 1] * w0 + o1[c + 1] * w1).bits;
              }
              *reinterpret_cast<uint4*>(orow + 32 * c4 + 8 * v) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
          }
        }
        tc_fence_before_sync();
        mbar_arrive(o_free);  // O_0 and O_1 may now be overwritten by the next unit
      }
      pend_row = -2;
    };
    UnitCursor cur;
    cur.start(p);
    Unit w;
    while (cur.next(p, &w)) {
      const bool row_valid = tl < w.ntok;
      const int pos = w.p_min + tl;
      const int lo_row = p.window > 0 ? max(0, pos - p.window + 1) : 0;
      float m_run = -FLT_MAX, l = 0.f;
      for (int j = 0; j < w.n && ok; ++j) {
        const int t = gt + j;
        const int b = t % 2, st = t % kRing;
        if (!__all_sync(0xffffffffu, wait_or_abort(s_full0 + 8 * b, (t / 2) & 1, abort))) {
          ok = false;
          break;
        }
        const int kv0 = (w.j_lo + j) * kKv;
        const int c0 = 64 * half;  // this warp's first column
        const uint32_t s_col = tmem + lane_addr + b * kKv + c0;
        float sc[64];
        tc_fence_after_sync();
        tmem_load64(s_col, sc);
        // Interior tiles (every row attends every column) skip the mask.
        const bool interior = w.ntok == p.tq && kv0 + kKv - 1 <= w.p_min &&
                              (p.window <= 0 || kv0 >= w.p_max - p.window + 1);
        if (!interior) {
          const int c_lo = lo_row - kv0 - c0, c_hi = row_valid ? pos - kv0 - c0 : -1;
#pragma unroll
          for (int c = 0; c < 64; ++c) sc[c] = (c >= c_lo && c <= c_hi) ? sc[c] : -INFINITY;
        }
        float mx[8];  // eight independent chains of three-input maxima over columns k + 8i
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(sc[k], sc[8 + k]);
#pragma unroll
        for (int c = 16; c < 64; c += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sc[c + k], sc[c + 8 + k]);
        const float mraw =
            fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const float mt = mraw * p.qscale;  // scores in base-2 units (qscale > 0 keeps the order)
        float alpha = 1.f;
        bool rescale = false;
        if (mt > m_run + kRescaleThreshold) {  // move the reference maximum
          alpha = ex2_ftz(m_run - mt);
          rescale = l > 0.f;                   // O_h holds earlier contributions of this row
          l *= alpha;
          m_run = mt;
        }
        // O_h may be rescaled only after the previous value MMA.
        if (__any_sync(0xffffffffu, rescale)) {
          if (!wait_pv(t - 1)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const float a = rescale ? alpha : 1.f;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {  // the 64 * nhalf columns of O_h in use
            if (c4 >= 2 * nhalf) break;
            float o[32];
            tmem_load32(o_col + 32 * c4, o);
#pragma unroll
            for (int k = 0; k < 32; ++k) o[k] *= a;
            tmem_store32(o_col + 32 * c4, o);
          }
        }
        // V rows of tokens outside the loaded blocks or past the context may hold anything
        // (NaN); their weights are 0, so give the value MMA zeros there (kv row r; half 0
        // clears its 64-dim lo half, half 1 the hi half; at head_dim 64 the two halves clear
        // four 16-byte chunks each of the lo half).
        const TileBlocks tb = tile_blocks(w.j_lo + j, bs, w.kv_lo, w.p_max);
        const int clean_lo = tb.lo * bs - kv0, clean_hi = min(w.ctx, (tb.hi + 1) * bs) - kv0;
        if (!kQuant && (clean_lo > 0 || clean_hi < kKv)) {  // (8-bit: the widening warps wrote the zeros)
          if (!__all_sync(0xffffffffu, wait_or_abort(v_full0 + 8 * st, (t / kRing) & 1, abort))) {
            ok = false;
            break;
          }
          if (r < clean_lo || r >= clean_hi) {
            const uint32_t zrow = nhalf == 2 ? sV(st) + half * kHalf + r * 128 : sV(st) + r * 128 + 64 * half;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              if (k < 4 * nhalf) st_shared_v4(zrow + 16 * k, 0, 0, 0, 0);
          }
        }
        // Probabilities of this half's 64 tokens, written over its own score columns as the
        // A operand of the value MMA.  exp2(s * qscale - m) is one FFMA and one MUFU op; two
        // weights are rounded and packed by one conversion.  (Moving a quarter of them to a
        // polynomial on the FMA pipe measured slower: the transcendental unit is not what
        // limits this loop.)  The denominator sums the
        // unrounded weights (fp16 rounding errors of the packed weights average out).
        // The scale-and-subtract and the running sum work on packed fp32 pairs.
        uint64_t ls2[4] = {0, 0, 0, 0};
        const uint64_t q2 = f2_pack(p.qscale, p.qscale), nm2 = f2_pack(-m_run, -m_run);
#pragma unroll
        for (int q = 0; q < 2; ++q) {  // two stores of 16 columns (32 tokens) each
          uint32_t w_hi[16], w_lo[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const int c = 32 * q + 2 * k;
            float y0, y1;
            f2_unpack(f2_fma(f2_pack(sc[c], sc[c + 1]), q2, nm2), y0, y1);
            const float x0 = ex2_ftz(y0), x1 = ex2_ftz(y1);
            const Pair<PW> hi(x0, x1);
            w_hi[k] = hi.bits;
            if (kSplit) w_lo[k] = Pair<PW>(x0 - hi.lo_f(), x1 - hi.hi_f()).bits;
            ls2[k & 3] = f2_add(ls2[k & 3], f2_pack(x0, x1));
          }
          tmem_store16_bits(s_col + 16 * q, w_hi);
          if (kSplit) tmem_store16_bits(s_col + 32 + 16 * q, w_lo);
        }
        tmem_wait_store();
        float ls[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) f2_unpack(ls2[k], ls[2 * k], ls[2 * k + 1]);
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        fence_proxy_async_shared();  // zeroed V rows (if any) are read by the tensor core
        tc_fence_before_sync();
        mbar_arrive(p_full0 + 8 * b);
        if (pend_row != -2) finish();  // first tile of this unit done: finish the previous one
      }
      if (pend_row != -2) finish();  // the tile loop ended early (a failed wait)
      pend_m = m_run;
      pend_l = l;
      pend_row = row_valid ? (w.q_start + w.i0 + tl) * p.Hq + w.kh * p.GQ + g : -1;
      gt += w.n;
    }
    if (pend_row != -2) finish();
    end_barrier();
  }
}

cudaError_t read_prefill_error(uint32_t* flags, int clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_prefill_error, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (clear && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_prefill_error, &z, sizeof z);
  }
  return e;
}

struct RegisterPrefill {
  RegisterPrefill() { register_device_error_reader(read_prefill_error); }
} g_register_prefill;

}  // namespace
}  // namespace pa

using namespace pa;

namespace {

template <typename IO>
const void* prefill_kernel_for(pa_dtype cache) {
  return cache == PA_I8 ? reinterpret_cast<const void*>(&prefill_tc_kernel<IO, int8_t>)
         : cache == PA_FP8_E4M3 ? reinterpret_cast<const void*>(&prefill_tc_kernel<IO, __nv_fp8_e4m3>)
                                : reinterpret_cast<const void*>(&prefill_tc_kernel<IO, IO>);
}

pa_status prefill_launch(void* out, const void* q, const void* k_cache, const void* v_cache, const void* k_scale,
                         const void* v_scale, const int32_t* block_tables, const int32_t* cu_q_lens,
                         const int32_t* context_lens, int num_seqs, int num_q_tokens, int max_q_len, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                         float scale, int window, pa_dtype dtype, pa_dtype cache_dtype, void* stream) {
  if (num_seqs < 0 || num_q_tokens < 0 || max_q_len < 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: negative size");
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: num_q_heads must be a positive multiple of num_kv_heads");
  if (block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: block_size, num_blocks and max_blocks_per_seq must be > 0");
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: dtype must be PA_F16 or PA_BF16");
  const bool eight_bit = cache_dtype == PA_I8 || cache_dtype == PA_FP8_E4M3;
  if (cache_dtype != dtype && !eight_bit)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: the cache must hold the I/O dtype, PA_I8 or PA_FP8_E4M3");
  if (head_dim != kDim && (head_dim != 64 || eight_bit))
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: head_dim must be 128 (or 64 with a 16-bit cache)");
  const int GQ = num_q_heads / num_kv_heads;
  if (GQ > kRows || (GQ & (GQ - 1)) != 0)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: query heads per cached head must be a power of two up to 128");
  if (block_size % 8 != 0 || kKv % block_size != 0)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: block_size must be 8, 16, 32, 64 or 128");
  if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !cu_q_lens || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: NULL pointer");
  if (eight_bit && (!k_scale || !v_scale || reinterpret_cast<uintptr_t>(k_scale) % 2 ||
                    reinterpret_cast<uintptr_t>(v_scale) % 2))
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: an 8-bit cache needs 2-byte aligned k_scale and v_scale");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: out, q and the caches must be 16-byte aligned");
  if (num_seqs > 65535 || num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: at most 65535 sequences and cached heads");
  if (static_cast<long long>(max_blocks_per_seq) * block_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: max_blocks_per_seq * block_size too large");
  if (static_cast<long long>(num_q_tokens) * num_q_heads >= (1LL << 31))
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: num_q_tokens * num_q_heads must be below 2^31");

  EncodeTiledFn enc = nullptr;
  pa_status st = get_encoder(&enc);
  if (st != PA_OK) return st;
  const CUtensorMapDataType ttype = dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int tq = kRows / GQ;
  CUtensorMap tmK, tmV, tmQ;
  {
    // [NB*bs rows][Hkv][head_dim]: boxes of one block's rows x one head x 64 dims (16-bit
    // cache) or all 128 one-byte codes (8-bit cache), 128-byte swizzle
    const cuuint64_t e = eight_bit ? 1 : 2, D = static_cast<cuuint64_t>(head_dim);
    const cuuint64_t dims[3] = {D, static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[2] = {D * e, static_cast<cuuint64_t>(num_kv_heads) * D * e};
    const cuuint32_t box[3] = {eight_bit ? 128u : 64u, 1, static_cast<cuuint32_t>(block_size)};
    const CUtensorMapDataType ctype = eight_bit ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : ttype;
    if ((st = encode(enc, &tmK, ctype, 3, k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    if ((st = encode(enc, &tmV, ctype, 3, v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
  }
  {
    // q as [T][Hq][head_dim]: tq tokens x the GQ heads of one cached head x 64 dims
    const cuuint64_t D = static_cast<cuuint64_t>(head_dim);
    const cuuint64_t dims[3] = {D, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(num_q_tokens)};
    const cuuint64_t strides[2] = {D * 2, static_cast<cuuint64_t>(num_q_heads) * D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(GQ), static_cast<cuuint32_t>(tq)};
    if ((st = encode(enc, &tmQ, ttype, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
  }
  PrefillParams prm = {};
  prm.out = out;
  prm.k_scale = static_cast<const uint16_t*>(k_scale);
  prm.v_scale = static_cast<const uint16_t*>(v_scale);
  prm.block_tables = block_tables;
  prm.cu_q = cu_q_lens;
  prm.context_lens = context_lens;
  prm.S = num_seqs;
  prm.T = num_q_tokens;
  prm.Hq = num_q_heads;
  prm.Hkv = num_kv_heads;
  prm.GQ = GQ;
  prm.gq_shift = __builtin_ctz(static_cast<unsigned>(GQ));
  prm.tq = tq;
  prm.bs = block_size;
  prm.MB = max_blocks_per_seq;
  prm.NB = num_blocks;
  prm.window = window > 0 ? window : 0;
  prm.max_q_len = max_q_len;
  prm.dim = head_dim;
  prm.qtiles = (max_q_len + tq - 1) / tq;
  prm.qscale = scale * 1.4426950408889634f;

  const bool bf16 = dtype == PA_BF16;
  const void* fn = bf16 ? prefill_kernel_for<__nv_bfloat16>(cache_dtype) : prefill_kernel_for<__half>(cache_dtype);
  const size_t smem = kSmemBytes;
  // Once per kernel: the dynamic shared-memory limit, and the kernel's register count.  The
  // warpgroups' register split (setmaxnreg) adds up to exactly what a 128-register launch
  // provides; with any other allocation the kernel is not launched.
  {
    struct Entry { const void* fn; int regs; };
    static std::mutex m;
    static std::vector<Entry> seen;
    std::lock_guard<std::mutex> lock(m);
    int regs = -1;
    for (const Entry& en : seen)
      if (en.fn == fn) regs = en.regs;
    if (regs < 0) {
      cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      cudaFuncAttributes fa;
      if (e == cudaSuccess) e = cudaFuncGetAttributes(&fa, fn);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
      regs = fa.numRegs;
      seen.push_back(Entry{fn, regs});
    }
    if (regs != kRegsLaunch)
      return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: kernel built with an unexpected register count");
  }
  const long long units = static_cast<long long>(num_seqs) * num_kv_heads * prm.qtiles;
  if (units > (1LL << 30)) return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: too many query tiles");
  prm.units = static_cast<int>(units);
  int dev = 0, sms = 0;
  st = current_device(&dev, &sms);
  if (st != PA_OK) return st;
  const dim3 grid(static_cast<unsigned>(units < sms ? units : sms));  // persistent: one CTA per SM
  void* args[] = {&tmK, &tmV, &tmQ, &prm};
  cudaError_t err = launch_dependent(fn, grid, dim3(kThreads), smem, static_cast<cudaStream_t>(stream), args);
  if (err != cudaSuccess) return cuda_fail(err, "launching the prefill kernel");
  return PA_OK;
}

}  // namespace

extern "C" pa_status paged_attention_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables, const int32_t* cu_q_lens,
                                             const int32_t* context_lens, int num_seqs, int num_q_tokens,
                                             int max_q_len, int num_q_heads, int num_kv_heads, int head_dim,
                                             int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                                             int window, pa_dtype dtype, void* stream) {
  return prefill_launch(out, q, k_cache, v_cache, nullptr, nullptr, block_tables, cu_q_lens, context_lens, num_seqs,
                        num_q_tokens, max_q_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                        max_blocks_per_seq, scale, window, dtype, dtype, stream);
}

extern "C" pa_status paged_attention_prefill_quant(void* out, const void* q, const void* k_cache, const void* v_cache,
                                                   const void* k_scale, const void* v_scale,
                                                   const int32_t* block_tables, const int32_t* cu_q_lens,
                                                   const int32_t* context_lens, int num_seqs, int num_q_tokens,
                                                   int max_q_len, int num_q_heads, int num_kv_heads, int head_dim,
                                                   int block_size, int num_blocks, int max_blocks_per_seq,
                                                   float scale, int window, pa_dtype io_dtype, pa_dtype cache_dtype,
                                                   void* stream) {
  if (cache_dtype != PA_I8 && cache_dtype != PA_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill_quant: cache_dtype must be PA_I8 or PA_FP8_E4M3");
  return prefill_launch(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, cu_q_lens, context_lens, num_seqs,
                        num_q_tokens, max_q_len, num_q_heads, num_kv_heads, head_dim, block_size, num_blocks,
                        max_blocks_per_seq, scale, window, io_dtype, cache_dtype, stream);
}
