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
// One CTA owns 128 query rows of one cached head: tq = 128 / GQ consecutive query tokens
// times the GQ query heads that share the cached head (row = token * GQ + head).  Per
// 128-token KV tile:
//
//   S[128 rows x 128 kv]  = Q[128 x 128 d] . K^T          (K-major A and B; fp32 in TMEM)
//   O[128 rows x 128 d]  += P[128 x 128 kv] . V           (K-major A, MN-major B; fp32 in TMEM)
//
// Roles (one CTA per SM, 6 warps):
//   warp 0      TMA producer: the q rows once, then per tile the attended blocks' K and V
//               (64-dim halves, 128-byte swizzle) into separate 2-deep K and V rings; block
//               ids for the next tile are fetched while the current one is issued.
//   warp 1      TMEM owner and MMA issuer (one lane), polling: score MMA of the next tile
//               whose K landed, value MMA of the tile whose probabilities are written.
//   warps 2..5  softmax, thread = query row = TMEM lane: scale, causal/window mask, online
//               softmax in base 2 with a lazily moved reference maximum (O in TMEM is
//               rescaled only when a row's maximum grows by more than 2^8), probabilities
//               to shared memory as the A operand, final O / l to the output.
// bf16 probabilities are split into hi + lo bf16 parts (two value MMAs) so the weights keep
// ~16 significant bits.  Every wait is bounded; one that gives up raises PA_DEVERR_TIMEOUT
// and an abort flag that ends the others.
#include <cfloat>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_host.h"
#include "pa_tmap.h"

namespace pa {

static __device__ unsigned int g_prefill_error;

__device__ __forceinline__ void prefill_error(unsigned int bits) { atomicOr(&g_prefill_error, bits); }

namespace {

constexpr int kRows = 128;                // query rows per CTA (MMA M)
constexpr int kKv = 128;                  // kv tokens per tile
constexpr int kDim = 128;                 // head_dim
constexpr int kHalf = 128 * 128;          // one 64-element half of a 128-row operand: 16 KiB
constexpr int kOpBytes = 2 * kHalf;       // a whole 128 x 128 operand (Q, K, V or P)
constexpr int kRing = 2;                  // depth of the K ring and of the V ring
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;       // S0 [0,128)  S1 [128,256)  O [256,384)
constexpr uint32_t kColO = 256;
constexpr float kRescaleThreshold = 8.f;  // log2 units: probabilities stay below 2^8

template <bool SPLIT>
constexpr size_t smem_bytes() {
  return 1024 + kOpBytes + 2 * kRing * kOpBytes + (SPLIT ? 2 : 1) * kOpBytes;
}

struct PrefillParams {
  void* out;
  const int32_t* block_tables;
  const int32_t* cu_q;
  const int32_t* context_lens;
  int S, T, Hq, Hkv, GQ, gq_shift, tq, bs, MB, NB, window, max_q_len;
  float qscale;  // scale * log2(e)
};

struct PfShared {
  uint64_t q_full;
  uint64_t k_full[kRing], k_empty[kRing], v_full[kRing], v_empty[kRing];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_full, mma_done;
  uint32_t tmem_base;
  int abort;
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

__device__ __forceinline__ uint32_t pack2(__half a, __half b) {
  return static_cast<uint32_t>(__half_as_ushort(a)) | (static_cast<uint32_t>(__half_as_ushort(b)) << 16);
}
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 a, __nv_bfloat16 b) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

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

template <typename IO>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ, const PrefillParams p) {
  constexpr bool kSplit = std::is_same<IO, __nv_bfloat16>::value;
  constexpr uint32_t kFmt = kSplit ? 1u : 0u;
  constexpr uint32_t kIdescS = mma_idesc_f16(kFmt, 0, 0, kRows, kKv);  // K-major Q and K
  constexpr uint32_t kIdescO = mma_idesc_f16(kFmt, 0, 1, kRows, kDim);  // K-major P, MN-major V

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ PfShared sh;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  grid_dependency_launch_next();
  grid_dependency_wait();

  // ---- this CTA's work: query tile qt (heaviest first) of sequence s, cached head kh ----
  const int s = blockIdx.z, kh = blockIdx.y;
  const int qt = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
  const int q_start = __ldg(p.cu_q + s);
  const int q_len = __ldg(p.cu_q + s + 1) - q_start;
  const int ctx = __ldg(p.context_lens + s);
  if (q_start < 0 || q_len < 0 || q_start + q_len > p.T || q_len > ctx || ctx > p.MB * p.bs || q_len > p.max_q_len) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) prefill_error(PA_DEVERR_CONTEXT);
    return;
  }
  const int i0 = qt * p.tq;
  if (i0 >= q_len) return;
  const int ntok = min(p.tq, q_len - i0);
  const int p_min = ctx - q_len + i0, p_max = p_min + ntok - 1;  // positions of the first / last query
  const int kv_lo = p.window > 0 ? max(0, p_min - p.window + 1) : 0;
  const int j_lo = kv_lo / kKv;
  const int n = p_max / kKv - j_lo + 1;  // KV tiles
  const int bs = p.bs;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;  // swizzle atoms are 1024-B aligned
  const uint32_t sQ = base;
  auto sK = [&](int st) { return base + kOpBytes + st * kOpBytes; };
  auto sV = [&](int st) { return base + (1 + kRing) * kOpBytes + st * kOpBytes; };
  const uint32_t sP = base + (1 + 2 * kRing) * kOpBytes;  // hi part; the lo part follows (bf16)
  const uint32_t q_full = smem_u32(&sh.q_full);
  const uint32_t k_full0 = smem_u32(&sh.k_full[0]), k_empty0 = smem_u32(&sh.k_empty[0]);
  const uint32_t v_full0 = smem_u32(&sh.v_full[0]), v_empty0 = smem_u32(&sh.v_empty[0]);
  const uint32_t s_full0 = smem_u32(&sh.s_full[0]), s_empty0 = smem_u32(&sh.s_empty[0]);
  const uint32_t p_full = smem_u32(&sh.p_full), o_full = smem_u32(&sh.o_full);
  const uint32_t mma_done = smem_u32(&sh.mma_done);
  volatile int* abort = &sh.abort;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int st = 0; st < kRing; ++st) {
      mbar_init(k_full0 + 8 * st, 1);
      mbar_init(k_empty0 + 8 * st, 1);
      mbar_init(v_full0 + 8 * st, 1);
      mbar_init(v_empty0 + 8 * st, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full0 + 8 * b, 1);
      mbar_init(s_empty0 + 8 * b, 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(mma_done, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(smem_u32(&sh.tmem_base), kTmemCols);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer --
    const uint64_t keep = l2_policy_evict_last();    // K/V tiles are shared by the sequence's q tiles
    const uint64_t once = l2_policy_evict_first();   // q rows are read once
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      prefetch_tensormap(&tmQ);
      mbar_arrive_expect_tx(q_full, kOpBytes);
      tma_load_3d(sQ, &tmQ, q_full, 0, kh * p.GQ, q_start + i0, once);
      tma_load_3d(sQ + kHalf, &tmQ, q_full, 64, kh * p.GQ, q_start + i0, once);
    }
    const int32_t* table = p.block_tables + static_cast<size_t>(s) * p.MB;
    TileBlocks tb = tile_blocks(j_lo, bs, kv_lo, p_max);
    int pb_next = lane <= tb.hi - tb.lo ? __ldg(table + tb.lo + lane) : 0;
    int k_issued = 0, v_issued = 0;
    for (int j = 0; j < n; ++j) {
      const TileBlocks cur = tb;
      int pb = pb_next;
      if (j + 1 < n) {  // next tile's block ids, in flight while this tile is issued
        tb = tile_blocks(j_lo + j + 1, bs, kv_lo, p_max);
        pb_next = lane <= tb.hi - tb.lo ? __ldg(table + tb.lo + lane) : 0;
      }
      const int nload = cur.hi - cur.lo + 1;
      if (lane < nload && (pb < 0 || pb >= p.NB)) {
        prefill_error(PA_DEVERR_TABLE);
        pb = 0;
      }
      const int st = j % kRing;
      const uint32_t bytes = static_cast<uint32_t>(nload) * 2u * bs * 128u;
      // K of tile j, then V of tile j; each copy is one 64-dim half of one block, one per lane.
      for (int which = 0; which < 2; ++which) {
        const uint32_t full = (which ? v_full0 : k_full0) + 8 * st;
        const uint32_t empty = (which ? v_empty0 : k_empty0) + 8 * st;
        bool ok = true;
        if (lane == 0) {
          if (j >= kRing) ok = wait_or_abort(empty, ((j / kRing) - 1) & 1, abort);
          if (ok) mbar_arrive_expect_tx(full, bytes);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const int cp = lane;  // 2 * nload <= 32 copies
        const int b = __shfl_sync(0xffffffffu, pb, (cp >> 1) & 31);
        if (cp < 2 * nload) {
          const uint32_t row = static_cast<uint32_t>(cur.lo + (cp >> 1) - cur.first) * bs * 128u;
          const uint32_t dst = (which ? sV(st) : sK(st)) + (cp & 1) * kHalf + row;
          tma_load_3d(dst, which ? &tmV : &tmK, full, (cp & 1) * 64, kh, b * bs, keep);
        }
        if (which) ++v_issued; else ++k_issued;
      }
      if (v_issued != j + 1) break;
    }
    if (lane == 0) {  // never leave with copies in flight
      mbar_wait_bounded(q_full, 0);
      for (int k = k_issued - kRing < 0 ? 0 : k_issued - kRing; k < k_issued; ++k)
        mbar_wait_bounded(k_full0 + 8 * (k % kRing), (k / kRing) & 1);
      for (int k = v_issued - kRing < 0 ? 0 : v_issued - kRing; k < v_issued; ++k)
        mbar_wait_bounded(v_full0 + 8 * (k % kRing), (k / kRing) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      int s_next = 0, o_next = 0;
      uint32_t idle = 0;
      bool ok = wait_or_abort(q_full, 0, abort);
      while (ok && o_next < n) {
        bool progressed = false;
        if (s_next < n) {
          const int st = s_next % kRing, b = s_next % 2;
          if (mbar_try_wait(k_full0 + 8 * st, (s_next / kRing) & 1) &&
              (s_next < 2 || mbar_try_wait(s_empty0 + 8 * b, ((s_next / 2) - 1) & 1))) {
            tc_fence_after_sync();
#pragma unroll
            for (int kk = 0; kk < kDim / 16; ++kk) {  // S[b] = Q . K^T, 16 dims per MMA
              const uint32_t off = (kk / 4) * kHalf + (kk % 4) * 32;
              tc_mma_f16(tmem + b * kKv, smem_desc(sQ + off, 16, 1024, kSwizzle128B),
                         smem_desc(sK(st) + off, 16, 1024, kSwizzle128B), kIdescS, kk > 0);
            }
            tc_commit(s_full0 + 8 * b);
            tc_commit(k_empty0 + 8 * st);
            ++s_next;
            progressed = true;
          }
        }
        if (o_next < s_next) {
          const int st = o_next % kRing;
          if (mbar_try_wait(p_full, o_next & 1) && mbar_try_wait(v_full0 + 8 * st, (o_next / kRing) & 1)) {
            tc_fence_after_sync();
#pragma unroll
            for (int part = 0; part < (kSplit ? 2 : 1); ++part) {
#pragma unroll
              for (int kk = 0; kk < kKv / 16; ++kk) {  // O += P . V, 16 kv tokens per MMA
                tc_mma_f16(tmem + kColO,
                           smem_desc(sP + part * kOpBytes + (kk / 4) * kHalf + (kk % 4) * 32, 16, 1024, kSwizzle128B),
                           smem_desc(sV(st) + kk * 2048, kHalf, 1024, kSwizzle128B), kIdescO,
                           o_next > 0 || part > 0 || kk > 0);
              }
            }
            tc_commit(o_full);
            tc_commit(v_empty0 + 8 * st);
            ++o_next;
            progressed = true;
          }
        }
        if (progressed) {
          idle = 0;
        } else if (*abort || ++idle > 4 * kWaitLimit) {
          if (!*abort) prefill_error(PA_DEVERR_TIMEOUT);
          *abort = 1;
          break;
        }
      }
      tc_commit(mma_done);  // every MMA issued above has finished before TMEM is released
      mbar_wait_bounded(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- softmax warps --
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // query row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q4) << 16;
    const int tl = r >> p.gq_shift, g = r & (p.GQ - 1);
    const bool row_valid = tl < ntok;
    const int pos = p_min + tl;
    const int lo_row = p.window > 0 ? max(0, pos - p.window + 1) : 0;
    float m_run = -FLT_MAX, l = 0.f;
    bool done = false;
    for (int j = 0; j < n; ++j) {
      const int b = j % 2, st = j % kRing;
      if (!__all_sync(0xffffffffu, wait_or_abort(s_full0 + 8 * b, (j / 2) & 1, abort))) break;
      tc_fence_after_sync();
      float sc[kKv];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_load32(tmem + lane_addr + b * kKv + 32 * c4, sc + 32 * c4);
      tc_fence_before_sync();
      mbar_arrive(s_empty0 + 8 * b);

      const int kv0 = (j_lo + j) * kKv;
      const int c_lo = lo_row - kv0, c_hi = row_valid ? pos - kv0 : -1;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kKv; ++c) {
        sc[c] = (c >= c_lo && c <= c_hi) ? sc[c] * p.qscale : -INFINITY;
        mt = fmaxf(mt, sc[c]);
      }
      float alpha = 1.f;
      bool rescale = false;
      if (mt > m_run + kRescaleThreshold) {  // move the reference maximum
        alpha = exp2f(m_run - mt);
        rescale = l > 0.f;                   // O holds earlier contributions of this row
        l *= alpha;
        m_run = mt;
      }
      // The previous value MMA must be done before P is overwritten or O rescaled.
      if (j > 0 && !__all_sync(0xffffffffu, wait_or_abort(o_full, (j - 1) & 1, abort))) break;
      if (__any_sync(0xffffffffu, rescale)) {
        tc_fence_after_sync();
        const float a = rescale ? alpha : 1.f;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float o[32];
          tmem_load32(tmem + lane_addr + kColO + 32 * c4, o);
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] *= a;
          tmem_store32(tmem + lane_addr + kColO + 32 * c4, o);
        }
      }
      // V rows of tokens outside the loaded blocks or past the context may hold anything
      // (NaN); their weights are 0, so give the value MMA zeros there (thread r: kv row r).
      const TileBlocks tb = tile_blocks(j_lo + j, bs, kv_lo, p_max);
      const int clean_lo = tb.lo * bs - kv0, clean_hi = min(ctx, (tb.hi + 1) * bs) - kv0;
      if (clean_lo > 0 || clean_hi < kKv) {
        if (!__all_sync(0xffffffffu, wait_or_abort(v_full0 + 8 * st, (j / kRing) & 1, abort))) break;
        if (r < clean_lo || r >= clean_hi) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            st_shared_v4(sV(st) + r * 128 + 16 * k, 0, 0, 0, 0);
            st_shared_v4(sV(st) + kHalf + r * 128 + 16 * k, 0, 0, 0, 0);
          }
        }
      }
      // Probabilities, written as row r of the K-major, 128-byte-swizzled A operand.
      float ls = 0.f;
      const uint32_t prow = (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w_hi[4], w_lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = exp2f(sc[64 * h + 8 * c + 2 * e] - m_run);
            const float x1 = exp2f(sc[64 * h + 8 * c + 2 * e + 1] - m_run);
            const IO h0 = float_to<IO>(x0), h1 = float_to<IO>(x1);
            w_hi[e] = pack2(h0, h1);
            if (kSplit) {
              w_lo[e] = pack2(float_to<IO>(x0 - static_cast<float>(h0)), float_to<IO>(x1 - static_cast<float>(h1)));
              ls += x0 + x1;
            } else {
              ls += static_cast<float>(h0) + static_cast<float>(h1);  // the rounded weights the MMA uses
            }
          }
          const uint32_t addr = sP + h * kHalf + prow + ((c ^ (r & 7)) << 4);
          st_shared_v4(addr, w_hi[0], w_hi[1], w_hi[2], w_hi[3]);
          if (kSplit) st_shared_v4(addr + kOpBytes, w_lo[0], w_lo[1], w_lo[2], w_lo[3]);
        }
      }
      l += ls;
      fence_proxy_async_shared();
      tc_fence_before_sync();
      mbar_arrive(p_full);
      if (j == n - 1) done = true;
    }
    if (done && __all_sync(0xffffffffu, wait_or_abort(o_full, (n - 1) & 1, abort))) {
      tc_fence_after_sync();
      const float inv = row_valid ? 1.f / l : 0.f;
      IO* orow = reinterpret_cast<IO*>(p.out) +
                 (static_cast<size_t>(q_start + i0 + tl) * p.Hq + static_cast<size_t>(kh) * p.GQ + g) * kDim;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        float o[32];
        tmem_load32(tmem + lane_addr + kColO + 32 * c4, o);
        if (row_valid) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = pack2(float_to<IO>(o[8 * v + 2 * e] * inv), float_to<IO>(o[8 * v + 2 * e + 1] * inv));
            *reinterpret_cast<uint4*>(orow + 32 * c4 + 8 * v) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
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

extern "C" pa_status paged_attention_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                                             const int32_t* block_tables, const int32_t* cu_q_lens,
                                             const int32_t* context_lens, int num_seqs, int num_q_tokens,
                                             int max_q_len, int num_q_heads, int num_kv_heads, int head_dim,
                                             int block_size, int num_blocks, int max_blocks_per_seq, float scale,
                                             int window, pa_dtype dtype, void* stream) {
  if (num_seqs < 0 || num_q_tokens < 0 || max_q_len < 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: negative size");
  if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: num_q_heads must be a positive multiple of num_kv_heads");
  if (block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: block_size, num_blocks and max_blocks_per_seq must be > 0");
  if (dtype != PA_F16 && dtype != PA_BF16)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: dtype must be PA_F16 or PA_BF16");
  if (head_dim != kDim) return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: head_dim must be 128");
  const int GQ = num_q_heads / num_kv_heads;
  if (GQ > 16 || (GQ & (GQ - 1)) != 0)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: query heads per cached head must be 1, 2, 4, 8 or 16");
  if (block_size % 8 != 0 || kKv % block_size != 0)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: block_size must be 8, 16, 32, 64 or 128");
  if (num_seqs == 0 || num_q_tokens == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !cu_q_lens || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: NULL pointer");
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "paged_attention_prefill: out, q and the caches must be 16-byte aligned");
  if (num_seqs > 65535 || num_kv_heads > 65535)
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: at most 65535 sequences and cached heads");
  if (static_cast<long long>(max_blocks_per_seq) * block_size > (1LL << 30))
    return fail(PA_ERR_UNSUPPORTED, "paged_attention_prefill: max_blocks_per_seq * block_size too large");

  EncodeTiledFn enc = nullptr;
  pa_status st = get_encoder(&enc);
  if (st != PA_OK) return st;
  const CUtensorMapDataType ttype = dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int tq = kRows / GQ;
  CUtensorMap tmK, tmV, tmQ;
  {
    // [NB*bs rows][Hkv][128]: boxes of one block's rows x one head x 64 dims, 128-byte swizzle
    const cuuint64_t dims[3] = {kDim, static_cast<cuuint64_t>(num_kv_heads),
                                static_cast<cuuint64_t>(num_blocks) * block_size};
    const cuuint64_t strides[2] = {kDim * 2, static_cast<cuuint64_t>(num_kv_heads) * kDim * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(block_size)};
    if ((st = encode(enc, &tmK, ttype, 3, k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
    if ((st = encode(enc, &tmV, ttype, 3, v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
  }
  {
    // q as [T][Hq][128]: tq tokens x the GQ heads of one cached head x 64 dims
    const cuuint64_t dims[3] = {kDim, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(num_q_tokens)};
    const cuuint64_t strides[2] = {kDim * 2, static_cast<cuuint64_t>(num_q_heads) * kDim * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(GQ), static_cast<cuuint32_t>(tq)};
    if ((st = encode(enc, &tmQ, ttype, 3, q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) != PA_OK) return st;
  }
  PrefillParams prm = {};
  prm.out = out;
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
  prm.qscale = scale * 1.4426950408889634f;

  const bool bf16 = dtype == PA_BF16;
  const void* fn = bf16 ? reinterpret_cast<const void*>(&prefill_tc_kernel<__nv_bfloat16>)
                        : reinterpret_cast<const void*>(&prefill_tc_kernel<__half>);
  const size_t smem = bf16 ? smem_bytes<true>() : smem_bytes<false>();
  static std::once_flag once[2];
  cudaError_t attr_err = cudaSuccess;
  std::call_once(once[bf16 ? 1 : 0], [&] {
    attr_err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  });
  if (attr_err != cudaSuccess) return cuda_fail(attr_err, "cudaFuncSetAttribute(prefill)");
  const dim3 grid(static_cast<unsigned>((max_q_len + tq - 1) / tq), static_cast<unsigned>(num_kv_heads),
                  static_cast<unsigned>(num_seqs));
  void* args[] = {&tmK, &tmV, &tmQ, &prm};
  cudaError_t err = launch_dependent(fn, grid, dim3(kThreads), smem, static_cast<cudaStream_t>(stream), args);
  if (err != cudaSuccess) return cuda_fail(err, "launching the prefill kernel");
  return PA_OK;
}
