// pa_decode_shared.cuh -- pieces shared by the decode partition kernels (CUDA-core and
// tensor-core): parameters, the (sequence, head group, tile) work stream and its device-side
// plan, and the error word.  Internal header.
#pragma once

#include "pa_device.cuh"

namespace pa {

static __device__ unsigned int g_decode_error;

__device__ __forceinline__ void decode_error(unsigned int bits) { atomicOr(&g_decode_error, bits); }

constexpr int kMaxCtasPerSm = 4;    // persistent-grid CTAs per SM (upper bound)
constexpr int kMaxHeadGroup = 8;    // heads per CTA (upper bound)
constexpr int kMaxThreads = 32 * (kMaxHeadGroup + 1);  // CUDA-core kernel: TMA warp + head warps
// Threads per CTA of any kernel that plans with plan_slice (the tensor-core kernels have up to 448);
// PlanScratch holds one entry each.
constexpr int kMaxPlanThreads = 448;
static_assert(kMaxPlanThreads >= kMaxThreads, "plan scratch must cover the CUDA-core kernel");
constexpr int kBarrierBytes = 128;  // mbarriers at the front of dynamic smem (<= 8 stages)

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  long long* ws_prefix;  // [S + 1] per-sequence tile prefix (written by CTA 0)
  float* ws_ml;          // [nslot][QW][2] partial (max, sum) per query head of the tile
  float* ws_acc;         // [nslot][QW][D] partial accumulators
  int S, H, bs, MB, NB, window;
  int tt, tpb;           // rows per tile (a divisor of bs) and tiles per physical block
  int HG, G, num_ctas, nstage;   // cached heads per tile, head groups, grid size, ring depth
  int Hq, GQ, QW;        // query heads, query heads per cached head (per sub-group), query heads per tile
  int sub;               // tensor-core kernel: head groups per cached head (1, or query sub-groups of
                         // one cached head when it has more than 16 query heads)
  int dim;               // head_dim (the tensor-core kernel takes 64 or 128 at run time)
  float qscale;          // softmax scale * log2(e): scores are kept in base 2
  uint32_t stage_bytes;  // bytes per pipeline stage
  uint32_t v_off, ks_off, vs_off;  // offsets of the V tile and the INT8 scale tiles in a stage
  uint32_t tx_bytes;     // TMA transaction bytes per stage
};

// Attended span of one sequence: tokens [lo, ctx), tiles first_t .. first_t + nb - 1.  Tile ti
// holds the tt rows of logical block ti / tpb starting at row (ti % tpb) * tt.
struct Span {
  int ctx, lo, first_t, nb;
};

__device__ __forceinline__ Span seq_span(const DecodeParams& p, int s, bool report) {
  int ctx = __ldg(p.context_lens + s);
  const int cap = p.MB * p.bs;
  if (ctx < 0 || ctx > cap) {
    if (report) decode_error(PA_DEVERR_CONTEXT);
    ctx = ctx < 0 ? 0 : cap;
  }
  Span r;
  r.ctx = ctx;
  r.lo = (p.window > 0 && ctx > p.window) ? ctx - p.window : 0;
  r.first_t = r.lo / p.tt;
  r.nb = ctx > 0 ? (ctx - 1) / p.tt - r.first_t + 1 : 0;
  return r;
}

// Position in the tile stream: sequence s, head group g, tile j of the segment.
struct Cursor {
  int s, g, j;
  Span sp;
};

__device__ __forceinline__ void advance(Cursor& c, const DecodeParams& p) {
  if (++c.j < c.sp.nb) return;
  c.j = 0;
  if (++c.g < p.G) return;
  c.g = 0;
  for (++c.s; c.s < p.S; ++c.s) {
    c.sp = seq_span(p, c.s, false);
    if (c.sp.nb > 0) return;
  }
}

// Slice [t0, t0 + count) of the T-tile stream owned by CTA c of C (equal split, the
// first T % C CTAs take one extra tile).
__device__ __forceinline__ void cta_slice(long long T, int C, int c, long long* t0, long long* count) {
  const long long base = T / C, rem = T % C;
  *t0 = c * base + (c < rem ? c : rem);
  *count = base + (c < rem ? 1 : 0);
}

// CTA owning tile t (inverse of cta_slice).
__device__ __forceinline__ int cta_of(long long t, long long T, int C) {
  const long long base = T / C, rem = T % C;
  const long long big = rem * (base + 1);
  return static_cast<int>(t < big ? t / (base + 1) : rem + (t - big) / base);
}

// Load n consecutive elements of type IO as floats (n * sizeof(IO) is a multiple of 16).
template <typename IO, int N>
__device__ __forceinline__ void load_floats(const IO* src, float* dst) {
  constexpr int EVIO = Elem<IO>::kEV;
  static_assert(N % EVIO == 0, "vector multiple");
#pragma unroll
  for (int i = 0; i < N / EVIO; ++i) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
    Elem<IO>::to_float(v, dst + i * EVIO);
  }
}

template <typename IO, int N>
__device__ __forceinline__ void store_floats(IO* dst, const float* src) {
  static_assert((N * sizeof(IO)) % 16 == 0, "vector multiple");
  IO tmp[N];
#pragma unroll
  for (int i = 0; i < N; ++i) tmp[i] = float_to<IO>(src[i]);
#pragma unroll
  for (int i = 0; i < static_cast<int>(N * sizeof(IO) / 16); ++i)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(tmp)[i];
}


// Device-side plan shared by the partition kernels: count every sequence's tiles, prefix-sum
// them over the CTA (CTA 0 also publishes the prefix for the merge kernel), and locate this
// CTA's slice [t0, t0 + count) of the (sequence, head group, tile) stream.  Every thread of
// the CTA must call it.  Returns count (0: nothing to do, or an impossible plan reported as
// PA_DEVERR_TIMEOUT); *start is the cursor of tile t0.
struct PlanScratch {
  long long warp_sum[kMaxPlanThreads / 32];  // tiles counted by each warp, then their exclusive prefix
  long long total;
  long long first_prefix;
  int first_seq;
};

__device__ __forceinline__ long long plan_slice(const DecodeParams& p, PlanScratch& sc, long long* t0_out,
                                                Cursor* start) {
  const int nthr = blockDim.x;
  const int G = p.G;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nwarps = (nthr + 31) >> 5;
  const int chunk = (p.S + nthr - 1) / nthr;
  const int s_lo = min(p.S, static_cast<int>(threadIdx.x) * chunk), s_hi = min(p.S, s_lo + chunk);
  long long mine = 0;
  for (int s = s_lo; s < s_hi; ++s) mine += seq_span(p, s, blockIdx.x == 0).nb;
  // Exclusive prefix over the threads: a shuffle scan inside each warp, then over the warps'
  // totals (a thread-serial scan measured ~6 us at 448 threads).
  long long incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) sc.warp_sum[wid] = incl;
  if (threadIdx.x == 0) sc.first_seq = -1;
  __syncthreads();
  if (wid == 0) {
    const long long v = lane < nwarps ? sc.warp_sum[lane] : 0;
    long long w = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < nwarps) sc.warp_sum[lane] = w - v;
    if (lane == 31) sc.total = w;
  }
  __syncthreads();
  const long long per_group = sc.total;  // tiles of one head group over all sequences
  const long long T = per_group * G;
  const long long my_prefix = sc.warp_sum[wid] + incl - mine;
  if (blockIdx.x == 0) {  // publish the per-sequence prefix for the merge kernel
    long long r = my_prefix;
    for (int s = s_lo; s < s_hi; ++s) {
      p.ws_prefix[s] = r;
      r += seq_span(p, s, false).nb;
    }
    if (threadIdx.x == 0) p.ws_prefix[p.S] = per_group;
  }
  long long t0, count;
  cta_slice(T, p.num_ctas, blockIdx.x, &t0, &count);
  if (count == 0) return 0;  // uniform across the CTA
  // Sequence holding t0: sequence s starts at tile G * prefix(s).
  if (t0 >= G * my_prefix && t0 < G * (my_prefix + mine)) {
    long long r = my_prefix;
    for (int s = s_lo; s < s_hi; ++s) {
      const int nb = seq_span(p, s, false).nb;
      if (t0 < G * (r + nb)) {
        sc.first_seq = s;
        sc.first_prefix = r;
        break;
      }
      r += nb;
    }
  }
  __syncthreads();
  if (sc.first_seq < 0) {  // cannot happen when count > 0; never index with it
    if (threadIdx.x == 0) decode_error(PA_DEVERR_TIMEOUT);
    return 0;
  }
  start->s = sc.first_seq;
  start->sp = seq_span(p, start->s, false);
  const long long rem = t0 - G * sc.first_prefix;
  start->g = static_cast<int>(rem / start->sp.nb);
  start->j = static_cast<int>(rem % start->sp.nb);
  *t0_out = t0;
  return count;
}

}  // namespace pa

namespace pa {
// Tensor-core grouped-query decode (pa_decode_tc.cu).
bool tc_decode_eligible(pa_dtype io, pa_dtype cache, int head_dim, int block_size, int group);
// Query heads per head group of the tensor-core kernel: the group itself up to 16, else the
// largest divisor of it in [4, 16] (0: none).
int tc_decode_subgroup(int group);
int tc_decode_tile_tokens();
// tmKs / tmVs: fp16 scale maps of an 8-bit cache (ignored when cache == io).
pa_status tc_decode_launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                           const CUtensorMap& tmKs, const CUtensorMap& tmVs, const DecodeParams& prm, pa_dtype io,
                           pa_dtype cache, int grid, cudaStream_t stream);
// 8-bit caches (pa_decode_tc8.cu): tmK / tmV map the codes, tmKs / tmVs the fp16 scales.
pa_status tc8_decode_launch(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmKs,
                            const CUtensorMap& tmVs, const DecodeParams& prm, pa_dtype io, pa_dtype cache, int grid,
                            cudaStream_t stream);
}  // namespace pa
