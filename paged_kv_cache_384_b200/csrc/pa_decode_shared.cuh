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
  int seg_units;         // cost of a segment's end, in tiles: the stream is split into equal
                         // shares of (tiles + seg_units per segment) among the CTAs
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


// Device-side plan shared by the partition kernels.  The (sequence, head group, tile) stream
// is split into equal shares of cost units: each tile is one unit and each segment (one
// head group of one sequence) adds p.seg_units more before its first tile (the work at a
// segment's end, which made CTAs with many short segments finish last).  Tile j of segment
// (s, g) sits at unit G * U(s) + g * (nb + w) + w + j, where U(s) counts the units of the
// sequences before s for one head group and w = p.seg_units; CTA c takes the tiles whose
// units fall in its share.  Every thread of the CTA must call plan_slice: it counts every
// sequence's tiles, prefix-sums the units over the CTA (CTA 0 also publishes U for the
// merge kernel) and locates this CTA's first and one-past-last tile.  Returns the number of
// tiles (0: nothing to do, or an impossible plan reported as PA_DEVERR_TIMEOUT); *start is
// the cursor of the first.
struct PlanScratch {
  long long warp_sum[kMaxPlanThreads / 32][2];  // units and tiles of each warp, then their exclusive prefixes
  long long total_units, total_tiles;
  long long tile_at[2];                         // stream index of the first tile at or after u0, u1
  int first_seq, first_g, first_j;
};

// Units of one head group's segment of a sequence with nb tiles.
__device__ __forceinline__ long long seg_units_of(int nb, int w) { return nb > 0 ? nb + w : 0; }

// Units -> CTA (the inverse of the equal split of the units).
__device__ __forceinline__ int cta_of_unit(long long u, long long U, int C) { return cta_of(u, U, C); }

__device__ __forceinline__ long long plan_slice(const DecodeParams& p, PlanScratch& sc, long long* t0_out,
                                                Cursor* start) {
  const int nthr = blockDim.x;  // a multiple of 32
  const int G = p.G, w = p.seg_units;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nwarps = (nthr + 31) >> 5;
  const int chunk = (p.S + nthr - 1) / nthr;
  const int s_lo = min(p.S, static_cast<int>(threadIdx.x) * chunk), s_hi = min(p.S, s_lo + chunk);
  long long mine_t = 0, mine_u = 0;
  for (int s = s_lo; s < s_hi; ++s) {
    const int nb = seq_span(p, s, blockIdx.x == 0).nb;
    mine_t += nb;
    mine_u += seg_units_of(nb, w);
  }
  // Exclusive prefixes over the threads: shuffle scans inside each warp, then over the warps'
  // totals (a thread-serial scan measured ~6 us at 448 threads).
  long long inc_t = mine_t, inc_u = mine_u;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const long long yt = __shfl_up_sync(0xffffffffu, inc_t, off);
    const long long yu = __shfl_up_sync(0xffffffffu, inc_u, off);
    if (lane >= off) inc_t += yt, inc_u += yu;
  }
  if (lane == 31) sc.warp_sum[wid][0] = inc_u, sc.warp_sum[wid][1] = inc_t;
  if (threadIdx.x == 0) sc.first_seq = -1;
  __syncthreads();
  if (wid == 0) {
    const long long vu = lane < nwarps ? sc.warp_sum[lane][0] : 0, vt = lane < nwarps ? sc.warp_sum[lane][1] : 0;
    long long au = vu, at = vt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const long long yu = __shfl_up_sync(0xffffffffu, au, off);
      const long long yt = __shfl_up_sync(0xffffffffu, at, off);
      if (lane >= off) au += yu, at += yt;
    }
    if (lane < nwarps) sc.warp_sum[lane][0] = au - vu, sc.warp_sum[lane][1] = at - vt;
    if (lane == 31) sc.total_units = au, sc.total_tiles = at;
  }
  __syncthreads();
  const long long per_group = sc.total_units;  // units of one head group over all sequences
  const long long U = per_group * G, T = sc.total_tiles * G;
  const long long pre_u = sc.warp_sum[wid][0] + inc_u - mine_u, pre_t = sc.warp_sum[wid][1] + inc_t - mine_t;
  if (blockIdx.x == 0) {  // publish the per-sequence unit prefix for the merge kernel
    long long r = pre_u;
    for (int s = s_lo; s < s_hi; ++s) {
      p.ws_prefix[s] = r;
      r += seg_units_of(seq_span(p, s, false).nb, w);
    }
    if (threadIdx.x == 0) p.ws_prefix[p.S] = per_group;
  }
  long long u0, ucount;
  cta_slice(U, p.num_ctas, blockIdx.x, &u0, &ucount);
  if (ucount == 0) return 0;  // uniform across the CTA
  // The first tile at or after unit u0 and after u0 + ucount: located by the thread whose
  // sequences hold that unit (an end at U has no owner: T).
  if (threadIdx.x == 0 && u0 + ucount >= U) sc.tile_at[1] = T;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const long long u = e == 0 ? u0 : u0 + ucount;
    if (u < U && u >= G * pre_u && u < G * (pre_u + mine_u)) {
      long long ru = pre_u, rt = pre_t;
      for (int s = s_lo; s < s_hi; ++s) {
        const int nb = seq_span(p, s, false).nb;
        const long long su = seg_units_of(nb, w);
        if (u < G * (ru + su)) {
          const long long rem = u - G * ru;
          const int g = static_cast<int>(rem / su);
          const int j = static_cast<int>(max(0ll, rem % su - w));
          sc.tile_at[e] = G * rt + static_cast<long long>(g) * nb + j;
          if (e == 0) {
            sc.first_seq = s;
            sc.first_g = g;
            sc.first_j = j;
          }
          break;
        }
        ru += su;
        rt += nb;
      }
    }
  }
  __syncthreads();
  if (sc.first_seq < 0) {  // cannot happen when ucount > 0; never index with it
    if (threadIdx.x == 0) decode_error(PA_DEVERR_TIMEOUT);
    return 0;
  }
  const long long count = sc.tile_at[1] - sc.tile_at[0];
  if (count <= 0) return 0;  // a share of segment-end units only
  start->s = sc.first_seq;
  start->sp = seq_span(p, start->s, false);
  start->g = sc.first_g;
  start->j = sc.first_j;
  *t0_out = sc.tile_at[0];
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
// CTAs per SM of the 8-bit kernel for a head group of `group` query heads (1 or 2).
int tc8_ctas_per_sm(int group);
}  // namespace pa
