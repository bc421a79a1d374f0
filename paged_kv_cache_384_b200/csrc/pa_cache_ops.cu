// pa_cache_ops.cu -- reshape_and_cache, copy_blocks and swap_blocks for sm_100a.
//
// Both are pure data movement and HBM-bound.  Each thread moves 16-byte vectors; a CTA
// covers a contiguous byte range so every warp issues fully coalesced 512-byte
// transactions.  Slot and pair indices are bounds-checked on the device: an index outside
// the pool skips the copy and sets a bit in the device error word instead of faulting.
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

static __device__ unsigned int g_cache_error;

__device__ __forceinline__ void cache_error(unsigned int bits) { atomicOr(&g_cache_error, bits); }

// ---------------------------------------------------------------------------------------
// reshape_and_cache: token t's row of H*D elements (row_bytes) goes to slot slot_mapping[t]
// ("vLLM source first look: PagedAttention memory design" (trdm.cn), section 一: the cache
// gains one row per generated token).  Grid: (vector chunks of a row, tokens).
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
reshape_and_cache_kernel(const uint8_t* __restrict__ k, const uint8_t* __restrict__ v, uint8_t* __restrict__ kc,
                         uint8_t* __restrict__ vc, const int64_t* __restrict__ slots, long long row_bytes,
                         long long k_stride_bytes, long long v_stride_bytes, long long num_slots,
                         const uint16_t* __restrict__ ks_src, const uint16_t* __restrict__ vs_src,
                         uint16_t* __restrict__ ks_cache, uint16_t* __restrict__ vs_cache, int H) {
  grid_dependency_launch_next();
  grid_dependency_wait();  // launched as a programmatic dependent: inputs may come from the previous kernel
  const int t = blockIdx.y;
  const long long slot = __ldg(slots + t);
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (threadIdx.x == 0 && blockIdx.x == 0) cache_error(PA_DEVERR_SLOT);
    return;
  }
  const long long nvec = row_bytes / 16;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < nvec) {
    const uint4 kv = __ldg(reinterpret_cast<const uint4*>(k + t * k_stride_bytes) + i);
    const uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + t * v_stride_bytes) + i);
    reinterpret_cast<uint4*>(kc + slot * row_bytes)[i] = kv;
    reinterpret_cast<uint4*>(vc + slot * row_bytes)[i] = vv;
  }
  if (ks_src && blockIdx.x == 0) {
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      ks_cache[slot * H + h] = ks_src[static_cast<long long>(t) * H + h];
      vs_cache[slot * H + h] = vs_src[static_cast<long long>(t) * H + h];
    }
  }
}

// ---------------------------------------------------------------------------------------
// Whole-block copies, dst pool block d <- src pool block s for each (s, d) pair.
//  * copy_blocks: source and destination are the same GPU pool ("vLLM source first look:
//    PagedAttention memory design" (trdm.cn), section 二, BlockManager.copy_on_write).
//  * swap_blocks: one pool is page-locked host memory mapped into the device address
//    space ("KV Cache memory optimisation and PagedAttention" (yunthe.com), section
//    "vLLM调度器与PagedAttention协同工作", item 3: preempted requests' blocks move to CPU
//    memory and back).  The threads read or write the host pool directly; the many
//    16-byte requests in flight across the grid keep the host link busy.
// Grid: (chunks of a block, pairs, 2 or 4 pools).  VEC = 16 moves uint4; VEC = 1 moves bytes.
// ---------------------------------------------------------------------------------------
struct BlockPools {
  const uint8_t* src[4];  // K, V, K scales, V scales
  uint8_t* dst[4];
};

template <int VEC>
__global__ void __launch_bounds__(256)
block_copy_kernel(BlockPools pools, const int64_t* pairs, long long block_bytes, long long scale_block_bytes,
                  long long num_src, long long num_dst) {
  grid_dependency_launch_next();
  grid_dependency_wait();
  const int pool = blockIdx.z;
  const long long src = pairs[2 * blockIdx.y], dst = pairs[2 * blockIdx.y + 1];
  if (src < 0 || src >= num_src || dst < 0 || dst >= num_dst) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && pool == 0) cache_error(PA_DEVERR_PAIR);
    return;
  }
  const long long bytes = pool < 2 ? block_bytes : scale_block_bytes;
  const uint8_t* from = pools.src[pool] + src * bytes;
  uint8_t* to = pools.dst[pool] + dst * bytes;
  if (VEC == 16 && pool < 2) {
    constexpr int kPerThread = 4;  // 4 independent 16-byte loads in flight per thread
    const long long nvec = bytes / 16;
    const long long first = (static_cast<long long>(blockIdx.x) * blockDim.x * kPerThread) + threadIdx.x;
    uint4 tmp[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const long long i = first + static_cast<long long>(u) * blockDim.x;
      if (i < nvec) tmp[u] = reinterpret_cast<const uint4*>(from)[i];
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const long long i = first + static_cast<long long>(u) * blockDim.x;
      if (i < nvec) reinterpret_cast<uint4*>(to)[i] = tmp[u];
    }
  } else {
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < bytes; i += stride)
      to[i] = from[i];
  }
}

namespace {

cudaError_t read_cache_error(uint32_t* flags, int clear) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_cache_error, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (clear && v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_cache_error, &z, sizeof z);
  }
  return e;
}

struct RegisterCache {
  RegisterCache() { register_device_error_reader(read_cache_error); }
} g_register_cache;

size_t elem_size(pa_dtype t) { return t == PA_F32 ? 4 : ((t == PA_I8 || t == PA_FP8_E4M3) ? 1 : 2); }

}  // namespace
}  // namespace pa

namespace pa {
namespace {

cudaError_t launch_block_copy(const BlockPools& pools, const int64_t* pairs, int num_pairs, size_t block_bytes,
                              size_t scale_block_bytes, long long num_src, long long num_dst, bool scales,
                              cudaStream_t s) {
  const bool vec_ok = block_bytes % 16 == 0 && aligned16(pools.src[0]) && aligned16(pools.src[1]) &&
                      aligned16(pools.dst[0]) && aligned16(pools.dst[1]);
  const int threads = 256;
  const long long per_cta = vec_ok ? 16LL * threads * 4 : threads * 64LL;
  const long long longest = static_cast<long long>(block_bytes > scale_block_bytes ? block_bytes : scale_block_bytes);
  dim3 grid(static_cast<unsigned>((longest + per_cta - 1) / per_cta), static_cast<unsigned>(num_pairs), scales ? 4u : 2u);
  BlockPools p = pools;
  long long bb = static_cast<long long>(block_bytes), sb = static_cast<long long>(scale_block_bytes);
  void* args[] = {&p, &pairs, &bb, &sb, &num_src, &num_dst};
  const void* fn = vec_ok ? reinterpret_cast<const void*>(&block_copy_kernel<16>)
                          : reinterpret_cast<const void*>(&block_copy_kernel<1>);
  return launch_dependent(fn, grid, dim3(threads), 0, s, args);
}

// The address under which the device reaches `p`: device memory as it is, page-locked host
// memory through its mapping.  Pageable host memory has no such address.
pa_status device_view(const void* p, const char* what, const void** out) {
  cudaPointerAttributes a;
  const cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return cuda_fail(e, what);
  }
  if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
    *out = p;
    return PA_OK;
  }
  if (a.type == cudaMemoryTypeHost && a.devicePointer) {
    *out = a.devicePointer;
    return PA_OK;
  }
  return fail(PA_ERR_INVALID_ARG, "swap_blocks: %s is pageable (or unmapped) host memory; use page-locked, mapped memory",
              what);
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" pa_status reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                                       const int64_t* slot_mapping, int num_tokens, int num_heads, int head_dim,
                                       int block_size, int num_blocks, int64_t k_token_stride, int64_t v_token_stride,
                                       pa_dtype dtype, const void* k_scale_src, const void* v_scale_src,
                                       void* k_scale_cache, void* v_scale_cache, void* stream) {
  if (num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: sizes must be positive (num_tokens >= 0)");
  if (dtype != PA_F32 && dtype != PA_F16 && dtype != PA_BF16 && dtype != PA_I8 && dtype != PA_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: unknown dtype %d", static_cast<int>(dtype));
  const long long row_elems = static_cast<long long>(num_heads) * head_dim;
  const size_t e = elem_size(dtype);
  const long long row_bytes = row_elems * static_cast<long long>(e);
  if (row_bytes % 16) return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: a token row (%lld bytes) must be a multiple of 16 bytes", row_bytes);
  if (k_token_stride < row_elems || v_token_stride < row_elems)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: token strides must be >= num_heads*head_dim");
  if ((k_token_stride * static_cast<long long>(e)) % 16 || (v_token_stride * static_cast<long long>(e)) % 16)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: token strides must be multiples of 16 bytes");
  const bool int8 = dtype == PA_I8 || dtype == PA_FP8_E4M3;  // 8-bit codes travel with their scales
  if (int8 != (k_scale_src && v_scale_src && k_scale_cache && v_scale_cache) ||
      (!int8 && (k_scale_src || v_scale_src || k_scale_cache || v_scale_cache)))
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: the four scale pointers are required for PA_I8 / PA_FP8_E4M3 and must be NULL otherwise");
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: NULL pointer");
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      reinterpret_cast<uintptr_t>(slot_mapping) % 8)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: k, v and caches must be 16-byte aligned, slot_mapping 8-byte aligned");
  if (int8 && ((reinterpret_cast<uintptr_t>(k_scale_src) | reinterpret_cast<uintptr_t>(v_scale_src) |
                reinterpret_cast<uintptr_t>(k_scale_cache) | reinterpret_cast<uintptr_t>(v_scale_cache)) & 1))
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache: scale pointers must be 2-byte aligned");
  if (num_tokens > 65535) return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache: at most 65535 tokens per call");

  const long long nvec = row_bytes / 16;
  const int threads = 256;
  dim3 grid(static_cast<unsigned>((nvec + threads - 1) / threads), static_cast<unsigned>(num_tokens));
  const uint8_t* kp = static_cast<const uint8_t*>(k);
  const uint8_t* vp = static_cast<const uint8_t*>(v);
  uint8_t* kcp = static_cast<uint8_t*>(k_cache);
  uint8_t* vcp = static_cast<uint8_t*>(v_cache);
  long long kst = k_token_stride * static_cast<long long>(e), vst = v_token_stride * static_cast<long long>(e);
  long long nslots = static_cast<long long>(num_blocks) * block_size;
  const uint16_t* kss = static_cast<const uint16_t*>(k_scale_src);
  const uint16_t* vss = static_cast<const uint16_t*>(v_scale_src);
  uint16_t* ksc = static_cast<uint16_t*>(k_scale_cache);
  uint16_t* vsc = static_cast<uint16_t*>(v_scale_cache);
  int H = num_heads;
  long long rb = row_bytes;
  void* args[] = {&kp, &vp, &kcp, &vcp, &slot_mapping, &rb, &kst, &vst, &nslots, &kss, &vss, &ksc, &vsc, &H};
  cudaError_t err = launch_dependent(reinterpret_cast<const void*>(&reshape_and_cache_kernel), grid, dim3(threads), 0,
                                     static_cast<cudaStream_t>(stream), args);
  if (err != cudaSuccess) return cuda_fail(err, "launching reshape_and_cache");
  return PA_OK;
}

extern "C" pa_status copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs,
                                 int num_blocks, size_t block_bytes, void* k_scale_cache, void* v_scale_cache,
                                 size_t scale_block_bytes, void* stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_bytes == 0)
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: num_pairs >= 0, num_blocks > 0 and block_bytes > 0 required");
  const bool scales = k_scale_cache || v_scale_cache;
  if (scales && (!k_scale_cache || !v_scale_cache || scale_block_bytes == 0))
    return fail(PA_ERR_INVALID_ARG, "copy_blocks: pass both scale pools with scale_block_bytes > 0, or neither");
  if (num_pairs == 0) return PA_OK;
  if (!k_cache || !v_cache || !src_dst_pairs) return fail(PA_ERR_INVALID_ARG, "copy_blocks: NULL pointer");
  if (reinterpret_cast<uintptr_t>(src_dst_pairs) % 8) return fail(PA_ERR_INVALID_ARG, "copy_blocks: pairs must be 8-byte aligned");
  if (num_pairs > 65535) return fail(PA_ERR_UNSUPPORTED, "copy_blocks: at most 65535 pairs per call");

  BlockPools pools{{static_cast<const uint8_t*>(k_cache), static_cast<const uint8_t*>(v_cache),
                    static_cast<const uint8_t*>(k_scale_cache), static_cast<const uint8_t*>(v_scale_cache)},
                   {static_cast<uint8_t*>(k_cache), static_cast<uint8_t*>(v_cache),
                    static_cast<uint8_t*>(k_scale_cache), static_cast<uint8_t*>(v_scale_cache)}};
  cudaError_t err = launch_block_copy(pools, src_dst_pairs, num_pairs, block_bytes, scale_block_bytes, num_blocks,
                                      num_blocks, scales, static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "launching copy_blocks");
  return PA_OK;
}

extern "C" pa_status swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                                 const int64_t* src_dst_pairs, int num_pairs, int num_src_blocks, int num_dst_blocks,
                                 size_t block_bytes, const void* src_k_scale, const void* src_v_scale,
                                 void* dst_k_scale, void* dst_v_scale, size_t scale_block_bytes, void* stream) {
  if (num_pairs < 0 || num_src_blocks <= 0 || num_dst_blocks <= 0 || block_bytes == 0)
    return fail(PA_ERR_INVALID_ARG, "swap_blocks: num_pairs >= 0, pool sizes > 0 and block_bytes > 0 required");
  const int nscale = !!src_k_scale + !!src_v_scale + !!dst_k_scale + !!dst_v_scale;
  if (nscale != 0 && (nscale != 4 || scale_block_bytes == 0))
    return fail(PA_ERR_INVALID_ARG, "swap_blocks: pass all four scale pools with scale_block_bytes > 0, or none");
  if (num_pairs == 0) return PA_OK;
  if (!src_k || !src_v || !dst_k || !dst_v || !src_dst_pairs) return fail(PA_ERR_INVALID_ARG, "swap_blocks: NULL pointer");
  if (reinterpret_cast<uintptr_t>(src_dst_pairs) % 8) return fail(PA_ERR_INVALID_ARG, "swap_blocks: pairs must be 8-byte aligned");
  if (num_pairs > 65535) return fail(PA_ERR_UNSUPPORTED, "swap_blocks: at most 65535 pairs per call");

  const void* in[9] = {src_k, src_v, src_k_scale, src_v_scale, dst_k, dst_v, dst_k_scale, dst_v_scale, src_dst_pairs};
  static const char* const names[9] = {"src_k", "src_v", "src_k_scale", "src_v_scale", "dst_k",
                                       "dst_v", "dst_k_scale", "dst_v_scale", "src_dst_pairs"};
  const void* dev[9] = {};
  for (int i = 0; i < 9; ++i) {
    if (!in[i]) continue;
    const pa_status st = device_view(in[i], names[i], &dev[i]);
    if (st != PA_OK) return st;
  }
  BlockPools pools{{static_cast<const uint8_t*>(dev[0]), static_cast<const uint8_t*>(dev[1]),
                    static_cast<const uint8_t*>(dev[2]), static_cast<const uint8_t*>(dev[3])},
                   {static_cast<uint8_t*>(const_cast<void*>(dev[4])), static_cast<uint8_t*>(const_cast<void*>(dev[5])),
                    static_cast<uint8_t*>(const_cast<void*>(dev[6])), static_cast<uint8_t*>(const_cast<void*>(dev[7]))}};
  cudaError_t err = launch_block_copy(pools, static_cast<const int64_t*>(dev[8]), num_pairs, block_bytes,
                                      scale_block_bytes, num_src_blocks, num_dst_blocks, nscale != 0,
                                      static_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "launching swap_blocks");
  return PA_OK;
}

// ---------------------------------------------------------------------------------------
// Quantise-on-write ("KV Cache optimisation strategies in deployment" (yunthe.com),
// section "量化压缩KV Cache的INT8与FP8方案": an 8-bit KV cache; the per-(token, head) scheme
// is this library's).  One warp per (token, head, K-or-V) row: the row's max |x| by a warp
// reduction, scale = fp16(max / QMAX) with an IEEE fp32 division, then every element's code
// from an IEEE fp32 division by the fp16 scale, rounded to nearest even.
// ---------------------------------------------------------------------------------------
namespace pa {

template <typename CODE> struct Code;
template <> struct Code<int8_t> {
  static constexpr float kMax = 127.f;
  static __device__ __forceinline__ uint8_t encode(float r) {
    const float c = fminf(fmaxf(rintf(r), -127.f), 127.f);
    return static_cast<uint8_t>(static_cast<int8_t>(c));
  }
};
template <> struct Code<__nv_fp8_e4m3> {
  static constexpr float kMax = 448.f;
  static __device__ __forceinline__ uint8_t encode(float r) {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3));
  }
};

template <typename SRC, typename CODE, int D>
__global__ void __launch_bounds__(256)
reshape_and_cache_quant_kernel(const SRC* __restrict__ k, const SRC* __restrict__ v, uint8_t* __restrict__ kc,
                               uint8_t* __restrict__ vc, __half* __restrict__ ks, __half* __restrict__ vs,
                               const int64_t* __restrict__ slots, int T, int H, long long k_stride,
                               long long v_stride, long long num_slots) {
  constexpr int PER = D / 32;  // elements per lane: 2 or 4
  grid_dependency_launch_next();
  grid_dependency_wait();
  const long long row = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= 2LL * T * H) return;
  const int which = static_cast<int>(row & 1);  // 0: K, 1: V
  const long long th = row >> 1;
  const int t = static_cast<int>(th / H), h = static_cast<int>(th % H);
  const long long slot = __ldg(slots + t);
  if (slot < 0) return;
  if (slot >= num_slots) {
    if (lane == 0 && which == 0 && h == 0) cache_error(PA_DEVERR_SLOT);
    return;
  }
  const SRC* src = (which ? v + t * v_stride : k + t * k_stride) + static_cast<long long>(h) * D + lane * PER;
  float x[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) x[i] = static_cast<float>(src[i]);
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const __half scale = __float2half_rn(__fdiv_rn(amax, Code<CODE>::kMax));
  const float s = __half2float(scale);
  uint8_t c[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) c[i] = s > 0.f ? Code<CODE>::encode(__fdiv_rn(x[i], s)) : 0;
  uint8_t* dst = (which ? vc : kc) + (slot * H + h) * D + lane * PER;
  if (PER == 4) {
    *reinterpret_cast<uint32_t*>(dst) = c[0] | (c[1] << 8) | (c[2] << 16) | (static_cast<uint32_t>(c[3]) << 24);
  } else {
    *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(c[0] | (c[1] << 8));
  }
  if (lane == 0) (which ? vs : ks)[slot * H + h] = scale;
}

template <typename SRC, typename CODE>
const void* quant_kernel_for(int D) {
  return D == 64 ? reinterpret_cast<const void*>(&reshape_and_cache_quant_kernel<SRC, CODE, 64>)
                 : reinterpret_cast<const void*>(&reshape_and_cache_quant_kernel<SRC, CODE, 128>);
}

}  // namespace pa

extern "C" pa_status reshape_and_cache_quant(const void* k, const void* v, pa_dtype src_dtype, void* k_cache,
                                             void* v_cache, void* k_scale_cache, void* v_scale_cache,
                                             pa_dtype cache_dtype, const int64_t* slot_mapping, int num_tokens,
                                             int num_heads, int head_dim, int block_size, int num_blocks,
                                             int64_t k_token_stride, int64_t v_token_stride, void* stream) {
  if (num_tokens < 0 || num_heads <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: sizes must be positive (num_tokens >= 0)");
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache_quant: head_dim %d (supported: 64, 128)", head_dim);
  if (src_dtype != PA_F16 && src_dtype != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: src_dtype must be PA_F16 or PA_BF16");
  if (cache_dtype != PA_I8 && cache_dtype != PA_FP8_E4M3)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: cache_dtype must be PA_I8 or PA_FP8_E4M3");
  const long long row_elems = static_cast<long long>(num_heads) * head_dim;
  if (k_token_stride < row_elems || v_token_stride < row_elems)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: token strides must be >= num_heads*head_dim");
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !k_scale_cache || !v_scale_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: NULL pointer");
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) % 8 ||
      (reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache)) % 4 ||
      (reinterpret_cast<uintptr_t>(k_scale_cache) | reinterpret_cast<uintptr_t>(v_scale_cache)) % 2 ||
      reinterpret_cast<uintptr_t>(slot_mapping) % 8 || (k_token_stride * 2) % 8 || (v_token_stride * 2) % 8)
    return fail(PA_ERR_INVALID_ARG, "reshape_and_cache_quant: misaligned pointer or stride");
  const long long rows = 2LL * num_tokens * num_heads;
  const int threads = 256;
  const long long blocks = (rows + (threads / 32) - 1) / (threads / 32);
  if (blocks > 0x7fffffffLL) return fail(PA_ERR_UNSUPPORTED, "reshape_and_cache_quant: too many rows");
  const void* fn;
  if (src_dtype == PA_F16)
    fn = cache_dtype == PA_I8 ? quant_kernel_for<__half, int8_t>(head_dim) : quant_kernel_for<__half, __nv_fp8_e4m3>(head_dim);
  else
    fn = cache_dtype == PA_I8 ? quant_kernel_for<__nv_bfloat16, int8_t>(head_dim)
                              : quant_kernel_for<__nv_bfloat16, __nv_fp8_e4m3>(head_dim);
  const void* kp = k;
  const void* vp = v;
  void* kcp = k_cache;
  void* vcp = v_cache;
  void* ksp = k_scale_cache;
  void* vsp = v_scale_cache;
  int T = num_tokens, H = num_heads;
  long long kst = k_token_stride, vst = v_token_stride, nslots = static_cast<long long>(num_blocks) * block_size;
  void* args[] = {&kp, &vp, &kcp, &vcp, &ksp, &vsp, &slot_mapping, &T, &H, &kst, &vst, &nslots};
  cudaError_t err = launch_dependent(fn, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
                                     static_cast<cudaStream_t>(stream), args);
  if (err != cudaSuccess) return cuda_fail(err, "launching reshape_and_cache_quant");
  return PA_OK;
}
