/*
 * pagedattn.h -- C ABI of libpagedattn.so: paged decode attention on NVIDIA B200 (sm_100a).
 *
 * The method (sources: three web pages on PagedAttention):
 *   "KV Cache memory optimisation and PagedAttention" (yunthe.com)              [page A]
 *   "KV Cache optimisation strategies in deployment" (yunthe.com)               [page B]
 *   "vLLM source first look: PagedAttention memory design" (trdm.cn)             [page C]
 *
 * The KV cache is cut into fixed-size physical blocks of block_size tokens (page A,
 * section "PagedAttention分页内存管理原理").  A sequence finds token i through its block
 * table: logical block i / block_size, offset i % block_size (page C, section 二,
 * BlockTable.get_physical_block / get_offset).  Cache layout, from the pseudocode
 * kernel's address h*D + (pb*bs + off)*H*D (page A, section "PagedAttention注意力计算流程"):
 *
 *     k_cache, v_cache : [num_blocks, block_size, num_heads, head_dim]   (row-major)
 *     k_scale, v_scale : [num_blocks, block_size, num_heads] fp16        (INT8 / FP8 caches only)
 *
 * A *slot* is pb*block_size + off: one token row of num_heads*head_dim values.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller (cudaMalloc or any
 *     allocator; swap_blocks also takes mapped page-locked host memory); the library
 *     never allocates, frees or keeps them.  Tensors are dense,
 *     row-major, and their base addresses must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued
 *     asynchronously; the call returns once it is launched.
 *   - Arguments are validated on the host before anything is launched; a non-PA_OK
 *     status means nothing was enqueued.  pa_last_error() then gives a message.
 *   - Device-side checks never fault: a block-table entry outside [0, num_blocks), a
 *     context length above max_blocks_per_seq*block_size, a slot or copy pair outside
 *     the pool is skipped or clamped and recorded in a device error word, read with
 *     pa_device_error().  Results of such a call are unspecified.
 *   - No call aborts, throws across the ABI or spins without a bound.
 */
#ifndef PAGEDATTN_H_
#define PAGEDATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_dtype {
  PA_F32 = 0,  /* IEEE binary32 */
  PA_F16 = 1,  /* IEEE binary16 */
  PA_BF16 = 2, /* bfloat16 */
  PA_I8 = 3,   /* signed 8-bit code with a per-(token, head) fp16 scale */
  PA_FP8_E4M3 = 4 /* OCP FP8 E4M3 code with a per-(token, head) fp16 scale */
} pa_dtype;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,   /* a pointer, size, alignment or dtype is not acceptable */
  PA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. head_dim 96) */
  PA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (message has the CUDA error) */
  PA_ERR_OUT_OF_BLOCKS = 4, /* block manager: fewer free blocks than requested */
  PA_ERR_BAD_BLOCK = 5      /* block manager: id out of range, or reference count would go negative */
} pa_status;

/* Bits of the device error word (pa_device_error). */
#define PA_DEVERR_TABLE 0x1u   /* block-table entry outside [0, num_blocks): block 0 read instead */
#define PA_DEVERR_CONTEXT 0x2u /* context_len < 0 or > max_blocks_per_seq*block_size: clamped */
#define PA_DEVERR_SLOT 0x4u    /* reshape_and_cache slot >= num_blocks*block_size: token skipped */
#define PA_DEVERR_PAIR 0x8u    /* copy_blocks / swap_blocks pair outside its pool: pair skipped */
#define PA_DEVERR_TIMEOUT 0x10u /* a bounded pipeline wait gave up (a library bug; results invalid) */

/* Message for the last non-PA_OK status returned on the calling thread ("" if none). */
const char* pa_last_error(void);

/* Library version string. */
const char* pa_version(void);

/*
 * Read (and if clear != 0, reset) the device error word of the current device.
 * Synchronises the device first.  *flags receives an OR of PA_DEVERR_* bits.
 */
pa_status pa_device_error(uint32_t* flags, int clear);

/* ------------------------------------------------------------------------------------ */
/* Decode attention                                                                     */
/* ------------------------------------------------------------------------------------ */

/*
 * Bytes of scratch workspace paged_attention_decode needs on the CURRENT device for a
 * batch of num_seqs sequences x num_heads heads of size head_dim (any block_size,
 * dtype or context length).  Returns 0 for invalid sizes or when no device is present.
 */
size_t pa_decode_workspace_bytes(int num_seqs, int num_heads, int head_dim);

/*
 * Paged decode attention: one query token per sequence attends over its cached keys
 * and values.  Source: page A, section "PagedAttention注意力计算流程" (score =
 * dot(q, k) * scale through the block table; softmax and the probability-weighted
 * sum of values), page C, section 三 (walk the cache block by block), page B,
 * section "Sliding Window Attention控制长序列显存" (window).
 *
 * For sequence s, head h, with ctx = context_lens[s] and lo = window > 0 ?
 * max(0, ctx - window) : 0, the attended tokens are i in [lo, ctx):
 *     k_i  = k_cache[block_tables[s][i / block_size], i % block_size, h, :]
 *     p    = softmax_i(scale * <q[s,h,:], k_i>)
 *     out[s,h,:] = sum_i p_i * v_i                      (ctx == 0: zeros)
 * An INT8 or FP8 (E4M3) cache holds codes c with k = value(c) * k_scale[slot, h] (likewise v).
 *
 *   out            [num_seqs, num_heads, head_dim]        io_dtype, written
 *   q              [num_seqs, num_heads, head_dim]        io_dtype
 *   k_cache,
 *   v_cache        [num_blocks, block_size, num_heads, head_dim]   cache_dtype
 *   k_scale,
 *   v_scale        [num_blocks, block_size, num_heads] fp16; required iff cache_dtype is PA_I8 or PA_FP8_E4M3
 *   block_tables   [num_seqs, max_blocks_per_seq] int32; only entries of blocks that hold
 *                  attended tokens are read (others may hold anything, e.g. -1)
 *   context_lens   [num_seqs] int32, 0 <= ctx <= max_blocks_per_seq*block_size
 *   head_dim       64 or 128;  block_size 1..32;  num_heads >= 1 (multiple of 8 for 8-bit caches)
 *   scale          softmax scale (typically 1/sqrt(head_dim))
 *   window         0 = full attention, W > 0 = the last W tokens only
 *   io_dtype       PA_F32, PA_F16 or PA_BF16; cache_dtype == io_dtype, or PA_I8 / PA_FP8_E4M3 with
 *                  io_dtype PA_F16 / PA_BF16
 *   workspace      device scratch of >= pa_decode_workspace_bytes(...) bytes; contents
 *                  need no initialisation and are clobbered.  Two calls that may run
 *                  concurrently need distinct workspaces.
 *
 * Two kernels are enqueued (partition pass, then merge of split partitions).
 * Accumulation is fp32; out is rounded to io_dtype (round to nearest even).
 */
pa_status paged_attention_decode(void* out, const void* q, const void* k_cache,
                                 const void* v_cache, const void* k_scale, const void* v_scale,
                                 const int32_t* block_tables, const int32_t* context_lens,
                                 int num_seqs, int num_heads, int head_dim, int block_size,
                                 int num_blocks, int max_blocks_per_seq, float scale, int window,
                                 pa_dtype io_dtype, pa_dtype cache_dtype, void* workspace,
                                 size_t workspace_bytes, void* stream);

/*
 * Grouped-query (and multi-query) paged decode: num_q_heads query heads share
 * num_kv_heads cached heads, query head h reading cached head h / (num_q_heads /
 * num_kv_heads).  Not on the pages (which size Llama-2-70B with 64 cached heads); the
 * usual grouped-query definition.  Arguments as paged_attention_decode, except
 *   q, out         [num_seqs, num_q_heads, head_dim]
 *   k_cache,
 *   v_cache        [num_blocks, block_size, num_kv_heads, head_dim]
 *   k_scale, v_scale [num_blocks, block_size, num_kv_heads] (8-bit caches)
 *   num_q_heads    a multiple of num_kv_heads
 * and the workspace is sized by pa_decode_workspace_bytes(num_seqs, num_q_heads, head_dim).
 * paged_attention_decode(..., num_heads, ...) is this call with both head counts equal.
 */
pa_status paged_attention_decode_gqa(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const void* k_scale, const void* v_scale,
                                     const int32_t* block_tables, const int32_t* context_lens,
                                     int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                     int block_size, int num_blocks, int max_blocks_per_seq,
                                     float scale, int window, pa_dtype io_dtype, pa_dtype cache_dtype,
                                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * Process-wide switch (default 1): let grouped-query decode run on the tensor cores when
 * the call qualifies -- fp16 or bf16 io_dtype with a cache of the same type (head_dim 64 or
 * 128) or an INT8 / FP8 E4M3 cache (head_dim 128), block_size a multiple of 8 dividing 128, and 4..16 query heads
 * per cached head, or more with a divisor in [4, 16] (multi-query attention: the query heads
 * of a cached head are split into sub-groups of that size, each reading the cached head).  Then each 128-token tile of one cached head is two tcgen05 MMAs (scores
 * K.q^T and the weighted sum V^T.p^T, fp32 accumulators in tensor memory) instead of
 * CUDA-core dot products.  8-bit codes are the MMA operands as stored (INT8: integer MMAs,
 * FP8: E4M3 MMAs); q and the softmax weights enter as 8-bit digits (INT8: the two bytes of
 * a 16-bit fixed-point value; FP8: three E4M3 digits, ~12 significant bits), the per-token
 * K scale multiplies the score and the V scale is folded into the weight.  0 forces the
 * CUDA-core kernel (same results within the tolerances).  Not thread-safe against concurrent decode calls; set it
 * once at start-up.
 */
pa_status pa_decode_use_tensor_cores(int enable);

/*
 * paged_attention_decode for callers that cannot allocate device memory.  No counterpart
 * on the pages: it exists for callers with no device allocator of their own -- e.g. a
 * plugin inside a host framework that owns all device memory and passes only the op's
 * tensors, or a latency-critical loop that cannot afford cudaMalloc's implicit device
 * synchronisation.
 *
 * Same arguments and results as paged_attention_decode, minus the workspace.  The
 * scratch is a fixed 16 MiB array inside the library's device memory, present on every
 * GPU that loads the library until the process exits; this call allocates nothing.
 *   - Batches whose pa_decode_workspace_bytes() exceeds 16 MiB are rejected with
 *     PA_ERR_INVALID_ARG (nothing is launched).
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current); make that first call before any stream capture.
 *   - `stream` must belong to the current device: the address looked up and the size
 *     check both refer to the current device.
 *   - The address is kept for the life of the process.  Do not call this entry point
 *     again on a device after cudaDeviceReset() of that device: the reset unloads the
 *     library's device code together with the array, and the kept address then points
 *     to nothing.
 *   - Every call on a device shares the one array: calls that may overlap on the GPU
 *     (different streams, no ordering between them) race and corrupt each other's
 *     results.  Calls ordered on one stream are fine.
 *   - The array keeps the last call's contents; the kernels overwrite every part of it
 *     that they read, so nothing has to be cleared between calls.
 */
pa_status paged_attention_decode_static_scratch(void* out, const void* q, const void* k_cache,
                                                const void* v_cache, const void* k_scale,
                                                const void* v_scale, const int32_t* block_tables,
                                                const int32_t* context_lens, int num_seqs,
                                                int num_heads, int head_dim, int block_size,
                                                int num_blocks, int max_blocks_per_seq, float scale,
                                                int window, pa_dtype io_dtype, pa_dtype cache_dtype,
                                                void* stream);

/* ------------------------------------------------------------------------------------ */
/* Cache maintenance                                                                    */
/* ------------------------------------------------------------------------------------ */

/*
 * Write each new token's key/value rows into its slot.  Source: the cache grows by one
 * row per generated token (page C, section 一) into blocks allocated on demand (page A,
 * section "vLLM调度器与PagedAttention协同工作").
 *
 *   k, v           [num_tokens, num_heads, head_dim] rows of `dtype`; consecutive tokens
 *                  k_token_stride / v_token_stride ELEMENTS apart (>= num_heads*head_dim,
 *                  so rows of a fused QKV tensor can be passed directly)
 *   k_cache,
 *   v_cache        [num_blocks, block_size, num_heads, head_dim] of `dtype`
 *   slot_mapping   [num_tokens] int64: token t goes to slot slot_mapping[t]
 *                  (= block*block_size + offset); a negative slot skips the token
 *   dtype          PA_F32 / PA_F16 / PA_BF16 / PA_I8 / PA_FP8_E4M3 (codes are copied as they are)
 *   k_scale_src,   [num_tokens, num_heads] fp16 scales of the new rows, and
 *   v_scale_src    k_scale_cache, v_scale_cache [num_blocks, block_size, num_heads] fp16:
 *   k_scale_cache, required iff dtype is PA_I8 or PA_FP8_E4M3, NULL otherwise
 *   v_scale_cache
 * Bit-exact copy.  Slots must be distinct (otherwise which token lands is unspecified).
 */
pa_status reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                            const int64_t* slot_mapping, int num_tokens, int num_heads,
                            int head_dim, int block_size, int num_blocks, int64_t k_token_stride,
                            int64_t v_token_stride, pa_dtype dtype, const void* k_scale_src,
                            const void* v_scale_src, void* k_scale_cache, void* v_scale_cache,
                            void* stream);

/*
 * Paged prefill / chunked-prefill attention: several new query tokens per sequence, each
 * attending causally to the paged cache.  The pages motivate it (page C, section 四: the
 * prompt stage writes many tokens' K/V at once; page A, section
 * "PagedAttention在不同推理场景下的适用性": long single-sequence contexts) but give no
 * formula; this is the usual causal attention with the cache layout, block-table walk and
 * window rule of paged_attention_decode:
 *   the chunk's own K/V rows are already in the cache (reshape_and_cache first), so
 *   sequence s holds context_lens[s] tokens and its q_len newest are the queries; query i
 *   sits at position p = ctx - q_len + i and attends tokens [lo, p], lo = max(0, p + 1 -
 *   window) for window > 0, else 0.  q_len == 1 is decode.
 *
 *   out, q         [num_q_tokens, num_q_heads, head_dim] in dtype (PA_F16 or PA_BF16); the
 *                  rows of sequence s are cu_q_lens[s] .. cu_q_lens[s+1]-1;
 *                  num_q_tokens * num_q_heads < 2^31 (else PA_ERR_UNSUPPORTED)
 *   k_cache,       [num_blocks, block_size, num_kv_heads, head_dim] in dtype
 *   v_cache
 *   head_dim       128 or 64 (else PA_ERR_UNSUPPORTED)
 *   block_tables   [num_seqs, max_blocks_per_seq] int32
 *   cu_q_lens      [num_seqs + 1] int32 device array, cu_q_lens[0] = 0, non-decreasing
 *   context_lens   [num_seqs] int32 device array, q_len <= context_len <= max_blocks_per_seq*block_size
 *   max_q_len      an upper bound of every q_len (sizes the grid; a larger q_len is an error)
 *   num_q_heads    a multiple of num_kv_heads with a power of two up to 128 query heads per cached head
 *   block_size     8, 16, 32, 64 or 128
 * Tensor cores (tcgen05), fp32 accumulation; bf16 probabilities keep ~16 bits (hi + lo
 * parts).  A sequence whose q_len exceeds max_q_len or its context, whose rows run
 * past num_q_tokens, or whose context exceeds the table, is skipped and sets
 * PA_DEVERR_CONTEXT; a table entry outside
 * [0, num_blocks) reads block 0 and sets PA_DEVERR_TABLE.  Needs no workspace.
 */
pa_status paged_attention_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, const int32_t* cu_q_lens,
                                  const int32_t* context_lens, int num_seqs, int num_q_tokens,
                                  int max_q_len, int num_q_heads, int num_kv_heads, int head_dim,
                                  int block_size, int num_blocks, int max_blocks_per_seq,
                                  float scale, int window, pa_dtype dtype, void* stream);

/*
 * paged_attention_prefill over an 8-bit cache: INT8 or FP8 E4M3 codes with one fp16 scale
 * per (token, cached head), as written by reshape_and_cache_quant.  Source: page B, section
 * "量化压缩KV Cache的INT8与FP8方案" (8-bit KV caches), with the prefill reading above.
 *
 *   k_cache, v_cache  [num_blocks, block_size, num_kv_heads, 128] codes of cache_dtype
 *                     (head_dim must be 128: another value is PA_ERR_UNSUPPORTED)
 *   k_scale, v_scale  [num_blocks, block_size, num_kv_heads] fp16 (2-byte aligned)
 *   io_dtype          PA_F16 or PA_BF16 (q and out)
 *   cache_dtype       PA_I8 or PA_FP8_E4M3 (anything else: PA_ERR_INVALID_ARG)
 * Other arguments, layouts and errors as paged_attention_prefill.  Each cached value
 * code * scale enters the tensor-core products rounded once to io_dtype (relative error
 * 2^-11 for fp16, 2^-8 for bf16); accumulation is fp32.
 */
pa_status paged_attention_prefill_quant(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, const void* k_scale,
                                        const void* v_scale, const int32_t* block_tables,
                                        const int32_t* cu_q_lens, const int32_t* context_lens,
                                        int num_seqs, int num_q_tokens, int max_q_len,
                                        int num_q_heads, int num_kv_heads, int head_dim,
                                        int block_size, int num_blocks, int max_blocks_per_seq,
                                        float scale, int window, pa_dtype io_dtype,
                                        pa_dtype cache_dtype, void* stream);

/*
 * Copy whole physical blocks for copy-on-write.  Source: page C, section 二,
 * BlockManager.copy_on_write (the new block receives a copy of the old block's KV
 * data) and section 四 (the copy is a latency cost of forking).
 *
 *   k_cache, v_cache    pools of num_blocks blocks, block_bytes bytes each
 *                       (block_size*num_heads*head_dim*element size)
 *   src_dst_pairs       [num_pairs, 2] int64 device array of (src, dst) block ids
 *   k_scale_cache,      optional (both or neither) pools of scale_block_bytes bytes per
 *   v_scale_cache       block (INT8 cache: block_size*num_heads*2)
 * Destinations must be distinct and no destination may also be a source (otherwise the
 * result is unspecified).  Bit-exact copy.
 */
pa_status copy_blocks(void* k_cache, void* v_cache, const int64_t* src_dst_pairs, int num_pairs,
                      int num_blocks, size_t block_bytes, void* k_scale_cache, void* v_scale_cache,
                      size_t scale_block_bytes, void* stream);

/*
 * Quantise-on-write: like reshape_and_cache, but the new rows arrive in fp16 / bf16 and
 * are stored as 8-bit codes with one fp16 scale per (token, head) row.  Source: page B,
 * section "量化压缩KV Cache的INT8与FP8方案" (an INT8 KV cache halves the memory; FP8 --
 * printed "E4M1", read as E4M3 -- is the alternative); the scheme is this library's:
 *   PA_I8:        scale = max_d |x_d| / 127 (fp32, then rounded to fp16),
 *                 code  = clamp(rint(x_d / scale), -127, 127)      (fp32 division, ties to even)
 *   PA_FP8_E4M3:  scale = max_d |x_d| / 448 (fp32, then rounded to fp16),
 *                 code  = E4M3(x_d / scale)       (fp32 division, nearest even, saturating)
 *   a row whose fp16 scale is 0 stores scale 0 and zero codes.
 *
 *   k, v           [num_tokens, num_heads, head_dim] of src_dtype (PA_F16 or PA_BF16),
 *                  token strides in elements as in reshape_and_cache
 *   k_cache,       [num_blocks, block_size, num_heads, head_dim] of cache_dtype
 *   v_cache        (PA_I8 or PA_FP8_E4M3)
 *   k_scale_cache, [num_blocks, block_size, num_heads] fp16
 *   v_scale_cache
 *   slot_mapping   [num_tokens] int64 (negative = skip)
 *   head_dim       64 or 128
 * Results are bit-exact with the definition above (IEEE fp32 division, RNE roundings).
 */
pa_status reshape_and_cache_quant(const void* k, const void* v, pa_dtype src_dtype, void* k_cache,
                                  void* v_cache, void* k_scale_cache, void* v_scale_cache,
                                  pa_dtype cache_dtype, const int64_t* slot_mapping, int num_tokens,
                                  int num_heads, int head_dim, int block_size, int num_blocks,
                                  int64_t k_token_stride, int64_t v_token_stride, void* stream);

/*
 * Swap whole blocks between two pools that live in different address spaces: the GPU
 * pool and a page-locked host pool ("swap space").  Source: page A, section
 * "vLLM调度器与PagedAttention协同工作", item 3 (preemption: under memory pressure a
 * low-priority request's KV blocks move out to CPU memory, freeing GPU blocks, and move
 * back when room returns) and section "vLLM部署配置与PagedAttention参数调优" (swap_space,
 * the size of the CPU pool in GB).  Swap-out is (GPU pool -> host pool), swap-in the
 * reverse; one call moves every listed block in ONE kernel launch whose threads read and
 * write the host pool directly over the host link (no staging copy, no per-block call).
 *
 *   src_k, src_v          source pools, num_src_blocks blocks of block_bytes bytes each
 *   dst_k, dst_v          destination pools, num_dst_blocks blocks of block_bytes bytes
 *   src_dst_pairs         [num_pairs, 2] int64 of (source block id, destination block id)
 *   src_k_scale, ...      optional (all four or none) scale pools, scale_block_bytes per
 *                         block (8-bit caches: block_size*num_heads*2)
 * Every pool and the pair array may each be device memory (any allocator) or page-locked
 * host memory mapped into the device's address space (cudaHostAlloc, or cudaHostRegister
 * with the mapped flag; torch's pin_memory qualifies).  Pageable host memory is rejected
 * with PA_ERR_INVALID_ARG.  Pools passed as host pointers are translated to their device
 * addresses by the library.  Destinations must be distinct and, when source and
 * destination are the same pool, no destination may also be a source.  A pair outside
 * either pool is skipped and sets PA_DEVERR_PAIR.  Bit-exact copy.  The copy is ordered
 * on `stream` like a kernel: host code must synchronise the stream before it reads a
 * host destination or reuses a host source.
 */
pa_status swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                      const int64_t* src_dst_pairs, int num_pairs, int num_src_blocks,
                      int num_dst_blocks, size_t block_bytes, const void* src_k_scale,
                      const void* src_v_scale, void* dst_k_scale, void* dst_v_scale,
                      size_t scale_block_bytes, void* stream);

/* ------------------------------------------------------------------------------------ */
/* Host-side block manager (free list + reference counts)                               */
/* ------------------------------------------------------------------------------------ */

/*
 * Physical-block allocator of page C, section 二 (BlockManager): a free list popped
 * from its end, one reference count per block, copy-on-write.  Host memory only; not
 * thread-safe (one manager per thread, or external locking).
 */
typedef struct pa_block_manager pa_block_manager;

/* free_order: optional permutation of 0..num_blocks-1 giving the initial free list
 * (the last entry is allocated first); NULL means 0..num_blocks-1.  NULL on bad input. */
pa_block_manager* pa_bm_create(int num_blocks, int block_size, const int32_t* free_order);
void pa_bm_destroy(pa_block_manager* bm);

/* Take n blocks (reference count 1 each) into out_ids[n].  PA_ERR_OUT_OF_BLOCKS if fewer
 * than n are free (nothing allocated). */
pa_status pa_bm_allocate(pa_block_manager* bm, int n, int32_t* out_ids);

/* Drop one reference of each listed block; a block whose count reaches 0 returns to the
 * end of the free list.  PA_ERR_BAD_BLOCK (and no change at all) if any id is out of
 * range or would drop below zero (double free). */
pa_status pa_bm_free(pa_block_manager* bm, const int32_t* ids, int n);

/* Add one reference to each listed, allocated block (a sequence forks and shares it). */
pa_status pa_bm_share(pa_block_manager* bm, const int32_t* ids, int n);

/* Copy-on-write: a block referenced at most once is returned unchanged; otherwise a new
 * block is allocated (count 1), the old block loses one reference, and the new id is
 * returned -- the caller then copies the data with copy_blocks. */
pa_status pa_bm_copy_on_write(pa_block_manager* bm, int32_t block_id, int32_t* out_id);

int pa_bm_num_free(const pa_block_manager* bm);
int pa_bm_ref_count(const pa_block_manager* bm, int32_t block_id); /* -1 if out of range */
double pa_bm_usage_ratio(const pa_block_manager* bm);             /* 1 - free/num_blocks */
/* Copy the free list (bottom to top) into out[cap]; *n receives its length. */
pa_status pa_bm_free_list(const pa_block_manager* bm, int32_t* out, int cap, int* n);

/*
 * Slot of token position pos of a sequence (host arrays): for each of n entries,
 *   out[i] = block_tables[seq[i]*max_blocks_per_seq + pos[i]/block_size]*block_size
 *            + pos[i] % block_size
 * (page A, pseudocode kernel: physical_offset = physical_block*block_size + offset).
 * PA_ERR_INVALID_ARG if a position falls outside the table or hits a negative entry.
 */
pa_status pa_slot_mapping_host(const int32_t* block_tables, int num_seqs, int max_blocks_per_seq,
                               int block_size, const int32_t* seq, const int32_t* pos, int n,
                               int64_t* out);

/* ------------------------------------------------------------------------------------ */
/* Profiling hooks                                                                      */
/* ------------------------------------------------------------------------------------ */

/* When enabled, paged_attention_decode records CUDA events around each of its two
 * kernels on the launch stream (a few hundred ns of host time per call). */
pa_status pa_profile_enable(int on);
/* Synchronise the recorded events and return the summed device time of the partition
 * and merge kernels over *calls calls since the last reset (reset != 0 clears). */
pa_status pa_profile_read(double* partition_ms, double* merge_ms, int* calls, int reset);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H_ */
