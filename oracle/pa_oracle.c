/*
 * pa_oracle.c -- plain fp64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no code, header or constant with the
 * CUDA path.
 *
 * What it computes (sources are the three web pages the method is taken from):
 *
 *   - Cache layout and address of one key/value row.  The pseudocode kernel on
 *     "KV Cache memory optimisation and PagedAttention" (yunthe.com), section
 *     "PagedAttention注意力计算流程", reads element (head h, token in physical
 *     block pb at offset off) at  h*head_dim + (pb*block_size + off)*num_heads*head_dim,
 *     i.e. a cache laid out as [num_blocks, block_size, num_heads, head_dim].
 *   - Logical -> physical mapping.  Same pseudocode, and "vLLM source first look:
 *     PagedAttention memory design" (trdm.cn), section 二, BlockTable.get_physical_block
 *     and get_offset: logical block i // block_size, offset i % block_size, physical
 *     block = block_table[logical block].
 *   - The attention itself.  The pseudocode computes score = dot(q, k) * scale and
 *     elides "softmax and weighted sum"; the oracle writes out textbook softmax
 *     attention over the gathered, contiguous K/V rows.
 *   - Sliding window.  "KV Cache optimisation strategies in deployment"
 *     (yunthe.com), section "Sliding Window Attention控制长序列显存": only the most
 *     recent W tokens take part.  Reading: tokens [max(0, ctx - W), ctx), the current
 *     token included; window <= 0 means full attention.
 *   - INT8 cache.  Same page, section "量化压缩KV Cache的INT8与FP8方案", names an
 *     INT8 KV cache but not its scheme.  Reading: one fp16 scale per (token, head)
 *     row, value = int8 code * scale, both converted to fp64 exactly.  The same
 *     section names FP8 ("E4M1", read as E4M3): the same per-row fp16 scale with an
 *     OCP FP8 E4M3 code, value = e4m3 value * scale, exact in fp64.
 *
 * Steps, in the order the pages give them, per (sequence s, head h):
 *   1. lo = window > 0 ? max(0, ctx - window) : 0.
 *   2. Gather K and V rows of logical tokens lo..ctx-1 through the block table into
 *      contiguous fp64 arrays Kc[n][D], Vc[n][D]  (n = ctx - lo).
 *   3. score_i = scale * sum_d q[d] * Kc[i][d].
 *   4. m = max_i score_i;  p_i = exp(score_i - m) / sum_j exp(score_j - m).
 *   5. out[d] = sum_i p_i * Vc[i][d].
 *   ctx == 0 (nothing to attend): out = 0.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_I8 = 3, ORC_FP8 = 4 };

enum {
  ORC_OK = 0,
  ORC_BAD_ARG = 1,
  ORC_BAD_TABLE = 2,   /* a block-table entry outside [0, num_blocks) */
  ORC_BAD_CONTEXT = 3, /* context_len < 0 or > max_blocks_per_seq * block_size */
  ORC_NO_MEMORY = 4
};

/* IEEE-754 binary16 -> double, exactly (every binary16 value is a double). */
double orc_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int exponent = (h >> 10) & 0x1f;
  int mantissa = h & 0x3ff;
  double v;
  if (exponent == 0) {
    v = ldexp((double)mantissa, -24); /* subnormal: mantissa * 2^-24 */
  } else if (exponent == 31) {
    v = mantissa ? NAN : INFINITY;
  } else {
    v = ldexp((double)(mantissa | 0x400), exponent - 25); /* 1.m * 2^(e-15) */
  }
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32; widen, then convert exactly. */
double orc_bf16_to_f64(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* FP8 E4M3 (the OCP "fn" variant: no infinities, S.1111.111 is NaN) -> double, exactly:
 * exponent field 0 is subnormal, m * 2^-9; otherwise (1 + m/8) * 2^(e - 7). */
double orc_e4m3_to_f64(uint8_t c) {
  int sign = (c >> 7) & 1;
  int exponent = (c >> 3) & 0xf;
  int mantissa = c & 0x7;
  double v;
  if (exponent == 15 && mantissa == 7) return NAN;
  if (exponent == 0) v = ldexp((double)mantissa, -9);
  else v = ldexp((double)(8 + mantissa), exponent - 10);
  return sign ? -v : v;
}

static double load_value(const void* base, int dtype, size_t index) {
  switch (dtype) {
    case ORC_F32: return (double)((const float*)base)[index];
    case ORC_F16: return orc_f16_to_f64(((const uint16_t*)base)[index]);
    case ORC_BF16: return orc_bf16_to_f64(((const uint16_t*)base)[index]);
    case ORC_I8: return (double)((const int8_t*)base)[index];
    case ORC_FP8: return orc_e4m3_to_f64(((const uint8_t*)base)[index]);
    default: return NAN;
  }
}

/*
 * Paged decode attention, one query token per sequence.  Grouped-query attention (not on
 * the pages; the usual definition): query head h reads key/value head h / (Hq / Hkv), so
 * consecutive query heads share a cached head; Hq == Hkv is the pages' multi-head case.
 *
 *   out          [S, Hq, D] fp64, written
 *   q            [S, Hq, D] in q_dtype (F32 / F16 / BF16)
 *   k_cache,     [NB, bs, Hkv, D] in cache_dtype (F32 / F16 / BF16 / I8 / FP8)
 *   v_cache
 *   k_scale,     [NB, bs, Hkv] binary16 bit patterns; required for I8 and FP8, ignored otherwise
 *   v_scale
 *   block_tables [S, MB] int32; only entries of blocks that hold attended tokens are read
 *   context_lens [S] int32
 */
int orc_paged_decode_gqa(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                         const uint16_t* v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs, int MB,
                         int NB, double scale, int window) {
  if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || bs <= 0 || MB <= 0 || NB <= 0)
    return ORC_BAD_ARG;
  const int group = Hq / Hkv; /* query heads sharing one key/value head */
  if ((cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) && (!k_scale || !v_scale)) return ORC_BAD_ARG;

  int max_ctx = MB * bs;
  double* Kc = (double*)malloc(sizeof(double) * (size_t)max_ctx * D);
  double* Vc = (double*)malloc(sizeof(double) * (size_t)max_ctx * D);
  double* score = (double*)malloc(sizeof(double) * (size_t)max_ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)D);
  if (!Kc || !Vc || !score || !qv) {
    free(Kc); free(Vc); free(score); free(qv);
    return ORC_NO_MEMORY;
  }
  int status = ORC_OK;

  for (int s = 0; s < S && status == ORC_OK; ++s) {
    int ctx = context_lens[s];
    if (ctx < 0 || ctx > max_ctx) { status = ORC_BAD_CONTEXT; break; }
    int lo = 0;
    if (window > 0 && ctx > window) lo = ctx - window;
    int n = ctx - lo;

    for (int h = 0; h < Hq && status == ORC_OK; ++h) {
      double* o = out + ((size_t)s * Hq + h) * D;
      if (n == 0) {
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        continue;
      }

      /* step 2: gather through the block table */
      for (int i = lo; i < ctx; ++i) {
        int logical_block = i / bs;
        int offset = i % bs;
        int32_t pb = block_tables[(size_t)s * MB + logical_block];
        if (pb < 0 || pb >= NB) { status = ORC_BAD_TABLE; break; }
        size_t row = ((size_t)pb * bs + offset) * Hkv + h / group; /* (pb*bs+off)*Hkv + kv head */
        double ks = 1.0, vs = 1.0;
        if (cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) {
          ks = orc_f16_to_f64(k_scale[row]);
          vs = orc_f16_to_f64(v_scale[row]);
        }
        for (int d = 0; d < D; ++d) {
          Kc[(size_t)(i - lo) * D + d] = load_value(k_cache, cache_dtype, row * D + d) * ks;
          Vc[(size_t)(i - lo) * D + d] = load_value(v_cache, cache_dtype, row * D + d) * vs;
        }
      }
      if (status != ORC_OK) break;

      for (int d = 0; d < D; ++d) qv[d] = load_value(q, q_dtype, ((size_t)s * Hq + h) * D + d);

      /* step 3: scaled dot products */
      for (int i = 0; i < n; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += qv[d] * Kc[(size_t)i * D + d];
        score[i] = scale * dot;
      }

      /* step 4: textbook softmax */
      double m = score[0];
      for (int i = 1; i < n; ++i) if (score[i] > m) m = score[i];
      double z = 0.0;
      for (int i = 0; i < n; ++i) { score[i] = exp(score[i] - m); z += score[i]; }
      for (int i = 0; i < n; ++i) score[i] /= z;

      /* step 5: probability-weighted sum of the value rows */
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += score[i] * Vc[(size_t)i * D + d];
        o[d] = acc;
      }
    }
  }

  free(Kc); free(Vc); free(score); free(qv);
  return status;
}

/* Multi-head decode: every query head has its own cached key/value head. */
int orc_paged_decode(double* out, const void* q, int q_dtype, const void* k_cache,
                     const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                     const uint16_t* v_scale, const int32_t* block_tables,
                     const int32_t* context_lens, int S, int H, int D, int bs, int MB, int NB,
                     double scale, int window) {
  return orc_paged_decode_gqa(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                              block_tables, context_lens, S, H, H, D, bs, MB, NB, scale, window);
}

/*
 * Paged prefill / chunked-prefill attention: several new query tokens per sequence, each
 * attending causally to the cache.  The pages motivate it (the prompt stage writes many
 * tokens' K/V at once: "vLLM source first look: PagedAttention memory design" (trdm.cn),
 * section 四; long single-sequence contexts such as document summarisation: "KV Cache
 * memory optimisation and PagedAttention" (yunthe.com), section
 * "PagedAttention在不同推理场景下的适用性") but print no formula; this is the usual causal
 * attention, read with the same cache layout, block table, window and GQA rules as decode.
 *
 * Readings.  The chunk's K/V rows are already in the cache (written before attention, as
 * for decode), so sequence s holds context_lens[s] tokens and its q_len newest ones are the
 * queries: query i sits at position p = ctx - q_len + i and attends tokens [lo, p], with
 * lo = max(0, p + 1 - window) for window > 0 (the last `window` tokens up to and
 * including itself) and 0 otherwise.  q_len == 1 is exactly decode.
 *
 *   out          [T, Hq, D] fp64, T = cu_q[S]; row t = cu_q[s] + i
 *   q            [T, Hq, D] in q_dtype
 *   cu_q         [S + 1] int32, cu_q[0] = 0, non-decreasing; q_len = cu_q[s+1] - cu_q[s]
 *   other arguments as for orc_paged_decode_gqa; q_len <= context_lens[s] is required.
 */
int orc_paged_prefill(double* out, const void* q, int q_dtype, const void* k_cache,
                      const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                      const uint16_t* v_scale, const int32_t* block_tables, const int32_t* cu_q,
                      const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs, int MB,
                      int NB, double scale, int window) {
  if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || bs <= 0 || MB <= 0 || NB <= 0)
    return ORC_BAD_ARG;
  if ((cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) && (!k_scale || !v_scale)) return ORC_BAD_ARG;
  if (S > 0 && cu_q[0] != 0) return ORC_BAD_ARG;
  const int group = Hq / Hkv;
  const int max_ctx = MB * bs;
  double* Kc = (double*)malloc(sizeof(double) * (size_t)max_ctx * D);
  double* Vc = (double*)malloc(sizeof(double) * (size_t)max_ctx * D);
  double* score = (double*)malloc(sizeof(double) * (size_t)max_ctx);
  double* qv = (double*)malloc(sizeof(double) * (size_t)D);
  if (!Kc || !Vc || !score || !qv) {
    free(Kc); free(Vc); free(score); free(qv);
    return ORC_NO_MEMORY;
  }
  int status = ORC_OK;

  for (int s = 0; s < S && status == ORC_OK; ++s) {
    const int ctx = context_lens[s];
    const int q_len = cu_q[s + 1] - cu_q[s];
    if (ctx < 0 || ctx > max_ctx) { status = ORC_BAD_CONTEXT; break; }
    if (q_len < 0 || q_len > ctx) { status = ORC_BAD_ARG; break; }
    if (q_len == 0) continue;

    for (int kh = 0; kh < Hkv && status == ORC_OK; ++kh) {
      /* gather every cached token of this key/value head through the block table */
      for (int i = 0; i < ctx; ++i) {
        int32_t pb = block_tables[(size_t)s * MB + i / bs];
        if (pb < 0 || pb >= NB) { status = ORC_BAD_TABLE; break; }
        size_t row = ((size_t)pb * bs + i % bs) * Hkv + kh;
        double ks = 1.0, vs = 1.0;
        if (cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) {
          ks = orc_f16_to_f64(k_scale[row]);
          vs = orc_f16_to_f64(v_scale[row]);
        }
        for (int d = 0; d < D; ++d) {
          Kc[(size_t)i * D + d] = load_value(k_cache, cache_dtype, row * D + d) * ks;
          Vc[(size_t)i * D + d] = load_value(v_cache, cache_dtype, row * D + d) * vs;
        }
      }
      if (status != ORC_OK) break;

      for (int h = kh * group; h < (kh + 1) * group; ++h) {
        for (int i = 0; i < q_len; ++i) {
          const size_t t = (size_t)cu_q[s] + i;
          const int p = ctx - q_len + i;
          const int lo = (window > 0 && p + 1 > window) ? p + 1 - window : 0;
          const int n = p + 1 - lo;
          double* o = out + (t * Hq + h) * D;
          for (int d = 0; d < D; ++d) qv[d] = load_value(q, q_dtype, (t * Hq + h) * D + d);
          for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d) dot += qv[d] * Kc[(size_t)(lo + j) * D + d];
            score[j] = scale * dot;
          }
          double m = score[0];
          for (int j = 1; j < n; ++j) if (score[j] > m) m = score[j];
          double z = 0.0;
          for (int j = 0; j < n; ++j) { score[j] = exp(score[j] - m); z += score[j]; }
          for (int j = 0; j < n; ++j) score[j] /= z;
          for (int d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int j = 0; j < n; ++j) acc += score[j] * Vc[(size_t)(lo + j) * D + d];
            o[d] = acc;
          }
        }
      }
    }
  }
  free(Kc); free(Vc); free(score); free(qv);
  return status;
}
