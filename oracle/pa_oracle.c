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
 *
 * The (sequence, head) pairs are independent, so a caller may spread them over threads;
 * each pair is still computed by the same loops in the same order (see run_items).
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
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


/* ---------------------------------------------------------------------------------------
 * Work items and threads.
 *
 * Every output row of the decode oracle depends on one (sequence, query head) pair only,
 * and every output row of the prefill oracle on one (sequence, key/value head) pair, so
 * these pairs are independent "items".  Each item is computed by exactly the same loops,
 * in the same order, whether one thread runs every item or several threads share them;
 * the result is therefore bit-identical for any thread count.  Threads take the next
 * unclaimed item from a shared counter.  When items fail, the status returned is that of
 * the lowest-numbered failing item, as a single thread walking the items in order would
 * have stopped there first.
 * ------------------------------------------------------------------------------------- */
typedef struct {
  double* Kc;    /* [max_ctx][D] gathered keys   */
  double* Vc;    /* [max_ctx][D] gathered values */
  double* score; /* [max_ctx]                    */
  double* qv;    /* [D]                          */
} scratch_t;

typedef int (*item_fn)(const void* job, long item, scratch_t* buf);

typedef struct {
  const void* job;
  item_fn fn;
  long n_items;
  int max_ctx, D;
  atomic_long next;
  pthread_mutex_t lock;
  long bad_item; /* lowest failing item so far, or n_items */
  int bad_status;
} runner_t;

static void* run_worker(void* arg) {
  runner_t* r = (runner_t*)arg;
  scratch_t b;
  b.Kc = (double*)malloc(sizeof(double) * (size_t)r->max_ctx * r->D);
  b.Vc = (double*)malloc(sizeof(double) * (size_t)r->max_ctx * r->D);
  b.score = (double*)malloc(sizeof(double) * (size_t)r->max_ctx);
  b.qv = (double*)malloc(sizeof(double) * (size_t)r->D);
  if (!b.Kc || !b.Vc || !b.score || !b.qv) {
    pthread_mutex_lock(&r->lock);
    if (r->bad_item > 0) { r->bad_item = 0; r->bad_status = ORC_NO_MEMORY; }
    pthread_mutex_unlock(&r->lock);
  } else {
    for (;;) {
      long item = atomic_fetch_add(&r->next, 1);
      if (item >= r->n_items) break;
      int st = r->fn(r->job, item, &b);
      if (st != ORC_OK) {
        pthread_mutex_lock(&r->lock);
        if (item < r->bad_item) { r->bad_item = item; r->bad_status = st; }
        pthread_mutex_unlock(&r->lock);
      }
    }
  }
  free(b.Kc); free(b.Vc); free(b.score); free(b.qv);
  return NULL;
}

/* Run items 0 .. n_items-1 of `job` on `threads` threads (the caller's thread is one). */
static int run_items(const void* job, item_fn fn, long n_items, int max_ctx, int D, int threads) {
  runner_t r;
  r.job = job;
  r.fn = fn;
  r.n_items = n_items;
  r.max_ctx = max_ctx;
  r.D = D;
  atomic_init(&r.next, 0);
  pthread_mutex_init(&r.lock, NULL);
  r.bad_item = n_items;
  r.bad_status = ORC_OK;
  if (threads < 1) threads = 1;
  if (threads > n_items) threads = n_items > 0 ? (int)n_items : 1;
  pthread_t* tid = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)threads);
  int started = 0;
  if (tid)
    for (; started < threads - 1; ++started)
      if (pthread_create(&tid[started], NULL, run_worker, &r) != 0) break;
  run_worker(&r);
  for (int i = 0; i < started; ++i) pthread_join(tid[i], NULL);
  free(tid);
  pthread_mutex_destroy(&r.lock);
  return r.bad_status;
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
 *   threads      worker threads (>= 1); the result does not depend on it
 */
typedef struct {
  double* out;
  const void *q, *k_cache, *v_cache;
  int q_dtype, cache_dtype;
  const uint16_t *k_scale, *v_scale;
  const int32_t *block_tables, *context_lens;
  int S, Hq, Hkv, D, bs, MB, NB, window;
  double scale;
} decode_job;

/* One item: sequence s = item / Hq, query head h = item % Hq. */
static int decode_item(const void* jp, long item, scratch_t* b) {
  const decode_job* j = (const decode_job*)jp;
  const int s = (int)(item / j->Hq), h = (int)(item % j->Hq);
  const int D = j->D, bs = j->bs;
  const int group = j->Hq / j->Hkv; /* query heads sharing one key/value head */
  const int ctx = j->context_lens[s];
  if (ctx < 0 || ctx > j->MB * bs) return ORC_BAD_CONTEXT;
  int lo = 0;
  if (j->window > 0 && ctx > j->window) lo = ctx - j->window;
  const int n = ctx - lo;
  double* o = j->out + ((size_t)s * j->Hq + h) * D;
  if (n == 0) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    return ORC_OK;
  }

  /* step 2: gather through the block table */
  for (int i = lo; i < ctx; ++i) {
    int logical_block = i / bs;
    int offset = i % bs;
    int32_t pb = j->block_tables[(size_t)s * j->MB + logical_block];
    if (pb < 0 || pb >= j->NB) return ORC_BAD_TABLE;
    size_t row = ((size_t)pb * bs + offset) * j->Hkv + h / group; /* (pb*bs+off)*Hkv + kv head */
    double ks = 1.0, vs = 1.0;
    if (j->cache_dtype == ORC_I8 || j->cache_dtype == ORC_FP8) {
      ks = orc_f16_to_f64(j->k_scale[row]);
      vs = orc_f16_to_f64(j->v_scale[row]);
    }
    for (int d = 0; d < D; ++d) {
      b->Kc[(size_t)(i - lo) * D + d] = load_value(j->k_cache, j->cache_dtype, row * D + d) * ks;
      b->Vc[(size_t)(i - lo) * D + d] = load_value(j->v_cache, j->cache_dtype, row * D + d) * vs;
    }
  }

  for (int d = 0; d < D; ++d) b->qv[d] = load_value(j->q, j->q_dtype, ((size_t)s * j->Hq + h) * D + d);

  /* step 3: scaled dot products */
  for (int i = 0; i < n; ++i) {
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += b->qv[d] * b->Kc[(size_t)i * D + d];
    b->score[i] = j->scale * dot;
  }

  /* step 4: textbook softmax */
  double m = b->score[0];
  for (int i = 1; i < n; ++i) if (b->score[i] > m) m = b->score[i];
  double z = 0.0;
  for (int i = 0; i < n; ++i) { b->score[i] = exp(b->score[i] - m); z += b->score[i]; }
  for (int i = 0; i < n; ++i) b->score[i] /= z;

  /* step 5: probability-weighted sum of the value rows */
  for (int d = 0; d < D; ++d) {
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += b->score[i] * b->Vc[(size_t)i * D + d];
    o[d] = acc;
  }
  return ORC_OK;
}

int orc_paged_decode_gqa(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                         const uint16_t* v_scale, const int32_t* block_tables,
                         const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs, int MB,
                         int NB, double scale, int window, int threads) {
  if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || bs <= 0 || MB <= 0 || NB <= 0)
    return ORC_BAD_ARG;
  if ((cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) && (!k_scale || !v_scale)) return ORC_BAD_ARG;
  decode_job j = {out, q, k_cache, v_cache, q_dtype, cache_dtype, k_scale, v_scale,
                  block_tables, context_lens, S, Hq, Hkv, D, bs, MB, NB, window, scale};
  return run_items(&j, decode_item, (long)S * Hq, MB * bs, D, threads);
}

/* Multi-head decode: every query head has its own cached key/value head. */
int orc_paged_decode(double* out, const void* q, int q_dtype, const void* k_cache,
                     const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                     const uint16_t* v_scale, const int32_t* block_tables,
                     const int32_t* context_lens, int S, int H, int D, int bs, int MB, int NB,
                     double scale, int window) {
  return orc_paged_decode_gqa(out, q, q_dtype, k_cache, v_cache, cache_dtype, k_scale, v_scale,
                              block_tables, context_lens, S, H, H, D, bs, MB, NB, scale, window, 1);
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
typedef struct {
  double* out;
  const void *q, *k_cache, *v_cache;
  int q_dtype, cache_dtype;
  const uint16_t *k_scale, *v_scale;
  const int32_t *block_tables, *cu_q, *context_lens;
  int S, Hq, Hkv, D, bs, MB, NB, window;
  double scale;
} prefill_job;

/* One item: sequence s = item / Hkv, key/value head kh = item % Hkv, with every query head
 * that reads kh and every query token of s. */
static int prefill_item(const void* jp, long item, scratch_t* b) {
  const prefill_job* j = (const prefill_job*)jp;
  const int s = (int)(item / j->Hkv), kh = (int)(item % j->Hkv);
  const int D = j->D, bs = j->bs, Hq = j->Hq, Hkv = j->Hkv;
  const int group = Hq / Hkv;
  const int ctx = j->context_lens[s];
  const int q_len = j->cu_q[s + 1] - j->cu_q[s];
  if (ctx < 0 || ctx > j->MB * bs) return ORC_BAD_CONTEXT;
  if (q_len < 0 || q_len > ctx) return ORC_BAD_ARG;
  if (q_len == 0) return ORC_OK;

  /* gather every cached token of this key/value head through the block table */
  for (int i = 0; i < ctx; ++i) {
    int32_t pb = j->block_tables[(size_t)s * j->MB + i / bs];
    if (pb < 0 || pb >= j->NB) return ORC_BAD_TABLE;
    size_t row = ((size_t)pb * bs + i % bs) * Hkv + kh;
    double ks = 1.0, vs = 1.0;
    if (j->cache_dtype == ORC_I8 || j->cache_dtype == ORC_FP8) {
      ks = orc_f16_to_f64(j->k_scale[row]);
      vs = orc_f16_to_f64(j->v_scale[row]);
    }
    for (int d = 0; d < D; ++d) {
      b->Kc[(size_t)i * D + d] = load_value(j->k_cache, j->cache_dtype, row * D + d) * ks;
      b->Vc[(size_t)i * D + d] = load_value(j->v_cache, j->cache_dtype, row * D + d) * vs;
    }
  }

  for (int h = kh * group; h < (kh + 1) * group; ++h) {
    for (int i = 0; i < q_len; ++i) {
      const size_t t = (size_t)j->cu_q[s] + i;
      const int p = ctx - q_len + i;
      const int lo = (j->window > 0 && p + 1 > j->window) ? p + 1 - j->window : 0;
      const int n = p + 1 - lo;
      double* o = j->out + (t * Hq + h) * D;
      for (int d = 0; d < D; ++d) b->qv[d] = load_value(j->q, j->q_dtype, (t * Hq + h) * D + d);
      for (int k = 0; k < n; ++k) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += b->qv[d] * b->Kc[(size_t)(lo + k) * D + d];
        b->score[k] = j->scale * dot;
      }
      double m = b->score[0];
      for (int k = 1; k < n; ++k) if (b->score[k] > m) m = b->score[k];
      double z = 0.0;
      for (int k = 0; k < n; ++k) { b->score[k] = exp(b->score[k] - m); z += b->score[k]; }
      for (int k = 0; k < n; ++k) b->score[k] /= z;
      for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int k = 0; k < n; ++k) acc += b->score[k] * b->Vc[(size_t)(lo + k) * D + d];
        o[d] = acc;
      }
    }
  }
  return ORC_OK;
}

int orc_paged_prefill(double* out, const void* q, int q_dtype, const void* k_cache,
                      const void* v_cache, int cache_dtype, const uint16_t* k_scale,
                      const uint16_t* v_scale, const int32_t* block_tables, const int32_t* cu_q,
                      const int32_t* context_lens, int S, int Hq, int Hkv, int D, int bs, int MB,
                      int NB, double scale, int window, int threads) {
  if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || bs <= 0 || MB <= 0 || NB <= 0)
    return ORC_BAD_ARG;
  if ((cache_dtype == ORC_I8 || cache_dtype == ORC_FP8) && (!k_scale || !v_scale)) return ORC_BAD_ARG;
  if (S > 0 && cu_q[0] != 0) return ORC_BAD_ARG;
  prefill_job j = {out, q, k_cache, v_cache, q_dtype, cache_dtype, k_scale, v_scale,
                   block_tables, cu_q, context_lens, S, Hq, Hkv, D, bs, MB, NB, window, scale};
  return run_items(&j, prefill_item, (long)S * Hkv, MB * bs, D, threads);
}
