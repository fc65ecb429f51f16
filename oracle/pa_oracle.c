/*
 * pa_oracle.c -- plain CPU reference ("the oracle") for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg load this library. The CUDA product never calls it, and the two share no code: no headers,
 * no helpers, no tables, no constants.
 *
 * Every result is computed in double precision from the values stored in the cache, one output at a
 * time, in the plainest order the definition allows. Speed is not a goal; the only concession is that
 * independent (sequence, head) outputs may be spread over host threads, which changes no arithmetic.
 *
 * Pages this follows (cited by page title and section):
 *  [T] "企业官网建设流程全解析" -- the body of this page is a PagedAttention tutorial (its title is a
 *      scraping artefact):
 *        sec. 2.1 "基本数据结构设计": a block holds the keys and values of a fixed number of tokens
 *          (16 by default); a block table maps a sequence's logical blocks to physical blocks.
 *        sec. 2.2 "分块注意力计算过程": Attention(Q,K,V) = softmax(QK^T / sqrt(d)) V. The same section's
 *          loop applies softmax per block and sums the per-block outputs; that loop is NOT what this
 *          oracle computes (its weights do not sum to one once a context spans two blocks). The
 *          oracle normalises over the whole context, as the formula says.
 *        sec. 3.2 "关键性能优化": blocks may be stored in FP8.
 *  [V] "vLLM的诞生背景：大模型推理的痛点与PagedAttention的破局":
 *        "PagedAttention的破局思路": logically contiguous KV, physically scattered blocks, a block table
 *          mapping one to the other, blocks allocated on demand as the sequence grows.
 *        "PagedAttention的局限性": shared blocks are handled with reference counts and copy-on-write.
 *  [C] "PagedAttention 与连续批处理：LLM Serving 的底层架构拆解", section
 *        "PagedAttention：把显存做成虚拟内存": attention finds each page through the page table and then
 *          attends within it.
 *  FP8 E4M3 follows the OCP 8-bit Floating Point Specification (OFP8): 1 sign bit, 4 exponent bits
 *  (bias 7), 3 mantissa bits, subnormals, no infinities, S.1111.111 is NaN, largest finite 448.
 *
 * Readings where the pages are silent (each one is listed with its reason in the design notes):
 *  - cache layout [num_blocks][block_size][num_kv_heads][head_size], element (blk, off, h, i) at
 *    ((blk*block_size + off)*num_kv_heads + h)*head_size + i;
 *  - grouped-query heads: query head h reads kv head h / (num_heads / num_kv_heads);
 *  - a context of length 0 gives an all-zero output row;
 *  - FP8 values dequantise as code_value * scale[kv_head] (per-head format), or code_value *
 *    scale[block][kv_head] (per-block format: [T] sec. 3.2 stores blocks in FP8 one by one, so each
 *    block may carry its own scale); quantisation is
 *    code = nearest E4M3 value to (float)x / scale (IEEE single division), ties to the even code,
 *    magnitudes >= 448 (and infinities) saturate to +-448, every NaN maps to the canonical NaN code
 *    0x7F (the OCP spec does not fix the sign of a NaN produced by a conversion);
 *  - reshape_and_cache skips slots < 0 (padding) and slots past the pool.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* OR_E4M3_BLOCK: E4M3 codes like OR_E4M3, with one scale per (block, kv head) instead of per kv head. */
enum { OR_F16 = 0, OR_BF16 = 1, OR_E4M3 = 2, OR_E4M3_BLOCK = 3 };

enum {
  OR_OK = 0,
  OR_BAD_ARG = 1,
  OR_BAD_BLOCK = 2, /* a block table entry outside [0, num_blocks) was needed */
  OR_NO_MEMORY = 3
};

/* ------------------------------------------------------------------------------------------------
 * Scalar decoders, each written from its format's definition.
 * --------------------------------------------------------------------------------------------- */

/* IEEE 754 binary16: sign, 5 exponent bits (bias 15), 10 fraction bits. */
double or_f16_to_double(uint16_t bits) {
  int sign = bits >> 15;
  int exponent = (bits >> 10) & 0x1F;
  int fraction = bits & 0x3FF;
  double v;
  if (exponent == 0)
    v = ldexp((double)fraction, -24); /* subnormal: (fraction / 2^10) * 2^-14 */
  else if (exponent == 31)
    v = fraction ? NAN : INFINITY;
  else
    v = ldexp(1.0 + fraction / 1024.0, exponent - 15);
  return sign ? -v : v;
}

/* bfloat16: sign, 8 exponent bits (bias 127), 7 fraction bits. */
double or_bf16_to_double(uint16_t bits) {
  int sign = bits >> 15;
  int exponent = (bits >> 7) & 0xFF;
  int fraction = bits & 0x7F;
  double v;
  if (exponent == 0)
    v = ldexp((double)fraction, -133); /* subnormal: (fraction / 2^7) * 2^-126 */
  else if (exponent == 255)
    v = fraction ? NAN : INFINITY;
  else
    v = ldexp(1.0 + fraction / 128.0, exponent - 127);
  return sign ? -v : v;
}

/* OCP E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; S.1111.111 is NaN; no infinities. */
double or_e4m3_to_double(uint8_t code) {
  int sign = code >> 7;
  int exponent = (code >> 3) & 0xF;
  int mantissa = code & 0x7;
  double v;
  if (exponent == 15 && mantissa == 7)
    v = NAN;
  else if (exponent == 0)
    v = ldexp((double)mantissa, -9); /* subnormal: (mantissa / 8) * 2^-6 */
  else
    v = ldexp(1.0 + mantissa / 8.0, exponent - 7);
  return sign ? -v : v;
}

/* Encode a float to E4M3: the nearest finite E4M3 value, ties to the code with an even mantissa,
 * magnitudes at or above the largest finite value (448, including infinity) saturate to it, and every
 * NaN maps to the canonical NaN code 0x7F. The candidate set is searched directly: the 127
 * non-negative finite codes 0x00..0x7E have strictly increasing values. */
uint8_t or_e4m3_from_float(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7E;
  /* Find c with value(c) <= a < value(c + 1), 0 <= c <= 125. */
  int lo = 0, hi = 126; /* invariant: value(lo) <= a < value(hi) */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (or_e4m3_to_double((uint8_t)mid) <= a)
      lo = mid;
    else
      hi = mid;
  }
  double below = a - or_e4m3_to_double((uint8_t)lo);
  double above = or_e4m3_to_double((uint8_t)hi) - a;
  int pick;
  if (below < above)
    pick = lo;
  else if (above < below)
    pick = hi;
  else
    pick = (lo % 2 == 0) ? lo : hi; /* tie: the code whose mantissa is even */
  return (uint8_t)(sign | pick);
}

/* Bulk versions for the Python wrapper. */
void or_e4m3_to_double_n(const uint8_t* codes, double* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = or_e4m3_to_double(codes[i]);
}
void or_e4m3_from_float_n(const float* x, uint8_t* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = or_e4m3_from_float(x[i]);
}
void or_f16_to_double_n(const uint16_t* bits, double* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = or_f16_to_double(bits[i]);
}
void or_bf16_to_double_n(const uint16_t* bits, double* out, size_t n) {
  for (size_t i = 0; i < n; ++i) out[i] = or_bf16_to_double(bits[i]);
}

/* Value of element `index` of an array stored in `dtype`. For E4M3 the per-head scale is applied by
 * the caller. */
static double element(const void* base, int dtype, size_t index) {
  switch (dtype) {
    case OR_F16: return or_f16_to_double(((const uint16_t*)base)[index]);
    case OR_BF16: return or_bf16_to_double(((const uint16_t*)base)[index]);
    default: return or_e4m3_to_double(((const uint8_t*)base)[index]);
  }
}

/* Dequantisation scale of kv head kvh for a token in physical block blk: 1 for 16-bit caches, the
 * kv head's scale for the per-head E4M3 format, the (block, kv head) scale for the per-block one. */
static double kv_scale(const float* scale, int kv_dtype, int blk, int num_kv_heads, int kvh) {
  if (kv_dtype == OR_E4M3) return (double)scale[kvh];
  if (kv_dtype == OR_E4M3_BLOCK) return (double)scale[(size_t)blk * num_kv_heads + kvh];
  return 1.0;
}

/* ------------------------------------------------------------------------------------------------
 * Paged decode attention, by definition ([T] sec. 2.2 formula; indirection per [T] sec. 2.1,
 * [V] "PagedAttention的破局思路", [C] "PagedAttention：把显存做成虚拟内存").
 *
 * For every sequence s and query head h, with G = num_heads / num_kv_heads and kvh = h / G:
 *   for t = 0 .. L_s - 1: blk = block_tables[s][t / bs], off = t % bs,
 *                         k_t = K[blk][off][kvh][:], v_t = V[blk][off][kvh][:] (dequantised),
 *                         z_t = scale * sum_i q[s][h][i] * k_t[i]
 *   m = max_t z_t,  w_t = exp(z_t - m),  out[s][h][:] = sum_t w_t v_t / sum_t w_t
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  double* out;             /* [S][H][d] */
  const void* query;       /* [S][H][d] in q_dtype */
  int q_dtype;
  const void* key_cache;   /* [NB][bs][Hkv][d] in kv_dtype */
  const void* value_cache;
  int kv_dtype;
  const float* k_scale;    /* [Hkv], E4M3 only */
  const float* v_scale;
  const int32_t* block_tables; /* [S][max_blocks_per_seq] */
  int max_blocks_per_seq;
  const int32_t* context_lens; /* [S] */
  int num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks;
  double scale;
  int num_threads;
  int thread_index;
  int status;
} or_attention_job;

static int attend_one(const or_attention_job* a, int s, int h, double* z) {
  const int d = a->head_size;
  const int G = a->num_heads / a->num_kv_heads;
  const int kvh = h / G;
  const int L = a->context_lens[s];
  double* o = a->out + ((size_t)s * a->num_heads + h) * d;
  const size_t q_base = ((size_t)s * a->num_heads + h) * d;
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  if (L == 0) return OR_OK;

  /* Scores. */
  for (int t = 0; t < L; ++t) {
    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];
    int off = t % a->block_size;
    if (blk < 0 || blk >= a->num_blocks) return OR_BAD_BLOCK;
    size_t k_base = (((size_t)blk * a->block_size + off) * a->num_kv_heads + kvh) * d;
    const double ks = kv_scale(a->k_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);
    double dot = 0.0;
    for (int i = 0; i < d; ++i)
      dot += element(a->query, a->q_dtype, q_base + i) * (element(a->key_cache, a->kv_dtype, k_base + i) * ks);
    z[t] = a->scale * dot;
  }
  /* Softmax over the whole context: subtract the maximum, exponentiate, normalise. */
  double m = z[0];
  for (int t = 1; t < L; ++t)
    if (z[t] > m) m = z[t];
  double denom = 0.0;
  for (int t = 0; t < L; ++t) denom += exp(z[t] - m);
  /* Weighted sum of values. */
  for (int t = 0; t < L; ++t) {
    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];
    int off = t % a->block_size;
    size_t v_base = (((size_t)blk * a->block_size + off) * a->num_kv_heads + kvh) * d;
    const double vs = kv_scale(a->v_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);
    double w = exp(z[t] - m) / denom;
    for (int i = 0; i < d; ++i) o[i] += w * (element(a->value_cache, a->kv_dtype, v_base + i) * vs);
  }
  return OR_OK;
}

static void* attention_worker(void* arg) {
  or_attention_job* a = (or_attention_job*)arg;
  int max_len = 1;
  for (int s = 0; s < a->num_seqs; ++s)
    if (a->context_lens[s] > max_len) max_len = a->context_lens[s];
  double* z = (double*)malloc(sizeof(double) * (size_t)max_len);
  if (!z) {
    a->status = OR_NO_MEMORY;
    return NULL;
  }
  const long total = (long)a->num_seqs * a->num_heads;
  for (long item = a->thread_index; item < total; item += a->num_threads) {
    int st = attend_one(a, (int)(item / a->num_heads), (int)(item % a->num_heads), z);
    if (st != OR_OK) {
      a->status = st;
      break;
    }
  }
  free(z);
  return NULL;
}

int or_paged_attention(double* out, const void* query, int q_dtype, const void* key_cache,
                       const void* value_cache, int kv_dtype, const float* k_scale,
                       const float* v_scale, const int32_t* block_tables, int max_blocks_per_seq,
                       const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                       int head_size, int block_size, int num_blocks, double scale,
                       int num_threads) {
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens) return OR_BAD_ARG;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return OR_BAD_ARG;
  if (head_size <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq < 0) return OR_BAD_ARG;
  if (q_dtype != OR_F16 && q_dtype != OR_BF16) return OR_BAD_ARG;
  if (kv_dtype != OR_F16 && kv_dtype != OR_BF16 && kv_dtype != OR_E4M3 && kv_dtype != OR_E4M3_BLOCK) return OR_BAD_ARG;
  if ((kv_dtype == OR_E4M3 || kv_dtype == OR_E4M3_BLOCK) && (!k_scale || !v_scale)) return OR_BAD_ARG;
  for (int s = 0; s < num_seqs; ++s)
    if (context_lens[s] < 0 || (long)context_lens[s] > (long)max_blocks_per_seq * block_size) return OR_BAD_ARG;
  if (num_threads < 1) num_threads = 1;

  or_attention_job base = {out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                           block_tables, max_blocks_per_seq, context_lens, num_seqs, num_heads,
                           num_kv_heads, head_size, block_size, num_blocks, scale, num_threads, 0, OR_OK};
  or_attention_job* jobs = (or_attention_job*)malloc(sizeof(or_attention_job) * (size_t)num_threads);
  pthread_t* threads = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)num_threads);
  if (!jobs || !threads) {
    free(jobs);
    free(threads);
    return OR_NO_MEMORY;
  }
  int started = 0;
  for (int t = 0; t < num_threads; ++t) {
    jobs[t] = base;
    jobs[t].thread_index = t;
  }
  for (int t = 1; t < num_threads; ++t) {
    if (pthread_create(&threads[t], NULL, attention_worker, &jobs[t]) != 0) break;
    started = t;
  }
  /* Items owned by threads that failed to start are done here, in the calling thread. */
  for (int t = started + 1; t < num_threads; ++t) attention_worker(&jobs[t]);
  attention_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(threads[t], NULL);
  int status = OR_OK;
  for (int t = 0; t < num_threads; ++t)
    if (jobs[t].status != OR_OK) status = jobs[t].status;
  free(jobs);
  free(threads);
  return status;
}

/* ------------------------------------------------------------------------------------------------
 * Writing new tokens into their slots ([V] "PagedAttention的破局思路": blocks are filled as the
 * sequence grows). Token i of key/value [T][Hkv][d] goes to slot slot_mapping[i], i.e. block
 * slot / bs, offset slot % bs. E4M3 caches store or_e4m3_from_float((float)x / scale), with scale the
 * kv head's (scale[h]) or, in the per-block format, the slot's block's (scale[block][h]).
 * --------------------------------------------------------------------------------------------- */
int or_reshape_and_cache(const void* key, const void* value, int in_dtype, void* key_cache,
                         void* value_cache, int kv_dtype, const float* k_scale, const float* v_scale,
                         const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                         int head_size, int block_size, int64_t num_blocks) {
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return OR_BAD_ARG;
  if (in_dtype != OR_F16 && in_dtype != OR_BF16) return OR_BAD_ARG;
  const int fp8 = kv_dtype == OR_E4M3 || kv_dtype == OR_E4M3_BLOCK;
  if (kv_dtype != in_dtype && !fp8) return OR_BAD_ARG;
  if (fp8 && (!k_scale || !v_scale)) return OR_BAD_ARG;
  for (int64_t i = 0; i < num_tokens; ++i) {
    int64_t slot = slot_mapping[i];
    if (slot < 0 || slot >= num_blocks * block_size) continue;
    int64_t blk = slot / block_size, off = slot % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      for (int j = 0; j < head_size; ++j) {
        size_t src = ((size_t)i * num_kv_heads + h) * head_size + j;
        size_t dst = (((size_t)blk * block_size + off) * num_kv_heads + h) * head_size + j;
        if (kv_dtype == in_dtype) {
          ((uint16_t*)key_cache)[dst] = ((const uint16_t*)key)[src];
          ((uint16_t*)value_cache)[dst] = ((const uint16_t*)value)[src];
        } else {
          /* The input value is exact in float; the division is IEEE single precision. */
          float kx = (float)element(key, in_dtype, src);
          float vx = (float)element(value, in_dtype, src);
          size_t sidx = (kv_dtype == OR_E4M3_BLOCK) ? (size_t)blk * num_kv_heads + h : (size_t)h;
          float ky = kx / k_scale[sidx];
          float vy = vx / v_scale[sidx];
          ((uint8_t*)key_cache)[dst] = or_e4m3_from_float(ky);
          ((uint8_t*)value_cache)[dst] = or_e4m3_from_float(vy);
        }
      }
    }
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------------------------------
 * Copy-on-write ([V] "PagedAttention的局限性"; sharing by reference count in [T] sec. 2.3): for each
 * pair (src, dst) the whole key block and the whole value block are copied.
 * --------------------------------------------------------------------------------------------- */
int or_copy_blocks(void* key_cache, void* value_cache, int kv_dtype, const int64_t* block_mapping,
                   int64_t num_pairs, int num_kv_heads, int head_size, int block_size,
                   int64_t num_blocks) {
  if (!key_cache || !value_cache || (!block_mapping && num_pairs > 0)) return OR_BAD_ARG;
  size_t elem = (kv_dtype == OR_E4M3 || kv_dtype == OR_E4M3_BLOCK) ? 1 : 2;
  size_t block_bytes = (size_t)block_size * num_kv_heads * head_size * elem;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return OR_BAD_BLOCK;
    memcpy((char*)key_cache + dst * block_bytes, (const char*)key_cache + src * block_bytes, block_bytes);
    memcpy((char*)value_cache + dst * block_bytes, (const char*)value_cache + src * block_bytes, block_bytes);
  }
  return OR_OK;
}

/* ------------------------------------------------------------------------------------------------
 * Swapping blocks between two pools ([C] "PagedAttention：把显存做成虚拟内存": pages of inactive
 * sequences are moved to CPU memory and brought back when needed): for each pair (src, dst) the whole
 * key block and the whole value block of the source pool are copied into block dst of the other pool.
 * --------------------------------------------------------------------------------------------- */
int or_swap_blocks(void* dst_key_cache, void* dst_value_cache, const void* src_key_cache,
                   const void* src_value_cache, int kv_dtype, const int64_t* block_mapping,
                   int64_t num_pairs, int num_kv_heads, int head_size, int block_size,
                   int64_t src_num_blocks, int64_t dst_num_blocks) {
  if (!dst_key_cache || !dst_value_cache || !src_key_cache || !src_value_cache || (!block_mapping && num_pairs > 0))
    return OR_BAD_ARG;
  size_t elem = (kv_dtype == OR_E4M3 || kv_dtype == OR_E4M3_BLOCK) ? 1 : 2;
  size_t block_bytes = (size_t)block_size * num_kv_heads * head_size * elem;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return OR_BAD_BLOCK;
    memcpy((char*)dst_key_cache + dst * block_bytes, (const char*)src_key_cache + src * block_bytes, block_bytes);
    memcpy((char*)dst_value_cache + dst * block_bytes, (const char*)src_value_cache + src * block_bytes, block_bytes);
  }
  return OR_OK;
}


/* ------------------------------------------------------------------------------------------------
 * Paged prefill attention: a chunk of new query tokens per sequence over the paged cache, causal.
 * Prefill (the prompt) is the compute-bound phase ([C] "对 agent 开发者的启示"); each token attends
 * only to the keys and values of its prefix ([C] "PagedAttention：把显存做成虚拟内存": a token needs
 * the KV of the tokens before it), with the [T] sec. 2.2 formula over that prefix.
 *
 * Sequence s has n_s = q_start[s+1] - q_start[s] query rows (rows q_start[s] .. q_start[s+1]-1 of
 * query/out), and L_s = context_lens[s] cached tokens that already include the chunk's own keys and
 * values. The chunk is the last n_s of those tokens (reading: a chunk continues the sequence), so
 * query j of the chunk sits at position p = L_s - n_s + j and attends to t = 0 .. p:
 *   z_t = scale * sum_i q[row][h][i] * k_t[i],  out[row][h][:] = sum_t exp(z_t - m) v_t / sum_t exp(z_t - m)
 * with m = max_t z_t, k_t and v_t found through block_tables[s] as in decode, and dequantised as in
 * decode for the FP8 formats (code x the kv head's scale, or x the scale of the token's physical
 * block and kv head).
 * --------------------------------------------------------------------------------------------- */
typedef struct {
  double* out;                 /* [T][H][d] */
  const void* query;           /* [T][H][d] in q_dtype */
  int q_dtype;
  const void* key_cache;
  const void* value_cache;
  int kv_dtype;
  const float* k_scale;
  const float* v_scale;
  const int32_t* block_tables; /* [S][max_blocks_per_seq] */
  int max_blocks_per_seq;
  const int32_t* context_lens; /* [S] */
  const int32_t* q_start;      /* [S + 1] */
  int num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks;
  double scale;
  int num_threads, thread_index, status;
} or_prefill_job;

static int prefill_one(const or_prefill_job* a, int s, int row, int h, double* z) {
  const int d = a->head_size;
  const int kvh = h / (a->num_heads / a->num_kv_heads);
  const int n = a->q_start[s + 1] - a->q_start[s];
  const int j = row - a->q_start[s];
  const int p = a->context_lens[s] - n + j; /* position of this query token */
  const size_t q_base = ((size_t)row * a->num_heads + h) * d;
  double* o = a->out + q_base;
  for (int i = 0; i < d; ++i) o[i] = 0.0;
  for (int t = 0; t <= p; ++t) {
    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];
    if (blk < 0 || blk >= a->num_blocks) return OR_BAD_BLOCK;
    size_t k_base = (((size_t)blk * a->block_size + t % a->block_size) * a->num_kv_heads + kvh) * d;
    const double ks = kv_scale(a->k_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);
    double dot = 0.0;
    for (int i = 0; i < d; ++i)
      dot += element(a->query, a->q_dtype, q_base + i) * (element(a->key_cache, a->kv_dtype, k_base + i) * ks);
    z[t] = a->scale * dot;
  }
  double m = z[0];
  for (int t = 1; t <= p; ++t)
    if (z[t] > m) m = z[t];
  double denom = 0.0;
  for (int t = 0; t <= p; ++t) denom += exp(z[t] - m);
  for (int t = 0; t <= p; ++t) {
    int blk = a->block_tables[(size_t)s * a->max_blocks_per_seq + t / a->block_size];
    size_t v_base = (((size_t)blk * a->block_size + t % a->block_size) * a->num_kv_heads + kvh) * d;
    const double vs = kv_scale(a->v_scale, a->kv_dtype, blk, a->num_kv_heads, kvh);
    double w = exp(z[t] - m) / denom;
    for (int i = 0; i < d; ++i) o[i] += w * (element(a->value_cache, a->kv_dtype, v_base + i) * vs);
  }
  return OR_OK;
}

static void* prefill_worker(void* arg) {
  or_prefill_job* a = (or_prefill_job*)arg;
  int max_len = 1;
  for (int s = 0; s < a->num_seqs; ++s)
    if (a->context_lens[s] > max_len) max_len = a->context_lens[s];
  double* z = (double*)malloc(sizeof(double) * (size_t)max_len);
  if (!z) {
    a->status = OR_NO_MEMORY;
    return NULL;
  }
  const long rows = a->q_start[a->num_seqs];
  const long total = rows * a->num_heads;
  int s = 0;
  for (long item = a->thread_index; item < total; item += a->num_threads) {
    int row = (int)(item / a->num_heads), h = (int)(item % a->num_heads);
    while (a->q_start[s + 1] <= row) ++s; /* rows are visited in increasing order */
    int st = prefill_one(a, s, row, h, z);
    if (st != OR_OK) {
      a->status = st;
      break;
    }
  }
  free(z);
  return NULL;
}

int or_paged_prefill(double* out, const void* query, int q_dtype, const void* key_cache,
                     const void* value_cache, int kv_dtype, const float* k_scale, const float* v_scale,
                     const int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                     const int32_t* q_start, int num_seqs, int num_heads, int num_kv_heads, int head_size,
                     int block_size, int num_blocks, double scale, int num_threads) {
  if (!out || !query || !key_cache || !value_cache || !block_tables || !context_lens || !q_start) return OR_BAD_ARG;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return OR_BAD_ARG;
  if (head_size <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq < 0) return OR_BAD_ARG;
  if (q_dtype != OR_F16 && q_dtype != OR_BF16) return OR_BAD_ARG;
  if (kv_dtype != OR_F16 && kv_dtype != OR_BF16 && kv_dtype != OR_E4M3 && kv_dtype != OR_E4M3_BLOCK)
    return OR_BAD_ARG;
  if ((kv_dtype == OR_E4M3 || kv_dtype == OR_E4M3_BLOCK) && (!k_scale || !v_scale)) return OR_BAD_ARG;
  if (q_start[0] != 0) return OR_BAD_ARG;
  for (int s = 0; s < num_seqs; ++s) {
    int n = q_start[s + 1] - q_start[s];
    if (n < 0 || n > context_lens[s]) return OR_BAD_ARG; /* a chunk lies inside its context */
    if ((long)context_lens[s] > (long)max_blocks_per_seq * block_size) return OR_BAD_ARG;
  }
  if (num_threads < 1) num_threads = 1;
  or_prefill_job base = {out, query, q_dtype, key_cache, value_cache, kv_dtype, k_scale, v_scale,
                         block_tables, max_blocks_per_seq, context_lens, q_start, num_seqs, num_heads,
                         num_kv_heads, head_size, block_size, num_blocks, scale, num_threads, 0, OR_OK};
  or_prefill_job* jobs = (or_prefill_job*)malloc(sizeof(or_prefill_job) * (size_t)num_threads);
  pthread_t* threads = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)num_threads);
  if (!jobs || !threads) {
    free(jobs);
    free(threads);
    return OR_NO_MEMORY;
  }
  int started = 0;
  for (int t = 0; t < num_threads; ++t) {
    jobs[t] = base;
    jobs[t].thread_index = t;
  }
  for (int t = 1; t < num_threads; ++t) {
    if (pthread_create(&threads[t], NULL, prefill_worker, &jobs[t]) != 0) break;
    started = t;
  }
  for (int t = started + 1; t < num_threads; ++t) prefill_worker(&jobs[t]);
  prefill_worker(&jobs[0]);
  for (int t = 1; t <= started; ++t) pthread_join(threads[t], NULL);
  int status = OR_OK;
  for (int t = 0; t < num_threads; ++t)
    if (jobs[t].status != OR_OK) status = jobs[t].status;
  free(jobs);
  free(threads);
  return status;
}
