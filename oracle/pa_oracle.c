/*
 * pa_oracle.c -- plain fp64 CPU oracle for paged decode attention and the two
 * cache operations that feed it.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke() entry and the
 * bench's CPU-baseline / reference arm may load this library.  It shares no code
 * with the CUDA path (no headers, no helpers, no tables) and is deliberately
 * slow: every loop follows the definition of the operation, with no blocking,
 * no online softmax and no split over partitions.
 *
 * Sources (web pages on vLLM / PagedAttention):
 *  - "详解vLLM推理引擎架构" (tbr8.org), section "PagedAttention 的核心思想":
 *    the KV cache is cut into fixed-size blocks of 16 or 32 tokens; a per-sequence
 *    block table maps logical block b to a physical block anywhere in the pool.
 *  - same page, section "Copy-on-Write 与内存共享": a write to a block whose
 *    refcount exceeds 1 first copies the block (copy_block(old, new)).
 *  - "vLLM 深度解读" (luoboask.github.io), section 3 "PagedAttention CUDA Kernel":
 *    k_cache / v_cache are [num_blocks, block_size, num_kv_heads, head_size];
 *    q and out are [num_seqs, num_heads, head_size]; the element of token t of a
 *    sequence lives at physical_block*block_size*num_kv_heads*head_size
 *    + (t % block_size)*num_kv_heads*head_size + head*head_size, with
 *    physical_block = block_table[t / block_size]; the score is
 *    scale * sum_d q[d]*k[d] and the result is softmax(scores) applied to V.
 *  - "vLLM 深度解读", section 7 (Llama attention): new K/V are stored into the
 *    paged cache before attention runs, so the context includes the new token.
 *  - "详解vLLM推理引擎架构", section "量化集成与部署": the KV cache may be stored in FP8
 *    (--kv-cache-dtype fp8).  The page names no format; read here as OCP E4M3 with one
 *    fp32 scale for K and one for V: stored code = e4m3(x / scale), value = code * scale.
 *  - same page, sections "量化集成与部署" (speculative decoding: the large model checks N
 *    draft tokens at once) and "Chunked Prefill" (a prompt is processed in chunks): several
 *    query tokens of one sequence attend to the paged cache in one call.  The page gives no
 *    formula; read as causal attention of the sequence's last T tokens, already in the
 *    cache: query token tq (position L - T + tq) sees tokens 0 .. L - T + tq.
 *
 * Readings where the pages are silent or inconsistent:
 *  - the printed kernel indexes K with the query head although it receives
 *    num_kv_heads; under grouped-query attention query head hq reads KV head
 *    hq / (num_q_heads / num_kv_heads) (contiguous groups);
 *  - the softmax is the textbook one, computed here in two passes in fp64 with
 *    libm exp; a sequence of length 0 yields an all-zero output row;
 *  - a negative slot in slot_mapping means "no write".
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_E4M3 = 3 };

enum {
  OR_OK = 0,
  OR_ERR_ARG = -1,      /* bad sizes, dtype or null pointer */
  OR_ERR_RANGE = -2,    /* an index (block id, slot, pair) is out of range */
  OR_ERR_NOMEM = -3,
};

/* IEEE-754 binary16 -> double, from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; exponent 0 encodes
 * subnormals m * 2^-24, exponent 31 encodes inf / NaN. */
double oracle_f16_to_f64(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24);
  } else if (e == 31) {
    v = m ? NAN : INFINITY;
  } else {
    v = ldexp((double)(m + 1024), e - 25);
  }
  return sign ? -v : v;
}

/* bfloat16 -> double: a bfloat16 is the upper half of an IEEE binary32. */
double oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* FP8 E4M3 (the OCP "e4m3fn" format) -> double, from the format's definition:
 * 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits; exponent 0 encodes subnormals
 * m * 2^-9; there is no infinity and S.1111.111 is NaN; the largest finite value is 448. */
double oracle_e4m3_to_f64(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xf;
  int m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp((double)(8 + m), e - 10);
  return sign ? -v : v;
}

/* float -> FP8 E4M3: round to nearest, ties to even, saturating to +-448; NaN -> 0x7f.
 * The value is scaled to an integer count of the quantum of its binade (2^-9 below 2^-6,
 * otherwise 2^(exponent - 3)) and rounded with rint (default rounding: ties to even); a
 * count of 16 carries into the next binade, which the code layout does by itself. */
uint8_t oracle_f32_to_e4m3(float x) {
  if (isnan(x)) return 0x7f;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double a = fabs((double)x);
  if (a > 448.0) return sign | 0x7e;
  if (a == 0.0) return sign;
  int E;
  frexp(a, &E);              /* a = f * 2^E, f in [0.5, 1): a's binade is 2^(E-1) */
  int code;
  if (E - 1 < -6) {
    code = (int)rint(a / ldexp(1.0, -9));                 /* subnormal quantum 2^-9 */
  } else {
    int q = (int)rint(a / ldexp(1.0, E - 1 - 3));        /* 8 <= q <= 16 */
    code = ((E - 1 + 7) << 3) + (q - 8);
  }
  return sign | (uint8_t)code;
}

static double load_elem(const void* base, int64_t idx, int dtype) {
  switch (dtype) {
    case OR_F32: return (double)((const float*)base)[idx];
    case OR_F16: return oracle_f16_to_f64(((const uint16_t*)base)[idx]);
    case OR_E4M3: return oracle_e4m3_to_f64(((const uint8_t*)base)[idx]);
    default:     return oracle_bf16_to_f64(((const uint16_t*)base)[idx]);
  }
}

/* copy_blocks: apply the (src, dst) pairs in order; each pair duplicates the
 * whole physical block src into dst, for the K cache and for the V cache. */
int oracle_copy_blocks(uint8_t* k_cache, uint8_t* v_cache, const int32_t* pairs,
                       int64_t num_pairs, int64_t num_blocks, int64_t block_bytes) {
  if (num_pairs < 0 || block_bytes <= 0 || num_blocks <= 0) return OR_ERR_ARG;
  if (num_pairs > 0 && (!k_cache || !v_cache || !pairs)) return OR_ERR_ARG;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return OR_ERR_RANGE;
  }
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
    memmove(k_cache + dst * block_bytes, k_cache + src * block_bytes, (size_t)block_bytes);
    memmove(v_cache + dst * block_bytes, v_cache + src * block_bytes, (size_t)block_bytes);
  }
  return OR_OK;
}

/* swap_blocks: block pairs[p][0] of the source pool is copied to block pairs[p][1] of the
 * destination pool (K and V), for every pair in order -- moving a preempted sequence's blocks
 * to CPU memory and back ("详解vLLM推理引擎架构", scheduler section: the KV cache of
 * low-priority requests is swapped out to CPU memory when GPU memory runs short and
 * swapped back later; --swap-space). */
int oracle_swap_blocks(uint8_t* dst_k, uint8_t* dst_v, const uint8_t* src_k, const uint8_t* src_v,
                       const int32_t* pairs, int64_t num_pairs, int64_t num_src_blocks,
                       int64_t num_dst_blocks, int64_t block_bytes) {
  if (num_pairs < 0 || block_bytes <= 0 || num_src_blocks <= 0 || num_dst_blocks <= 0) return OR_ERR_ARG;
  if (num_pairs > 0 && (!dst_k || !dst_v || !src_k || !src_v || !pairs)) return OR_ERR_ARG;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
    if (s < 0 || s >= num_src_blocks || d < 0 || d >= num_dst_blocks) return OR_ERR_RANGE;
  }
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
    memcpy(dst_k + d * block_bytes, src_k + s * block_bytes, (size_t)block_bytes);
    memcpy(dst_v + d * block_bytes, src_v + s * block_bytes, (size_t)block_bytes);
  }
  return OR_OK;
}

/* reshape_and_cache: token t with slot s >= 0 goes to physical block s / block_size,
 * position s % block_size, for every KV head.  k / v are [num_tokens, num_kv_heads,
 * head_dim] with a row stride of token_stride elements between tokens. */
int oracle_reshape_and_cache(const uint8_t* k, const uint8_t* v, uint8_t* k_cache,
                             uint8_t* v_cache, const int64_t* slot_mapping,
                             int64_t num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int64_t num_blocks, int elem_bytes,
                             int64_t k_token_stride, int64_t v_token_stride) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      num_blocks <= 0 || elem_bytes <= 0)
    return OR_ERR_ARG;
  if (num_tokens > 0 && (!k || !v || !k_cache || !v_cache || !slot_mapping)) return OR_ERR_ARG;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s >= num_blocks * block_size) return OR_ERR_RANGE;
  }
  const int64_t row = (int64_t)head_dim * elem_bytes;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    int64_t blk = s / block_size, pos = s % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((blk * block_size + pos) * num_kv_heads + h) * row;
      memcpy(k_cache + dst, k + (t * k_token_stride + (int64_t)h * head_dim) * elem_bytes, (size_t)row);
      memcpy(v_cache + dst, v + (t * v_token_stride + (int64_t)h * head_dim) * elem_bytes, (size_t)row);
    }
  }
  return OR_OK;
}

/* reshape_and_cache into an FP8 E4M3 cache with per-tensor scales: each element x of the
 * new token (in_dtype f32 / f16 / bf16) is stored as e4m3(x / scale), the division done
 * in fp32 (round to nearest); the slot rule is the one of oracle_reshape_and_cache. */
int oracle_reshape_and_cache_e4m3(const void* k, const void* v, uint8_t* k_cache, uint8_t* v_cache,
                                  const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                                  int head_dim, int block_size, int64_t num_blocks, int in_dtype,
                                  float k_scale, float v_scale, int64_t k_token_stride,
                                  int64_t v_token_stride) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return OR_ERR_ARG;
  if (in_dtype < OR_F32 || in_dtype > OR_BF16) return OR_ERR_ARG;
  if (num_tokens > 0 && (!k || !v || !k_cache || !v_cache || !slot_mapping)) return OR_ERR_ARG;
  for (int64_t t = 0; t < num_tokens; ++t)
    if (slot_mapping[t] >= num_blocks * block_size) return OR_ERR_RANGE;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    int64_t blk = s / block_size, pos = s % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      int64_t dst = ((blk * block_size + pos) * num_kv_heads + h) * head_dim;
      for (int d = 0; d < head_dim; ++d) {
        float xk = (float)load_elem(k, t * k_token_stride + (int64_t)h * head_dim + d, in_dtype);
        float xv = (float)load_elem(v, t * v_token_stride + (int64_t)h * head_dim + d, in_dtype);
        float qk = xk / k_scale;
        float qv = xv / v_scale;
        k_cache[dst + d] = oracle_f32_to_e4m3(qk);
        v_cache[dst + d] = oracle_f32_to_e4m3(qv);
      }
    }
  }
  return OR_OK;
}

typedef struct {
  double* out;
  const void* q;
  int q_dtype;
  const void* k_cache;
  const void* v_cache;
  int kv_dtype;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int num_q_tokens;          /* query tokens per sequence (1 = decode) */
  int num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
  double scale;
  double k_scale, v_scale;   /* dequantisation scales of an E4M3 cache (1 otherwise) */
  int seq_begin, seq_end;
  int status;
} decode_job;

/* Offset (in elements) of element d of token t's KV row for kv head h, reached
 * through the sequence's block table -- the index formula of the kernel on the
 * "vLLM 深度解读" page, with the KV head in place of the query head. */
static int64_t kv_offset(const int32_t* table, int t, int h, int d, int block_size,
                         int num_kv_heads, int head_dim) {
  int64_t phys = table[t / block_size];
  return phys * block_size * num_kv_heads * head_dim + (int64_t)(t % block_size) * num_kv_heads * head_dim +
         (int64_t)h * head_dim + d;
}

static void* decode_worker(void* arg) {
  decode_job* J = (decode_job*)arg;
  const int G = J->num_q_heads / J->num_kv_heads;
  const int D = J->head_dim;
  double* scores = NULL;
  size_t cap = 0;
  for (int i = J->seq_begin; i < J->seq_end; ++i) {
    const int L = J->seq_lens[i];
    const int32_t* table = J->block_tables + (int64_t)i * J->max_blocks_per_seq;
    if ((size_t)L > cap) {
      free(scores);
      cap = (size_t)L;
      scores = (double*)malloc(cap * sizeof(double));
      if (!scores) { J->status = OR_ERR_NOMEM; return NULL; }
    }
    const int T = J->num_q_tokens;
    for (int tq = 0; tq < T; ++tq)
    for (int hq = 0; hq < J->num_q_heads; ++hq) {
      const int h = hq / G;                       /* KV head shared by this query head */
      const int64_t qo = (((int64_t)i * T + tq) * J->num_q_heads + hq) * D;
      double* o = J->out + qo;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (L == 0) continue;
      /* query token tq sits at position L - T + tq and sees the tokens up to its own */
      const int n = L - T + tq + 1;
      /* pass 1: scores and their maximum */
      double m = -INFINITY;
      for (int t = 0; t < n; ++t) {
        double s = 0.0;
        for (int d = 0; d < D; ++d)
          s += load_elem(J->q, qo + d, J->q_dtype) *
               load_elem(J->k_cache, kv_offset(table, t, h, d, J->block_size, J->num_kv_heads, D), J->kv_dtype);
        if (J->kv_dtype == OR_E4M3) s *= J->k_scale;   /* K_t = code * k_scale */
        s *= J->scale;
        scores[t] = s;
        if (s > m) m = s;
      }
      /* pass 2: softmax weights and the weighted sum of V rows */
      double z = 0.0;
      for (int t = 0; t < n; ++t) {
        double w = exp(scores[t] - m);
        z += w;
        for (int d = 0; d < D; ++d)
          o[d] += w * load_elem(J->v_cache, kv_offset(table, t, h, d, J->block_size, J->num_kv_heads, D), J->kv_dtype);
      }
      for (int d = 0; d < D; ++d) o[d] /= z;
      if (J->kv_dtype == OR_E4M3)                      /* V_t = code * v_scale */
        for (int d = 0; d < D; ++d) o[d] *= J->v_scale;
    }
  }
  free(scores);
  return NULL;
}

static int decode_common(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int kv_dtype, const int32_t* block_tables,
                         const int32_t* seq_lens, int num_seqs, int num_q_tokens, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                         int64_t num_blocks, float scale, float k_scale, float v_scale, int num_threads);

/* Decode attention: out[i, hq, :] = softmax_t(scale * q[i,hq,:] . K_t) V_t over the
 * seq_lens[i] tokens of sequence i, K_t / V_t gathered through block_tables.
 * out is fp64 [num_seqs, num_q_heads, head_dim].  Sequences are split across
 * num_threads POSIX threads; each output element is computed by one thread in
 * the same order whatever the thread count. */
int oracle_decode_scaled(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int kv_dtype, const int32_t* block_tables,
                         const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                         float scale, float k_scale, float v_scale, int num_threads);

int oracle_decode(double* out, const void* q, int q_dtype, const void* k_cache,
                  const void* v_cache, int kv_dtype, const int32_t* block_tables,
                  const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                  int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                  float scale, int num_threads) {
  return oracle_decode_scaled(out, q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens,
                              num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                              max_blocks_per_seq, num_blocks, scale, 1.0f, 1.0f, num_threads);
}

/* Decode attention over a cache of any element type; for an E4M3 cache the stored codes are
 * multiplied by k_scale (keys) and v_scale (values) -- the scales are ignored otherwise. */
int oracle_decode_scaled(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int kv_dtype, const int32_t* block_tables,
                         const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                         float scale, float k_scale, float v_scale, int num_threads) {
  return decode_common(out, q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens, num_seqs, 1,
                       num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale,
                       k_scale, v_scale, num_threads);
}

/* Multi-token causal attention over the paged cache: q and out are
 * [num_seqs, num_q_tokens, num_q_heads, head_dim]; query token tq of sequence i is the
 * token at position seq_lens[i] - num_q_tokens + tq and attends to the tokens 0 .. that
 * position.  A sequence must hold 0 or at least num_q_tokens tokens. */
int oracle_decode_multi(double* out, const void* q, int q_dtype, const void* k_cache,
                        const void* v_cache, int kv_dtype, const int32_t* block_tables,
                        const int32_t* seq_lens, int num_seqs, int num_q_tokens, int num_q_heads,
                        int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                        int64_t num_blocks, float scale, int num_threads) {
  return decode_common(out, q, q_dtype, k_cache, v_cache, kv_dtype, block_tables, seq_lens, num_seqs,
                       num_q_tokens, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                       num_blocks, scale, 1.0f, 1.0f, num_threads);
}

static int decode_common(double* out, const void* q, int q_dtype, const void* k_cache,
                         const void* v_cache, int kv_dtype, const int32_t* block_tables,
                         const int32_t* seq_lens, int num_seqs, int num_q_tokens, int num_q_heads,
                         int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                         int64_t num_blocks, float scale, float k_scale, float v_scale, int num_threads) {
  if (num_seqs < 0 || num_q_tokens <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || max_blocks_per_seq < 0 || num_blocks <= 0)
    return OR_ERR_ARG;
  if (num_q_heads % num_kv_heads) return OR_ERR_ARG;
  if (q_dtype < OR_F32 || q_dtype > OR_BF16 || kv_dtype < OR_F32 || kv_dtype > OR_E4M3) return OR_ERR_ARG;
  if (num_seqs == 0) return OR_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return OR_ERR_ARG;
  /* every block the definition will touch must exist */
  for (int i = 0; i < num_seqs; ++i) {
    int L = seq_lens[i];
    if (L < 0 || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) return OR_ERR_RANGE;
    if (L > 0 && L < num_q_tokens) return OR_ERR_RANGE;
    int nb = (L + block_size - 1) / block_size;
    for (int b = 0; b < nb; ++b) {
      int32_t p = block_tables[(int64_t)i * max_blocks_per_seq + b];
      if (p < 0 || p >= num_blocks) return OR_ERR_RANGE;
    }
  }
  if (num_threads < 1) num_threads = 1;
  if (num_threads > num_seqs) num_threads = num_seqs;
  decode_job* jobs = (decode_job*)calloc((size_t)num_threads, sizeof(decode_job));
  pthread_t* tids = (pthread_t*)calloc((size_t)num_threads, sizeof(pthread_t));
  if (!jobs || !tids) { free(jobs); free(tids); return OR_ERR_NOMEM; }
  for (int w = 0; w < num_threads; ++w) {
    decode_job* J = &jobs[w];
    J->out = out; J->q = q; J->q_dtype = q_dtype; J->k_cache = k_cache; J->v_cache = v_cache;
    J->kv_dtype = kv_dtype; J->block_tables = block_tables; J->seq_lens = seq_lens;
    J->num_q_tokens = num_q_tokens;
    J->num_q_heads = num_q_heads; J->num_kv_heads = num_kv_heads; J->head_dim = head_dim;
    J->block_size = block_size; J->max_blocks_per_seq = max_blocks_per_seq;
    J->scale = (double)scale;
    J->k_scale = (double)k_scale;
    J->v_scale = (double)v_scale;
    J->seq_begin = (int)((int64_t)num_seqs * w / num_threads);
    J->seq_end = (int)((int64_t)num_seqs * (w + 1) / num_threads);
    J->status = OR_OK;
  }
  int status = OR_OK;
  int started = 0;
  for (int w = 1; w < num_threads; ++w) {
    if (pthread_create(&tids[w], NULL, decode_worker, &jobs[w]) != 0) break;
    started = w;
  }
  decode_worker(&jobs[0]);
  for (int w = 1; w <= started; ++w) pthread_join(tids[w], NULL);
  /* any range not covered by a started thread runs here */
  for (int w = started + 1; w < num_threads; ++w) decode_worker(&jobs[w]);
  for (int w = 0; w < num_threads; ++w)
    if (jobs[w].status != OR_OK) status = jobs[w].status;
  free(jobs);
  free(tids);
  return status;
}
