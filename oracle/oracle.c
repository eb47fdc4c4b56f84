/*
 * CPU oracle for paged-attention decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline do.  It shares no code, header, table or constant with the CUDA
 * path.
 *
 * Sources (the three web pages on vLLM / PagedAttention):
 *   [KV]    "vLLM 推理加速原理详解：大模型服务吞吐量为何能提升 10 倍",
 *           section "真正吃显存的是 KV Cache，不是模型权重" — the worked
 *           KV-cache size formula 2 x seq_len x layers x heads x head_dim x bytes.
 *   [PA]    same page, section "PagedAttention：把操作系统的虚拟内存搬进 GPU" —
 *           the cache lives in fixed-size physical blocks; a per-sequence
 *           block table maps logically contiguous positions to physically
 *           scattered blocks; the kernel must read K/V correctly from
 *           non-contiguous blocks.  Paging only changes addresses, so the
 *           result is plain attention over the sequence's own tokens.
 *   [FP8]   same page, section "vLLM 也不是银弹：真实部署中的坑", third pitfall —
 *           FP8 KV cache as the remedy for long-context memory pressure.  The
 *           page fixes neither the FP8 format nor the scale granularity; the
 *           reading taken is OCP FP8 E4M3 ("fn": bias 7, no infinities,
 *           S.1111.111 = NaN, max 448) with one fp32 scale per (block, kv head).
 *
 * Everything here is written from those definitions and from the IEEE 754
 * binary16 / bfloat16 formats: decode each stored element exactly to double,
 * rebuild each sequence's contiguous K and V from its block table, and run
 * textbook softmax attention in double precision.
 *
 * Pool layout (a choice of this library, which the pages leave open): per
 * layer, K and V are each [num_blocks][kv_heads][block_size][head_dim]
 * elements, row-major.  Element (blk, h, off, d) sits at
 *   ((blk * kv_heads + h) * block_size + off) * head_dim + d.
 * FP8 scales are [num_blocks][kv_heads] fp32, separately for K and V; the
 * stored code times the scale is the value.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F16 = 0, OR_BF16 = 1, OR_E4M3 = 2, OR_F32 = 3 };

/* ---------------------------------------------------------------- formats */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 mantissa bits. */
double oracle_f16_to_double(uint16_t h) {
  int s = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)m, -24); /* subnormal: m/1024 * 2^-14 */
  } else if (e == 31) {
    v = (m == 0) ? INFINITY : NAN;
  } else {
    v = ldexp(1.0 + (double)m / 1024.0, e - 15);
  }
  return s ? -v : v;
}

/* bfloat16 is the upper half of an IEEE 754 binary32. */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t bits = (uint32_t)b << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there
 * is no infinity, so S.1111.110 = 448 is the largest magnitude. */
double oracle_e4m3_to_double(uint8_t c) {
  int s = (c >> 7) & 1;
  int e = (c >> 3) & 0xf;
  int m = c & 0x7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) {
    v = ldexp((double)m, -9);
  } else {
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  }
  return s ? -v : v;
}

/* Round a non-negative double to the nearest integer, ties to even. */
static double round_half_even(double r) {
  double f = floor(r);
  double d = r - f;
  if (d > 0.5) return f + 1.0;
  if (d < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* float -> E4M3 with round-to-nearest-even and saturation to the largest
 * finite magnitude (448).  NaN maps to the NaN code 0x7f.  Steps: take |x|,
 * find the quantum of its binade (2^(E-3) for normals, 2^-9 below the
 * smallest normal 2^-6), round |x|/quantum to an integer with ties to even,
 * clamp to 448, then write sign, exponent and mantissa fields. */
uint8_t oracle_e4m3_from_float(float x) {
  if (isnan(x)) return 0x7f;
  int s = signbit(x) ? 1 : 0;
  double a = fabs((double)x);
  double v;
  if (isinf(a)) {
    v = 448.0;
  } else if (a < ldexp(1.0, -6)) {
    v = round_half_even(a / ldexp(1.0, -9)) * ldexp(1.0, -9);
  } else {
    int E;
    (void)frexp(a, &E); /* a = f * 2^E with f in [0.5, 1) */
    E -= 1;             /* a in [2^E, 2^(E+1)) */
    double q = ldexp(1.0, E - 3);
    v = round_half_even(a / q) * q;
  }
  if (v > 448.0) v = 448.0;
  uint8_t code;
  if (v == 0.0) {
    code = 0;
  } else if (v < ldexp(1.0, -6)) {
    code = (uint8_t)(v / ldexp(1.0, -9)); /* subnormal: exponent field 0 */
  } else {
    int E;
    double f = frexp(v, &E); /* v = f * 2^E, f in [0.5,1) */
    int e = (E - 1) + 7;
    int m = (int)((f * 2.0 - 1.0) * 8.0);
    code = (uint8_t)((e << 3) | m);
  }
  return (uint8_t)(code | (s << 7));
}

/* Element-wise helpers over arrays, so Python can call the codecs in bulk. */
void oracle_decode_array(const void* src, int dtype, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    if (dtype == OR_F16) out[i] = oracle_f16_to_double(((const uint16_t*)src)[i]);
    else if (dtype == OR_BF16) out[i] = oracle_bf16_to_double(((const uint16_t*)src)[i]);
    else if (dtype == OR_E4M3) out[i] = oracle_e4m3_to_double(((const uint8_t*)src)[i]);
    else out[i] = (double)((const float*)src)[i];
  }
}

void oracle_e4m3_encode_array(const float* src, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_from_float(src[i]);
}

/* [KV]: bytes of K and V for one request,
 *   2 (K and V) x seq_len x layers x heads x head_dim x bytes per element. */
int64_t oracle_kv_cache_bytes(int64_t seq_len, int64_t layers, int64_t heads,
                              int64_t head_dim, int64_t elem_bytes) {
  return 2 * seq_len * layers * heads * head_dim * elem_bytes;
}

/* ------------------------------------------------------------- attention */

static double elem(const void* pool, int dtype, int64_t idx) {
  if (dtype == OR_F16) return oracle_f16_to_double(((const uint16_t*)pool)[idx]);
  if (dtype == OR_BF16) return oracle_bf16_to_double(((const uint16_t*)pool)[idx]);
  return oracle_e4m3_to_double(((const uint8_t*)pool)[idx]);
}

typedef struct {
  const void* k_pool;
  const void* v_pool;
  int kv_dtype;
  const float* k_scale; /* [num_blocks][kv_heads], FP8 only */
  const float* v_scale;
  int num_blocks, kv_heads, block_size, head_dim;
  const void* q; /* [batch][num_q_heads][head_dim] */
  int q_dtype;
  int num_q_heads;
  const int32_t* block_tables; /* [batch][max_blocks] */
  int max_blocks;
  const int32_t* context_lens; /* [batch] */
  int batch;
  double scale;
} oracle_decode_args;

/* Rebuild the contiguous K (or V) rows of sequence s, kv head kvh, from the
 * block table ([PA]): token t lives in physical block bt[s][t / block_size]
 * at offset t % block_size.  Values are decoded exactly and, for FP8, times
 * the (block, head) scale.  Returns 0, or -1 on a block id outside the pool. */
static int gather_from(const oracle_decode_args* a, const void* pool, const float* scales,
                       int s, int kvh, int t_first, int n, double* rows) {
  int D = a->head_dim, bs = a->block_size;
  for (int t = t_first; t < n; ++t) {
    int32_t blk = a->block_tables[(int64_t)s * a->max_blocks + t / bs];
    if (blk < 0 || blk >= a->num_blocks) return -1;
    int off = t % bs;
    int64_t base = (((int64_t)blk * a->kv_heads + kvh) * bs + off) * D;
    double sc = 1.0;
    if (a->kv_dtype == OR_E4M3) sc = (double)scales[(int64_t)blk * a->kv_heads + kvh];
    for (int d = 0; d < D; ++d) rows[(int64_t)t * D + d] = elem(pool, a->kv_dtype, base + d) * sc;
  }
  return 0;
}

static int gather(const oracle_decode_args* a, const void* pool, const float* scales,
                  int s, int kvh, int n, double* rows) {
  return gather_from(a, pool, scales, s, kvh, 0, n, rows);
}

static double qval(const oracle_decode_args* a, int s, int h, int d) {
  int64_t idx = ((int64_t)s * a->num_q_heads + h) * a->head_dim + d;
  if (a->q_dtype == OR_F16) return oracle_f16_to_double(((const uint16_t*)a->q)[idx]);
  if (a->q_dtype == OR_BF16) return oracle_bf16_to_double(((const uint16_t*)a->q)[idx]);
  return (double)((const float*)a->q)[idx];
}

/* Logits z_t = scale * q . K_t over tokens [t0, t1) of (s, h). */
static void logits(const oracle_decode_args* a, int s, int h, const double* K,
                   int t0, int t1, double* z) {
  int D = a->head_dim;
  for (int t = t0; t < t1; ++t) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += qval(a, s, h, d) * K[(int64_t)t * D + d];
    z[t - t0] = a->scale * acc;
  }
}

/* One (sequence, query head): out = sum_t softmax(z)_t V_t, all in double.
 * GQA reading: query head h uses kv head h / (num_q_heads / kv_heads).
 * context_len <= 0 gives an all-zero output.  Returns -1 on a bad block id. */
static int decode_one(const oracle_decode_args* a, int s, int h, double* out) {
  int D = a->head_dim;
  int g = a->num_q_heads / a->kv_heads;
  int kvh = h / g;
  int n = a->context_lens[s];
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  if (n <= 0) return 0;
  double* K = (double*)malloc(sizeof(double) * (size_t)n * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)n * D);
  double* z = (double*)malloc(sizeof(double) * (size_t)n);
  int rc = 0;
  if (!K || !V || !z) { rc = -2; goto done; }
  if (gather(a, a->k_pool, a->k_scale, s, kvh, n, K) || gather(a, a->v_pool, a->v_scale, s, kvh, n, V)) {
    rc = -1;
    goto done;
  }
  logits(a, s, h, K, 0, n, z);
  double m = -INFINITY;
  for (int t = 0; t < n; ++t) if (z[t] > m) m = z[t];
  double l = 0.0;
  for (int t = 0; t < n; ++t) {
    double w = exp(z[t] - m);
    l += w;
    for (int d = 0; d < D; ++d) out[d] += w * V[(int64_t)t * D + d];
  }
  for (int d = 0; d < D; ++d) out[d] /= l;
done:
  free(K);
  free(V);
  free(z);
  return rc;
}

/* Decode every (sequence, query head); out is [batch][num_q_heads][head_dim]
 * doubles.  Parallel over (sequence, head) pairs only; each pair is computed
 * by the plain serial formula above.  Returns 0, -1 (bad block id), -2 (OOM). */
int oracle_paged_decode(const void* k_pool, const void* v_pool, int kv_dtype,
                        const float* k_scale, const float* v_scale, int num_blocks,
                        int kv_heads, int block_size, int head_dim, const void* q,
                        int q_dtype, int num_q_heads, const int32_t* block_tables,
                        int max_blocks, const int32_t* context_lens, int batch,
                        double scale, double* out) {
  oracle_decode_args a = {k_pool, v_pool, kv_dtype, k_scale, v_scale, num_blocks, kv_heads,
                          block_size, head_dim, q, q_dtype, num_q_heads, block_tables,
                          max_blocks, context_lens, batch, scale};
  int rc = 0;
  int64_t pairs = (int64_t)batch * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
  for (int64_t i = 0; i < pairs; ++i) {
    int s = (int)(i / num_q_heads), h = (int)(i % num_q_heads);
    int r = decode_one(&a, s, h, out + i * head_dim);
    if (r < rc) rc = r;
  }
  return rc;
}

/* Split-K partials (the context-partition step of the decode): partition p
 * covers tokens [p*P, min((p+1)*P, n)).  For each (s, h, p):
 *   m_p = max_t z_t,  l_p = sum_t exp(z_t - m_p),  o_p = sum_t exp(z_t - m_p) V_t.
 * An empty partition has m_p = -inf, l_p = 0, o_p = 0.  Outputs are
 * [batch][num_q_heads][num_parts] (x head_dim for o). */
int oracle_paged_decode_partials(const void* k_pool, const void* v_pool, int kv_dtype,
                                 const float* k_scale, const float* v_scale,
                                 int num_blocks, int kv_heads, int block_size,
                                 int head_dim, const void* q, int q_dtype,
                                 int num_q_heads, const int32_t* block_tables,
                                 int max_blocks, const int32_t* context_lens, int batch,
                                 double scale, int partition_tokens, int num_parts,
                                 double* o_part, double* m_part, double* l_part) {
  oracle_decode_args a = {k_pool, v_pool, kv_dtype, k_scale, v_scale, num_blocks, kv_heads,
                          block_size, head_dim, q, q_dtype, num_q_heads, block_tables,
                          max_blocks, context_lens, batch, scale};
  int D = head_dim;
  int g = num_q_heads / kv_heads;
  int rc = 0;
  int64_t pairs = (int64_t)batch * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
  for (int64_t i = 0; i < pairs; ++i) {
    int s = (int)(i / num_q_heads), h = (int)(i % num_q_heads);
    int n = context_lens[s];
    if (n < 0) n = 0;
    double* K = (double*)malloc(sizeof(double) * ((size_t)n * D + 1));
    double* V = (double*)malloc(sizeof(double) * ((size_t)n * D + 1));
    double* z = (double*)malloc(sizeof(double) * ((size_t)partition_tokens + 1));
    if (!K || !V || !z) { rc = -2; free(K); free(V); free(z); continue; }
    int bad = gather(&a, k_pool, k_scale, s, h / g, n, K) || gather(&a, v_pool, v_scale, s, h / g, n, V);
    if (bad) rc = -1;
    for (int p = 0; p < num_parts; ++p) {
      double* o = o_part + (i * num_parts + p) * D;
      double m = -INFINITY, l = 0.0;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      int t0 = p * partition_tokens;
      int t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;
      if (t0 < t1 && !bad) {
        logits(&a, s, h, K, t0, t1, z);
        for (int t = t0; t < t1; ++t) if (z[t - t0] > m) m = z[t - t0];
        for (int t = t0; t < t1; ++t) {
          double w = exp(z[t - t0] - m);
          l += w;
          for (int d = 0; d < D; ++d) o[d] += w * V[(int64_t)t * D + d];
        }
      }
      m_part[i * num_parts + p] = m;
      l_part[i * num_parts + p] = l;
    }
    free(K);
    free(V);
    free(z);
  }
  return rc;
}

/* Log-sum-exp merge of partials (the reduce step):
 *   m = max_p m_p,  l = sum_p l_p exp(m_p - m),  out = sum_p o_p exp(m_p - m) / l.
 * All partitions empty (m = -inf) gives zeros.  rows = number of (s, h)
 * pairs; o_part is [rows][num_parts][D]. */
void oracle_lse_merge(int64_t rows, int num_parts, int head_dim, const double* o_part,
                      const double* m_part, const double* l_part, double* out) {
  for (int64_t i = 0; i < rows; ++i) {
    double m = -INFINITY;
    for (int p = 0; p < num_parts; ++p)
      if (m_part[i * num_parts + p] > m) m = m_part[i * num_parts + p];
    double* o = out + i * head_dim;
    for (int d = 0; d < head_dim; ++d) o[d] = 0.0;
    if (m == -INFINITY) continue;
    double l = 0.0;
    for (int p = 0; p < num_parts; ++p) {
      double mp = m_part[i * num_parts + p];
      if (mp == -INFINITY) continue;
      double w = exp(mp - m);
      l += l_part[i * num_parts + p] * w;
      for (int d = 0; d < head_dim; ++d) o[d] += o_part[(i * num_parts + p) * head_dim + d] * w;
    }
    for (int d = 0; d < head_dim; ++d) o[d] /= l;
  }
}

/* ------------------------------------------------ multi-token attention */

/* Query element d of head h in packed row `row` of a [rows][num_q_heads]
 * [head_dim] array (multi-token layout: one row per new token). */
static double qrow_val(const oracle_decode_args* a, int64_t row, int h, int d) {
  int64_t idx = (row * a->num_q_heads + h) * a->head_dim + d;
  if (a->q_dtype == OR_F16) return oracle_f16_to_double(((const uint16_t*)a->q)[idx]);
  if (a->q_dtype == OR_BF16) return oracle_bf16_to_double(((const uint16_t*)a->q)[idx]);
  return (double)((const float*)a->q)[idx];
}

/* Multi-token attention over the paged cache: the step that processes a
 * prompt (or a chunk of one, or several drafted tokens) before decoding
 * continues ([PA] plus the time-to-first-token discussion of the same page's
 * "连续批处理" section; the pages describe no kernel for it).  Reading taken:
 * sequence s holds n = context_lens[s] tokens in the cache, the last
 * q_len = cu_q[s+1] - cu_q[s] of which are its new tokens (already written);
 * new token i sits at position p = n - q_len + i and attends to the cached
 * positions t with lo <= t <= p (causal), where lo = 0 without a window and
 * lo = max(0, p - window + 1) with a sliding window of `window` tokens (the
 * long-context remedy named in the pitfalls section).  q and out are
 * [cu_q[batch]][num_q_heads][head_dim]; row cu_q[s] + i belongs to token i
 * of s.  Returns 0, -1 (bad block id), -2 (OOM), -3 (q_len > n, q_len < 0,
 * or a negative window). */
static int prefill_one(const oracle_decode_args* a, const int32_t* cu_q, int window, int s,
                       int h, double* out) {
  int D = a->head_dim;
  int g = a->num_q_heads / a->kv_heads;
  int n = a->context_lens[s];
  int q_len = cu_q[s + 1] - cu_q[s];
  if (q_len < 0 || q_len > n || window < 0) return -3;
  if (q_len == 0) return 0;
  double* K = (double*)malloc(sizeof(double) * (size_t)n * D);
  double* V = (double*)malloc(sizeof(double) * (size_t)n * D);
  double* z = (double*)malloc(sizeof(double) * (size_t)n);
  int rc = 0;
  if (!K || !V || !z) { rc = -2; goto done; }
  /* positions before the first row's window are never read (with a sliding
   * window their blocks may already be released) */
  int t_first = (window > 0 && n - q_len - window + 1 > 0) ? n - q_len - window + 1 : 0;
  if (gather_from(a, a->k_pool, a->k_scale, s, h / g, t_first, n, K) ||
      gather_from(a, a->v_pool, a->v_scale, s, h / g, t_first, n, V)) {
    rc = -1;
    goto done;
  }
  for (int i = 0; i < q_len; ++i) {
    int64_t row = (int64_t)cu_q[s] + i;
    int p = n - q_len + i;
    int lo = (window > 0 && p - window + 1 > 0) ? p - window + 1 : 0;
    double* o = out + (row * a->num_q_heads + h) * D;
    double m = -INFINITY;
    for (int t = lo; t <= p; ++t) {
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += qrow_val(a, row, h, d) * K[(int64_t)t * D + d];
      z[t] = a->scale * acc;
      if (z[t] > m) m = z[t];
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int t = lo; t <= p; ++t) {
      double w = exp(z[t] - m);
      l += w;
      for (int d = 0; d < D; ++d) o[d] += w * V[(int64_t)t * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
  }
done:
  free(K);
  free(V);
  free(z);
  return rc;
}

int oracle_paged_prefill(const void* k_pool, const void* v_pool, int kv_dtype,
                         const float* k_scale, const float* v_scale, int num_blocks,
                         int kv_heads, int block_size, int head_dim, const void* q, int q_dtype,
                         int num_q_heads, const int32_t* cu_q, const int32_t* block_tables,
                         int max_blocks, const int32_t* context_lens, int batch, double scale,
                         int window, double* out) {
  oracle_decode_args a = {k_pool, v_pool, kv_dtype, k_scale, v_scale, num_blocks, kv_heads,
                          block_size, head_dim, q, q_dtype, num_q_heads, block_tables,
                          max_blocks, context_lens, batch, scale};
  int rc = 0;
  int64_t pairs = (int64_t)batch * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1) reduction(min : rc)
  for (int64_t i = 0; i < pairs; ++i) {
    int r = prefill_one(&a, cu_q, window, (int)(i / num_q_heads), (int)(i % num_q_heads), out);
    if (r < rc) rc = r;
  }
  return rc;
}
