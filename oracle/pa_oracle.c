/*
 * pa_oracle.c -- plain, slow, obviously correct CPU oracle for paged-KV decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or
 * constant with the CUDA path and includes nothing from it.
 *
 * Sources (page title, then the passage):
 *   [P1] "vLLM推理引擎PagedAttention原理与性能优化实战"
 *        sec 2.2 (16-token blocks, per-request block table), sec 3.2 (copy-on-write),
 *        sec 5.2 (FP8 KV cache), sec 6 (chunked prefill).
 *   [P2] "vLLM 是什么：PagedAttention 让大模型推理快 2-4 倍，还能撑起更长思维链"
 *        sec 2 (logically contiguous, physically scattered blocks; a new block only
 *        when the current one is full), sec 5 misconception 3 (block swapping to
 *        CPU memory when GPU memory runs out).
 *   [P3] "vLLM 推理优化技术深度调研报告"
 *        dim. 1 sec 1 misconception 2 (attention is the standard Softmax(QK^T/sqrt d)V),
 *        sec 3 formula 3 (logical -> physical page mapping through BlockTable[s]),
 *        sec 3 formula 4 (K_paged, V_paged gathered from physical pages, then standard
 *        attention), sec 2 memory flow (KV block request -> table registration ->
 *        attention read -> release/reuse).
 *
 * Readings where the pages are silent or garbled (the formula bodies of [P3] sec 3
 * were lost; only captions and symbol definitions survive):
 *   - mapping: token l of sequence s lives in physical block BlockTable[s][l / P] at
 *     in-block offset l % P (P = block size);
 *   - pool layout: one K pool and one V pool per layer, [num_blocks][kv_heads][P][D];
 *   - GQA: query head h reads kv head h / (H / H_kv);
 *   - FP8 is OCP E4M3 (bias 7, no infinities, S.1111.111 = NaN) with one fp32 scale
 *     per cache tensor: stored code = RNE_satfinite(float(x) / scale) with the
 *     division done in IEEE fp32, value read back = decode(code) * scale;
 *   - a slot < 0 is padding and is skipped; seq_len 0 yields a zero output.
 *
 * Every floating-point step of the attention is fp64 and textbook: an explicit
 * gather into contiguous K, V arrays, then scores, max, exponentials, sum and the
 * weighted sum of V rows.  No online softmax, no tiling, no partitions (except in
 * oracle_decode_partition_stats, which applies the same textbook definition to each
 * token range separately, and oracle_lse_merge, which merges such ranges).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* dtype codes understood by this file (independent of any other header) */
enum { ORC_F16 = 0, ORC_BF16 = 1, ORC_F32 = 2, ORC_E4M3 = 3 };

static int elt_size(int dt) {
  switch (dt) {
    case ORC_F16: return 2;
    case ORC_BF16: return 2;
    case ORC_F32: return 4;
    case ORC_E4M3: return 1;
    default: return 0;
  }
}

/* ---------------------------------------------------------------------------
 * Number formats, decoded from their definitions.
 * ------------------------------------------------------------------------- */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h) {
  int s = h >> 15, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24); /* subnormal: (m / 2^10) * 2^-14 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25); /* (1 + m/2^10) * 2^(e-15) */
  return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double orc_bf16_to_f64(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* OCP OFP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 * exponent 1111 with mantissa 111 is NaN; exponent 0000 is subnormal. */
double orc_e4m3_to_f64(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = ldexp((double)m, -9); /* (m / 8) * 2^-6 */
  else
    v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
  return s ? -v : v;
}

/* Round a float to E4M3: nearest representable value, ties to the even code,
 * magnitudes at or above the largest finite value (448) saturate to it, NaN maps
 * to 0x7F.  The 127 non-negative finite codes 0x00..0x7E are increasing in value,
 * so the two candidates are the largest code whose value is <= |y| and the next
 * one; the sign bit is carried separately. */
uint8_t orc_f32_to_e4m3_satfinite(float y) {
  if (isnan(y)) return 0x7F;
  uint8_t sign = signbit(y) ? 0x80 : 0x00;
  double a = fabs((double)y);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  int lo = 0, hi = 0x7E; /* invariant: value(lo) <= a < value(hi) */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (orc_e4m3_to_f64((uint8_t)mid) <= a)
      lo = mid;
    else
      hi = mid;
  }
  double dl = a - orc_e4m3_to_f64((uint8_t)lo);
  double dh = orc_e4m3_to_f64((uint8_t)hi) - a;
  int c;
  if (dl < dh)
    c = lo;
  else if (dh < dl)
    c = hi;
  else
    c = (lo & 1) ? hi : lo; /* tie: the even code */
  return (uint8_t)(sign | c);
}

/* Batch form of the rounding above. */
void oracle_f32_to_e4m3(uint8_t* dst, const float* src, int64_t n) {
  for (int64_t i = 0; i < n; ++i) dst[i] = orc_f32_to_e4m3_satfinite(src[i]);
}

static double load_elt(const void* base, int64_t idx, int dt) {
  switch (dt) {
    case ORC_F16: return orc_f16_to_f64(((const uint16_t*)base)[idx]);
    case ORC_BF16: return orc_bf16_to_f64(((const uint16_t*)base)[idx]);
    case ORC_F32: return (double)((const float*)base)[idx];
    case ORC_E4M3: return orc_e4m3_to_f64(((const uint8_t*)base)[idx]);
    default: return NAN;
  }
}

/* float value of a 16-bit source element, exactly (both formats embed in fp32) */
static float load_src_f32(const void* base, int64_t idx, int dt) {
  return (float)load_elt(base, idx, dt);
}

/* ---------------------------------------------------------------------------
 * reshape_and_cache: write each new token's K and V rows into the slot the
 * slot mapping names ([P3] sec 2 memory flow; [P2] sec 2 on-demand blocks).
 * slot s -> block s / P, offset s % P.  Same-format copies are bit copies;
 * an E4M3 cache stores RNE_satfinite(float(x) / scale).
 * Returns 0, or -1 for an invalid argument / out-of-range slot.
 * ------------------------------------------------------------------------- */
int oracle_reshape_and_cache(const void* key, const void* value, void* key_cache,
                             void* value_cache, const int64_t* slot_mapping,
                             int64_t num_tokens, int num_kv_heads, int head_dim,
                             int block_size, int64_t num_blocks, int src_dtype,
                             int cache_dtype, float k_scale, float v_scale) {
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return -1;
  int es = elt_size(src_dtype), ec = elt_size(cache_dtype);
  if (!es || !ec) return -1;
  int quant = (cache_dtype == ORC_E4M3);
  if (!quant && cache_dtype != src_dtype) return -1;
  if (quant && src_dtype != ORC_F16 && src_dtype != ORC_BF16) return -1;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue; /* padding token */
    if (s >= num_blocks * (int64_t)block_size) return -1;
    int64_t b = s / block_size, o = s % block_size;
    for (int h = 0; h < num_kv_heads; ++h) {
      int64_t src_row = (t * num_kv_heads + h) * (int64_t)head_dim;
      int64_t dst_row = ((b * num_kv_heads + h) * block_size + o) * (int64_t)head_dim;
      if (!quant) {
        memcpy((char*)key_cache + dst_row * ec, (const char*)key + src_row * es,
               (size_t)head_dim * es);
        memcpy((char*)value_cache + dst_row * ec, (const char*)value + src_row * es,
               (size_t)head_dim * es);
      } else {
        for (int d = 0; d < head_dim; ++d) {
          float xk = load_src_f32(key, src_row + d, src_dtype);
          float xv = load_src_f32(value, src_row + d, src_dtype);
          float yk = xk / k_scale; /* IEEE fp32 division */
          float yv = xv / v_scale;
          ((uint8_t*)key_cache)[dst_row + d] = orc_f32_to_e4m3_satfinite(yk);
          ((uint8_t*)value_cache)[dst_row + d] = orc_f32_to_e4m3_satfinite(yv);
        }
      }
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * copy_blocks: the copy step of copy-on-write ([P1] sec 3.2): for each (src, dst)
 * pair in order, the whole src block is copied to dst, K and V, every layer.
 * ------------------------------------------------------------------------- */
int oracle_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                       const int64_t* block_mapping, int64_t num_pairs, int64_t block_bytes) {
  if (num_layers < 0 || num_pairs < 0 || block_bytes <= 0) return -1;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || dst < 0) return -1;
    for (int l = 0; l < num_layers; ++l) {
      memcpy((char*)key_caches[l] + dst * block_bytes, (char*)key_caches[l] + src * block_bytes,
             (size_t)block_bytes);
      memcpy((char*)value_caches[l] + dst * block_bytes,
             (char*)value_caches[l] + src * block_bytes, (size_t)block_bytes);
    }
  }
  return 0;
}

/* ---------------------------------------------------------------------------
 * swap_blocks: whole blocks moved between two pools (device <-> host memory when
 * GPU memory runs out: [P2] sec 5 misconception 3, block swapping to CPU memory):
 * for each (src, dst) pair in order, block src of the source pool is copied to
 * block dst of the destination pool, K and V, every layer.
 * ------------------------------------------------------------------------- */
int oracle_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                       void* const* src_key_caches, void* const* src_value_caches,
                       int num_layers, const int64_t* block_mapping, int64_t num_pairs,
                       int64_t block_bytes, int64_t src_num_blocks, int64_t dst_num_blocks) {
  if (num_layers < 0 || num_pairs < 0 || block_bytes <= 0) return -1;
  for (int64_t p = 0; p < num_pairs; ++p) {
    int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return -1;
    for (int l = 0; l < num_layers; ++l) {
      memcpy((char*)dst_key_caches[l] + dst * block_bytes,
             (const char*)src_key_caches[l] + src * block_bytes, (size_t)block_bytes);
      memcpy((char*)dst_value_caches[l] + dst * block_bytes,
             (const char*)src_value_caches[l] + src * block_bytes, (size_t)block_bytes);
    }
  }
  return 0;
}

/* Explicit gather ([P3] sec 3 formula 4, mapping of formula 3): rows 0..L-1 of
 * sequence `seq`, kv head `kvh`, into contiguous fp64 arrays, dequantised. */
static int gather_kv(double* K, double* V, const void* key_cache, const void* value_cache,
                     const int32_t* table, int L, int kvh, int num_kv_heads, int head_dim,
                     int block_size, int64_t num_blocks, int cache_dtype, double k_scale,
                     double v_scale) {
  int quant = (cache_dtype == ORC_E4M3);
  for (int l = 0; l < L; ++l) {
    int64_t phys = table[l / block_size];
    int64_t off = l % block_size;
    if (phys < 0 || phys >= num_blocks) return -1;
    int64_t row = ((phys * num_kv_heads + kvh) * block_size + off) * (int64_t)head_dim;
    for (int d = 0; d < head_dim; ++d) {
      double k = load_elt(key_cache, row + d, cache_dtype);
      double v = load_elt(value_cache, row + d, cache_dtype);
      if (quant) {
        k *= k_scale;
        v *= v_scale;
      }
      K[(int64_t)l * head_dim + d] = k;
      V[(int64_t)l * head_dim + d] = v;
    }
  }
  return 0;
}

/* Textbook attention of one query row over contiguous K, V rows [lo, hi):
 * s_j = scale * q.k_j ; m = max s ; p_j = exp(s_j - m) ; out = sum p_j v_j / sum p_j.
 * Optionally returns m and the sum of p (for the partition statistics). */
static void attend_rows(double* out, double* m_out, double* l_out, const double* q,
                        const double* K, const double* V, int lo, int hi, int head_dim,
                        double scale, double* scratch) {
  if (hi <= lo) {
    for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (m_out) *m_out = -INFINITY;
    if (l_out) *l_out = 0.0;
    return;
  }
  double m = -INFINITY;
  for (int j = lo; j < hi; ++j) {
    double s = 0.0;
    for (int d = 0; d < head_dim; ++d) s += q[d] * K[(int64_t)j * head_dim + d];
    s *= scale;
    scratch[j - lo] = s;
    if (s > m) m = s;
  }
  double sum = 0.0;
  for (int j = lo; j < hi; ++j) {
    double p = exp(scratch[j - lo] - m);
    scratch[j - lo] = p;
    sum += p;
  }
  for (int d = 0; d < head_dim; ++d) {
    double acc = 0.0;
    for (int j = lo; j < hi; ++j) acc += scratch[j - lo] * V[(int64_t)j * head_dim + d];
    out[d] = acc / sum;
  }
  if (m_out) *m_out = m;
  if (l_out) *l_out = sum;
}

/* ---------------------------------------------------------------------------
 * Decode attention ([P3] dim.1 misconception 2 and sec 3 formula 4): for each
 * sequence i and query head h, out[i][h] = softmax(scale * q K_i^T) V_i where
 * K_i, V_i are gathered through block_tables[i] for kv head h / (H / H_kv).
 * out is fp64 [num_seqs][num_heads][head_dim].  Returns 0, or -1 on bad input.
 * ------------------------------------------------------------------------- */
int oracle_paged_attention_decode(double* out, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                                  int num_heads, int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, double scale, int q_dtype, int cache_dtype,
                                  double k_scale, double v_scale) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return -1;
  if (num_heads % num_kv_heads != 0) return -1;
  if (!elt_size(q_dtype) || !elt_size(cache_dtype)) return -1;
  int group = num_heads / num_kv_heads;
  int failed = 0;
  int64_t npairs = (int64_t)num_seqs * num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (int64_t pr = 0; pr < npairs; ++pr) {
    int i = (int)(pr / num_kv_heads), kvh = (int)(pr % num_kv_heads);
    int L = seq_lens[i];
    if (L < 0 || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) {
      failed = 1;
      continue;
    }
    int Lc = L > 0 ? L : 1;
    double* K = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* sc = (double*)malloc(sizeof(double) * (size_t)Lc);
    double* q = (double*)malloc(sizeof(double) * (size_t)head_dim);
    if (!K || !V || !sc || !q) {
      failed = 1;
    } else if (gather_kv(K, V, key_cache, value_cache,
                         block_tables + (int64_t)i * max_blocks_per_seq, L, kvh, num_kv_heads,
                         head_dim, block_size, num_blocks, cache_dtype, k_scale,
                         v_scale) != 0) {
      failed = 1;
    } else {
      for (int g = 0; g < group; ++g) {
        int h = kvh * group + g;
        int64_t qrow = ((int64_t)i * num_heads + h) * head_dim;
        for (int d = 0; d < head_dim; ++d) q[d] = load_elt(query, qrow + d, q_dtype);
        attend_rows(out + qrow, NULL, NULL, q, K, V, 0, L, head_dim, scale, sc);
      }
    }
    free(K);
    free(V);
    free(sc);
    free(q);
  }
  return failed ? -1 : 0;
}

/* ---------------------------------------------------------------------------
 * Multi-query attention over the paged cache (chunked prefill, [P1] sec 6: a
 * long prompt is processed in chunks interleaved with decode steps; several
 * query tokens per sequence).  Sequence i has q_i = query_start[i+1] -
 * query_start[i] query tokens, the last q_i positions of its context (their K/V
 * already in the cache); query token j sits at position L_i - q_i + j and attends
 * to positions 0 .. its own (causal).  Each query row is the textbook attention
 * of attend_rows over that prefix of the gathered K, V.
 * out: fp64 [total_queries][num_heads][head_dim].
 * ------------------------------------------------------------------------- */
int oracle_paged_attention_prefill(double* out, const void* query, const void* key_cache,
                                   const void* value_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* seq_lens,
                                   const int32_t* query_start, int num_seqs, int num_heads,
                                   int num_kv_heads, int head_dim, int block_size,
                                   int64_t num_blocks, double scale, int q_dtype, int cache_dtype,
                                   double k_scale, double v_scale) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return -1;
  if (num_heads % num_kv_heads != 0) return -1;
  if (!elt_size(q_dtype) || !elt_size(cache_dtype)) return -1;
  int group = num_heads / num_kv_heads;
  int failed = 0;
  int64_t npairs = (int64_t)num_seqs * num_kv_heads;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (int64_t pr = 0; pr < npairs; ++pr) {
    int i = (int)(pr / num_kv_heads), kvh = (int)(pr % num_kv_heads);
    int L = seq_lens[i];
    int q0 = query_start[i], nq = query_start[i + 1] - query_start[i];
    if (L < 0 || nq < 0 || nq > L || (int64_t)L > (int64_t)max_blocks_per_seq * block_size) {
      failed = 1;
      continue;
    }
    int Lc = L > 0 ? L : 1;
    double* K = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* sc = (double*)malloc(sizeof(double) * (size_t)Lc);
    double* q = (double*)malloc(sizeof(double) * (size_t)head_dim);
    if (!K || !V || !sc || !q ||
        gather_kv(K, V, key_cache, value_cache, block_tables + (int64_t)i * max_blocks_per_seq,
                  L, kvh, num_kv_heads, head_dim, block_size, num_blocks, cache_dtype, k_scale,
                  v_scale) != 0) {
      failed = 1;
    } else {
      for (int j = 0; j < nq; ++j) {
        int pos = L - nq + j; /* this query token's position */
        for (int g = 0; g < group; ++g) {
          int h = kvh * group + g;
          int64_t row = ((int64_t)(q0 + j) * num_heads + h) * head_dim;
          for (int d = 0; d < head_dim; ++d) q[d] = load_elt(query, row + d, q_dtype);
          attend_rows(out + row, NULL, NULL, q, K, V, 0, pos + 1, head_dim, scale, sc);
        }
      }
    }
    free(K);
    free(V);
    free(sc);
    free(q);
  }
  return failed ? -1 : 0;
}

/* ---------------------------------------------------------------------------
 * Per-partition statistics: the same textbook definition applied to the token
 * range [p * part, min(L, (p+1) * part)) of each (sequence, head):
 *   m_p = max score, l_p = sum exp(s - m_p), o_p = sum exp(s - m_p) v / l_p.
 * Ranges past the end get m = -inf, l = 0, o = 0.
 * m, l: [num_seqs][num_heads][max_parts]; o: [num_seqs][num_heads][max_parts][D].
 * ------------------------------------------------------------------------- */
int oracle_decode_partition_stats(double* m, double* l, double* o, int max_parts,
                                  int partition_size, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                                  int num_heads, int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, double scale, int q_dtype, int cache_dtype,
                                  double k_scale, double v_scale) {
  if (partition_size <= 0 || max_parts <= 0) return -1;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0)
    return -1;
  if (num_heads % num_kv_heads != 0) return -1;
  int group = num_heads / num_kv_heads;
  int failed = 0;
  for (int i = 0; i < num_seqs && !failed; ++i) {
    int L = seq_lens[i];
    if (L < 0 || (int64_t)L > (int64_t)max_parts * partition_size ||
        (int64_t)L > (int64_t)max_blocks_per_seq * block_size)
      return -1;
    int Lc = L > 0 ? L : 1;
    double* K = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)Lc * head_dim);
    double* sc = (double*)malloc(sizeof(double) * (size_t)Lc);
    double* q = (double*)malloc(sizeof(double) * (size_t)head_dim);
    for (int kvh = 0; kvh < num_kv_heads && !failed; ++kvh) {
      if (!K || !V || !sc || !q ||
          gather_kv(K, V, key_cache, value_cache, block_tables + (int64_t)i * max_blocks_per_seq,
                    L, kvh, num_kv_heads, head_dim, block_size, num_blocks, cache_dtype, k_scale,
                    v_scale) != 0) {
        failed = 1;
        break;
      }
      for (int g = 0; g < group; ++g) {
        int h = kvh * group + g;
        int64_t row = (int64_t)i * num_heads + h;
        for (int d = 0; d < head_dim; ++d) q[d] = load_elt(query, row * head_dim + d, q_dtype);
        for (int p = 0; p < max_parts; ++p) {
          int lo = p * partition_size, hi = lo + partition_size;
          if (hi > L) hi = L;
          int64_t ix = row * max_parts + p;
          attend_rows(o + ix * head_dim, m + ix, l + ix, q, K, V, lo, hi, head_dim, scale, sc);
        }
      }
    }
    free(K);
    free(V);
    free(sc);
    free(q);
  }
  return failed ? -1 : 0;
}

/* ---------------------------------------------------------------------------
 * Log-sum-exp merge of partition statistics, row by row:
 *   M = max_p m_p ; w_p = l_p * exp(m_p - M) ; out = sum_p w_p o_p / sum_p w_p.
 * Partitions with l_p = 0 carry no weight; a row with no weight gives zeros.
 * ------------------------------------------------------------------------- */
void oracle_lse_merge(double* out, const double* m, const double* l, const double* o,
                      int64_t num_rows, int max_parts, int head_dim) {
  for (int64_t r = 0; r < num_rows; ++r) {
    double M = -INFINITY;
    for (int p = 0; p < max_parts; ++p)
      if (l[r * max_parts + p] > 0.0 && m[r * max_parts + p] > M) M = m[r * max_parts + p];
    double W = 0.0;
    for (int d = 0; d < head_dim; ++d) out[r * head_dim + d] = 0.0;
    if (M == -INFINITY) continue;
    for (int p = 0; p < max_parts; ++p) {
      double lp = l[r * max_parts + p];
      if (!(lp > 0.0)) continue;
      double w = lp * exp(m[r * max_parts + p] - M);
      W += w;
      for (int d = 0; d < head_dim; ++d)
        out[r * head_dim + d] += w * o[(r * max_parts + p) * head_dim + d];
    }
    for (int d = 0; d < head_dim; ++d) out[r * head_dim + d] /= W;
  }
}

/* Number of OpenMP threads the decode loop would use (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Set the number of OpenMP threads later calls use (n >= 1); returns the new count. */
int oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* Convert n values of a format to fp64 (used by tests to read device outputs). */
int oracle_to_f64(double* dst, const void* src, int64_t n, int dtype) {
  if (!elt_size(dtype)) return -1;
  for (int64_t i = 0; i < n; ++i) dst[i] = load_elt(src, i, dtype);
  return 0;
}
