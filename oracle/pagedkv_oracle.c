/*
 * CPU oracle for paged KV append and PagedAttention decode.
 *
 * TEST INFRASTRUCTURE ONLY. This file is a plain, slow, obviously-correct
 * restatement of what the paged decode path computes, in fp64. Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may build, load
 * or call it; the product library never does, and this file shares no code,
 * header or constant with it.
 *
 * Sources (page title, address, section):
 *   [T] "vLLM 推理引擎源码级拆解：PagedAttention 显存虚拟化、Continuous Batching
 *        调度与量化落地全指南" (chenxutan.com/d/5333)
 *        §2.1 fixed-size KV blocks, per-sequence block table, shared blocks
 *        §2.2 block-table figure; a new token fills the last block's next slot
 *        §2.3 the PagedAttention kernel: per token, logical block = tok / bs,
 *             offset = tok % bs, physical block = block_table[logical block],
 *             score = dot(query, k) * scale, online softmax, write back; GQA/MQA
 *   [P] "vLLM 深度实战：当 PagedAttention 遇上生产级 LLM 推理" (chenxutan.com/d/3332)
 *        §1.2 Block / Block Table: blocks of 16 tokens, allocated on demand,
 *             shared through a reference count
 *   [D] "vLLM 0.5 深度拆解" (chenxutan.com/d/4924) §4.2 FP8 KV cache
 *
 * Readings of points the pages leave open (each is listed in the design notes):
 *   - the cache is indexed by KV head: element (blk, off, h, d) of a pool laid
 *     out [num_blocks, block_size, num_kv_heads, head_dim]; the §2.3 address
 *     omits the head term, which is added here;
 *   - GQA groups consecutive query heads: query head j reads KV head
 *     j / (num_heads / num_kv_heads);
 *   - seq_len counts the token appended in this step; seq_len <= 0 gives zeros;
 *   - a negative slot in slot_mapping, or one past the pool, writes nothing;
 *     a block-table entry outside [0, num_blocks) reads as a row of zeros;
 *   - "fp8" is OCP E4M3 (bias 7, 3 mantissa bits, subnormals, max 448, no
 *     infinities, S.1111.111 = NaN); quantising divides by the per-tensor scale
 *     in IEEE binary32 and rounds to nearest-even with saturation to +-448;
 *     decoding multiplies the E4M3 value by the scale;
 *   - softmax is computed in two passes (max, then exp-weighted sums), which is
 *     the exact result the pages' online softmax reaches up to rounding order.
 *
 * Everything is fp64 except the binary32 division the FP8 quantiser performs.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Element type codes of this oracle (its own numbering). */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_E4M3 = 3 };

static int orc_elem_bytes(int dt) {
  switch (dt) {
    case ORC_F32: return 4;
    case ORC_F16: return 2;
    case ORC_BF16: return 2;
    case ORC_E4M3: return 1;
    default: return 0;
  }
}

/* ---- element decoding, straight from each format's bit layout ---------- */

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
static double orc_f16_value(uint16_t b) {
  int s = (b >> 15) & 1, e = (b >> 10) & 31, m = b & 1023;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp((double)(1024 + m), e - 25);
  return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
static double orc_bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* OCP E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; S.1111.111 is NaN. */
double orc_e4m3_value(uint8_t b) {
  int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);           /* subnormal: m/8 * 2^-6 */
  else v = ldexp((double)(8 + m), e - 10);        /* (1 + m/8) * 2^(e-7)   */
  return s ? -v : v;
}

static double orc_load(const void* base, int64_t idx, int dt) {
  switch (dt) {
    case ORC_F32: { float f; memcpy(&f, (const char*)base + 4 * idx, 4); return (double)f; }
    case ORC_F16: { uint16_t b; memcpy(&b, (const char*)base + 2 * idx, 2); return orc_f16_value(b); }
    case ORC_BF16: { uint16_t b; memcpy(&b, (const char*)base + 2 * idx, 2); return orc_bf16_value(b); }
    case ORC_E4M3: return orc_e4m3_value(((const uint8_t*)base)[idx]);
    default: return NAN;
  }
}

/* ---- E4M3 encoding: round to nearest, ties to even, saturate to +-448 --- */

uint8_t orc_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);                 /* exact */
  if (a >= 448.0) return sign | 0x7E;         /* saturate (also infinities) */
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: value = m * 2^-9, m in [0, 8]; m == 8 is the smallest normal */
    double m = nearbyint(ldexp(a, 9));        /* default mode: ties to even */
    return sign | (uint8_t)m;                 /* m == 8 encodes e=1, m=0 */
  }
  int ex;
  frexp(a, &ex);                              /* a = f * 2^ex, f in [0.5, 1) */
  int u = ex - 1;                             /* a in [2^u, 2^(u+1)) */
  double m = nearbyint((ldexp(a, -u) - 1.0) * 8.0);
  if (m == 8.0) { m = 0.0; u += 1; }
  int e = u + 7;
  if (e > 15 || (e == 15 && m == 7.0)) return sign | 0x7E;  /* rounds past 448 */
  return sign | (uint8_t)((e << 3) | (int)m);
}

/* ---- block-table arithmetic ([T] §2.3, [P] §1.2) ---------------------- */

/* Number of blocks a sequence of seq_len tokens occupies: ceil(seq_len / bs). */
int64_t orc_num_blocks(int64_t seq_len, int block_size) {
  if (seq_len <= 0) return 0;
  return (seq_len + block_size - 1) / block_size;
}

/* Flat slot of token `tok` of a sequence: physical block * bs + offset. */
int64_t orc_slot_of_token(const int32_t* block_table_row, int64_t tok, int block_size) {
  int64_t logical = tok / block_size;
  int64_t offset = tok % block_size;
  int64_t physical = block_table_row[logical];
  return physical * block_size + offset;
}

/* ---- append ([T] §2.2: the new token goes into the next slot) ---------- */

/*
 * For every token t with 0 <= slot_mapping[t] < num_blocks*block_size, write
 * key[t] / value[t] ([num_tokens, num_kv_heads, head_dim], src_dtype) into the
 * caches at (slot / bs, slot % bs). Same dtype: bytes are copied. E4M3 cache:
 * each element is widened to binary32, divided by the scale in binary32 and
 * encoded. Caches are host copies updated in place.
 */
int orc_append(const void* key, const void* value, void* k_cache, void* v_cache,
               const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
               int head_dim, int block_size, int64_t num_blocks, int src_dtype,
               int cache_dtype, float k_scale, float v_scale) {
  int sb = orc_elem_bytes(src_dtype), cb = orc_elem_bytes(cache_dtype);
  if (!sb || !cb) return -1;
  if (cache_dtype != src_dtype && cache_dtype != ORC_E4M3) return -1;
  int64_t row = (int64_t)num_kv_heads * head_dim;
  for (int t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    if (slot < 0 || slot >= num_blocks * block_size) continue;
    int64_t blk = slot / block_size, off = slot % block_size;
    int64_t dst0 = (blk * block_size + off) * row;
    int64_t src0 = (int64_t)t * row;
    for (int64_t e = 0; e < row; ++e) {
      if (cache_dtype == src_dtype) {
        memcpy((char*)k_cache + (dst0 + e) * cb, (const char*)key + (src0 + e) * sb, cb);
        memcpy((char*)v_cache + (dst0 + e) * cb, (const char*)value + (src0 + e) * sb, cb);
      } else {
        float kx = (float)orc_load(key, src0 + e, src_dtype);   /* exact widening */
        float vx = (float)orc_load(value, src0 + e, src_dtype);
        volatile float kq = kx / k_scale;                        /* binary32 division */
        volatile float vq = vx / v_scale;
        ((uint8_t*)k_cache)[dst0 + e] = orc_e4m3_encode(kq);
        ((uint8_t*)v_cache)[dst0 + e] = orc_e4m3_encode(vq);
      }
    }
  }
  return 0;
}

/* ---- decode ([T] §2.3) -------------------------------------------------- */

typedef struct {
  const void* query; const void* k_cache; const void* v_cache;
  const int32_t* block_table; const int32_t* seq_lens;
  int num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq;
  int64_t num_blocks;
  double scale, k_scale, v_scale;
  int q_dtype, cache_dtype;
} orc_problem;

/*
 * Attention of one query row (query element offset qoff, KV head h) over the
 * first L cached tokens of sequence i:
 *   K[t] = cache element at (block_table[i][t / bs], t % bs, h, :)
 *   s_t  = scale * <q, K[t]>
 *   out  = sum_t exp(s_t - max s) V[t] / sum_t exp(s_t - max s)
 * out_row receives head_dim doubles (zeros if L <= 0); sbuf holds L doubles.
 */
static void orc_attend_row(const orc_problem* p, int64_t qoff, int i, int h, int64_t L,
                           double* out_row, double* sbuf) {
  int D = p->head_dim;
  for (int d = 0; d < D; ++d) out_row[d] = 0.0;
  if (L <= 0) return;
  const int32_t* bt = p->block_table + (int64_t)i * p->max_blocks_per_seq;
  int is8 = p->cache_dtype == ORC_E4M3;
  double ks = is8 ? p->k_scale : 1.0, vs = is8 ? p->v_scale : 1.0;

  double m = -INFINITY;
  for (int64_t t = 0; t < L; ++t) {
    int64_t slot = orc_slot_of_token(bt, t, p->block_size);
    int64_t base = (slot * p->num_kv_heads + h) * D;
    int inside = slot >= 0 && slot < p->num_blocks * p->block_size;
    double dot = 0.0;
    for (int d = 0; d < D && inside; ++d)
      dot += orc_load(p->query, qoff + d, p->q_dtype) * (orc_load(p->k_cache, base + d, p->cache_dtype) * ks);
    sbuf[t] = p->scale * dot;
    if (sbuf[t] > m) m = sbuf[t];
  }
  double denom = 0.0;
  for (int64_t t = 0; t < L; ++t) {
    int64_t slot = orc_slot_of_token(bt, t, p->block_size);
    int64_t base = (slot * p->num_kv_heads + h) * D;
    int inside = slot >= 0 && slot < p->num_blocks * p->block_size;
    double w = exp(sbuf[t] - m);
    denom += w;
    for (int d = 0; d < D && inside; ++d)
      out_row[d] += w * (orc_load(p->v_cache, base + d, p->cache_dtype) * vs);
  }
  for (int d = 0; d < D; ++d) out_row[d] /= denom;
}

/* Decode: query head j of sequence i (query row i) over all L_i cached tokens. */
static void orc_decode_item(const orc_problem* p, int i, int j, double* out_row, double* sbuf) {
  int g = p->num_heads / p->num_kv_heads;
  int64_t qoff = ((int64_t)i * p->num_heads + j) * p->head_dim;
  orc_attend_row(p, qoff, i, j / g, p->seq_lens[i], out_row, sbuf);
}

/*
 * Decode for a list of (sequence, query head) items. items holds 2*num_items
 * ints (i, j); out receives num_items*head_dim doubles in item order.
 * num_threads <= 0 uses every available thread. Returns the threads used.
 */
int orc_decode_items(double* out, const int32_t* items, int64_t num_items,
                     const void* query, const void* k_cache, const void* v_cache,
                     const int32_t* block_table, const int32_t* seq_lens,
                     int num_heads, int num_kv_heads, int head_dim, int block_size,
                     int max_blocks_per_seq, int64_t num_blocks, double scale,
                     int q_dtype, int cache_dtype, double k_scale, double v_scale,
                     int num_threads) {
  if (num_kv_heads <= 0 || num_heads % num_kv_heads) return -1;
  orc_problem p = {query, k_cache, v_cache, block_table, seq_lens, num_heads, num_kv_heads,
                   head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale,
                   v_scale, q_dtype, cache_dtype};
  int64_t max_len = 1;
  for (int64_t n = 0; n < num_items; ++n) {
    int64_t L = seq_lens[items[2 * n]];
    if (L > max_len) max_len = L;
  }
  int used = 1;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
  used = num_threads;
#pragma omp parallel num_threads(num_threads)
#endif
  {
    double* sbuf = (double*)malloc(sizeof(double) * max_len);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int64_t n = 0; n < num_items; ++n)
      orc_decode_item(&p, items[2 * n], items[2 * n + 1], out + n * head_dim, sbuf);
    free(sbuf);
  }
  return used;
}

/* Decode for every (sequence, query head): out is [num_seqs, num_heads, head_dim]. */
int orc_decode(double* out, const void* query, const void* k_cache, const void* v_cache,
               const int32_t* block_table, const int32_t* seq_lens, int num_seqs,
               int num_heads, int num_kv_heads, int head_dim, int block_size,
               int max_blocks_per_seq, int64_t num_blocks, double scale, int q_dtype,
               int cache_dtype, double k_scale, double v_scale, int num_threads) {
  int64_t n = (int64_t)num_seqs * num_heads;
  int32_t* items = (int32_t*)malloc(sizeof(int32_t) * 2 * (n ? n : 1));
  for (int64_t k = 0; k < n; ++k) { items[2 * k] = (int32_t)(k / num_heads); items[2 * k + 1] = (int32_t)(k % num_heads); }
  int r = orc_decode_items(out, items, n, query, k_cache, v_cache, block_table, seq_lens,
                           num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           num_blocks, scale, q_dtype, cache_dtype, k_scale, v_scale, num_threads);
  free(items);
  return r;
}

/* ---- array helpers for the Python wrapper ----------------------------- */

/* ---- multi-token queries: chunked prefill / prefix-cache continuation ---- */

/*
 * Query rows query_start[i] .. query_start[i+1]-1 belong to sequence i, whose
 * seq_lens[i] cached tokens include them as its last q_i = query_start[i+1] -
 * query_start[i] tokens ("vLLM 0.5 深度拆解" §2.3 chunked prefill: a long prompt
 * is filled in chunks, each chunk's tokens attending over everything before
 * them; "vLLM 推理引擎源码级拆解" §4.2: a request whose prefix blocks are cached
 * computes only the rest). Row r of sequence i sits at position
 *   pos = seq_lens[i] - q_i + (r - query_start[i])
 * and attends causally over tokens 0..pos. items holds (row, query head)
 * pairs; out receives num_items*head_dim doubles in item order. Returns the
 * threads used, or -1 for a bad head ratio.
 */
int orc_prefill_items(double* out, const int32_t* items, int64_t num_items,
                      const void* query, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens,
                      const int32_t* query_start, int num_seqs, int num_heads, int num_kv_heads,
                      int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                      double scale, int q_dtype, int cache_dtype, double k_scale,
                      double v_scale, int num_threads) {
  if (num_kv_heads <= 0 || num_heads % num_kv_heads) return -1;
  orc_problem p = {query, k_cache, v_cache, block_table, seq_lens, num_heads, num_kv_heads,
                   head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale,
                   v_scale, q_dtype, cache_dtype};
  int g = num_heads / num_kv_heads;
  int64_t max_len = 1;
  for (int i = 0; i < num_seqs; ++i)
    if (seq_lens[i] > max_len) max_len = seq_lens[i];
  int used = 1;
#ifdef _OPENMP
  if (num_threads <= 0) num_threads = omp_get_max_threads();
  used = num_threads;
#pragma omp parallel num_threads(num_threads)
#endif
  {
    double* sbuf = (double*)malloc(sizeof(double) * max_len);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int64_t n = 0; n < num_items; ++n) {
      int r = items[2 * n], j = items[2 * n + 1];
      int i = 0;
      while (i < num_seqs && !(query_start[i] <= r && r < query_start[i + 1])) ++i;
      double* row = out + n * head_dim;
      if (i == num_seqs) {
        for (int d = 0; d < head_dim; ++d) row[d] = 0.0;
        continue;
      }
      int64_t q_i = query_start[i + 1] - query_start[i];
      int64_t pos = (int64_t)seq_lens[i] - q_i + (r - query_start[i]);
      orc_attend_row(&p, ((int64_t)r * num_heads + j) * head_dim, i, j / g, pos + 1, row, sbuf);
    }
    free(sbuf);
  }
  return used;
}

void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
  for (int64_t k = 0; k < n; ++k) out[k] = orc_e4m3_encode(x[k]);
}

void orc_values_array(const void* src, int dtype, double* out, int64_t n) {
  for (int64_t k = 0; k < n; ++k) out[k] = orc_load(src, k, dtype);
}
