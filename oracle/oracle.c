/*
 * Plain, slow, single-threaded fp64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product calls this file: only the
 * tests, the smoke check and the benchmark's CPU-baseline leg load it. It
 * shares no source, header, helper or table with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [Ch7]    "第 7 章推理框架：vLLM 与 PagedAttention"
 *            (blog.lkad.net/posts/ai-infra-07-vllm-pagedattention/)
 *   [OSPage] "vLLM 与 PagedAttention：把 GPU 显存当操作系统内存管"
 *            (alishangtian.com/article/user-68cf17f91b)
 *   [Day28]  "GPU 学习日报 Day 28：vLLM 与 PagedAttention：GPU Memory 管理的艺术"
 *            (daoyuly.cn/2026/2026-10-17-gpu-learning-day-28/)
 * The fp8 format is the OCP 8-bit floating point E4M3 definition ("fn"
 * variant: bias 7, no infinities, S.1111.111 is NaN, max 448).
 *
 * Every function here is written from the plain definition of what it
 * computes. No blocking, fusion or reordering: attention gathers a sequence's
 * blocks into a contiguous array, then does a two-pass softmax in double.
 *
 * Status codes returned: 0 ok, 1 invalid argument (bad id, slot, size).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ sizes */

/* Per-token KV bytes: 2 (K and V) x layers x KV heads x head dim x bytes.
 * [Ch7] §7.1 "KV cache 的数学" formula and §"KV cache 显存估算". */
int64_t oracle_kv_bytes_per_token(int64_t layers, int64_t kv_heads,
                                  int64_t head_dim, int64_t dtype_bytes) {
  return 2 * layers * kv_heads * head_dim * dtype_bytes;
}

/* Total KV bytes: per-token bytes x tokens x concurrent requests.
 * [Ch7] §"KV cache 显存估算" (单 token KV x 平均上下文长度 x 并发请求数);
 * [Day28] §一 growth formula (x seq_len x batch_size). */
int64_t oracle_kv_cache_bytes(int64_t layers, int64_t kv_heads,
                              int64_t head_dim, int64_t dtype_bytes,
                              int64_t tokens, int64_t batch) {
  return oracle_kv_bytes_per_token(layers, kv_heads, head_dim, dtype_bytes) *
         tokens * batch;
}

/* Physical slot of logical token position `pos`: the block table maps
 * logical block pos / B to a physical block, and the token sits at offset
 * pos % B inside it. [Day28] §3.1 (Block Table [7, 1, 3] example);
 * [Ch7] §7.1 "Block 与 Block Table". */
int64_t oracle_slot(const int32_t *block_table_row, int64_t pos,
                    int64_t block_size) {
  return (int64_t)block_table_row[pos / block_size] * block_size +
         pos % block_size;
}

/* ------------------------------------------------------------- number types */

static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Value of an E4M3 code: sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 x 2^-6); S.1111.111 is NaN. */
double oracle_e4m3_decode(uint8_t code) {
  int sign = code >> 7;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6);
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* Round-half-to-even of a non-negative double to an integer. */
static double round_half_even(double x) {
  double f = floor(x);
  double r = x - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Encode a binary32 value to E4M3 with round-to-nearest-even and
 * saturation of finite overflow (and of infinities) to +-448; NaN maps to
 * the NaN code 0x7F. -0 keeps its sign (0x80). */
uint8_t oracle_e4m3_encode(float y) {
  double a;
  int sign;
  if (isnan(y)) return 0x7F;
  sign = signbit(y) ? 1 : 0;
  a = fabs((double)y);
  if (a > 448.0) return (uint8_t)((sign << 7) | 0x7E); /* satfinite */
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: multiples of 2^-9; q == 8 is the smallest normal */
    double q = round_half_even(a / ldexp(1.0, -9));
    return (uint8_t)((sign << 7) | (int)q);
  }
  {
    int E = (int)floor(log2(a));
    double mant, q;
    /* guard against log2 rounding at exact powers of two */
    if (ldexp(1.0, E) > a) E -= 1;
    if (ldexp(1.0, E + 1) <= a) E += 1;
    mant = a / ldexp(1.0, E) - 1.0; /* in [0, 1) */
    q = round_half_even(mant * 8.0);
    if (q == 8.0) {
      q = 0.0;
      E += 1;
    }
    /* a <= 448 keeps E <= 8 and never produces the NaN pattern */
    return (uint8_t)((sign << 7) | ((E + 7) << 3) | (int)q);
  }
}

/* Quantise one bf16 element: y = x / scale in binary32 (correctly rounded
 * IEEE division), then E4M3 RNE with saturation. The per-tensor scale and
 * the fp8_e4m3 cache type: [Ch7] §"vLLM 关键参数速记"
 * (--kv-cache-dtype fp8_e4m3 halves KV memory; precision must be checked). */
uint8_t oracle_quantize_bf16(uint16_t x, float scale) {
  volatile float num = bf16_bits_to_float(x);
  volatile float y = num / scale;
  return oracle_e4m3_encode(y);
}

/* Element-wise oracle_quantize_bf16 over an array (for exhaustive tests). */
void oracle_quantize_bf16_array(const uint16_t *x, int64_t n, float scale,
                                uint8_t *out) {
  int64_t i;
  for (i = 0; i < n; ++i) out[i] = oracle_quantize_bf16(x[i], scale);
}

/* ---------------------------------------------------------- cache writes */

/* Write the new tokens' K/V rows into their cache slots.
 * Cache layout [num_blocks][num_kv_heads][block_size][head_dim];
 * slot s lives in block s / B at offset s % B. A negative slot is skipped.
 * bf16 caches copy the bits; fp8 caches store E4M3(x / scale).
 * [Ch7] §7.1 "Block 与 Block Table" (a new token goes into the next slot,
 * a new block after 16); [Day28] §4.2 (按需分配) and FAQ Q4 (prefill KV is
 * written block-wise too). */
int oracle_reshape_and_cache(const uint16_t *key, const uint16_t *value,
                             void *k_cache, void *v_cache,
                             const int64_t *slot_mapping, int num_tokens,
                             int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int kv_dtype, float k_scale,
                             float v_scale) {
  int t, h, d;
  for (t = 0; t < num_tokens; ++t) {
    int64_t slot = slot_mapping[t];
    int64_t blk, off;
    if (slot < 0) continue;
    if (slot >= (int64_t)num_blocks * block_size) return 1;
    blk = slot / block_size;
    off = slot % block_size;
    for (h = 0; h < num_kv_heads; ++h) {
      int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
      int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * head_dim;
      for (d = 0; d < head_dim; ++d) {
        if (kv_dtype == 0) {
          ((uint16_t *)k_cache)[dst + d] = key[src + d];
          ((uint16_t *)v_cache)[dst + d] = value[src + d];
        } else {
          ((uint8_t *)k_cache)[dst + d] = oracle_quantize_bf16(key[src + d], k_scale);
          ((uint8_t *)v_cache)[dst + d] = oracle_quantize_bf16(value[src + d], v_scale);
        }
      }
    }
  }
  return 0;
}

/* Copy-on-write: for each (src, dst) pair copy the whole physical block,
 * K and V independently. [OSPage] §"PagedAttention：向操作系统借思路"
 * (共享与写时复制); [Day28] §4.2 (Copy-on-Write 共享) and §六 item 4
 * (B allocates a new block, copies, refcount - 1). */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs,
                       int num_pairs, int64_t block_bytes, int num_blocks) {
  int i;
  for (i = 0; i < num_pairs; ++i) {
    int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return 1;
    memcpy((char *)k_cache + dst * block_bytes,
           (const char *)k_cache + src * block_bytes, (size_t)block_bytes);
    memcpy((char *)v_cache + dst * block_bytes,
           (const char *)v_cache + src * block_bytes, (size_t)block_bytes);
  }
  return 0;
}

/* Swap: copy physical blocks between two caches (GPU pool <-> host pool),
 * dst_cache[dst] = src_cache[src] for each (src, dst) pair, K and V alike.
 * Preemption moves a request's KV blocks to CPU memory and back ([Day28]
 * §六 question 4, §七 and FAQ Q3: watermark, preemption, swapping). */
int oracle_swap_blocks(void *dst_k, void *dst_v, const void *src_k,
                       const void *src_v, const int64_t *pairs, int num_pairs,
                       int64_t block_bytes, int src_num_blocks,
                       int dst_num_blocks) {
  int i;
  for (i = 0; i < num_pairs; ++i) {
    int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return 1;
    memcpy((char *)dst_k + dst * block_bytes,
           (const char *)src_k + src * block_bytes, (size_t)block_bytes);
    memcpy((char *)dst_v + dst * block_bytes,
           (const char *)src_v + src * block_bytes, (size_t)block_bytes);
  }
  return 0;
}

/* --------------------------------------------------------------- attention */

static double cache_value(const void *cache, int kv_dtype, double scale,
                          int64_t idx) {
  if (kv_dtype == 0) return bf16_bits_to_double(((const uint16_t *)cache)[idx]);
  return oracle_e4m3_decode(((const uint8_t *)cache)[idx]) * scale;
}

/* Gather K and V of (sequence s, KV head h) into contiguous [L][D] arrays
 * through the block table: logical block j -> physical block table[s][j].
 * [Day28] §3.1 (注意力 kernel 通过 Block Table 间接寻址, Gather 散落的 K/V)
 * and §3.2 (块内连续访存、块间通过指针跳转). */
static int gather_kv(double *Kc, double *Vc, const void *k_cache,
                     const void *v_cache, int kv_dtype, double k_scale,
                     double v_scale, const int32_t *bt_row, int L, int h,
                     int num_kv_heads, int head_dim, int block_size,
                     int num_blocks) {
  int t, d;
  for (t = 0; t < L; ++t) {
    int64_t p = bt_row[t / block_size];
    int64_t base;
    if (p < 0 || p >= num_blocks) return 1;
    base = ((p * num_kv_heads + h) * block_size + t % block_size) * head_dim;
    for (d = 0; d < head_dim; ++d) {
      Kc[(int64_t)t * head_dim + d] = cache_value(k_cache, kv_dtype, k_scale, base + d);
      Vc[(int64_t)t * head_dim + d] = cache_value(v_cache, kv_dtype, v_scale, base + d);
    }
  }
  return 0;
}

/* Decode-step attention for every (sequence, query head):
 *   z_t = sm_scale * sum_d q[d] K[t][d]           (t < context_lens[s])
 *   out = sum_t softmax(z)_t V[t]
 * with the query head hq reading KV head hq / (num_q_heads / num_kv_heads).
 * Two passes over z (max, then normalised weights), all in double.
 * context_lens[s] == 0 gives a zero output row.
 * If seq_subset is non-null only those sequences are computed.
 * [Day28] §一 (each new token's Query attends to all past K/V) and §3.1. */
int oracle_paged_decode(double *out, const uint16_t *q, const void *k_cache,
                        const void *v_cache, int kv_dtype, double k_scale,
                        double v_scale, const int32_t *block_tables,
                        int max_blocks_per_seq, const int32_t *context_lens,
                        int num_seqs, int num_q_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks,
                        double sm_scale, const int32_t *seq_subset,
                        int n_subset) {
  int group, i, n_iter;
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return 1;
  group = num_q_heads / num_kv_heads;
  n_iter = seq_subset ? n_subset : num_seqs;
  for (i = 0; i < n_iter; ++i) {
    int s = seq_subset ? seq_subset[i] : i;
    int L = context_lens[s];
    int hq;
    const int32_t *bt_row = block_tables + (int64_t)s * max_blocks_per_seq;
    if (s < 0 || s >= num_seqs || L < 0) return 1;
    if ((L + block_size - 1) / block_size > max_blocks_per_seq) return 1;
    for (hq = 0; hq < num_q_heads; ++hq) {
      double *o = out + ((int64_t)s * num_q_heads + hq) * head_dim;
      const uint16_t *qv = q + ((int64_t)s * num_q_heads + hq) * head_dim;
      int h = hq / group, t, d;
      double *Kc, *Vc, *z, zmax, denom;
      for (d = 0; d < head_dim; ++d) o[d] = 0.0;
      if (L == 0) continue;
      Kc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
      Vc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
      z = (double *)malloc(sizeof(double) * (size_t)L);
      if (!Kc || !Vc || !z) {
        free(Kc); free(Vc); free(z);
        return 2;
      }
      if (gather_kv(Kc, Vc, k_cache, v_cache, kv_dtype, k_scale, v_scale,
                    bt_row, L, h, num_kv_heads, head_dim, block_size,
                    num_blocks)) {
        free(Kc); free(Vc); free(z);
        return 1;
      }
      zmax = -INFINITY;
      for (t = 0; t < L; ++t) {
        double acc = 0.0;
        for (d = 0; d < head_dim; ++d)
          acc += bf16_bits_to_double(qv[d]) * Kc[(int64_t)t * head_dim + d];
        z[t] = sm_scale * acc;
        if (z[t] > zmax) zmax = z[t];
      }
      denom = 0.0;
      for (t = 0; t < L; ++t) {
        z[t] = exp(z[t] - zmax);
        denom += z[t];
      }
      for (t = 0; t < L; ++t) {
        double p = z[t] / denom;
        for (d = 0; d < head_dim; ++d) o[d] += p * Vc[(int64_t)t * head_dim + d];
      }
      free(Kc); free(Vc); free(z);
    }
  }
  return 0;
}

/* The split-context form of the same attention, step by step: cut the
 * context into partitions of `partition_size` tokens; for partition p keep
 *   m_p = max z,  l_p = sum exp(z - m_p),  o_p = sum exp(z - m_p) V
 * and combine with M = max_p m_p:
 *   out = sum_p exp(m_p - M) o_p / sum_p exp(m_p - M) l_p.
 * Computed in double; equals oracle_paged_decode up to rounding. The pages
 * only name the long-context ("v2") kernel ([Day28] §二, CUDA Kernel layer);
 * the partition/reduce steps above are the plain reading of that name. */
int oracle_paged_decode_split(double *out, const uint16_t *q,
                              const void *k_cache, const void *v_cache,
                              int kv_dtype, double k_scale, double v_scale,
                              const int32_t *block_tables,
                              int max_blocks_per_seq,
                              const int32_t *context_lens, int num_seqs,
                              int num_q_heads, int num_kv_heads, int head_dim,
                              int block_size, int num_blocks, double sm_scale,
                              int partition_size) {
  int group, s;
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return 1;
  if (partition_size <= 0) return 1;
  group = num_q_heads / num_kv_heads;
  for (s = 0; s < num_seqs; ++s) {
    int L = context_lens[s];
    int hq;
    const int32_t *bt_row = block_tables + (int64_t)s * max_blocks_per_seq;
    if (L < 0 || (L + block_size - 1) / block_size > max_blocks_per_seq) return 1;
    for (hq = 0; hq < num_q_heads; ++hq) {
      double *o = out + ((int64_t)s * num_q_heads + hq) * head_dim;
      const uint16_t *qv = q + ((int64_t)s * num_q_heads + hq) * head_dim;
      int h = hq / group, P = (L + partition_size - 1) / partition_size;
      int p, t, d;
      double *Kc, *Vc, *mp, *lp, *op, M, num_l;
      for (d = 0; d < head_dim; ++d) o[d] = 0.0;
      if (L == 0) continue;
      Kc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
      Vc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
      mp = (double *)malloc(sizeof(double) * (size_t)P);
      lp = (double *)malloc(sizeof(double) * (size_t)P);
      op = (double *)calloc((size_t)P * head_dim, sizeof(double));
      if (!Kc || !Vc || !mp || !lp || !op) {
        free(Kc); free(Vc); free(mp); free(lp); free(op);
        return 2;
      }
      if (gather_kv(Kc, Vc, k_cache, v_cache, kv_dtype, k_scale, v_scale,
                    bt_row, L, h, num_kv_heads, head_dim, block_size,
                    num_blocks)) {
        free(Kc); free(Vc); free(mp); free(lp); free(op);
        return 1;
      }
      for (p = 0; p < P; ++p) {
        int t0 = p * partition_size;
        int t1 = t0 + partition_size < L ? t0 + partition_size : L;
        double m = -INFINITY, l = 0.0;
        for (t = t0; t < t1; ++t) {
          double acc = 0.0, zt;
          for (d = 0; d < head_dim; ++d)
            acc += bf16_bits_to_double(qv[d]) * Kc[(int64_t)t * head_dim + d];
          zt = sm_scale * acc;
          if (zt > m) m = zt;
        }
        for (t = t0; t < t1; ++t) {
          double acc = 0.0, w;
          for (d = 0; d < head_dim; ++d)
            acc += bf16_bits_to_double(qv[d]) * Kc[(int64_t)t * head_dim + d];
          w = exp(sm_scale * acc - m);
          l += w;
          for (d = 0; d < head_dim; ++d)
            op[(int64_t)p * head_dim + d] += w * Vc[(int64_t)t * head_dim + d];
        }
        mp[p] = m;
        lp[p] = l;
      }
      M = -INFINITY;
      for (p = 0; p < P; ++p)
        if (mp[p] > M) M = mp[p];
      num_l = 0.0;
      for (p = 0; p < P; ++p) num_l += exp(mp[p] - M) * lp[p];
      for (p = 0; p < P; ++p) {
        double w = exp(mp[p] - M) / num_l;
        for (d = 0; d < head_dim; ++d) o[d] += w * op[(int64_t)p * head_dim + d];
      }
      free(Kc); free(Vc); free(mp); free(lp); free(op);
    }
  }
  return 0;
}

/* Chunked prefill attention through block tables. Sequence s holds
 * context_lens[s] tokens in the cache; its last n_s = query_start[s+1] -
 * query_start[s] tokens are this chunk's queries (rows query_start[s] ..
 * query_start[s+1]-1 of q and out). The query at position p attends to the
 * keys at positions 0..p (causal):
 *   z_t = sm_scale * q . K_t (t <= p),  out = sum_t softmax(z)_t V_t.
 * Prefill KV is written block-wise into the same pool ([Day28] FAQ Q4,
 * chunked prefill mixes prompt chunks with decode), so a chunk attends to
 * the cached prefix and to itself. Two-pass softmax in double. */
int oracle_paged_prefill(double *out, const uint16_t *q, const void *k_cache,
                         const void *v_cache, int kv_dtype, double k_scale,
                         double v_scale, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *query_start,
                         const int32_t *context_lens, int num_seqs,
                         int num_q_heads, int num_kv_heads, int head_dim,
                         int block_size, int num_blocks, double sm_scale) {
  int group, s;
  if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0) return 1;
  group = num_q_heads / num_kv_heads;
  for (s = 0; s < num_seqs; ++s) {
    int L = context_lens[s];
    int q0 = query_start[s], n = query_start[s + 1] - query_start[s];
    const int32_t *bt_row = block_tables + (int64_t)s * max_blocks_per_seq;
    int h, i, t, d;
    double *Kc, *Vc, *z;
    if (n < 0 || n > L || (L + block_size - 1) / block_size > max_blocks_per_seq) return 1;
    if (L == 0) continue;
    Kc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
    Vc = (double *)malloc(sizeof(double) * (size_t)L * head_dim);
    z = (double *)malloc(sizeof(double) * (size_t)L);
    if (!Kc || !Vc || !z) {
      free(Kc); free(Vc); free(z);
      return 2;
    }
    for (h = 0; h < num_kv_heads; ++h) {
      if (gather_kv(Kc, Vc, k_cache, v_cache, kv_dtype, k_scale, v_scale, bt_row, L,
                    h, num_kv_heads, head_dim, block_size, num_blocks)) {
        free(Kc); free(Vc); free(z);
        return 1;
      }
      for (i = 0; i < n; ++i) {
        int p = L - n + i, g;
        for (g = 0; g < group; ++g) {
          int hq = h * group + g;
          const uint16_t *qv = q + ((int64_t)(q0 + i) * num_q_heads + hq) * head_dim;
          double *o = out + ((int64_t)(q0 + i) * num_q_heads + hq) * head_dim;
          double zmax = -INFINITY, denom = 0.0;
          for (t = 0; t <= p; ++t) {
            double acc = 0.0;
            for (d = 0; d < head_dim; ++d)
              acc += bf16_bits_to_double(qv[d]) * Kc[(int64_t)t * head_dim + d];
            z[t] = sm_scale * acc;
            if (z[t] > zmax) zmax = z[t];
          }
          for (t = 0; t <= p; ++t) {
            z[t] = exp(z[t] - zmax);
            denom += z[t];
          }
          for (d = 0; d < head_dim; ++d) o[d] = 0.0;
          for (t = 0; t <= p; ++t) {
            double w = z[t] / denom;
            for (d = 0; d < head_dim; ++d) o[d] += w * Vc[(int64_t)t * head_dim + d];
          }
        }
      }
    }
    free(Kc); free(Vc); free(z);
  }
  return 0;
}
