/*
 * ORACLE — test infrastructure only.
 *
 * A plain, slow, fp64 CPU statement of exact decode attention against a
 * paged grouped-query KV cache.  It exists so that the CUDA path can be
 * checked against something obviously correct.  Only the tests, the smoke
 * check and the CPU-baseline leg of the benchmark may load it; the product
 * library never does, and the two share no code.
 *
 * What it computes (per batch row b, query position t, query head h):
 *
 *   O[b,t,h,:] = softmax(scale * q . K^T) . V          (exact, fp64)
 *   LSE[b,h,t] = ln sum_j exp(scale * q . k_j)          (natural log)
 *
 * Sources:
 *  - "SmallQ FlashAttention (Vector)" README, section 接口 (Interface): the
 *    formula O = softmax(Q K^T / sqrt(headDim)) V for small qLen, long kvLen.
 *  - "ops-transformer FlashAttention" walkthrough, section "标准 Attention 的
 *    问题" (standard attention) and "FlashAttention 的数学细节" (math
 *    details): softmax with the max subtracted for stability,
 *    attn_i = exp(s_i - m) / sum_j exp(s_j - m).
 *  - "Flash-Attention GQA 性能调优: pack_gqa 与 num_splits", section
 *    "两个开关在 kernel 层面各做了什么": query head h belongs to KV head
 *    h / qhead_per_khead (the groups are contiguous).
 *  - "MixedQuantSparseFlashMlaMetadata 算子解析", section 参数说明
 *    (ori_mask_mode 3, RightDownCausal): with qLen draft tokens already in
 *    the cache, query t (0-based) sees the first L - qLen + t + 1 keys.
 *  - "MXFlashAttn 1.4.0" project page, 能力矩阵 (capability matrix): paged KV
 *    cache; the block table maps a logical page of a sequence to a page of
 *    the shared pool.
 *
 * There is no tiling, no split and no online rescaling here: the scores of a
 * row are materialised as a vector, its maximum is taken, and the weights
 * are formed from it directly.  Every input element is widened exactly from
 * its 16-bit storage format to double before any arithmetic.
 *
 * A row that sees no key (L = 0, or a causal row with L - qLen + t + 1 <= 0)
 * has no softmax; the reading used throughout is O = 0 and LSE = -inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits.  Exponent 0 encodes zero and subnormals (fraction * 2^-24);
 * exponent 31 encodes infinities and NaNs. */
double oracle_f16_to_double(uint16_t bits) {
  int sign = (bits >> 15) & 1;
  int expo = (bits >> 10) & 0x1f;
  int frac = bits & 0x3ff;
  double v;
  if (expo == 0) {
    v = ldexp((double)frac, -24);
  } else if (expo == 31) {
    v = frac ? NAN : INFINITY;
  } else {
    v = ldexp((double)(frac + 1024), expo - 25);
  }
  return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE 754 binary32: 1 sign bit, 8
 * exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_to_double(uint16_t bits) {
  uint32_t w = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &w, sizeof f);
  return (double)f;
}

static double widen(uint16_t bits, int dtype) {
  return dtype == ORACLE_BF16 ? oracle_bf16_to_double(bits)
                              : oracle_f16_to_double(bits);
}

/* Address of element d of key/value row j (logical position j in sequence
 * b) for KV head kvh.  Paged layout: cache[num_pages, page_size, Hkv, D]
 * with page = block_table[b * max_pages_per_seq + j / page_size].
 * Contiguous layout (block_table == NULL): cache[B, page_size, Hkv, D],
 * i.e. row b is its own single page of page_size (= max_seqlen_k) slots. */
static size_t kv_index(const int32_t *block_table, int max_pages_per_seq,
                       int page_size, int Hkv, int D, int b, int j, int kvh) {
  long page;
  if (block_table) {
    page = block_table[(size_t)b * max_pages_per_seq + j / page_size];
  } else {
    page = b;
  }
  long slot = j % page_size;
  return (((size_t)page * page_size + slot) * Hkv + kvh) * (size_t)D;
}

/*
 * Exact attention for every (b, t, h).
 *   q          [B, q_len, Hq, D]        16-bit storage (dtype)
 *   k_cache    [num_pages, page_size, Hkv, D]  (or [B, page_size, Hkv, D])
 *   v_cache    same as k_cache
 *   block_table [B, max_pages_per_seq] int32, or NULL for contiguous
 *   cache_seqlens [B] int32, the number of valid keys L_b of each row
 *   out        [B, q_len, Hq, D] double
 *   lse        [B, Hq, q_len]    double (natural log)
 * Returns 0, or -1 on a bad shape argument.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k_cache,
                  const uint16_t *v_cache, const int32_t *block_table,
                  const int32_t *cache_seqlens, int B, int q_len, int Hq,
                  int Hkv, int D, int page_size, int max_pages_per_seq,
                  int dtype, double scale, int causal, double *out,
                  double *lse) {
  if (B < 0 || q_len < 1 || Hq < 1 || Hkv < 1 || D < 1 || page_size < 1 ||
      Hq % Hkv != 0)
    return -1;
  const int G = Hq / Hkv; /* query heads per KV head */
  const long rows = (long)B * q_len * Hq;

#pragma omp parallel for schedule(dynamic, 1)
  for (long r = 0; r < rows; ++r) {
    const int h = (int)(r % Hq);
    const int t = (int)((r / Hq) % q_len);
    const int b = (int)(r / ((long)Hq * q_len));
    const int kvh = h / G;
    const int L = cache_seqlens[b];

    int n = causal ? L - q_len + t + 1 : L;
    if (n > L) n = L;
    if (n < 0) n = 0;

    double *o = out + (((size_t)b * q_len + t) * Hq + h) * (size_t)D;
    double *lse_row = lse + ((size_t)b * Hq + h) * q_len + t;

    if (n == 0) {
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      *lse_row = -INFINITY;
      continue;
    }

    const uint16_t *qrow = q + (((size_t)b * q_len + t) * Hq + h) * (size_t)D;
    double *qd = (double *)malloc(sizeof(double) * (size_t)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    for (int d = 0; d < D; ++d) qd[d] = widen(qrow[d], dtype);

    /* scores s_j = scale * sum_d q[d] k_j[d] */
    for (int j = 0; j < n; ++j) {
      const uint16_t *krow =
          k_cache + kv_index(block_table, max_pages_per_seq, page_size, Hkv,
                             D, b, j, kvh);
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qd[d] * widen(krow[d], dtype);
      s[j] = scale * dot;
    }

    /* softmax with the maximum subtracted */
    double m = s[0];
    for (int j = 1; j < n; ++j)
      if (s[j] > m) m = s[j];
    double l = 0.0;
    for (int j = 0; j < n; ++j) {
      s[j] = exp(s[j] - m); /* s now holds the unnormalised weights p_j */
      l += s[j];
    }

    /* O = sum_j p_j v_j / l */
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int j = 0; j < n; ++j) {
      const uint16_t *vrow =
          v_cache + kv_index(block_table, max_pages_per_seq, page_size, Hkv,
                             D, b, j, kvh);
      for (int d = 0; d < D; ++d) o[d] += s[j] * widen(vrow[d], dtype);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    *lse_row = m + log(l);

    free(s);
    free(qd);
  }
  return 0;
}

/*
 * Exact merge of per-split partial results (the reduce that follows a
 * split of the key axis; "Flash-Attention GQA 性能调优", section
 * "两个开关在 kernel 层面各做了什么": each split yields a partial
 * attention output and its logsumexp, and a reduce merges them).
 *
 * With split s covering key set J_s, lse_s = ln sum_{j in J_s} e^{s_j} and
 * O_s = sum_{j in J_s} e^{s_j} v_j / e^{lse_s}.  Then over all keys
 *   LSE = ln sum_s e^{lse_s}
 *   O   = sum_s e^{lse_s - LSE} O_s
 * written with the maximum split LSE subtracted for stability.  Splits with
 * lse_s = -inf hold no key and carry zero weight; if every split is empty
 * the result is O = 0, LSE = -inf.
 *
 *   o_part   [S, rows, D] double, lse_part [S, rows] double
 *   out      [rows, D] double,    lse      [rows] double
 */
int oracle_combine(const double *o_part, const double *lse_part, int S,
                   long rows, int D, double *out, double *lse) {
  if (S < 1 || rows < 0 || D < 1) return -1;
  for (long r = 0; r < rows; ++r) {
    double mx = -INFINITY;
    for (int s = 0; s < S; ++s)
      if (lse_part[(size_t)s * rows + r] > mx) mx = lse_part[(size_t)s * rows + r];
    double *o = out + (size_t)r * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (mx == -INFINITY) {
      lse[r] = -INFINITY;
      continue;
    }
    double sum = 0.0;
    for (int s = 0; s < S; ++s) sum += exp(lse_part[(size_t)s * rows + r] - mx);
    double L = mx + log(sum);
    for (int s = 0; s < S; ++s) {
      double w = exp(lse_part[(size_t)s * rows + r] - L);
      const double *os = o_part + ((size_t)s * rows + r) * D;
      for (int d = 0; d < D; ++d) o[d] += w * os[d];
    }
    lse[r] = L;
  }
  return 0;
}
