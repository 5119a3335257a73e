/*
 * NOSA sparse decode attention -- CPU oracle (test infrastructure).
 *
 * This file is the plain, slow, obviously-correct definition of what the
 * per-step sparse decode attention of NOSA (Native and Offloadable Sparse
 * Attention) computes.  It is TEST INFRASTRUCTURE: only the test-suite, the
 * smoke check and the benchmark's CPU-baseline leg may load it.  The CUDA
 * library never links, includes or calls it, and it shares no code with it.
 *
 * Sources (web pages, cited by title and section):
 *   [P1] "从论文到代码：手把手教你理解NOSA-8B的高效注意力机制实现" (nzsm.cn),
 *        section "NOSA-8B的核心实现模块", item 2 (forward: k = cis_pooling(k, cu_seqlens)).
 *   [P2] "NOSA-1B 模型家族全景：从 1B 到 8B，三款稀疏注意力模型怎么选"
 *        (demingchina.com), section "核心原理 3 句话讲清" (local window 1024,
 *        two-level retrieval: compressed attention screens top-k blocks, then
 *        the blocks are read exactly).
 *   [P3] "NOSA-1B 性能基准全解析：5.04× 解码吞吐提升是怎么测出来的" (wmrh.cn),
 *        section 三.2 "显式局部性约束" (window 1024, block 64, about 16 local
 *        blocks, TopK 64), section 三.3 "两阶段注意力" (pooling kernel 32 /
 *        stride 16, coarse scores, top-k, exact attention on the selected
 *        blocks), section 四 "NOSA-1B 模型配置速览" (table: 16 q / 2 KV heads,
 *        bfloat16, TopK64 / window 1024 / block 64 / kernel32 / stride16).
 *   [P5] "NOSA 技术架构解析" (devpress.csdn.net), section "1.1 双阶段稀疏注意力设计"
 *        ("关键技巧": 32-bit prefill, decode switchable to 16-bit or 8-bit integers).
 *
 * Conventions (all readings are listed in the design notes of the repo):
 *   * bf16 values are passed as their 16-bit patterns and widened exactly
 *     (bits << 16) to fp32, then to fp64.
 *   * Sums are taken in fp64.  Pooled keys, compressed scores and block
 *     scores are rounded to fp32 once, at the end of their definition.
 *   * Window j of a sequence covers tokens [j*stride, j*stride + kernel).
 *     nc(L) = number of complete windows = L >= kernel ? (L-kernel)/stride+1 : 0.
 *   * Blocks: block b covers tokens [b*bs, (b+1)*bs); nb(L) = ceil(L/bs).
 *     The local window is the last `local_blocks` blocks; the candidates are
 *     blocks [0, ncand), ncand = max(0, nb - local_blocks).
 *   * Block score (reading of [P3] 三.3 with the rule "max over the windows
 *     that overlap the block, summed over the query heads of the GQA group"):
 *        S[g][b] = sum over heads h of group g (ascending h) of
 *                  max over windows j overlapping block b of s[h][j].
 *   * Top-k: the min(topk, ncand) candidates with the largest S, ties broken
 *     towards the lowest block index, reported in ascending index order and
 *     padded with -1.  -0.0 compares equal to +0.0; NaN ranks as -inf.
 *   * Attention: softmax over the token set (selected blocks) U [ncand*bs, L),
 *     clipped to [0, L), of scale * q.k, applied to v; fp64 throughout.
 *   * INT8 cache variant (reading of [P5] "1.1 双阶段稀疏注意力设计",
 *     "关键技巧": the decode stage may switch to 8-bit integers): each cache
 *     row (token, KV head) of d bf16 values x is kept as d int8 codes and one
 *     fp32 scale, symmetric per row:
 *        amax = max_c |x_c|;  s = amax / 127;  code_c = clamp(rint(x_c / s), -127, 127)
 *     with both divisions in fp32 (IEEE, round to nearest) and rint rounding
 *     half to even; an all-zero row has s = 0 and zero codes.  The value the
 *     method sees is s * code_c (exact in fp64); pooling and attention read
 *     those values in place of the bf16 keys and values.
 *
 * Parity pins for every function live in the CPU test-suite (closed forms,
 * brute force on tiny inputs, dense-attention equivalence via a library
 * attention routine).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1

static int g_threads = 1;

/* Number of OpenMP threads the oracle uses for its loops over independent
 * (sequence, KV head) pairs.  1 (the default) means plain serial loops. */
int nosa_oracle_set_threads(int n) {
  g_threads = n < 1 ? 1 : n;
#ifdef _OPENMP
  return g_threads;
#else
  g_threads = 1;
  return 1;
#endif
}

static double bf16_to_f64(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* A key or value cache as the oracle reads it: bf16 patterns [T, hkv, d], or
 * INT8 codes [T, hkv, d] with one fp32 scale per (row, KV head), scales
 * [T, hkv] (the INT8 cache variant). */
typedef struct {
  const uint16_t* bf16;
  const int8_t* codes;
  const float* scales;
} kv_view;

static double kv_at(const kv_view* v, int64_t row, int hkv, int h, int d, int c) {
  int64_t at = (row * hkv + h) * d + c;
  if (v->bf16) return bf16_to_f64(v->bf16[at]);
  return (double)v->scales[row * hkv + h] * (double)v->codes[at];
}

static int kv_ok(const kv_view* v) { return v->bf16 || (v->codes && v->scales); }

/* INT8 cache variant ([P5] 1.1 "关键技巧", reading in the header): quantizes
 * `rows` rows of d bf16 values (x, [rows, d]) into codes [rows, d] and scales
 * [rows]:  amax = max |x_c|, s = amax / 127, code_c = clamp(rint(x_c / s),
 * -127, 127), divisions in fp32, half to even; s = 0 and zero codes for an
 * all-zero row. */
int nosa_oracle_quantize_int8(const uint16_t* x, int64_t rows, int d, int8_t* codes, float* scales) {
  if (!x || !codes || !scales || rows < 0 || d < 1) return ORACLE_BAD_ARG;
  for (int64_t r = 0; r < rows; ++r) {
    float amax = 0.0f;
    for (int c = 0; c < d; ++c) {
      float v = (float)bf16_to_f64(x[r * d + c]);
      if (fabsf(v) > amax) amax = fabsf(v);
    }
    float s = amax / 127.0f;
    scales[r] = s;
    for (int c = 0; c < d; ++c) {
      float v = (float)bf16_to_f64(x[r * d + c]);
      float code = s > 0.0f ? rintf(v / s) : 0.0f;
      if (code > 127.0f) code = 127.0f;
      if (code < -127.0f) code = -127.0f;
      codes[r * d + c] = (int8_t)code;
    }
  }
  return ORACLE_OK;
}

static int64_t n_windows(int64_t L, int kernel, int stride) {
  return L >= kernel ? (L - kernel) / stride + 1 : 0;
}

static int64_t n_blocks(int64_t L, int bs) { return (L + bs - 1) / bs; }

static int64_t n_candidates(int64_t L, int bs, int local_blocks) {
  int64_t c = n_blocks(L, bs) - local_blocks;
  return c > 0 ? c : 0;
}

/* CIS mean pooling of keys, [P1] item 2 and [P3] 三.3: every window j in
 * [nc(len_old), nc(len_new)) of sequence i and KV head h gets
 *   pooled[i][h][j][:] = (1/kernel) * sum_{t = j*stride}^{j*stride+kernel-1} K[seq_start[i]+t][h][:]
 * K is [T, hkv, d] bf16; pooled is [batch, hkv, nc_cap, d] fp32.
 * Windows outside [nc(len_old), nc(len_new)) are left untouched. */
static int pool_view(const kv_view* k, const int64_t* seq_start,
                     const int32_t* len_old, const int32_t* len_new, int batch,
                     int hkv, int d, int kernel, int stride, float* pooled,
                     int64_t nc_cap) {
  if (!kv_ok(k) || !seq_start || !len_new || !pooled || batch < 0 || hkv < 1 ||
      d < 1 || kernel < 1 || stride < 1)
    return ORACLE_BAD_ARG;
  int npairs = batch * hkv;
#pragma omp parallel for schedule(dynamic) num_threads(g_threads)
  for (int p = 0; p < npairs; ++p) {
    int i = p / hkv, h = p % hkv;
    int64_t j0 = len_old ? n_windows(len_old[i], kernel, stride) : 0;
    int64_t j1 = n_windows(len_new[i], kernel, stride);
    if (j1 > nc_cap) j1 = nc_cap;
    for (int64_t j = j0; j < j1; ++j) {
      float* dst = pooled + (((int64_t)i * hkv + h) * nc_cap + j) * d;
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int t = 0; t < kernel; ++t) {
          int64_t row = seq_start[i] + j * stride + t;
          acc += kv_at(k, row, hkv, h, d, c);
        }
        dst[c] = (float)(acc / kernel);
      }
    }
  }
  return ORACLE_OK;
}

int nosa_oracle_pool(const uint16_t* k_cache, const int64_t* seq_start,
                     const int32_t* len_old, const int32_t* len_new, int batch,
                     int hkv, int d, int kernel, int stride, float* pooled,
                     int64_t nc_cap) {
  kv_view k = {k_cache, NULL, NULL};
  return pool_view(&k, seq_start, len_old, len_new, batch, hkv, d, kernel, stride, pooled, nc_cap);
}

/* The same pooling over an INT8 cache: the mean of the dequantized keys
 * s_t * code_t of the window (scales [T, hkv]). */
int nosa_oracle_pool_int8(const int8_t* k_codes, const float* k_scales, const int64_t* seq_start,
                          const int32_t* len_old, const int32_t* len_new, int batch, int hkv, int d,
                          int kernel, int stride, float* pooled, int64_t nc_cap) {
  kv_view k = {NULL, k_codes, k_scales};
  return pool_view(&k, seq_start, len_old, len_new, batch, hkv, d, kernel, stride, pooled, nc_cap);
}

/* Compressed attention scores, [P3] 三.3 / [P2] 核心原理 (coarse screen):
 *   s[i][hq][j] = scale * q[i][hq][:] . pooled[i][hq / G][j][:],  j < nc(L_i)
 * q is [batch, hq, d] bf16; s is [batch, hq, nc_cap] fp32.  Entries j >= nc(L_i)
 * are set to -inf so that a caller can tell them apart. */
int nosa_oracle_comp_scores(const uint16_t* q, const float* pooled,
                            int64_t nc_cap, const int32_t* seq_len, int batch,
                            int hq, int hkv, int d, int kernel, int stride,
                            double scale, float* s) {
  if (!q || !pooled || !seq_len || !s || hkv < 1 || hq % hkv != 0)
    return ORACLE_BAD_ARG;
  int G = hq / hkv;
#pragma omp parallel for schedule(dynamic) num_threads(g_threads)
  for (int p = 0; p < batch * hq; ++p) {
    int i = p / hq, h = p % hq, g = h / G;
    int64_t nc = n_windows(seq_len[i], kernel, stride);
    if (nc > nc_cap) nc = nc_cap;
    const uint16_t* qv = q + ((int64_t)i * hq + h) * d;
    float* out = s + ((int64_t)i * hq + h) * nc_cap;
    for (int64_t j = 0; j < nc_cap; ++j) {
      if (j >= nc) {
        out[j] = -INFINITY;
        continue;
      }
      const float* kv = pooled + (((int64_t)i * hkv + g) * nc_cap + j) * d;
      double acc = 0.0;
      for (int c = 0; c < d; ++c) acc += bf16_to_f64(qv[c]) * (double)kv[c];
      out[j] = (float)(scale * acc);
    }
  }
  return ORACLE_OK;
}

/* Block scores from compressed scores (reading of [P3] 三.2/三.3, block 64;
 * rule: max over the windows overlapping the block, then summed over the
 * query heads of the GQA group in ascending head order).  Window j overlaps
 * block b when the token ranges [j*stride, j*stride+kernel) and
 * [b*bs, (b+1)*bs) intersect.  Only candidate blocks b < ncand(L_i) get a
 * score; the rest of S[i][g][:] is set to -inf. */
int nosa_oracle_block_scores(const float* s, int64_t nc_cap,
                             const int32_t* seq_len, int batch, int hq, int hkv,
                             int kernel, int stride, int bs, int local_blocks,
                             float* S, int64_t nb_cap) {
  if (!s || !seq_len || !S || hkv < 1 || hq % hkv != 0) return ORACLE_BAD_ARG;
  int G = hq / hkv;
#pragma omp parallel for schedule(dynamic) num_threads(g_threads)
  for (int p = 0; p < batch * hkv; ++p) {
    int i = p / hkv, g = p % hkv;
    int64_t L = seq_len[i];
    int64_t nc = n_windows(L, kernel, stride);
    if (nc > nc_cap) nc = nc_cap;
    int64_t ncand = n_candidates(L, bs, local_blocks);
    float* out = S + ((int64_t)i * hkv + g) * nb_cap;
    for (int64_t b = 0; b < nb_cap; ++b) {
      if (b >= ncand) {
        out[b] = -INFINITY;
        continue;
      }
      int64_t blo = b * bs, bhi = (b + 1) * bs;
      double total = 0.0;
      for (int hh = 0; hh < G; ++hh) {
        int h = g * G + hh;
        const float* sh = s + ((int64_t)i * hq + h) * nc_cap;
        double best = -INFINITY;
        for (int64_t j = 0; j < nc; ++j) {
          int64_t wlo = j * stride, whi = j * stride + kernel;
          if (wlo < bhi && whi > blo && (double)sh[j] > best) best = sh[j];
        }
        total += best;
      }
      out[b] = (float)total;
    }
  }
  return ORACLE_OK;
}

typedef struct {
  float score;
  int64_t index;
} ranked_block;

static float canonical(float x) {
  if (isnan(x)) return -INFINITY;
  if (x == 0.0f) return 0.0f; /* -0.0 -> +0.0 */
  return x;
}

/* Descending score, then ascending index. */
static int by_score_then_index(const void* a, const void* b) {
  const ranked_block* x = (const ranked_block*)a;
  const ranked_block* y = (const ranked_block*)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->index > y->index) - (x->index < y->index);
}

static int by_index(const void* a, const void* b) {
  int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* Top-k block selection, [P3] 三.2 ("TopK 选择 64 个高分块") and 四 (TopK64):
 * the k_eff = min(topk, ncand) candidates with the largest block score; ties
 * go to the lower block index.  sel_idx[i][g][:] lists them in ascending
 * order, padded with -1; sel_cnt[i][g] = k_eff. */
int nosa_oracle_topk(const float* S, int64_t nb_cap, const int32_t* seq_len,
                     int batch, int hkv, int bs, int local_blocks, int topk,
                     int32_t* sel_idx, int32_t* sel_cnt) {
  if (!S || !seq_len || !sel_idx || !sel_cnt || topk < 0) return ORACLE_BAD_ARG;
#pragma omp parallel for schedule(dynamic) num_threads(g_threads)
  for (int p = 0; p < batch * hkv; ++p) {
    int i = p / hkv;
    int64_t ncand = n_candidates(seq_len[i], bs, local_blocks);
    if (ncand > nb_cap) ncand = nb_cap;
    int64_t k_eff = ncand < topk ? ncand : topk;
    ranked_block* r = (ranked_block*)malloc(sizeof(ranked_block) * (ncand > 0 ? ncand : 1));
    for (int64_t b = 0; b < ncand; ++b) {
      r[b].score = canonical(S[(int64_t)p * nb_cap + b]);
      r[b].index = b;
    }
    qsort(r, (size_t)ncand, sizeof(ranked_block), by_score_then_index);
    int32_t* out = sel_idx + (int64_t)p * topk;
    for (int t = 0; t < topk; ++t) out[t] = t < k_eff ? (int32_t)r[t].index : -1;
    qsort(out, (size_t)k_eff, sizeof(int32_t), by_index);
    sel_cnt[p] = (int32_t)k_eff;
    free(r);
  }
  return ORACLE_OK;
}

/* Exact attention over the selected blocks plus the local window, [P3] 三.3
 * ("通过 TopK 选出高分块做精确注意力") and 三.2 (fixed local window):
 *   T = (U_{b in sel} [b*bs, (b+1)*bs)  U  [ncand*bs, L)) n [0, L)
 *   out[i][h] = sum_{t in T} softmax_t(scale * q.k_t) v_t
 *   lse[i][h] = log sum_{t in T} exp(scale * q.k_t)
 * q is [batch, hq, d] bf16; K, V are [T_total, hkv, d] bf16 with sequence i
 * starting at row seq_start[i]; out is fp64 [batch, hq, d]; lse fp64 [batch, hq]
 * (nullable).  Indices outside [0, ncand) are rejected. */
static int attention_view(const uint16_t* q, const kv_view* kc, const kv_view* vc,
                          const int64_t* seq_start, const int32_t* seq_len,
                          int batch, int hq, int hkv, int d, int bs,
                          int local_blocks, const int32_t* sel_idx,
                          const int32_t* sel_cnt, int topk, double scale,
                          double* out, double* lse) {
  if (!q || !kv_ok(kc) || !kv_ok(vc) || !seq_start || !seq_len || !out ||
      hkv < 1 || hq % hkv != 0 || topk < 0 || (topk > 0 && (!sel_idx || !sel_cnt)))
    return ORACLE_BAD_ARG;
  int G = hq / hkv;
  int bad = 0;
#pragma omp parallel for schedule(dynamic) num_threads(g_threads) reduction(| : bad)
  for (int p = 0; p < batch * hkv; ++p) {
    int i = p / hkv, g = p % hkv;
    int64_t L = seq_len[i];
    int64_t nb = n_blocks(L, bs);
    int64_t ncand = n_candidates(L, bs, local_blocks);
    /* Membership mask over tokens [0, L). */
    unsigned char* in_set = (unsigned char*)calloc((size_t)(L > 0 ? L : 1), 1);
    int cnt = topk > 0 ? sel_cnt[p] : 0;
    if (cnt < 0 || cnt > topk) {
      bad = 1;
      cnt = 0;
    }
    for (int t = 0; t < cnt; ++t) {
      int32_t b = sel_idx[(int64_t)p * topk + t];
      if (b < 0 || b >= ncand) {
        bad = 1;
        continue;
      }
      for (int64_t tok = (int64_t)b * bs; tok < (int64_t)(b + 1) * bs && tok < L; ++tok)
        in_set[tok] = 1;
    }
    for (int64_t tok = ncand * bs; tok < L; ++tok) in_set[tok] = 1;
    (void)nb;
    double* logit = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    for (int hh = 0; hh < G; ++hh) {
      int h = g * G + hh;
      const uint16_t* qv = q + ((int64_t)i * hq + h) * d;
      double m = -INFINITY;
      for (int64_t tok = 0; tok < L; ++tok) {
        if (!in_set[tok]) continue;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += bf16_to_f64(qv[c]) * kv_at(kc, seq_start[i] + tok, hkv, g, d, c);
        logit[tok] = scale * acc;
        if (logit[tok] > m) m = logit[tok];
      }
      double denom = 0.0;
      double* o = out + ((int64_t)i * hq + h) * d;
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      for (int64_t tok = 0; tok < L; ++tok) {
        if (!in_set[tok]) continue;
        double w = exp(logit[tok] - m);
        denom += w;
        for (int c = 0; c < d; ++c) o[c] += w * kv_at(vc, seq_start[i] + tok, hkv, g, d, c);
      }
      for (int c = 0; c < d; ++c) o[c] = denom > 0.0 ? o[c] / denom : 0.0;
      if (lse) lse[(int64_t)i * hq + h] = denom > 0.0 ? m + log(denom) : -INFINITY;
    }
    free(logit);
    free(in_set);
  }
  return bad ? ORACLE_BAD_ARG : ORACLE_OK;
}

int nosa_oracle_sparse_attention(const uint16_t* q, const uint16_t* k_cache,
                                 const uint16_t* v_cache,
                                 const int64_t* seq_start, const int32_t* seq_len,
                                 int batch, int hq, int hkv, int d, int bs,
                                 int local_blocks, const int32_t* sel_idx,
                                 const int32_t* sel_cnt, int topk, double scale,
                                 double* out, double* lse) {
  kv_view k = {k_cache, NULL, NULL}, v = {v_cache, NULL, NULL};
  return attention_view(q, &k, &v, seq_start, seq_len, batch, hq, hkv, d, bs, local_blocks, sel_idx,
                        sel_cnt, topk, scale, out, lse);
}

/* The same attention over INT8 caches: keys and values are s_t * code_t
 * (scales [T, hkv]). */
int nosa_oracle_sparse_attention_int8(const uint16_t* q, const int8_t* k_codes, const float* k_scales,
                                      const int8_t* v_codes, const float* v_scales,
                                      const int64_t* seq_start, const int32_t* seq_len, int batch,
                                      int hq, int hkv, int d, int bs, int local_blocks,
                                      const int32_t* sel_idx, const int32_t* sel_cnt, int topk,
                                      double scale, double* out, double* lse) {
  kv_view k = {NULL, k_codes, k_scales}, v = {NULL, v_codes, v_scales};
  return attention_view(q, &k, &v, seq_start, seq_len, batch, hq, hkv, d, bs, local_blocks, sel_idx,
                        sel_cnt, topk, scale, out, lse);
}
