/*
 * attn_oracle.c -- plain, slow, float64 CPU oracle for the three attention operations.
 *
 * TEST INFRASTRUCTURE ONLY. This file is not part of the product. Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg may load it. It shares no code with the CUDA
 * path: no headers, no helpers, no tables.
 *
 * Every function is the plain definition of the result, written out with no blocking, no
 * fusion and no online (streaming) softmax:
 *
 *   attention   o_i = sum_j softmax_j(scale * q_i . k_j + mask_ij) v_j
 *               "paddle.nn.functional.sparse_attention" (Paddle 2.3 API doc), formula
 *               result = softmax(Q K^T / sqrt(d)) V; the same formula as the manual_attention
 *               section of "高效 AI 模型开发：PyTorch torch.nn.attention 报错排查与高效替代方法".
 *   varlen TND  "aclnnFlashAttentionVarLenScore" (CANN 8.5 API doc), 功能说明 and 约束说明:
 *               packed [T, N, D] tensors, cumulative lengths with B entries and no leading 0,
 *               GQA/MQA when Nq/Nkv > 1, lower-triangular (causal) masks.
 *   CSR sparse  "paddle.nn.functional.sparse_attention", 参数: offset [B,H,S+1] row pointer,
 *               columns [B,H,nnz]; softmax over the stored entries of each row only.
 *   merge       "npu_ring_attention_update" (MindSpeed op doc), 小算子等价计算逻辑: lane-wise
 *               max/sum update over [B,N,S,8] statistics, output rescaled with lane 0.
 *   masked      "aclnnFlashAttentionVarLenScore", 约束说明: band limits (preTokens/nextTokens),
 *               an explicit mask (attenMaskOptional) and a value head size with qD == kD >= vD;
 *               the readings are stated above oracle_attn_fwd_ext.
 *
 * Statistics convention (the pages only imply it through the merge, which takes exp of
 * differences of maxima): softmax_max = max_j of the scaled score in natural-log units and
 * softmax_sum = sum_j exp(score_j - softmax_max).
 *
 * Rows with no visible key (an empty key range, or a causal bottom-right row above the band)
 * give out = 0, max = -inf, sum = 0.
 *
 * Element types of the inputs: 0 = float64, 1 = float32, 2 = bfloat16 (raw 16-bit patterns).
 * Widening float32 or bf16 to double is exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F64 0
#define ORC_F32 1
#define ORC_BF16 2

#define ORC_BHSD 0
#define ORC_TND 1

#define ORC_MASK_NONE 0
#define ORC_MASK_TOPLEFT 1      /* key j visible iff j <= i                 */
#define ORC_MASK_BOTTOMRIGHT 2  /* key j visible iff j <= i + Skv_b - Sq_b  */

static double ld(const void *base, int64_t idx, int et) {
  if (et == ORC_F64) return ((const double *)base)[idx];
  if (et == ORC_F32) return (double)((const float *)base)[idx];
  {
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
}

/* Offset of element (sequence b, token i of that sequence, head h, dim d).
 * BHSD: tensor [B, N, S, D]; TND: tensor [T, N, D] with the sequence starting at token t0. */
static int64_t offs(int layout, int64_t b, int64_t t0, int64_t i, int64_t h, int64_t d,
                    int64_t N, int64_t S, int64_t D) {
  if (layout == ORC_BHSD) return ((b * N + h) * S + i) * D + d;
  return ((t0 + i) * N + h) * D + d;
}

/* Start token and length of sequence b. */
static void seq_range(int layout, const int32_t *cu, int64_t b, int64_t S, int64_t *t0, int64_t *len) {
  if (layout == ORC_BHSD) {
    *t0 = 0;
    *len = S;
  } else {
    int64_t lo = b == 0 ? 0 : cu[b - 1];
    *t0 = lo;
    *len = (int64_t)cu[b] - lo;
  }
}

/* Number of keys visible to query row i: keys 0 .. n-1 (masks here are prefixes). */
static int64_t visible_keys(int mask_mode, int64_t i, int64_t sq, int64_t sk) {
  int64_t last;
  if (mask_mode == ORC_MASK_NONE) return sk;
  last = (mask_mode == ORC_MASK_TOPLEFT) ? i : i + sk - sq;
  if (last < 0) return 0;
  return last + 1 < sk ? last + 1 : sk;
}

/*
 * One query row of dense / varlen attention (the definition, over all visible keys).
 * o[D] receives the output row; *m and *l the statistics. s is scratch of length >= nk.
 */
static void attn_row(const void *q, const void *k, const void *v, int et, int layout,
                     int64_t b, int64_t tq0, int64_t tk0, int64_t i, int64_t h, int64_t g,
                     int64_t nk, int64_t Nq, int64_t Nkv, int64_t Sq, int64_t Skv, int64_t D,
                     double scale, double *s, double *o, double *m, double *l) {
  int64_t j, d;
  double mx = -INFINITY, sum = 0.0;
  for (d = 0; d < D; ++d) o[d] = 0.0;
  if (nk <= 0) {
    *m = -INFINITY;
    *l = 0.0;
    return;
  }
  /* scores s_j = scale * sum_d q[i,h,d] k[j,g,d] */
  for (j = 0; j < nk; ++j) {
    double acc = 0.0;
    for (d = 0; d < D; ++d)
      acc += ld(q, offs(layout, b, tq0, i, h, d, Nq, Sq, D), et) *
             ld(k, offs(layout, b, tk0, j, g, d, Nkv, Skv, D), et);
    s[j] = scale * acc;
    if (s[j] > mx) mx = s[j];
  }
  /* softmax weights relative to the row maximum, and their sum */
  for (j = 0; j < nk; ++j) {
    s[j] = exp(s[j] - mx);
    sum += s[j];
  }
  /* o = sum_j p_j v_j with p_j = s_j / sum */
  for (j = 0; j < nk; ++j)
    for (d = 0; d < D; ++d) o[d] += s[j] * ld(v, offs(layout, b, tk0, j, g, d, Nkv, Skv, D), et);
  for (d = 0; d < D; ++d) o[d] /= sum;
  *m = mx;
  *l = sum;
}

static int check_cu(const int32_t *cu, int64_t B, int64_t T) {
  int64_t b, prev = 0;
  for (b = 0; b < B; ++b) {
    if (cu[b] < prev) return -2;
    prev = cu[b];
  }
  if (B > 0 && prev != T) return -2;
  return 0;
}

/*
 * Dense (BHSD) or packed varlen (TND) attention forward, all rows.
 * out: double, same layout as q ([B,Nq,Sq,D] or [Tq,Nq,D]).
 * smax/ssum: double, [B,Nq,Sq] (BHSD) or [Tq,Nq] (TND).
 * GQA: query head h reads key/value head h / (Nq/Nkv).
 * Returns 0, -1 on bad shapes, -2 on bad cumulative lengths.
 */
int oracle_attn_fwd(const void *q, const void *k, const void *v, int et,
                    const int32_t *cu_q, const int32_t *cu_kv, int B, int Sq, int Skv,
                    int Nq, int Nkv, int D, double scale, int mask_mode, int layout,
                    double *out, double *smax, double *ssum) {
  int64_t nrows, r;
  int64_t group;
  if (B < 0 || Sq < 0 || Skv < 0 || Nq <= 0 || Nkv <= 0 || D <= 0 || Nq % Nkv) return -1;
  if (layout == ORC_TND && (check_cu(cu_q, B, Sq) || check_cu(cu_kv, B, Skv))) return -2;
  group = Nq / Nkv;
  /* one work item per (query token, head) */
  nrows = (layout == ORC_BHSD ? (int64_t)B * Sq : (int64_t)Sq) * Nq;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 16)
    for (r = 0; r < nrows; ++r) {
      int64_t h = r % Nq, tok = r / Nq, b, i, tq0, tk0, lq, lk, nk;
      double m, l;
      if (layout == ORC_BHSD) {
        b = tok / Sq;
        i = tok % Sq;
      } else {
        b = 0;
        while (cu_q[b] <= tok) ++b; /* sequence holding token tok */
        i = tok - (b == 0 ? 0 : cu_q[b - 1]);
      }
      seq_range(layout, cu_q, b, Sq, &tq0, &lq);
      seq_range(layout, cu_kv, b, Skv, &tk0, &lk);
      nk = visible_keys(mask_mode, i, lq, lk);
      {
        int64_t oo = offs(layout, b, tq0, i, h, 0, Nq, Sq, D);
        int64_t so = layout == ORC_BHSD ? ((int64_t)b * Nq + h) * Sq + i : (tq0 + i) * Nq + h;
        attn_row(q, k, v, et, layout, b, tq0, tk0, i, h, h / group, nk, Nq, Nkv, Sq, Skv, D,
                 scale, s, out + oo, &m, &l);
        smax[so] = m;
        ssum[so] = l;
      }
    }
    free(s);
  }
  return 0;
}

/*
 * The same forward for a chosen set of rows only (for checks at full problem sizes).
 * Row r is (head rows_h[r], query token rows_t[r]); the token is b*Sq + i for BHSD and the
 * packed token index for TND. out_rows is [n, D]; m_rows and l_rows are [n].
 */
int oracle_attn_fwd_rows(const void *q, const void *k, const void *v, int et,
                         const int32_t *cu_q, const int32_t *cu_kv, int B, int Sq, int Skv,
                         int Nq, int Nkv, int D, double scale, int mask_mode, int layout,
                         const int32_t *rows_h, const int64_t *rows_t, int64_t n,
                         double *out_rows, double *m_rows, double *l_rows) {
  int64_t r, group;
  if (B < 0 || Sq < 0 || Skv < 0 || Nq <= 0 || Nkv <= 0 || D <= 0 || Nq % Nkv) return -1;
  if (layout == ORC_TND && (check_cu(cu_q, B, Sq) || check_cu(cu_kv, B, Skv))) return -2;
  group = Nq / Nkv;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 1)
    for (r = 0; r < n; ++r) {
      int64_t h = rows_h[r], tok = rows_t[r], b, i, tq0, tk0, lq, lk, nk;
      if (layout == ORC_BHSD) {
        b = tok / Sq;
        i = tok % Sq;
      } else {
        b = 0;
        while (cu_q[b] <= tok) ++b;
        i = tok - (b == 0 ? 0 : cu_q[b - 1]);
      }
      seq_range(layout, cu_q, b, Sq, &tq0, &lq);
      seq_range(layout, cu_kv, b, Skv, &tk0, &lk);
      nk = visible_keys(mask_mode, i, lq, lk);
      attn_row(q, k, v, et, layout, b, tq0, tk0, i, h, h / group, nk, Nq, Nkv, Sq, Skv, D, scale,
               s, out_rows + r * D, m_rows + r, l_rows + r);
    }
    free(s);
  }
  return 0;
}

/*
 * Masked forward with band limits, an explicit mask and a value head size of its own
 * ("aclnnFlashAttentionVarLenScore", 约束说明: preTokens / nextTokens band, attenMaskOptional,
 * qD == kD >= vD). The page only lists these inputs; the table that defines the sparse modes is
 * not on it, so the readings are:
 *   band (mode 3):      key j is visible to query row i iff i - pre <= j <= i + next, with i and j
 *                       positions within the sequence (top-left aligned); pre + next >= 0 so the
 *                       band is not empty ("preTokens and nextTokens must intersect").
 *   explicit mask:      uint8, 1 = masked out (the page forbids a row of all 1s, so 1 excludes);
 *                       element (b, i, j) at mask[b * mask_bstride + i * mask_rstride + j].
 *                       Combined with the mode by AND: a key must pass both.
 *   value head size Dv: v is [.., Nkv, Dv] in the q/k layout, out is [.., Nq, Dv].
 * Rows with no visible key give out = 0, max = -inf, sum = 0, as elsewhere here.
 */
#define ORC_MASK_BAND 3

static int key_visible(int mask_mode, int64_t i, int64_t j, int64_t sq, int64_t sk, int64_t pre,
                       int64_t next, const uint8_t *mask, int64_t mrow, int64_t mask_rstride) {
  if (j < 0 || j >= sk) return 0;
  if (mask_mode == ORC_MASK_TOPLEFT && j > i) return 0;
  if (mask_mode == ORC_MASK_BOTTOMRIGHT && j > i + sk - sq) return 0;
  if (mask_mode == ORC_MASK_BAND && (j < i - pre || j > i + next)) return 0;
  if (mask != NULL && mask[mrow + i * mask_rstride + j] != 0) return 0;
  return 1;
}

/* One query row over every key of its sequence, each tested by key_visible. */
static void attn_row_ext(const void *q, const void *k, const void *v, int et, int layout,
                         int64_t b, int64_t tq0, int64_t tk0, int64_t i, int64_t h, int64_t g,
                         int64_t lq, int64_t lk, int64_t Nq, int64_t Nkv, int64_t Sq, int64_t Skv,
                         int64_t Dqk, int64_t Dv, double scale, int mask_mode, int64_t pre,
                         int64_t next, const uint8_t *mask, int64_t mask_bstride,
                         int64_t mask_rstride, double *s, double *o, double *m, double *l) {
  int64_t j, d, nvis = 0;
  double mx = -INFINITY, sum = 0.0;
  for (d = 0; d < Dv; ++d) o[d] = 0.0;
  for (j = 0; j < lk; ++j) {
    double acc = 0.0;
    if (!key_visible(mask_mode, i, j, lq, lk, pre, next, mask, b * mask_bstride, mask_rstride)) {
      s[j] = -INFINITY;
      continue;
    }
    for (d = 0; d < Dqk; ++d)
      acc += ld(q, offs(layout, b, tq0, i, h, d, Nq, Sq, Dqk), et) *
             ld(k, offs(layout, b, tk0, j, g, d, Nkv, Skv, Dqk), et);
    s[j] = scale * acc;
    if (s[j] > mx) mx = s[j];
    ++nvis;
  }
  if (nvis == 0) {
    *m = -INFINITY;
    *l = 0.0;
    return;
  }
  for (j = 0; j < lk; ++j) {
    s[j] = s[j] == -INFINITY ? 0.0 : exp(s[j] - mx);
    sum += s[j];
  }
  for (j = 0; j < lk; ++j)
    if (s[j] != 0.0)
      for (d = 0; d < Dv; ++d) o[d] += s[j] * ld(v, offs(layout, b, tk0, j, g, d, Nkv, Skv, Dv), et);
  for (d = 0; d < Dv; ++d) o[d] /= sum;
  *m = mx;
  *l = sum;
}

static int ext_args_bad(int B, int Sq, int Skv, int Nq, int Nkv, int Dqk, int Dv, int mask_mode,
                        int64_t pre, int64_t next) {
  if (B < 0 || Sq < 0 || Skv < 0 || Nq <= 0 || Nkv <= 0 || Dqk <= 0 || Nq % Nkv) return 1;
  if (Dv <= 0 || Dv > Dqk) return 1;
  if (mask_mode < ORC_MASK_NONE || mask_mode > ORC_MASK_BAND) return 1;
  if (mask_mode == ORC_MASK_BAND && pre + next < 0) return 1;
  return 0;
}

/* Sequence b and position i of query token tok (b*Sq + i for BHSD, packed index for TND). */
static void locate(int layout, const int32_t *cu_q, int64_t Sq, int64_t tok, int64_t *b, int64_t *i) {
  if (layout == ORC_BHSD) {
    *b = tok / Sq;
    *i = tok % Sq;
  } else {
    int64_t bb = 0;
    while (cu_q[bb] <= tok) ++bb;
    *b = bb;
    *i = tok - (bb == 0 ? 0 : cu_q[bb - 1]);
  }
}

/*
 * All rows: out is [B,Nq,Sq,Dv] (BHSD) or [Tq,Nq,Dv] (TND); smax/ssum as for oracle_attn_fwd.
 * Returns 0, -1 on bad arguments, -2 on bad cumulative lengths.
 */
int oracle_attn_fwd_ext(const void *q, const void *k, const void *v, int et, const int32_t *cu_q,
                        const int32_t *cu_kv, int B, int Sq, int Skv, int Nq, int Nkv, int Dqk,
                        int Dv, double scale, int mask_mode, int64_t pre, int64_t next,
                        const uint8_t *mask, int64_t mask_bstride, int64_t mask_rstride,
                        int layout, double *out, double *smax, double *ssum) {
  int64_t nrows, r, group;
  if (ext_args_bad(B, Sq, Skv, Nq, Nkv, Dqk, Dv, mask_mode, pre, next)) return -1;
  if (layout == ORC_TND && (check_cu(cu_q, B, Sq) || check_cu(cu_kv, B, Skv))) return -2;
  group = Nq / Nkv;
  nrows = (layout == ORC_BHSD ? (int64_t)B * Sq : (int64_t)Sq) * Nq;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 16)
    for (r = 0; r < nrows; ++r) {
      int64_t h = r % Nq, b, i, tq0, tk0, lq, lk, so;
      locate(layout, cu_q, Sq, r / Nq, &b, &i);
      seq_range(layout, cu_q, b, Sq, &tq0, &lq);
      seq_range(layout, cu_kv, b, Skv, &tk0, &lk);
      so = layout == ORC_BHSD ? ((int64_t)b * Nq + h) * Sq + i : (tq0 + i) * Nq + h;
      attn_row_ext(q, k, v, et, layout, b, tq0, tk0, i, h, h / group, lq, lk, Nq, Nkv, Sq, Skv,
                   Dqk, Dv, scale, mask_mode, pre, next, mask, mask_bstride, mask_rstride, s,
                   out + offs(layout, b, tq0, i, h, 0, Nq, Sq, Dv), smax + so, ssum + so);
    }
    free(s);
  }
  return 0;
}

/* Chosen rows only (head rows_h[r], query token rows_t[r]); out_rows is [n, Dv]. */
int oracle_attn_fwd_ext_rows(const void *q, const void *k, const void *v, int et,
                             const int32_t *cu_q, const int32_t *cu_kv, int B, int Sq, int Skv,
                             int Nq, int Nkv, int Dqk, int Dv, double scale, int mask_mode,
                             int64_t pre, int64_t next, const uint8_t *mask, int64_t mask_bstride,
                             int64_t mask_rstride, int layout, const int32_t *rows_h,
                             const int64_t *rows_t, int64_t n, double *out_rows, double *m_rows,
                             double *l_rows) {
  int64_t r, group;
  if (ext_args_bad(B, Sq, Skv, Nq, Nkv, Dqk, Dv, mask_mode, pre, next)) return -1;
  if (layout == ORC_TND && (check_cu(cu_q, B, Sq) || check_cu(cu_kv, B, Skv))) return -2;
  group = Nq / Nkv;
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(Skv > 0 ? Skv : 1));
#pragma omp for schedule(dynamic, 1)
    for (r = 0; r < n; ++r) {
      int64_t h = rows_h[r], b, i, tq0, tk0, lq, lk;
      locate(layout, cu_q, Sq, rows_t[r], &b, &i);
      seq_range(layout, cu_q, b, Sq, &tq0, &lq);
      seq_range(layout, cu_kv, b, Skv, &tk0, &lk);
      attn_row_ext(q, k, v, et, layout, b, tq0, tk0, i, h, h / group, lq, lk, Nq, Nkv, Sq, Skv,
                   Dqk, Dv, scale, mask_mode, pre, next, mask, mask_bstride, mask_rstride, s,
                   out_rows + r * Dv, m_rows + r, l_rows + r);
    }
    free(s);
  }
  return 0;
}

/*
 * CSR-sparse attention ("paddle.nn.functional.sparse_attention"): for every (b, h, i) the
 * softmax runs over the stored entries c in [offset[i], offset[i+1]) of that (b, h) slice,
 * key j = columns[c], scale 1/sqrt(D). q, k, v, out are [B, H, S, D].
 * offset is [B, H, S+1] (a row pointer: offset[0] = 0, non-decreasing, offset[S] <= nnz_cap);
 * columns is [B, H, nnz_cap]. An empty row gives out = 0.
 * Returns 0, -1 on bad shapes, -2 on a bad row pointer or a column out of [0, S).
 */
int oracle_sparse_csr(const void *q, const void *k, const void *v, int et, const int32_t *offset,
                      const int32_t *columns, int B, int H, int S, int D, int64_t nnz_cap,
                      double *out) {
  int64_t bh, r, nrows = (int64_t)B * H * S;
  double scale = 1.0 / sqrt((double)D);
  int bad = 0;
  if (B < 0 || H < 0 || S < 0 || D <= 0 || nnz_cap < 0) return -1;
  for (bh = 0; bh < (int64_t)B * H; ++bh) {
    const int32_t *op = offset + bh * (S + 1);
    const int32_t *cp = columns + bh * nnz_cap;
    if (op[0] != 0 || op[S] > nnz_cap) return -2;
    for (r = 0; r < S; ++r)
      if (op[r + 1] < op[r]) return -2;
    for (r = 0; r < op[S]; ++r)
      if (cp[r] < 0 || cp[r] >= S) return -2;
  }
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(nnz_cap > 0 ? nnz_cap : 1));
#pragma omp for schedule(dynamic, 16)
    for (r = 0; r < nrows; ++r) {
      int64_t bhi = r / S, i = r % S, c, d;
      const int32_t *op = offset + bhi * (S + 1);
      const int32_t *cp = columns + bhi * nnz_cap;
      int64_t c0 = op[i], c1 = op[i + 1];
      double mx = -INFINITY, sum = 0.0;
      double *o = out + r * D;
      const int64_t rowq = r * D, base = bhi * (int64_t)S * D;
      for (d = 0; d < D; ++d) o[d] = 0.0;
      if (c1 <= c0) continue;
      for (c = c0; c < c1; ++c) {
        int64_t j = cp[c];
        double acc = 0.0;
        for (d = 0; d < D; ++d) acc += ld(q, rowq + d, et) * ld(k, base + j * D + d, et);
        s[c - c0] = scale * acc;
        if (s[c - c0] > mx) mx = s[c - c0];
      }
      for (c = c0; c < c1; ++c) {
        s[c - c0] = exp(s[c - c0] - mx);
        sum += s[c - c0];
      }
      for (c = c0; c < c1; ++c) {
        int64_t j = cp[c];
        for (d = 0; d < D; ++d) o[d] += s[c - c0] * ld(v, base + j * D + d, et);
      }
      for (d = 0; d < D; ++d) o[d] /= sum;
    }
    free(s);
  }
  return bad;
}

/*
 * Ring-attention partial merge ("npu_ring_attention_update", 小算子等价计算逻辑 and 前向接口).
 * Lane-wise over the 8 statistic lanes of each row:
 *     m = max(pm, cm), ps' = ps * exp(pm - m), cs' = cs * exp(cm - m), l = ps' + cs'.
 * Output: out = prev * (ps'[0] / l[0]) + cur * (cs'[0] / l[0]) with lane 0 of each row, in
 * double (the caller rounds to the output type).
 * Layouts (layout argument):
 *   ORC_BHSD ("SBH" on the page): outputs [S, B, N*D], statistics [B, N, S, 8];
 *   ORC_TND: outputs [T, N*D] with T = S (B unused), statistics [T, N, 8] (token-major, as
 *            the TND tensors themselves).
 * Where both maxima are -inf (both sides empty) the lane gives m = -inf, ps' = cs' = 0, l = 0,
 * and where the lane-0 sum l is 0 the output scales are 0 (the plain formula would divide
 * 0 by 0).
 */
int oracle_merge(const void *prev_out, const double *prev_max, const double *prev_sum,
                 const void *cur_out, const double *cur_max, const double *cur_sum, int et,
                 int S, int B, int N, int D, int layout, double *out, double *out_max,
                 double *out_sum) {
  int64_t row, nrows;
  if (S < 0 || N <= 0 || D <= 0) return -1;
  if (layout == ORC_BHSD && B < 0) return -1;
  nrows = layout == ORC_BHSD ? (int64_t)B * N * S : (int64_t)S * N;
#pragma omp parallel for schedule(static)
  for (row = 0; row < nrows; ++row) {
    int64_t lane, d, obase;
    double ps_scaled[8], cs_scaled[8], l[8], po, co;
    if (layout == ORC_BHSD) {
      /* row = (b * N + n) * S + s, the statistics' own order; output (s, b, n*D + d) */
      int64_t s = row % S, bn = row / S, n = bn % N, b = bn / N;
      obase = ((s * B + b) * N + n) * (int64_t)D;
    } else {
      /* row = t * N + n for both the statistics and the output */
      obase = row * (int64_t)D;
    }
    for (lane = 0; lane < 8; ++lane) {
      int64_t x = row * 8 + lane;
      double pm = prev_max[x], cm = cur_max[x];
      double m = pm > cm ? pm : cm;
      if (m == -INFINITY) {
        ps_scaled[lane] = 0.0;
        cs_scaled[lane] = 0.0;
      } else {
        ps_scaled[lane] = prev_sum[x] * exp(pm - m);
        cs_scaled[lane] = cur_sum[x] * exp(cm - m);
      }
      l[lane] = ps_scaled[lane] + cs_scaled[lane];
      out_max[x] = m;
      out_sum[x] = l[lane];
    }
    po = l[0] != 0.0 ? ps_scaled[0] / l[0] : 0.0;
    co = l[0] != 0.0 ? cs_scaled[0] / l[0] : 0.0;
    for (d = 0; d < D; ++d) {
      int64_t x = obase + d;
      out[x] = ld(prev_out, x, et) * po + ld(cur_out, x, et) * co;
    }
  }
  return 0;
}

/*
 * Round a double to bfloat16 (8 significant bits, float32's exponent range), round to
 * nearest with ties to even, and return the 16-bit pattern. The rounding is done once, on
 * the double itself: the significand is scaled to an integer grid and rounded with
 * nearbyint (the default rounding mode is to-nearest-even), then scaled back exactly.
 */
uint16_t oracle_round_bf16(double x) {
  double a, r;
  int e;
  float f;
  uint32_t bits;
  if (isnan(x)) return 0x7FC0;
  if (isinf(x)) return signbit(x) ? 0xFF80 : 0x7F80;
  a = fabs(x);
  if (a < 0x1p-126) {
    r = nearbyint(a * 0x1p133) * 0x1p-133; /* subnormal grid: spacing 2^-133 */
  } else {
    double m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
    r = ldexp(nearbyint(m * 256.0), e - 8);
  }
  f = r >= 0x1p128 ? INFINITY : (float)r; /* exact: r has at most 8 significant bits */
  if (signbit(x)) f = -f;
  memcpy(&bits, &f, 4);
  return (uint16_t)(bits >> 16);
}

void oracle_round_bf16_array(const double *x, int64_t n, uint16_t *out) {
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < n; ++i) out[i] = oracle_round_bf16(x[i]);
}

/*
 * Round a double to IEEE binary16 (11 significant bits, exponents -14 .. 15, subnormal spacing
 * 2^-24), round to nearest with ties to even, and return the 16-bit pattern. The merge page
 * lists float16 among its output types and casts the float32 result once to the output type
 * ("npu_ring_attention_update", 小算子等价计算逻辑: the final .to(origin_dtype)); this is that
 * cast, done once on the double itself with nearbyint on the integer grid of the value's binade.
 */
uint16_t oracle_round_f16(double x) {
  double a, r, m;
  int e;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return 0x7E00;
  if (isinf(x)) return (uint16_t)(sign | 0x7C00);
  a = fabs(x);
  if (a < 0x1p-14) {
    r = nearbyint(a * 0x1p24); /* subnormal grid; 1024 is the smallest normal, 0x0400 */
    return (uint16_t)(sign | (uint16_t)r);
  }
  m = frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
  r = ldexp(nearbyint(m * 2048.0), e - 11);
  if (r >= 65536.0) return (uint16_t)(sign | 0x7C00); /* past the largest finite value */
  m = frexp(r, &e);                                    /* r = 2^(e-1) * (2m), 2m in [1, 2) */
  return (uint16_t)(sign | (uint16_t)((e - 1 + 15) << 10) | (uint16_t)((2.0 * m - 1.0) * 1024.0));
}

void oracle_round_f16_array(const double *x, int64_t n, uint16_t *out) {
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < n; ++i) out[i] = oracle_round_f16(x[i]);
}
