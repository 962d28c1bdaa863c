/*
 * oracle.c -- plain, slow, fp64 CPU oracle for masked scaled-dot-product
 * attention over packed variable-length sequences, with K/V read either from
 * a contiguous packed tensor or from a paged cache through a block table.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file.  Only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it computes (for every sequence b, query head h, query row i):
 *
 *   s_j = qkScale * sum_k q[i,h,k] * K[j, h/g, k] + bias_h(i, j)   (j allowed)
 *   O[i,h,:] = sum_j softmax(s)_j * V[j, h/g, :]
 *   lse[i,h] = log sum_j exp(s_j)                                  (natural log)
 *
 * Sources (page titles as published):
 *  - nalar.dev article on padding masks, section "Masking mengubah kelayakan
 *    relasi attention": the attention formula A = softmax(QK^T/sqrt(d) + M),
 *    O = AV, and the rule that a masked pair gets zero probability.
 *  - ATB "PrefixEncoder" page, parameter table: qkScale multiplies Q*K^T;
 *    seqLen / kvSeqLen per batch on the host; key/value paged as
 *    [numBlocks, blockSize, kvHeads, headSize]; blockTables [batch, maxBlockNum];
 *    slopes per head; maskType 3/4/5/9; headNum / kvHeadNum (grouped heads).
 *  - ATB "压缩mask" (compressed mask) page, alibi section: the alibi mask is
 *    slope_h times an alibi bias plus a lower-triangular mask, with the
 *    right-aligned, square-root right-aligned and left-aligned bias forms.
 *  - ATB "MLA" page, parameter table: qNope/qRope, ctKV/kRope paged latent
 *    cache, contextLens, qseqlen, lse output.
 *  - nalar.dev article, section "Packing mengeluarkan padding dari
 *    representasi": packed tokens addressed through cumulative offsets.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *  - prefix offset: row i of sequence b sits at absolute key position
 *    iabs = i + (kvSeqLen_b - seqLen_b); causal allows j <= iabs;
 *  - right-aligned bias = slope*(j - iabs); square-root form
 *    = -slope*sqrt(iabs - j); left-aligned bias = slope*j;
 *  - masked value = -infinity (exact zero weight);
 *  - query head h uses kv head floor(h / (headNum/kvHeadNum));
 *  - blockTables row index is the batch index;
 *  - MLA: key = [ctKV ; kRope], value = ctKV, query t of batch b allows
 *    j <= contextLens_b - qseqlen_b + t.
 *  - MLA with an int8 latent cache (the MLA page's qkDescale / pvDescale
 *    rows, both [num_heads] float): qkDescale[h] turns the qNope . ctKV dot
 *    product of the stored numbers into a score (the qRope . kRope part is
 *    not rescaled), and pvDescale[h] turns the probability-weighted sum of
 *    the stored ctKV rows into the output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* element types of the tensors handed to the oracle */
#define ORC_F16 0
#define ORC_BF16 1
#define ORC_F32 2
#define ORC_I8 3 /* two's-complement signed 8-bit integer */
#define ORC_F64 4 /* already decoded (oracle_decode) */

/* mask types, numbered as on the ATB PrefixEncoder page (maskType row) plus
 * 0 = no mask (all keys of the sequence allowed). */
#define ORC_MASK_NONE 0
#define ORC_MASK_ALIBI 3
#define ORC_MASK_ALIBI_SQRT 4
#define ORC_MASK_ALIBI_LEFT 5
#define ORC_MASK_CAUSAL 9

/* ---- exact decoding of stored elements to double --------------------------
 * IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
 * bfloat16: the top 16 bits of an IEEE binary32.                           */
static double orc_half_to_double(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0) {
    v = ldexp((double)f, -24); /* subnormal: f * 2^-14 * 2^-10 */
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = ldexp((double)(f + 1024), e - 25); /* (1 + f/1024) * 2^(e-15) */
  }
  return sign ? -v : v;
}

static double orc_bf16_to_double(uint16_t b) {
  uint32_t bits = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static double orc_load(const void* base, int dtype, int64_t idx) {
  switch (dtype) {
    case ORC_F16: return orc_half_to_double(((const uint16_t*)base)[idx]);
    case ORC_BF16: return orc_bf16_to_double(((const uint16_t*)base)[idx]);
    case ORC_I8: return (double)((const int8_t*)base)[idx];
    case ORC_F64: return ((const double*)base)[idx];
    default: return (double)((const float*)base)[idx];
  }
}

/* Decodes n stored elements into doubles once (exact for every type above),
 * so that the attention loops, which read each key and value row once per
 * query row, read plain doubles instead of decoding the same element again. */
int oracle_decode(const void* src, int dtype, int64_t n, double* dst) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) dst[i] = orc_load(src, dtype, i);
  return 0;
}

/* ---- the mask rule ------------------------------------------------------
 * Returns 1 and sets *bias when key j is allowed for the query at absolute
 * position iabs, 0 when the pair is masked out.                           */
static int orc_mask_rule(int mask_type, double slope, int64_t iabs, int64_t j,
                         int64_t kv_len, double* bias) {
  *bias = 0.0;
  if (j < 0 || j >= kv_len) return 0;
  if (mask_type == ORC_MASK_NONE) return 1;
  if (j > iabs) return 0; /* lower-triangular part of every other mask type */
  switch (mask_type) {
    case ORC_MASK_ALIBI: *bias = slope * (double)(j - iabs); break;
    case ORC_MASK_ALIBI_SQRT: *bias = -slope * sqrt((double)(iabs - j)); break;
    case ORC_MASK_ALIBI_LEFT: *bias = slope * (double)j; break;
    default: break; /* causal: no bias */
  }
  return 1;
}

/* Address of key/value position j of sequence b, kv head g, element 0.
 * Contiguous: packed [nKvTokens, kvHeads, dim] with sequence b starting at
 * cu_kv[b].  Paged: [numBlocks, blockSize, kvHeads, dim]; position j lives
 * in physical block blockTables[b][j / blockSize], slot j % blockSize.     */
static int64_t orc_kv_index(const int32_t* block_tables, int64_t max_blocks,
                            int32_t block_size, int64_t cu_kv_b, int32_t b,
                            int64_t j, int32_t kv_heads, int32_t g, int32_t dim) {
  int64_t row;
  if (block_tables) {
    int64_t blk = block_tables[(int64_t)b * max_blocks + j / block_size];
    row = blk * block_size + j % block_size;
  } else {
    row = cu_kv_b + j;
  }
  return (row * kv_heads + g) * (int64_t)dim;
}

/* ---- rule-based attention ----------------------------------------------
 * q:     [nTokens, heads, d_qk]      (dtype q_dtype)
 * k:     contiguous [nKvTokens, kv_heads, d_qk] or paged [nb, bs, kv_heads, d_qk]
 * v:     same layouts with d_v
 * seq_len, kv_seq_len: [batch] (host)
 * slopes: [heads] fp32 or NULL (treated as 0)
 * rows:  flattened (token * heads + h) indices to compute, or NULL for all
 * out:   [n_rows or nTokens*heads, d_v] doubles; lse: [n_rows or ...] or NULL
 * Returns 0, or -1 on inconsistent arguments.                              */
int oracle_attention(const void* q, int q_dtype, const void* k, const void* v,
                     int kv_dtype, const int32_t* block_tables, int64_t max_blocks,
                     int32_t block_size, const int32_t* seq_len,
                     const int32_t* kv_seq_len, int32_t batch, const float* slopes,
                     int mask_type, int32_t heads, int32_t kv_heads, int32_t d_qk,
                     int32_t d_v, double qk_scale, const int64_t* rows, int64_t n_rows,
                     double* out, double* lse) {
  if (batch < 0 || heads <= 0 || kv_heads <= 0 || heads % kv_heads) return -1;
  int64_t* cu_q = (int64_t*)malloc(sizeof(int64_t) * (batch + 1));
  int64_t* cu_kv = (int64_t*)malloc(sizeof(int64_t) * (batch + 1));
  cu_q[0] = cu_kv[0] = 0;
  for (int32_t b = 0; b < batch; ++b) {
    if (seq_len[b] < 0 || kv_seq_len[b] < seq_len[b]) {
      free(cu_q); free(cu_kv);
      return -1;
    }
    cu_q[b + 1] = cu_q[b] + seq_len[b];
    cu_kv[b + 1] = cu_kv[b] + kv_seq_len[b];
  }
  const int64_t n_tokens = cu_q[batch];
  const int64_t total = rows ? n_rows : n_tokens * heads;
  const int32_t group = heads / kv_heads;

#pragma omp parallel
  {
    int64_t max_kv = 0;
    for (int32_t b = 0; b < batch; ++b)
      if (kv_seq_len[b] > max_kv) max_kv = kv_seq_len[b];
    double* s = (double*)malloc(sizeof(double) * (max_kv > 0 ? max_kv : 1));
    char* ok = (char*)malloc(max_kv > 0 ? max_kv : 1);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < total; ++r) {
      const int64_t flat = rows ? rows[r] : r;
      const int64_t t = flat / heads;
      const int32_t h = (int32_t)(flat % heads);
      int32_t b = 0;
      while (b + 1 <= batch && cu_q[b + 1] <= t) ++b; /* sequence of token t */
      const int64_t i = t - cu_q[b];
      const int64_t kv_len = kv_seq_len[b];
      const int64_t iabs = i + (kv_len - seq_len[b]);
      const int32_t g = h / group;
      const double slope = slopes ? (double)slopes[h] : 0.0;
      double m = -INFINITY;
      for (int64_t j = 0; j < kv_len; ++j) {
        double bias;
        ok[j] = (char)orc_mask_rule(mask_type, slope, iabs, j, kv_len, &bias);
        if (!ok[j]) continue;
        const int64_t kb = orc_kv_index(block_tables, max_blocks, block_size,
                                        cu_kv[b], b, j, kv_heads, g, d_qk);
        double dot = 0.0;
        for (int32_t c = 0; c < d_qk; ++c)
          dot += orc_load(q, q_dtype, (t * heads + h) * (int64_t)d_qk + c) *
                 orc_load(k, kv_dtype, kb + c);
        s[j] = qk_scale * dot + bias;
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < kv_len; ++j)
        if (ok[j]) l += exp(s[j] - m);
      double* o = out + r * (int64_t)d_v;
      for (int32_t c = 0; c < d_v; ++c) o[c] = 0.0;
      for (int64_t j = 0; j < kv_len; ++j) {
        if (!ok[j]) continue;
        const double p = exp(s[j] - m) / l;
        const int64_t vb = orc_kv_index(block_tables, max_blocks, block_size,
                                        cu_kv[b], b, j, kv_heads, g, d_v);
        for (int32_t c = 0; c < d_v; ++c) o[c] += p * orc_load(v, kv_dtype, vb + c);
      }
      if (lse) lse[r] = m + log(l);
    }
    free(s);
    free(ok);
  }
  free(cu_q);
  free(cu_kv);
  return 0;
}

/* ---- explicit full mask ---------------------------------------------------
 * Materialises M[h, i, j] for one sequence from the same rule (masked pairs
 * -inf), the way a non-compressed mask tensor would be passed.             */
int oracle_build_mask(int mask_type, const float* slopes, int32_t heads,
                      int64_t seq_len, int64_t kv_len, double* m_out) {
  if (kv_len < seq_len) return -1;
  for (int32_t h = 0; h < heads; ++h)
    for (int64_t i = 0; i < seq_len; ++i)
      for (int64_t j = 0; j < kv_len; ++j) {
        double bias;
        const double slope = slopes ? (double)slopes[h] : 0.0;
        const int ok = orc_mask_rule(mask_type, slope, i + kv_len - seq_len, j,
                                     kv_len, &bias);
        m_out[((int64_t)h * seq_len + i) * kv_len + j] = ok ? bias : -INFINITY;
      }
  return 0;
}

/* Literal evaluation of softmax(qkScale * Q K^T + M) V for ONE sequence with
 * contiguous q [L, heads, d_qk], k/v [Lkv, kv_heads, d], and a full mask
 * M [heads, L, Lkv]: forms the whole score matrix row, adds M, normalises,
 * multiplies by V.  No rule is applied here; M alone decides.             */
int oracle_attention_explicit(const void* q, int q_dtype, const void* k,
                              const void* v, int kv_dtype, int64_t seq_len,
                              int64_t kv_len, int32_t heads, int32_t kv_heads,
                              int32_t d_qk, int32_t d_v, double qk_scale,
                              const double* mask, double* out, double* lse) {
  if (heads <= 0 || kv_heads <= 0 || heads % kv_heads) return -1;
  const int32_t group = heads / kv_heads;
  double* s = (double*)malloc(sizeof(double) * (kv_len > 0 ? kv_len : 1));
  double* p = (double*)malloc(sizeof(double) * (kv_len > 0 ? kv_len : 1));
  for (int64_t i = 0; i < seq_len; ++i)
    for (int32_t h = 0; h < heads; ++h) {
      const int32_t g = h / group;
      double m = -INFINITY;
      for (int64_t j = 0; j < kv_len; ++j) {
        double dot = 0.0;
        for (int32_t c = 0; c < d_qk; ++c)
          dot += orc_load(q, q_dtype, (i * heads + h) * (int64_t)d_qk + c) *
                 orc_load(k, kv_dtype, (j * kv_heads + g) * (int64_t)d_qk + c);
        s[j] = qk_scale * dot + mask[((int64_t)h * seq_len + i) * kv_len + j];
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < kv_len; ++j) {
        p[j] = (s[j] == -INFINITY) ? 0.0 : exp(s[j] - m);
        l += p[j];
      }
      double* o = out + (i * heads + h) * (int64_t)d_v;
      for (int32_t c = 0; c < d_v; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j < kv_len; ++j)
          acc += (p[j] / l) * orc_load(v, kv_dtype, (j * kv_heads + g) * (int64_t)d_v + c);
        o[c] = acc;
      }
      if (lse) lse[i * heads + h] = m + log(l);
    }
  free(s);
  free(p);
  return 0;
}

/* Expansion of the compressed causal mask (the 128 x 128 triangle of the
 * compressed-mask page, norm scenario) into the full [seq_len, kv_len] mask
 * of one sequence.  tri[r][c] is the triangle entry for row r, column c of a
 * 128 x 128 tile; the full mask is tiled with it along the prefix-shifted
 * diagonal: a pair (i, j) whose absolute distance iabs - j lies in
 * (-128, 128) reads the triangle at the position that distance gives;
 * pairs further above the diagonal are masked, pairs further below are not. */
int oracle_expand_causal_compressed(const double* tri, int64_t seq_len,
                                    int64_t kv_len, double* m_out) {
  if (kv_len < seq_len) return -1;
  for (int64_t i = 0; i < seq_len; ++i)
    for (int64_t j = 0; j < kv_len; ++j) {
      const int64_t dist = i + kv_len - seq_len - j; /* iabs - j */
      double val;
      if (dist >= 128) val = 0.0;
      else if (dist <= -128) val = -INFINITY;
      else if (dist >= 0) val = tri[dist * 128 + 0];  /* row dist, column 0 */
      else val = tri[0 * 128 + (-dist)];               /* row 0, column -dist */
      m_out[i * kv_len + j] = val;
    }
  return 0;
}

/* ---- MLA (latent attention) ------------------------------------------------
 * qNope [tokens, heads, 512-ish d_nope], qRope [tokens, heads, d_rope]
 * ctKV  [numBlocks, blockSize, kv_heads(=1), d_nope], kRope [.., d_rope]
 * key_j = [ctKV_j ; kRope_j], value_j = ctKV_j.
 * Query t (0 <= t < qs_b) of batch b allows j <= contextLens_b - qs_b + t
 * (qs_b = 1 gives all j < contextLens_b).  Rows as in oracle_attention.
 *
 * Dequantised form (qk_descale / pv_descale non-NULL, one float per head):
 *   s_j = qkScale * (qkDescale[h] * qNope . ctKV_j + qRope . kRope_j)
 *   O   = pvDescale[h] * sum_j softmax(s)_j ctKV_j
 * with qNope and ctKV read as stored (int8 integers, or floats).  NULL
 * descales mean 1, which is the plain MLA definition above.
 *
 * Explicit mask (MLA page, parameter table, rows mask and maskType: the
 * MASK_TYPE_SPEC mask is [num_tokens, max_seq_len], fp16/bf16).  With `mask`
 * non-NULL, packed token t of batch b considers every key j < contextLens_b
 * and its score becomes s_j + mask[t * mask_cols + j] (the mask is added after
 * the scale, as in the padding-mask article's formula); the generated
 * speculative rule is not applied.  A row whose every score is -inf has no
 * allowed key: O = 0 and lse = -inf.                                      */
int oracle_mla_dequant(const void* q_nope, int qn_dtype, const void* q_rope,
                       int rope_dtype, const void* ct_kv, int kv_dtype,
                       const void* k_rope, const float* qk_descale,
                       const float* pv_descale, const int32_t* block_tables,
                       int64_t max_blocks, int32_t block_size,
                       const int32_t* context_lens, const int32_t* q_seq_len,
                       int32_t batch, int32_t heads, int32_t d_nope,
                       int32_t d_rope, double qk_scale, const void* mask,
                       int mask_dtype, int64_t mask_cols, const int64_t* rows,
                       int64_t n_rows, double* out, double* lse) {
  if (batch < 0 || heads <= 0) return -1;
  int64_t* cu_q = (int64_t*)malloc(sizeof(int64_t) * (batch + 1));
  cu_q[0] = 0;
  int64_t max_ctx = 1;
  for (int32_t b = 0; b < batch; ++b) {
    const int32_t qs = q_seq_len ? q_seq_len[b] : 1;
    if (qs < 1 || context_lens[b] < qs) { free(cu_q); return -1; }
    cu_q[b + 1] = cu_q[b] + qs;
    if (context_lens[b] > max_ctx) max_ctx = context_lens[b];
    if (mask && context_lens[b] > mask_cols) { free(cu_q); return -1; }
  }
  const int64_t total = rows ? n_rows : cu_q[batch] * heads;
#pragma omp parallel
  {
    double* s = (double*)malloc(sizeof(double) * max_ctx);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < total; ++r) {
      const int64_t flat = rows ? rows[r] : r;
      const int64_t t = flat / heads;
      const int32_t h = (int32_t)(flat % heads);
      int32_t b = 0;
      while (b + 1 <= batch && cu_q[b + 1] <= t) ++b;
      const int64_t qs = cu_q[b + 1] - cu_q[b];
      const int64_t ti = t - cu_q[b];
      const int64_t ctx = context_lens[b];
      /* last key considered: the speculative rule, or every key with an explicit mask */
      const int64_t last = mask ? ctx - 1 : ctx - qs + ti;
      const double qk_d = qk_descale ? (double)qk_descale[h] : 1.0;
      const double pv_d = pv_descale ? (double)pv_descale[h] : 1.0;
      double m = -INFINITY;
      for (int64_t j = 0; j <= last; ++j) {
        const int64_t blk = block_tables[(int64_t)b * max_blocks + j / block_size];
        const int64_t slot = blk * block_size + j % block_size;
        double dot_nope = 0.0, dot_rope = 0.0;
        for (int32_t c = 0; c < d_nope; ++c)
          dot_nope += orc_load(q_nope, qn_dtype, (t * heads + h) * (int64_t)d_nope + c) *
                      orc_load(ct_kv, kv_dtype, slot * d_nope + c);
        for (int32_t c = 0; c < d_rope; ++c)
          dot_rope += orc_load(q_rope, rope_dtype, (t * heads + h) * (int64_t)d_rope + c) *
                      orc_load(k_rope, rope_dtype, slot * d_rope + c);
        s[j] = qk_scale * (qk_d * dot_nope + dot_rope);
        if (mask) s[j] += orc_load(mask, mask_dtype, t * mask_cols + j);
        if (s[j] > m) m = s[j];
      }
      double* o = out + r * (int64_t)d_nope;
      for (int32_t c = 0; c < d_nope; ++c) o[c] = 0.0;
      if (m == -INFINITY) { /* no allowed key */
        if (lse) lse[r] = -INFINITY;
        continue;
      }
      double l = 0.0;
      for (int64_t j = 0; j <= last; ++j) l += exp(s[j] - m);
      for (int64_t j = 0; j <= last; ++j) {
        const double p = exp(s[j] - m) / l;
        const int64_t blk = block_tables[(int64_t)b * max_blocks + j / block_size];
        const int64_t slot = blk * block_size + j % block_size;
        for (int32_t c = 0; c < d_nope; ++c)
          o[c] += p * orc_load(ct_kv, kv_dtype, slot * d_nope + c);
      }
      for (int32_t c = 0; c < d_nope; ++c) o[c] *= pv_d;
      if (lse) lse[r] = m + log(l);
    }
    free(s);
  }
  free(cu_q);
  return 0;
}

/* The MLA definition with every tensor in one floating dtype. */
int oracle_mla(const void* q_nope, const void* q_rope, const void* ct_kv,
               const void* k_rope, int dtype, const int32_t* block_tables,
               int64_t max_blocks, int32_t block_size, const int32_t* context_lens,
               const int32_t* q_seq_len, int32_t batch, int32_t heads,
               int32_t d_nope, int32_t d_rope, double qk_scale,
               const int64_t* rows, int64_t n_rows, double* out, double* lse) {
  return oracle_mla_dequant(q_nope, dtype, q_rope, dtype, ct_kv, dtype, k_rope, NULL, NULL,
                            block_tables, max_blocks, block_size, context_lens, q_seq_len,
                            batch, heads, d_nope, d_rope, qk_scale, NULL, 0, 0, rows, n_rows,
                            out, lse);
}

/* ---- merge of partial results over disjoint key ranges --------------------
 * Given, for each row, n_parts partial outputs O_p (each normalised over its
 * own key range) and their log-sum-exps lse_p, the result over the union of
 * the ranges is lse = log sum_p exp(lse_p), O = sum_p exp(lse_p - lse) O_p.
 * This is the combination the MLA page's ring mode returns the lse for.
 * o_parts [n_parts, n_rows, d_v], lse_parts [n_parts, n_rows].           */
int oracle_lse_merge(int32_t n_parts, int64_t n_rows, int32_t d_v,
                     const double* o_parts, const double* lse_parts, double* out,
                     double* lse) {
  for (int64_t r = 0; r < n_rows; ++r) {
    double m = -INFINITY;
    for (int32_t p = 0; p < n_parts; ++p)
      if (lse_parts[p * n_rows + r] > m) m = lse_parts[p * n_rows + r];
    double l = 0.0;
    for (int32_t p = 0; p < n_parts; ++p) {
      const double x = lse_parts[p * n_rows + r];
      l += (x == -INFINITY) ? 0.0 : exp(x - m);
    }
    const double total = m + log(l);
    for (int32_t c = 0; c < d_v; ++c) {
      double acc = 0.0;
      for (int32_t p = 0; p < n_parts; ++p) {
        const double x = lse_parts[p * n_rows + r];
        if (x == -INFINITY) continue;
        acc += exp(x - total) * o_parts[((int64_t)p * n_rows + r) * d_v + c];
      }
      out[r * d_v + c] = acc;
    }
    if (lse) lse[r] = total;
  }
  return 0;
}
