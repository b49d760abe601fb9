/*
 * hs2_oracle.c -- plain, slow, single-threaded fp64 definition of the
 * HySparse2 Cross-Decoder Hybrid-Block decode attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header or constant
 * generator with the CUDA library.
 *
 * What it follows (HySparse2 announcement, "KV Reuse" section and the
 * token-level selection / forced-window paragraphs that follow it):
 *   - each Hybrid Block is one full-attention layer followed by sparse layers;
 *     the full layer, while computing its own attention, picks important
 *     positions from its attention scores, and the sparse layers reuse its
 *     KV cache and its selection indices directly;
 *   - selection is per token (not per block): the most recent 128 tokens are
 *     always taken, plus 1,024 global tokens chosen from outside that window;
 *   - the window and the global tokens are read from the same shared KV cache
 *     in one sparse-attention computation (no separate sliding-window branch);
 *   - (paragraphs on first-generation HySparse) the block-level selection it
 *     used, as a comparator at the same token budget (orc_select_blocks);
 *   - ("KV Bridging" paragraphs) each Cross-Decoder full-attention layer
 *     builds its KV cache from the matching Self-Decoder layer's input hidden
 *     state through its own K/V projections (orc_kv_bridge and the encoders
 *     at the end of this file).
 *
 * Readings fixed where the pages are silent:
 *   - score[t] for a KV head = sum over the query heads of its GQA group of
 *     the full layer's softmax probability p_{h,t};
 *   - top-k over t < T-W by (score descending, index ascending); if there
 *     are no more than k_global such positions, all of them are taken;
 *   - query head h uses KV head floor(h / G); softmax scale 1/sqrt(d);
 *   - the current token is already in the cache at position T-1, so the
 *     window is [max(0,T-W), T);
 *   - E4M3 values are dequantised as decode(code) * scale[slot, kv_head].
 *
 * Every value is widened exactly to double from the stored bytes (fp32, the
 * bf16 bit pattern, or the E4M3 code times its fp32 scale); all arithmetic
 * is double.  Parity-pinned by tests/test_oracle_pins.py (brute force in
 * extended precision, closed forms, invariants, exhaustive ranking).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };

/* ---- exact widening of the stored element types ------------------------ */

/* OCP FP8 E4M3 ("fn" flavour): 1 sign, 4 exponent (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN.  Exponent field 0 is subnormal. */
double orc_e4m3_value(uint8_t code) {
  int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m, -9); /* (m/8) * 2^(1-7) */
  else
    mag = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -mag : mag;
}

static double bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

static double elem(const void *base, int dtype, int64_t i) {
  switch (dtype) {
  case ORC_F32: return (double)((const float *)base)[i];
  case ORC_BF16: return bf16_value(((const uint16_t *)base)[i]);
  case ORC_E4M3: return orc_e4m3_value(((const uint8_t *)base)[i]);
  }
  return NAN;
}

/* One K or V cache: rows [num_slots, num_kv_heads, head_dim]. */
typedef struct {
  const void *data;
  const float *scale; /* [num_slots, num_kv_heads], E4M3 only */
  int dtype;
  int num_kv_heads;
  int head_dim;
} orc_cache;

static void cache_row(const orc_cache *c, int64_t slot, int kvh, double *row) {
  int64_t base = (slot * c->num_kv_heads + kvh) * (int64_t)c->head_dim;
  double s = 1.0;
  if (c->dtype == ORC_E4M3) s = (double)c->scale[slot * c->num_kv_heads + kvh];
  for (int i = 0; i < c->head_dim; ++i) row[i] = elem(c->data, c->dtype, base + i) * s;
}

/* Logical position t of sequence b -> physical slot.  A NULL page table means
 * the contiguous layout, where sequence b owns slots [b*page_size, (b+1)*page_size). */
static int64_t slot_of(const int32_t *page_table, int max_pages, int page_size, int b, int64_t t) {
  if (!page_table) return (int64_t)b * page_size + t;
  int64_t page = page_table[(int64_t)b * max_pages + t / page_size];
  return page * page_size + t % page_size;
}

/* ---- selection: the definition, written as a sort ----------------------- */

typedef struct {
  double score;
  int64_t t;
} orc_cand;

/* score descending, then position ascending */
static int cand_order(const void *a, const void *b) {
  const orc_cand *x = (const orc_cand *)a, *y = (const orc_cand *)b;
  if (x->score > y->score) return -1;
  if (x->score < y->score) return 1;
  return (x->t > y->t) - (x->t < y->t);
}

/*
 * Full-attention layer + token selection for one (sequence b, KV head kvh).
 *
 * q        : [num_q_heads, head_dim] elements of the query for sequence b
 *            (dtype q_dtype; the caller points at q + b*Hq*d)
 * T        : context length of sequence b (>= 1)
 * outputs  : out   [G, head_dim]  attention output of heads kvh*G .. kvh*G+G-1
 *            lse   [G]            log-sum-exp of the scaled logits
 *            score [T]            group probability sum, every position
 *            idx   [window + k_global] selected slots, ascending logical
 *                                 position, -1 padded
 * returns the number of selected positions, or -1 on allocation failure.
 */
int orc_full_unit(const void *q, int q_dtype, int num_q_heads, const orc_cache *kc,
                  const orc_cache *vc, const int32_t *page_table, int max_pages, int page_size,
                  int b, int kvh, int64_t T, int window, int k_global, double *out, double *lse,
                  double *score, int32_t *idx) {
  const int d = kc->head_dim, G = num_q_heads / kc->num_kv_heads;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  double *krow = malloc(sizeof(double) * d), *vrow = malloc(sizeof(double) * d);
  double *qh = malloc(sizeof(double) * (size_t)G * d);
  double *s = malloc(sizeof(double) * (size_t)G * T); /* logits, then probabilities */
  char *taken = calloc((size_t)T, 1);
  orc_cand *cand = NULL;
  int rc = -1;
  if (!krow || !vrow || !qh || !s || !taken) goto done;

  for (int g = 0; g < G; ++g)
    for (int i = 0; i < d; ++i) qh[g * d + i] = elem(q, q_dtype, (int64_t)(kvh * G + g) * d + i);

  /* logits s_{h,t} = q_h . k_t / sqrt(d) */
  for (int64_t t = 0; t < T; ++t) {
    cache_row(kc, slot_of(page_table, max_pages, page_size, b, t), kvh, krow);
    for (int g = 0; g < G; ++g) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += qh[g * d + i] * krow[i];
      s[(size_t)g * T + t] = acc * inv_sqrt_d;
    }
  }
  /* softmax over all T positions, per query head; out = sum_t p v_t */
  for (int g = 0; g < G; ++g) {
    double *sg = s + (size_t)g * T, M = -INFINITY, Z = 0.0;
    for (int64_t t = 0; t < T; ++t) M = fmax(M, sg[t]);
    for (int64_t t = 0; t < T; ++t) Z += exp(sg[t] - M);
    for (int64_t t = 0; t < T; ++t) sg[t] = exp(sg[t] - M) / Z;
    lse[g] = M + log(Z);
    for (int i = 0; i < d; ++i) out[g * d + i] = 0.0;
  }
  for (int64_t t = 0; t < T; ++t) {
    cache_row(vc, slot_of(page_table, max_pages, page_size, b, t), kvh, vrow);
    for (int g = 0; g < G; ++g) {
      double p = s[(size_t)g * T + t];
      for (int i = 0; i < d; ++i) out[g * d + i] += p * vrow[i];
    }
  }
  /* group score: sum of the group's probabilities at each position */
  for (int64_t t = 0; t < T; ++t) {
    double acc = 0.0;
    for (int g = 0; g < G; ++g) acc += s[(size_t)g * T + t];
    score[t] = acc;
  }

  /* window [max(0,T-W), T) always; top-k_global of the candidates [0, T-W) */
  int64_t n_cand = T > window ? T - window : 0;
  for (int64_t t = n_cand; t < T; ++t) taken[t] = 1;
  if (n_cand <= k_global) {
    for (int64_t t = 0; t < n_cand; ++t) taken[t] = 1;
  } else {
    cand = malloc(sizeof(orc_cand) * (size_t)n_cand);
    if (!cand) goto done;
    for (int64_t t = 0; t < n_cand; ++t) {
      cand[t].score = score[t];
      cand[t].t = t;
    }
    qsort(cand, (size_t)n_cand, sizeof(orc_cand), cand_order);
    for (int i = 0; i < k_global; ++i) taken[cand[i].t] = 1;
  }
  int n = 0;
  for (int64_t t = 0; t < T; ++t)
    if (taken[t]) idx[n++] = (int32_t)slot_of(page_table, max_pages, page_size, b, t);
  for (int i = n; i < window + k_global; ++i) idx[i] = -1;
  rc = n;
done:
  free(krow);
  free(vrow);
  free(qh);
  free(s);
  free(taken);
  free(cand);
  return rc;
}

/*
 * Block-level selection, the first-generation HySparse comparator (the
 * announcement's paragraphs on HySparse v1: it selected whole blocks, so one
 * important token brought in the block around it; HySparse2's token-level
 * selection was compared with it at the same token budget).  Readings: the
 * candidates [0, T-W) are cut into blocks [j*block, (j+1)*block), the last
 * one cut short at T-W; a block's score is the sum of its positions' group
 * scores; k_global / block blocks are taken by (block score descending, block
 * index ascending), all of them when there are no more; the window
 * [max(0,T-W), T) is always taken.  idx gets the slots of the taken positions
 * in position order, -1 padded to window + k_global.  Returns the count, or
 * -1 for a block size that does not divide k_global (or no memory).
 */
int orc_select_blocks(const double *score, int64_t T, int window, int k_global, int block,
                      const int32_t *page_table, int max_pages, int page_size, int b, int32_t *idx) {
  if (block < 1 || k_global % block != 0) return -1;
  const int64_t n_cand = T > window ? T - window : 0;
  const int64_t n_blocks = (n_cand + block - 1) / block, keep = k_global / block;
  char *taken = calloc((size_t)(T > 0 ? T : 1), 1);
  orc_cand *blk = NULL;
  int rc = -1;
  if (!taken) return -1;
  for (int64_t t = n_cand; t < T; ++t) taken[t] = 1;
  if (n_blocks <= keep) {
    for (int64_t t = 0; t < n_cand; ++t) taken[t] = 1;
  } else {
    blk = malloc(sizeof(orc_cand) * (size_t)n_blocks);
    if (!blk) goto done;
    for (int64_t j = 0; j < n_blocks; ++j) {
      const int64_t t1 = (j + 1) * block < n_cand ? (j + 1) * block : n_cand;
      double sum = 0.0;
      for (int64_t t = j * block; t < t1; ++t) sum += score[t];
      blk[j].score = sum;
      blk[j].t = j;
    }
    qsort(blk, (size_t)n_blocks, sizeof(orc_cand), cand_order);
    for (int64_t i = 0; i < keep; ++i) {
      const int64_t j = blk[i].t, t1 = (j + 1) * block < n_cand ? (j + 1) * block : n_cand;
      for (int64_t t = j * block; t < t1; ++t) taken[t] = 1;
    }
  }
  int n = 0;
  for (int64_t t = 0; t < T; ++t)
    if (taken[t]) idx[n++] = (int32_t)slot_of(page_table, max_pages, page_size, b, t);
  for (int i = n; i < window + k_global; ++i) idx[i] = -1;
  rc = n;
done:
  free(taken);
  free(blk);
  return rc;
}

/*
 * Sparse-attention layer for one (sequence b, KV head kvh): softmax over the
 * listed rows only (the window and the global tokens together), with the
 * layer's own query.  idx holds slots, -1 entries are ignored.
 * q : [num_q_heads, head_dim] of sequence b.   out : [G, head_dim].
 */
int orc_sparse_unit(const void *q, int q_dtype, int num_q_heads, const orc_cache *kc,
                    const orc_cache *vc, int kvh, const int32_t *idx, int n_idx, double *out) {
  const int d = kc->head_dim, G = num_q_heads / kc->num_kv_heads;
  const double inv_sqrt_d = 1.0 / sqrt((double)d);
  double *row = malloc(sizeof(double) * d), *qh = malloc(sizeof(double) * d);
  double *s = malloc(sizeof(double) * (n_idx > 0 ? n_idx : 1));
  int rc = -1;
  if (!row || !qh || !s) goto done;
  for (int g = 0; g < G; ++g) {
    for (int i = 0; i < d; ++i) qh[i] = elem(q, q_dtype, (int64_t)(kvh * G + g) * d + i);
    double M = -INFINITY, Z = 0.0;
    for (int j = 0; j < n_idx; ++j) {
      s[j] = -INFINITY;
      if (idx[j] < 0) continue;
      cache_row(kc, idx[j], kvh, row);
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += qh[i] * row[i];
      s[j] = acc * inv_sqrt_d;
      M = fmax(M, s[j]);
    }
    for (int i = 0; i < d; ++i) out[g * d + i] = 0.0;
    if (M == -INFINITY) continue; /* no rows: output 0 */
    for (int j = 0; j < n_idx; ++j)
      if (idx[j] >= 0) Z += exp(s[j] - M);
    for (int j = 0; j < n_idx; ++j) {
      if (idx[j] < 0) continue;
      double p = exp(s[j] - M) / Z;
      cache_row(vc, idx[j], kvh, row);
      for (int i = 0; i < d; ++i) out[g * d + i] += p * row[i];
    }
  }
  rc = 0;
done:
  free(row);
  free(qh);
  free(s);
  return rc;
}

/* ---- batched entry points (loops over the per-unit definitions) --------- */

/*
 * Full layer + selection for a whole batch.
 *   q [B, Hq, d];  caches [num_slots, Hkv, d];  seq_lens [B];
 *   page_table [B, max_pages] or NULL (contiguous, capacity page_size each).
 * Outputs: out [B, Hq, d], lse [B, Hq], score [B, Hkv, t_cap] (positions
 * >= T_b left untouched), idx [B, Hkv, window+k_global], n_sel [B, Hkv].
 */
int orc_full_attn_select(const void *q, int q_dtype, int B, int num_q_heads, const void *k,
                         const float *k_scale, const void *v, const float *v_scale, int kv_dtype,
                         int num_kv_heads, int head_dim, const int32_t *seq_lens,
                         const int32_t *page_table, int max_pages, int page_size, int window,
                         int k_global, int64_t t_cap, double *out, double *lse, double *score,
                         int32_t *idx, int32_t *n_sel) {
  orc_cache kc = {k, k_scale, kv_dtype, num_kv_heads, head_dim};
  orc_cache vc = {v, v_scale, kv_dtype, num_kv_heads, head_dim};
  const int G = num_q_heads / num_kv_heads, d = head_dim, L = window + k_global;
  const size_t q_elem = q_dtype == ORC_F32 ? 4 : 2;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < num_kv_heads; ++h) {
      const char *qb = (const char *)q + (size_t)b * num_q_heads * d * q_elem;
      size_t u = (size_t)b * num_kv_heads + h;
      int n = orc_full_unit(qb, q_dtype, num_q_heads, &kc, &vc, page_table, max_pages, page_size,
                            b, h, seq_lens[b], window, k_global,
                            out + ((size_t)b * num_q_heads + (size_t)h * G) * d,
                            lse + (size_t)b * num_q_heads + (size_t)h * G, score + u * t_cap,
                            idx + u * L);
      if (n < 0) return -1;
      n_sel[u] = n;
    }
  return 0;
}

/*
 * Sparse layer for a whole batch: q [B, Hq, d], idx [B, Hkv, idx_stride]
 * (slots, -1 padded), out [B, Hq, d].
 */
int orc_sparse_attn(const void *q, int q_dtype, int B, int num_q_heads, const void *k,
                    const float *k_scale, const void *v, const float *v_scale, int kv_dtype,
                    int num_kv_heads, int head_dim, const int32_t *idx, int idx_stride,
                    double *out) {
  orc_cache kc = {k, k_scale, kv_dtype, num_kv_heads, head_dim};
  orc_cache vc = {v, v_scale, kv_dtype, num_kv_heads, head_dim};
  const int G = num_q_heads / num_kv_heads, d = head_dim;
  const size_t q_elem = q_dtype == ORC_F32 ? 4 : 2;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < num_kv_heads; ++h) {
      const char *qb = (const char *)q + (size_t)b * num_q_heads * d * q_elem;
      int rc = orc_sparse_unit(qb, q_dtype, num_q_heads, &kc, &vc, h,
                               idx + ((size_t)b * num_kv_heads + h) * idx_stride, idx_stride,
                               out + ((size_t)b * num_q_heads + (size_t)h * G) * d);
      if (rc < 0) return -1;
    }
  return 0;
}

/* ---- KV Bridging append ------------------------------------------------
 * HySparse2 announcement, "KV Bridging" paragraphs: each Cross-Decoder
 * full-attention layer builds its own KV cache from the input hidden state of
 * the matching Self-Decoder full-attention layer, through its own K and V
 * projections, so the cache exists before the Cross-Decoder runs.  For one
 * decode step the new token's rows are
 *     k = h W_k,   v = h W_v      (h [d_model], W [d_model, Hkv * d])
 * in double.  Readings where the pages are silent: the projections are plain
 * matrix products without bias; storage follows the cache type -- bf16
 * rounded to nearest (ties to even), or E4M3 per (token, kv head) with
 * scale = max|x| / 448 stored as fp32 (1 for an all-zero row) and each code
 * the E4M3 value nearest to x / scale (ties to the even code), saturated at
 * +-448. */

/* The E4M3 code nearest to x, ties to the code with an even mantissa, |x| >=
 * 448 saturating to +-448, NaN to 0x7F.  Plain definition: a scan of the 127
 * finite non-negative codes, whose values increase with the code. */
uint8_t orc_e4m3_encode(double x) {
  if (x != x) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  int lo = 0;
  while (lo + 1 <= 0x7E && orc_e4m3_value((uint8_t)(lo + 1)) <= a) ++lo;
  /* value(lo) <= a < value(lo + 1) */
  const double vl = orc_e4m3_value((uint8_t)lo), vh = orc_e4m3_value((uint8_t)(lo + 1));
  int c;
  if (a - vl < vh - a) c = lo;
  else if (a - vl > vh - a) c = lo + 1;
  else c = (lo & 1) ? lo + 1 : lo;
  return sign | (uint8_t)c;
}

/* bf16 bit pattern nearest to x (8 significant bits, ties to even), for
 * values in the normal fp32 range. */
uint16_t orc_bf16_encode(double x) {
  if (x == 0.0) return signbit(x) ? 0x8000 : 0;
  int e;
  const double f = frexp(x, &e);          /* x = f 2^e, 0.5 <= |f| < 1 */
  const double r = nearbyint(ldexp(f, 8)); /* 8 significant bits, ties to even */
  const float y = (float)ldexp(r, e - 8);  /* exact */
  uint32_t u;
  memcpy(&u, &y, sizeof u);
  return (uint16_t)(u >> 16);
}

/* One (token, kv head) row of d values into E4M3 codes and its fp32 scale. */
void orc_e4m3_row(const double *x, int d, uint8_t *codes, float *scale) {
  double amax = 0.0;
  for (int i = 0; i < d; ++i) amax = fmax(amax, fabs(x[i]));
  const float s = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
  for (int i = 0; i < d; ++i) codes[i] = orc_e4m3_encode(x[i] / (double)s);
  *scale = s;
}

/* k[b][n] = sum_i h[b][i] wk[i][n], v likewise; h, w are bf16 bit patterns. */
int orc_kv_bridge(const uint16_t *h, int B, int d_model, const uint16_t *wk, const uint16_t *wv, int n_out,
                  double *k, double *v) {
  for (int b = 0; b < B; ++b)
    for (int n = 0; n < n_out; ++n) {
      double sk = 0.0, sv = 0.0;
      for (int i = 0; i < d_model; ++i) {
        const double hi = bf16_value(h[(size_t)b * d_model + i]);
        sk += hi * bf16_value(wk[(size_t)i * n_out + n]);
        sv += hi * bf16_value(wv[(size_t)i * n_out + n]);
      }
      k[(size_t)b * n_out + n] = sk;
      v[(size_t)b * n_out + n] = sv;
    }
  return 0;
}
