/*
 * oracle.c -- plain, slow, obviously-correct CPU statement of the hybrid
 * sparse attention forward (HCA + MLA-DSA), and of the gradients of its
 * attention and compression steps (the backward pass, at the end).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * Sources (the pages describe the method in prose; no listing exists):
 *  [P1] "Baidu open-sourced a brand-new pretraining model, still focusing on
 *       efficiency with Flash" (blog.mirrorspeed.com), section
 *       "Hybrid sparse attention, 1/7 full context access".
 *  [P3] "Baidu Open-Sources ERNIE 5.5 Flash Base: Efficient 280B MoE for
 *       Agents" (besthub.dev), section "Core Architectural Innovations",
 *       item 1 "Hybrid Sparse Attention: MLA + HCA".
 *  [P5] ai-club.cn article on ERNIE 5.5 Flash Base, section
 *       "混合注意力（MLA + HCA）" (head widths 512 / 256, DSA).
 *
 * What the pages leave open is fixed by the problem statement this library
 * implements: compressor = weighted sum with a per-position weight vector
 * w[blk], fp32 accumulation, bf16 result; window W; indexer = int8 dot
 * products summed over indexer heads with integer weights; top-k with ties
 * going to the lower position.  Readings taken where even that is silent
 * (visibility rule, softmax scale, candidate set) are stated at each function.
 *
 * Precision: the compressor follows the fixed fp32 accumulation (ascending
 * position order, one fused multiply-add per term) and rounds to bf16 with
 * round-to-nearest-even; attention is evaluated in fp64; indexer scores are
 * exact integers.
 *
 * Tensor layouts (row-major, last dimension contiguous; bf16 as uint16 bits):
 *   K, V            [B, L, H, d]
 *   Kc, Vc          [B, n_c, H, d]
 *   Q, O            [B, Lq, Hq, d]
 *   q_idx           [B, Lq, H_idx, d_idx] int8
 *   k_idx           [B, Lk, d_idx]        int8  (one key shared by all indexer heads)
 *   w_idx           [H_idx]               int32
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG (-1)
#define ORACLE_ERR_RANGE (-2)

int oracle_version(void) { return 1; }

/* ------------------------------------------------------------------ */
/* bf16 <-> fp32 (IEEE binary32 with the low 16 mantissa bits dropped)  */
/* ------------------------------------------------------------------ */

static float bf16_bits_to_float(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round-to-nearest, ties-to-even, from the definition: add half an ulp of the
 * 16-bit result minus one, plus the result's low bit, then truncate. */
static uint16_t float_to_bf16_bits_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
  uint32_t keep_lsb = (u >> 16) & 1u;
  u += 0x7fffu + keep_lsb;
  return (uint16_t)(u >> 16);
}

void oracle_f32_to_bf16(const float* x, uint16_t* y, long n) {
  for (long i = 0; i < n; ++i) y[i] = float_to_bf16_bits_rne(x[i]);
}

void oracle_bf16_to_f32(const uint16_t* x, float* y, long n) {
  for (long i = 0; i < n; ++i) y[i] = bf16_bits_to_float(x[i]);
}

/* ------------------------------------------------------------------ */
/* HCA block compression                                               */
/* ------------------------------------------------------------------ */

/* [P1]/[P3]: the cache keeps one entry per 128 tokens.
 * Entry j of head h, channel c:
 *     acc = 0;  for i = 0 .. blk-1:  acc = fma(w[i], X[blk*j + i, h, c], acc)
 *     Xc[j, h, c] = bf16_rne(acc)
 * Only complete blocks exist: n_c = floor(L / blk).  The same w serves every
 * block, head and channel (and K and V alike: the caller applies it to both). */
int oracle_hca_compress(const uint16_t* X, const float* w, uint16_t* Xc,
                        int B, int L, int H, int d, int blk) {
  if (!X || !w || !Xc || B < 0 || L < 0 || H <= 0 || d <= 0 || blk <= 0) return ORACLE_ERR_ARG;
  const int n_c = L / blk;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < n_c; ++j)
      for (int h = 0; h < H; ++h)
        for (int c = 0; c < d; ++c) {
          float acc = 0.0f;
          for (int i = 0; i < blk; ++i) {
            const long src = (((long)b * L + (long)blk * j + i) * H + h) * (long)d + c;
            acc = fmaf(w[i], bf16_bits_to_float(X[src]), acc);
          }
          const long dst = (((long)b * n_c + j) * H + h) * (long)d + c;
          Xc[dst] = float_to_bf16_bits_rne(acc);
        }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* HCA visible set                                                     */
/* ------------------------------------------------------------------ */

/* [P1]/[P3]/[P5]: a query attends to the compressed entries and to a short
 * window of the latest raw tokens.  Reading taken (the pages do not say how the two
 * meet):
 *   window   = raw positions s with  max(0, t-W+1) <= s <= t
 *   entries  = blocks j whose every position lies before the window start,
 *              i.e. blk*(j+1) <= t-W+1, so n_c(t) = max(0, floor((t-W+1)/blk)).
 * With W >= t+1 no entry is visible (dense causal attention); with blk = 1 and
 * w = [1] the entries are the raw tokens before the window (dense causal again). */
int oracle_hca_window_start(int t, int W) {
  int s = t - W + 1;
  return s > 0 ? s : 0;
}

int oracle_hca_n_compressed(int t, int W, int blk) {
  int s = t - W + 1;
  return s > 0 ? s / blk : 0;
}

/* ------------------------------------------------------------------ */
/* Softmax attention of one query row over an explicit key list         */
/* ------------------------------------------------------------------ */

/* out[d] = sum_k p_k v_k / sum_k p_k with p_k = exp(s_k - max s), s_k =
 * scale * <q, k_k>; lse = max s + log(sum p).  Everything in fp64.
 * keys[i] / vals[i] point at bf16 rows of length d. */
static void attend_row(const uint16_t* q, const uint16_t* const* keys, const uint16_t* const* vals,
                       int n, int d, double scale, double* s_buf, double* out, double* lse) {
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (n == 0) {
    if (lse) *lse = -INFINITY;
    return;
  }
  double m = -INFINITY;
  for (int i = 0; i < n; ++i) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += (double)bf16_bits_to_float(q[c]) * (double)bf16_bits_to_float(keys[i][c]);
    s_buf[i] = scale * dot;
    if (s_buf[i] > m) m = s_buf[i];
  }
  double l = 0.0;
  for (int i = 0; i < n; ++i) {
    double p = exp(s_buf[i] - m);
    l += p;
    for (int c = 0; c < d; ++c) out[c] += p * (double)bf16_bits_to_float(vals[i][c]);
  }
  for (int c = 0; c < d; ++c) out[c] /= l;
  if (lse) *lse = m + log(l);
}

/* ------------------------------------------------------------------ */
/* HCA attention                                                       */
/* ------------------------------------------------------------------ */

/* [P1]/[P3]/[P5] HCA attention: one softmax over the union of the visible
 * compressed entries (in entry order) and the raw window (in position order).
 *   Query row r of batch b has absolute position t = q_offset + r.
 *   Window position s is read from Kw[b, s - win_start], Vw likewise.
 *   Head h reads K/V head h / (Hq / Hkv).
 *   scale is the softmax temperature (1/sqrt(d) by the plainest reading).
 * Only the rows listed in `rows` (flat b*Lq + r) are evaluated; O is
 * [n_rows, Hq, d] fp64 and lse (nullable) [n_rows, Hq] fp64. */
int oracle_hca_attn(const uint16_t* Q, const uint16_t* Kc, const uint16_t* Vc, int n_c,
                    const uint16_t* Kw, const uint16_t* Vw, int win_start, int n_w,
                    int B, int Lq, int q_offset, int Hq, int Hkv, int d, int blk, int W,
                    double scale, const int64_t* rows, int n_rows, double* O, double* lse) {
  if (!Q || !Kw || !Vw || !rows || !O || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || blk <= 0 || W <= 0)
    return ORACLE_ERR_ARG;
  if (n_c > 0 && (!Kc || !Vc)) return ORACLE_ERR_ARG;
  const int group = Hq / Hkv;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    const int max_keys = n_c + n_w;
    const uint16_t** keys = (const uint16_t**)malloc(sizeof(void*) * (size_t)(max_keys + 1));
    const uint16_t** vals = (const uint16_t**)malloc(sizeof(void*) * (size_t)(max_keys + 1));
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      const int64_t flat = rows[i];
      const int b = (int)(flat / Lq), r = (int)(flat % Lq);
      const int t = q_offset + r;
      const int ws = oracle_hca_window_start(t, W);
      const int nc_t = oracle_hca_n_compressed(t, W, blk);
      if (b < 0 || b >= B || nc_t > n_c || ws < win_start || t - win_start >= n_w) {
#pragma omp atomic write
        status = ORACLE_ERR_RANGE;
        continue;
      }
      for (int h = 0; h < Hq; ++h) {
        const int hk = h / group;
        int n = 0;
        for (int j = 0; j < nc_t; ++j) {
          const long off = (((long)b * n_c + j) * Hkv + hk) * (long)d;
          keys[n] = Kc + off;
          vals[n] = Vc + off;
          ++n;
        }
        for (int s = ws; s <= t; ++s) {
          const long off = (((long)b * n_w + (s - win_start)) * Hkv + hk) * (long)d;
          keys[n] = Kw + off;
          vals[n] = Vw + off;
          ++n;
        }
        const uint16_t* q = Q + (((long)b * Lq + r) * Hq + h) * (long)d;
        attend_row(q, keys, vals, n, d, scale, s_buf, O + ((long)i * Hq + h) * d,
                   lse ? lse + (long)i * Hq + h : NULL);
      }
    }
    free(keys);
    free(vals);
    free(s_buf);
  }
  return status;
}

/* HCA attention with FlashMask-4's head shape ([P1] "More structural improvements, data, and
 * infrastructure"; [P5] "训练：Muon 优化器 + 自研注意力算子": qk head dim 576, v head dim 512, for
 * HCA's 512-wide heads).  Reading taken (MLA-style shared latent): a key row is dqk wide
 * (the dv-wide latent plus a dqk - dv positional slice), and the value of a key is the first dv
 * columns of the same row -- one cache tensor per part (entries Kc, window Kw), no separate V.
 * Visible set, softmax and scale as oracle_hca_attn; scores over dqk, outputs over dv.
 * O is [n_rows, Hq, dv] fp64; lse (nullable) [n_rows, Hq]. */
int oracle_hca_attn_latent(const uint16_t* Q, const uint16_t* Kc, int n_c, const uint16_t* Kw, int win_start,
                           int n_w, int B, int Lq, int q_offset, int Hq, int Hkv, int dqk, int dv, int blk, int W,
                           double scale, const int64_t* rows, int n_rows, double* O, double* lse) {
  if (!Q || !Kw || !rows || !O || Hq <= 0 || Hkv <= 0 || Hq % Hkv || dqk <= 0 || dv <= 0 || dv > dqk || blk <= 0 ||
      W <= 0)
    return ORACLE_ERR_ARG;
  if (n_c > 0 && !Kc) return ORACLE_ERR_ARG;
  const int group = Hq / Hkv;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    const int max_keys = n_c + n_w;
    const uint16_t** keys = (const uint16_t**)malloc(sizeof(void*) * (size_t)(max_keys + 1));
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)(max_keys + 1));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      const int64_t flat = rows[i];
      const int b = (int)(flat / Lq), r = (int)(flat % Lq);
      const int t = q_offset + r;
      const int ws = oracle_hca_window_start(t, W);
      const int nc_t = oracle_hca_n_compressed(t, W, blk);
      if (b < 0 || b >= B || nc_t > n_c || ws < win_start || t - win_start >= n_w) {
#pragma omp atomic write
        status = ORACLE_ERR_RANGE;
        continue;
      }
      for (int h = 0; h < Hq; ++h) {
        const int hk = h / group;
        int n = 0;
        for (int j = 0; j < nc_t; ++j) keys[n++] = Kc + (((long)b * n_c + j) * Hkv + hk) * (long)dqk;
        for (int s = ws; s <= t; ++s) keys[n++] = Kw + (((long)b * n_w + (s - win_start)) * Hkv + hk) * (long)dqk;
        const uint16_t* q = Q + (((long)b * Lq + r) * Hq + h) * (long)dqk;
        double* out = O + ((long)i * Hq + h) * dv;
        for (int c = 0; c < dv; ++c) out[c] = 0.0;
        if (n == 0) {
          if (lse) lse[(long)i * Hq + h] = -INFINITY;
          continue;
        }
        double m = -INFINITY;
        for (int e = 0; e < n; ++e) {
          double dot = 0.0;
          for (int c = 0; c < dqk; ++c) dot += (double)bf16_bits_to_float(q[c]) * (double)bf16_bits_to_float(keys[e][c]);
          s_buf[e] = scale * dot;
          if (s_buf[e] > m) m = s_buf[e];
        }
        double l = 0.0;
        for (int e = 0; e < n; ++e) {
          const double pe = exp(s_buf[e] - m);
          l += pe;
          for (int c = 0; c < dv; ++c) out[c] += pe * (double)bf16_bits_to_float(keys[e][c]);  // value = first dv columns
        }
        for (int c = 0; c < dv; ++c) out[c] /= l;
        if (lse) lse[(long)i * Hq + h] = m + log(l);
      }
    }
    free(keys);
    free(s_buf);
  }
  return status;
}

/* ------------------------------------------------------------------ */
/* DSA lightning indexer                                               */
/* ------------------------------------------------------------------ */

/* [P1]/[P3]: a small scoring network rates every earlier position for each
 * query.  Form fixed by the problem statement:
 *   score[t, s] = sum_j w_idx[j] * sum_c q_idx[t, j, c] * k_idx[s, c]
 * exact in integers.  Writes the scores of query row (b, r) against key
 * positions 0 .. n-1 into out[0 .. n-1]. */
int oracle_dsa_scores(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx,
                      int B, int Lq, int Lk, int H_idx, int d_idx, int b, int r, int n, int64_t* out) {
  if (!q_idx || !k_idx || !w_idx || !out || b < 0 || b >= B || r < 0 || r >= Lq || n < 0 || n > Lk)
    return ORACLE_ERR_ARG;
  const int8_t* q = q_idx + ((long)b * Lq + r) * H_idx * (long)d_idx;
  for (int s = 0; s < n; ++s) {
    const int8_t* k = k_idx + ((long)b * Lk + s) * (long)d_idx;
    int64_t total = 0;
    for (int j = 0; j < H_idx; ++j) {
      int64_t dot = 0;
      for (int c = 0; c < d_idx; ++c) dot += (int64_t)q[j * d_idx + c] * (int64_t)k[c];
      total += (int64_t)w_idx[j] * dot;
    }
    out[s] = total;
  }
  return ORACLE_OK;
}

typedef struct {
  int64_t score;
  int32_t pos;
} scored_pos;

/* Order: higher score first; equal scores go to the lower position. */
static int by_score_then_position(const void* a, const void* b) {
  const scored_pos* x = (const scored_pos*)a;
  const scored_pos* y = (const scored_pos*)b;
  if (x->score != y->score) return x->score > y->score ? -1 : 1;
  return (x->pos > y->pos) - (x->pos < y->pos);
}

static int ascending_int32(const void* a, const void* b) {
  const int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
  return (x > y) - (x < y);
}

/* [P1]/[P3]: attention covers only the k positions with the best scores.
 * Candidates of a query at t are the positions 0 .. t
 * (the query's own position included; reading needed so that k >= t+1 gives
 * dense causal attention), restricted to s < Lk.  All candidates are sorted by
 * (score descending, position ascending); the first min(k, count) are kept and
 * written in ascending position order, padded with -1 up to k.
 * idx_out is [n_rows, k]. */
int oracle_dsa_topk(const int8_t* q_idx, const int8_t* k_idx, const int32_t* w_idx,
                    int B, int Lq, int q_offset, int Lk, int H_idx, int d_idx, int k,
                    const int64_t* rows, int n_rows, int32_t* idx_out) {
  if (!q_idx || !k_idx || !w_idx || !rows || !idx_out || k <= 0 || Lk < 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    int64_t* sc = (int64_t*)malloc(sizeof(int64_t) * (size_t)(Lk + 1));
    scored_pos* cand = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)(Lk + 1));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      const int b = (int)(rows[i] / Lq), r = (int)(rows[i] % Lq);
      const int t = q_offset + r;
      int n = t + 1 < Lk ? t + 1 : Lk;
      if (n < 0) n = 0;
      if (oracle_dsa_scores(q_idx, k_idx, w_idx, B, Lq, Lk, H_idx, d_idx, b, r, n, sc) != ORACLE_OK) {
#pragma omp atomic write
        status = ORACLE_ERR_RANGE;
        continue;
      }
      for (int s = 0; s < n; ++s) {
        cand[s].score = sc[s];
        cand[s].pos = s;
      }
      qsort(cand, (size_t)n, sizeof(scored_pos), by_score_then_position);
      const int keep = n < k ? n : k;
      int32_t* out = idx_out + (long)i * k;
      for (int m = 0; m < keep; ++m) out[m] = cand[m].pos;
      qsort(out, (size_t)keep, sizeof(int32_t), ascending_int32);
      for (int m = keep; m < k; ++m) out[m] = -1;
    }
    free(sc);
    free(cand);
  }
  return status;
}

/* ------------------------------------------------------------------ */
/* CSA: top-k over compressed entries                                  */
/* ------------------------------------------------------------------ */

/* [P1] "Hybrid sparse attention, 1/7 full context access" (and [P3] item 1)
 * name the alternative the pages compare against: CSA, which compresses the
 * history 4:1 and then selects sparsely.  Reading taken here (the pages give
 * no more): the entries are the compressor's output for blocks of blk tokens
 * (the HCA compressor form with a blk-long weight vector), each entry has its
 * own indexer key, and a query at t may select entry j once the block it
 * summarises is complete, blk*(j+1) <= t+1, i.e. j < floor((t+1)/blk).  No
 * raw window.  Selection as in DSA: the k entries with the largest (score,
 * -j), written ascending, -1 padded.
 * kc_idx is [B, n_c, d_idx] (one key per entry); idx_out [n_rows, k]. */
int oracle_csa_n_candidates(int t, int blk, int n_c) {
  if (blk <= 0 || t < 0) return 0;
  const int n = (t + 1) / blk;
  return n < n_c ? n : n_c;
}

int oracle_csa_topk(const int8_t* q_idx, const int8_t* kc_idx, const int32_t* w_idx,
                    int B, int Lq, int q_offset, int n_c, int H_idx, int d_idx, int k, int blk,
                    const int64_t* rows, int n_rows, int32_t* idx_out) {
  if (!q_idx || !kc_idx || !w_idx || !rows || !idx_out || k <= 0 || n_c < 0 || blk <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    int64_t* sc = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_c + 1));
    scored_pos* cand = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)(n_c + 1));
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      const int b = (int)(rows[i] / Lq), r = (int)(rows[i] % Lq);
      const int n = oracle_csa_n_candidates(q_offset + r, blk, n_c);
      if (oracle_dsa_scores(q_idx, kc_idx, w_idx, B, Lq, n_c, H_idx, d_idx, b, r, n, sc) != ORACLE_OK) {
#pragma omp atomic write
        status = ORACLE_ERR_RANGE;
        continue;
      }
      for (int j = 0; j < n; ++j) {
        cand[j].score = sc[j];
        cand[j].pos = j;
      }
      qsort(cand, (size_t)n, sizeof(scored_pos), by_score_then_position);
      const int keep = n < k ? n : k;
      int32_t* out = idx_out + (long)i * k;
      for (int m = 0; m < keep; ++m) out[m] = cand[m].pos;
      qsort(out, (size_t)keep, sizeof(int32_t), ascending_int32);
      for (int m = keep; m < k; ++m) out[m] = -1;
    }
    free(sc);
    free(cand);
  }
  return status;
}

/* ------------------------------------------------------------------ */
/* DSA sparse attention                                                */
/* ------------------------------------------------------------------ */

/* [P1]/[P3]/[P5]: dense attention of each query over its selected positions
 * only; 256-wide heads; all query heads read one shared K/V head (the MLA
 * latent reading) and share the index set.  idx_rows is [n_rows, k], entries
 * < 0 are padding and ignored; the order of the entries does not matter.
 * O is [n_rows, Hq, d] fp64; lse (nullable) [n_rows, Hq]. */
int oracle_dsa_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx_rows,
                    int B, int Lq, int Lk, int Hq, int d, int k, double scale,
                    const int64_t* rows, int n_rows, double* O, double* lse) {
  if (!Q || !K || !V || !idx_rows || !rows || !O || Hq <= 0 || d <= 0 || k <= 0) return ORACLE_ERR_ARG;
  int status = ORACLE_OK;
#pragma omp parallel
  {
    const uint16_t** keys = (const uint16_t**)malloc(sizeof(void*) * (size_t)k);
    const uint16_t** vals = (const uint16_t**)malloc(sizeof(void*) * (size_t)k);
    double* s_buf = (double*)malloc(sizeof(double) * (size_t)k);
#pragma omp for schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
      const int b = (int)(rows[i] / Lq), r = (int)(rows[i] % Lq);
      int n = 0, bad = 0;
      for (int m = 0; m < k; ++m) {
        const int32_t s = idx_rows[(long)i * k + m];
        if (s < 0) continue;
        if (s >= Lk) {
          bad = 1;
          break;
        }
        keys[n] = K + ((long)b * Lk + s) * (long)d;
        vals[n] = V + ((long)b * Lk + s) * (long)d;
        ++n;
      }
      if (bad || b < 0 || b >= B) {
#pragma omp atomic write
        status = ORACLE_ERR_RANGE;
        continue;
      }
      for (int h = 0; h < Hq; ++h) {
        const uint16_t* q = Q + (((long)b * Lq + r) * Hq + h) * (long)d;
        attend_row(q, keys, vals, n, d, scale, s_buf, O + ((long)i * Hq + h) * d,
                   lse ? lse + (long)i * Hq + h : NULL);
      }
    }
    free(keys);
    free(vals);
    free(s_buf);
  }
  return status;
}

/* ------------------------------------------------------------------ */
/* Output gate + virtual-head mix (the attention epilogue)              */
/* ------------------------------------------------------------------ */

/* [P1] "Hybrid sparse attention, 1/7 full context access", last paragraph, and
 * [P3] "Core Architectural Innovations" (low-rank gated attention, VHA): the
 * output gate is computed from the layer's low-rank query latent (a quarter of
 * the hidden width), and VHA mixes the heads with a light low-rank term on top
 * of an identity path.  Readings taken (the pages give no formulas): the gate
 * is elementwise per head and channel, Z = c_q . W_g^T, and VHA acts on the
 * attention output of one token, channel by channel, before the gate:
 *   Ohat[t,h,c] = O[t,h,c] + sum_m U[h,m] sum_h' V[h',m] O[t,h',c]
 *   Z[t,h,c]    = sum_i cq[t,i] Wg[h*dv + c, i]
 *   Y[t,h,c]    = sigmoid(Z[t,h,c]) * Ohat[t,h,c]
 * O [B,L,H,dv], cq [B,L,rq], Wg [H*dv, rq] bf16; U, V [H, r] fp32; Y fp64
 * [B,L,H,dv].  Rows t are independent; OpenMP over them. */
int oracle_gate_vha(const uint16_t* O, const uint16_t* cq, const uint16_t* Wg, const float* U, const float* V,
                    int B, int L, int H, int dv, int rq, int r, double* Y) {
  if (!O || !cq || !Wg || !Y || B < 0 || L < 0 || H <= 0 || dv <= 0 || rq <= 0 || r < 0 || (r > 0 && (!U || !V)))
    return ORACLE_ERR_ARG;
  const long rows = (long)B * L;
#pragma omp parallel
  {
    double* proj = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1) * (size_t)dv);
#pragma omp for schedule(static)
    for (long t = 0; t < rows; ++t) {
      const uint16_t* o = O + t * (long)H * dv;
      const uint16_t* q = cq + t * (long)rq;
      for (int m = 0; m < r; ++m)
        for (int c = 0; c < dv; ++c) {
          double acc = 0.0;
          for (int h2 = 0; h2 < H; ++h2) acc += (double)V[h2 * r + m] * (double)bf16_bits_to_float(o[h2 * dv + c]);
          proj[m * dv + c] = acc;
        }
      for (int h = 0; h < H; ++h)
        for (int c = 0; c < dv; ++c) {
          double ohat = (double)bf16_bits_to_float(o[h * dv + c]);
          for (int m = 0; m < r; ++m) ohat += (double)U[h * r + m] * proj[m * dv + c];
          const uint16_t* wrow = Wg + ((long)h * dv + c) * rq;
          double z = 0.0;
          for (int i = 0; i < rq; ++i) z += (double)bf16_bits_to_float(q[i]) * (double)bf16_bits_to_float(wrow[i]);
          Y[(t * H + h) * (long)dv + c] = ohat / (1.0 + exp(-z));
        }
    }
    free(proj);
  }
  return ORACLE_OK;
}

/* ================================================================== */
/* Backward pass (gradients of a scalar loss through O)                */
/* ================================================================== */

/* Gradient of one query row of attend_row.  With s_i = scale <q, k_i>,
 * p = softmax(s) and O = sum_i p_i v_i, a loss with dL/dO = dO gives
 *   dL/dv_i = p_i dO
 *   dL/ds_i = p_i (<dO, v_i> - <dO, O>)
 *   dL/dq   = scale sum_i dL/ds_i k_i,   dL/dk_i = scale dL/ds_i q.
 * Keys and values are given by element offsets into K/V (bf16) so that the
 * key and value gradients land at the same offsets of dK/dV (fp64, added to).
 * dq (d doubles) is added to as well.  p_buf holds n doubles. */
static void attend_row_bwd(const uint16_t* q, const uint16_t* K, const uint16_t* V, const long* offs, int n,
                           int d, double scale, const double* dO, double* p_buf, double* dq, double* dK,
                           double* dV) {
  if (n == 0) return;
  double m = -INFINITY;
  for (int i = 0; i < n; ++i) {
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += (double)bf16_bits_to_float(q[c]) * (double)bf16_bits_to_float(K[offs[i] + c]);
    p_buf[i] = scale * dot;
    if (p_buf[i] > m) m = p_buf[i];
  }
  double l = 0.0;
  for (int i = 0; i < n; ++i) {
    p_buf[i] = exp(p_buf[i] - m);
    l += p_buf[i];
  }
  for (int i = 0; i < n; ++i) p_buf[i] /= l;
  /* <dO, O> = sum_i p_i <dO, v_i> */
  double dO_O = 0.0;
  for (int i = 0; i < n; ++i) {
    double dp = 0.0;
    for (int c = 0; c < d; ++c) dp += dO[c] * (double)bf16_bits_to_float(V[offs[i] + c]);
    dO_O += p_buf[i] * dp;
  }
  for (int i = 0; i < n; ++i) {
    double dp = 0.0;
    for (int c = 0; c < d; ++c) dp += dO[c] * (double)bf16_bits_to_float(V[offs[i] + c]);
    const double ds = p_buf[i] * (dp - dO_O);
    for (int c = 0; c < d; ++c) {
      dV[offs[i] + c] += p_buf[i] * dO[c];
      dq[c] += scale * ds * (double)bf16_bits_to_float(K[offs[i] + c]);
      dK[offs[i] + c] += scale * ds * (double)bf16_bits_to_float(q[c]);
    }
  }
}

/* Backward of oracle_hca_attn over every query row: dO is [B, Lq, Hq, d]
 * fp64; dQ [B, Lq, Hq, d], dKc/dVc [B, n_c, Hkv, d], dKw/dVw [B, n_w, Hkv, d]
 * are fp64 and overwritten.  The visible set, head mapping and scale are those
 * of the forward.  Serial (keys are shared between rows and heads). */
int oracle_hca_attn_bwd(const uint16_t* Q, const uint16_t* Kc, const uint16_t* Vc, int n_c,
                        const uint16_t* Kw, const uint16_t* Vw, int win_start, int n_w, const double* dO,
                        int B, int Lq, int q_offset, int Hq, int Hkv, int d, int blk, int W, double scale,
                        double* dQ, double* dKc, double* dVc, double* dKw, double* dVw) {
  if (!Q || !Kw || !Vw || !dO || !dQ || !dKw || !dVw || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 ||
      blk <= 0 || W <= 0 || B < 0 || Lq < 0 || n_c < 0 || n_w < 0)
    return ORACLE_ERR_ARG;
  if (n_c > 0 && (!Kc || !Vc || !dKc || !dVc)) return ORACLE_ERR_ARG;
  const int group = Hq / Hkv;
  memset(dQ, 0, sizeof(double) * (size_t)B * Lq * Hq * d);
  if (n_c > 0) {
    memset(dKc, 0, sizeof(double) * (size_t)B * n_c * Hkv * d);
    memset(dVc, 0, sizeof(double) * (size_t)B * n_c * Hkv * d);
  }
  memset(dKw, 0, sizeof(double) * (size_t)B * n_w * Hkv * d);
  memset(dVw, 0, sizeof(double) * (size_t)B * n_w * Hkv * d);
  long* offs_c = (long*)malloc(sizeof(long) * (size_t)(n_c + 1));
  long* offs_w = (long*)malloc(sizeof(long) * (size_t)(n_w + 1));
  double* p_buf = (double*)malloc(sizeof(double) * (size_t)(n_c + n_w + 1));
  double* dq_tmp = (double*)malloc(sizeof(double) * (size_t)d);
  int status = ORACLE_OK;
  for (int b = 0; b < B && status == ORACLE_OK; ++b)
    for (int r = 0; r < Lq && status == ORACLE_OK; ++r) {
      const int t = q_offset + r;
      const int ws = oracle_hca_window_start(t, W);
      const int nc_t = oracle_hca_n_compressed(t, W, blk);
      if (nc_t > n_c || ws < win_start || t - win_start >= n_w) {
        status = ORACLE_ERR_RANGE;
        break;
      }
      for (int h = 0; h < Hq; ++h) {
        const int hk = h / group;
        int n_cv = 0, n_wv = 0;
        for (int j = 0; j < nc_t; ++j) offs_c[n_cv++] = (((long)b * n_c + j) * Hkv + hk) * (long)d;
        for (int s = ws; s <= t; ++s) offs_w[n_wv++] = (((long)b * n_w + (s - win_start)) * Hkv + hk) * (long)d;
        const long qo = (((long)b * Lq + r) * Hq + h) * (long)d;
        /* the row's keys: its entries, then its window (one softmax over both, as in the
         * forward); the same steps as attend_row_bwd, with two key tensors */
        const int n = n_cv + n_wv;
        if (n == 0) continue;
        double m = -INFINITY;
        for (int i = 0; i < n; ++i) {
          const uint16_t* kr = i < n_cv ? Kc + offs_c[i] : Kw + offs_w[i - n_cv];
          double dot = 0.0;
          for (int c = 0; c < d; ++c) dot += (double)bf16_bits_to_float(Q[qo + c]) * (double)bf16_bits_to_float(kr[c]);
          p_buf[i] = scale * dot;
          if (p_buf[i] > m) m = p_buf[i];
        }
        double l = 0.0;
        for (int i = 0; i < n; ++i) {
          p_buf[i] = exp(p_buf[i] - m);
          l += p_buf[i];
        }
        for (int i = 0; i < n; ++i) p_buf[i] /= l;
        const double* g = dO + qo;
        double dO_O = 0.0;
        for (int i = 0; i < n; ++i) {
          const uint16_t* vr = i < n_cv ? Vc + offs_c[i] : Vw + offs_w[i - n_cv];
          double dp = 0.0;
          for (int c = 0; c < d; ++c) dp += g[c] * (double)bf16_bits_to_float(vr[c]);
          dO_O += p_buf[i] * dp;
        }
        for (int c = 0; c < d; ++c) dq_tmp[c] = 0.0;
        for (int i = 0; i < n; ++i) {
          const int entry = i < n_cv;
          const long o = entry ? offs_c[i] : offs_w[i - n_cv];
          const uint16_t* kr = (entry ? Kc : Kw) + o;
          const uint16_t* vr = (entry ? Vc : Vw) + o;
          double* dk = (entry ? dKc : dKw) + o;
          double* dv = (entry ? dVc : dVw) + o;
          double dp = 0.0;
          for (int c = 0; c < d; ++c) dp += g[c] * (double)bf16_bits_to_float(vr[c]);
          const double ds = p_buf[i] * (dp - dO_O);
          for (int c = 0; c < d; ++c) {
            dv[c] += p_buf[i] * g[c];
            dq_tmp[c] += scale * ds * (double)bf16_bits_to_float(kr[c]);
            dk[c] += scale * ds * (double)bf16_bits_to_float(Q[qo + c]);
          }
        }
        for (int c = 0; c < d; ++c) dQ[qo + c] = dq_tmp[c];
      }
    }
  free(offs_c);
  free(offs_w);
  free(p_buf);
  free(dq_tmp);
  return status;
}

/* Backward of oracle_dsa_attn over every query row: idx_rows is [B*Lq, k]
 * (row b*Lq + r; entries < 0 are padding), dO [B, Lq, Hq, d] fp64; dQ
 * [B, Lq, Hq, d], dK/dV [B, Lk, d] fp64, overwritten.  Serial. */
int oracle_dsa_attn_bwd(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const int32_t* idx_rows,
                        const double* dO, int B, int Lq, int Lk, int Hq, int d, int k, double scale, double* dQ,
                        double* dK, double* dV) {
  if (!Q || !K || !V || !idx_rows || !dO || !dQ || !dK || !dV || B < 0 || Lq < 0 || Lk < 0 || Hq <= 0 ||
      d <= 0 || k <= 0)
    return ORACLE_ERR_ARG;
  memset(dQ, 0, sizeof(double) * (size_t)B * Lq * Hq * d);
  memset(dK, 0, sizeof(double) * (size_t)B * Lk * d);
  memset(dV, 0, sizeof(double) * (size_t)B * Lk * d);
  long* offs = (long*)malloc(sizeof(long) * (size_t)k);
  double* p_buf = (double*)malloc(sizeof(double) * (size_t)k);
  int status = ORACLE_OK;
  for (int b = 0; b < B && status == ORACLE_OK; ++b)
    for (int r = 0; r < Lq; ++r) {
      int n = 0;
      for (int m = 0; m < k; ++m) {
        const int32_t s = idx_rows[((long)b * Lq + r) * k + m];
        if (s < 0) continue;
        if (s >= Lk) {
          status = ORACLE_ERR_RANGE;
          break;
        }
        offs[n++] = ((long)b * Lk + s) * (long)d;
      }
      if (status != ORACLE_OK) break;
      for (int h = 0; h < Hq; ++h) {
        const long qo = (((long)b * Lq + r) * Hq + h) * (long)d;
        attend_row_bwd(Q + qo, K, V, offs, n, d, scale, dO + qo, p_buf, dQ + qo, dK, dV);
      }
    }
  free(offs);
  free(p_buf);
  return status;
}

/* Backward of the compressor, taken as the exact linear map
 *   Xc[b, j, h, c] = sum_i w[i] X[b, blk*j + i, h, c]
 * (the forward's fp32 chain and bf16 rounding are not differentiated):
 *   dX[b, blk*j + i, h, c] = w[i] dXc[b, j, h, c]   (0 for the partial tail block)
 *   dw[i] = sum_{b, j, h, c} X[b, blk*j + i, h, c] dXc[b, j, h, c]
 * dXc is [B, L/blk, H, d] fp64; dX [B, L, H, d] and dw [blk] fp64, overwritten. */
int oracle_hca_compress_bwd(const uint16_t* X, const float* w, const double* dXc, int B, int L, int H, int d,
                            int blk, double* dX, double* dw) {
  if (!X || !w || !dXc || !dX || !dw || B < 0 || L < 0 || H <= 0 || d <= 0 || blk <= 0) return ORACLE_ERR_ARG;
  const int n_c = L / blk;
  memset(dX, 0, sizeof(double) * (size_t)B * L * H * d);
  for (int i = 0; i < blk; ++i) dw[i] = 0.0;
  for (int b = 0; b < B; ++b)
    for (int j = 0; j < n_c; ++j)
      for (int i = 0; i < blk; ++i)
        for (int h = 0; h < H; ++h)
          for (int c = 0; c < d; ++c) {
            const long src = (((long)b * L + (long)blk * j + i) * H + h) * (long)d + c;
            const double g = dXc[(((long)b * n_c + j) * H + h) * (long)d + c];
            dX[src] = (double)w[i] * g;
            dw[i] += (double)bf16_bits_to_float(X[src]) * g;
          }
  return ORACLE_OK;
}
