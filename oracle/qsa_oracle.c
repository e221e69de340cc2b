/*
 * qsa_oracle.c -- CPU oracle for the Qwen Sparse Attention (QSA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA path is checked against.  Only the tests, __graft_entry__.smoke() and
 * bench.py's cpu_baseline / reference leg may load or call it.  The product
 * library (libqsa.so) never links, loads or calls it, and the two share no
 * code: no headers, tables, helpers or constants.
 *
 * What it computes (sources are the web pages on Qwen3.8-Flash-Next):
 *   - "Qwen3.8-Next architecture design report" (macin.top summary of
 *     "On the Design of Qwen3.8-Next Architecture"), section "Four architecture
 *     components", item 2 "Qwen Sparse Attention (QSA)": the indexer scores at
 *     micro-block granularity r=4; keys are first average-pooled, then given a
 *     position encoding; the indexer uses 4 query heads (MQA); the token budget
 *     is K=2048.
 *   - Miles docs page "Qwen3.8-Flash-Next", section 1 "Model Introduction":
 *     each QSA layer projects its own indexer queries and compressed keys,
 *     scores them, keeps indexer_budget key tokens per query, and attention
 *     reads only those; 24 attention heads, 2 query groups, kv-channels 256,
 *     rotary base 1e7 at rotary percent 0.25.
 *   - tahou.com article "Qwen3.8-Flash-Next open-sourced ...", section
 *     "GDN+QSA": a lightweight indexer aggregates the sequence into
 *     micro-blocks, scores importance per block, then attends to the most
 *     relevant regions.
 * Readings fixed where the pages are silent (the score is the DSA form
 * s(t,b) = sum_h w[t,h] * ReLU(q~[t,h] . k^[b]); RoPE on k^[b] at the block
 * start b*r; partial rotary on the first rope_dims dims with rotate-half
 * pairs (i, i + rope_dims/2) and theta_i = base^(-2i/rope_dims); the query's
 * own partial block is always kept and causally masked; ties break toward the
 * lower block index) are listed with the rest in the repository's design notes.
 *
 * Precision.  Storage is fp32.  The two rounding points that the method's
 * definition fixes (the pooled+rotated key k^ and the rotated indexer query q~
 * are held in the I/O dtype) are computed in fp32 in a fixed order with no
 * fused multiply-add (build with -ffp-contract=off) and rounded to bf16
 * round-to-nearest-even when the I/O dtype is bf16.  Cosines and sines come
 * from angles formed in fp64 and are rounded to fp32.  Every other sum (dot
 * products, softmax, weighted V sums) accumulates in acc_t: fp64 by default,
 * fp32 when built with -DQSA_ORACLE_ACC_F32 (the second build is used only to
 * cross-check the first).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "qsa_oracle.h"

#ifdef _OPENMP
#include <omp.h>
#endif

#ifdef QSA_ORACLE_ACC_F32
typedef float acc_t;
#define ACC_EXP expf
#define ACC_LOG logf
#else
typedef double acc_t;
#define ACC_EXP exp
#define ACC_LOG log
#endif

/* ------------------------------------------------------------------------ */
/* bf16 round-to-nearest-even of an fp32 value, written from the IEEE        */
/* definition: keep the top 16 bits, rounding on the 16 dropped bits with    */
/* ties to even.  NaN stays NaN.                                             */
/* ------------------------------------------------------------------------ */
static float to_bf16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u) {       /* Inf or NaN */
    if (u & 0x007fffffu) u |= 0x00400000u;      /* keep NaN quiet */
    u &= 0xffff0000u;
  } else {
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    u &= 0xffff0000u;
  }
  memcpy(&x, &u, sizeof u);
  return x;
}

static float round_io(const qsa_ref_config* c, float x) {
  return c->round_bf16 ? to_bf16_rne(x) : x;
}

double qsa_ref_round_bf16(double x) { return (double)to_bf16_rne((float)x); }

/* ------------------------------------------------------------------------ */
/* Rotary position encoding (partial, rotate-half pairing).                  */
/* Miles docs "Qwen3.8-Flash-Next" section 1: rotary base 1e7, rotary        */
/* percent 0.25.  The design report says pooled keys get a position          */
/* encoding after pooling; this oracle applies the same rotary encoding the  */
/* main attention uses, at the block's first token position.                 */
/* ------------------------------------------------------------------------ */
double qsa_ref_rope_theta(const qsa_ref_config* c, int i) {
  /* theta_i = base^(-2i / rope_dims), i in [0, rope_dims/2) */
  return pow(c->rope_base, -(2.0 * (double)i) / (double)c->rope_dims);
}

void qsa_ref_rope_cos_sin(const qsa_ref_config* c, int64_t pos, float* cos_out,
                          float* sin_out) {
  int half = c->rope_dims / 2;
  for (int i = 0; i < half; ++i) {
    double angle = (double)pos * qsa_ref_rope_theta(c, i);
    cos_out[i] = (float)cos(angle);
    sin_out[i] = (float)sin(angle);
  }
}

/* Rotate x (length idx_dim) for position pos, fp32 arithmetic, products
 * rounded separately (no FMA), then round to the I/O dtype. */
void qsa_ref_rope_vec(const qsa_ref_config* c, const float* x, int64_t pos,
                      float* out) {
  int d = c->idx_dim, half = c->rope_dims / 2;
  float cs[512], sn[512];
  qsa_ref_rope_cos_sin(c, pos, cs, sn);
  for (int j = 0; j < d; ++j) out[j] = x[j];
  for (int i = 0; i < half; ++i) {
    float a = x[i], b = x[i + half];
    float ac = a * cs[i], bs = b * sn[i];
    float bc = b * cs[i], as = a * sn[i];
    out[i] = ac - bs;
    out[i + half] = bc + as;
  }
  for (int j = 0; j < d; ++j) out[j] = round_io(c, out[j]);
}

/* ------------------------------------------------------------------------ */
/* Step 1: key pooling into micro-blocks + block position encoding.          */
/* Design report, QSA item: the indexer keys of each micro-block (r = 4      */
/* tokens) are averaged first; the position encoding is added afterwards.    */
/* k_idx: the sequence's indexer keys, row-major [n][idx_dim], row 0 = token 0.
 * Writes k^ for blocks [b0, b1) to khat[(b - b0)][idx_dim].                  */
/* ------------------------------------------------------------------------ */
void qsa_ref_compress_keys(const qsa_ref_config* c, const float* k_idx,
                           int64_t b0, int64_t b1, float* khat) {
  int d = c->idx_dim, r = c->r;
  float mean[1024];
  for (int64_t b = b0; b < b1; ++b) {
    const float* rows = k_idx + (b * r) * (int64_t)d;
    for (int j = 0; j < d; ++j) {
      float s = rows[j];
      for (int k = 1; k < r; ++k) s = s + rows[(int64_t)k * d + j];
      mean[j] = s / (float)r;
    }
    qsa_ref_rope_vec(c, mean, b * r, khat + (b - b0) * (int64_t)d);
  }
}

/* ------------------------------------------------------------------------ */
/* Step 2: indexer scores of one query token at position t against every    */
/* complete block before its own block b_t = floor(t / r).                   */
/* s(t,b) = sum_h w[h] * max(0, q~[h] . k^[b]),  b in [0, b_t).               */
/* Design report, QSA item: 4-head MQA indexer, scores per micro-block.       */
/* q_idx: [idx_heads][idx_dim] as projected (not yet rotated).               */
/* khat: k^ of blocks 0 .. b_t-1, [b][idx_dim].  s: out, [b_t].              */
/* ------------------------------------------------------------------------ */
void qsa_ref_index_scores(const qsa_ref_config* c, const float* q_idx,
                          const float* w, int64_t t, const float* khat,
                          double* s) {
  int d = c->idx_dim, hi = c->idx_heads;
  int64_t bt = t / c->r;
  float* qr = (float*)malloc(sizeof(float) * (size_t)hi * (size_t)d);
  for (int h = 0; h < hi; ++h) qsa_ref_rope_vec(c, q_idx + h * d, t, qr + h * d);
  for (int64_t b = 0; b < bt; ++b) {
    const float* kb = khat + b * (int64_t)d;
    acc_t total = 0;
    for (int h = 0; h < hi; ++h) {
      acc_t dot = 0;
      for (int j = 0; j < d; ++j) dot += (acc_t)qr[h * d + j] * (acc_t)kb[j];
      acc_t relu = dot > 0 ? dot : 0;
      total += (acc_t)w[h] * relu;
    }
    s[b] = (double)total;
  }
  free(qr);
}

/* ------------------------------------------------------------------------ */
/* Step 3: top-k block selection.                                            */
/* Budget S = budget_tokens / r blocks (2048 tokens = 512 blocks on the      */
/* pages).  If the query has at most S blocks in reach (b_t + 1 <= S), every */
/* block 0..b_t is kept.  Otherwise the own block b_t is kept and the S-1    */
/* best candidates b < b_t under the order (score descending, block index    */
/* ascending) are added.  The list is returned sorted ascending and padded   */
/* with -1 to S entries.  Returns the count.                                 */
/* ------------------------------------------------------------------------ */
typedef struct {
  double s;
  int64_t b;
} cand_t;

static int cand_order(const void* pa, const void* pb) {
  const cand_t* a = (const cand_t*)pa;
  const cand_t* b = (const cand_t*)pb;
  if (a->s > b->s) return -1;
  if (a->s < b->s) return 1;
  return (a->b < b->b) ? -1 : (a->b > b->b);
}

static int int32_ascending(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a > b) - (a < b);
}

int qsa_ref_select(const qsa_ref_config* c, const double* s, int64_t t,
                   int32_t* sel) {
  int S = c->budget_tokens / c->r;
  int64_t bt = t / c->r;
  int n = 0;
  if (bt + 1 <= S) {
    for (int64_t b = 0; b <= bt; ++b) sel[n++] = (int32_t)b;
  } else {
    cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)bt);
    for (int64_t b = 0; b < bt; ++b) {
      cand[b].s = (s[b] == 0.0) ? 0.0 : s[b];   /* -0 and +0 are one value */
      cand[b].b = b;
    }
    qsort(cand, (size_t)bt, sizeof(cand_t), cand_order);
    for (int i = 0; i < S - 1; ++i) sel[n++] = (int32_t)cand[i].b;
    free(cand);
    qsort(sel, (size_t)n, sizeof(int32_t), int32_ascending);
    sel[n++] = (int32_t)bt;                     /* own block, largest index */
  }
  for (int i = n; i < S; ++i) sel[i] = -1;
  return n;
}

/* ------------------------------------------------------------------------ */
/* Step 4: GQA softmax attention over the selected tokens of one query.      */
/* Miles docs section 1: attention reads only the kept key tokens; 24 heads, */
/* 2 query groups, head dim 256.  Head h reads group h / (n_heads/n_groups). */
/* Token j is attended iff its block j / r is selected and j <= t.           */
/* q: [n_heads][head_dim].  k, v: the sequence's cache, [n_groups][ld][head_dim].
 * o: out [n_heads][head_dim].  lse: out [n_heads] (natural log), may be NULL.
 * ------------------------------------------------------------------------ */
void qsa_ref_attend(const qsa_ref_config* c, const float* q, const float* k,
                    const float* v, int64_t ld, int64_t t, const int32_t* sel,
                    int nsel, double* o, double* lse) {
  int H = c->n_heads, G = c->n_groups, D = c->head_dim, r = c->r;
  int hpg = H / G;
  int64_t maxtok = (int64_t)nsel * r;
  acc_t* sc = (acc_t*)malloc(sizeof(acc_t) * (size_t)(maxtok > 0 ? maxtok : 1));
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)(maxtok > 0 ? maxtok : 1));
  acc_t* acc = (acc_t*)malloc(sizeof(acc_t) * (size_t)D);
  for (int h = 0; h < H; ++h) {
    int g = h / hpg;
    const float* qh = q + (int64_t)h * D;
    const float* kg = k + (int64_t)g * ld * D;
    const float* vg = v + (int64_t)g * ld * D;
    int64_t n = 0;
    acc_t m = -INFINITY;
    for (int i = 0; i < nsel; ++i) {
      int64_t b = sel[i];
      for (int64_t j = b * r; j < b * r + r; ++j) {
        if (j > t) continue;
        acc_t dot = 0;
        for (int e = 0; e < D; ++e) dot += (acc_t)qh[e] * (acc_t)kg[j * D + e];
        acc_t sj = (acc_t)c->softmax_scale * dot;
        sc[n] = sj;
        tok[n] = j;
        ++n;
        if (sj > m) m = sj;
      }
    }
    acc_t l = 0;
    for (int e = 0; e < D; ++e) acc[e] = 0;
    for (int64_t i = 0; i < n; ++i) {
      acc_t p = ACC_EXP(sc[i] - m);
      l += p;
      const float* vj = vg + tok[i] * D;
      for (int e = 0; e < D; ++e) acc[e] += p * (acc_t)vj[e];
    }
    for (int e = 0; e < D; ++e) o[(int64_t)h * D + e] = (double)(acc[e] / l);
    if (lse) lse[h] = (double)(m + ACC_LOG(l));
  }
  free(acc);
  free(tok);
  free(sc);
}

/* ------------------------------------------------------------------------ */
/* Backward of one query's sparse attention (Miles docs "Qwen3.8-Flash-Next",  */
/* section 1: the QSA kernel has a forward and a backward pass).  For the     */
/* loss sum_h dout_h . o_h, with P_hj = softmax_j(scale q_h . k_j) over the     */
/* same kept tokens as qsa_ref_attend, the derivative of softmax attention:   */
/*   dv_j  += P_hj dout_h                                                      */
/*   dp_hj  = dout_h . v_j,  delta_h = sum_j P_hj dp_hj                        */
/*   ds_hj  = P_hj (dp_hj - delta_h)                                           */
/*   dq_h   = scale sum_j ds_hj k_j,   dk_j += scale ds_hj q_h                 */
/* q, dout: [n_heads][head_dim]; k, v: [n_groups][ld][head_dim];              */
/* dq: out [n_heads][head_dim]; dk, dv: accumulated, [n_groups][ld][head_dim]. */
/* ------------------------------------------------------------------------ */
void qsa_ref_attend_bwd(const qsa_ref_config* c, const float* q, const float* k,
                        const float* v, int64_t ld, int64_t t, const int32_t* sel,
                        int nsel, const float* dout, double* dq, double* dk, double* dv) {
  int H = c->n_heads, G = c->n_groups, D = c->head_dim, r = c->r;
  int hpg = H / G;
  int64_t maxtok = (int64_t)nsel * r;
  acc_t* p = (acc_t*)malloc(sizeof(acc_t) * (size_t)(maxtok > 0 ? maxtok : 1));
  acc_t* dp = (acc_t*)malloc(sizeof(acc_t) * (size_t)(maxtok > 0 ? maxtok : 1));
  int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)(maxtok > 0 ? maxtok : 1));
  for (int h = 0; h < H; ++h) {
    int g = h / hpg;
    const float* qh = q + (int64_t)h * D;
    const float* doh = dout + (int64_t)h * D;
    const float* kg = k + (int64_t)g * ld * D;
    const float* vg = v + (int64_t)g * ld * D;
    /* probabilities, as in the forward pass */
    int64_t n = 0;
    acc_t m = -INFINITY;
    for (int i = 0; i < nsel; ++i) {
      int64_t b = sel[i];
      for (int64_t j = b * r; j < b * r + r; ++j) {
        if (j > t) continue;
        acc_t dot = 0;
        for (int e = 0; e < D; ++e) dot += (acc_t)qh[e] * (acc_t)kg[j * D + e];
        p[n] = (acc_t)c->softmax_scale * dot;
        tok[n] = j;
        if (p[n] > m) m = p[n];
        ++n;
      }
    }
    acc_t l = 0;
    for (int64_t i = 0; i < n; ++i) {
      p[i] = ACC_EXP(p[i] - m);
      l += p[i];
    }
    for (int64_t i = 0; i < n; ++i) p[i] /= l;
    /* dp and delta */
    acc_t delta = 0;
    for (int64_t i = 0; i < n; ++i) {
      const float* vj = vg + tok[i] * D;
      acc_t dot = 0;
      for (int e = 0; e < D; ++e) dot += (acc_t)doh[e] * (acc_t)vj[e];
      dp[i] = dot;
      delta += p[i] * dot;
    }
    /* gradients */
    for (int e = 0; e < D; ++e) dq[(int64_t)h * D + e] = 0;
    for (int64_t i = 0; i < n; ++i) {
      const int64_t j = tok[i];
      const acc_t ds = p[i] * (dp[i] - delta);
      const acc_t sds = (acc_t)c->softmax_scale * ds;
      for (int e = 0; e < D; ++e) {
        dq[(int64_t)h * D + e] += (double)(sds * (acc_t)kg[j * D + e]);
        dk[((int64_t)g * ld + j) * D + e] += (double)(sds * (acc_t)qh[e]);
        dv[((int64_t)g * ld + j) * D + e] += (double)(p[i] * (acc_t)doh[e]);
      }
    }
  }
  free(tok);
  free(dp);
  free(p);
}

/* ------------------------------------------------------------------------ */
/* The whole path for nq query tokens of ONE sequence.                       */
/* q: [nq][n_heads][head_dim]; q_idx: [nq][idx_heads][idx_dim]; w: [nq][idx_heads];
 * pos: [nq] absolute positions.  k_idx: [>= n][idx_dim]; k, v: [n_groups][ld][head_dim]
 * (the sequence's caches; every position <= max(pos) must be filled).
 * sel: out [nq][S]; nsel: out [nq]; o: out [nq][n_heads][head_dim];
 * lse: out [nq][n_heads] or NULL.  n_threads <= 0 lets OpenMP decide.       */
/* ------------------------------------------------------------------------ */
void qsa_ref_forward(const qsa_ref_config* c, const float* q, const float* q_idx,
                     const float* w, const int64_t* pos, int64_t nq,
                     const float* k_idx, const float* k, const float* v,
                     int64_t ld, int32_t* sel, int32_t* nsel, double* o,
                     double* lse, int n_threads) {
  int S = c->budget_tokens / c->r;
  int64_t maxpos = 0;
  for (int64_t i = 0; i < nq; ++i) if (pos[i] > maxpos) maxpos = pos[i];
  int64_t nblk = maxpos / c->r;                 /* complete blocks needed */
  float* khat = (float*)malloc(sizeof(float) * (size_t)(nblk > 0 ? nblk : 1) * c->idx_dim);
  qsa_ref_compress_keys(c, k_idx, 0, nblk, khat);
  int64_t H = c->n_heads, D = c->head_dim, HI = c->idx_heads, DI = c->idx_dim;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
#endif
  for (int64_t i = 0; i < nq; ++i) {
    int64_t t = pos[i];
    int64_t bt = t / c->r;
    double* s = (double*)malloc(sizeof(double) * (size_t)(bt > 0 ? bt : 1));
    qsa_ref_index_scores(c, q_idx + i * HI * DI, w + i * HI, t, khat, s);
    nsel[i] = qsa_ref_select(c, s, t, sel + i * S);
    qsa_ref_attend(c, q + i * H * D, k, v, ld, t, sel + i * S, nsel[i],
                   o + i * H * D, lse ? lse + i * H : NULL);
    free(s);
  }
  free(khat);
}

int qsa_ref_acc_bits(void) { return (int)(8 * sizeof(acc_t)); }
