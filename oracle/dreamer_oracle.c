/*
 * Dreamer depth-recurrent core forward: CPU oracle.  TEST INFRASTRUCTURE ONLY — loaded by
 * tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg, never by the product.
 *
 * Plain C, float64 throughout, loops in the order the pages give the block (papernotes.org
 * notes on "Depth-Recurrent Attention Mixtures", section "Overall framework", flowchart:
 * RMSNorm -> DA + SA -> residual -> EA -> next depth).  OpenMP, when enabled, only splits
 * loops over independent tokens; no sum is reordered.
 *
 * Readings where the pages leave a step open (each one is named where it is used):
 *  R1  one RMSNorm per depth on the residual stream; the stream continues from x^_l;
 *      no final norm.
 *  R2  DA over depths 0..l inclusive.
 *  R3  separate SA and DA weights, fused as one [h][6h] QKV (qSA kSA vSA qDA kDA vDA, each
 *      head-major) and one [2h][h] O applied to [a_SA | a_DA].
 *  R4  softmax scale 1/sqrt(d); SA causal (key j <= query i).
 *  R5  SA RoPE: rotate-half (pair i with i + d/2), theta_i = base^(-2i/d), position = token
 *      index in its sequence (decode: the cache length).
 *  R6  depth RoPE: each head vector split into two halves of d/2; each half gets rotate-half
 *      RoPE over d/2 dims (theta_i = base^(-2i/(d/2))); first half at position l, second
 *      half at L-1-l.
 *  R7  DA keys/values of depth j come from x^_j, rotated at depth j, stored once.
 *  R8  EA query q_E = y W_qE unrotated; expert keys depth-RoPE'd (R6) at the current depth;
 *      z = q_E . k~_e / sqrt(d_r).
 *  R9  the bias is added to the logit for selection: order by z + b.
 *  R10 ties in z + b go to the lower expert index; w_e = sigmoid(z_e) / sum over picks.
 *  R11 expert FFN SiLU(y W1_e) W2_e, no gate, no biases.
 *  R12 projection router: q_P = x^ W_qP, z_P = q_P . (depth-RoPE'd K_P) / sqrt(d_r), no
 *      bias, p* = argmax (lower index on ties), sigma = sigmoid(z_P[p*]) = max sigma^;
 *      QKV and O share p* and sigma.
 *  R13 decode: one SA cache per depth; the new token writes slot `len` and attends over
 *      len + 1 keys; the DA buffer is per token and rewritten.
 */
#include "dreamer_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void orc_set_threads(int n) {
#ifdef _OPENMP
  omp_set_num_threads(n > 0 ? n : 1);
#else
  (void)n;
#endif
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Round to bfloat16 (nearest even, through float32): the precision in which the bf16 path
 * stores the states its routers read.  Where a float decides an integer (an argmax, a
 * top-k) both sides take the decision on the same stored input.                         */
static double round_bf16(double v) {
  float f = (float)v;
  uint32_t b;
  memcpy(&b, &f, 4);
  b = (b + 0x7FFFu + ((b >> 16) & 1u)) & 0xFFFF0000u;
  memcpy(&f, &b, 4);
  return (double)f;
}

static void *xcalloc(size_t n, size_t sz) {
  void *p = calloc(n ? n : 1, sz);
  return p;
}

/* RMSNorm on the residual stream (notes, "Overall framework": residual RMSNorm; gist,
 * "Methodology": RMSNorm on the residual stream to steer residual scales).
 * out_i = g_i * x_i / sqrt(mean(x^2) + eps).                                           */
void orc_rmsnorm(int h, const double *x, const float *g, double eps, double *out) {
  double ss = 0.0;
  for (int i = 0; i < h; i++) ss += x[i] * x[i];
  double r = 1.0 / sqrt(ss / (double)h + eps);
  for (int i = 0; i < h; i++) out[i] = (double)g[i] * x[i] * r;
}

/* Rotate-half RoPE over n dims at position pos (R5): pair (i, i + n/2), angle
 * pos * base^(-2i/n).                                                                   */
void orc_rope(double *v, int n, double pos, double base) {
  int half = n / 2;
  for (int i = 0; i < half; i++) {
    double theta = pos * pow(base, -2.0 * (double)i / (double)n);
    double c = cos(theta), s = sin(theta);
    double a = v[i], b = v[i + half];
    v[i] = a * c - b * s;
    v[i + half] = b * c + a * s;
  }
}

/* Depth RoPE with a reversed half (notes, "Key design 1": RoPE over the depth index with
 * half of the rotary dims reversed to encode the distance to the maximum depth; gist,
 * "Methodology"): reading R6.                                                            */
void orc_depth_rope(double *v, int n, int l, int L, double base) {
  orc_rope(v, n / 2, (double)l, base);
  orc_rope(v + n / 2, n / 2, (double)(L - 1 - l), base);
}

/* Scaled dot-product attention of one query over nk keys (row stride ldk), R4.
 * probs: scratch of nk doubles, left holding the softmax row.                          */
void orc_attend(const double *q, const double *K, const double *V, int nk, int d, long ldk,
                double *out, double *probs) {
  double scale = 1.0 / sqrt((double)d);
  double mx = -INFINITY;
  for (int j = 0; j < nk; j++) {
    double s = 0.0;
    for (int i = 0; i < d; i++) s += q[i] * K[(long)j * ldk + i];
    s *= scale;
    probs[j] = s;
    if (s > mx) mx = s;
  }
  double Z = 0.0;
  for (int j = 0; j < nk; j++) {
    probs[j] = exp(probs[j] - mx);
    Z += probs[j];
  }
  for (int j = 0; j < nk; j++) probs[j] /= Z;
  for (int i = 0; i < d; i++) out[i] = 0.0;
  for (int j = 0; j < nk; j++)
    for (int i = 0; i < d; i++) out[i] += probs[j] * V[(long)j * ldk + i];
}

/* Routing sigma(x) = norm(TopK(sigmoid(x), x + b, k)) (notes, "Key design 2"):
 * pick k experts by z + b (R9, ties to the lower index, R10), weight each by sigmoid(z)
 * normalised over the picks.  margin = (z+b) of the k-th pick minus the best unpicked.  */
void orc_topk(const double *z, const float *bias, int E, int k, int32_t *idx, double *w,
              double *margin) {
  char *taken = (char *)xcalloc((size_t)E, 1);
  double kth = 0.0;
  for (int s = 0; s < k; s++) {
    int bi = -1;
    double best = 0.0;
    for (int e = 0; e < E; e++) {
      if (taken[e]) continue;
      double v = z[e] + (double)bias[e];
      if (bi < 0 || v > best) {
        best = v;
        bi = e;
      }
    }
    taken[bi] = 1;
    idx[s] = bi;
    kth = best;
  }
  if (margin) {
    if (k < E) {
      double bu = -INFINITY;
      for (int e = 0; e < E; e++)
        if (!taken[e] && z[e] + (double)bias[e] > bu) bu = z[e] + (double)bias[e];
      *margin = kth - bu;
    } else {
      *margin = INFINITY;
    }
  }
  double sum = 0.0;
  for (int s = 0; s < k; s++) sum += sigmoid(z[idx[s]]);
  for (int s = 0; s < k; s++) w[s] = sigmoid(z[idx[s]]) / sum;
  free(taken);
}

/* Linear-MoE projection, top-1 with a shared expert (notes, "Key design 3"):
 * sigma x W_p + max(sigma^) x W_shared, and under top-1 max(sigma^) = sigma.            */
void orc_linear_moe(int in, int out, const double *x, const float *Wp, const float *Wsh,
                    double sigma, double *y) {
  for (int j = 0; j < out; j++) {
    double ap = 0.0, as = 0.0;
    for (int i = 0; i < in; i++) {
      ap += x[i] * (double)Wp[(long)i * out + j];
      as += x[i] * (double)Wsh[(long)i * out + j];
    }
    y[j] = sigma * ap + sigma * as;
  }
}

/* The absorbed right-hand side of the same identity: sigma x (W_p + W_shared).        */
void orc_linear_moe_absorbed(int in, int out, const double *x, const float *Wp,
                             const float *Wsh, double sigma, double *y) {
  for (int j = 0; j < out; j++) {
    double a = 0.0;
    for (int i = 0; i < in; i++)
      a += x[i] * ((double)Wp[(long)i * out + j] + (double)Wsh[(long)i * out + j]);
    y[j] = sigma * a;
  }
}

/* Expert "value" FFN, R11: out = SiLU(y W1_e) W2_e.                                     */
void orc_expert(int h, int m, const double *y, const float *w1e, const float *w2e,
                double *out) {
  double *u = (double *)xcalloc((size_t)m, sizeof(double));
  for (int i = 0; i < h; i++)
    for (int j = 0; j < m; j++) u[j] += y[i] * (double)w1e[(long)i * m + j];
  for (int j = 0; j < m; j++) u[j] = u[j] * sigmoid(u[j]);
  for (int i = 0; i < h; i++) out[i] = 0.0;
  for (int j = 0; j < m; j++)
    for (int i = 0; i < h; i++) out[i] += u[j] * (double)w2e[(long)j * h + i];
  free(u);
}

/* Bias balance update (notes, "Key design 2"): b <- b + lambda sign(median(N) - N),
 * N_e summed over depths; the median of an even count is the lower middle value.       */
static int cmp_i64(const void *a, const void *b) {
  long long x = *(const long long *)a, y = *(const long long *)b;
  return (x > y) - (x < y);
}
void orc_bias_update(int L, int E, const int32_t *counts, double lambda, double *bias) {
  long long *N = (long long *)xcalloc((size_t)E, sizeof(long long));
  long long *srt = (long long *)xcalloc((size_t)E, sizeof(long long));
  for (int l = 0; l < L; l++)
    for (int e = 0; e < E; e++) N[e] += counts[(long)l * E + e];
  memcpy(srt, N, sizeof(long long) * (size_t)E);
  qsort(srt, (size_t)E, sizeof(long long), cmp_i64);
  long long med = srt[(E - 1) / 2];
  for (int e = 0; e < E; e++) {
    double sg = (med > N[e]) ? 1.0 : (med < N[e] ? -1.0 : 0.0);
    bias[e] += lambda * sg;
  }
  free(N);
  free(srt);
}

/* ------------------------------------------------------------------------------------ */
/* projections                                                                           */

/* out[j] = sum_i x[i] * W[(row0 + i) * ld + col0 + j] for j < ncol, over the routed
 * expert's matrix Wp and, for the linear MoE, plus the shared matrix, both scaled by
 * sigma (R12 with the identity of "Key design 3").  Dense projections: Wsh == NULL.
 * Loops run over the rows of W (i outer) so W streams once; every out[j] is still the sum
 * over i = 0, 1, ... in that order.                                                       */
static void proj(const double *x, int nin, const float *Wp, const float *Wsh, long ld, int row0,
                 int col0, int ncol, double sigma, double *out) {
  double *ap = (double *)xcalloc((size_t)ncol, sizeof(double));
  double *as = Wsh ? (double *)xcalloc((size_t)ncol, sizeof(double)) : NULL;
  for (int i = 0; i < nin; i++) {
    const double xi = x[i];
    const float *wr = Wp + (long)(row0 + i) * ld + col0;
    for (int j = 0; j < ncol; j++) ap[j] += xi * (double)wr[j];
    if (Wsh) {
      const float *sr = Wsh + (long)(row0 + i) * ld + col0;
      for (int j = 0; j < ncol; j++) as[j] += xi * (double)sr[j];
    }
  }
  for (int j = 0; j < ncol; j++) out[j] = Wsh ? (sigma * ap[j] + sigma * as[j]) : ap[j];
  free(ap);
  free(as);
}

/* depth-RoPE'd key table for depth l: rot[e][:] = R_l key[e][:] (R6, R8)               */
static void rotate_keys(const float *key, int n, int dr, int l, int L, double base,
                        double *rot) {
  for (int e = 0; e < n; e++) {
    for (int i = 0; i < dr; i++) rot[(long)e * dr + i] = (double)key[(long)e * dr + i];
    orc_depth_rope(rot + (long)e * dr, dr, l, L, base);
  }
}

/* Projection router for one token (R12).                                                */
static void proj_route(const orc_cfg *c, const orc_weights *W, const double *krotP,
                       const double *xh, int32_t *pstar, double *sigma, double *pmargin) {
  int dr = c->dr, P = c->P;
  double q[1024];
  double z[256] = {0.0};
  for (int j = 0; j < dr; j++) q[j] = 0.0;
  for (int i = 0; i < c->h; i++) {
    const double xi = c->route_bf16 ? round_bf16(xh[i]) : xh[i];
    for (int j = 0; j < dr; j++) q[j] += xi * (double)W->w_qP[(long)i * dr + j];
  }
  for (int p = 0; p < P; p++) {
    double s = 0.0;
    for (int j = 0; j < dr; j++) s += q[j] * krotP[(long)p * dr + j];
    z[p] = s / sqrt((double)dr);
  }
  int best = 0;
  for (int p = 1; p < P; p++)
    if (z[p] > z[best]) best = p;
  double second = -INFINITY;
  for (int p = 0; p < P; p++)
    if (p != best && z[p] > second) second = z[p];
  *pstar = best;
  *sigma = sigmoid(z[best]);
  if (pmargin) *pmargin = z[best] - second;
}

/* EA router query and scores for one token (R8): z_e = (x W_qE) . k~_e / sqrt(d_r).    */
static void ea_scores(const orc_cfg *c, const orc_weights *W, const double *krotE,
                      const double *x, double *z) {
  int dr = c->dr;
  double q[1024];
  for (int j = 0; j < dr; j++) q[j] = 0.0;
  for (int i = 0; i < c->h; i++) {
    const double xi = c->route_bf16 ? round_bf16(x[i]) : x[i];
    for (int j = 0; j < dr; j++) q[j] += xi * (double)W->w_qE[(long)i * dr + j];
  }
  for (int e = 0; e < c->E; e++) {
    double s = 0.0;
    for (int j = 0; j < dr; j++) s += q[j] * krotE[(long)e * dr + j];
    z[e] = s / sqrt((double)dr);
  }
}

/* EA for one token: route, then x_next = base + sum_s w_s Expert_{idx_s}(x_in).         */
static void ea_token(const orc_cfg *c, const orc_weights *W, const double *krotE,
                     const double *x_in, const double *base, double *x_next, int32_t *idx,
                     double *w, double *margin, double *zsel) {
  int h = c->h, k = c->k, E = c->E, m = c->m;
  double *z = (double *)xcalloc((size_t)E, sizeof(double));
  double *ye = (double *)xcalloc((size_t)h, sizeof(double));
  double mg;
  ea_scores(c, W, krotE, x_in, z);
  orc_topk(z, W->bias, E, k, idx, w, &mg);
  if (margin) *margin = mg;
  if (zsel) {
    for (int s = 0; s < k; s++) zsel[s] = z[idx[s]] + (double)W->bias[idx[s]];
    zsel[k] = (k < E) ? zsel[k - 1] - mg : -INFINITY;
  }
  for (int i = 0; i < h; i++) x_next[i] = base[i];
  for (int s = 0; s < k; s++) {
    int e = idx[s];
    orc_expert(h, m, x_in, W->w1 + (long)e * h * m, W->w2 + (long)e * m * h, ye);
    for (int i = 0; i < h; i++) x_next[i] += w[s] * ye[i];
  }
  free(z);
  free(ye);
}

static const float *wsel(const float *base, int P, long per, int p) {
  return base + (P > 0 ? (long)p * per : 0);
}

/* ------------------------------------------------------------------------------------ */
/* First depth that depth attention at depth l reads: 0 (all earlier depths, R2), or the
 * first of the last W depths with a sliding window (the pages' sparse-DA outlook); -1 when
 * the layout has no depth attention (variant 3).                                        */
static int da_first(const orc_cfg *c, int l) {
  if (c->variant == 3) return -1;
  if (c->da_window > 0 && l + 1 > c->da_window) return l + 1 - c->da_window;
  return 0;
}

/* prefill forward                                                                       */

static int forward_impl(const orc_cfg *c, const orc_weights *W, const float *x_in, int l0,
                        int l1, double *da_kv, double *x_out, orc_trace *tr, int da_loops) {
  const int B = c->B, S = c->S, h = c->h, H = c->H, d = c->d, L = c->L, k = c->k;
  const int P = c->P, dr = c->dr;
  const long T = (long)B * S;
  const long h6 = 6L * h;
  if (h != H * d || d % 4 || dr % 4 || l0 < 0 || l1 > L || l0 > l1 || k > c->E) return -1;
  if (P > 256 || dr > 1024 || h > 4096 || L > 1024) return -2;

  double *x = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *xh = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *u = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *qkv_sa = (double *)xcalloc((size_t)(T * 3 * h), sizeof(double));
  double *q_da = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *a_sa = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *a_da = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *y = (double *)xcalloc((size_t)(T * h), sizeof(double));
  double *xn = (double *)xcalloc((size_t)(T * h), sizeof(double));
  int32_t *pst = (int32_t *)xcalloc((size_t)T, sizeof(int32_t));
  double *sig = (double *)xcalloc((size_t)T, sizeof(double));
  double *pmg = (double *)xcalloc((size_t)T, sizeof(double));
  int32_t *idx = (int32_t *)xcalloc((size_t)(T * k), sizeof(int32_t));
  double *wts = (double *)xcalloc((size_t)(T * k), sizeof(double));
  double *mg = (double *)xcalloc((size_t)T, sizeof(double));
  double *zs = (double *)xcalloc((size_t)(T * (k + 1)), sizeof(double));
  double *krotE = (double *)xcalloc((size_t)c->E * dr, sizeof(double));
  double *krotP = (double *)xcalloc((size_t)(P > 0 ? P : 1) * dr, sizeof(double));
  const long perQKV = (long)h * h6, perO = 2L * h * h;

  for (long i = 0; i < T * h; i++) x[i] = (double)x_in[i];

  for (int l = l0; l < l1; l++) {
    rotate_keys(W->k_E, c->E, dr, l, L, c->rope_base, krotE);
    if (P > 0) rotate_keys(W->k_P, P, dr, l, L, c->rope_base, krotP);

    /* RMSNorm, projection routing, DA projections (q, k, v of depth attention) */
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      double tmp[3 * 4096];
      orc_rmsnorm(h, x + t * h, W->g, c->eps, xh + t * h);
      if (P > 0) {
        proj_route(c, W, krotP, xh + t * h, &pst[t], &sig[t], &pmg[t]);
      } else {
        pst[t] = 0;
        sig[t] = 1.0;
        pmg[t] = INFINITY;
      }
      const float *Wq = wsel(W->w_qkv, P, perQKV, pst[t]);
      proj(xh + t * h, h, Wq, P > 0 ? W->w_qkv_sh : NULL, h6, 0, 3 * h, 3 * h, sig[t], tmp);
      for (int hd = 0; hd < H; hd++) {
        orc_depth_rope(tmp + hd * d, d, l, L, c->rope_base);          /* q_DA (R6) */
        orc_depth_rope(tmp + h + hd * d, d, l, L, c->rope_base);      /* k_DA (R6) */
      }
      for (int i = 0; i < h; i++) {
        q_da[t * h + i] = tmp[i];
        da_kv[((t * L + l) * 2 + 0) * h + i] = tmp[h + i];            /* R7 */
        da_kv[((t * L + l) * 2 + 1) * h + i] = tmp[2 * h + i];
      }
    }

    /* depth attention over depths j0..l of the same token (R2; j0 > 0 with a window) */
    const int j0 = da_first(c, l);
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      double probs[1024];
      for (int hd = 0; hd < H; hd++) {
        const double *q = q_da + t * h + hd * d;
        double *o = a_da + t * h + hd * d;
        if (j0 < 0) {  /* no depth attention */
          for (int i = 0; i < d; i++) o[i] = 0.0;
        } else if (!da_loops) {
          /* reshape view (notes, "Key design 1"; gist, "Methodology"): the b*s tokens are
           * the batch, the depth index is the sequence; the token's query sits at depth
           * position l and attends over its own depth sequence 0..l.                    */
          const double *Kseq = da_kv + ((t * L + j0) * 2 + 0) * h + hd * d;
          const double *Vseq = da_kv + ((t * L + j0) * 2 + 1) * h + hd * d;
          orc_attend(q, Kseq, Vseq, l + 1 - j0, d, 2L * h, o, probs);
        } else {
          /* explicit loops over depths j = j0..l */
          double sc[1024], mx = -INFINITY, Z = 0.0;
          for (int j = j0; j <= l; j++) {
            double s = 0.0;
            for (int i = 0; i < d; i++)
              s += q[i] * da_kv[((t * L + j) * 2 + 0) * h + hd * d + i];
            sc[j] = s / sqrt((double)d);
            if (sc[j] > mx) mx = sc[j];
          }
          for (int j = j0; j <= l; j++) {
            sc[j] = exp(sc[j] - mx);
            Z += sc[j];
          }
          for (int i = 0; i < d; i++) {
            double acc = 0.0;
            for (int j = j0; j <= l; j++)
              acc += (sc[j] / Z) * da_kv[((t * L + j) * 2 + 1) * h + hd * d + i];
            o[i] = acc;
          }
        }
      }
    }

    /* SA input: x^ (parallel layouts) or x^ + DA output (serial layout DA -> SA -> EA) */
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      double tmp[4096];
      if (c->variant == 1) {
        const float *Wo = wsel(W->w_o, P, perO, pst[t]);
        proj(a_da + t * h, h, Wo, P > 0 ? W->w_o_sh : NULL, h, h, 0, h, sig[t], tmp);
        for (int i = 0; i < h; i++) u[t * h + i] = xh[t * h + i] + tmp[i];
      } else {
        for (int i = 0; i < h; i++) u[t * h + i] = xh[t * h + i];
      }
      const float *Wq = wsel(W->w_qkv, P, perQKV, pst[t]);
      double *o = qkv_sa + t * 3 * h;
      proj(u + t * h, h, Wq, P > 0 ? W->w_qkv_sh : NULL, h6, 0, 0, 3 * h, sig[t], o);
      double pos = (double)(t % S);
      for (int hd = 0; hd < H; hd++) {
        orc_rope(o + hd * d, d, pos, c->rope_base);      /* q_SA (R5) */
        orc_rope(o + h + hd * d, d, pos, c->rope_base);  /* k_SA (R5) */
      }
    }

    /* causal sequence attention inside each sequence (R4) */
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      long b = t / S, i = t % S;
      double *probs = (double *)xcalloc((size_t)S, sizeof(double));
      for (int hd = 0; hd < H; hd++) {
        const double *q = qkv_sa + t * 3 * h + hd * d;
        const double *K = qkv_sa + (b * S) * 3 * h + h + hd * d;
        const double *V = qkv_sa + (b * S) * 3 * h + 2 * h + hd * d;
        orc_attend(q, K, V, (int)i + 1, d, 3L * h, a_sa + t * h + hd * d, probs);
      }
      free(probs);
    }

    /* residual: y = x^ + DA + SA through the O projection (notes, "Key design 1") */
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      double cat[2 * 4096], tmp[4096];
      const float *Wo = wsel(W->w_o, P, perO, pst[t]);
      const float *Wsh = P > 0 ? W->w_o_sh : NULL;
      if (c->variant == 1) {
        proj(a_sa + t * h, h, Wo, Wsh, h, 0, 0, h, sig[t], tmp);
        for (int i = 0; i < h; i++) y[t * h + i] = u[t * h + i] + tmp[i];
      } else {
        for (int i = 0; i < h; i++) {
          cat[i] = a_sa[t * h + i];
          cat[h + i] = a_da[t * h + i];
        }
        proj(cat, 2 * h, Wo, Wsh, h, 0, 0, h, sig[t], tmp);
        for (int i = 0; i < h; i++) y[t * h + i] = xh[t * h + i] + tmp[i];
      }
    }

    /* expert attention (notes, "Key design 2"); fully parallel layout routes x^ */
#pragma omp parallel for schedule(dynamic, 4)
    for (long t = 0; t < T; t++) {
      const double *ein = (c->variant == 2) ? xh + t * h : y + t * h;
      ea_token(c, W, krotE, ein, y + t * h, xn + t * h, idx + t * k, wts + t * k, &mg[t],
               zs + t * (k + 1));
    }

    if (tr) {
      long off = (long)l * T;
      if (tr->xhat) memcpy(tr->xhat + off * h, xh, sizeof(double) * T * h);
      if (tr->y) memcpy(tr->y + off * h, y, sizeof(double) * T * h);
      if (tr->idx) memcpy(tr->idx + off * k, idx, sizeof(int32_t) * T * k);
      if (tr->w) memcpy(tr->w + off * k, wts, sizeof(double) * T * k);
      if (tr->margin) memcpy(tr->margin + off, mg, sizeof(double) * T);
      if (tr->zsel) memcpy(tr->zsel + off * (k + 1), zs, sizeof(double) * T * (k + 1));
      if (tr->pidx) memcpy(tr->pidx + off, pst, sizeof(int32_t) * T);
      if (tr->psig) memcpy(tr->psig + off, sig, sizeof(double) * T);
      if (tr->pmargin) memcpy(tr->pmargin + off, pmg, sizeof(double) * T);
      if (tr->counts)
        for (long t = 0; t < T * k; t++) tr->counts[(long)l * c->E + idx[t]] += 1;
      for (long t = 0; t < T; t++)
        for (int i = 0; i < h; i++) {
          if (tr->sa_k) tr->sa_k[(off + t) * h + i] = qkv_sa[t * 3 * h + h + i];
          if (tr->sa_v) tr->sa_v[(off + t) * h + i] = qkv_sa[t * 3 * h + 2 * h + i];
        }
    }
    memcpy(x, xn, sizeof(double) * T * h);
  }
  memcpy(x_out, x, sizeof(double) * T * h);

  free(x); free(xh); free(u); free(qkv_sa); free(q_da); free(a_sa); free(a_da); free(y);
  free(xn); free(pst); free(sig); free(pmg); free(idx); free(wts); free(mg); free(zs);
  free(krotE); free(krotP);
  return 0;
}

int orc_forward(const orc_cfg *c, const orc_weights *W, const float *x_in, int l0, int l1,
                double *da_kv, double *x_out, orc_trace *tr) {
  return forward_impl(c, W, x_in, l0, l1, da_kv, x_out, tr, 0);
}

int orc_forward_da_loops(const orc_cfg *c, const orc_weights *W, const float *x_in, int l0,
                         int l1, double *da_kv, double *x_out, orc_trace *tr) {
  return forward_impl(c, W, x_in, l0, l1, da_kv, x_out, tr, 1);
}

/* ------------------------------------------------------------------------------------ */
/* one depth for selected tokens of one sequence                                         */

int orc_step_tokens(const orc_cfg *c, const orc_weights *W, int l, const float *x_seq,
                    int n_ctx, const double *da_hist, const int32_t *pos, int n_s,
                    double *x_out, orc_trace *tr) {
  const int h = c->h, H = c->H, d = c->d, L = c->L, k = c->k, P = c->P, dr = c->dr;
  const long h6 = 6L * h, perQKV = (long)h * h6, perO = 2L * h * h;
  if (c->variant == 1) return -2; /* serial layout needs every context token's DA */
  if (h != H * d || d % 4 || l < 0 || l >= L || P > 256 || dr > 1024) return -1;
  int n_need = 0;
  for (int s = 0; s < n_s; s++) {
    if (pos[s] < 0 || pos[s] >= n_ctx) return -1;
    if (pos[s] + 1 > n_need) n_need = pos[s] + 1;
  }
  double *xh = (double *)xcalloc((size_t)n_need * h, sizeof(double));
  double *kv = (double *)xcalloc((size_t)n_need * 2 * h, sizeof(double));
  int32_t *pst = (int32_t *)xcalloc((size_t)n_need, sizeof(int32_t));
  double *sig = (double *)xcalloc((size_t)n_need, sizeof(double));
  double *pmg = (double *)xcalloc((size_t)n_need, sizeof(double));
  double *krotE = (double *)xcalloc((size_t)c->E * dr, sizeof(double));
  double *krotP = (double *)xcalloc((size_t)(P > 0 ? P : 1) * dr, sizeof(double));
  rotate_keys(W->k_E, c->E, dr, l, L, c->rope_base, krotE);
  if (P > 0) rotate_keys(W->k_P, P, dr, l, L, c->rope_base, krotP);

  /* x^, routing and post-RoPE SA keys/values of every context token up to the last one
   * selected */
#pragma omp parallel for schedule(dynamic, 4)
  for (long t = 0; t < n_need; t++) {
    double xd[4096];
    for (int i = 0; i < h; i++) xd[i] = (double)x_seq[t * h + i];
    orc_rmsnorm(h, xd, W->g, c->eps, xh + t * h);
    if (P > 0) {
      proj_route(c, W, krotP, xh + t * h, &pst[t], &sig[t], &pmg[t]);
    } else {
      pst[t] = 0;
      sig[t] = 1.0;
      pmg[t] = INFINITY;
    }
    const float *Wq = wsel(W->w_qkv, P, perQKV, pst[t]);
    proj(xh + t * h, h, Wq, P > 0 ? W->w_qkv_sh : NULL, h6, 0, h, 2 * h, sig[t],
         kv + t * 2 * h);
    for (int hd = 0; hd < H; hd++) orc_rope(kv + t * 2 * h + hd * d, d, (double)t, c->rope_base);
  }

#pragma omp parallel for schedule(dynamic, 1)
  for (int s = 0; s < n_s; s++) {
    long t = pos[s];
    double *qs = (double *)xcalloc((size_t)h, sizeof(double));
    double *qkvd = (double *)xcalloc((size_t)3 * h, sizeof(double));
    double *dkv = (double *)xcalloc((size_t)L * 2 * h, sizeof(double));
    double *cat = (double *)xcalloc((size_t)2 * h, sizeof(double));
    double *yv = (double *)xcalloc((size_t)h, sizeof(double));
    double *tmp = (double *)xcalloc((size_t)h, sizeof(double));
    double *probs = (double *)xcalloc((size_t)(n_ctx > L ? n_ctx : L), sizeof(double));
    const float *Wq = wsel(W->w_qkv, P, perQKV, pst[t]);
    const float *Wqs = P > 0 ? W->w_qkv_sh : NULL;
    proj(xh + t * h, h, Wq, Wqs, h6, 0, 0, h, sig[t], qs);
    proj(xh + t * h, h, Wq, Wqs, h6, 0, 3 * h, 3 * h, sig[t], qkvd);
    for (int hd = 0; hd < H; hd++) {
      orc_rope(qs + hd * d, d, (double)t, c->rope_base);
      orc_depth_rope(qkvd + hd * d, d, l, L, c->rope_base);
      orc_depth_rope(qkvd + h + hd * d, d, l, L, c->rope_base);
    }
    for (int j = 0; j < l; j++)
      for (int i = 0; i < 2 * h; i++)
        dkv[(long)j * 2 * h + i] = da_hist[((long)s * L + j) * 2 * h + i];
    for (int i = 0; i < 2 * h; i++) dkv[(long)l * 2 * h + i] = qkvd[h + i];
    const int j0 = da_first(c, l);
    for (int hd = 0; hd < H; hd++) {
      orc_attend(qs + hd * d, kv + hd * d, kv + h + hd * d, (int)t + 1, d, 2L * h,
                 cat + hd * d, probs);
      if (j0 < 0)
        for (int i = 0; i < d; i++) cat[h + hd * d + i] = 0.0;
      else
        orc_attend(qkvd + hd * d, dkv + (long)j0 * 2 * h + hd * d, dkv + (long)j0 * 2 * h + h + hd * d,
                   l + 1 - j0, d, 2L * h, cat + h + hd * d, probs);
    }
    const float *Wo = wsel(W->w_o, P, perO, pst[t]);
    proj(cat, 2 * h, Wo, P > 0 ? W->w_o_sh : NULL, h, 0, 0, h, sig[t], tmp);
    for (int i = 0; i < h; i++) yv[i] = xh[t * h + i] + tmp[i];
    double mgs;
    int32_t *ix = (int32_t *)xcalloc((size_t)k, sizeof(int32_t));
    double *wv = (double *)xcalloc((size_t)k, sizeof(double));
    double *zs = (double *)xcalloc((size_t)k + 1, sizeof(double));
    const double *ein = (c->variant == 2) ? xh + t * h : yv;
    ea_token(c, W, krotE, ein, yv, x_out + (long)s * h, ix, wv, &mgs, zs);
    if (tr) {
      if (tr->xhat) memcpy(tr->xhat + (long)s * h, xh + t * h, sizeof(double) * h);
      if (tr->y) memcpy(tr->y + (long)s * h, yv, sizeof(double) * h);
      if (tr->idx) memcpy(tr->idx + (long)s * k, ix, sizeof(int32_t) * k);
      if (tr->w) memcpy(tr->w + (long)s * k, wv, sizeof(double) * k);
      if (tr->margin) tr->margin[s] = mgs;
      if (tr->zsel) memcpy(tr->zsel + (long)s * (k + 1), zs, sizeof(double) * (k + 1));
      if (tr->pidx) tr->pidx[s] = pst[t];
      if (tr->psig) tr->psig[s] = sig[t];
      if (tr->pmargin) tr->pmargin[s] = pmg[t];
      if (tr->sa_k) memcpy(tr->sa_k + (long)s * h, kv + t * 2 * h, sizeof(double) * h);
      if (tr->sa_v) memcpy(tr->sa_v + (long)s * h, kv + t * 2 * h + h, sizeof(double) * h);
    }
    free(qs); free(qkvd); free(dkv); free(cat); free(yv); free(tmp); free(probs);
    free(ix); free(wv); free(zs);
  }
  if (tr && tr->counts && tr->idx)
    for (long i = 0; i < (long)n_s * k; i++) tr->counts[tr->idx[i]] += 1;

  free(xh); free(kv); free(pst); free(sig); free(pmg); free(krotE); free(krotP);
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* decode: one new token of one sequence through all depths (R13)                        */

int orc_decode_seq(const orc_cfg *c, const orc_weights *W, const float *x_new, double *kc,
                   double *vc, int cap, int len, double *x_out, orc_trace *tr) {
  const int h = c->h, H = c->H, d = c->d, L = c->L, k = c->k, P = c->P, dr = c->dr;
  const long h6 = 6L * h, perQKV = (long)h * h6, perO = 2L * h * h;
  if (h != H * d || d % 4 || len < 0 || len >= cap || P > 256 || dr > 1024) return -1;
  double *x = (double *)xcalloc((size_t)h, sizeof(double));
  double *xh = (double *)xcalloc((size_t)h, sizeof(double));
  double *u = (double *)xcalloc((size_t)h, sizeof(double));
  double *qkv = (double *)xcalloc((size_t)h6, sizeof(double));
  double *dkv = (double *)xcalloc((size_t)L * 2 * h, sizeof(double));
  double *cat = (double *)xcalloc((size_t)2 * h, sizeof(double));
  double *tmp = (double *)xcalloc((size_t)h, sizeof(double));
  double *y = (double *)xcalloc((size_t)h, sizeof(double));
  double *xn = (double *)xcalloc((size_t)h, sizeof(double));
  double *probs = (double *)xcalloc((size_t)(cap > L ? cap : L), sizeof(double));
  double *krotE = (double *)xcalloc((size_t)c->E * dr, sizeof(double));
  double *krotP = (double *)xcalloc((size_t)(P > 0 ? P : 1) * dr, sizeof(double));
  int32_t *ix = (int32_t *)xcalloc((size_t)k, sizeof(int32_t));
  double *wv = (double *)xcalloc((size_t)k, sizeof(double));
  double *zs = (double *)xcalloc((size_t)k + 1, sizeof(double));
  for (int i = 0; i < h; i++) x[i] = (double)x_new[i];

  for (int l = 0; l < L; l++) {
    rotate_keys(W->k_E, c->E, dr, l, L, c->rope_base, krotE);
    if (P > 0) rotate_keys(W->k_P, P, dr, l, L, c->rope_base, krotP);
    int32_t ps = 0;
    double sg = 1.0, pm = INFINITY;
    orc_rmsnorm(h, x, W->g, c->eps, xh);
    if (P > 0) proj_route(c, W, krotP, xh, &ps, &sg, &pm);
    const float *Wq = wsel(W->w_qkv, P, perQKV, ps);
    const float *Wqs = P > 0 ? W->w_qkv_sh : NULL;
    const float *Wo = wsel(W->w_o, P, perO, ps);
    const float *Wos = P > 0 ? W->w_o_sh : NULL;
    /* DA part */
    proj(xh, h, Wq, Wqs, h6, 0, 3 * h, 3 * h, sg, qkv + 3 * h);
    for (int hd = 0; hd < H; hd++) {
      orc_depth_rope(qkv + 3 * h + hd * d, d, l, L, c->rope_base);
      orc_depth_rope(qkv + 4 * h + hd * d, d, l, L, c->rope_base);
    }
    for (int i = 0; i < 2 * h; i++) dkv[(long)l * 2 * h + i] = qkv[4 * h + i];
    const int j0 = da_first(c, l);
    for (int hd = 0; hd < H; hd++) {
      if (j0 < 0)
        for (int i = 0; i < d; i++) cat[h + hd * d + i] = 0.0;
      else
        orc_attend(qkv + 3 * h + hd * d, dkv + (long)j0 * 2 * h + hd * d,
                   dkv + (long)j0 * 2 * h + h + hd * d, l + 1 - j0, d, 2L * h,
                   cat + h + hd * d, probs);
    }
    if (c->variant == 1) {
      proj(cat + h, h, Wo, Wos, h, h, 0, h, sg, tmp);
      for (int i = 0; i < h; i++) u[i] = xh[i] + tmp[i];
    } else {
      for (int i = 0; i < h; i++) u[i] = xh[i];
    }
    /* SA part: the new key/value go to slot len of this depth's cache */
    proj(u, h, Wq, Wqs, h6, 0, 0, 3 * h, sg, qkv);
    for (int hd = 0; hd < H; hd++) {
      orc_rope(qkv + hd * d, d, (double)len, c->rope_base);
      orc_rope(qkv + h + hd * d, d, (double)len, c->rope_base);
      double *kh = kc + (((long)l * H + hd) * cap) * d;
      double *vh = vc + (((long)l * H + hd) * cap) * d;
      for (int i = 0; i < d; i++) {
        kh[(long)len * d + i] = qkv[h + hd * d + i];
        vh[(long)len * d + i] = qkv[2 * h + hd * d + i];
      }
      orc_attend(qkv + hd * d, kh, vh, len + 1, d, d, cat + hd * d, probs);
    }
    if (c->variant == 1) {
      proj(cat, h, Wo, Wos, h, 0, 0, h, sg, tmp);
      for (int i = 0; i < h; i++) y[i] = u[i] + tmp[i];
    } else {
      proj(cat, 2 * h, Wo, Wos, h, 0, 0, h, sg, tmp);
      for (int i = 0; i < h; i++) y[i] = xh[i] + tmp[i];
    }
    double mgs;
    ea_token(c, W, krotE, c->variant == 2 ? xh : y, y, xn, ix, wv, &mgs, zs);
    if (tr) {
      if (tr->xhat) memcpy(tr->xhat + (long)l * h, xh, sizeof(double) * h);
      if (tr->y) memcpy(tr->y + (long)l * h, y, sizeof(double) * h);
      if (tr->idx) memcpy(tr->idx + (long)l * k, ix, sizeof(int32_t) * k);
      if (tr->w) memcpy(tr->w + (long)l * k, wv, sizeof(double) * k);
      if (tr->margin) tr->margin[l] = mgs;
      if (tr->zsel) memcpy(tr->zsel + (long)l * (k + 1), zs, sizeof(double) * (k + 1));
      if (tr->pidx) tr->pidx[l] = ps;
      if (tr->psig) tr->psig[l] = sg;
      if (tr->pmargin) tr->pmargin[l] = pm;
      if (tr->counts)
        for (int s = 0; s < k; s++) tr->counts[(long)l * c->E + ix[s]] += 1;
    }
    memcpy(x, xn, sizeof(double) * h);
  }
  memcpy(x_out, x, sizeof(double) * h);
  free(x); free(xh); free(u); free(qkv); free(dkv); free(cat); free(tmp); free(y); free(xn);
  free(probs); free(krotE); free(krotP); free(ix); free(wv); free(zs);
  return 0;
}

/* ------------------------------------------------------------------------------------ */

int orc_route(const orc_cfg *c, const orc_weights *W, int l, const float *y, int T,
              int32_t *idx, double *w, double *margin, double *zsel, int32_t *counts) {
  const int h = c->h, k = c->k, dr = c->dr, E = c->E;
  if (l < 0 || l >= c->L || dr > 1024 || k > E) return -1;
  double *krotE = (double *)xcalloc((size_t)E * dr, sizeof(double));
  rotate_keys(W->k_E, E, dr, l, c->L, c->rope_base, krotE);
#pragma omp parallel for schedule(dynamic, 8)
  for (long t = 0; t < T; t++) {
    double *yd = (double *)xcalloc((size_t)h, sizeof(double));
    double *z = (double *)xcalloc((size_t)E, sizeof(double));
    double mg;
    for (int i = 0; i < h; i++) yd[i] = (double)y[t * h + i];
    ea_scores(c, W, krotE, yd, z);
    orc_topk(z, W->bias, E, k, idx + t * k, w + t * k, &mg);
    if (margin) margin[t] = mg;
    if (zsel) {
      for (int s = 0; s < k; s++) zsel[t * (k + 1) + s] = z[idx[t * k + s]] + W->bias[idx[t * k + s]];
      zsel[t * (k + 1) + k] = (k < E) ? zsel[t * (k + 1) + k - 1] - mg : -INFINITY;
    }
    free(yd);
    free(z);
  }
  if (counts)
    for (long i = 0; i < (long)T * k; i++) counts[idx[i]] += 1;
  free(krotE);
  return 0;
}

/* Projection router alone on given normalised states (R12): x^ [T][h] at depth l ->
 * p* [T], sigma [T], margin z_P[p*] - runner-up [T] (margin may be NULL).             */
int orc_proj_route(const orc_cfg *c, const orc_weights *W, int l, const float *xh, int T,
                   int32_t *pstar, double *sigma, double *pmargin) {
  const int h = c->h, dr = c->dr, P = c->P;
  if (P < 1 || P > 256 || l < 0 || l >= c->L || dr > 1024) return -1;
  double *krotP = (double *)xcalloc((size_t)P * dr, sizeof(double));
  rotate_keys(W->k_P, P, dr, l, c->L, c->rope_base, krotP);
#pragma omp parallel for schedule(dynamic, 8)
  for (long t = 0; t < T; t++) {
    double *xd = (double *)xcalloc((size_t)h, sizeof(double));
    for (int i = 0; i < h; i++) xd[i] = (double)xh[t * h + i];
    proj_route(c, W, krotP, xd, &pstar[t], &sigma[t], pmargin ? &pmargin[t] : NULL);
    free(xd);
  }
  free(krotP);
  return 0;
}
