/*
 * Dreamer depth-recurrent core forward: CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference leg may load
 * this library.  The product path (libdreamer.so) never calls it and shares no code with it.
 *
 * Plain C, every sum in float64, no blocking, fusion or reordering beyond the definitions.
 * Inputs are float32 arrays (bf16 and fp32 values are exact in float32); all arithmetic and
 * all outputs are float64.
 *
 * Sources (web pages about arXiv 2601.21582, "Depth-Recurrent Attention Mixtures"):
 *   [notes]  papernotes.org notes "Depth-Recurrent Attention Mixtures: Giving Latent
 *            Reasoning the Attention it Deserves": section "Overall framework" (flowchart),
 *            "Key design 1" (depth attention, residual equation y = x_l + DA(x_:l) + SA(x_l)),
 *            "Key design 2" (expert attention, sigma(x) = norm(TopK(sigmoid(x), x + b, k)),
 *            bias update), "Key design 3" (linear-MoE projections, shared-expert identity).
 *   [gist]   gist.science technical summary, section "Methodology" (DA treats the sequence
 *            as batch and depth as sequence; depth RoPE with a reversed half; top-k routing
 *            with a balancing bias; shared expert scaled by the max score).
 *
 * Readings where the pages leave a step open are listed next to each function.
 */
#ifndef DREAMER_ORACLE_H
#define DREAMER_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int B, S;        /* sequences, tokens per sequence (prefill)                       */
  int h, H, d;     /* hidden = H * d                                                  */
  int L;           /* depths                                                          */
  int E, k, m, dr; /* experts, top-k, expert hidden, router key dim                    */
  int P;           /* projection experts (0 = dense QKV/O)                            */
  double rope_base, eps;
  int variant;     /* block layout: 0 DA||SA then EA; 1 serial DA->SA->EA; 2 all parallel;
                      3 no depth attention (the DR-without-DA comparison arm) */
  int route_bf16;  /* 1: routing decisions read their input rounded to bf16, the precision
                      the bf16 kernels store it in (the decision itself stays float64)     */
  int da_window;   /* 0: DA over depths 0..l; W > 0: over the last W depths max(0,l-W+1)..l
                      (sliding-window depth attention)                                   */
} orc_cfg;

typedef struct {
  const float *g;        /* [h]                                   */
  const float *w_qkv;    /* [max(P,1)][h][6h]  x @ W convention    */
  const float *w_qkv_sh; /* [h][6h] (P > 0)                       */
  const float *w_o;      /* [max(P,1)][2h][h]                     */
  const float *w_o_sh;   /* [2h][h] (P > 0)                       */
  const float *w_qP;     /* [h][dr] (P > 0)                       */
  const float *k_P;      /* [P][dr] (P > 0)                       */
  const float *w_qE;     /* [h][dr]                               */
  const float *k_E;      /* [E][dr]                               */
  const float *bias;     /* [E]                                   */
  const float *w1;       /* [E][h][m]                             */
  const float *w2;       /* [E][m][h]                             */
} orc_weights;

/* Optional per-depth outputs; any pointer may be NULL.  Depth-major: [L][T][...]. */
typedef struct {
  double *xhat;     /* [L][T][h]  normalised residual stream            */
  double *y;        /* [L][T][h]  x^ + DA + SA (input of EA)             */
  int32_t *idx;     /* [L][T][k]  selected experts, in selection order   */
  double *w;        /* [L][T][k]  routing weights                        */
  double *margin;   /* [L][T]     (z+b) of k-th pick minus best unpicked */
  double *zsel;     /* [L][T][k+1] biased scores of the k picks and the best unpicked */
  int32_t *counts;  /* [L][E]     selections per expert (added to)       */
  double *sa_k;     /* [L][T][h]  post-RoPE SA keys                      */
  double *sa_v;     /* [L][T][h]  SA values                              */
  int32_t *pidx;    /* [L][T]     projection expert p*                    */
  double *psig;     /* [L][T]     projection weight sigma                 */
  double *pmargin;  /* [L][T]     z_P[p*] minus the runner-up            */
} orc_trace;

void orc_set_threads(int n);

/* Prefill forward over depths [l0, l1) for all B*S tokens.
 * x_in:  [T][h] residual stream at depth l0 (x_0 when l0 = 0).
 * da_kv: [T][L][2][h] depth KV buffer: depths < l0 are read, depths l0..l1-1 are written
 *        (float64, caller-owned).
 * x_out: [T][h] residual stream at depth l1.                                           */
int orc_forward(const orc_cfg *c, const orc_weights *W, const float *x_in, int l0, int l1,
                double *da_kv, double *x_out, orc_trace *tr);

/* Same block, DA computed by explicit per-token, per-head, per-depth loops instead of the
 * reshape-to-batch form; used by the reshape-equivalence pin.                         */
int orc_forward_da_loops(const orc_cfg *c, const orc_weights *W, const float *x_in, int l0,
                         int l1, double *da_kv, double *x_out, orc_trace *tr);

/* One depth l for selected tokens of one sequence (sampled checks at full size).
 * x_seq:   [n_ctx][h] residual stream at depth l of tokens 0..n_ctx-1 of the sequence.
 * da_hist: [n_s][L][2][h] depth KV of the selected tokens (depths < l read).
 * pos:     [n_s] token positions (< n_ctx).
 * Outputs per selected token: x_out [n_s][h]; trace arrays indexed [n_s] (depth slot 0). */
int orc_step_tokens(const orc_cfg *c, const orc_weights *W, int l, const float *x_seq,
                    int n_ctx, const double *da_hist, const int32_t *pos, int n_s,
                    double *x_out, orc_trace *tr);

/* Decode: one new token of ONE sequence through all L depths.
 * kc, vc: [L][H][cap][d] this sequence's SA caches (float64, updated in place at slot len).
 * x_new:  [h].  x_out: [h].  Trace arrays indexed [L][1][...].                         */
int orc_decode_seq(const orc_cfg *c, const orc_weights *W, const float *x_new, double *kc,
                   double *vc, int cap, int len, double *x_out, orc_trace *tr);

/* EA router alone on given states: y [T][h] at depth l -> idx [T][k], w [T][k],
 * margin [T], zsel [T][k+1] (may be NULL), counts [E] (added to).                     */
int orc_route(const orc_cfg *c, const orc_weights *W, int l, const float *y, int T,
              int32_t *idx, double *w, double *margin, double *zsel, int32_t *counts);

/* Projection router alone on given states (R12): x^ [T][h] at depth l -> p* [T],
 * sigma [T], margin [T] (z_P of p* minus the runner-up; may be NULL).  P > 0 only.    */
int orc_proj_route(const orc_cfg *c, const orc_weights *W, int l, const float *xh, int T,
                   int32_t *pstar, double *sigma, double *pmargin);

/* Building blocks exposed for the pins. */
void orc_rmsnorm(int h, const double *x, const float *g, double eps, double *out);
void orc_rope(double *v, int n, double pos, double base);
void orc_depth_rope(double *v, int n, int l, int L, double base);
void orc_attend(const double *q, const double *K, const double *V, int nk, int d,
                long ldk, double *out, double *probs);
void orc_topk(const double *z, const float *bias, int E, int k, int32_t *idx, double *w,
              double *margin);
void orc_linear_moe(int in, int out, const double *x, const float *Wp, const float *Wsh,
                    double sigma, double *y);
void orc_linear_moe_absorbed(int in, int out, const double *x, const float *Wp,
                             const float *Wsh, double sigma, double *y);
void orc_expert(int h, int m, const double *y, const float *w1e, const float *w2e,
                double *out);
/* bias balance update: b <- b + lambda * sign(median(N) - N), N_e = sum_l counts[l][e]. */
void orc_bias_update(int L, int E, const int32_t *counts, double lambda, double *bias);

#ifdef __cplusplus
}
#endif
#endif
