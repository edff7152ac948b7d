/*
 * libdreamer — B200 (sm_100a) forward pass of Dreamer's single depth-recurrent layer.
 *
 * Method (web pages about arXiv 2601.21582, "Depth-Recurrent Attention Mixtures: Giving
 * Latent Reasoning the Attention it Deserves"; [notes] = papernotes.org notes, [gist] =
 * gist.science technical summary):
 *   one shared layer is applied for depths l = 0 .. L-1 ([notes] "Overall framework",
 *   flowchart).  Each depth:
 *     x^_l   = RMSNorm(x_l)                                      ([notes] flowchart)
 *     y_l    = x^_l + DA(x^_0..l) + SA(x^_l)                     ([notes] "Key design 1")
 *     x_l+1  = y_l + sum_{e in TopK} w_e FFN_e(y_l)               ([notes] "Key design 2")
 *   with DA attending over the token's own depth states under a depth RoPE whose second
 *   half is reversed, SA causal over tokens, expert selection
 *   sigma(x) = norm(TopK(sigmoid(x), x + b, k)) against depth-RoPE'd expert keys, and
 *   (optionally) top-1 linear-MoE QKV/O projections whose shared expert is absorbed into
 *   each routed expert ([notes] "Key design 3": sigma x W + max(sigma^) x W_shared =
 *   sigma x (W + W_shared)).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated, row-major, densely packed,
 *     16-byte aligned, of the element type given by dreamer_config.dtype ("dtype" below:
 *     0 = float32, 1 = bfloat16).  Routing weights, biases and counts have fixed types.
 *   - Weight matrices use the x @ W convention: W[in][out].
 *   - The caller owns every buffer it passes; the library never frees them.
 *   - Calls are asynchronous on the given stream (0 = legacy default stream) and return
 *     DREAMER_OK or a negative code.  A device-side error (a bounded wait that expired)
 *     is reported by the next call on the handle and by dreamer_route_counts(on_host=1),
 *     which synchronises.
 *   - One handle per stream: calls on one handle must not overlap.
 */
#ifndef DREAMER_H
#define DREAMER_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DREAMER_OK 0
#define DREAMER_ERR_ARG (-1)         /* null/misaligned pointer, inconsistent config     */
#define DREAMER_ERR_UNSUPPORTED (-2) /* shape outside what the kernels implement         */
#define DREAMER_ERR_CUDA (-3)        /* a CUDA runtime call failed                        */
#define DREAMER_ERR_OOM (-4)         /* device allocation failed                          */
#define DREAMER_ERR_TIMEOUT (-5)     /* a kernel's bounded wait expired                   */
#define DREAMER_ERR_STATE (-6)       /* call not valid for this handle's configuration   */

typedef struct dreamer_handle dreamer_handle;
typedef void *dreamer_stream; /* a cudaStream_t */

typedef struct {
  int batch;          /* b: sequences (prefill) or decode sequences                       */
  int seq;            /* s: tokens per sequence for core_forward (1 for decode-only)       */
  int hidden;         /* h = n_heads * head_dim                                           */
  int n_heads;        /* H                                                                */
  int head_dim;       /* d, multiple of 16                                                */
  int depth;          /* L: number of depth steps (unrolled applications of the layer)    */
  int n_experts;      /* E: expert-attention experts                                      */
  int top_k;          /* k <= E, k <= 16                                                  */
  int expert_hidden;  /* m: expert FFN hidden size, multiple of 16                        */
  int router_dim;     /* d_r: expert/projection router key dim, multiple of 16            */
  int n_proj_experts; /* P: 0 = dense QKV/O; else top-1 linear-MoE QKV/O with P experts   */
  int dtype;          /* 0 = float32, 1 = bfloat16 (weights, activations, caches)         */
  float rope_base;    /* 10000                                                            */
  float rms_eps;      /* 1e-6                                                             */
  int max_cache_len;  /* decode: SA cache capacity per sequence (0 = no decode)           */
  int variant;        /* block layout ([notes] ablation table): 0 DA||SA then EA (default),
                         1 serial DA->SA->EA, 2 fully parallel DA+SA+EA, 3 without depth
                         attention (the pages' DR-without-DA comparison arm: y = x^ + SA)  */
  int da_window;      /* 0: DA at depth l over depths 0..l; W > 0: over the last W depths
                         max(0, l-W+1)..l (sliding-window depth attention)                */
} dreamer_config;

typedef struct {
  const void *rms_gain;     /* [h]                                                          */
  const void *w_qkv;        /* [max(P,1)][h][6h]: columns qSA|kSA|vSA|qDA|kDA|vDA, each
                               h wide and head-major (head j at columns j*d .. j*d+d-1)      */
  const void *w_qkv_shared; /* [h][6h] shared expert, P > 0 only (NULL otherwise)           */
  const void *w_o;          /* [max(P,1)][2h][h]: rows 0..h-1 take a_SA, rows h..2h-1 a_DA   */
  const void *w_o_shared;   /* [2h][h], P > 0 only                                          */
  const void *w_qP;         /* [h][d_r] projection-router query, P > 0 only                 */
  const void *k_P;          /* [P][d_r] projection-expert keys, P > 0 only                  */
  const void *w_qE;         /* [h][d_r] expert-router query                                 */
  const void *k_E;          /* [E][d_r] expert keys (depth RoPE applied per depth inside)   */
  const float *bias_E;      /* [E] float32 selection bias b                                 */
  const void *w1;           /* [E][h][m] expert up-projections                              */
  const void *w2;           /* [E][m][h] expert down-projections                            */
} dreamer_weights;

/* Optional per-depth dumps for checking and analysis; any member may be NULL.
 * Layout [L][T][...] with T = batch*seq (forward) or batch (decode); only the depths a
 * call runs are written.                                                                  */
typedef struct {
  void *xhat;      /* [L][T][h] dtype: RMSNorm output                                      */
  void *y;         /* [L][T][h] dtype: y_l = x^_l + DA + SA, the state entering expert
                      attention (the fully parallel layout routes x^_l instead)             */
  int32_t *idx;    /* [L][T][k]: selected experts                                          */
  float *w;        /* [L][T][k]: routing weights                                           */
  void *sa_k;      /* [L][T][h] dtype: post-RoPE SA keys (forward only)                    */
  void *sa_v;      /* [L][T][h] dtype: SA values (forward only)                            */
  int32_t *pidx;   /* [L][T]: projection expert p* (P > 0)                                 */
  float *psig;     /* [L][T]: projection weight sigma (P > 0)                              */
  float *y_f32;    /* [L][T][h] float32: y_l as the residual stream carries it, before its
                      rounding to dtype (in bf16 mode `y` above is this value rounded)     */
  float *x_f32;    /* [L][T][h] float32: x_{l+1} = y_l + expert attention, before rounding
                      (the last depth's x_out is this value rounded to dtype)              */
} dreamer_trace;

/* Shapes the bfloat16 path takes (every contraction and attention on the tcgen05 tensor
 * cores or in the purpose-built streaming kernels; there is no CUDA-core fallback):
 * head_dim 64 or 128, hidden a multiple of 256 and at most 2048 where rows are few per expert
 * (decode), n_heads <= 32, expert_hidden 16, 32 or 64, router_dim 64 or 128, n_experts a
 * multiple of 4; dreamer_core_forward also needs seq a multiple of 128.  dreamer_init returns
 * DREAMER_ERR_UNSUPPORTED for any other bf16 shape (dreamer_core_forward on a handle whose seq
 * is not a multiple of 128 returns it too).  float32 mode runs every shape on CUDA cores.  */

/* Create a handle: validates the configuration, copies the weights (device pointers) into
 * handle-owned buffers in the kernels' layouts, absorbs the shared projection expert into
 * every routed one (W~_p = round(W_p + W_shared), [notes] "Key design 3"), precomputes the
 * RoPE tables and allocates the workspace for batch*seq tokens.  Synchronises `stream`.
 * Returns DREAMER_ERR_ARG / _UNSUPPORTED / _OOM / _CUDA on failure (*out = NULL).         */
int dreamer_init(const dreamer_config *cfg, const dreamer_weights *weights,
                 dreamer_stream stream, dreamer_handle **out);

/* Prefill forward over depths [depth_begin, depth_end) for all batch*seq tokens
 * ([notes] "Overall framework" flowchart; "Key design 1" residual equation).
 *   x_in   [T][h] dtype: residual stream x at depth_begin (x_0 when depth_begin = 0).
 *   x_out  [T][h] dtype: residual stream at depth_end (no final norm).
 *   da_kv  [T][L][2][h] dtype or NULL.  The depth KV buffer: slot [t][j][0] holds the
 *          post-depth-RoPE DA key of token t at depth j, [t][j][1] its value.  Depths below
 *          depth_begin are read, depths depth_begin .. depth_end-1 are written.  NULL uses
 *          a handle-owned buffer and then requires depth_begin == 0.
 *   trace  NULL or dump pointers.
 * Route counts of the run depths are kept in the handle (zeroed at the start of the call).
 * x_in and x_out may alias.                                                               */
int dreamer_core_forward(dreamer_handle *h, const void *x_in, void *x_out, int depth_begin,
                         int depth_end, void *da_kv, const dreamer_trace *trace,
                         dreamer_stream stream);

/* One decode step: one new token for each of the `batch` sequences through all L depths
 * ([notes] "Overall framework": the SA KV cache persists across tokens while the DA KV
 * cache is overwritten for the next token).
 *   x_new   [B][h] dtype: the new tokens' embeddings.
 *   k_cache, v_cache [L][B][H][max_cache_len][d] dtype: per-depth SA caches holding
 *           post-RoPE keys and values of past tokens.  Slot cache_len[b] of every depth is
 *           written with the new token's key/value; the call attends over cache_len[b]+1
 *           keys.  The caller advances cache_len afterwards.
 *   cache_len [B] int32, device: past tokens per sequence (< max_cache_len).
 *   x_out   [B][h] dtype.                                                                 */
int dreamer_decode_step(dreamer_handle *h, const void *x_new, void *k_cache, void *v_cache,
                        const int32_t *cache_len, void *x_out, const dreamer_trace *trace,
                        dreamer_stream stream);

/* Route counts N[l][e] of the last forward/decode call ([notes] "Key design 2": the usage
 * counts the bias update balances).  counts: [L][E] int32, device pointer (on_host = 0) or
 * host pointer (on_host = 1; the call then synchronises `stream` and also reports any
 * device-side error).  Depths the call did not run hold 0.                                 */
int dreamer_route_counts(dreamer_handle *h, int32_t *counts, int on_host,
                         dreamer_stream stream);

/* Expert routing alone on given states ([notes] "Key design 2", routing equation):
 * z_e = (y W_qE) . (depth-RoPE_l k_e) / sqrt(d_r); pick the k experts with the largest
 * z_e + b_e (ties to the lower index); w_e = sigmoid(z_e) / sum over picks.
 *   y [n_tokens][h] dtype; idx [n_tokens][k] int32; w [n_tokens][k] float32;
 *   counts [E] int32 (overwritten with this call's histogram) or NULL.
 * n_tokens <= batch*seq (or batch for a decode-only handle).                              */
int dreamer_route_experts(dreamer_handle *h, int depth, const void *y, int n_tokens,
                          int32_t *idx, float *w, int32_t *counts, dreamer_stream stream);

/* Expert routing that allocates no device memory and needs no handle.  The pages have no
 * counterpart of this entry point: it exists for callers that cannot call cudaMalloc where
 * they route — a host application that gives all device memory to its own pool and allows no
 * outside allocation, a real-time loop where an allocation (which can synchronise the
 * device) is not acceptable, a plugin that only receives buffers from its host.
 * Computes the same routing as dreamer_route_experts, on CUDA cores.
 *   cfg      hidden, depth (L), n_experts (E), top_k (k <= 16), router_dim (d_r = 32, 64 or
 *            128), dtype and rope_base are read; other fields are ignored.
 *   y        [n_tokens][h] dtype, w_qE [h][d_r] dtype, k_E [E][d_r] dtype (unrotated),
 *            bias_E [E] float32: inputs, device pointers, caller-owned.
 *   idx      [n_tokens][k] int32, w [n_tokens][k] float32: outputs.  counts [E] int32 or
 *            NULL: cleared, then the histogram of idx.
 * Scratch: a fixed array of 4 MiB (1,048,576 floats) inside the library holds the expert keys
 * turned by the depth RoPE of `depth`; E * d_r above 1,048,576 returns
 * DREAMER_ERR_UNSUPPORTED before anything runs.  Every GPU that loads the library keeps the
 * array until the process exits.  All calls share it and it keeps the last call's contents,
 * so calls that overlap on the GPU (other streams, other host threads) race: serialise them.
 * The first call on a device looks up the array's device address and caches it (per device
 * and CUDA context: a new context, e.g. after cudaDeviceReset, looks it up again); make that
 * first call before any stream capture on the device.  Routing weights are formed in a form
 * that stays finite when every pick's sigmoid underflows.                                  */
int dreamer_route_experts_noalloc(const dreamer_config *cfg, int depth, const void *y,
                                  int n_tokens, const void *w_qE, const void *k_E,
                                  const float *bias_E, int32_t *idx, float *w,
                                  int32_t *counts, dreamer_stream stream);

/* Bias balance update from the handle's last route counts ([notes] "Key design 2"):
 * b_e <- b_e + lambda * sign(median(N) - N_e), N_e = sum over depths, lower median for an
 * even E.  Updates the handle's bias; if bias_out is not NULL also copies the new bias
 * ([E] float32, device) there.                                                            */
int dreamer_bias_update(dreamer_handle *h, float lambda, float *bias_out,
                        dreamer_stream stream);

/* The same update from caller-given counts: counts [n_rows][E] int32, device pointer (read
 * only), N_e = sum over the rows.  With data-parallel replicas (one handle per GPU, each
 * routing its own batch) the counts are the [L][E] output of dreamer_route_counts summed over
 * the replicas by one all-reduce, so every replica applies the same update to its bias.
 * DREAMER_ERR_ARG for a NULL handle or counts or n_rows < 1.                              */
int dreamer_bias_update_counts(dreamer_handle *h, float lambda, const int32_t *counts,
                               int n_rows, float *bias_out, dreamer_stream stream);

/* Balance summary of the expert route counts N of the last call ([notes] "Key design 2":
 * the bias keeps expert use balanced; this measures how balanced): N_e = counts of depth
 * `depth`, or summed over depths for depth < 0.  Writes the Lorenz curve of N (sorted
 * ascending, cumulative share at e/E for e = 0..E; [E+1] float32, device, may be NULL) and
 * the Gini coefficient G = 1 - (1/E) sum_e (L_{e-1} + L_e) ([1] float32, device).  E up to
 * 8192 (DREAMER_ERR_UNSUPPORTED beyond).  Asynchronous on `stream`.                        */
int dreamer_route_balance(dreamer_handle *h, int depth, float *lorenz, float *gini,
                          dreamer_stream stream);

/* Instrumentation.  Stages of the depth step, in launch order: */
enum {
  DREAMER_STAGE_NORM = 0,     /* RMSNorm of the residual stream                          */
  DREAMER_STAGE_PROJ_ROUTE,   /* projection router + grouping (linear-MoE QKV/O)         */
  DREAMER_STAGE_QKV,          /* fused QKV projection, RoPE / depth RoPE, DA KV write    */
  DREAMER_STAGE_DA,           /* depth attention                                         */
  DREAMER_STAGE_SA,           /* causal sequence attention (prefill) / cache attention   */
  DREAMER_STAGE_O,            /* O projection + residual                                 */
  DREAMER_STAGE_EA_ROUTE,     /* expert router: query, scores, top-k, counts             */
  DREAMER_STAGE_PERMUTE,      /* counting sort of routed slots by expert                 */
  DREAMER_STAGE_EXPERTS,      /* expert FFNs with weighted scatter-add                   */
  DREAMER_STAGE_FINISH,       /* final residual store and call overhead                  */
  DREAMER_N_STAGES
};
typedef struct {
  uint64_t launches;                 /* kernels launched by the library since the reset    */
  double ms[DREAMER_N_STAGES];       /* device time per stage (profiling enabled only)     */
  uint64_t count[DREAMER_N_STAGES];  /* timed stage executions                             */
  uint64_t launches_tc;              /* of `launches`: tcgen05 kernels (GEMM engine, flash
                                        SA, fused expert FFN)                              */
  uint64_t launches_simt;            /* of `launches`: the generic CUDA-core GEMM, attention
                                        and top-k kernels of float32 mode (0 in bf16 mode)   */
} dreamer_stats;

/* Enable (1) or disable (0) per-stage CUDA-event timing on the streams of later calls.
 * Timing adds one event record per stage boundary; it is meant for measurement runs.     */
int dreamer_set_profiling(dreamer_handle *h, int enable);

/* Read the launch counter and the per-stage times accumulated since the last reset
 * (synchronises the device when profiling is on); reset = 1 clears them afterwards.      */
int dreamer_get_stats(dreamer_handle *h, dreamer_stats *out, int reset);

/* Free the handle and everything it owns (synchronises the device).                      */
void dreamer_destroy(dreamer_handle *h);

/* Static description of an error code.                                                    */
const char *dreamer_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* DREAMER_H */
