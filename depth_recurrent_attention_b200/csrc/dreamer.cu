// libdreamer: C ABI of the Dreamer depth-recurrent core forward on B200 (sm_100a).
// The depth step (papernotes.org notes on "Depth-Recurrent Attention Mixtures", section
// "Overall framework", flowchart): RMSNorm -> [DA || SA] -> residual -> EA -> next depth.
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <utility>
#include <vector>

#include "../../include/dreamer.h"
#include "common.cuh"
#include "kernels_simt.cuh"
#include "attn_rows.cuh"

using namespace dreamer;

struct dreamer_handle {
  dreamer_config cfg;
  int T;        // token capacity of the workspace
  int esz;      // element size
  int max_pos;  // RoPE table rows
  int ldz;      // router score row stride (E rounded up to 8)
  int ldzp;     // projection router score row stride
  // weights in kernel layouts ([N][K], K contiguous)
  void *g = nullptr, *wqkv_t = nullptr, *wo_t = nullptr, *wqE_t = nullptr, *wqP_t = nullptr;
  void *w1_t = nullptr, *w2_t = nullptr;
  void *kE_raw = nullptr;        // [E][dr] dtype (unrotated)
  float *bias = nullptr;         // [E]
  float *kE_rot = nullptr;       // [L][E][dr]
  float *kP_rot = nullptr;       // [L][P][dr]
  float2 *rope_tok = nullptr;    // [max_pos][d/2]
  float2 *rope_dep = nullptr;    // [L][d/2]
  float2 *rope_dr = nullptr;     // [L][dr/2] depth RoPE table of the router key dim
  // workspace
  void *xh = nullptr, *qkv_sa = nullptr, *q_da = nullptr, *attn = nullptr, *y = nullptr;
  void *u = nullptr, *da_kv_int = nullptr, *Hbuf = nullptr, *qsplit = nullptr;
  void *xh_sorted = nullptr;     // x^ in the projection experts' group order (P > 0)
  float *acc = nullptr, *zbuf = nullptr, *qbuf = nullptr, *psig = nullptr, *ew = nullptr;
  float *inv_rms = nullptr;      // [T] 1/rms of the current depth's residual
  float *part = nullptr;         // decode attention split partials [B][H][nsplit][d + 2]
  int nsplit = 1;
  int *pidx = nullptr, *eidx = nullptr, *counts = nullptr, *ecnt = nullptr, *eoffs = nullptr;
  int *etiles_a = nullptr, *etiles_b = nullptr, *ecursor = nullptr, *erows = nullptr;
  int *einv = nullptr;           // [T k] sorted position of each routed slot
  int2 *etab = nullptr;          // 128-row tiles of the expert groups (written by the sort)
  int2 *ptab = nullptr;          // 128-row tiles of the projection groups
  void *Ybuf = nullptr;          // [T k + 128][h] expert outputs in sorted order
  int *pcnt = nullptr, *poffs = nullptr, *ptiles_a = nullptr, *ptiles_b = nullptr;
  int *pcursor = nullptr, *prows = nullptr, *pinv = nullptr;
  int *err = nullptr;
  void *k3 = nullptr;            // [E][3 d_r] bf16: router keys repeated for split scores
  void *kEt = nullptr;           // [d_r][E] bf16: router keys transposed (CUDA-core scores)
  int num_sms = 148;
  int prio_hi = 0;   // the device's most urgent launch priority (depth attention beside SA)
  int qkv_perm = 0;  // q_SA / k_SA columns of the fused QKV weight in EpiQKV perm order
  int prefill_ok = 1;  // bf16: the prefill shapes are ones the tcgen05 kernels take
#ifdef DREAMER_TEST_HOOKS
  int inject_skip = 0;  // the next QKV GEMM's TMA producer issues no loads (timeout test)
#endif
  int path_err = 0;    // a bf16 step found no kernel for its shape while enqueuing (a bug)
  std::vector<void *> allocs;
  int *err_host = nullptr;       // pinned copy of the device error flag (async)
  cudaStream_t side = nullptr;   // second stream: DA runs beside SA
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  cudaStream_t side2 = nullptr;  // third stream: expert attention beside DA/SA/O (layout 2)
  cudaEvent_t ev_fork2 = nullptr, ev_join2 = nullptr;
  int use_graph = 1;
  int use_pdl = 1;               // programmatic dependent launch between kernels of a stream
  bool pdl_ok[3] = {false, false, false};  // main / side / side2: the last operation was a kernel
  struct GraphEntry {
    int kind;                    // 0 forward, 1 decode
    const void *key[5];
    int l0, l1, prof;
    int captured;                // 0: seen once (ran directly), 1: graph ready
    cudaGraphExec_t exec;
    uint64_t launches, launches_tc, launches_simt;
    std::vector<cudaEvent_t> evs;
    std::vector<int> stages;
    uint64_t last_use;
  };
  std::vector<GraphEntry> graphs;
  uint64_t use_clock = 0;
  // instrumentation
  uint64_t launches = 0, launches_tc = 0, launches_simt = 0;
  int prof = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> ev_stage;
  size_t ev_used = 0;
  double stage_ms[DREAMER_N_STAGES] = {0};
  uint64_t stage_count[DREAMER_N_STAGES] = {0};
};

// stage boundary: with profiling on, an event tagged with the stage that starts here
static void mark(dreamer_handle *h, cudaStream_t s, int stage) {
  if (!h->prof) return;
  if (h->ev_used == h->ev.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    h->ev.push_back(e);
    h->ev_stage.push_back(0);
  }
  cudaEventRecord(h->ev[h->ev_used], s);
  h->ev_stage[h->ev_used] = stage;
  h->ev_used++;
}

static void accumulate_marks(dreamer_handle *h, const std::vector<cudaEvent_t> &evs,
                             const std::vector<int> &stages) {
  for (size_t i = 0; i + 1 < evs.size(); i++) {
    const int st = stages[i];
    if (st >= DREAMER_N_STAGES) continue;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, evs[i], evs[i + 1]) == cudaSuccess) {
      h->stage_ms[st] += ms;
      h->stage_count[st] += 1;
    }
  }
}



#define CK(call)                                                  \
  do {                                                            \
    cudaError_t e_ = (call);                                      \
    if (e_ != cudaSuccess) {                                      \
      fprintf(stderr, "libdreamer: %s failed: %s\n", #call,      \
              cudaGetErrorString(e_));                            \
      return e_ == cudaErrorMemoryAllocation ? DREAMER_ERR_OOM    \
                                             : DREAMER_ERR_CUDA;  \
    }                                                             \
  } while (0)

static int dalloc(dreamer_handle *h, void **p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    *p = nullptr;
    return e == cudaErrorMemoryAllocation ? DREAMER_ERR_OOM : DREAMER_ERR_CUDA;
  }
  h->allocs.push_back(*p);
  return DREAMER_OK;
}
#define DALLOC(ptr, bytes)                                     \
  do {                                                         \
    int rc_ = dalloc(h, (void **)&(ptr), (size_t)(bytes));     \
    if (rc_ != DREAMER_OK) return rc_;                         \
  } while (0)

static inline int cdiv(long a, long b) { return (int)((a + b - 1) / b); }
// kernels launched by this thread through the library (read as deltas around each call):
// all of them, the tcgen05 ones, and the generic CUDA-core GEMM / attention / top-k kernels
static thread_local uint64_t g_launches = 0;
static thread_local uint64_t g_launches_tc = 0;
static thread_local uint64_t g_launches_simt = 0;

// ---- kernel launches with programmatic dependent launch -------------------------------
// A kernel may start while the previous operation on its stream is still running only if that
// operation is a kernel (whose completion its pdl_wait() then waits for).  pdl_take() answers
// that for the stream and records that a kernel is now last; pdl_break() records any other
// operation (copy, memset, event wait).  Off while stages are timed by events.
static bool pdl_take(dreamer_handle *h, cudaStream_t s) {
  bool &ok = h->pdl_ok[s == h->side ? 1 : (s == h->side2 ? 2 : 0)];
  const bool r = ok && h->use_pdl && !h->prof;
  ok = true;
  return r;
}
static void pdl_break(dreamer_handle *h, cudaStream_t s) {
  h->pdl_ok[s == h->side ? 1 : (s == h->side2 ? 2 : 0)] = false;
}

// launch_kx: with thread-block clusters of `cluster` CTAs along x and, for prio != 0, the
// launch priority prio (lower = more urgent: its CTAs are placed before pending CTAs of
// kernels launched with the default priority)
template <typename... P, typename... A>
static void launch_kx(dreamer_handle *h, int cluster, int prio, void (*kern)(P...), dim3 grid,
                      dim3 block, size_t smem, cudaStream_t s, A &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[3];
  int na = 0;
  if (prio != 0) {
    at[na].id = cudaLaunchAttributePriority;
    at[na].val.priority = prio;
    na++;
  }
  if (pdl_take(h, s)) {
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    na++;
  }
  if (cluster > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = cluster;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    na++;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  ++g_launches;
  cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}
template <typename... P, typename... A>
static void launch_kc(dreamer_handle *h, int cluster, void (*kern)(P...), dim3 grid, dim3 block,
                      size_t smem, cudaStream_t s, A &&...args) {
  launch_kx(h, cluster, 0, kern, grid, block, smem, s, std::forward<A>(args)...);
}
template <typename... P, typename... A>
static void launch_k(dreamer_handle *h, void (*kern)(P...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t s, A &&...args) {
  launch_kc(h, 1, kern, grid, block, smem, s, std::forward<A>(args)...);
}

// top-k: eight warps a token when there are too few tokens to fill the GPU with one warp each
static void launch_topk(dreamer_handle *h, const TopkArgs &t, cudaStream_t s) {
  ++g_launches_simt;
  if ((long)t.n_tok * 4 < (long)h->num_sms * 32)
    launch_k(h, topk_kernel<8>, dim3(t.n_tok), dim3(256), 0, s, t);
  else
    launch_k(h, topk_kernel<1>, dim3((t.n_tok + 7) / 8), dim3(256), 0, s, t);
}

#include "tc_kernels.cuh"

static inline int round8(int v) { return (v + 7) / 8 * 8; }

extern "C" const char *dreamer_strerror(int code) {
  switch (code) {
    case DREAMER_OK: return "ok";
    case DREAMER_ERR_ARG: return "invalid argument";
    case DREAMER_ERR_UNSUPPORTED: return "unsupported configuration";
    case DREAMER_ERR_CUDA: return "CUDA runtime error";
    case DREAMER_ERR_OOM: return "out of device memory";
    case DREAMER_ERR_TIMEOUT: return "device wait timed out";
    case DREAMER_ERR_STATE: return "call not valid for this handle";
    default: return "unknown error";
  }
}

static int validate(const dreamer_config *c) {
  if (!c) return DREAMER_ERR_ARG;
  if (c->batch < 1 || c->seq < 1 || c->depth < 1 || c->n_heads < 1 || c->head_dim < 1)
    return DREAMER_ERR_ARG;
  if (c->hidden != c->n_heads * c->head_dim) return DREAMER_ERR_ARG;
  if (c->top_k < 1 || c->top_k > c->n_experts) return DREAMER_ERR_ARG;
  if (c->dtype != 0 && c->dtype != 1) return DREAMER_ERR_ARG;
  if (c->n_proj_experts < 0 || c->max_cache_len < 0) return DREAMER_ERR_ARG;
  if (c->variant < 0 || c->variant > 3 || c->da_window < 0) return DREAMER_ERR_ARG;
  if (!(c->rope_base > 0.f) || !(c->rms_eps >= 0.f)) return DREAMER_ERR_ARG;
  const int d = c->head_dim;
  if (d != 16 && d != 32 && d != 64 && d != 128) return DREAMER_ERR_UNSUPPORTED;
  if (c->top_k > 16 || c->n_experts > 65536 || c->n_proj_experts > 64) return DREAMER_ERR_UNSUPPORTED;
  if (c->expert_hidden % 16 || c->router_dim % 16 || c->router_dim > 256 || c->hidden % 64)
    return DREAMER_ERR_UNSUPPORTED;
  if (c->depth > 1024 || c->hidden > 4096) return DREAMER_ERR_UNSUPPORTED;
  // routed rows (tokens x k) are indexed with 24 bits in the grouping tables
  if ((long)c->batch * c->seq * c->top_k >= (1L << 24)) return DREAMER_ERR_UNSUPPORTED;
  if (c->dtype == 1) {
    // bf16 runs only on the tcgen05 kernels and the purpose-built streaming kernels: shapes
    // they do not take are refused here instead of being routed to CUDA-core fallbacks
    if (d != 64 && d != 128) return DREAMER_ERR_UNSUPPORTED;             // GEMM / flash SA
    if (c->hidden % 256 || c->n_heads > 32) return DREAMER_ERR_UNSUPPORTED;  // N tiles; DA CTA
    const int m = c->expert_hidden;
    if (m != 16 && m != 32 && m != 64) return DREAMER_ERR_UNSUPPORTED;     // expert FFN
    if (c->router_dim != 64 && c->router_dim != 128) return DREAMER_ERR_UNSUPPORTED;
    if (c->n_experts % 4) return DREAMER_ERR_UNSUPPORTED;                  // router scorer
  }
  return DREAMER_OK;
}

// ---------------------------------------------------------------------------------------
// host-side tables
// RoPE rotate-half tables in double, stored as float2 (cos, sin).
static void rope_table(std::vector<float2> &t, int rows, int n, double base) {
  // rows positions x n/2 pairs, angle pos * base^(-2i/n)
  t.resize((size_t)rows * (n / 2));
  for (int p = 0; p < rows; p++)
    for (int i = 0; i < n / 2; i++) {
      double th = (double)p * pow(base, -2.0 * i / (double)n);
      t[(size_t)p * (n / 2) + i] = make_float2((float)cos(th), (float)sin(th));
    }
}
// depth table [L][n/2]: first n/4 entries at position l over n/2 dims, next n/4 at L-1-l.
static void depth_table(std::vector<float2> &t, int L, int n, double base) {
  t.resize((size_t)L * (n / 2));
  const int q = n / 4;
  for (int l = 0; l < L; l++)
    for (int half = 0; half < 2; half++)
      for (int i = 0; i < q; i++) {
        double pos = half == 0 ? l : (L - 1 - l);
        double th = pos * pow(base, -2.0 * i / (double)(n / 2));
        t[(size_t)l * (n / 2) + half * q + i] = make_float2((float)cos(th), (float)sin(th));
      }
}

static float host_to_f(const void *p, size_t i, int dtype) {
  if (dtype == 0) return ((const float *)p)[i];
  uint16_t b = ((const uint16_t *)p)[i];
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// keys [n][dr] (dtype, device) -> rotated fp32 [L][n][dr] by the depth RoPE of each depth.
static int rotated_keys(dreamer_handle *h, const void *keys_dev, int n, float **out) {
  const dreamer_config &c = h->cfg;
  const int dr = c.router_dim, L = c.depth;
  std::vector<uint8_t> raw((size_t)n * dr * h->esz);
  CK(cudaMemcpy(raw.data(), keys_dev, raw.size(), cudaMemcpyDeviceToHost));
  std::vector<float> rot((size_t)L * n * dr);
  const int half = dr / 2, q = dr / 4;
  for (int l = 0; l < L; l++)
    for (int e = 0; e < n; e++) {
      std::vector<double> v(dr);
      for (int i = 0; i < dr; i++) v[i] = host_to_f(raw.data(), (size_t)e * dr + i, c.dtype);
      for (int hh = 0; hh < 2; hh++) {
        double pos = hh == 0 ? l : (L - 1 - l);
        for (int i = 0; i < q; i++) {
          double th = pos * pow((double)c.rope_base, -2.0 * i / (double)half);
          double cs = cos(th), sn = sin(th);
          double a = v[hh * half + i], b = v[hh * half + i + q];
          v[hh * half + i] = a * cs - b * sn;
          v[hh * half + i + q] = b * cs + a * sn;
        }
      }
      for (int i = 0; i < dr; i++) rot[((size_t)l * n + e) * dr + i] = (float)v[i];
    }
  DALLOC(*out, rot.size() * sizeof(float));
  CK(cudaMemcpy(*out, rot.data(), rot.size() * sizeof(float), cudaMemcpyHostToDevice));
  return DREAMER_OK;
}

template <typename T>
static void launch_transpose(const void *src, const void *sh, void *dst, int rows, int cols,
                             int G, cudaStream_t s) {
  dim3 grid(cdiv(cols, 32), cdiv(rows, 32), G), block(32, 8);
  ++g_launches;
  transpose_absorb_kernel<T><<<grid, block, 0, s>>>((const T *)src, (const T *)sh, (T *)dst,
                                                     rows, cols, G);
}

extern "C" int dreamer_init(const dreamer_config *cfg, const dreamer_weights *w,
                            dreamer_stream stream, dreamer_handle **out) {
  if (!out) return DREAMER_ERR_ARG;
  *out = nullptr;
  int rc = validate(cfg);
  if (rc) return rc;
  if (!w || !w->rms_gain || !w->w_qkv || !w->w_o || !w->w_qE || !w->k_E || !w->bias_E ||
      !w->w1 || !w->w2)
    return DREAMER_ERR_ARG;
  if (cfg->n_proj_experts > 0 &&
      (!w->w_qkv_shared || !w->w_o_shared || !w->w_qP || !w->k_P))
    return DREAMER_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  dreamer_handle *h = new dreamer_handle();
  h->cfg = *cfg;
  rc = [&]() -> int {
    const dreamer_config &c = h->cfg;
    const int hd = c.hidden, E = c.n_experts, m = c.expert_hidden, dr = c.router_dim;
    const int P = c.n_proj_experts, G = P > 0 ? P : 1, L = c.depth, d = c.head_dim;
    h->esz = c.dtype == 0 ? 4 : 2;
    h->prefill_ok = c.dtype == 0 || c.seq % 128 == 0;  // bf16 flash SA: 128-token query tiles
    h->T = c.batch * c.seq > c.batch ? c.batch * c.seq : c.batch;
    h->max_pos = c.seq > c.max_cache_len ? c.seq : c.max_cache_len;
    h->ldz = round8(E);
    h->ldzp = round8(P > 0 ? P : 1);
    const size_t es = h->esz;
    const long T = h->T;
    {
      int dev = 0, sms = 0;
      if (cudaGetDevice(&dev) == cudaSuccess &&
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
        h->num_sms = sms;
    }
    if (const char *ev = getenv("DREAMER_NO_GRAPH")) h->use_graph = atoi(ev) ? 0 : 1;
    if (const char *ev = getenv("DREAMER_NO_PDL")) h->use_pdl = atoi(ev) ? 0 : 1;
    {
      int least = 0, greatest = 0;
      if (cudaDeviceGetStreamPriorityRange(&least, &greatest) == cudaSuccess) h->prio_hi = greatest;
    }
    CK(cudaHostAlloc((void **)&h->err_host, sizeof(int), cudaHostAllocDefault));
    *h->err_host = 0;
    CK(cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
    CK(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
    CK(cudaStreamCreateWithFlags(&h->side2, cudaStreamNonBlocking));
    CK(cudaEventCreateWithFlags(&h->ev_fork2, cudaEventDisableTiming));
    CK(cudaEventCreateWithFlags(&h->ev_join2, cudaEventDisableTiming));
    // ---- weights
    DALLOC(h->g, hd * es);
    CK(cudaMemcpyAsync(h->g, w->rms_gain, hd * es, cudaMemcpyDeviceToDevice, s));
    DALLOC(h->wqkv_t, (size_t)G * hd * 6 * hd * es);
    DALLOC(h->wo_t, (size_t)G * 2 * hd * hd * es);
    DALLOC(h->wqE_t, (size_t)hd * dr * es);
    DALLOC(h->w1_t, (size_t)E * hd * m * es);
    DALLOC(h->w2_t, (size_t)E * hd * m * es);
    DALLOC(h->kE_raw, (size_t)E * dr * es);
    CK(cudaMemcpyAsync(h->kE_raw, w->k_E, (size_t)E * dr * es, cudaMemcpyDeviceToDevice, s));
    DALLOC(h->bias, E * sizeof(float));
    CK(cudaMemcpyAsync(h->bias, w->bias_E, E * sizeof(float), cudaMemcpyDeviceToDevice, s));
    auto tr = c.dtype == 0 ? launch_transpose<float> : launch_transpose<bf16>;
    // W_qkv [G][h][6h] (+ shared) -> [G][6h][h]; W_o [G][2h][h] -> [G][h][2h]
    tr(w->w_qkv, P > 0 ? w->w_qkv_shared : nullptr, h->wqkv_t, hd, 6 * hd, G, s);
    tr(w->w_o, P > 0 ? w->w_o_shared : nullptr, h->wo_t, 2 * hd, hd, G, s);
    if (c.dtype == 1 && d == 128) {  // RoPE partners 32 columns apart (EpiQKV perm order)
      h->qkv_perm = 1;
      ++g_launches;
      perm_qk_rows_kernel<bf16><<<4 * 148, 256, 0, s>>>((bf16 *)h->wqkv_t, hd, G);
    }
    tr(w->w_qE, nullptr, h->wqE_t, hd, dr, 1, s);
    tr(w->w1, nullptr, h->w1_t, hd, m, E, s);     // [E][h][m] -> [E][m][h]
    tr(w->w2, nullptr, h->w2_t, m, hd, E, s);     // [E][m][h] -> [E][h][m]
    if (P > 0) {
      DALLOC(h->wqP_t, (size_t)hd * dr * es);
      tr(w->w_qP, nullptr, h->wqP_t, hd, dr, 1, s);
    }
    CK(cudaGetLastError());
    CK(cudaStreamSynchronize(s));
    int r2 = rotated_keys(h, w->k_E, E, &h->kE_rot);
    if (r2) return r2;
    if (P > 0) {
      r2 = rotated_keys(h, w->k_P, P, &h->kP_rot);
      if (r2) return r2;
    }
    std::vector<float2> tt, td, tq;
    rope_table(tt, h->max_pos + 1, d, c.rope_base);
    depth_table(td, L, d, c.rope_base);
    depth_table(tq, L, dr, c.rope_base);
    DALLOC(h->rope_tok, tt.size() * sizeof(float2));
    DALLOC(h->rope_dep, td.size() * sizeof(float2));
    DALLOC(h->rope_dr, tq.size() * sizeof(float2));
    CK(cudaMemcpy(h->rope_tok, tt.data(), tt.size() * sizeof(float2), cudaMemcpyHostToDevice));
    CK(cudaMemcpy(h->rope_dep, td.data(), td.size() * sizeof(float2), cudaMemcpyHostToDevice));
    CK(cudaMemcpy(h->rope_dr, tq.data(), tq.size() * sizeof(float2), cudaMemcpyHostToDevice));
    // ---- workspace
    const long Tk = T * c.top_k;
    DALLOC(h->xh, T * hd * es);
    DALLOC(h->u, T * hd * es);
    if (P > 0) DALLOC(h->xh_sorted, T * hd * es);
    DALLOC(h->qkv_sa, T * 3 * hd * es);
    DALLOC(h->q_da, T * hd * es);
    DALLOC(h->attn, T * 2 * hd * es);
    DALLOC(h->y, T * hd * es);
    DALLOC(h->acc, T * hd * sizeof(float));
    DALLOC(h->inv_rms, T * sizeof(float));
    if (c.variant != 3) DALLOC(h->da_kv_int, (size_t)T * L * 2 * hd * es);
    DALLOC(h->Hbuf, (Tk + 128) * m * es);
    DALLOC(h->qsplit, T * 3 * dr * 2);
    DALLOC(h->zbuf, (size_t)T * (h->ldz > h->ldzp ? h->ldz : h->ldzp) * sizeof(float));
    DALLOC(h->qbuf, T * dr * sizeof(float));
    DALLOC(h->psig, T * sizeof(float));
    DALLOC(h->pidx, T * sizeof(int));
    DALLOC(h->ew, Tk * sizeof(float));
    DALLOC(h->eidx, Tk * sizeof(int));
    DALLOC(h->counts, (size_t)L * E * sizeof(int));
    DALLOC(h->ecnt, 2 * E * sizeof(int));  // counts | rank counters, zero between depths
    h->ecursor = h->ecnt + E;
    DALLOC(h->eoffs, (E + 1) * sizeof(int));
    DALLOC(h->etiles_a, (E + 1) * sizeof(int));
    DALLOC(h->etiles_b, (E + 1) * sizeof(int));
    DALLOC(h->erows, Tk * sizeof(int));
    DALLOC(h->einv, Tk * sizeof(int));
    DALLOC(h->etab, (Tk / 128 + E + 2) * sizeof(int2));
    DALLOC(h->ptab, (T / 128 + G + 2) * sizeof(int2));
    DALLOC(h->Ybuf, (size_t)(Tk + 128) * hd * es);
    DALLOC(h->pcnt, 2 * (G + 1) * sizeof(int));  // counts | rank counters
    h->pcursor = h->pcnt + G + 1;
    DALLOC(h->poffs, (G + 1) * sizeof(int));
    DALLOC(h->ptiles_a, (G + 1) * sizeof(int));
    DALLOC(h->ptiles_b, (G + 1) * sizeof(int));
    DALLOC(h->prows, T * sizeof(int));
    DALLOC(h->pinv, T * sizeof(int));
    DALLOC(h->err, sizeof(int));
    if (c.max_cache_len > 0) {
      // key ranges per (sequence, head): about ten waves of three CTAs per SM, at least 16
      // keys a range, at most 64 ranges
      const long pairs = (long)c.batch * c.n_heads;
      long ns = (30L * h->num_sms + pairs - 1) / pairs;
      const long by_len = (c.max_cache_len + 1 + 15) / 16;
      if (ns > by_len) ns = by_len;
      h->nsplit = (int)(ns < 1 ? 1 : ns > 64 ? 64 : ns);
      DALLOC(h->part, (size_t)c.batch * c.n_heads * h->nsplit * (d + 2) * sizeof(float));
    }
    CK(cudaMemset(h->err, 0, sizeof(int)));
    CK(cudaMemset(h->counts, 0, (size_t)L * E * sizeof(int)));
    CK(cudaMemset(h->ecnt, 0, 2 * E * sizeof(int)));
    CK(cudaMemset(h->pcnt, 0, 2 * (G + 1) * sizeof(int)));
    int r3 = tc_init(h);
    if (r3) return r3;
    CK(cudaDeviceSynchronize());
    return DREAMER_OK;
  }();
  if (rc != DREAMER_OK) {
    dreamer_destroy(h);
    return rc;
  }
  *out = h;
  return DREAMER_OK;
}

extern "C" int dreamer_set_profiling(dreamer_handle *h, int enable) {
  if (!h) return DREAMER_ERR_ARG;
  h->prof = enable ? 1 : 0;
  return DREAMER_OK;
}

extern "C" int dreamer_get_stats(dreamer_handle *h, dreamer_stats *out, int reset) {
  if (!h || !out) return DREAMER_ERR_ARG;
  if (h->ev_used > 1) {
    CK(cudaEventSynchronize(h->ev[h->ev_used - 1]));
    std::vector<cudaEvent_t> evs(h->ev.begin(), h->ev.begin() + h->ev_used);
    std::vector<int> st(h->ev_stage.begin(), h->ev_stage.begin() + h->ev_used);
    accumulate_marks(h, evs, st);
  }
  h->ev_used = 0;
  out->launches = h->launches;
  out->launches_tc = h->launches_tc;
  out->launches_simt = h->launches_simt;
  for (int i = 0; i < DREAMER_N_STAGES; i++) {
    out->ms[i] = h->stage_ms[i];
    out->count[i] = h->stage_count[i];
  }
  if (reset) {
    h->launches = 0;
    h->launches_tc = 0;
    h->launches_simt = 0;
    for (int i = 0; i < DREAMER_N_STAGES; i++) {
      h->stage_ms[i] = 0;
      h->stage_count[i] = 0;
    }
  }
  return DREAMER_OK;
}

extern "C" void dreamer_destroy(dreamer_handle *h) {
  if (!h) return;
  cudaDeviceSynchronize();
  tc_destroy(h);
  for (cudaEvent_t e : h->ev) cudaEventDestroy(e);
  for (auto &g : h->graphs) {
    if (g.captured) cudaGraphExecDestroy(g.exec);
    for (cudaEvent_t e : g.evs) cudaEventDestroy(e);
  }
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  if (h->ev_fork2) cudaEventDestroy(h->ev_fork2);
  if (h->ev_join2) cudaEventDestroy(h->ev_join2);
  if (h->side2) cudaStreamDestroy(h->side2);
  if (h->err_host) cudaFreeHost(h->err_host);
  for (void *p : h->allocs) cudaFree(p);
  delete h;
}

// ---------------------------------------------------------------------------------------
// launch helpers
template <typename TA, typename TB, int SEG, class Epi>
static void gemm_simt(const GemmArgs &a, int max_tiles, const Epi &epi, cudaStream_t s) {
  dim3 grid(max_tiles, cdiv(a.N, 128));
  ++g_launches;
  ++g_launches_simt;
  gemm_simt_kernel<TA, TB, SEG, Epi><<<grid, 256, 0, s>>>(a, epi);
}

static GemmArgs dense_args(int M, int N, int K, const void *A, long lda, const void *B,
                           long ldb) {
  GemmArgs a{};
  a.N = N; a.K = K; a.G = 1; a.M = M; a.goffs = nullptr; a.tile_offs = nullptr;
  a.arow = nullptr; a.arow_div = 1; a.A = A; a.lda = lda; a.B = B; a.ldb = ldb; a.bgstride = 0;
  return a;
}

template <typename T>
static void launch_attn(const AttnArgs &a, int d, cudaStream_t s) {
  const int warps = a.n_q * a.H;
  const int blocks = cdiv(warps, 8);
  ++g_launches_simt;
  switch (d) {
    case 16: ++g_launches; attn_warp_kernel<T, 16><<<blocks, 256, 0, s>>>(a); break;
    case 32: ++g_launches; attn_warp_kernel<T, 32><<<blocks, 256, 0, s>>>(a); break;
    case 64: ++g_launches; attn_warp_kernel<T, 64><<<blocks, 256, 0, s>>>(a); break;
    default: ++g_launches; attn_warp_kernel<T, 128><<<blocks, 256, 0, s>>>(a); break;
  }
}

// Depth attention: persistent CTAs, each streaming its tokens' depth runs through shared
// memory.  sms = 0: as many CTAs as are resident at once on the whole GPU (two buffers, two
// CTAs an SM).  sms > 0 (beside SA): sms CTAs that each own an SM (four buffers, at least
// 116 KB of shared memory so that no other CTA fits beside), launched at the most urgent
// priority so that they take their SMs before SA's pending CTAs.
template <typename T>
static void launch_da_bulk(dreamer_handle *h, const RowsArgs &r, int d, cudaStream_t s, int sms) {
  DaBulkArgs a{};
  a.n_tok = r.n_q; a.H = r.H; a.h = r.h; a.L = r.L; a.l = r.l; a.r0 = r.r0;
  const long row_bytes = 2L * r.h * sizeof(T);
  int chunk = (int)((48 * 1024) / row_bytes);
  if (chunk < 1) chunk = 1;
  if (chunk > r.l + 1 - r.r0) chunk = r.l + 1 - r.r0;
  a.chunk = chunk;
  a.q = r.q; a.kv = r.kv; a.out = r.out; a.ldo = r.ldo; a.col0 = r.col0; a.err = r.err;
  a.out_rows = r.out_rows;
  const bool own = sms > 0;
  const int nb = own ? 4 : 2;
  int smem = (int)(nb * (chunk * row_bytes + r.h * (long)sizeof(T)));
  if (own && smem < 116 * 1024) smem = 116 * 1024;
  const int threads = 32 * r.H;
  auto go = [&](void (*kern)(DaBulkArgs)) {
    // the largest dynamic shared memory any launch of the kernel asks for: a call captured
    // into a graph holds launches of several depths, each with its own size
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 220 * 1024);
    long grid;
    if (own) {
      grid = sms;
    } else {  // as many CTAs as are resident at once (registers, shared memory, threads)
      int per_sm = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      grid = (long)h->num_sms * per_sm;
    }
    if (grid > a.n_tok) grid = a.n_tok;
    if (grid < 1) grid = 1;
    launch_kx(h, 1, own ? h->prio_hi : 0, kern, dim3((unsigned)grid), dim3(threads), smem, s, a);
  };
  if (sizeof(T) == 2 && (d == 64 || d == 128)) {
    // bf16, head dim 64 / 128: batches of 8 rows, chunks of a multiple of 8 rows (about
    // 64 KB), three buffers
    int c8 = (int)((64 * 1024) / row_bytes) / 8 * 8;
    if (c8 < 8) c8 = 8;
    a.chunk = c8 < r.l + 1 - r.r0 ? c8 : r.l + 1 - r.r0;
    smem = (int)(3 * (a.chunk * row_bytes + r.h * (long)sizeof(T)));
    if (own && smem < 116 * 1024) smem = 116 * 1024;
    if (d == 64) go(da_fast_kernel<64>);
    else go(da_fast_kernel<128>);
  } else if (own) {
    switch (d) {
      case 16: go(da_bulk_kernel<T, 16, 4>); break;
      case 32: go(da_bulk_kernel<T, 32, 4>); break;
      case 64: go(da_bulk_kernel<T, 64, 4>); break;
      default: go(da_bulk_kernel<T, 128, 4>); break;
    }
  } else {
    switch (d) {
      case 16: go(da_bulk_kernel<T, 16, 2>); break;
      case 32: go(da_bulk_kernel<T, 32, 2>); break;
      case 64: go(da_bulk_kernel<T, 64, 2>); break;
      default: go(da_bulk_kernel<T, 128, 2>); break;
    }
  }
}

// decode attention over the SA cache: streamed key ranges, then the merge of the partials
template <typename T>
static void launch_dec_bulk(dreamer_handle *h, const RowsArgs &r, int d, cudaStream_t s) {
  DecBulkArgs a{};
  a.B = r.B; a.H = r.H; a.L = r.L; a.l = r.l; a.cap = r.cap; a.nsplit = r.nsplit;
  int chunk = (int)(8192 / (d * (long)sizeof(T)));  // 8 KB of keys (and of values) a stage
  // bf16 at head dim 64 / 128 takes 8-row batches, one a warp: 64 rows a stage
  if (sizeof(T) == 2 && (d == 64 || d == 128)) chunk = 64;
  a.chunk = chunk > 256 ? 256 : chunk;
  a.q = r.q; a.ldq = r.ldq; a.kc = r.kv; a.vc = r.vc; a.cache_len = r.cache_len;
  a.part = r.part; a.err = r.err;
  const int smem = (int)(4 * 2 * (long)a.chunk * d * sizeof(T));
  const dim3 grid((unsigned)(r.B * r.H * r.nsplit));
  auto go = [&](void (*kern)(DecBulkArgs)) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    launch_k(h, kern, grid, dim3(256), smem, s, a);
  };
  switch (d) {
    case 16: go(dec_bulk_kernel<T, 16>); break;
    case 32: go(dec_bulk_kernel<T, 32>); break;
    case 64: go(dec_bulk_kernel<T, 64>); break;
    default: go(dec_bulk_kernel<T, 128>); break;
  }
}

// depth attention (mode 0) or split decode attention + merge (mode 2)
template <typename T>
static void launch_rows(dreamer_handle *h, const RowsArgs &a, int d, cudaStream_t s,
                        int da_sms = 0) {
  if (a.mode == 0 && a.H <= 32 && 2L * a.h * (long)sizeof(T) <= 48 * 1024) {
    launch_da_bulk<T>(h, a, d, s, da_sms);
    return;
  }
  if (a.mode == 2) {
    launch_dec_bulk<T>(h, a, d, s);
  } else if (sizeof(T) == 2) {
    h->path_err = 1;  // bf16 depth attention is the bulk-copy kernel only
    return;
  } else {
    const long warps = (long)a.n_q * a.H;
    const int blocks = cdiv(warps, 8);
    ++g_launches_simt;
    switch (d) {
      case 16: launch_k(h, attn_rows_kernel<T, 16, 4>, dim3(blocks), dim3(256), 0, s, a); break;
      case 32: launch_k(h, attn_rows_kernel<T, 32, 4>, dim3(blocks), dim3(256), 0, s, a); break;
      case 64: launch_k(h, attn_rows_kernel<T, 64, 4>, dim3(blocks), dim3(256), 0, s, a); break;
      default: launch_k(h, attn_rows_kernel<T, 128, 4>, dim3(blocks), dim3(256), 0, s, a); break;
    }
  }
  if (a.mode == 2) {
    const int mb = cdiv((long)a.n_q * a.H, 8);
    switch (d) {
      case 16: launch_k(h, attn_merge_kernel<T, 16>, dim3(mb), dim3(256), 0, s, a); break;
      case 32: launch_k(h, attn_merge_kernel<T, 32>, dim3(mb), dim3(256), 0, s, a); break;
      case 64: launch_k(h, attn_merge_kernel<T, 64>, dim3(mb), dim3(256), 0, s, a); break;
      default: launch_k(h, attn_merge_kernel<T, 128>, dim3(mb), dim3(256), 0, s, a); break;
    }
  }
}

// SMs depth attention gets when it runs beside causal SA in a prefill depth step (papernotes
// "Key design 1": DA and SA computed in parallel).  Both kernels fill whole SMs, so run side
// by side at full width they would take turns; instead DA takes n SMs of its own and SA the
// rest.  n balances DA's streamed K/V bytes on n SMs against SA's tensor-core work on the
// other SMs, from per-SM rates measured on B200: DA about DA_BYTES_SM bytes/s an SM, up to
// DA_BYTES_ALL over the whole chip; flash SA about SA_FLOPS_SM_D128 (head dim 128) or
// SA_FLOPS_SM_D64 flop/s an SM.  0 when the split does not pay (DA then runs at full width).
static constexpr double DA_BYTES_SM = 26e9, DA_BYTES_ALL = 4.7e12;
static constexpr double SA_FLOPS_SM_D128 = 5.3e12, SA_FLOPS_SM_D64 = 2.5e12;
static int da_beside_sa_sms(const dreamer_handle *h, int l, int r0) {
  const dreamer_config &c = h->cfg;
  const double hd = c.hidden, T = (double)c.batch * c.seq;
  const double bytes = T * (double)(l + 1 - r0) * 4.0 * hd;  // the depths' bf16 K and V rows
  const double flops = 2.0 * hd * c.batch * (double)c.seq * (c.seq + 1.0);  // causal half
  const double r_sa = c.head_dim == 128 ? SA_FLOPS_SM_D128 : SA_FLOPS_SM_D64;
  const int S = h->num_sms;
  double best = 1e30;
  int bn = 0;
  for (int n = 8; n <= S - 8; n++) {
    const double t = fmax(bytes / fmin(n * DA_BYTES_SM, DA_BYTES_ALL), flops / ((S - n) * r_sa));
    if (t < best) {
      best = t;
      bn = n;
    }
  }
  const double apart = bytes / DA_BYTES_ALL + flops / (S * r_sa);
  return best < 0.9 * apart ? bn : 0;
}

template <typename T, int SEG>
static void gemm_qkv(dreamer_handle *h, const GemmArgs &a, int max_tiles, const EpiQKV<T> &e,
                     cudaStream_t s) {
  gemm_simt<T, T, SEG>(a, max_tiles, e, s);
}

// Routing of n rows X [n][h] at depth l (router query projection, scores against the
// depth-RoPE'd keys, top-k).  mode 0: expert attention; mode 1: projection router.
template <typename T>
static void route_rows(dreamer_handle *h, int mode, int l, const void *X, int n, int *idx,
                       float *wout, int *counts_a, int *counts_b, cudaStream_t s) {
  const dreamer_config &c = h->cfg;
  const int dr = c.router_dim, hd = c.hidden;
  const int E = mode == 0 ? c.n_experts : c.n_proj_experts;
  const int ldz = mode == 0 ? h->ldz : h->ldzp;
  const void *Wq = mode == 0 ? h->wqE_t : h->wqP_t;
  const float *krot = (mode == 0 ? h->kE_rot : h->kP_rot) + (size_t)l * E * dr;
  if (mode == 0 && (long)n * 4 < (long)h->num_sms * 32 && (dr == 32 || dr == 64 || dr == 128) &&
      hd % 8 == 0) {
    // few tokens: query, scores and top-k in one kernel, a cluster of CTAs a token
    TopkArgs t{};
    t.n_tok = n; t.E = E; t.k = c.top_k; t.mode = 0;
    t.zscale = 1.0f / sqrtf((float)dr); t.bias = h->bias;
    t.idx = idx; t.w = wout; t.counts_a = counts_a; t.counts_b = counts_b;
    const int ncl = E >= 1024 ? 8 : (E >= 256 ? 4 : 1);
    auto kern = dr == 32 ? route_cluster_kernel<T, 32>
                         : (dr == 64 ? route_cluster_kernel<T, 64> : route_cluster_kernel<T, 128>);
    launch_kc(h, ncl, kern, dim3(n * ncl), dim3(256), 0, s, (const T *)X, hd, (const T *)Wq,
              (const T *)h->kE_raw, (const float2 *)(h->rope_dr + (size_t)l * (dr / 2)), t);
    return;
  }
  if (c.dtype == 1) {
    // bf16: query GEMM on tcgen05, then the fused top-k score GEMM or the warp scorer
    if (!(mode == 0 && tc_route(h, l, X, n, idx, wout, counts_a, counts_b, s))) h->path_err = 1;
    return;
  }
  // float32: q = X W_q (fp32 accumulation), z = q . k~ (fp32), on CUDA cores
  GemmArgs a = dense_args(n, dr, hd, X, hd, Wq, hd);
  gemm_simt<T, T, 8>(a, cdiv(n, 64), EpiStoreF32{h->qbuf, dr, dr}, s);
  GemmArgs b = dense_args(n, E, dr, h->qbuf, dr, krot, dr);
  gemm_simt<float, float, 8>(b, cdiv(n, 64), EpiStoreF32{h->zbuf, ldz, E}, s);
  TopkArgs t{};
  t.n_tok = n; t.E = E; t.k = mode == 0 ? c.top_k : 1; t.mode = mode;
  t.z = h->zbuf; t.ldz = ldz; t.zscale = 1.0f / sqrtf((float)dr);
  t.bias = mode == 0 ? h->bias : nullptr;
  t.idx = idx; t.w = wout; t.counts_a = counts_a; t.counts_b = counts_b;
  launch_topk(h, t, s);
}

static void trace_depth(dreamer_handle *h, const dreamer_trace *tr, int l, int n, bool prefill,
                        cudaStream_t s) {
  if (!tr) return;
  pdl_break(h, s);
  const dreamer_config &c = h->cfg;
  const size_t es = h->esz, hd = c.hidden, k = c.top_k;
  const size_t off = (size_t)l * n;
  if (tr->xhat) cudaMemcpyAsync((char *)tr->xhat + off * hd * es, h->xh, n * hd * es, cudaMemcpyDeviceToDevice, s);
  if (tr->y) cudaMemcpyAsync((char *)tr->y + off * hd * es, h->y, n * hd * es, cudaMemcpyDeviceToDevice, s);
  if (tr->idx) cudaMemcpyAsync(tr->idx + off * k, h->eidx, n * k * sizeof(int), cudaMemcpyDeviceToDevice, s);
  if (tr->w) cudaMemcpyAsync(tr->w + off * k, h->ew, n * k * sizeof(float), cudaMemcpyDeviceToDevice, s);
  if (prefill && tr->sa_k)
    cudaMemcpy2DAsync((char *)tr->sa_k + off * hd * es, hd * es, (char *)h->qkv_sa + hd * es,
                      3 * hd * es, hd * es, n, cudaMemcpyDeviceToDevice, s);
  if (prefill && tr->sa_v)
    cudaMemcpy2DAsync((char *)tr->sa_v + off * hd * es, hd * es, (char *)h->qkv_sa + 2 * hd * es,
                      3 * hd * es, hd * es, n, cudaMemcpyDeviceToDevice, s);
  if (c.n_proj_experts > 0) {
    if (tr->pidx) cudaMemcpyAsync(tr->pidx + off, h->pidx, n * sizeof(int), cudaMemcpyDeviceToDevice, s);
    if (tr->psig) cudaMemcpyAsync(tr->psig + off, h->psig, n * sizeof(float), cudaMemcpyDeviceToDevice, s);
  }
  // the residual accumulator holds y_l in float32 between the O projection and the combine
  if (tr->y_f32) cudaMemcpyAsync(tr->y_f32 + off * hd, h->acc, n * hd * sizeof(float), cudaMemcpyDeviceToDevice, s);
}

// after the combine: the accumulator holds x_{l+1} in float32
static void trace_next(dreamer_handle *h, const dreamer_trace *tr, int l, int n, cudaStream_t s) {
  if (!tr || !tr->x_f32) return;
  pdl_break(h, s);
  const size_t hd = h->cfg.hidden, off = (size_t)l * n;
  cudaMemcpyAsync(tr->x_f32 + off * hd, h->acc, n * hd * sizeof(float), cudaMemcpyDeviceToDevice, s);
}

struct DepthIO {
  int mode;               // 0 prefill, 1 decode
  int n_tok;
  const void *x_in;       // first depth only
  void *x_out;            // written by the last depth's combine
  const dreamer_trace *tr;
  void *da_kv;
  void *k_cache, *v_cache;
  const int *cache_len;
};

// One depth step for all n_tok tokens.
template <typename T>
static void run_depth(dreamer_handle *h, int l, bool first, bool last, const DepthIO &io,
                      cudaStream_t s) {
  const dreamer_config &c = h->cfg;
  const int hd = c.hidden, d = c.head_dim, L = c.depth, E = c.n_experts, k = c.top_k;
  const int m = c.expert_hidden, P = c.n_proj_experts, G = P > 0 ? P : 1;
  const int n = io.n_tok;
  const bool tc = c.dtype == 1;  // bf16: tcgen05 and streaming kernels only

  // 1. RMSNorm of the residual stream on the first depth of the call (later depths get x^
  // from the previous depth's fused combine + norm)
  mark(h, s, DREAMER_STAGE_NORM);
  if (first)
    launch_k(h, rmsnorm_kernel<T>, dim3(cdiv(n, 8)), dim3(256), 0, s, (const T *)io.x_in,
             (const float *)nullptr, (const T *)h->g, (T *)h->xh, h->inv_rms, n, hd, c.rms_eps);
  // Expert attention (steps 6-7 below): routing on y (fully parallel layout: on x^), token
  // grouping and the expert FFNs, enqueued on stream st.  Defined here so that the fully
  // parallel layout can start it first, on a stream of its own.
  const void *ein = c.variant == 2 ? h->xh : h->y;
  // few rows per expert (decode): every routed row computes its own expert FFN, unsorted
  const bool by_rows = (long)n * k < 8L * E && (m == 16 || m == 32 || m == 64) &&
                       hd <= 2048 && hd % 8 == 0;
  auto run_ea = [&](cudaStream_t st) {
    mark(h, s, DREAMER_STAGE_EA_ROUTE);
    if (by_rows) {
      route_rows<T>(h, 0, l, ein, n, h->eidx, h->ew, h->counts + (size_t)l * E, nullptr, st);
    } else {
      // ecnt / ecursor are zero here: cleared at init and by every depth's combine kernel
      route_rows<T>(h, 0, l, ein, n, h->eidx, h->ew, h->counts + (size_t)l * E, h->ecnt, st);
      mark(h, s, DREAMER_STAGE_PERMUTE);
      if (E <= 8192) {
        launch_k(h, permute_kernel, dim3(cdiv((long)n * k, 1024)), dim3(1024),
                 (size_t)(E + 1) * sizeof(int), st, (const int *)h->ecnt, E, (const int *)h->eidx,
                 n * k, h->eoffs, h->etiles_a, 64, h->etiles_b, 128, h->ecursor, h->erows, h->einv,
                 h->etab);
      } else {
        launch_k(h, scan_kernel, dim3(1), dim3(1024), 0, st, (const int *)h->ecnt, E, h->eoffs,
                 h->etiles_a, 64, h->etiles_b, 128, h->ecursor);
        launch_k(h, scatter_kernel, dim3(cdiv((long)n * k, 256)), dim3(256), 0, st,
                 (const int *)h->eidx, n * k, h->ecursor, h->erows, h->einv);
      }
    }
    // 7. expert FFNs: H = SiLU(X W1_e), acc[token] += w * H W2_e
    mark(h, s, DREAMER_STAGE_EXPERTS);
    if (by_rows) {
      auto kern = m == 16 ? expert_rows_kernel<T, 16>
                          : (m == 32 ? expert_rows_kernel<T, 32> : expert_rows_kernel<T, 64>);
      launch_k(h, kern, dim3(n * k), dim3(256), 0, st, (const T *)ein, (const int *)h->eidx,
               n * k, k, hd, (const T *)h->w1_t, (const T *)h->w2_t, (T *)h->Ybuf);
    } else if (tc) {
      if (!(tc_expert_ok(h) && tc_expert(h, ein, n, st))) h->path_err = 1;
    } else {
      const int etiles = cdiv((long)n * k, 64) + E;
      GemmArgs up{};
      up.N = m; up.K = hd; up.G = E; up.M = n * k; up.goffs = h->eoffs; up.tile_offs = h->etiles_a;
      up.arow = h->erows; up.arow_div = k; up.A = ein; up.lda = hd; up.B = h->w1_t; up.ldb = hd;
      up.bgstride = (long)m * hd;
      gemm_simt<T, T, 16>(up, etiles, EpiUp<T>{m, (T *)h->Hbuf}, st);
      GemmArgs dn{};
      dn.N = hd; dn.K = m; dn.G = E; dn.M = n * k; dn.goffs = h->eoffs; dn.tile_offs = h->etiles_a;
      dn.arow = nullptr; dn.arow_div = 1; dn.A = h->Hbuf; dn.lda = m; dn.B = h->w2_t; dn.ldb = m;
      dn.bgstride = (long)m * hd;
      gemm_simt<T, T, 16>(dn, etiles, EpiDownStore<T>{hd, (T *)h->Ybuf}, st);
    }
  };
  // the fully parallel layout ([notes] ablation table): expert attention reads x^ only, so
  // with bf16 it runs on a third stream beside the projections, DA, SA and O (one more branch
  // of the captured graph), joined before the combine; with stage profiling on it runs in line
  const bool ea_beside = c.variant == 2 && c.dtype == 1 && !h->prof;
  if (ea_beside) {
    cudaEventRecord(h->ev_fork2, s);
    cudaStreamWaitEvent(h->side2, h->ev_fork2, 0);
    pdl_break(h, h->side2);
    run_ea(h->side2);
    cudaEventRecord(h->ev_join2, h->side2);
  }
  // 2. projection router and token grouping (linear-MoE QKV/O).  In bf16 prefill (not the
  // serial layout) the grouped projections read their A rows in group order with TMA: x^ is
  // gathered into that order once, and SA and DA write their outputs at the tokens' sorted
  // rows, so that the O projection reads them in order too.
  const int *prow = nullptr;
  const float *psig = nullptr;
  const bool sorted = P > 0 && tc && io.mode == 0 && c.variant != 1;
  if (P > 0) {
    mark(h, s, DREAMER_STAGE_PROJ_ROUTE);
    // pcnt / pcursor are zero here: cleared at init and by every depth's combine kernel
    if (!tc)
      route_rows<T>(h, 1, l, h->xh, n, h->pidx, h->psig, nullptr, h->pcnt, s);
    else if (!tc_proj_route(h, l, h->xh, n, s))
      h->path_err = 1;
    launch_k(h, permute_kernel, dim3(cdiv(n, 1024)), dim3(1024), (size_t)(G + 1) * sizeof(int), s,
             (const int *)h->pcnt, G, (const int *)h->pidx, n, h->poffs, h->ptiles_a, 64,
             h->ptiles_b, 128, h->pcursor, h->prows, h->pinv, h->ptab);
    prow = h->prows;
    psig = h->psig;
    if (sorted) {
      // four rows a CTA at a time, a thread a 16-byte chunk of each
      const int threads = hd / 8 < 32 ? 32 : (hd / 8 > 256 ? 256 : hd / 8);
      const long groups = cdiv(n, 4);
      const long cap = 2048L / threads * h->num_sms;  // the CTAs resident at once
      launch_k(h, gather_rows_kernel, dim3((unsigned)(groups < cap ? groups : cap)), dim3(threads),
               0, s, (const bf16 *)h->xh, (const int *)h->prows, (bf16 *)h->xh_sorted, n, hd);
    }
  }
  auto grouped = [&](int N, int K, const void *A, long lda, const void *B, long bgs) {
    GemmArgs a{};
    a.N = N; a.K = K; a.G = G; a.M = n;
    a.goffs = P > 0 ? h->poffs : nullptr;
    a.tile_offs = P > 0 ? h->ptiles_a : nullptr;
    a.arow = prow; a.arow_div = 1; a.A = A; a.lda = lda; a.B = B; a.ldb = K; a.bgstride = bgs;
    a.a_sorted = sorted ? 1 : 0;
    return a;
  };
  const int ptiles = cdiv(n, 64) + (P > 0 ? G : 0);

  EpiQKV<T> eq{};
  eq.h = hd; eq.d = d; eq.L = L; eq.l = l; eq.S = c.seq; eq.mode = io.mode; eq.col_lo = 0;
  eq.perm = h->qkv_perm;
  eq.psig = psig; eq.rope_tok = h->rope_tok; eq.rope_dep = h->rope_dep;
  eq.qkv_sa = (T *)h->qkv_sa; eq.q_da = (T *)h->q_da; eq.da_kv = (T *)io.da_kv;
  eq.k_cache = (T *)io.k_cache; eq.v_cache = (T *)io.v_cache; eq.cache_len = io.cache_len;
  eq.B = c.batch; eq.cap = c.max_cache_len; eq.err = h->err;

  RowsArgs da{};
  da.mode = 0; da.n_q = n; da.H = c.n_heads; da.h = hd; da.L = L; da.l = l;
  da.r0 = (c.da_window > 0 && l + 1 > c.da_window) ? l + 1 - c.da_window : 0;
  da.q = h->q_da; da.ldq = hd; da.kv = io.da_kv;
  da.out = h->attn; da.ldo = 2 * hd; da.col0 = hd; da.err = h->err;
  da.out_rows = sorted ? h->pinv : nullptr;
  RowsArgs sd{};  // decode: attention over the per-depth SA cache, split over key ranges
  sd.mode = 2; sd.n_q = n; sd.H = c.n_heads; sd.h = hd; sd.L = L; sd.l = l;
  sd.q = h->qkv_sa; sd.ldq = 3 * hd; sd.kv = io.k_cache; sd.vc = io.v_cache;
  sd.B = c.batch; sd.cap = c.max_cache_len; sd.nsplit = h->nsplit; sd.cache_len = io.cache_len;
  sd.err = h->err; sd.out = h->attn; sd.ldo = 2 * hd; sd.col0 = 0; sd.part = h->part;
  AttnArgs sa{};
  sa.mode = io.mode == 0 ? 1 : 2; sa.n_q = n; sa.H = c.n_heads; sa.d = d; sa.h = hd;
  sa.q = h->qkv_sa; sa.ldq = 3 * hd; sa.kv = io.mode == 0 ? h->qkv_sa : io.k_cache;
  sa.vc = io.v_cache; sa.L = L; sa.l = l; sa.S = c.seq; sa.B = c.batch;
  sa.cap = c.max_cache_len; sa.cache_len = io.cache_len; sa.err = h->err;
  sa.out = h->attn; sa.ldo = 2 * hd; sa.col0 = 0;

  // SA: tcgen05 flash kernel for bf16 prefill, split decode attention for decode, the warp
  // kernel for float32 prefill
  auto run_sa = [&](cudaStream_t st) {
    if (io.mode == 1) {
      launch_rows<T>(h, sd, d, st);
      return;
    }
    if (!tc)
      launch_attn<T>(sa, d, st);
    else if (!(tc_sa_ok(h) && tc_sa(h, st, sorted ? h->pinv : nullptr)))
      h->path_err = 1;
  };
  auto qkv_gemm = [&](const void *A, int col0, int ncols) {
    // columns [col0, col0 + ncols) of the fused QKV projection
    mark(h, s, DREAMER_STAGE_QKV);
    GemmArgs a = grouped(ncols, hd, A, hd, (const T *)h->wqkv_t + (size_t)col0 * hd,
                         (long)6 * hd * hd);
    EpiQKV<T> e2 = eq;
    e2.col_lo = col0;
    if (tc) {
      if (!(tc_gemm_ok(h, a) && tc_gemm_qkv(h, a, e2, s))) h->path_err = 1;
      return;
    }
    switch (d) {
      case 16: gemm_qkv<T, 16>(h, a, ptiles, e2, s); break;
      case 32: gemm_qkv<T, 32>(h, a, ptiles, e2, s); break;
      case 64: gemm_qkv<T, 64>(h, a, ptiles, e2, s); break;
      default: gemm_qkv<T, 128>(h, a, ptiles, e2, s); break;
    }
  };
  // residual source of the O epilogue: x^ rebuilt from x_l (first depth: the input,
  // else the fp32 accumulator rounded to dtype) or, for the serial layout's second half, u
  const int res_xhat = first ? 0 : 1;
  auto o_gemm = [&](const void *A, int row0, int nrows, int res_mode, void *yout) {
    // O projection over input rows [row0, row0 + nrows) of W_O ([a_SA | a_DA] order)
    mark(h, s, DREAMER_STAGE_O);
    GemmArgs a = grouped(hd, nrows, A, 2 * hd, (const T *)h->wo_t + row0, (long)2 * hd * hd);
    a.ldb = 2 * hd;
    EpiO<T> eo{hd, psig, res_mode, (const T *)io.x_in, h->inv_rms, (const T *)h->g,
               (T *)yout, h->acc};
    if (tc) {
      if (!(tc_gemm_ok(h, a) && tc_gemm_o(h, a, eo, s))) h->path_err = 1;
      return;
    }
    gemm_simt<T, T, 16>(a, ptiles, eo, s);
  };

  if (c.variant == 3) {
    // without depth attention (the DR-without-DA arm): the SA columns of the projection
    // only, y = x^ + SA W_O[SA rows]
    qkv_gemm(sorted ? h->xh_sorted : h->xh, 0, 3 * hd);
    mark(h, s, DREAMER_STAGE_SA);
    run_sa(s);
    o_gemm(h->attn, 0, hd, res_xhat, h->y);
  } else if (c.variant == 1) {
    // serial DA -> SA -> EA: DA on x^, then SA on u = x^ + DA-part of O, then EA
    qkv_gemm(h->xh, 3 * hd, 3 * hd);
    mark(h, s, DREAMER_STAGE_DA);
    launch_rows<T>(h, da, d, s);
    o_gemm((const T *)h->attn + hd, hd, hd, res_xhat, h->u);   // u = x^ + DA part (acc = u)
    qkv_gemm(h->u, 0, 3 * hd);
    mark(h, s, DREAMER_STAGE_SA);
    run_sa(s);
    o_gemm(h->attn, 0, hd, 2, h->y);                            // y = u + SA part
  } else {
    // 3. fused QKV projection with RoPE / depth RoPE epilogue, DA KV write
    qkv_gemm(sorted ? h->xh_sorted : h->xh, 0, 6 * hd);
    // 4. DA || SA (papernotes "Key design 1": run in parallel for throughput).  DA runs
    // on the side stream beside SA (two branches of the captured graph), on SMs of its own
    // where that pays; with stage profiling on they run one after the other (same launch
    // shapes) so each stage's time is its own.
    const int da_sms = io.mode == 0 && c.dtype == 1 ? da_beside_sa_sms(h, l, da.r0) : 0;
    if (h->prof) {
      mark(h, s, DREAMER_STAGE_DA);
      launch_rows<T>(h, da, d, s, da_sms);
    } else {
      cudaEventRecord(h->ev_fork, s);
      cudaStreamWaitEvent(h->side, h->ev_fork, 0);
      pdl_break(h, h->side);
      launch_rows<T>(h, da, d, h->side, da_sms);
      cudaEventRecord(h->ev_join, h->side);
    }
    mark(h, s, DREAMER_STAGE_SA);
    // with DA on its own SMs, SA starts after the projection has completed, as DA does, so that
    // DA's urgent CTAs are placed first (no early launch of SA's CTAs into the projection's tail)
    if (da_sms > 0) pdl_break(h, s);
    run_sa(s);
    if (!h->prof) {
      cudaStreamWaitEvent(s, h->ev_join, 0);
      pdl_break(h, s);
    }
    // 5. O projection, residual y = x^ + DA + SA
    o_gemm(h->attn, 0, 2 * hd, res_xhat, h->y);
  }
  // 6-7. expert attention in line, or the join of its own stream
  if (!ea_beside) {
    run_ea(s);
  } else {
    cudaStreamWaitEvent(s, h->ev_join2, 0);
    pdl_break(h, s);
  }
  // per-depth dumps (before the combine replaces x^ with the next depth's)
  trace_depth(h, io.tr, l, n, io.mode == 0, s);
  // 8. x_{l+1} = y + sum_s w_s Y_s, then the next depth's RMSNorm (or the call's output)
  mark(h, s, DREAMER_STAGE_FINISH);
  if (c.dtype == 1) {  // bf16: a CTA of h / 8 threads per token (h <= 4096, k <= 16)
    auto kern = k <= 4 ? combine_norm_row_kernel<4>
                       : (k <= 8 ? combine_norm_row_kernel<8> : combine_norm_row_kernel<16>);
    launch_k(h, kern, dim3(n), dim3(hd / 8), 0, s, h->acc,
             (const bf16 *)h->Ybuf, by_rows ? (const int *)nullptr : (const int *)h->einv,
             (const float *)h->ew, k, (const bf16 *)h->g, (bf16 *)h->xh, h->inv_rms,
             last ? (bf16 *)io.x_out : (bf16 *)nullptr, n, hd, c.rms_eps, h->ecnt, 2 * E,
             h->pcnt, P > 0 ? 2 * (G + 1) : 0);
  } else {
    const int cb = cdiv(n, 8);
    auto combine = hd <= 2048 ? combine_norm_kernel<T, 64> : combine_norm_kernel<T, 128>;
    launch_k(h, combine, dim3(cb), dim3(256), 0, s, h->acc, (const T *)h->Ybuf,
             by_rows ? (const int *)nullptr : (const int *)h->einv, (const float *)h->ew, k,
             (const T *)h->g, (T *)h->xh,
             h->inv_rms, last ? (T *)io.x_out : (T *)nullptr, n, hd, c.rms_eps, h->ecnt, 2 * E,
             h->pcnt, P > 0 ? 2 * (G + 1) : 0);
  }
  trace_next(h, io.tr, l, n, s);
}

// The device error flag is copied to pinned host memory at the end of every call; the next
// call reads that copy without synchronising (errors of calls still running show up one call
// later, or at dreamer_route_counts(on_host = 1), which synchronises and reads it exactly).
static int dev_error_code(int e) { return e == DEV_TIMEOUT ? DREAMER_ERR_TIMEOUT : DREAMER_ERR_ARG; }
static int check_dev_error(dreamer_handle *h) {
  const int e = *(volatile int *)h->err_host;
  if (e) {
    cudaDeviceSynchronize();
    cudaMemset(h->err, 0, sizeof(int));
    *h->err_host = 0;
    return dev_error_code(e);
  }
  return DREAMER_OK;
}
static int check_dev_error_sync(dreamer_handle *h) {
  int e = 0;
  if (cudaMemcpy(&e, h->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DREAMER_ERR_CUDA;
  if (e) {
    cudaMemset(h->err, 0, sizeof(int));
    *h->err_host = 0;
    return dev_error_code(e);
  }
  return DREAMER_OK;
}

static bool aligned16(const void *p) { return ((uintptr_t)p & 15) == 0; }

// ---------------------------------------------------------------------------------------
// CUDA graphs: the whole call (every depth, ~10 kernels each) is captured once per set of
// argument pointers and replayed, so the host enqueues one graph instead of ~10 L kernels.
// A pointer set runs directly the first time it is seen (this also sets every kernel's
// attributes outside capture) and is captured on its second use.  Calls with a trace run
// directly.  Up to 8 graphs are cached per handle (least recently used evicted).
template <class F>
static int run_graphed(dreamer_handle *h, int kind, const void *const key[5], int l0, int l1,
                       cudaStream_t s, F &&enqueue) {
  if (!h->use_graph) return enqueue();
#ifdef DREAMER_TEST_HOOKS
  if (h->inject_skip) return enqueue();  // an injected call runs directly, never from a graph
#endif
  dreamer_handle::GraphEntry *e = nullptr;
  for (auto &g : h->graphs)
    if (g.kind == kind && g.l0 == l0 && g.l1 == l1 && g.prof == h->prof &&
        !memcmp(g.key, key, sizeof(g.key))) {
      e = &g;
      break;
    }
  if (!e) {
    if (h->graphs.size() >= 8) {
      size_t old = 0;
      for (size_t i = 1; i < h->graphs.size(); i++)
        if (h->graphs[i].last_use < h->graphs[old].last_use) old = i;
      auto &g = h->graphs[old];
      if (g.captured) cudaGraphExecDestroy(g.exec);
      for (cudaEvent_t ev : g.evs) cudaEventDestroy(ev);
      h->graphs.erase(h->graphs.begin() + old);
    }
    dreamer_handle::GraphEntry g{};
    g.kind = kind;
    memcpy(g.key, key, sizeof(g.key));
    g.l0 = l0; g.l1 = l1; g.prof = h->prof; g.captured = 0;
    g.last_use = ++h->use_clock;
    h->graphs.push_back(g);
    return enqueue();  // first use: direct
  }
  e->last_use = ++h->use_clock;
  if (!e->captured) {
    const size_t ev0 = h->ev_used;
    const uint64_t l_before = g_launches, tc_before = g_launches_tc, simt_before = g_launches_simt;
    cudaGraph_t graph = nullptr;
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      cudaGetLastError();
      return enqueue();
    }
    int rc = enqueue();
    cudaError_t ce = cudaStreamEndCapture(s, &graph);
    const uint64_t n_launch = g_launches - l_before;
    const uint64_t n_tc = g_launches_tc - tc_before, n_simt = g_launches_simt - simt_before;
    // captured kernels run when the graph is launched
    g_launches = l_before;
    g_launches_tc = tc_before;
    g_launches_simt = simt_before;
    if (rc != DREAMER_OK || ce != cudaSuccess || !graph) {
      if (graph) cudaGraphDestroy(graph);
      cudaGetLastError();
      h->ev_used = ev0;
      h->use_graph = 0;  // capture is not available here: run directly from now on
      return rc != DREAMER_OK ? rc : enqueue();
    }
    cudaError_t ie = cudaGraphInstantiate(&e->exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ie != cudaSuccess) {
      cudaGetLastError();
      h->ev_used = ev0;
      h->use_graph = 0;
      return enqueue();
    }
    e->captured = 1;
    e->launches = n_launch;
    e->launches_tc = n_tc;
    e->launches_simt = n_simt;
    // the graph records into the events its marks captured: they now belong to it
    e->evs.assign(h->ev.begin() + ev0, h->ev.begin() + h->ev_used);
    e->stages.assign(h->ev_stage.begin() + ev0, h->ev_stage.begin() + h->ev_used);
    h->ev.erase(h->ev.begin() + ev0, h->ev.begin() + h->ev_used);
    h->ev_stage.erase(h->ev_stage.begin() + ev0, h->ev_stage.begin() + h->ev_used);
    h->ev_used = ev0;
  }
  CK(cudaGraphLaunch(e->exec, s));
  g_launches += e->launches;
  g_launches_tc += e->launches_tc;
  g_launches_simt += e->launches_simt;
  if (e->prof && !e->evs.empty()) {
    CK(cudaStreamSynchronize(s));
    accumulate_marks(h, e->evs, e->stages);
  }
  return DREAMER_OK;
}

template <typename T>
static int forward_impl(dreamer_handle *h, const void *x_in, void *x_out, int l0, int l1,
                        void *da_kv, const dreamer_trace *tr, cudaStream_t s) {
  const dreamer_config &c = h->cfg;
  const int n = c.batch * c.seq;
  CK(cudaMemsetAsync(h->counts, 0, (size_t)c.depth * c.n_experts * sizeof(int), s));
  // grouping counters: zero between depths by construction; cleared here as well so that a
  // call after a failed one starts clean
  CK(cudaMemsetAsync(h->ecnt, 0, 2 * (size_t)c.n_experts * sizeof(int), s));
  CK(cudaMemsetAsync(h->pcnt, 0, 2 * (size_t)((c.n_proj_experts > 0 ? c.n_proj_experts : 1) + 1) * sizeof(int), s));
  pdl_break(h, s);
  pdl_break(h, h->side);
  pdl_break(h, h->side2);
  DepthIO io{};
  io.mode = 0; io.n_tok = n; io.x_in = x_in; io.x_out = x_out; io.tr = tr;
  io.da_kv = da_kv ? da_kv : h->da_kv_int;
  h->path_err = 0;
  for (int l = l0; l < l1; l++) run_depth<T>(h, l, l == l0, l == l1 - 1, io, s);
  if (h->path_err) return DREAMER_ERR_UNSUPPORTED;
  if (l1 == l0 && x_out != x_in) {
    CK(cudaMemcpyAsync(x_out, x_in, (size_t)n * c.hidden * h->esz, cudaMemcpyDeviceToDevice, s));
  }
  CK(cudaMemcpyAsync(h->err_host, h->err, sizeof(int), cudaMemcpyDeviceToHost, s));
  mark(h, s, DREAMER_N_STAGES);
  CK(cudaGetLastError());
  return DREAMER_OK;
}

extern "C" int dreamer_core_forward(dreamer_handle *h, const void *x_in, void *x_out,
                                    int depth_begin, int depth_end, void *da_kv,
                                    const dreamer_trace *trace, dreamer_stream stream) {
  if (!h || !x_in || !x_out) return DREAMER_ERR_ARG;
  const dreamer_config &c = h->cfg;
  if (depth_begin < 0 || depth_end > c.depth || depth_begin > depth_end) return DREAMER_ERR_ARG;
  if (!da_kv && depth_begin != 0 && c.variant != 3) return DREAMER_ERR_ARG;
  if (!aligned16(x_in) || !aligned16(x_out) || (da_kv && !aligned16(da_kv))) return DREAMER_ERR_ARG;
  if (!h->prefill_ok) return DREAMER_ERR_UNSUPPORTED;
  int e = check_dev_error(h);
  if (e) return e;
  cudaStream_t s = (cudaStream_t)stream;
  auto enqueue = [&]() -> int {
    return c.dtype == 0 ? forward_impl<float>(h, x_in, x_out, depth_begin, depth_end, da_kv, trace, s)
                        : forward_impl<bf16>(h, x_in, x_out, depth_begin, depth_end, da_kv, trace, s);
  };
  const uint64_t l0c = g_launches, l0tc = g_launches_tc, l0simt = g_launches_simt;
  int rc;
  if (trace) {
    rc = enqueue();
  } else {
    const void *key[5] = {x_in, x_out, da_kv, nullptr, nullptr};
    rc = run_graphed(h, 0, key, depth_begin, depth_end, s, enqueue);
  }
  h->launches += g_launches - l0c;
  h->launches_tc += g_launches_tc - l0tc;
  h->launches_simt += g_launches_simt - l0simt;
  return rc;
}

template <typename T>
static int decode_impl(dreamer_handle *h, const void *x_new, void *kc, void *vc,
                       const int32_t *len, void *x_out, const dreamer_trace *tr, cudaStream_t s) {
  const dreamer_config &c = h->cfg;
  const int n = c.batch;
  CK(cudaMemsetAsync(h->counts, 0, (size_t)c.depth * c.n_experts * sizeof(int), s));
  // grouping counters: zero between depths by construction; cleared here as well so that a
  // call after a failed one starts clean
  CK(cudaMemsetAsync(h->ecnt, 0, 2 * (size_t)c.n_experts * sizeof(int), s));
  CK(cudaMemsetAsync(h->pcnt, 0, 2 * (size_t)((c.n_proj_experts > 0 ? c.n_proj_experts : 1) + 1) * sizeof(int), s));
  pdl_break(h, s);
  pdl_break(h, h->side);
  pdl_break(h, h->side2);
  DepthIO io{};
  io.mode = 1; io.n_tok = n; io.x_in = x_new; io.x_out = x_out; io.tr = tr;
  io.da_kv = h->da_kv_int;
  io.k_cache = kc; io.v_cache = vc; io.cache_len = len;
  h->path_err = 0;
  for (int l = 0; l < c.depth; l++) run_depth<T>(h, l, l == 0, l == c.depth - 1, io, s);
  if (h->path_err) return DREAMER_ERR_UNSUPPORTED;
  CK(cudaMemcpyAsync(h->err_host, h->err, sizeof(int), cudaMemcpyDeviceToHost, s));
  mark(h, s, DREAMER_N_STAGES);
  CK(cudaGetLastError());
  return DREAMER_OK;
}

extern "C" int dreamer_decode_step(dreamer_handle *h, const void *x_new, void *k_cache,
                                   void *v_cache, const int32_t *cache_len, void *x_out,
                                   const dreamer_trace *trace, dreamer_stream stream) {
  if (!h || !x_new || !k_cache || !v_cache || !cache_len || !x_out) return DREAMER_ERR_ARG;
  if (h->cfg.max_cache_len < 1) return DREAMER_ERR_STATE;
  if (!aligned16(x_new) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(x_out))
    return DREAMER_ERR_ARG;
  int e = check_dev_error(h);
  if (e) return e;
  cudaStream_t s = (cudaStream_t)stream;
  auto enqueue = [&]() -> int {
    return h->cfg.dtype == 0
               ? decode_impl<float>(h, x_new, k_cache, v_cache, cache_len, x_out, trace, s)
               : decode_impl<bf16>(h, x_new, k_cache, v_cache, cache_len, x_out, trace, s);
  };
  const uint64_t l0c = g_launches, l0tc = g_launches_tc, l0simt = g_launches_simt;
  int rc;
  if (trace) {
    rc = enqueue();
  } else {
    const void *key[5] = {x_new, k_cache, v_cache, cache_len, x_out};
    rc = run_graphed(h, 1, key, 0, h->cfg.depth, s, enqueue);
  }
  h->launches += g_launches - l0c;
  h->launches_tc += g_launches_tc - l0tc;
  h->launches_simt += g_launches_simt - l0simt;
  return rc;
}

extern "C" int dreamer_route_counts(dreamer_handle *h, int32_t *counts, int on_host,
                                    dreamer_stream stream) {
  if (!h || !counts) return DREAMER_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = (size_t)h->cfg.depth * h->cfg.n_experts * sizeof(int);
  if (on_host) {
    CK(cudaMemcpyAsync(counts, h->counts, bytes, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    return check_dev_error_sync(h);
  }
  CK(cudaMemcpyAsync(counts, h->counts, bytes, cudaMemcpyDeviceToDevice, s));
  return DREAMER_OK;
}

extern "C" int dreamer_route_experts(dreamer_handle *h, int depth, const void *y, int n_tokens,
                                     int32_t *idx, float *w, int32_t *counts,
                                     dreamer_stream stream) {
  if (!h || !y || !idx || !w) return DREAMER_ERR_ARG;
  if (depth < 0 || depth >= h->cfg.depth || n_tokens < 0 || n_tokens > h->T) return DREAMER_ERR_ARG;
  if (!aligned16(y)) return DREAMER_ERR_ARG;
  if (n_tokens == 0) return DREAMER_OK;
  cudaStream_t s = (cudaStream_t)stream;
  if (counts) CK(cudaMemsetAsync(counts, 0, h->cfg.n_experts * sizeof(int), s));
  pdl_break(h, s);  // the caller's stream: whatever ran last is not ours
  h->path_err = 0;
  if (h->cfg.dtype == 0)
    route_rows<float>(h, 0, depth, y, n_tokens, idx, w, counts, nullptr, s);
  else
    route_rows<bf16>(h, 0, depth, y, n_tokens, idx, w, counts, nullptr, s);
  if (h->path_err) return DREAMER_ERR_UNSUPPORTED;
  CK(cudaGetLastError());
  return DREAMER_OK;
}

extern "C" int dreamer_route_balance(dreamer_handle *h, int depth, float *lorenz, float *gini,
                                     dreamer_stream stream) {
  if (!h || !gini) return DREAMER_ERR_ARG;
  const int E = h->cfg.n_experts, L = h->cfg.depth;
  if (depth >= L) return DREAMER_ERR_ARG;
  if (E > 8192) return DREAMER_ERR_UNSUPPORTED;
  int n2 = 1;
  while (n2 < E) n2 <<= 1;
  const size_t smem = (size_t)n2 * sizeof(int);
  if (smem > 48 * 1024)
    CK(cudaFuncSetAttribute(balance_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaStream_t s = (cudaStream_t)stream;
  pdl_break(h, s);
  launch_k(h, balance_kernel, dim3(1), dim3(1024), smem, s, (const int *)h->counts, L, E, depth,
           lorenz, gini);
  CK(cudaGetLastError());
  return DREAMER_OK;
}

static int launch_bias_update(dreamer_handle *h, const int *counts, int rows, float lambda,
                              float *bias_out, cudaStream_t s) {
  const int E = h->cfg.n_experts;
  int n2 = 1;
  while (n2 < E) n2 <<= 1;
  const size_t smem = (size_t)(n2 + E) * sizeof(int);
  if (smem > 200 * 1024) return DREAMER_ERR_UNSUPPORTED;
  if (smem > 48 * 1024)
    CK(cudaFuncSetAttribute(bias_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  ++g_launches;
  bias_update_kernel<<<1, 1024, smem, s>>>(counts, rows, E, lambda, h->bias, bias_out);
  CK(cudaGetLastError());
  return DREAMER_OK;
}

extern "C" int dreamer_bias_update(dreamer_handle *h, float lambda, float *bias_out,
                                   dreamer_stream stream) {
  if (!h) return DREAMER_ERR_ARG;
  return launch_bias_update(h, h->counts, h->cfg.depth, lambda, bias_out, (cudaStream_t)stream);
}

#ifdef DREAMER_TEST_HOOKS
// Test-hook build only (not in libdreamer.so): what = 1 makes the TMA producer of the next
// call's first QKV projection GEMM issue no loads, so that its MMA issuer's bounded wait
// expires; the call's error then surfaces as DREAMER_ERR_TIMEOUT.
extern "C" int dreamer_test_inject(dreamer_handle *h, int what) {
  if (!h || what < 0 || what > 1) return DREAMER_ERR_ARG;
  h->inject_skip = what;
  return DREAMER_OK;
}
#endif

extern "C" int dreamer_bias_update_counts(dreamer_handle *h, float lambda, const int32_t *counts,
                                          int n_rows, float *bias_out, dreamer_stream stream) {
  if (!h || !counts || n_rows < 1) return DREAMER_ERR_ARG;
  return launch_bias_update(h, counts, n_rows, lambda, bias_out, (cudaStream_t)stream);
}
