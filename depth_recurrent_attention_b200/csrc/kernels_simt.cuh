// CUDA-core kernels of the Dreamer depth step.  These carry the float32 mode end to end and
// the parts of the bfloat16 mode that are not dense contractions (norm, depth attention,
// routing top-k, permutation, decode attention).
#pragma once
#include "common.cuh"

namespace dreamer {

// =======================================================================================
// Epilogue parameter blocks (shared by the CUDA-core and the tcgen05 GEMM engines).
// Every epilogue is called per (sorted row r, token, group g, column segment starting at
// n0) with the fp32 accumulator values v[0..SEG).
// =======================================================================================

// QKV projection epilogue: scale by the projection weight sigma (linear MoE), apply token
// RoPE to q_SA/k_SA and depth RoPE to q_DA/k_DA, and scatter into the attention layouts.
// (papernotes "Key design 1": depth RoPE with a reversed half; "Key design 3": sigma x W~.)
template <typename T> struct EpiQKV {
  int h, d, L, l, S;
  int mode;                  // 0 prefill (position = token % S), 1 decode (position = cache_len[b])
  int col_lo;                // first column of the fused projection this GEMM computes
  const float *psig;         // [T] or null (dense)
  const float2 *rope_tok;    // [max_pos][d/2]
  const float2 *rope_dep;    // [L][d/2]
  T *qkv_sa;                 // [T][3h]
  T *q_da;                   // [T][h]
  T *da_kv;                  // [T][L][2][h]
  T *k_cache, *v_cache;      // decode: [L][B][H][cap][d]
  const int *cache_len;      // decode: [B]
  int B, cap;
  int *err;                  // device error flag

  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    static_assert(SEG % 16 == 0, "segment");
    const int nc = n0 + col_lo;        // column of the full [6h] projection
    const int blk = nc / h;            // 0 qSA 1 kSA 2 vSA 3 qDA 4 kDA 5 vDA
    const int head = (nc % h) / d;
    const int hc = nc % h;             // column inside the block
    if (psig) {
      const float s = psig[token];
#pragma unroll
      for (int i = 0; i < SEG; i++) v[i] *= s;
    }
    if (mode == 1 && blk <= 2) {
      const int p = cache_len[token];
      if (p < 0 || p >= cap) {  // slot outside the cache: report, write nothing
        raise_dev_error(err, DEV_BAD_INDEX);
        return;
      }
    }
    if (blk <= 1) {  // token RoPE, rotate-half over d (pair i, i + d/2)
      const int pos = mode == 0 ? (token % S) : cache_len[token];
      const float2 *cs = rope_tok + (long)pos * (d / 2);
#pragma unroll
      for (int i = 0; i < SEG / 2; i++) {
        float c = cs[i].x, s = cs[i].y;
        float a = v[i], b = v[i + SEG / 2];
        v[i] = a * c - b * s;
        v[i + SEG / 2] = b * c + a * s;
      }
    } else if (blk == 3 || blk == 4) {  // depth RoPE: halves at l and L-1-l
      const float2 *cs = rope_dep + (long)l * (d / 2);
      const int q4 = SEG / 4;
#pragma unroll
      for (int half = 0; half < 2; half++) {
#pragma unroll
        for (int i = 0; i < q4; i++) {
          float c = cs[half * q4 + i].x, s = cs[half * q4 + i].y;
          float a = v[half * (SEG / 2) + i], b = v[half * (SEG / 2) + i + q4];
          v[half * (SEG / 2) + i] = a * c - b * s;
          v[half * (SEG / 2) + i + q4] = b * c + a * s;
        }
      }
    }
    T *dst;
    if (blk <= 2) {
      if (mode == 0 || blk == 0) {
        dst = qkv_sa + (long)token * 3 * h + blk * h + hc;
      } else {
        const int pos = cache_len[token];
        T *base = (blk == 1) ? k_cache : v_cache;
        dst = base + ((((long)l * B + token) * (h / d) + head) * cap + pos) * d;
      }
    } else if (blk == 3) {
      dst = q_da + (long)token * h + hc;
    } else {
      dst = da_kv + (((long)token * L + l) * 2 + (blk - 4)) * h + hc;
    }
#pragma unroll
    for (int i = 0; i < SEG; i += 8) store8(dst + i, v + i);
  }
};

// O projection epilogue: y = x^ + sigma [a_SA | a_DA] W~_O (papernotes "Key design 1"
// residual equation).  The residual is carried in fp32: x^ is rebuilt from the residual x_l
// (dtype: the input on the first depth, else the fp32 accumulator rounded to dtype), the gain
// and the token's 1/rms, so the only rounding of y is its own store.  acc receives the fp32 y
// (the base that the expert outputs are added to); y itself is stored in dtype for the
// router and the experts.
//   res_mode 0: residual x^ from xin;  1: x^ from acc (fp32 x_l);  2: residual = acc as is
//   (the serial layout's u).
template <typename T> struct EpiO {
  int h;
  const float *psig;
  int res_mode;
  const T *xin;
  const float *inv_rms;
  const T *gain;
  T *y;             // [T][h] or null
  float *acc;       // [T][h] read (res_mode 1, 2) and written
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    const float s = psig ? psig[token] : 1.0f;
    const float ir = res_mode == 2 ? 0.f : inv_rms[token];
#pragma unroll
    for (int i = 0; i < SEG; i += 8) {
      float xr[8], gv[8], o[8];
      float *ap = acc + (long)token * h + n0 + i;
      if (res_mode == 0) load8(xin + (long)token * h + n0 + i, xr);
      else load8(ap, xr);
      if (res_mode != 2) {
        load8(gain + n0 + i, gv);
#pragma unroll
        for (int j = 0; j < 8; j++) {
          xr[j] = gv[j] * xr[j] * ir;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; j++) o[j] = xr[j] + s * v[i + j];
      if (y) store8(y + (long)token * h + n0 + i, o);
      store8(ap, o);
    }
  }
};

// Expert up-projection epilogue: H[r] = SiLU(X W1_e) (papernotes "Key design 2": each
// expert is a small FFN acting as the value transform).
template <typename T> struct EpiUp {
  int m;
  T *H;  // [rows][m] in expert-sorted order
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
#pragma unroll
    for (int i = 0; i < SEG; i++) v[i] = v[i] / (1.0f + __expf(-v[i]));
#pragma unroll
    for (int i = 0; i < SEG; i += 8) store8(H + (long)r * m + n0 + i, v + i);
  }
};

// Expert down-projection epilogue: acc[token] += w_slot * (H W2_e).
struct EpiDown {
  int h, k;
  const int *rows;    // sorted row -> token*k + slot
  const float *wts;   // [T][k]
  float *acc;         // [T][h]
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    const int slot = rows[r];
    const float w = wts[slot];
    float *dst = acc + (long)(slot / k) * h + n0;
#pragma unroll
    for (int i = 0; i < SEG; i++) atomicAdd(dst + i, w * v[i]);
  }
};

// Expert down-projection epilogue, store form: the routed row's expert output Y (sorted row
// r) is written once in dtype; the weighted sum over a token's k rows happens in
// combine_norm_kernel (no atomics, fixed summation order).
template <typename T> struct EpiDownStore {
  int h;
  T *Y;  // [rows][h], expert-sorted order
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
#pragma unroll
    for (int i = 0; i < SEG; i += 8) store8(Y + (long)r * h + n0 + i, v + i);
  }
};

// Plain fp32 store of columns < N (router queries and scores).
struct EpiStoreF32 {
  float *C;
  long ldc;
  int N;
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
#pragma unroll
    for (int i = 0; i < SEG; i++)
      if (n0 + i < N) C[(long)r * ldc + n0 + i] = v[i];
  }
};

// =======================================================================================
// Grouped GEMM on CUDA cores: for group g, C[r][n] = sum_k A[arow(r)][k] * B_g[n][k] for
// sorted rows r in [goffs[g], goffs[g+1]); B_g stored [N][K] (K contiguous).
// =======================================================================================
struct GemmArgs {
  int N, K;
  int G;                  // number of groups
  int M;                  // rows (single group, goffs == null)
  const int *goffs;       // [G+1] or null
  const int *tile_offs;   // [G+1] cumulative row tiles (of this engine's BM) or null
  const int *arow;        // sorted row -> source id, or null (identity)
  int arow_div;           // A row = arow[r] / arow_div
  const void *A;
  long lda;
  const void *B;
  long ldb, bgstride;
};

__device__ __forceinline__ bool gemm_tile_coords(const GemmArgs &a, int tile, int BM, int &g,
                                                 int &m0, int &m1) {
  if (!a.goffs) {
    g = 0;
    m0 = tile * BM;
    m1 = min(m0 + BM, a.M);
    return m0 < a.M;
  }
  int total = a.tile_offs[a.G];
  if (tile >= total) return false;
  int lo = 0, hi = a.G - 1;  // largest g with tile_offs[g] <= tile
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (a.tile_offs[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  g = lo;
  m0 = a.goffs[g] + (tile - a.tile_offs[g]) * BM;
  m1 = min(m0 + BM, a.goffs[g + 1]);
  return m0 < m1;
}

template <typename TA, typename TB, int SEG, class Epi>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs a, Epi epi) {
  constexpr int BM = 64, BN = 128, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  __shared__ float Cs[BM][BN + 4];
  int g, m0, m1;
  if (!gemm_tile_coords(a, blockIdx.x, BM, g, m0, m1)) return;
  const int n0 = blockIdx.y * BN;
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const TA *A = reinterpret_cast<const TA *>(a.A);
  const TB *B = reinterpret_cast<const TB *>(a.B) + (long)g * a.bgstride;
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 8; j++) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < a.K; k0 += BK) {
    for (int e = tid; e < BM * BK; e += 256) {
      int rr = e / BK, kk = e % BK;
      int r = m0 + rr;
      float v = 0.f;
      if (r < m1) {
        long src = a.arow ? (long)(a.arow[r] / a.arow_div) : (long)r;
        v = to_f(A[src * a.lda + k0 + kk]);
      }
      As[kk][rr] = v;
    }
    for (int e = tid; e < BN * BK; e += 256) {
      int nn = e / BK, kk = e % BK;
      int n = n0 + nn;
      Bs[kk][nn] = (n < a.N) ? to_f(B[(long)n * a.ldb + k0 + kk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; kk++) {
      float ar[4], br[8];
#pragma unroll
      for (int i = 0; i < 4; i++) ar[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 8; j++) br[j] = Bs[kk][tx * 8 + j];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = fmaf(ar[i], br[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < 8; j++) Cs[ty * 4 + i][tx * 8 + j] = acc[i][j];
  __syncthreads();
  constexpr int NSEG = BN / SEG;
  for (int item = tid; item < BM * NSEG; item += 256) {
    int rr = item / NSEG, sg = item % NSEG;
    int r = m0 + rr;
    int n = n0 + sg * SEG;
    if (r >= m1 || n >= a.N) continue;
    float v[SEG];
#pragma unroll
    for (int i = 0; i < SEG; i++) v[i] = Cs[rr][sg * SEG + i];
    int token = a.arow ? a.arow[r] / a.arow_div : r;
    epi.template operator()<SEG>(r, token, g, n, v);
  }
}

// =======================================================================================
// RMSNorm (papernotes "Overall framework": RMSNorm on the residual stream; R1: one norm per
// depth, the stream continues from x^).  One warp per token.  The input is either the
// dtype residual x (first depth of a call) or the fp32 accumulator of the previous depth:
// inside a call the residual stream stays in fp32, it is rounded to dtype only when it
// leaves the call.
// =======================================================================================
template <typename T>
__global__ void rmsnorm_kernel(const T *x_in, const float *acc, const T *gain, T *xh,
                               float *inv_rms, int n_tok, int h, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok) return;
  float ss = 0.f;
  for (int c = lane * 8; c < h; c += 256) {
    float v[8];
    if (acc) load8(acc + (long)warp * h + c, v);
    else load8(x_in + (long)warp * h + c, v);
#pragma unroll
    for (int j = 0; j < 8; j++) ss += v[j] * v[j];
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)h + eps);
  if (lane == 0 && inv_rms) inv_rms[warp] = r;
  for (int c = lane * 8; c < h; c += 256) {
    float v[8], gv[8], o[8];
    if (acc) load8(acc + (long)warp * h + c, v);
    else load8(x_in + (long)warp * h + c, v);
    load8(gain + c, gv);
#pragma unroll
    for (int j = 0; j < 8; j++) o[j] = gv[j] * v[j] * r;
    store8(xh + (long)warp * h + c, o);
  }
}

// Combine, residual and RMSNorm fused (one warp per token): x_{l+1} = y + sum_s w_s Y_s over
// the token's k routed rows (papernotes "Key design 2": the expert outputs mixed by the
// normalised routing weights; fixed order s = 0..k-1), kept in fp32 in acc; then either the
// next depth's x^ = g x / rms(x) and 1/rms (RMSNorm on the residual stream, "Overall
// framework"), or, after the last depth, the output x_L rounded to dtype.
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) combine_norm_kernel(float *acc, const T *Y, const int *pos,
                                                          const float *wts, int k, const T *gain,
                                                          T *xh, float *inv_rms, T *x_out,
                                                          int n_tok, int h, float eps) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok) return;
  float xv[MAXV];  // this lane's 8-element chunks of the row, in fp32
  float ss = 0.f;
  long prow[16];
  float pw[16];
  for (int s = 0; s < k; s++) {
    prow[s] = (long)pos[(long)warp * k + s] * h;
    pw[s] = wts[(long)warp * k + s];
  }
#pragma unroll
  for (int ci = 0; ci < MAXV / 8; ci++) {
    const int c = ci * 256 + lane * 8;
    if (c >= h) break;
    float x[8];
    load8(acc + (long)warp * h + c, x);
    for (int s = 0; s < k; s++) {
      float yv[8];
      load8(Y + prow[s] + c, yv);
#pragma unroll
      for (int j = 0; j < 8; j++) x[j] = fmaf(pw[s], yv[j], x[j]);
    }
#pragma unroll
    for (int j = 0; j < 8; j++) {
      xv[ci * 8 + j] = x[j];
      ss += x[j] * x[j];
    }
    if (x_out) store8(x_out + (long)warp * h + c, x);
    else store8(acc + (long)warp * h + c, x);
  }
  if (x_out) return;
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)h + eps);
  if (lane == 0) inv_rms[warp] = r;
#pragma unroll
  for (int ci = 0; ci < MAXV / 8; ci++) {
    const int c = ci * 256 + lane * 8;
    if (c >= h) break;
    float gv[8], o[8];
    load8(gain + c, gv);
#pragma unroll
    for (int j = 0; j < 8; j++) o[j] = gv[j] * xv[ci * 8 + j] * r;
    store8(xh + (long)warp * h + c, o);
  }
}

// Final residual: x_L = dtype(acc).
template <typename T>
__global__ void finish_kernel(const float *acc, T *x_out, long n) {
  long i = ((long)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i >= n) return;
  float v[8];
  load8(acc + i, v);
  store8(x_out + i, v);
}

// =======================================================================================
// Attention of one query row over a run of keys (R4: scale 1/sqrt(d), fp32 softmax).
// One warp per (query, head).  Keys are processed 32 at a time: lane j scores key j of the
// chunk over all d dims, the chunk's softmax statistics are combined with warp shuffles,
// then lanes switch to owning output dims and accumulate p_j v_j.
// Used for depth attention (keys = the token's depth states 0..l), causal sequence
// attention on CUDA cores (keys = earlier tokens) and decode (keys = the SA cache).
// =======================================================================================
struct AttnArgs {
  int mode;          // 0 depth attention, 1 sequence attention (prefill), 2 decode
  int n_q, H, d, h;
  // queries
  const void *q;     // [n_q][ldq] at column head*d
  long ldq;
  // keys/values
  const void *kv;    // mode 0: da_kv [T][L][2][h]; mode 1: qkv_sa [T][3h]; mode 2: cache
  const void *vc;    // mode 2: v cache
  int L, l, S, B, cap;
  const int *cache_len;
  int *err;
  // output
  void *out;         // [n_q][ldo] at column col0 + head*d
  long ldo;
  int col0;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) attn_warp_kernel(AttnArgs a) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.n_q * a.H) return;
  const int qi = gw / a.H, head = gw % a.H;
  const T *Q = reinterpret_cast<const T *>(a.q) + (long)qi * a.ldq + head * D;
  const T *Kb, *Vb;
  long ldk;
  int nk;
  if (a.mode == 0) {
    const T *base = reinterpret_cast<const T *>(a.kv);
    Kb = base + ((long)qi * a.L * 2 + 0) * a.h + head * D;
    Vb = Kb + a.h;
    ldk = 2L * a.h;
    nk = a.l + 1;
  } else if (a.mode == 1) {
    const T *base = reinterpret_cast<const T *>(a.kv);
    const int b = qi / a.S, i = qi % a.S;
    Kb = base + ((long)b * a.S) * 3 * a.h + a.h + head * D;
    Vb = Kb + a.h;
    ldk = 3L * a.h;
    nk = i + 1;
  } else {
    const long off = ((((long)a.l * a.B + qi) * a.H + head) * a.cap) * D;
    Kb = reinterpret_cast<const T *>(a.kv) + off;
    Vb = reinterpret_cast<const T *>(a.vc) + off;
    ldk = D;
    nk = a.cache_len[qi] + 1;
    if (nk < 1 || nk > a.cap) {  // length outside the cache: report, attend to nothing
      if (lane == 0) raise_dev_error(a.err, DEV_BAD_INDEX);
      return;
    }
  }
  float q[D];
#pragma unroll
  for (int i = 0; i < D; i += 8) load8(Q + i, q + i);
  const float scale = rsqrtf((float)D);
  constexpr int DPL = (D + 31) / 32;  // output dims per lane
  float o[DPL];
#pragma unroll
  for (int i = 0; i < DPL; i++) o[i] = 0.f;
  float m = -INFINITY, lsum = 0.f;
  for (int j0 = 0; j0 < nk; j0 += 32) {
    const int j = j0 + lane;
    float s = -INFINITY;
    if (j < nk) {
      s = 0.f;
      const T *kr = Kb + (long)j * ldk;
#pragma unroll
      for (int i = 0; i < D; i += 8) {
        float kv8[8];
        load8(kr + i, kv8);
#pragma unroll
        for (int t = 0; t < 8; t++) s = fmaf(q[i + t], kv8[t], s);
      }
      s *= scale;
    }
    const float cm = warp_max(s);
    const float mn = fmaxf(m, cm);
    const float alpha = __expf(m - mn);
    const float p = (j < nk) ? __expf(s - mn) : 0.f;
    lsum = lsum * alpha + warp_sum(p);
#pragma unroll
    for (int i = 0; i < DPL; i++) o[i] *= alpha;
    const int cnt = min(32, nk - j0);
    for (int jj = 0; jj < cnt; jj++) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const T *vr = Vb + (long)(j0 + jj) * ldk;
#pragma unroll
      for (int i = 0; i < DPL; i++) {
        const int dd = lane + 32 * i;
        if (dd < D) o[i] = fmaf(pj, to_f(vr[dd]), o[i]);
      }
    }
    m = mn;
  }
  T *O = reinterpret_cast<T *>(a.out) + (long)qi * a.ldo + a.col0 + head * D;
  const float inv = 1.0f / lsum;
#pragma unroll
  for (int i = 0; i < DPL; i++) {
    const int dd = lane + 32 * i;
    if (dd < D) O[dd] = from_f<T>(o[i] * inv);
  }
}

// =======================================================================================
// Top-k over router scores (papernotes "Key design 2": sigma(x) = norm(TopK(sigmoid(x),
// x + b, k))).  One warp per token: each lane keeps its own best-k list of (z + b, e) over
// experts e = lane (mod 32); the warp then pops the global best k (ties to the lower
// index).  mode 0: expert attention (bias, weights normalised over the picks);
// mode 1: projection router (k = 1, no bias, weight sigmoid(z) kept as is).
// =======================================================================================
struct TopkArgs {
  int n_tok, E, k, mode;
  const float *z;      // [n_tok][ldz]
  long ldz;
  float zscale;        // applied to z (1/sqrt(d_r))
  const float *bias;   // [E] or null
  int *idx;            // [n_tok][k]
  float *w;            // [n_tok][k]
  int *counts_a;       // [E] histogram (may be null)
  int *counts_b;       // [E] second histogram (may be null)
};

__device__ __forceinline__ bool better(float v1, int e1, float v2, int e2) {
  return v1 > v2 || (v1 == v2 && e1 < e2);
}

__global__ void __launch_bounds__(256) topk_kernel(TopkArgs a) {
  constexpr int KMAX = 16;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.n_tok) return;
  const float *zr = a.z + (long)warp * a.ldz;
  float lv[KMAX];
  int le[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; i++) {
    lv[i] = -INFINITY;
    le[i] = 0x7fffffff;
  }
  const int k = a.k;
  for (int e = lane; e < a.E; e += 32) {
    float v = zr[e] * a.zscale + (a.bias ? a.bias[e] : 0.f);
    if (v != v) v = -INFINITY;  // a NaN score ranks last; indices stay valid
    if (!better(v, e, lv[k - 1], le[k - 1])) continue;
    // insert keeping descending order
    int p = k - 1;
    while (p > 0 && better(v, e, lv[p - 1], le[p - 1])) {
      lv[p] = lv[p - 1];
      le[p] = le[p - 1];
      p--;
    }
    lv[p] = v;
    le[p] = e;
  }
  int head = 0;
  float wsum = 0.f;
  int myidx = 0;
  float myz = 0.f;
  for (int s = 0; s < k; s++) {
    float v = head < k ? lv[head] : -INFINITY;
    int e = head < k ? le[head] : 0x7fffffff;
    // warp argmax with lower-index tie break
    float bv = v;
    int be = e;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (better(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be == e && head < k) head++;
    const float zv = zr[be] * a.zscale;
    const float sg = 1.0f / (1.0f + __expf(-zv));
    wsum += sg;
    if (lane == s) {
      myidx = be;
      myz = sg;
    }
  }
  if (lane < k) {
    a.idx[(long)warp * k + lane] = myidx;
    a.w[(long)warp * k + lane] = (a.mode == 0) ? myz / wsum : myz;
    if (a.counts_a) atomicAdd(a.counts_a + myidx, 1);
    if (a.counts_b) atomicAdd(a.counts_b + myidx, 1);
  }
}

// =======================================================================================
// Counting sort of routed slots by expert (the permutation feeding the grouped GEMMs).
// scan: offs = exclusive prefix of cnt; tile_offs = exclusive prefix of ceil(cnt/BM) for
// two tile heights; cursor = offs.  One block.
// =======================================================================================
__global__ void __launch_bounds__(1024) scan_kernel(const int *cnt, int G, int *offs,
                                                    int *tiles_a, int bm_a, int *tiles_b,
                                                    int bm_b, int *cursor) {
  __shared__ int s0[1024], s1[1024], s2[1024];
  const int tid = threadIdx.x;
  const int per = (G + 1023) / 1024;
  int a0 = 0, a1 = 0, a2 = 0;
  for (int i = 0; i < per; i++) {
    int g = tid * per + i;
    if (g < G) {
      int c = cnt[g];
      a0 += c;
      a1 += (c + bm_a - 1) / bm_a;
      a2 += (c + bm_b - 1) / bm_b;
    }
  }
  s0[tid] = a0;
  s1[tid] = a1;
  s2[tid] = a2;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    int v0 = tid >= o ? s0[tid - o] : 0;
    int v1 = tid >= o ? s1[tid - o] : 0;
    int v2 = tid >= o ? s2[tid - o] : 0;
    __syncthreads();
    s0[tid] += v0;
    s1[tid] += v1;
    s2[tid] += v2;
    __syncthreads();
  }
  int b0 = tid ? s0[tid - 1] : 0, b1 = tid ? s1[tid - 1] : 0, b2 = tid ? s2[tid - 1] : 0;
  for (int i = 0; i < per; i++) {
    int g = tid * per + i;
    if (g < G) {
      int c = cnt[g];
      offs[g] = b0;
      cursor[g] = b0;
      tiles_a[g] = b1;
      if (tiles_b) tiles_b[g] = b2;
      b0 += c;
      b1 += (c + bm_a - 1) / bm_a;
      b2 += (c + bm_b - 1) / bm_b;
    }
  }
  if (tid == 1023) {
    offs[G] = s0[1023];
    tiles_a[G] = s1[1023];
    if (tiles_b) tiles_b[G] = s2[1023];
  }
}

// rows[offs[e] + rank] = slot for every slot (token*k + j) routed to e.
__global__ void scatter_kernel(const int *idx, int n, int *cursor, int *rows, int *inv) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int p = atomicAdd(cursor + idx[i], 1);
  rows[p] = i;
  if (inv) inv[i] = p;
}

// =======================================================================================
// Bias balance update (papernotes "Key design 2"): b += lambda * sign(median(N) - N),
// N_e = sum over depths of counts[l][e]; lower median for even E.  One block, bitonic sort.
// =======================================================================================
__global__ void __launch_bounds__(1024) bias_update_kernel(const int *counts, int L, int E,
                                                           float lambda, float *bias,
                                                           float *bias_out) {
  extern __shared__ int sm[];  // [pow2 >= E] sorted copy, then [E] totals
  int n2 = 1;
  while (n2 < E) n2 <<= 1;
  int *srt = sm;
  int *tot = sm + n2;
  for (int e = threadIdx.x; e < n2; e += blockDim.x) {
    int s = 0x7fffffff;
    if (e < E) {
      s = 0;
      for (int l = 0; l < L; l++) s += counts[(long)l * E + e];
      tot[e] = s;
    }
    srt[e] = s;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        int j = i ^ stride;
        if (j > i) {
          bool up = (i & size) == 0;
          int x = srt[i], y = srt[j];
          if ((x > y) == up) {
            srt[i] = y;
            srt[j] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  const int med = srt[(E - 1) / 2];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    float sg = med > tot[e] ? 1.f : (med < tot[e] ? -1.f : 0.f);
    bias[e] += lambda * sg;
    if (bias_out) bias_out[e] = bias[e];
  }
}

// =======================================================================================
// init-time layout kernels
// =======================================================================================
// dst[g][j][i] = src[g][i][j] (+ sh[i][j]), rounded to T once (absorption, papernotes
// "Key design 3": W~ = W_p + W_shared folded after training).
template <typename T>
__global__ void transpose_absorb_kernel(const T *src, const T *sh, T *dst, int rows, int cols,
                                        int G) {
  __shared__ float tile[32][33];
  const int g = blockIdx.z;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  const T *S = src + (long)g * rows * cols;
  for (int i = threadIdx.y; i < 32; i += 8) {
    int r = r0 + i, c = c0 + threadIdx.x;
    float v = 0.f;
    if (r < rows && c < cols) {
      v = to_f(S[(long)r * cols + c]);
      if (sh) v += to_f(sh[(long)r * cols + c]);
    }
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  T *D = dst + (long)g * rows * cols;
  for (int i = threadIdx.y; i < 32; i += 8) {
    int c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) D[(long)c * rows + r] = from_f<T>(tile[threadIdx.x][i]);
  }
}

}  // namespace dreamer
