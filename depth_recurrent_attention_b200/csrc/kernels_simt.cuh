// CUDA-core kernels of the Dreamer depth step.  These carry the float32 mode end to end and
// the parts of the bfloat16 mode that are not dense contractions (norm, depth attention,
// routing top-k, permutation, decode attention).
#pragma once
#include <cooperative_groups.h>

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
//
// Column order.  With perm set (head dim 128 on the tensor-core path) the q_SA and k_SA
// columns of each head come out of the GEMM in the order [0,32) [64,96) [32,64) [96,128), so
// that rotate-half partners (i, i + 64) sit 32 columns apart like every other RoPE pair;
// unperm() maps a computed column back to its head column.
template <typename T> struct EpiQKV {
  int h, d, L, l, S;
  int mode;                  // 0 prefill (position = token % S), 1 decode (position = cache_len[b])
  int col_lo;                // first column of the fused projection this GEMM computes
  int perm;                  // q_SA / k_SA column order as above
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

  __device__ __forceinline__ static int unperm(int c) {  // c in [0, 128)
    const int q = c >> 5;
    return q == 1 ? c + 32 : (q == 2 ? c - 32 : c);
  }

  // Destination of (token, column nc of the full [6h] projection in head order), or null when
  // a decode cache slot is out of range (reported by the caller).
  __device__ __forceinline__ T *dest(int token, int nc) const {
    const int blk = nc / h, head = (nc % h) / d, hc = nc % h;
    if (blk <= 2) {
      if (mode == 0 || blk == 0) return qkv_sa + (long)token * 3 * h + blk * h + hc;
      const int pos = cache_len[token];
      if (pos < 0 || pos >= cap) return nullptr;
      T *base = (blk == 1) ? k_cache : v_cache;
      return base + ((((long)l * B + token) * (h / d) + head) * cap + pos) * d + (hc % d);
    }
    if (blk == 3) return q_da + (long)token * h + hc;
    return da_kv + (((long)token * L + l) * 2 + (blk - 4)) * h + hc;
  }

  __device__ __forceinline__ int position(int token) const {  // -1: outside the cache
    if (mode == 0) return token % S;
    const int p = cache_len[token];
    return (p < 0 || p >= cap) ? -1 : p;
  }

  // Row layout (SEG = d columns of one head, in computed order): sigma only; the rotations
  // run in the coalesced layout.
  template <int SEG>
  __device__ __forceinline__ void transform(int r, int token, int g, int n0, float *v) const {
    if (psig) {
      const float s = psig[token];
#pragma unroll
      for (int i = 0; i < SEG; i++) v[i] *= s;
    }
  }

  // Coalesced layout: a pass of 64 columns inside one head; the lane holds columns col..col+3
  // (v[i][0..3]) and col+32..col+35 (v[i][4..7]) of rows r[i]; ax[i] is the row's position
  // (-1: decode slot outside the cache).
  static constexpr bool STAGED = true;
  using Aux = int;
  __device__ __forceinline__ int row_aux(int r, int token) const {
    return r < 0 ? 0 : position(token);
  }
  // the token-RoPE table rows of the tile's rows, into L2 while the tile's MMAs run
  template <int NR>
  __device__ __forceinline__ void prefetch(const int *r, const int *, const int *ax, int n0,
                                           int bn, int cj, int lpr) const {
    if ((n0 + col_lo) / h > 1) return;
    const int lines = (d / 2) * 8 / 128;
#pragma unroll
    for (int i = 0; i < NR; i++)
      if (r[i] >= 0 && ax[i] >= 0 && cj < lines)
        prefetch_l2(reinterpret_cast<const char *>(rope_tok + (long)ax[i] * (d / 2)) + cj * 128);
  }
  template <int NR, int NV>
  __device__ __forceinline__ void store_rows(const int *r, const int *tok, const int *ax, int g,
                                             int col, const float (*v)[NV]) const {
    static_assert(NV == 8, "QKV passes are 64 columns wide");
    const int nc = col + col_lo;
    const int blk = nc / h, hc = nc % h;
    const int cin = hc % d;                 // computed column inside the head (cin % 64 < 32)
    const int hd0 = hc - cin;               // first column of the head inside the block
    // token-strided destinations (everything but the decode caches): base + token * stride
    T *base = nullptr;
    long stride = 0;
    const bool cache = mode == 1 && (blk == 1 || blk == 2);
    if (blk <= 2) { base = qkv_sa + blk * h + hd0; stride = 3L * h; }
    else if (blk == 3) { base = q_da + hd0; stride = h; }
    else { base = da_kv + ((long)l * 2 + (blk - 4)) * h + hd0; stride = 2L * L * h; }
    auto row_dst = [&](int i) -> T * {  // head base of row i, or null
      if (!cache) return base + (long)tok[i] * stride;
      if (ax[i] < 0) return nullptr;
      T *cb = blk == 1 ? k_cache : v_cache;
      return cb + ((((long)l * B + tok[i]) * (h / d) + hd0 / d) * cap + ax[i]) * d;
    };
    if (blk <= 1) {
      // token RoPE: head columns o and o + d/2, frequency o; every row's table entries are
      // requested before the first store (one memory round trip a pass)
      const int o = perm ? unperm(cin) : cin;
      float4 t01[NR], t23[NR];
#pragma unroll
      for (int i = 0; i < NR; i++) {
        const float4 *cs = reinterpret_cast<const float4 *>(
            rope_tok + (long)(r[i] >= 0 && ax[i] >= 0 ? ax[i] : 0) * (d / 2) + o);
        t01[i] = __ldg(cs);
        t23[i] = __ldg(cs + 1);
      }
#pragma unroll
      for (int i = 0; i < NR; i++) {
        if (r[i] < 0) continue;
        if (ax[i] < 0) {
          raise_dev_error(err, DEV_BAD_INDEX);
          continue;
        }
        const float4 c01 = t01[i], c23 = t23[i];
        const float cc[4] = {c01.x, c01.z, c23.x, c23.z}, sn[4] = {c01.y, c01.w, c23.y, c23.w};
        float a[4], b[4];
#pragma unroll
        for (int j = 0; j < 4; j++) {
          a[j] = v[i][j] * cc[j] - v[i][4 + j] * sn[j];
          b[j] = v[i][4 + j] * cc[j] + v[i][j] * sn[j];
        }
        T *dst = row_dst(i);
        store4(dst + o, a);
        store4(dst + o + d / 2, b);
      }
      return;
    }
    if (blk == 3 || blk == 4) {
      // depth RoPE: two halves of d/2 (positions l and L-1-l), rotate-half inside each
      const float2 *tab = rope_dep + (long)l * (d / 2);
      float w[NR][8];
      if (d == 128) {
        // the pass is one half; columns col and col + 32 are partners, frequency cin % 32
        const int half = cin >> 6, f = cin & 31;
        const float4 *cs = reinterpret_cast<const float4 *>(tab + half * 32 + f);
        const float4 c01 = cs[0], c23 = cs[1];
        const float cc[4] = {c01.x, c01.z, c23.x, c23.z}, sn[4] = {c01.y, c01.w, c23.y, c23.w};
#pragma unroll
        for (int i = 0; i < NR; i++)
#pragma unroll
          for (int j = 0; j < 4; j++) {
            w[i][j] = v[i][j] * cc[j] - v[i][4 + j] * sn[j];
            w[i][4 + j] = v[i][4 + j] * cc[j] + v[i][j] * sn[j];
          }
      } else {
        // d = 64: the pass is the head; columns col (half 0) and col + 32 (half 1) each pair
        // with the column 16 away, held by lane ^ 4
        const int f = cin & 15;
        const bool first = (cin & 31) < 16;
        const float4 *c0 = reinterpret_cast<const float4 *>(tab + f);
        const float4 *c1 = reinterpret_cast<const float4 *>(tab + 16 + f);
        const float4 a01 = c0[0], a23 = c0[1], b01 = c1[0], b23 = c1[1];
        const float ca[4] = {a01.x, a01.z, a23.x, a23.z}, sa[4] = {a01.y, a01.w, a23.y, a23.w};
        const float cb[4] = {b01.x, b01.z, b23.x, b23.z}, sb[4] = {b01.y, b01.w, b23.y, b23.w};
        const float sg = first ? -1.f : 1.f;
#pragma unroll
        for (int i = 0; i < NR; i++)
#pragma unroll
          for (int j = 0; j < 4; j++) {
            const float pa = __shfl_xor_sync(0xffffffffu, v[i][j], 4);
            const float pb = __shfl_xor_sync(0xffffffffu, v[i][4 + j], 4);
            w[i][j] = v[i][j] * ca[j] + sg * pa * sa[j];
            w[i][4 + j] = v[i][4 + j] * cb[j] + sg * pb * sb[j];
          }
      }
#pragma unroll
      for (int i = 0; i < NR; i++) {
        if (r[i] < 0) continue;
        T *dst = base + (long)tok[i] * stride + cin;
        store4(dst, w[i]);
        store4(dst + 32, w[i] + 4);
      }
      return;
    }
#pragma unroll
    for (int i = 0; i < NR; i++) {  // v_SA, v_DA: as they are
      if (r[i] < 0) continue;
      T *dst = row_dst(i);
      if (!dst) {
        raise_dev_error(err, DEV_BAD_INDEX);
        continue;
      }
      store4(dst + cin, v[i]);
      store4(dst + cin + 32, v[i] + 4);
    }
  }

  // CUDA-core engine: one row's SEG = d columns of one head at once, in computed order.
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    static_assert(SEG % 16 == 0, "segment");
    const int nc = n0 + col_lo;        // column of the full [6h] projection
    const int blk = nc / h;            // 0 qSA 1 kSA 2 vSA 3 qDA 4 kDA 5 vDA
    if (psig) {
      const float s = psig[token];
#pragma unroll
      for (int i = 0; i < SEG; i++) v[i] *= s;
    }
    if (SEG == 128 && perm && blk <= 1) {  // back to head order (the permutation swaps
#pragma unroll                             // the middle two 32-column blocks)
      for (int i = 32; i < 64; i++) {
        const float t = v[i];
        v[i] = v[i + 32];
        v[i + 32] = t;
      }
    }
    if (mode == 1 && blk <= 2 && position(token) < 0) {  // slot outside the cache
      raise_dev_error(err, DEV_BAD_INDEX);
      return;
    }
    if (blk <= 1) {  // token RoPE, rotate-half over d (pair i, i + d/2)
      const float2 *cs = rope_tok + (long)position(token) * (d / 2);
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
    T *dst = dest(token, n0 + col_lo);
    if (!dst) return;
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

  static constexpr bool STAGED = true;
  template <int SEG>
  __device__ __forceinline__ void transform(int, int, int, int, float *) const {}
  struct Aux {
    float s, ir;  // sigma and 1/rms of the row's token
  };
  __device__ __forceinline__ Aux row_aux(int r, int token) const {
    if (r < 0) return Aux{0.f, 0.f};
    return Aux{psig ? psig[token] : 1.0f, res_mode == 2 ? 1.f : inv_rms[token]};
  }
  // the residual rows of the tile, into L2 while the tile's MMAs run
  template <int NR>
  __device__ __forceinline__ void prefetch(const int *r, const int *tok, const Aux *, int n0,
                                           int bn, int cj, int lpr) const {
    const bool from_x = res_mode == 0;
    const int lines = bn * (from_x ? (int)sizeof(T) : 4) / 128;
#pragma unroll
    for (int i = 0; i < NR; i++) {
      if (r[i] < 0) continue;
      const char *row = from_x ? reinterpret_cast<const char *>(xin + (long)tok[i] * h + n0)
                               : reinterpret_cast<const char *>(acc + (long)tok[i] * h + n0);
      for (int ln = cj; ln < lines; ln += lpr) prefetch_l2(row + ln * 128);
    }
  }
  // Coalesced layout (NV values a lane and row: 4 at col, and with NV = 8 four more at
  // col + 32); every row's residual loads are issued before the first store.
  template <int NR, int NV>
  __device__ __forceinline__ void store_rows(const int *r, const int *tok, const Aux *ax, int g,
                                             int col, const float (*v)[NV]) const {
    float gv[NV];
#pragma unroll
    for (int hh = 0; hh < NV / 4; hh++) {
      if (res_mode != 2) load4(gain + col + 32 * hh, gv + 4 * hh);
      else gv[4 * hh] = gv[4 * hh + 1] = gv[4 * hh + 2] = gv[4 * hh + 3] = 1.f;
    }
    constexpr int GR = NR;
#pragma unroll
    for (int i0 = 0; i0 < NR; i0 += GR) {
      float xr[GR][NV];
#pragma unroll
      for (int i = 0; i < GR; i++) {
        if (r[i0 + i] < 0) continue;
#pragma unroll
        for (int hh = 0; hh < NV / 4; hh++) {
          const long off = (long)tok[i0 + i] * h + col + 32 * hh;
          if (res_mode == 0) load4(xin + off, xr[i] + 4 * hh);
          else load4(acc + off, xr[i] + 4 * hh);
        }
      }
#pragma unroll
      for (int i = 0; i < GR; i++) {
        if (r[i0 + i] < 0) continue;
        const float s = ax[i0 + i].s, ir = ax[i0 + i].ir;
        float o[NV];
#pragma unroll
        for (int j = 0; j < NV; j++)
          o[j] = (res_mode == 2 ? xr[i][j] : gv[j] * xr[i][j] * ir) + s * v[i0 + i][j];
#pragma unroll
        for (int hh = 0; hh < NV / 4; hh++) {
          const long off = (long)tok[i0 + i] * h + col + 32 * hh;
          if (y) store4(y + off, o + 4 * hh);
          store4(acc + off, o + 4 * hh);
        }
      }
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

// Expert down-projection epilogue, store form: the routed row's expert output Y (sorted row
// r) is written once in dtype; the weighted sum over a token's k rows happens in
// combine_norm_kernel (no atomics, fixed summation order).
template <typename T> struct EpiDownStore {
  static constexpr bool TMA_STORE = true;  // tcgen05 engine: tile stores through a tensor map
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
    float *p = C + (long)r * ldc + n0;
    if (n0 + SEG <= N && (ldc & 3) == 0) {
#pragma unroll
      for (int i = 0; i < SEG; i += 4) store4(p + i, v + i);
    } else {
#pragma unroll
      for (int i = 0; i < SEG; i++)
        if (n0 + i < N) p[i] = v[i];
    }
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
  int a_sorted;           // tcgen05 engine: A is already in sorted-row order (TMA tiles);
                          // arow then only maps rows to tokens for the epilogue
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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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

// Expert FFN of single routed rows, for batches with few rows per expert (decode): one CTA
// per routed slot (token t, slot s) computes Y[t k + s] = SiLU(x_t W1_e) W2_e for its expert
// e (papernotes "Key design 2": each expert is a small SiLU FFN), reading the expert's two
// weight blocks once; no sorting by expert is needed.  The hidden activations are rounded to
// dtype as the grouped path stores them.  w1t: [E][M][h], w2t: [E][h][M] (K contiguous).
template <typename T, int M>
__global__ void __launch_bounds__(256) expert_rows_kernel(const T *X, const int *eidx,
                                                          int nslots, int k, int h,
                                                          const T *w1t, const T *w2t, T *Y) {
  pdl_wait();
  pdl_trigger();
  constexpr int XC = 8;  // 16-byte x chunks a lane covers (h <= 2048)
  // the row x in shared memory as fp32 (in registers it would take 64 a thread and cap the
  // CTAs an SM holds at two)
  __shared__ __align__(16) float xs[XC * 256];
  __shared__ float hs[M];
  const int slot = blockIdx.x;
  if (slot >= nslots) return;
  const int e = eidx[slot], tok = slot / k;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T *x = X + (long)tok * h;
  const T *W1 = w1t + (long)e * M * h;
  const T *W2 = w2t + (long)e * h * M;
  for (int i = threadIdx.x * 8; i < h; i += 256 * 8) {
    float xv[8];
    load8(x + i, xv);
    *reinterpret_cast<float4 *>(xs + i) = make_float4(xv[0], xv[1], xv[2], xv[3]);
    *reinterpret_cast<float4 *>(xs + i + 4) = make_float4(xv[4], xv[5], xv[6], xv[7]);
  }
  __syncthreads();
  // up: one hidden unit a warp at a time, two in flight
#pragma unroll 2
  for (int jj = 0; jj < M / 8; jj++) {
    const int j = warp + 8 * jj;
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < XC; t++) {
      const int i = t * 256 + lane * 8;
      if (i < h) {
        float wv[8];
        load8(W1 + (long)j * h + i, wv);
        const float4 x0 = *reinterpret_cast<const float4 *>(xs + i);
        const float4 x1 = *reinterpret_cast<const float4 *>(xs + i + 4);
        a = fmaf(x0.x, wv[0], a); a = fmaf(x0.y, wv[1], a);
        a = fmaf(x0.z, wv[2], a); a = fmaf(x0.w, wv[3], a);
        a = fmaf(x1.x, wv[4], a); a = fmaf(x1.y, wv[5], a);
        a = fmaf(x1.z, wv[6], a); a = fmaf(x1.w, wv[7], a);
      }
    }
    a = warp_sum(a);
    if (lane == 0) hs[j] = to_f(from_f<T>(a / (1.0f + __expf(-a))));
  }
  __syncthreads();
#pragma unroll 4
  for (int c = threadIdx.x; c < h; c += blockDim.x) {  // down: one output column a thread
    const T *w = W2 + (long)c * M;
    float a = 0.f;
#pragma unroll
    for (int j = 0; j < M; j += 8) {
      float wv[8];
      load8(w + j, wv);
#pragma unroll
      for (int q = 0; q < 8; q++) a = fmaf(hs[j + q], wv[q], a);
    }
    Y[(long)slot * h + c] = from_f<T>(a);
  }
}

// Combine, residual and RMSNorm fused (one warp per token): x_{l+1} = y + sum_s w_s Y_s over
// the token's k routed rows (papernotes "Key design 2": the expert outputs mixed by the
// normalised routing weights; fixed order s = 0..k-1), kept in fp32 in acc; then either the
// next depth's x^ = g x / rms(x) and 1/rms (RMSNorm on the residual stream, "Overall
// framework"), or, after the last depth, the output x_L rounded to dtype.
template <typename T, int MAXV>
__global__ void __launch_bounds__(256, 4) combine_norm_kernel(float *acc, const T *Y, const int *pos,
                                                          const float *wts, int k, const T *gain,
                                                          T *xh, float *inv_rms, T *x_out,
                                                          int n_tok, int h, float eps,
                                                          int *zero_a, int na, int *zero_b,
                                                          int nb) {
  pdl_wait();
  pdl_trigger();
  {  // the depth's grouping counters, cleared for the next depth (nothing reads them now)
    const int t = blockIdx.x * blockDim.x + threadIdx.x, nt = gridDim.x * blockDim.x;
    for (int i = t; i < na; i += nt) zero_a[i] = 0;
    for (int i = t; i < nb; i += nt) zero_b[i] = 0;
  }
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_tok) return;
  // slot s's row in Y (its sorted position, or the slot itself when pos == null) and weight,
  // held by lane s (k <= 16) and passed round by shuffles
  const long slot0 = (long)warp * k;
  long my_row = 0;
  float my_w = 0.f;
  if (lane < k) {
    my_row = (pos ? (long)pos[slot0 + lane] : slot0 + lane) * h;
    my_w = wts[slot0 + lane];
  }
  float ss = 0.f;
#pragma unroll 1
  for (int ci = 0; ci < MAXV / 8; ci++) {
    if (ci * 256 >= h) break;  // uniform across the warp
    const int c = ci * 256 + lane * 8;
    const bool on = c < h;
    float x[8];
    if (on) load8(acc + (long)warp * h + c, x);
    // four slot rows requested before any is used; the sum runs over s = 0..k-1 in order
    for (int s0 = 0; s0 < k; s0 += 4) {
      float yv[4][8];
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const long pr = __shfl_sync(0xffffffffu, my_row, (s0 + u) & 31);
        if (on && s0 + u < k) load8(Y + pr + c, yv[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const float pw = __shfl_sync(0xffffffffu, my_w, (s0 + u) & 31);
        if (on && s0 + u < k) {
#pragma unroll
          for (int j = 0; j < 8; j++) x[j] = fmaf(pw, yv[u][j], x[j]);
        }
      }
    }
    if (on) {
#pragma unroll
      for (int j = 0; j < 8; j++) ss += x[j] * x[j];
      // the accumulator always keeps x_{l+1} in fp32 (the last depth also stores it rounded)
      if (x_out) store8(x_out + (long)warp * h + c, x);
      store8(acc + (long)warp * h + c, x);
    }
  }
  if (x_out) return;
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)h + eps);
  if (lane == 0) inv_rms[warp] = r;
  // the next depth's x^ from the row just stored (this thread's own writes, still in L1/L2):
  // the row is not kept in registers, so more warps fit on an SM to hide the slot loads
#pragma unroll 1
  for (int ci = 0; ci < MAXV / 8; ci++) {
    const int c = ci * 256 + lane * 8;
    if (c >= h) break;
    float gv[8], xr[8], o[8];
    load8(gain + c, gv);
    load8(acc + (long)warp * h + c, xr);
#pragma unroll
    for (int j = 0; j < 8; j++) o[j] = gv[j] * xr[j] * r;
    store8(xh + (long)warp * h + c, o);
  }
}

// The same combine for bf16 with one CTA per token and h / 8 threads (8 elements each): every
// thread requests its acc chunk and all k <= KMAX slot chunks (16-byte loads, kept packed)
// before the first use, so a token costs one memory round trip; the sum over the slots runs in the same
// fixed order s = 0..k-1, and the row's squares are reduced over the CTA for the next norm.
template <int KMAX>
__global__ void __launch_bounds__(512) combine_norm_row_kernel(
    float *acc, const bf16 *Y, const int *pos, const float *wts, int k, const bf16 *gain,
    bf16 *xh, float *inv_rms, bf16 *x_out, int n_tok, int h, float eps, int *zero_a, int na,
    int *zero_b, int nb) {
  pdl_wait();
  pdl_trigger();
  {  // the depth's grouping counters, cleared for the next depth (nothing reads them now)
    const int t = blockIdx.x * blockDim.x + threadIdx.x, nt = gridDim.x * blockDim.x;
    for (int i = t; i < na; i += nt) zero_a[i] = 0;
    for (int i = t; i < nb; i += nt) zero_b[i] = 0;
  }
  __shared__ long srow[16];
  __shared__ float sw[16];
  __shared__ float red[32];
  const int tok = blockIdx.x;
  const long slot0 = (long)tok * k;
  if (threadIdx.x < k) {
    srow[threadIdx.x] = (pos ? (long)pos[slot0 + threadIdx.x] : slot0 + threadIdx.x) * h;
    sw[threadIdx.x] = wts[slot0 + threadIdx.x];
  }
  __syncthreads();
  const int c = threadIdx.x * 8;
  float x[8];
  load8(acc + (long)tok * h + c, x);
  uint4 yv[KMAX];
#pragma unroll
  for (int s = 0; s < KMAX; s++)
    if (s < k) yv[s] = *reinterpret_cast<const uint4 *>(Y + srow[s] + c);
#pragma unroll
  for (int s = 0; s < KMAX; s++) {
    if (s < k) {
      const float pw = sw[s];
      const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&yv[s]);
#pragma unroll
      for (int i = 0; i < 4; i++) {
        const float2 f = __bfloat1622float2(h2[i]);
        x[2 * i] = fmaf(pw, f.x, x[2 * i]);
        x[2 * i + 1] = fmaf(pw, f.y, x[2 * i + 1]);
      }
    }
  }
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < 8; j++) ss += x[j] * x[j];
  // the accumulator always keeps x_{l+1} in fp32 (the last depth also stores it rounded)
  if (x_out) store8(x_out + (long)tok * h + c, x);
  store8(acc + (long)tok * h + c, x);
  if (x_out) return;  // uniform over the CTA
  ss = warp_sum(ss);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (lane == 0) red[wid] = ss;
  __syncthreads();
  float tot = lane < nw ? red[lane] : 0.f;
  tot = warp_sum(tot);
  const float r = rsqrtf(tot / (float)h + eps);
  if (threadIdx.x == 0) inv_rms[tok] = r;
  float gv[8], o[8];
  load8(gain + c, gv);
#pragma unroll
  for (int j = 0; j < 8; j++) o[j] = gv[j] * x[j] * r;
  store8(xh + (long)tok * h + c, o);
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
  pdl_wait();
  pdl_trigger();
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

// Running top k (k <= 32) of one warp, distributed over its lanes: lane j holds the j-th best
// (biased score v, expert e, raw score z).  The first 32 candidates are sorted by a warp
// bitonic network; later ones that beat entry k-1 are inserted by a ballot for the position and
// a one-lane shift.  No per-lane arrays, nothing in local memory.  Order: higher v first, the
// lower expert index on ties; a NaN score ranks last.
struct WarpTopK {
  static constexpr unsigned FULL = 0xffffffffu;
  static constexpr int NONE = 0x7fffffff;
  int k, lane;
  bool started = false;
  float lv = -INFINITY, lz = 0.f, tv = -INFINITY;
  int le = NONE, te = NONE;
  __device__ WarpTopK(int k_, int lane_) : k(k_), lane(lane_) {}
  __device__ __forceinline__ void threshold() {
    tv = __shfl_sync(FULL, lv, k - 1);
    te = __shfl_sync(FULL, le, k - 1);
  }
  __device__ __forceinline__ void insert(float cv, int ce, float cz) {
    const int pos = __popc(__ballot_sync(FULL, lane < k && better(lv, le, cv, ce)));
    const float uv = __shfl_up_sync(FULL, lv, 1), uz = __shfl_up_sync(FULL, lz, 1);
    const int ue = __shfl_up_sync(FULL, le, 1);
    if (lane > pos) {
      lv = uv; lz = uz; le = ue;
    } else if (lane == pos) {
      lv = cv; lz = cz; le = ce;
    }
    threshold();
  }
  // the first batch: sort the warp's 32 candidates (descending) and keep the best k
  __device__ __forceinline__ void start(float v, int e, float z) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const float ov = __shfl_xor_sync(FULL, v, stride), oz = __shfl_xor_sync(FULL, z, stride);
        const int oe = __shfl_xor_sync(FULL, e, stride);
        const bool desc = (lane & size) == 0 || size == 32;
        const bool lower = (lane & stride) == 0;
        const bool mine = better(v, e, ov, oe);
        if ((lower == desc) != mine) {
          v = ov; e = oe; z = oz;
        }
      }
    }
    lv = lane < k ? v : -INFINITY;
    le = lane < k ? e : NONE;
    lz = z;
    started = true;
    threshold();
  }
  // one candidate a lane (e == NONE: none); warp-uniform call
  __device__ __forceinline__ void offer(float v, int e, float z) {
    if (!started) {
      start(v, e, z);
      return;
    }
    unsigned m = __ballot_sync(FULL, e != NONE && better(v, e, tv, te));
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      const float cv = __shfl_sync(FULL, v, src), cz = __shfl_sync(FULL, z, src);
      const int ce = __shfl_sync(FULL, e, src);
      if (better(cv, ce, tv, te)) insert(cv, ce, cz);
    }
  }
  // the candidate of expert e with raw score z (already scaled)
  __device__ __forceinline__ void offer_score(float z, int e, bool valid, const float *bias) {
    float v = -INFINITY;
    if (valid) {
      v = z + (bias ? bias[e] : 0.f);
      if (v != v) v = -INFINITY;
    }
    offer(v, valid ? e : NONE, z);
  }
};

// Lanes < k of a warp write the k picks (descending), their weights (sigmoid of the raw score,
// normalised over the k in mode 0) and count them.
__device__ __forceinline__ void emit_topk(int lane, int k, float v, int e, float z, long tok,
                                          int mode, int *idx, float *w, int *ca, int *cb) {
  // mode 0: normalised routing weights (stable form); mode 1: the projection weight sigmoid(z)
  const float ls = lane < k ? log_sigmoidf_(z) : -INFINITY;
  const float m = warp_max(ls);
  const float ex = lane < k ? expf(ls - m) : 0.f;
  const float ssum = warp_sum(ex);
  if (lane < k) {
    idx[tok * k + lane] = e;
    w[tok * k + lane] = mode == 0 ? ex / ssum : 1.0f / (1.0f + expf(-z));
    if (ca) atomicAdd(ca + e, 1);
    if (cb) atomicAdd(cb + e, 1);
  }
}

// Candidates as one ordered 64-bit key: larger key = better (higher biased score, then the
// lower expert index); 0 = no candidate.  -0 counts as +0, as in better().
__device__ __forceinline__ unsigned long long topk_key(float v, int e) {
  if (e == WarpTopK::NONE) return 0ull;
  if (v == 0.f) v = 0.f;
  unsigned u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)u << 32) | (unsigned)(~e);
}
__device__ __forceinline__ int topk_key_expert(unsigned long long key) {
  return (int)(~(unsigned)(key & 0xffffffffull));
}

// Top k of n listed candidates (keys, raw scores; distinct experts) by rank counting: the
// threads of the block each rank one entry against all n (no serial chain) and write the k
// best to out[rank].  Ends with a block barrier.
__device__ __forceinline__ void rank_select(const unsigned long long *key, const float *z, int n,
                                            int k, unsigned long long *okey, float *oz) {
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const unsigned long long ki = key[i];
    if (ki == 0ull) continue;
    int r = 0;
    for (int j = 0; j < n; j++) r += key[j] > ki ? 1 : 0;
    if (r < k) {
      okey[r] = ki;
      oz[r] = z[i];
    }
  }
  __syncthreads();
}

// Top-k of stored raw router scores, one warp a token, E = 32 EPL experts (EPL a multiple of
// 4, at most 64): lane j holds experts 4j..4j+3 of every 128 (float4 loads) as biased scores
// v = fma(z, zscale, b) (NaN ranks last).  The k-th largest of the 32 lane maxima is at most
// the k-th largest v, so only values at or above it can be picks: when there are at most 32
// such candidates (the usual case) the warp sorts them once (bitonic, by better(): higher v,
// then the lower index); otherwise it takes k rounds of a warp-wide best.  Either way the
// picks and their order are those of a full sort.  The weights are emit_topk's, from the
// picks' scaled raw scores.
template <int KT, int EPL>
__global__ void __launch_bounds__(256, 2) topk_rows_kernel(TopkArgs a) {
  pdl_wait();
  pdl_trigger();
  static_assert(EPL % 4 == 0 && EPL <= 64 && KT <= 32, "experts a lane");
  constexpr unsigned FULL = 0xffffffffu;
  constexpr int NONE = WarpTopK::NONE, NJ = EPL / 4;
  extern __shared__ float bsh[];  // bias [E]
  __shared__ float cvs[8][32];
  __shared__ int ces[8][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < a.E; i += blockDim.x) bsh[i] = a.bias ? a.bias[i] : 0.f;
  __syncthreads();
  for (long tok = (long)blockIdx.x * 8 + wib; tok < a.n_tok; tok += (long)gridDim.x * 8) {
    const float4 *src = reinterpret_cast<const float4 *>(a.z + tok * a.ldz);
    float v[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int j = 0; j < NJ; j++) {
      const float4 q = src[j * 32 + lane];
      const int c = (j * 32 + lane) * 4;
      v[4 * j] = fmaxf(fmaf(q.x, a.zscale, bsh[c]), -INFINITY);
      v[4 * j + 1] = fmaxf(fmaf(q.y, a.zscale, bsh[c + 1]), -INFINITY);
      v[4 * j + 2] = fmaxf(fmaf(q.z, a.zscale, bsh[c + 2]), -INFINITY);
      v[4 * j + 3] = fmaxf(fmaf(q.w, a.zscale, bsh[c + 3]), -INFINITY);
      mx = max3f(mx, fmaxf(v[4 * j], v[4 * j + 1]), fmaxf(v[4 * j + 2], v[4 * j + 3]));
    }
    // the KT-th largest lane maximum: bitonic sort of the 32 maxima, descending
    float sm = mx;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const float o = __shfl_xor_sync(FULL, sm, stride);
        const bool desc = (lane & size) == 0 || size == 32;
        const bool lower = (lane & stride) == 0;
        sm = (lower == desc) ? fmaxf(sm, o) : fminf(sm, o);
      }
    }
    const float tau = __shfl_sync(FULL, sm, KT - 1);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < EPL; i++) cnt += v[i] >= tau ? 1 : 0;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(FULL, incl, o);
      if (lane >= o) incl += t;
    }
    const int C = __shfl_sync(FULL, incl, 31);
    float bv = -INFINITY;
    int be = NONE;
    if (C <= 32) {
      int off = incl - cnt;
#pragma unroll
      for (int i = 0; i < EPL; i++)
        if (v[i] >= tau) {
          cvs[wib][off] = v[i];
          ces[wib][off] = ((i >> 2) * 32 + lane) * 4 + (i & 3);
          off++;
        }
      __syncwarp();
      float cv = lane < C ? cvs[wib][lane] : -INFINITY;
      int ce = lane < C ? ces[wib][lane] : NONE;
      __syncwarp();  // the lists are read before the next token writes them
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const float ov = __shfl_xor_sync(FULL, cv, stride);
          const int oe = __shfl_xor_sync(FULL, ce, stride);
          const bool desc = (lane & size) == 0 || size == 32;
          const bool lower = (lane & stride) == 0;
          if ((lower == desc) != better(cv, ce, ov, oe)) {
            cv = ov;
            ce = oe;
          }
        }
      }
      bv = cv;
      be = ce;
    } else {
      // many values tied at the bound: KT rounds of the warp-wide best not yet taken
      unsigned long long taken = 0ull;
#pragma unroll 1
      for (int t = 0; t < KT; t++) {
        float lv = -INFINITY;
        int le = NONE, li = -1;
#pragma unroll
        for (int i = 0; i < EPL; i++) {
          const int e = ((i >> 2) * 32 + lane) * 4 + (i & 3);
          if (!((taken >> i) & 1ull) && better(v[i], e, lv, le)) {
            lv = v[i];
            le = e;
            li = i;
          }
        }
        float wv = lv;
        int we = le;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float ov = __shfl_xor_sync(FULL, wv, o);
          const int oe = __shfl_xor_sync(FULL, we, o);
          if (better(ov, oe, wv, we)) {
            wv = ov;
            we = oe;
          }
        }
        if (li >= 0 && we == le) taken |= 1ull << li;  // the owner marks its pick
        if (lane == t) {
          bv = wv;
          be = we;
        }
      }
    }
    const float z = (lane < KT && be != NONE) ? a.z[tok * a.ldz + be] * a.zscale : 0.f;
    emit_topk(lane, KT, bv, be, z, tok, 0, a.idx, a.w, a.counts_a, a.counts_b);
  }
}

// Top-k of stored scores z (one token's row of E), WPT warps a token; each warp scans a slice
// of the experts 32 at a time, then the block ranks the WPT lists.
template <int WPT>
__global__ void __launch_bounds__(256) topk_kernel(TopkArgs a) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long mk[WPT * 32], fk[32];
  __shared__ float mz[WPT * 32], fz[32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int tok = WPT == 1 ? blockIdx.x * 8 + wib : blockIdx.x;
  if (tok >= a.n_tok) return;  // whole warp (WPT 1) or whole block (WPT > 1)
  const float *zr = a.z + (long)tok * a.ldz;
  WarpTopK t(a.k, lane);
  const int per = (a.E + WPT - 1) / WPT;
  const int e0 = WPT > 1 ? wib * per : 0, e1 = WPT > 1 ? min(a.E, e0 + per) : a.E;
  for (int b = e0; b < e1; b += 32) {
    const int e = b + lane;
    t.offer_score(e < e1 ? zr[e] * a.zscale : 0.f, e, e < e1, a.bias);
  }
  if (WPT == 1) {
    emit_topk(lane, a.k, t.lv, t.le, t.lz, tok, a.mode, a.idx, a.w, a.counts_a, a.counts_b);
    return;
  }
  if (lane < a.k) {  // the warps' lists, compacted
    mk[wib * a.k + lane] = topk_key(t.lv, t.le);
    mz[wib * a.k + lane] = t.lz;
  }
  __syncthreads();
  rank_select(mk, mz, WPT * a.k, a.k, fk, fz);
  if (wib == 0)
    emit_topk(lane, a.k, 0.f, lane < a.k ? topk_key_expert(fk[lane]) : 0, fz[lane], tok, a.mode,
              a.idx, a.w, a.counts_a, a.counts_b);
}

// Scores and top-k from a stored router query, WPT warps a token: q arrives as the three bf16
// parts q_hi + q_mid + q_lo of R_l^T q (the split the tensor-core query GEMM writes), the
// keys unrotated and transposed [d_r][E].  The token's warps sum the parts once into shared
// memory; warp w of the token then scores the experts of its slice [w E/WPT, (w+1) E/WPT),
// lane j taking experts b + 4j .. b + 4j + 3 of each batch of 128 (one 256-byte row read a key
// dimension, shared through L1 by the block's warps; four independent sums a lane),
// z_e = q . k_e in fp32 summed in dimension order, and keeps the slice's top k; the token's
// first warp ranks the WPT lists.  For batches too short to fill the GPU with fused score
// tiles.  E a multiple of 4 WPT.
template <int DR, int WPT>
__global__ void __launch_bounds__(256, 3) route_q_topk_kernel(const bf16 *qs3, const bf16 *kt,
                                                           TopkArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int TPB = 8 / WPT;  // tokens a block
  __shared__ __align__(16) float qsh[TPB][DR];
  __shared__ unsigned long long mk[TPB][WPT * 32], ok[TPB][32];
  __shared__ float mz[TPB][WPT * 32], oz[TPB][32];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int g = wib / WPT, w = wib % WPT;  // token of the block, warp of the token
  const long tok = (long)blockIdx.x * TPB + g;
  const bool live = tok < a.n_tok;
  for (int j = w * 32 + lane; j < DR; j += WPT * 32) {
    float v = 0.f;
    if (live) {
      const bf16 *qr = qs3 + tok * 3 * DR + j;
      v = (to_f(qr[0]) + to_f(qr[DR])) + to_f(qr[2 * DR]);
    }
    qsh[g][j] = v;
  }
  __syncthreads();
  WarpTopK t(a.k, lane);
  if (live) {
    const int per = a.E / WPT, e0 = w * per, e1 = e0 + per;
    for (int b = e0; b < e1; b += 128) {
      const int e = b + 4 * lane;
      float z[4] = {0.f, 0.f, 0.f, 0.f};
      if (e < e1) {
        const bf16 *kc = kt + e;
#pragma unroll
        for (int j = 0; j < DR; j += 4) {
          const float4 q4 = *reinterpret_cast<const float4 *>(&qsh[g][j]);
          const float qj[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
          for (int jj = 0; jj < 4; jj++) {
            const uint2 u = *reinterpret_cast<const uint2 *>(kc + (long)(j + jj) * a.E);
            const float2 f0 =
                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
            const float2 f1 =
                __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
            z[0] = fmaf(qj[jj], f0.x, z[0]);
            z[1] = fmaf(qj[jj], f0.y, z[1]);
            z[2] = fmaf(qj[jj], f1.x, z[2]);
            z[3] = fmaf(qj[jj], f1.y, z[3]);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; u++) t.offer_score(z[u] * a.zscale, e + u, e + u < e1, a.bias);
    }
  }
  if (WPT == 1) {
    if (live) emit_topk(lane, a.k, t.lv, t.le, t.lz, tok, a.mode, a.idx, a.w, a.counts_a, a.counts_b);
    return;
  }
  if (lane < a.k) {  // the warps' lists, compacted
    mk[g][w * a.k + lane] = topk_key(t.lv, t.le);
    mz[g][w * a.k + lane] = t.lz;
  }
  __syncthreads();
  if (w != 0 || !live) return;
  const int nc = WPT * a.k;  // rank every listed candidate against all (distinct experts)
  for (int i = lane; i < nc; i += 32) {
    const unsigned long long ki = mk[g][i];
    if (ki == 0ull) continue;
    int r = 0;
    for (int c = 0; c < nc; c++) r += mk[g][c] > ki ? 1 : 0;
    if (r < a.k) {
      ok[g][r] = ki;
      oz[g][r] = mz[g][i];
    }
  }
  __syncwarp();
  emit_topk(lane, a.k, 0.f, lane < a.k ? topk_key_expert(ok[g][lane]) : 0,
            lane < a.k ? oz[g][lane] : 0.f, tok, a.mode, a.idx, a.w, a.counts_a, a.counts_b);
}

// Routing of few tokens (decode): a cluster of NCL CTAs per token (papernotes "Key design 2":
// router query, sigmoid scores against depth-RoPE'd expert keys, biased top-k).  Each CTA
// computes DR/NCL entries of the query q = y W_q (fp32), the cluster gathers q through
// distributed shared memory and turns it back by the depth rotation (q . R_l k = R_l^T q . k),
// each CTA scores its slice of the experts against the unrotated keys and ranks its warps'
// lists, and CTA 0 ranks the NCL lists read from its peers' shared memory.  wqt: W_q
// transposed [d_r][h]; kraw: [E][d_r]; rope: the router dim's depth-RoPE row of this depth.
template <typename T, int DR>
__global__ void __launch_bounds__(256, 4) route_cluster_kernel(const T *y, int h, const T *wqt,
                                                               const T *kraw, const float2 *rope,
                                                               TopkArgs a) {
  pdl_wait();
  pdl_trigger();
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int ncl = (int)cl.num_blocks(), rank = (int)cl.block_rank();
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const int tok = blockIdx.x / ncl;  // the same for the whole cluster
  __shared__ __align__(16) float qpart[DR], qv[DR];
  __shared__ unsigned long long mk[256], fk[32];
  __shared__ float mz[256], fz[32];
  const bool live = tok < a.n_tok;
  const int qn = DR / ncl;
  if (live) {
    const T *yr = y + (long)tok * h;
    for (int j = rank * qn + wib; j < (rank + 1) * qn; j += 8) {
      float acc = 0.f;
#pragma unroll 4
      for (int i = lane * 8; i < h; i += 256) {
        float yv[8], wv[8];
        load8(yr + i, yv);
        load8(wqt + (long)j * h + i, wv);
#pragma unroll
        for (int u = 0; u < 8; u++) acc = fmaf(yv[u], wv[u], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) qpart[j] = acc;
    }
  }
  cl.sync();
  if (threadIdx.x < DR) qv[threadIdx.x] = *cl.map_shared_rank(qpart + threadIdx.x, threadIdx.x / qn);
  __syncthreads();
  if (threadIdx.x < DR / 2) {  // R_l^T: pairs (i, i + d_r/4) inside each half
    const int q4 = DR / 4, half = threadIdx.x / q4, i = threadIdx.x % q4;
    const int ia = half * (DR / 2) + i, ib = ia + q4;
    const float c = rope[half * q4 + i].x, sn = rope[half * q4 + i].y;
    const float va = qv[ia], vb = qv[ib];
    qv[ia] = va * c + vb * sn;
    qv[ib] = vb * c - va * sn;
  }
  __syncthreads();
  WarpTopK t(a.k, lane);
  if (live) {
    // q stays in shared memory (every lane reads the same words): as registers it would
    // take DR of them a thread and halve the CTAs an SM holds
    const float4 *q4 = reinterpret_cast<const float4 *>(qv);
    const int per_cta = (a.E + ncl - 1) / ncl;
    const int c0 = rank * per_cta, c1 = min(a.E, c0 + per_cta);
    const int per_w = (c1 - c0 + 7) / 8;
    const int e0 = c0 + wib * per_w, e1 = min(c1, e0 + per_w);
    for (int b = e0; b < e1; b += 32) {
      const int e = b + lane;
      float z = 0.f;
      if (e < e1) {
        const T *kr = kraw + (long)e * DR;
#pragma unroll 4
        for (int j = 0; j < DR; j += 8) {
          float kv[8];
          load8(kr + j, kv);
          const float4 qa = q4[j / 4], qb = q4[j / 4 + 1];
          z = fmaf(qa.x, kv[0], z); z = fmaf(qa.y, kv[1], z);
          z = fmaf(qa.z, kv[2], z); z = fmaf(qa.w, kv[3], z);
          z = fmaf(qb.x, kv[4], z); z = fmaf(qb.y, kv[5], z);
          z = fmaf(qb.z, kv[6], z); z = fmaf(qb.w, kv[7], z);
        }
      }
      t.offer_score(z * a.zscale, e, e < e1, a.bias);
    }
  }
  if (lane < a.k) {  // the warps' lists, compacted
    mk[wib * a.k + lane] = topk_key(t.lv, t.le);
    mz[wib * a.k + lane] = t.lz;
  }
  if (threadIdx.x < 32) fk[threadIdx.x] = 0ull;
  __syncthreads();
  rank_select(mk, mz, 8 * a.k, a.k, fk, fz);  // this CTA's best k in fk / fz
  cl.sync();
  if (rank == 0) {  // gather the cluster's lists and rank them again
    for (int i = threadIdx.x; i < ncl * a.k; i += blockDim.x) {
      const int r = i / a.k, j = i % a.k;
      mk[i] = *cl.map_shared_rank(fk + j, r);
      mz[i] = *cl.map_shared_rank(fz + j, r);
    }
  }
  cl.sync();  // peers' lists read; they may exit
  if (rank == 0) {
    __syncthreads();
    rank_select(mk, mz, ncl * a.k, a.k, fk, fz);
    if (live && wib == 0)
      emit_topk(lane, a.k, 0.f, lane < a.k ? topk_key_expert(fk[lane]) : 0, fz[lane], tok,
                a.mode, a.idx, a.w, a.counts_a, a.counts_b);
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
  pdl_wait();
  pdl_trigger();
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

// Counting sort in one kernel (G <= 8192 groups): every CTA scans the group counts into its
// shared memory (exclusive prefix), CTA 0 also publishes offs and the row-tile prefixes for
// the grouped GEMMs, and each thread places one item: rows[offs[g] + rank] = i, inv[i] = that
// position, the rank within the group taken from ctr[g] (zero on entry; the order inside a
// group is not fixed, every row is computed on its own).
__global__ void __launch_bounds__(1024) permute_kernel(const int *cnt, int G, const int *idx,
                                                       int n, int *offs, int *tiles_a, int bm_a,
                                                       int *tiles_b, int bm_b, int *ctr, int *rows,
                                                       int *inv, int2 *ttab_b) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int so[];  // [G + 1]
  __shared__ int w0[32], w1[32], w2[32];
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const bool pub = blockIdx.x == 0;
  const int per = (G + 1023) / 1024;
  int a0 = 0, a1 = 0, a2 = 0;
  for (int i = 0; i < per; i++) {
    const int g = tid * per + i;
    if (g < G) {
      const int c = cnt[g];
      a0 += c;
      a1 += (c + bm_a - 1) / bm_a;
      a2 += (c + bm_b - 1) / bm_b;
    }
  }
  // exclusive prefix of the three per-thread sums: warp shuffles, then the warp totals
  int i0 = a0, i1 = a1, i2 = a2;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v0 = __shfl_up_sync(0xffffffffu, i0, o), v1 = __shfl_up_sync(0xffffffffu, i1, o);
    const int v2 = __shfl_up_sync(0xffffffffu, i2, o);
    if (lane >= o) {
      i0 += v0;
      i1 += v1;
      i2 += v2;
    }
  }
  if (lane == 31) {
    w0[wid] = i0;
    w1[wid] = i1;
    w2[wid] = i2;
  }
  __syncthreads();
  if (wid == 0) {
    int t0 = w0[lane], t1 = w1[lane], t2 = w2[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v0 = __shfl_up_sync(0xffffffffu, t0, o), v1 = __shfl_up_sync(0xffffffffu, t1, o);
      const int v2 = __shfl_up_sync(0xffffffffu, t2, o);
      if (lane >= o) {
        t0 += v0;
        t1 += v1;
        t2 += v2;
      }
    }
    w0[lane] = t0;  // inclusive prefix of the warp totals
    w1[lane] = t1;
    w2[lane] = t2;
  }
  __syncthreads();
  int b0 = i0 - a0 + (wid ? w0[wid - 1] : 0);
  int b1 = i1 - a1 + (wid ? w1[wid - 1] : 0);
  int b2 = i2 - a2 + (wid ? w2[wid - 1] : 0);
  for (int i = 0; i < per; i++) {
    const int g = tid * per + i;
    if (g < G) {
      const int c = cnt[g];
      so[g] = b0;
      if (pub) {
        offs[g] = b0;
        tiles_a[g] = b1;
        if (tiles_b) tiles_b[g] = b2;
        // the group's bm_b-row tiles: (group, first row | rows << 24), so a GEMM finds a tile's
        // rows with one load instead of a search over the tile offsets
        if (ttab_b)
          for (int t = 0; t * bm_b < c; t++) {
            const int r0 = b0 + t * bm_b, nr = min(bm_b, c - t * bm_b);
            ttab_b[b2 + t] = make_int2(g, (int)((unsigned)r0 | ((unsigned)nr << 24)));
          }
      }
      b0 += c;
      b1 += (c + bm_a - 1) / bm_a;
      b2 += (c + bm_b - 1) / bm_b;
    }
  }
  if (tid == 1023 && pub) {
    offs[G] = w0[31];
    tiles_a[G] = w1[31];
    if (tiles_b) tiles_b[G] = w2[31];
  }
  __syncthreads();
  const int i = blockIdx.x * 1024 + tid;
  if (i < n) {
    const int g = idx[i];
    const int p = so[g] + atomicAdd(ctr + g, 1);
    rows[p] = i;
    if (inv) inv[i] = p;
  }
}

// dst[r] = src[rows[r]] for r < n, rows of h bf16: the normalised states in the order of the
// projection experts' groups, so that the grouped QKV projection loads its A tiles with TMA.
// A CTA copies four rows at a time, its threads taking the rows' 16-byte chunks, so a thread
// keeps four independent loads in flight (one at a time left most of HBM idle).
__global__ void gather_rows_kernel(const bf16 *src, const int *rows, bf16 *dst, int n, int h) {
  pdl_wait();
  pdl_trigger();
  constexpr int RB = 4;
  const int cpr = h / 8;
  for (int r0 = blockIdx.x * RB; r0 < n; r0 += gridDim.x * RB) {
    const bf16 *sr[RB];
#pragma unroll
    for (int u = 0; u < RB; u++) sr[u] = r0 + u < n ? src + (long)rows[r0 + u] * h : nullptr;
    for (int c = threadIdx.x; c < cpr; c += blockDim.x) {
      uint4 v[RB];
#pragma unroll
      for (int u = 0; u < RB; u++)
        if (sr[u]) v[u] = *reinterpret_cast<const uint4 *>(sr[u] + c * 8);
#pragma unroll
      for (int u = 0; u < RB; u++)
        if (sr[u]) *reinterpret_cast<uint4 *>(dst + (long)(r0 + u) * h + c * 8) = v[u];
    }
  }
}

// rows[offs[e] + rank] = slot for every slot (token*k + j) routed to e.
__global__ void scatter_kernel(const int *idx, int n, int *cursor, int *rows, int *inv) {
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
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
// Column order of the tensor-core QKV GEMM for head dim 128: in the transposed weight
// [G][6h][h], swap rows [32, 64) and [64, 96) of every 128-row head of q_SA and k_SA (the
// EpiQKV perm order).  One thread per swapped element pair.
template <typename T>
__global__ void perm_qk_rows_kernel(T *w, int h, int G) {
  const int nh = h / 128;
  const long total = (long)G * 2 * nh * 32 * h;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long)gridDim.x * blockDim.x) {
    const int k = (int)(i % h);
    long t = i / h;
    const int r = (int)(t % 32);
    t /= 32;
    const int head = (int)(t % nh);
    t /= nh;
    const int blk = (int)(t % 2), g = (int)(t / 2);
    T *base = w + ((long)g * 6 * h + blk * h + head * 128) * h;
    T *a = base + (long)(32 + r) * h + k, *b = base + (long)(64 + r) * h + k;
    const T x = *a;
    *a = *b;
    *b = x;
  }
}

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

// =======================================================================================
// Balance summary of the route counts (f2 of the bias balance): the Lorenz curve of the
// per-expert totals N_e (sorted ascending, cumulative share at 0, 1/E, .., 1) and the Gini
// coefficient from it, G = 1 - (1/E) sum_i (L_{i-1} + L_i).  N_e = counts[depth][e], or the
// sum over depths for depth < 0.  One block; bitonic sort in shared memory; sums in double.
// All-zero counts give the diagonal and G = 0.
// =======================================================================================
__global__ void __launch_bounds__(1024) balance_kernel(const int *counts, int L, int E,
                                                       int depth, float *lorenz, float *gini) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int srt[];  // [pow2 >= E]
  __shared__ double part[1024];
  const int tid = threadIdx.x;
  int n2 = 1;
  while (n2 < E) n2 <<= 1;
  for (int e = tid; e < n2; e += blockDim.x) {
    int v = 0x7fffffff;
    if (e < E) {
      if (depth >= 0) {
        v = counts[(long)depth * E + e];
      } else {
        v = 0;
        for (int l = 0; l < L; l++) v += counts[(long)l * E + e];
      }
    }
    srt[e] = v;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < n2; i += blockDim.x) {
        const int j = i ^ stride;
        if (j > i) {
          const bool up = (i & size) == 0;
          const int x = srt[i], y = srt[j];
          if ((x > y) == up) {
            srt[i] = y;
            srt[j] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  // prefix sums: thread tid owns sorted entries [i0, i0 + per)
  const int per = (E + 1023) / 1024, i0 = tid * per;
  double loc = 0.0;
  for (int i = i0; i < i0 + per && i < E; i++) loc += (double)srt[i];
  part[tid] = loc;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const double v = tid >= o ? part[tid - o] : 0.0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  const double total = part[1023];
  double acc = tid ? part[tid - 1] : 0.0, tsum = 0.0;
  for (int i = i0; i < i0 + per && i < E; i++) {
    const double prev = acc;
    acc += (double)srt[i];
    if (lorenz) lorenz[i + 1] = total > 0.0 ? (float)(acc / total) : (float)(i + 1) / (float)E;
    tsum += prev + acc;
  }
  if (tid == 0 && lorenz) lorenz[0] = 0.f;
  __syncthreads();
  part[tid] = tsum;
  __syncthreads();
  for (int o = 512; o > 0; o >>= 1) {
    if (tid < o) part[tid] += part[tid + o];
    __syncthreads();
  }
  if (tid == 0) *gini = total > 0.0 ? (float)(1.0 - part[0] / ((double)E * total)) : 0.f;
}

}  // namespace dreamer
