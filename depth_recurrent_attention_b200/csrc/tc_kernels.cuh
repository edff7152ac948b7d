// Host side of the tcgen05 path: tensor maps, launch shapes and the bf16 contraction steps
// of the depth step (QKV / O projections, router scores, expert FFNs).  Included by
// dreamer.cu after the handle definition.
#pragma once
#include <cuda.h>

#include "tc_attn.cuh"
#include "tc_ffn.cuh"
#include "tc_gemm.cuh"

namespace dreamer {

// Router query epilogue (papernotes "Key design 2", reading R8): the thread holds the full
// fp32 row q = y W_qE.  z_e = q . (R_l k_e) = (R_l^T q) . k_e, so the query is turned back by
// the depth rotation of depth l (k_e then enters the contraction exactly as stored, bf16) and
// split into three bf16 parts hi + mid + lo that carry q to float32 precision; the score
// contraction against [k | k | k] then runs on the tensor cores with fp32 accumulation.
// Raw router scores z [n][ldz] in fp32 (read by topk_rows_kernel), through the staged
// epilogue: a pass's 32 rows x 64 columns leave the warp as four full 128-byte lines a store.
struct EpiScoreStore {
  float *z;
  long ldz;
  static constexpr bool STAGED = true;
  using Aux = int;
  __device__ __forceinline__ int row_aux(int, int) const { return 0; }
  template <int NR>
  __device__ __forceinline__ void prefetch(const int *, const int *, const int *, int, int, int,
                                           int) const {}
  template <int SEG>
  __device__ __forceinline__ void transform(int, int, int, int, float *) const {}
  // the lane holds columns col..col+3 (v[i][0..3]) and col+32..col+35 (v[i][4..7]) of rows r[i]
  template <int NR, int NV>
  __device__ __forceinline__ void store_rows(const int *r, const int *, const int *, int, int col,
                                             const float (*v)[NV]) const {
    static_assert(NV == 8, "passes of 64 columns");
#pragma unroll
    for (int i = 0; i < NR; i++) {
      if (r[i] < 0) continue;
      float *d = z + (long)r[i] * ldz + col;
      *reinterpret_cast<float4 *>(d) = make_float4(v[i][0], v[i][1], v[i][2], v[i][3]);
      *reinterpret_cast<float4 *>(d + 32) = make_float4(v[i][4], v[i][5], v[i][6], v[i][7]);
    }
  }
};

struct EpiRouterQ {
  int dr;
  const float2 *rope;  // depth-RoPE table row of depth l over d_r dims
  bf16 *qs;            // [n][3 d_r]
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    const int q4 = SEG / 4;
#pragma unroll
    for (int half = 0; half < 2; half++) {
#pragma unroll
      for (int i = 0; i < q4; i++) {
        const float c = rope[half * q4 + i].x, s = rope[half * q4 + i].y;
        const float a = v[half * (SEG / 2) + i], b = v[half * (SEG / 2) + i + q4];
        v[half * (SEG / 2) + i] = a * c + b * s;
        v[half * (SEG / 2) + i + q4] = b * c - a * s;
      }
    }
    bf16 *row = qs + (long)r * 3 * SEG;
#pragma unroll
    for (int i = 0; i < SEG; i += 8) {
      float hi[8], mid[8], lo[8];
#pragma unroll
      for (int j = 0; j < 8; j++) {
        hi[j] = __bfloat162float(__float2bfloat16_rn(v[i + j]));
        const float r1 = v[i + j] - hi[j];
        mid[j] = __bfloat162float(__float2bfloat16_rn(r1));
        lo[j] = r1 - mid[j];
      }
      store8(row + i, hi);
      store8(row + SEG + i, mid);
      store8(row + 2 * SEG + i, lo);
    }
  }
};

// Expert-attention top-k fused into the score GEMM (row-pass epilogue): each thread owns one
// token's row, walks all E scores tile by tile and keeps its best KT by z + b (lower expert
// index on exact ties) in registers (papernotes "Key design 2": sigma(x) = norm(TopK(
// sigmoid(x), x + b, k))); at the row's end it writes the picks, the weights
// sigmoid(z) / sum over the picks, and the two histograms (per-depth counts, per-call expert
// sizes for the permutation).
template <int KT>
struct EpiTopK {
  int E;
  float zscale;
  const float *bias;
  int *idx;
  float *w;
  int *counts_a, *counts_b;
  struct State {
    float v[KT], z[KT];
    int e[KT];
  };
  __device__ __forceinline__ static bool better(float v1, int e1, float v2, int e2) {
    return v1 > v2 || (v1 == v2 && e1 < e2);
  }
  __device__ __forceinline__ void row_begin(State &s) const {
#pragma unroll
    for (int i = 0; i < KT; i++) {
      s.v[i] = -INFINITY;
      s.z[i] = 0.f;
      s.e[i] = 0x7fffffff;
    }
  }
  template <int SEG>
  __device__ __forceinline__ void row_apply(State &s, int r, int token, int g, int n0,
                                            const float *vals) const {
    // candidates against the current k-th entry first (straight-line), then one insertion
    // per qualifying candidate, picked out of the registers by a select chain (a dynamically
    // indexed array would live in local memory) and placed by an unrolled compare-and-swap
    // A row's columns arrive in increasing order, so once the list is full a candidate can
    // only tie entry KT-1 with a larger index and lose: "v > v[KT-1]" is the exact test then.
    float vb[SEG];
    unsigned mask = 0;
    const float tv = s.v[KT - 1];
    const bool open = s.e[KT - 1] == 0x7fffffff;  // the list is not full yet
    const float4 *b4 = reinterpret_cast<const float4 *>(bias + n0);
#pragma unroll
    for (int i = 0; i < SEG; i += 4) {
      const float4 bq = b4[i / 4];
      const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
      for (int u = 0; u < 4; u++) {
        const float v = fmaxf(fmaf(vals[i + u], zscale, bb[u]), -INFINITY);  // NaN ranks last
        vb[i + u] = v;
        if (open || v > tv) mask |= 1u << (i + u);
      }
    }
    while (mask) {
      const int i = __ffs(mask) - 1;
      mask &= mask - 1;
      float cv = 0.f, cz = 0.f;
#pragma unroll
      for (int j = 0; j < SEG; j++)
        if (j == i) {
          cv = vb[j];
          cz = vals[j] * zscale;
        }
      int ce = n0 + i;
      if (!better(cv, ce, s.v[KT - 1], s.e[KT - 1])) continue;
#pragma unroll
      for (int j = 0; j < KT; j++) {  // insertion by compare-and-swap down the sorted list
        if (better(cv, ce, s.v[j], s.e[j])) {
          const float tv = s.v[j], tz = s.z[j];
          const int te = s.e[j];
          s.v[j] = cv; s.z[j] = cz; s.e[j] = ce;
          cv = tv; cz = tz; ce = te;
        }
      }
    }
  }
  // Two warps a lane quarter: half 1 writes its list for row slot `slot` (0..127) into xb
  // and arrives on xfull; half 0 waits for it (bounded), inserts it into its own list (sorted,
  // so the first entry that does not qualify ends the merge), frees the slot through xempty
  // and writes the row.  rb: row blocks this pair finished before.
  __device__ __forceinline__ void row_end_pair(State &s, int r, int token, bool valid, int half,
                                               int slot, uint8_t *xb, uint64_t *xfull,
                                               uint64_t *xempty, int rb, volatile int *abort_flag,
                                               int *err) const {
    float *xv = reinterpret_cast<float *>(xb) + slot * KT;
    float *xz = reinterpret_cast<float *>(xb) + 128 * KT + slot * KT;
    int *xe = reinterpret_cast<int *>(reinterpret_cast<float *>(xb) + 256 * KT) + slot * KT;
    if (half == 1) {
      if (rb > 0 && !tc::mbar_wait(tc::smem_u32(xempty), (rb - 1) & 1, abort_flag, err)) return;
#pragma unroll
      for (int i = 0; i < KT; i++) {
        xv[i] = s.v[i];
        xz[i] = s.z[i];
        xe[i] = s.e[i];
      }
      tc::mbar_arrive(tc::smem_u32(xfull));
      return;
    }
    if (!tc::mbar_wait(tc::smem_u32(xfull), rb & 1, abort_flag, err)) return;
#pragma unroll 1
    for (int i = 0; i < KT; i++) {
      float cv = xv[i], cz = xz[i];
      int ce = xe[i];
      if (!better(cv, ce, s.v[KT - 1], s.e[KT - 1])) break;
#pragma unroll
      for (int j = 0; j < KT; j++) {
        if (better(cv, ce, s.v[j], s.e[j])) {
          const float tv = s.v[j], tz = s.z[j];
          const int te = s.e[j];
          s.v[j] = cv; s.z[j] = cz; s.e[j] = ce;
          cv = tv; cz = tz; ce = te;
        }
      }
    }
    tc::mbar_arrive(tc::smem_u32(xempty));
    if (valid) row_end(s, r, token);
  }
  __device__ __forceinline__ void row_end(State &s, int r, int token) const {
    // normalised sigmoid weights in the stable form (log_sigmoidf_)
    float sg[KT], m = -INFINITY, sum = 0.f;
#pragma unroll
    for (int i = 0; i < KT; i++) {
      sg[i] = log_sigmoidf_(s.z[i]);
      m = fmaxf(m, sg[i]);
    }
#pragma unroll
    for (int i = 0; i < KT; i++) {
      sg[i] = expf(sg[i] - m);
      sum += sg[i];
    }
    const float inv = 1.0f / sum;
#pragma unroll
    for (int i = 0; i < KT; i++) {
      idx[(long)r * KT + i] = s.e[i];
      w[(long)r * KT + i] = sg[i] * inv;
      if (counts_a) atomicAdd(counts_a + s.e[i], 1);
      if (counts_b) atomicAdd(counts_b + s.e[i], 1);
    }
  }
};

// Projection router fused into its query GEMM epilogue (papernotes "Key design 3", reading
// R12): the thread holds q_P = x^ W_qP (fp32) of its token, scores it against the P
// depth-rotated projection keys, takes the argmax (lower index on ties), sigma = sigmoid(max)
// and counts the token into its group.
struct EpiProjRoute {
  int P, dr;
  float zscale;
  const float *keys;   // [P][d_r] fp32, rotated to the current depth
  int *pidx;
  float *psig;
  int *pcount;
  template <int SEG>
  __device__ __forceinline__ void operator()(int r, int token, int g, int n0, float *v) const {
    float best = -INFINITY;
    int bi = 0;
    for (int p = 0; p < P; p++) {
      const float *kr = keys + (long)p * SEG;
      float z = 0.f;
#pragma unroll
      for (int i = 0; i < SEG; i++) z = fmaf(v[i], kr[i], z);
      z *= zscale;
      if (z > best) {  // strict: the lower index keeps ties
        best = z;
        bi = p;
      }
    }
    pidx[r] = bi;
    psig[r] = 1.0f / (1.0f + __expf(-best));
    atomicAdd(pcount + bi, 1);
  }
};

}  // namespace dreamer

typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                      const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                      const cuuint32_t *, CUtensorMapInterleave,
                                      CUtensorMapSwizzle, CUtensorMapL2promotion,
                                      CUtensorMapFloatOOBfill);
static PFN_encodeTiled_t g_encode_tiled = nullptr;

// 2-D bf16 tensor map: `rows` rows of `inner` elements at `pitch_bytes`, box box_inner x
// box_rows, swizzle = box_inner * 2 bytes (32, 64 or 128).
static bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows) {
  if (!g_encode_tiled || ((uintptr_t)base & 15) || (pitch_bytes & 15) || rows == 0) return false;
  const uint32_t sw_bytes = box_inner * 2;
  CUtensorMapSwizzle sw = sw_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : sw_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                          : sw_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                           : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (sw == CU_TENSOR_MAP_SWIZZLE_NONE) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
                              dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

static int tc_init(dreamer_handle *h) {
  const dreamer_config &c = h->cfg;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (!g_encode_tiled) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode_tiled = (PFN_encodeTiled_t)fn;
  }
  if (c.dtype == 1) {
    // [E][3 d_r] = [k | k | k] for the split-precision score contraction
    const int E = c.n_experts, dr = c.router_dim;
    if (dalloc(h, &h->k3, (size_t)E * 3 * dr * 2)) return DREAMER_ERR_OOM;
    for (int i = 0; i < 3; i++)
      if (cudaMemcpy2D((char *)h->k3 + i * dr * 2, 3 * dr * 2, h->kE_raw, dr * 2, dr * 2, E,
                       cudaMemcpyDeviceToDevice) != cudaSuccess)
        return DREAMER_ERR_CUDA;
    // [d_r][E]: the keys transposed, so that a warp scoring 64 experts reads 128-byte rows
    if (dalloc(h, &h->kEt, (size_t)E * dr * 2)) return DREAMER_ERR_OOM;
    dreamer::transpose_absorb_kernel<dreamer::bf16>
        <<<dim3((dr + 31) / 32, (E + 31) / 32, 1), dim3(32, 8)>>>(
            (const dreamer::bf16 *)h->kE_raw, nullptr, (dreamer::bf16 *)h->kEt, E, dr, 1);
    if (cudaGetLastError() != cudaSuccess) return DREAMER_ERR_CUDA;
  }
  return tc_attn_init(h);
}

static void tc_destroy(dreamer_handle *h) {}

template <int BN, int BK, int ST, int GATHER, int SEG, class Epi, bool ROWPASS = false,
          int EW = 4>
static void tc_launch(dreamer_handle *h, const dreamer::tc::TcGemmArgs &a, const CUtensorMap &ta,
                      const CUtensorMap &tb, long max_tiles, const Epi &epi, cudaStream_t s,
                      const CUtensorMap *tc = nullptr) {
  constexpr bool STG = dreamer::tc::EpiStaged<Epi>::value && !ROWPASS;
  using Cfg = dreamer::tc::TcGemmCfg<BN, BK, ST, GATHER, STG, EW, ROWPASS,
                                     dreamer::tc::EpiTma<Epi>::value && !STG && !ROWPASS>;
  auto kern = dreamer::tc::tc_gemm_kernel<BN, BK, ST, GATHER, SEG, Epi, ROWPASS, EW>;
  if (ROWPASS) max_tiles /= (a.N / BN);  // one unit of work per row tile
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    attr_set = true;
  }
  long grid = max_tiles < h->num_sms ? max_tiles : h->num_sms;
  if (grid < 1) grid = 1;
  ++g_launches_tc;
  launch_k(h, kern, dim3((unsigned)grid), dim3(Cfg::THREADS), Cfg::SMEM, s, ta, tb,
           tc ? *tc : tb, a, epi);
}

// Build engine arguments and tensor maps from the generic GEMM description.  B rows of group
// g start at g * (bgstride / ldb); A is TMA-loaded unless rows are gathered.
template <int BN, int BK>
static bool tc_prepare(dreamer_handle *h, const dreamer::GemmArgs &a, const int *tiles,
                       long a_rows, dreamer::tc::TcGemmArgs &t, CUtensorMap &ta, CUtensorMap &tb,
                       long &max_tiles) {
  if (a.N % BN || a.K % BK) return false;
  const bool gather = a.arow != nullptr && !a.a_sorted;
  const long bgr = a.G > 1 ? a.bgstride / a.ldb : 0;
  if (!make_tmap(&tb, a.B, a.K, (uint64_t)((a.G - 1) * bgr + a.N), a.ldb * 2, BK, BN)) return false;
  if (!gather) {
    if (!make_tmap(&ta, a.A, a.K, (uint64_t)a_rows, a.lda * 2, BK, 128)) return false;
  } else {
    ta = tb;  // unused
    if (((uintptr_t)a.A & 15) || (a.lda * 2) % 16) return false;
  }
  t.N = a.N; t.K = a.K; t.G = a.G; t.M = a.M;
  t.goffs = a.goffs; t.tiles = a.goffs ? tiles : nullptr;
  t.arow = a.arow; t.arow_div = a.arow_div;
  t.A = (const dreamer::bf16 *)a.A; t.lda = a.lda;
  t.b_group_rows = (int)bgr; t.b_row0 = 0;
  t.err = h->err;
  // 128-row tile table of the grouping (written by the counting sort; the expert one only
  // when the sort ran in one kernel)
  t.ttab = nullptr;
  if (a.goffs && tiles == h->etiles_b && h->cfg.n_experts <= 8192) t.ttab = h->etab;
  if (a.goffs && tiles == h->ptiles_b) t.ttab = h->ptab;
  // projections whose weights (a group's N x K) do not stay in L2 next to the streams around
  // them: raster blocks of 16 row tiles, so each B tile comes from DRAM about once
  t.mswz = (tiles != h->etiles_b && a.N / BN >= 8 && 2L * a.N * a.K >= (32L << 20)) ? 16 : 1;
  max_tiles = ((a.M + 127) / 128 + (a.goffs ? a.G : 0)) * (long)(a.N / BN);
  return true;
}

static bool tc_gemm_ok(dreamer_handle *h, const dreamer::GemmArgs &a) {
  if (!g_encode_tiled) return false;
  const int d = h->cfg.head_dim;
  return a.N % 256 == 0 && a.K % 64 == 0 && (d == 64 || d == 128);
}

// N tile of the projection GEMMs (16 to 256): the wider tile reads A fewer times, the
// narrower one spreads a small problem over more SMs; take the one with the shorter critical
// path (waves of tiles x tile width plus a fixed per-tile cost of about 32 columns).
// min_bn: 64 for epilogues that pair columns 32 apart (the QKV RoPE), else 16
static int tc_pick_bn(dreamer_handle *h, const dreamer::GemmArgs &a, int min_bn = 64) {
  const long mt = (a.M + 127) / 128 + (a.goffs ? a.G : 0);
  auto cost = [&](int bn) {
    const long tiles = mt * (a.N / bn);
    return ((tiles + h->num_sms - 1) / h->num_sms) * (bn + 32);
  };
  int best = 128;
  if (a.N % 256 == 0 && cost(256) <= cost(best)) best = 256;
  if (cost(64) < cost(best)) best = 64;  // few tiles: narrower ones reach more SMs
  // a single row tile (decode): every N tile streams its own slice of B, so narrower tiles
  // put more SMs on the weights
  if (min_bn <= 32 && a.N % 32 == 0 && cost(32) < cost(best)) best = 32;
  if (min_bn <= 16 && a.N % 16 == 0 && cost(16) < cost(best)) best = 16;
  return best;
}

template <typename T>
static bool tc_gemm_qkv(dreamer_handle *h, const dreamer::GemmArgs &a, const dreamer::EpiQKV<T> &e,
                        cudaStream_t s) {
  if constexpr (sizeof(T) == 2) {
    dreamer::tc::TcGemmArgs t{};
    CUtensorMap ta, tb;
    long mt;
    const int *tiles = h->ptiles_b;
    const bool gather = a.arow != nullptr && !a.a_sorted;
    // 64-column segments: the staged epilogue rotates pairs 32 columns apart (head dim 64,
    // or 128 in perm order).  Short K leaves little MMA time per tile to hide the epilogue
    // behind: eight epilogue warps then, at one stage less of operand ring.
    const bool ew8 = a.K <= 1024;
    const int bn = tc_pick_bn(h, a);
#ifdef DREAMER_TEST_HOOKS
    const int skip = h->inject_skip;
    h->inject_skip = 0;
#endif
    if (bn == 64) {  // one 64-column pass a tile: four epilogue warps, eight stages
      if (!tc_prepare<64, 64>(h, a, tiles, a.M, t, ta, tb, mt)) return false;
#ifdef DREAMER_TEST_HOOKS
      t.skip_loads = skip;
#endif
      if (gather) tc_launch<64, 64, 8, 2, 64>(h, t, ta, tb, mt, e, s);
      else tc_launch<64, 64, 8, 0, 64>(h, t, ta, tb, mt, e, s);
    } else if (bn == 256) {
      if (!tc_prepare<256, 64>(h, a, tiles, a.M, t, ta, tb, mt)) return false;
#ifdef DREAMER_TEST_HOOKS
      t.skip_loads = skip;
#endif
      if (ew8) {
        if (gather) tc_launch<256, 64, 3, 2, 64, EpiQKV<T>, false, 8>(h, t, ta, tb, mt, e, s);
        else tc_launch<256, 64, 3, 0, 64, EpiQKV<T>, false, 8>(h, t, ta, tb, mt, e, s);
      } else {
        if (gather) tc_launch<256, 64, 4, 2, 64>(h, t, ta, tb, mt, e, s);
        else tc_launch<256, 64, 4, 0, 64>(h, t, ta, tb, mt, e, s);
      }
    } else {
      if (!tc_prepare<128, 64>(h, a, tiles, a.M, t, ta, tb, mt)) return false;
#ifdef DREAMER_TEST_HOOKS
      t.skip_loads = skip;
#endif
      if (ew8) {
        if (gather) tc_launch<128, 64, 5, 2, 64, EpiQKV<T>, false, 8>(h, t, ta, tb, mt, e, s);
        else tc_launch<128, 64, 5, 0, 64, EpiQKV<T>, false, 8>(h, t, ta, tb, mt, e, s);
      } else {
        if (gather) tc_launch<128, 64, 6, 2, 64>(h, t, ta, tb, mt, e, s);
        else tc_launch<128, 64, 6, 0, 64>(h, t, ta, tb, mt, e, s);
      }
    }
    return true;
  }
  return false;
}

template <typename T>
static bool tc_gemm_o(dreamer_handle *h, const dreamer::GemmArgs &a, const dreamer::EpiO<T> &e,
                      cudaStream_t s) {
  if constexpr (sizeof(T) == 2) {
    dreamer::tc::TcGemmArgs t{};
    CUtensorMap ta, tb;
    long mt;
    const bool ew8 = a.K <= 1024;  // as for the QKV projection
    const int bn = tc_pick_bn(h, a, 16);
    if (bn == 16) {
      if (!tc_prepare<16, 64>(h, a, h->ptiles_b, a.M, t, ta, tb, mt)) return false;
      if (a.arow && !a.a_sorted) tc_launch<16, 64, 8, 2, 16>(h, t, ta, tb, mt, e, s);
      else tc_launch<16, 64, 8, 0, 16>(h, t, ta, tb, mt, e, s);
    } else if (bn == 32) {
      if (!tc_prepare<32, 64>(h, a, h->ptiles_b, a.M, t, ta, tb, mt)) return false;
      if (a.arow && !a.a_sorted) tc_launch<32, 64, 8, 2, 32>(h, t, ta, tb, mt, e, s);
      else tc_launch<32, 64, 8, 0, 32>(h, t, ta, tb, mt, e, s);
    } else if (bn == 64) {
      if (!tc_prepare<64, 64>(h, a, h->ptiles_b, a.M, t, ta, tb, mt)) return false;
      if (a.arow && !a.a_sorted) tc_launch<64, 64, 8, 2, 64>(h, t, ta, tb, mt, e, s);
      else tc_launch<64, 64, 8, 0, 64>(h, t, ta, tb, mt, e, s);
    } else if (bn == 256) {
      if (!tc_prepare<256, 64>(h, a, h->ptiles_b, a.M, t, ta, tb, mt)) return false;
      if (ew8) {
        if (a.arow && !a.a_sorted) tc_launch<256, 64, 3, 2, 64, EpiO<T>, false, 8>(h, t, ta, tb, mt, e, s);
        else tc_launch<256, 64, 3, 0, 64, EpiO<T>, false, 8>(h, t, ta, tb, mt, e, s);
      } else {
        if (a.arow && !a.a_sorted) tc_launch<256, 64, 4, 2, 64>(h, t, ta, tb, mt, e, s);
        else tc_launch<256, 64, 4, 0, 64>(h, t, ta, tb, mt, e, s);
      }
    } else {
      if (!tc_prepare<128, 64>(h, a, h->ptiles_b, a.M, t, ta, tb, mt)) return false;
      if (ew8) {
        if (a.arow && !a.a_sorted) tc_launch<128, 64, 5, 2, 64, EpiO<T>, false, 8>(h, t, ta, tb, mt, e, s);
        else tc_launch<128, 64, 5, 0, 64, EpiO<T>, false, 8>(h, t, ta, tb, mt, e, s);
      } else {
        if (a.arow && !a.a_sorted) tc_launch<128, 64, 6, 2, 64>(h, t, ta, tb, mt, e, s);
        else tc_launch<128, 64, 6, 0, 64>(h, t, ta, tb, mt, e, s);
      }
    }
    return true;
  }
  return false;
}

static bool tc_route(dreamer_handle *h, int l, const void *X, int n, int *idx, float *w,
                     int *counts_a, int *counts_b, cudaStream_t s) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int dr = c.router_dim, hd = c.hidden, E = c.n_experts;
  if (!g_encode_tiled || !h->k3 || !(dr == 64 || dr == 128) || hd % 64 || E % 4) return false;
  // q = X W_qE, turned back by the depth rotation and split into hi/mid/lo bf16
  GemmArgs qa{};
  qa.N = dr; qa.K = hd; qa.G = 1; qa.M = n; qa.arow_div = 1;
  qa.A = X; qa.lda = hd; qa.B = h->wqE_t; qa.ldb = hd; qa.bgstride = 0;
  tc::TcGemmArgs t{}, t2{};
  CUtensorMap ta, tb, ta2, tb2;
  long mt, mt2;
  EpiRouterQ eq{dr, h->rope_dr + (size_t)l * (dr / 2), (bf16 *)h->qsplit};
  // z = [q_hi | q_mid | q_lo] . [k | k | k]
  GemmArgs za{};
  za.N = E; za.K = 3 * dr; za.G = 1; za.M = n; za.arow_div = 1;
  za.A = h->qsplit; za.lda = 3 * dr; za.B = h->k3; za.ldb = 3 * dr; za.bgstride = 0;
  // Scores on the tensor cores (then the top k of each row, from stored scores or inside the
  // GEMM's epilogue) only when there are enough 128-row tiles to fill the GPU; otherwise a warp
  // per token scores its row from the split query on the CUDA cores, which spreads the rows
  // over every SM.
  int k_fused = (n + 127) / 128 >= h->num_sms / 2 && E % 256 == 0 ? c.top_k : 0;
  if (k_fused != 4 && k_fused != 8 && k_fused != 16) k_fused = 0;
  if (k_fused && !tc_prepare<256, 64>(h, za, nullptr, n, t2, ta2, tb2, mt2)) return false;
  if (dr == 64) {
    if (!tc_prepare<64, 64>(h, qa, nullptr, n, t, ta, tb, mt)) return false;
    tc_launch<64, 64, 6, 0, 64>(h, t, ta, tb, mt, eq, s);
  } else {
    if (!tc_prepare<128, 64>(h, qa, nullptr, n, t, ta, tb, mt)) return false;
    tc_launch<128, 64, 6, 0, 128>(h, t, ta, tb, mt, eq, s);
  }
  const float zs = 1.0f / sqrtf((float)dr);
  // Up to 2048 experts: the score GEMM stores z and a warp a token picks the top k of its row
  // (a few hundred instructions a row); beyond that the top k is kept in the GEMM's epilogue.
  const int epl = E / 32;
  if (k_fused && E % 128 == 0 && E <= 2048 && h->ldz == E) {
    tc_launch<256, 64, 4, 0, 64>(h, t2, ta2, tb2, mt2, EpiScoreStore{h->zbuf, (long)h->ldz}, s);
    TopkArgs k{};
    k.n_tok = n; k.E = E; k.k = k_fused; k.mode = 0; k.z = h->zbuf; k.ldz = h->ldz; k.zscale = zs;
    k.bias = h->bias; k.idx = idx; k.w = w; k.counts_a = counts_a; k.counts_b = counts_b;
    void (*kern)(TopkArgs) = nullptr;
#define TOPK_ROWS_CASE(KT)                                                              \
  if (k_fused == KT)                                                                    \
    kern = epl == 64 ? topk_rows_kernel<KT, 64> : epl == 32 ? topk_rows_kernel<KT, 32>  \
         : epl == 16 ? topk_rows_kernel<KT, 16> : topk_rows_kernel<KT, 8>;
    TOPK_ROWS_CASE(4)
    TOPK_ROWS_CASE(8)
    TOPK_ROWS_CASE(16)
#undef TOPK_ROWS_CASE
    long grid = ((long)n + 7) / 8;
    if (grid > 2L * h->num_sms) grid = 2L * h->num_sms;
    launch_k(h, kern, dim3((unsigned)grid), dim3(256), (size_t)E * sizeof(float), s, k);
    return true;
  }
  switch (k_fused) {  // top-k fused into the score GEMM
    case 4:
      tc_launch<256, 64, 4, 0, 32, EpiTopK<4>, true, 8>(
          h, t2, ta2, tb2, mt2, EpiTopK<4>{E, zs, h->bias, idx, w, counts_a, counts_b}, s);
      return true;
    case 8:
      tc_launch<256, 64, 4, 0, 32, EpiTopK<8>, true, 8>(
          h, t2, ta2, tb2, mt2, EpiTopK<8>{E, zs, h->bias, idx, w, counts_a, counts_b}, s);
      return true;
    case 16:
      tc_launch<256, 64, 4, 0, 32, EpiTopK<16>, true>(
          h, t2, ta2, tb2, mt2, EpiTopK<16>{E, zs, h->bias, idx, w, counts_a, counts_b}, s);
      return true;
    default:
      break;
  }
  // scores straight from the split query: two warps a token, four tokens a block (each warp's
  // expert slice a multiple of 4), or one warp a token when E is not a multiple of 8
  TopkArgs k{};
  k.n_tok = n; k.E = E; k.k = c.top_k; k.mode = 0; k.zscale = zs;
  k.bias = h->bias; k.idx = idx; k.w = w; k.counts_a = counts_a; k.counts_b = counts_b;
  if (E % 8 == 0) {
    auto kern = dr == 64 ? route_q_topk_kernel<64, 2> : route_q_topk_kernel<128, 2>;
    launch_k(h, kern, dim3((n + 3) / 4), dim3(256), 0, s, (const bf16 *)h->qsplit,
             (const bf16 *)h->kEt, k);
  } else {
    auto kern = dr == 64 ? route_q_topk_kernel<64, 1> : route_q_topk_kernel<128, 1>;
    launch_k(h, kern, dim3((n + 7) / 8), dim3(256), 0, s, (const bf16 *)h->qsplit,
             (const bf16 *)h->kEt, k);
  }
  return true;
}

// Projection router: q_P = x^ W_qP on the tensor cores, argmax over the P keys in the
// epilogue.  Needs d_r in {64, 128} (the thread holds the whole query row).
static bool tc_proj_route(dreamer_handle *h, int l, const void *X, int n, cudaStream_t s) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int dr = c.router_dim, hd = c.hidden, P = c.n_proj_experts;
  if (!g_encode_tiled || !(dr == 64 || dr == 128) || hd % 64) return false;
  GemmArgs qa{};
  qa.N = dr; qa.K = hd; qa.G = 1; qa.M = n; qa.arow_div = 1;
  qa.A = X; qa.lda = hd; qa.B = h->wqP_t; qa.ldb = hd; qa.bgstride = 0;
  tc::TcGemmArgs t{};
  CUtensorMap ta, tb;
  long mt;
  EpiProjRoute e{P, dr, 1.0f / sqrtf((float)dr), h->kP_rot + (size_t)l * P * dr, h->pidx,
                 h->psig, h->pcnt};
  if (dr == 64) {
    if (!tc_prepare<64, 64>(h, qa, nullptr, n, t, ta, tb, mt)) return false;
    tc_launch<64, 64, 6, 0, 64>(h, t, ta, tb, mt, e, s);
  } else {
    if (!tc_prepare<128, 64>(h, qa, nullptr, n, t, ta, tb, mt)) return false;
    tc_launch<128, 64, 6, 0, 128>(h, t, ta, tb, mt, e, s);
  }
  return true;
}

static bool tc_expert_ok(dreamer_handle *h) {
  const dreamer_config &c = h->cfg;
  const int m = c.expert_hidden;
  return g_encode_tiled && (m == 16 || m == 32 || m == 64) && c.hidden % 256 == 0;
}

template <int M, int ST>
static void tc_ffn_launch(dreamer_handle *h, const CUtensorMap &t1, const CUtensorMap &t2,
                          const CUtensorMap &ty, const dreamer::tc::TcFfnArgs &a,
                          long max_tiles, cudaStream_t s) {
  using Cfg = dreamer::tc::TcFfnCfg<M, ST>;
  auto kern = dreamer::tc::tc_ffn_kernel<M, ST>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    attr_set = true;
  }
  long grid = max_tiles < h->num_sms ? max_tiles : h->num_sms;
  if (grid < 1) grid = 1;
  ++g_launches_tc;
  launch_k(h, kern, dim3((unsigned)grid), dim3(Cfg::THREADS), Cfg::SMEM, s, t1, t2, ty, a);
}

// Two grouped GEMMs: H = SiLU(X_gathered W1_e) stored in sorted order, then Y = H W2_e.  The
// up-projection's rows are gathered by four cp.async warps (its epilogue is light, and with
// about one short tile per expert the gather is what bounds it).
static bool tc_expert_two(dreamer_handle *h, const void *X, int n, cudaStream_t s) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int hd = c.hidden, m = c.expert_hidden, k = c.top_k, E = c.n_experts;
  const long rows = (long)n * k;
  // up: H = SiLU(X_gathered W1_e)
  GemmArgs up{};
  up.N = m; up.K = hd; up.G = E; up.M = (int)rows; up.goffs = h->eoffs; up.tile_offs = h->etiles_b;
  up.arow = h->erows; up.arow_div = k; up.A = X; up.lda = hd; up.B = h->w1_t; up.ldb = hd;
  up.bgstride = (long)m * hd;
  // down: acc[token] += w * H W2_e
  GemmArgs dn{};
  dn.N = hd; dn.K = m; dn.G = E; dn.M = (int)rows; dn.goffs = h->eoffs; dn.tile_offs = h->etiles_b;
  dn.arow = nullptr; dn.arow_div = 1; dn.A = h->Hbuf; dn.lda = m; dn.B = h->w2_t; dn.ldb = m;
  dn.bgstride = (long)m * hd;
  tc::TcGemmArgs tu{}, td{};
  CUtensorMap tau, tbu, tad, tbd, tyd;
  long mtu, mtd;
  EpiUp<bf16> eu{m, (bf16 *)h->Hbuf};
  EpiDownStore<bf16> ed{hd, (bf16 *)h->Ybuf};
  // Y [T k + 128][h]: the down-projection's tile stores (32 rows x 64 columns a box)
  if (!make_tmap(&tyd, h->Ybuf, hd, (uint64_t)rows + 128, (uint64_t)hd * 2, 64, 32)) return false;
  switch (m) {
    case 16:
      if (!tc_prepare<16, 64>(h, up, h->etiles_b, rows, tu, tau, tbu, mtu) ||
          !tc_prepare<256, 16>(h, dn, h->etiles_b, rows + 128, td, tad, tbd, mtd))
        return false;
      tc_launch<16, 64, 8, 4, 16>(h, tu, tau, tbu, mtu, eu, s);
      tc_launch<256, 16, 8, 0, 64>(h, td, tad, tbd, mtd, ed, s, &tyd);
      return true;
    case 32:
      if (!tc_prepare<32, 64>(h, up, h->etiles_b, rows, tu, tau, tbu, mtu) ||
          !tc_prepare<256, 32>(h, dn, h->etiles_b, rows + 128, td, tad, tbd, mtd))
        return false;
      tc_launch<32, 64, 8, 4, 32>(h, tu, tau, tbu, mtu, eu, s);
      tc_launch<256, 32, 6, 0, 64>(h, td, tad, tbd, mtd, ed, s, &tyd);
      return true;
    default:
      if (!tc_prepare<64, 64>(h, up, h->etiles_b, rows, tu, tau, tbu, mtu) ||
          !tc_prepare<256, 64>(h, dn, h->etiles_b, rows + 128, td, tad, tbd, mtd))
        return false;
      tc_launch<64, 64, 8, 4, 64>(h, tu, tau, tbu, mtu, eu, s);
      tc_launch<256, 64, 4, 0, 64>(h, td, tad, tbd, mtd, ed, s, &tyd);
      return true;
  }
}

// Expert FFNs of the routed rows (sorted by expert).  The two grouped GEMMs, each spread over
// all SMs on its own tiling (the up-projection with four gather warps, the down-projection
// with TMA tile stores), are the faster form at 32, 64 and 128 rows per expert (small, large,
// medium: the medium expert stage 2.97 ms fused against 2.43 ms); the fused kernel, which keeps
// H on chip (H = SiLU(X W1_e), Y = H W2_e stored in sorted order for the combine), serves
// experts with four or more full 128-row tiles.
static bool tc_expert(dreamer_handle *h, const void *X, int n, cudaStream_t s) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int hd = c.hidden, m = c.expert_hidden, k = c.top_k, E = c.n_experts;
  const long rows = (long)n * k;
  if (rows < 512L * E) return tc_expert_two(h, X, n, s);
  if (((uintptr_t)X & 15) || (hd * 2) % 16) return false;
  // W1^T [E m][h] in blocks of m x 64; W2^T [E h][m] in chunks of 256 x m; Y [T k + 128][h]
  // in 32 x 64 store boxes
  CUtensorMap t1, t2, ty;
  if (!make_tmap(&t1, h->w1_t, hd, (uint64_t)E * m, (uint64_t)hd * 2, 64, m) ||
      !make_tmap(&t2, h->w2_t, m, (uint64_t)E * hd, (uint64_t)m * 2, m, 256) ||
      !make_tmap(&ty, h->Ybuf, hd, (uint64_t)rows + 128, (uint64_t)hd * 2, 64, 32))
    return false;
  tc::TcFfnArgs a{};
  a.H = hd; a.G = E; a.M = (int)rows; a.goffs = h->eoffs; a.tiles = h->etiles_b;
  a.arow = h->erows; a.arow_div = k; a.X = (const bf16 *)X; a.ldx = hd;
  a.Y = (bf16 *)h->Ybuf; a.err = h->err;
  a.ttab = E <= 8192 ? h->etab : nullptr;
  const long max_tiles = (rows + 127) / 128 + E;
  switch (m) {
    case 16: tc_ffn_launch<16, 6>(h, t1, t2, ty, a, max_tiles, s); return true;
    case 32: tc_ffn_launch<32, 6>(h, t1, t2, ty, a, max_tiles, s); return true;
    default: tc_ffn_launch<64, 4>(h, t1, t2, ty, a, max_tiles, s); return true;
  }
}
