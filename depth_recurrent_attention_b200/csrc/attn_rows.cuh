// Attention of one query row over a run of key/value rows, HBM-bound forms (bf16 / fp32).
// Used for depth attention (the token's own depth states 0..l; papernotes "Key design 1":
// DA looks back over the token's earlier depth states) and for decode attention over the
// per-depth SA cache (split over key ranges, then merged).
//
// Layout of the work inside a warp: a key row of D elements is CH = D / VEC chunks of 16
// bytes; lane = r * CH + c owns chunk c of row r of a group of RPW = 32 / CH rows.  A warp
// issues U groups of K and V loads (2U independent 16-byte loads per lane) before using any
// of them, reduces the partial dot products over the CH lanes of a row with shuffles, keeps an
// online softmax over groups, and reduces the output chunks over the RPW rows at the end.
#pragma once
#include <type_traits>
#include "common.cuh"

namespace dreamer {

template <typename T> struct VecOf;
template <> struct VecOf<bf16> { static constexpr int N = 8; };
template <> struct VecOf<float> { static constexpr int N = 4; };

__device__ __forceinline__ void ld16(const bf16 *p, float *o) { load8(p, o); }
__device__ __forceinline__ void ld16(const float *p, float *o) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
}
__device__ __forceinline__ void st16(bf16 *p, const float *v) { store8(p, v); }
__device__ __forceinline__ void st16(float *p, const float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

struct RowsArgs {
  int mode;            // 0 depth attention, 2 decode attention (split)
  int n_q, H, h, L, l;
  int r0;              // mode 0: first depth attended (0, or l-W+1 with a window of W)
  const void *q;       // [n_q][ldq], head at column head * D
  long ldq;
  const void *kv;      // mode 0: da_kv [T][L][2][h]; mode 2: k cache [L][B][H][cap][D]
  const void *vc;      // mode 2: v cache
  int B, cap, nsplit;
  const int *cache_len;
  int *err;
  void *out;           // mode 0: attn [n_q][ldo] at column col0 + head * D
  long ldo;
  int col0;
  float *part;         // mode 2: [n_q][H][nsplit][D + 2] partial (o, m, l)
  const int *out_rows; // mode 0: output row of token t (grouped projections), or null: t
};

template <typename T, int D, int U>
__global__ void __launch_bounds__(256) attn_rows_kernel(RowsArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int VEC = VecOf<T>::N;
  constexpr int CH = D / VEC;
  static_assert(CH >= 1 && CH <= 32 && (32 % CH) == 0, "chunking");
  constexpr int RPW = 32 / CH;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int c = lane % CH, r = lane / CH;
  if (gw >= a.n_q * a.H) return;
  const int qi = gw / a.H, head = gw % a.H;
  const T *Kb = reinterpret_cast<const T *>(a.kv) + ((long)qi * a.L * 2) * a.h + head * D;
  const T *Vb = Kb + a.h;
  const long ldk = 2L * a.h;
  const int j0 = a.r0, j1 = a.l + 1;
  float q[VEC];
  ld16(reinterpret_cast<const T *>(a.q) + (long)qi * a.ldq + head * D + c * VEC, q);
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);
#pragma unroll
  for (int i = 0; i < VEC; i++) q[i] *= sl2;  // scores in log2 units

  float m = -INFINITY, lsum = 0.f;
  float o[VEC];
#pragma unroll
  for (int i = 0; i < VEC; i++) o[i] = 0.f;

  for (int g = j0; g < j1; g += U * RPW) {
    float kv[U][VEC], vv[U][VEC];
    bool ok[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      const int j = g + u * RPW + r;
      ok[u] = j < j1;
      if (ok[u]) {
        ld16(Kb + (long)j * ldk + c * VEC, kv[u]);
        ld16(Vb + (long)j * ldk + c * VEC, vv[u]);
      }
    }
    float s[U];
#pragma unroll
    for (int u = 0; u < U; u++) {
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; i++) p = fmaf(q[i], ok[u] ? kv[u][i] : 0.f, p);
#pragma unroll
      for (int o2 = 1; o2 < CH; o2 <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o2);
      s[u] = ok[u] ? p : -INFINITY;
    }
    float gm = s[0];
#pragma unroll
    for (int u = 1; u < U; u++) gm = fmaxf(gm, s[u]);
    gm = warp_max(gm);
    const float mn = fmaxf(m, gm);
    const float alpha = exp2f(m - mn);
    float ps = 0.f;
#pragma unroll
    for (int i = 0; i < VEC; i++) o[i] *= alpha;
#pragma unroll
    for (int u = 0; u < U; u++) {
      const float p = ok[u] ? exp2f(s[u] - mn) : 0.f;
      ps += p;
#pragma unroll
      for (int i = 0; i < VEC; i++) o[i] = fmaf(p, ok[u] ? vv[u][i] : 0.f, o[i]);
    }
    // row sums: each row's p sits on its CH lanes, count it once
    ps = warp_sum(c == 0 ? ps : 0.f);
    lsum = lsum * alpha + ps;
    m = mn;
  }
  // reduce the output chunks over the RPW rows of the warp
#pragma unroll
  for (int o2 = CH; o2 < 32; o2 <<= 1)
#pragma unroll
    for (int i = 0; i < VEC; i++) o[i] += __shfl_xor_sync(0xffffffffu, o[i], o2);
  if (r == 0) {
    const float inv = 1.0f / lsum;
#pragma unroll
    for (int i = 0; i < VEC; i++) o[i] *= inv;
    st16(reinterpret_cast<T *>(a.out) + (long)qi * a.ldo + a.col0 + head * D + c * VEC, o);
  }
}

// Merge the split partials of decode attention: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_merge_kernel(RowsArgs a) {
  pdl_wait();
  pdl_trigger();
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.n_q * a.H) return;
  const int qi = gw / a.H, head = gw % a.H;
  const float *pp = a.part + (long)gw * a.nsplit * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; s++) M = fmaxf(M, pp[s * (D + 2) + D]);
  float den = 0.f;
  constexpr int PER = (D + 31) / 32;
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; i++) acc[i] = 0.f;
  for (int s = 0; s < a.nsplit; s++) {
    const float ms = pp[s * (D + 2) + D];
    if (ms == -INFINITY) continue;  // empty split
    const float f = exp2f(ms - M);
    den += f * pp[s * (D + 2) + D + 1];
#pragma unroll
    for (int i = 0; i < PER; i++) {
      const int dd = lane + 32 * i;
      if (dd < D) acc[i] = fmaf(f, pp[s * (D + 2) + dd], acc[i]);
    }
  }
  T *dst = reinterpret_cast<T *>(a.out) + (long)qi * a.ldo + a.col0 + head * D;
  const float inv = 1.0f / den;
#pragma unroll
  for (int i = 0; i < PER; i++) {
    const int dd = lane + 32 * i;
    if (dd < D) dst[dd] = from_f<T>(acc[i] * inv);
  }
}


// =======================================================================================
// Depth attention as one stream per CTA: a token's depth KV rows 0..l for all heads are one
// contiguous run of the [T][L][2][h] buffer ((l + 1) * 2h elements).  A CTA takes the tokens
// blockIdx.x, blockIdx.x + gridDim.x, ... and cuts each run into chunks of CHUNK depths; the
// (token, chunk) items form one sequence that thread 0 streams into an NB-deep ring of
// shared-memory buffers with 1-D bulk copies (the token's query row rides with its first
// chunk), so the copies of the next token overlap the arithmetic of this one.  Warp `head`
// attends over its head's slice of every row in the row-group layout of the kernels above
// (papernotes "Key design 1": DA attends over the same token's states at depths 0..l).
// =======================================================================================
namespace tcda {
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
}  // namespace tcda

struct DaBulkArgs {
  int n_tok, H, h, L, l, chunk;  // chunk: depths per shared-memory buffer
  int r0;                        // first depth attended (0, or l-W+1 with a window of W)
  const void *q;                 // q_DA [T][h]
  const void *kv;                // [T][L][2][h]
  void *out;                     // attn [T][ldo], DA part at column col0
  long ldo;
  int col0;
  int *err;
  const int *out_rows;           // output row of token t (grouped projections), or null: t
};

// NB chunk buffers: 2 (two CTAs share an SM) or 4 (a CTA owns its SM: the launch beside SA
// gives depth attention a set of whole SMs, and more chunks in flight per SM).
template <typename T, int D, int NB>
__global__ void __launch_bounds__(1024) da_bulk_kernel(DaBulkArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ __align__(8) uint64_t bars[NB];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrow = a.l + 1 - a.r0;                     // depths r0..l
  const int nch = (nrow + a.chunk - 1) / a.chunk;
  const long row_el = 2L * a.h;                        // elements of one depth row (K then V)
  const uint32_t chunk_bytes = (uint32_t)(a.chunk * row_el * sizeof(T));
  const uint32_t q_bytes = (uint32_t)(a.h * sizeof(T));
  const int ntok = a.n_tok > (int)blockIdx.x ? (a.n_tok - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nitems = ntok * nch;
  if (nitems == 0) return;  // the whole CTA
  auto kv_slot = [&](int b) { return dsm + (size_t)b * chunk_bytes; };
  auto q_slot = [&](int b) { return dsm + (size_t)NB * chunk_bytes + (size_t)b * q_bytes; };
  if (threadIdx.x == 0) {
    for (int i = 0; i < NB; i++)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tcda::smem_u32(&bars[i])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  auto issue = [&](int j) {
    const int b = j % NB, c = j % nch;
    const int tok = (int)blockIdx.x + (j / nch) * (int)gridDim.x;
    const int r0 = c * a.chunk, nr = min(a.chunk, nrow - r0);
    const uint32_t kvb = (uint32_t)(nr * row_el * sizeof(T));
    const uint32_t bar = tcda::smem_u32(&bars[b]);
    const uint32_t total = kvb + (c == 0 ? q_bytes : 0u);
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(total)
                 : "memory");
    tcda::bulk_load(tcda::smem_u32(kv_slot(b)),
                    reinterpret_cast<const T *>(a.kv) + ((long)tok * a.L + a.r0 + r0) * row_el,
                    kvb, bar);
    if (c == 0)
      tcda::bulk_load(tcda::smem_u32(q_slot(b)), reinterpret_cast<const T *>(a.q) + (long)tok * a.h,
                      q_bytes, bar);
  };
  int issued = 0;  // items issued (thread 0's count)
  if (threadIdx.x == 0)
    for (; issued < NB && issued < nitems; issued++) issue(issued);
  // row-group layout: CH lanes of 16 bytes cover a row, RPW rows per warp step
  constexpr int VEC = VecOf<T>::N;
  constexpr int CH = D / VEC;
  constexpr int RPW = 32 / CH;
  constexpr int U = 2;  // row groups per iteration (one max / sum reduction for U * RPW rows)
  const int cc = lane % CH, rr = lane / CH;
  const int head = warp;
  const bool active = head < a.H;
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);
  float q[VEC], o[VEC];
  float m = -INFINITY, lsum = 0.f;
  int consumed = 0;
  for (int j = 0; j < nitems; j++) {
    const int b = j % NB, c = j % nch;
    const uint32_t bar = tcda::smem_u32(&bars[b]);
    const uint32_t par = (uint32_t)((j / NB) & 1);
    if (!tcda::try_wait(bar, par)) {  // bounded; on expiry every thread stops after the barrier
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(bar, par)) {
        if (abort_flag) break;
        if (tcda::gtimer() - t0 > DREAMER_WAIT_LIMIT_NS) {
          abort_flag = 1;
          raise_dev_error(a.err, DEV_TIMEOUT);
          break;
        }
      }
    }
    if (!abort_flag) consumed = j + 1;
    const T *bk = reinterpret_cast<const T *>(kv_slot(b));  // stale after a timeout; nothing is stored then
    const int nr = min(a.chunk, nrow - c * a.chunk);
    if (active) {
      if (c == 0) {  // a new token: its query, a fresh softmax
        ld16(reinterpret_cast<const T *>(q_slot(b)) + head * D + cc * VEC, q);
#pragma unroll
        for (int i = 0; i < VEC; i++) {
          q[i] *= sl2;
          o[i] = 0.f;
        }
        m = -INFINITY;
        lsum = 0.f;
      }
      for (int g = 0; g < nr; g += U * RPW) {
        float s[U], vv[U][VEC];
#pragma unroll
        for (int u = 0; u < U; u++) {
          const int jr = g + u * RPW + rr;
          s[u] = -INFINITY;
          if (jr < nr) {
            float kv[VEC];
            const T *kr = bk + (long)jr * row_el + head * D + cc * VEC;
            ld16(kr, kv);
            ld16(kr + a.h, vv[u]);
            float p = 0.f;
#pragma unroll
            for (int i = 0; i < VEC; i++) p = fmaf(q[i], kv[i], p);
            s[u] = p;
          } else {
#pragma unroll
            for (int i = 0; i < VEC; i++) vv[u][i] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < U; u++) {
          float p = s[u] == -INFINITY ? 0.f : s[u];
#pragma unroll
          for (int o2 = 1; o2 < CH; o2 <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o2);
          if (s[u] != -INFINITY) s[u] = p;
        }
        float gm = s[0];
#pragma unroll
        for (int u = 1; u < U; u++) gm = fmaxf(gm, s[u]);
        gm = warp_max(gm);
        const float mn = fmaxf(m, gm);
        const float alpha = exp2f(m - mn);
        float ps = 0.f;
#pragma unroll
        for (int i = 0; i < VEC; i++) o[i] *= alpha;
#pragma unroll
        for (int u = 0; u < U; u++) {
          const float p = s[u] == -INFINITY ? 0.f : exp2f(s[u] - mn);
          ps += p;
#pragma unroll
          for (int i = 0; i < VEC; i++) o[i] = fmaf(p, vv[u][i], o[i]);
        }
        ps = warp_sum(cc == 0 ? ps : 0.f);
        lsum = lsum * alpha + ps;
        m = mn;
      }
      if (c == nch - 1) {  // the token's last chunk: fold the RPW rows, normalise, store
        float of[VEC];
#pragma unroll
        for (int i = 0; i < VEC; i++) of[i] = o[i];
#pragma unroll
        for (int o2 = CH; o2 < 32; o2 <<= 1)
#pragma unroll
          for (int i = 0; i < VEC; i++) of[i] += __shfl_xor_sync(0xffffffffu, of[i], o2);
        if (rr == 0 && !abort_flag) {
          const int tok = (int)blockIdx.x + (j / nch) * (int)gridDim.x;
          const float inv = 1.0f / lsum;
#pragma unroll
          for (int i = 0; i < VEC; i++) of[i] *= inv;
          const long orow = a.out_rows ? a.out_rows[tok] : tok;
          st16(reinterpret_cast<T *>(a.out) + orow * a.ldo + a.col0 + head * D + cc * VEC, of);
        }
      }
    }
    __syncthreads();        // buffer b is free again
    if (abort_flag) break;  // read after the barrier: the same decision in every thread
    if (threadIdx.x == 0 && issued < nitems) {
      issue(issued);
      issued++;
    }
  }
  // copies still in flight after an abort land before the CTA exits
  if (threadIdx.x == 0 && abort_flag) {
    for (int j = consumed; j < issued; j++) {
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(tcda::smem_u32(&bars[j % NB]), (uint32_t)((j / NB) & 1)) &&
             tcda::gtimer() - t0 < DREAMER_WAIT_LIMIT_NS) {
      }
    }
  }
}

// =======================================================================================
// Depth attention for bf16 and head dims 64 / 128, fewer instructions per streamed byte: the
// same (token, chunk) stream of bulk copies as da_bulk_kernel (three buffers, one CTA an SM),
// with the rows of a chunk taken in batches of 8.  A warp (one head) splits a row into CH =
// D / 8 lanes of 8 elements and its 32 lanes into G = 32 / CH groups; lane (g, c) forms the
// partial dot products of its chunk c with the NR = 8 / G rows of group g, and one transposed
// butterfly (log2 NR halving exchanges, then plain ones) leaves every row's full score in
// CH / NR lanes with NR - 1 + log2(CH / NR) shuffles for the batch instead of log2(CH) a row.
// The q.k products take the bf16 pairs as they are (fma.rn.f32.bf16: bf16 inputs, fp32
// accumulate, each product exact); the V accumulation uses packed fp32 pairs
// (fma.rn.f32x2) with V widened by a shift or a mask.  One online-softmax update a batch (max
// and sum by warp shuffles); each lane then fetches the NR weights of its group's rows and
// accumulates the V rows into its 8 output elements; the G groups' partial outputs are
// summed at the token's last chunk.  Batches with all 8 rows present (every one but a
// chunk's last partial batch) run without per-row checks: the kernel is bound by the
// instructions a streamed byte costs, and the checks' branches were a sixth of them.
// (papernotes "Key design 1": attention over the token's own states at depths 0..l.)
// =======================================================================================
namespace tcda {
// packed fp32 pairs: {lo, hi} in one 64-bit register
__device__ __forceinline__ uint64_t pk2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 up2(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
// two bf16 of one 32-bit word as an fp32 pair (low element, high element)
// acc + a.lo * b.lo + a.hi * b.hi for bf16 pairs a, b: mixed-precision FMAs (bf16 inputs,
// fp32 accumulate; each product is exact in fp32)
__device__ __forceinline__ float dot2_bf16(uint32_t a, uint32_t b, float acc) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;\n\tfma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
      : "+f"(acc)
      : "r"(a), "r"(b));
  return acc;
}
__device__ __forceinline__ uint64_t bf2_to_f2(uint32_t w) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w << 16), "r"(w & 0xffff0000u));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
}  // namespace tcda

template <int D>
__global__ void __launch_bounds__(1024) da_fast_kernel(DaBulkArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int NB = 3;
  constexpr int CH = D / 8, G = 32 / CH, NR = 8 / G, DUP = CH / NR;
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ __align__(8) uint64_t bars[NB];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrow = a.l + 1 - a.r0;                     // depths r0..l
  const int nch = (nrow + a.chunk - 1) / a.chunk;
  const long row_el = 2L * a.h;                        // elements of one depth row (K then V)
  const uint32_t chunk_bytes = (uint32_t)(a.chunk * row_el * sizeof(bf16));
  const uint32_t q_bytes = (uint32_t)(a.h * sizeof(bf16));
  const int ntok = a.n_tok > (int)blockIdx.x ? (a.n_tok - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int nitems = ntok * nch;
  if (nitems == 0) return;  // the whole CTA
  auto kv_slot = [&](int b) { return dsm + (size_t)b * chunk_bytes; };
  auto q_slot = [&](int b) { return dsm + (size_t)NB * chunk_bytes + (size_t)b * q_bytes; };
  if (threadIdx.x == 0) {
    for (int i = 0; i < NB; i++)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tcda::smem_u32(&bars[i])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  // the issuer's position in the (token, chunk) stream: no run-time divisions a chunk
  int is_c = 0, is_tok = (int)blockIdx.x;
  auto issue = [&](int j) {
    const int b = j % NB, c = is_c;
    const int tok = is_tok;
    if (++is_c == nch) {
      is_c = 0;
      is_tok += (int)gridDim.x;
    }
    const int r0 = c * a.chunk, nr = min(a.chunk, nrow - r0);
    const uint32_t kvb = (uint32_t)(nr * row_el * sizeof(bf16));
    const uint32_t bar = tcda::smem_u32(&bars[b]);
    const uint32_t total = kvb + (c == 0 ? q_bytes : 0u);
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(total)
                 : "memory");
    tcda::bulk_load(tcda::smem_u32(kv_slot(b)),
                    reinterpret_cast<const bf16 *>(a.kv) + ((long)tok * a.L + a.r0 + r0) * row_el,
                    kvb, bar);
    if (c == 0)
      tcda::bulk_load(tcda::smem_u32(q_slot(b)), reinterpret_cast<const bf16 *>(a.q) + (long)tok * a.h,
                      q_bytes, bar);
  };
  int issued = 0;  // items issued (thread 0's count)
  if (threadIdx.x == 0)
    for (; issued < NB && issued < nitems; issued++) issue(issued);
  const int cc = lane % CH, g = lane / CH;
  const int myrow = g * NR + cc / DUP;                 // the batch row whose score this lane ends with
  const int head = warp;
  const bool active = head < a.H;
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);
  uint64_t o2[4];
  uint32_t qb[4];  // the query slice as bf16 pairs
  float m = -INFINITY, lsum = 0.f;
  int consumed = 0;
  int c = 0, ctok = (int)blockIdx.x;  // the consumer's (chunk, token) position
  for (int j = 0; j < nitems; j++) {
    const int b = j % NB;
    const uint32_t bar = tcda::smem_u32(&bars[b]);
    const uint32_t par = (uint32_t)((j / NB) & 1);
    if (!tcda::try_wait(bar, par)) {  // bounded; on expiry every thread stops after the barrier
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(bar, par)) {
        if (abort_flag) break;
        if (tcda::gtimer() - t0 > DREAMER_WAIT_LIMIT_NS) {
          abort_flag = 1;
          raise_dev_error(a.err, DEV_TIMEOUT);
          break;
        }
      }
    }
    if (!abort_flag) consumed = j + 1;
    // stale after a timeout; nothing is stored then
    const uint8_t *bk = kv_slot(b) + (size_t)(head * D + cc * 8) * sizeof(bf16);
    const uint32_t vofs = (uint32_t)(a.h * sizeof(bf16));
    const uint32_t rstride = (uint32_t)(row_el * sizeof(bf16));
    const int nr = min(a.chunk, nrow - c * a.chunk);
    if (active) {
      if (c == 0) {  // a new token: its query, a fresh softmax
        const uint4 qw = *reinterpret_cast<const uint4 *>(q_slot(b) + (size_t)(head * D + cc * 8) * sizeof(bf16));
        qb[0] = qw.x; qb[1] = qw.y; qb[2] = qw.z; qb[3] = qw.w;
#pragma unroll
        for (int w = 0; w < 4; w++) o2[w] = 0ull;
        m = -INFINITY;
        lsum = 0.f;
      }
      // one batch of 8 rows; FULL: all 8 rows exist (no per-row checks)
      auto batch = [&](const int b0, auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        // partial dot products of this lane's 8 elements with the NR rows of its group
        float v[NR];
#pragma unroll
        for (int i = 0; i < NR; i++) {
          const int r = b0 + g * NR + i;
          v[i] = 0.f;
          if (FULL || r < nr) {
            const uint4 kw = *reinterpret_cast<const uint4 *>(bk + (size_t)r * rstride);
            // bf16 products are exact in fp32: no widening of q or k, two fp32 sums
            float a0 = tcda::dot2_bf16(qb[0], kw.x, 0.f), a1 = tcda::dot2_bf16(qb[1], kw.y, 0.f);
            a0 = tcda::dot2_bf16(qb[2], kw.z, a0);
            a1 = tcda::dot2_bf16(qb[3], kw.w, a1);
            v[i] = a0 + a1;
          }
        }
        // transposed butterfly: halving exchanges over the lanes of a row, then plain ones
#pragma unroll
        for (int st = 0; (NR >> st) > 1; st++) {
          const int mk = CH >> (st + 1), half = NR >> (st + 1);
          const bool upper = (lane & mk) != 0;
#pragma unroll
          for (int i = 0; i < half; i++) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mk);
          }
        }
#pragma unroll
        for (int mk = DUP / 2; mk >= 1; mk >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], mk);
        // online softmax over the batch (scores in log2 units)
        const bool valid = FULL || b0 + myrow < nr;
        const float x = valid ? v[0] * sl2 : -INFINITY;
        // max and sum over the batch's rows: a row's score sits in DUP neighbouring lanes
        // (bitwise equal), so the exchanges skip the low log2(DUP) lane bits
        float xm = x;
#pragma unroll
        for (int mk = DUP; mk < 32; mk <<= 1) xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, mk));
        const float mn = fmaxf(m, xm);
        const float alpha = tcda::ex2a(m - mn);
        const float p = valid ? tcda::ex2a(x - mn) : 0.f;
        float ps = p;
#pragma unroll
        for (int mk = DUP; mk < 32; mk <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, mk);
        lsum = lsum * alpha + ps;
        m = mn;
        const uint64_t al2 = tcda::pk2(alpha, alpha);
#pragma unroll
        for (int w = 0; w < 4; w++) o2[w] = tcda::mul2(o2[w], al2);
        // the weights of this group's rows, then their V rows into the 8 output elements
#pragma unroll
        for (int i = 0; i < NR; i++) {
          const float pi = __shfl_sync(0xffffffffu, p, g * CH + i * DUP);
          const int r = b0 + g * NR + i;
          if (FULL || r < nr) {
            const uint4 vw = *reinterpret_cast<const uint4 *>(bk + (size_t)r * rstride + vofs);
            const uint64_t p2 = tcda::pk2(pi, pi);
            o2[0] = tcda::fma2(p2, tcda::bf2_to_f2(vw.x), o2[0]);
            o2[1] = tcda::fma2(p2, tcda::bf2_to_f2(vw.y), o2[1]);
            o2[2] = tcda::fma2(p2, tcda::bf2_to_f2(vw.z), o2[2]);
            o2[3] = tcda::fma2(p2, tcda::bf2_to_f2(vw.w), o2[3]);
          }
        }
      };
      int b0 = 0;
#pragma unroll 1
      for (; b0 + 8 <= nr; b0 += 8) batch(b0, std::true_type{});
      if (b0 < nr) batch(b0, std::false_type{});
      if (c == nch - 1) {  // the token's last chunk: sum the groups, normalise, store
        float of[8];
#pragma unroll
        for (int w = 0; w < 4; w++) {
          const float2 f = tcda::up2(o2[w]);
          of[2 * w] = f.x;
          of[2 * w + 1] = f.y;
        }
#pragma unroll
        for (int mk = CH; mk < 32; mk <<= 1)
#pragma unroll
          for (int i = 0; i < 8; i++) of[i] += __shfl_xor_sync(0xffffffffu, of[i], mk);
        if (g == 0 && !abort_flag) {
          const int tok = ctok;
          const float inv = 1.0f / lsum;
#pragma unroll
          for (int i = 0; i < 8; i++) of[i] *= inv;
          const long orow = a.out_rows ? a.out_rows[tok] : tok;
          store8(reinterpret_cast<bf16 *>(a.out) + orow * a.ldo + a.col0 + head * D + cc * 8, of);
        }
      }
    }
    __syncthreads();        // buffer b is free again
    if (abort_flag) break;  // read after the barrier: the same decision in every thread
    if (threadIdx.x == 0 && issued < nitems) {
      issue(issued);
      issued++;
    }
    if (++c == nch) {
      c = 0;
      ctok += (int)gridDim.x;
    }
  }
  // copies still in flight after an abort land before the CTA exits
  if (threadIdx.x == 0 && abort_flag) {
    for (int j = consumed; j < issued; j++) {
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(tcda::smem_u32(&bars[j % NB]), (uint32_t)((j / NB) & 1)) &&
             tcda::gtimer() - t0 < DREAMER_WAIT_LIMIT_NS) {
      }
    }
  }
}

// =======================================================================================
// Decode attention over the per-depth SA cache, streamed: one CTA per (sequence, head, key
// range).  The range's keys and values are two contiguous runs of the [L][B][H][cap][D]
// caches, so thread 0 streams them into shared memory with 1-D bulk copies, NST chunks in
// flight; the eight warps take interleaved groups of rows of each chunk (row-group layout as
// above) with their own online softmax, and the CTA folds the eight (m, l, o) into one partial
// for attn_merge_kernel.  Every chunk wait is bounded; the decision to stop is taken after a
// block barrier so all threads take it together.
// =======================================================================================
struct DecBulkArgs {
  int B, H, L, l, cap, nsplit, chunk;  // chunk: keys per shared-memory stage
  const void *q;                       // [B][ldq], head at column head * D
  long ldq;
  const void *kc, *vc;                 // [L][B][H][cap][D]
  const int *cache_len;                // [B]
  float *part;                         // [B][H][nsplit][D + 2] partial (o, m, l)
  int *err;
};

template <typename T, int D>
__global__ void __launch_bounds__(256) dec_bulk_kernel(DecBulkArgs a) {
  pdl_wait();
  pdl_trigger();
  constexpr int NST = 4, NW = 8;
  constexpr int VEC = VecOf<T>::N;
  constexpr int CH = D / VEC;
  constexpr int RPW = 32 / CH;
  constexpr int U = 2;
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ __align__(8) uint64_t bars[NST];
  __shared__ int abort_flag;
  __shared__ float wm[NW], wl[NW];
  __shared__ __align__(16) float wo[NW][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sp = blockIdx.x % a.nsplit, bh = blockIdx.x / a.nsplit;
  const int b = bh / a.H, head = bh % a.H;
  float *pp = a.part + ((long)bh * a.nsplit + sp) * (D + 2);
  const int len = a.cache_len[b];
  if (len < 0 || len >= a.cap) {  // slot outside the cache: report, attend to nothing
    if (threadIdx.x == 0) {
      raise_dev_error(a.err, DEV_BAD_INDEX);
      pp[D] = -INFINITY;
      pp[D + 1] = 0.f;
    }
    return;
  }
  const int nk = len + 1;
  const int per = (nk + a.nsplit - 1) / a.nsplit;
  const int j0 = sp * per, j1 = min(nk, j0 + per);
  if (j0 >= j1) {  // empty range
    if (threadIdx.x == 0) {
      pp[D] = -INFINITY;
      pp[D + 1] = 0.f;
    }
    return;
  }
  const long off = ((((long)a.l * a.B + b) * a.H + head) * a.cap + j0) * D;
  const T *Ks = reinterpret_cast<const T *>(a.kc) + off;
  const T *Vs = reinterpret_cast<const T *>(a.vc) + off;
  const int nrow = j1 - j0;
  const int nch = (nrow + a.chunk - 1) / a.chunk;
  const uint32_t cbytes = (uint32_t)(a.chunk * D * sizeof(T));
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; i++)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tcda::smem_u32(&bars[i])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    abort_flag = 0;
  }
  __syncthreads();
  auto issue = [&](int c) {
    const int st = c % NST;
    const int nr = min(a.chunk, nrow - c * a.chunk);
    const uint32_t bytes = (uint32_t)(nr * D * sizeof(T));
    const uint32_t bar = tcda::smem_u32(&bars[st]);
    asm volatile("{\n\t.reg .b64 s;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 s, [%0], %1;\n\t}" ::"r"(bar),
                 "r"(2 * bytes)
                 : "memory");
    uint8_t *dst = dsm + (size_t)st * 2 * cbytes;
    tcda::bulk_load(tcda::smem_u32(dst), Ks + (long)c * a.chunk * D, bytes, bar);
    tcda::bulk_load(tcda::smem_u32(dst + cbytes), Vs + (long)c * a.chunk * D, bytes, bar);
  };
  int issued = 0;
  if (threadIdx.x == 0) {
    for (; issued < NST && issued < nch; issued++) issue(issued);
  }
  const int cc = lane % CH, rr = lane / CH;
  float q[VEC], o[VEC];
  const float sl2 = 1.4426950408889634f * rsqrtf((float)D);
  ld16(reinterpret_cast<const T *>(a.q) + (long)b * a.ldq + head * D + cc * VEC, q);
#pragma unroll
  for (int i = 0; i < VEC; i++) {
    q[i] *= sl2;
    o[i] = 0.f;
  }
  float m = -INFINITY, lsum = 0.f;
  // bf16 at head dim 64 / 128: depth attention's batch form (8 rows a warp batch, the
  // transposed butterfly, bf16 q.k products in mixed FMAs, check-free full batches); warp w
  // takes batches w, w + 8, ... of each chunk with its own online softmax
  constexpr bool FAST = std::is_same<T, bf16>::value && (D == 64 || D == 128);
  constexpr int FCH = FAST ? D / 8 : 16, FG = 32 / FCH, FNR = 8 / FG, FDUP = FCH / FNR;
  const int fg = lane / FCH;
  const int myrow = fg * FNR + cc / FDUP;
  uint32_t qb[4] = {0u, 0u, 0u, 0u};
  uint64_t o2[4] = {0ull, 0ull, 0ull, 0ull};
  if constexpr (FAST) {
    const uint4 qw = *reinterpret_cast<const uint4 *>(reinterpret_cast<const bf16 *>(a.q) +
                                                      (long)b * a.ldq + head * D + cc * 8);
    qb[0] = qw.x; qb[1] = qw.y; qb[2] = qw.z; qb[3] = qw.w;
  }
  int consumed = 0;
  for (int c = 0; c < nch; c++) {
    const int st = c % NST;
    const uint32_t bar = tcda::smem_u32(&bars[st]);
    const uint32_t par = (uint32_t)((c / NST) & 1);
    if (!tcda::try_wait(bar, par)) {
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(bar, par)) {
        if (abort_flag) break;
        if (tcda::gtimer() - t0 > DREAMER_WAIT_LIMIT_NS) {
          abort_flag = 1;
          raise_dev_error(a.err, DEV_TIMEOUT);
          break;
        }
      }
    }
    if (!abort_flag) consumed = c + 1;
    const T *sk = reinterpret_cast<const T *>(dsm + (size_t)st * 2 * cbytes);
    const T *sv = reinterpret_cast<const T *>(dsm + (size_t)st * 2 * cbytes + cbytes);
    const int nr = min(a.chunk, nrow - c * a.chunk);
    if constexpr (FAST) {
      const uint8_t *kb = reinterpret_cast<const uint8_t *>(sk) + cc * 16;
      const uint8_t *vb = reinterpret_cast<const uint8_t *>(sv) + cc * 16;
      constexpr uint32_t RS = D * 2;  // bytes of a key (value) row
      auto batch = [&](const int b0, auto full_tag) {
        constexpr bool FULL = decltype(full_tag)::value;
        float v[FNR];
#pragma unroll
        for (int i = 0; i < FNR; i++) {
          const int r = b0 + fg * FNR + i;
          v[i] = 0.f;
          if (FULL || r < nr) {
            const uint4 kw = *reinterpret_cast<const uint4 *>(kb + (size_t)r * RS);
            float a0 = tcda::dot2_bf16(qb[0], kw.x, 0.f), a1 = tcda::dot2_bf16(qb[1], kw.y, 0.f);
            a0 = tcda::dot2_bf16(qb[2], kw.z, a0);
            a1 = tcda::dot2_bf16(qb[3], kw.w, a1);
            v[i] = a0 + a1;
          }
        }
#pragma unroll
        for (int stp = 0; (FNR >> stp) > 1; stp++) {
          const int mk = FCH >> (stp + 1), half = FNR >> (stp + 1);
          const bool upper = (lane & mk) != 0;
#pragma unroll
          for (int i = 0; i < half; i++) {
            const float send = upper ? v[i] : v[i + half];
            const float keep = upper ? v[i + half] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mk);
          }
        }
#pragma unroll
        for (int mk = FDUP / 2; mk >= 1; mk >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], mk);
        const bool valid = FULL || b0 + myrow < nr;
        const float x = valid ? v[0] * sl2 : -INFINITY;
        float xm = x;
#pragma unroll
        for (int mk = FDUP; mk < 32; mk <<= 1) xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, mk));
        const float mn = fmaxf(m, xm);
        const float alpha = tcda::ex2a(m - mn);
        const float p = valid ? tcda::ex2a(x - mn) : 0.f;
        float ps = p;
#pragma unroll
        for (int mk = FDUP; mk < 32; mk <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, mk);
        lsum = lsum * alpha + ps;
        m = mn;
        const uint64_t al2 = tcda::pk2(alpha, alpha);
#pragma unroll
        for (int w = 0; w < 4; w++) o2[w] = tcda::mul2(o2[w], al2);
#pragma unroll
        for (int i = 0; i < FNR; i++) {
          const float pi = __shfl_sync(0xffffffffu, p, fg * FCH + i * FDUP);
          const int r = b0 + fg * FNR + i;
          if (FULL || r < nr) {
            const uint4 vw = *reinterpret_cast<const uint4 *>(vb + (size_t)r * RS);
            const uint64_t p2 = tcda::pk2(pi, pi);
            o2[0] = tcda::fma2(p2, tcda::bf2_to_f2(vw.x), o2[0]);
            o2[1] = tcda::fma2(p2, tcda::bf2_to_f2(vw.y), o2[1]);
            o2[2] = tcda::fma2(p2, tcda::bf2_to_f2(vw.z), o2[2]);
            o2[3] = tcda::fma2(p2, tcda::bf2_to_f2(vw.w), o2[3]);
          }
        }
      };
#pragma unroll 1
      for (int b0 = warp * 8; b0 < nr; b0 += NW * 8) {
        if (b0 + 8 <= nr) batch(b0, std::true_type{});
        else batch(b0, std::false_type{});
      }
    } else
    for (int g = warp * RPW; g < nr; g += NW * RPW * U) {
      float s[U], vv[U][VEC];
#pragma unroll
      for (int u = 0; u < U; u++) {
        const int j = g + u * NW * RPW + rr;
        s[u] = -INFINITY;
        if (j < nr) {
          float kv[VEC];
          ld16(sk + (long)j * D + cc * VEC, kv);
          ld16(sv + (long)j * D + cc * VEC, vv[u]);
          float p = 0.f;
#pragma unroll
          for (int i = 0; i < VEC; i++) p = fmaf(q[i], kv[i], p);
          s[u] = p;
        } else {
#pragma unroll
          for (int i = 0; i < VEC; i++) vv[u][i] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; u++) {
        float p = s[u] == -INFINITY ? 0.f : s[u];
#pragma unroll
        for (int o2 = 1; o2 < CH; o2 <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o2);
        if (s[u] != -INFINITY) s[u] = p;
      }
      float gm = s[0];
#pragma unroll
      for (int u = 1; u < U; u++) gm = fmaxf(gm, s[u]);
      gm = warp_max(gm);
      const float mn = fmaxf(m, gm);
      const float alpha = exp2f(m - mn);
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < VEC; i++) o[i] *= alpha;
#pragma unroll
      for (int u = 0; u < U; u++) {
        const float p = s[u] == -INFINITY ? 0.f : exp2f(s[u] - mn);
        ps += p;
#pragma unroll
        for (int i = 0; i < VEC; i++) o[i] = fmaf(p, vv[u][i], o[i]);
      }
      ps = warp_sum(cc == 0 ? ps : 0.f);
      lsum = lsum * alpha + ps;
      m = mn;
    }
    __syncthreads();        // stage st is free again
    if (abort_flag) break;  // read after the barrier: the same decision in every thread
    if (threadIdx.x == 0 && issued < nch) {
      issue(issued);
      issued++;
    }
  }
  if constexpr (FAST) {
#pragma unroll
    for (int w = 0; w < 4; w++) {
      const float2 f = tcda::up2(o2[w]);
      o[2 * w] = f.x;
      o[2 * w + 1] = f.y;
    }
  }
#pragma unroll
  for (int o2 = CH; o2 < 32; o2 <<= 1)
#pragma unroll
    for (int i = 0; i < VEC; i++) o[i] += __shfl_xor_sync(0xffffffffu, o[i], o2);
  if (rr == 0) {
#pragma unroll
    for (int i = 0; i < VEC; i++) wo[warp][cc * VEC + i] = o[i];
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = lsum;
  }
  __syncthreads();
  if (!abort_flag) {
    float M = wm[0];
#pragma unroll
    for (int w = 1; w < NW; w++) M = fmaxf(M, wm[w]);
    float f[NW];
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < NW; w++) {
      f[w] = wm[w] == -INFINITY ? 0.f : exp2f(wm[w] - M);
      den += f[w] * wl[w];
    }
    for (int dd = threadIdx.x; dd < D; dd += blockDim.x) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < NW; w++) acc = fmaf(f[w], wo[w][dd], acc);
      pp[dd] = acc;
    }
    if (threadIdx.x == 0) {
      pp[D] = M;
      pp[D + 1] = den;
    }
  }
  // copies still in flight after an abort land before the CTA exits
  if (threadIdx.x == 0 && abort_flag) {
    for (int c = consumed; c < issued; c++) {
      const uint64_t t0 = tcda::gtimer();
      while (!tcda::try_wait(tcda::smem_u32(&bars[c % NST]), (uint32_t)((c / NST) & 1)) &&
             tcda::gtimer() - t0 < DREAMER_WAIT_LIMIT_NS) {
      }
    }
  }
}

}  // namespace dreamer
