// Causal sequence attention for prefill on tcgen05 (flash-style, one 128-query tile of one
// (sequence, head) per CTA).  Sequence attention over tokens (papernotes "Overall framework":
// SA keeps the standard causal interaction across time steps; reading R4: scale 1/sqrt(d),
// key j <= query i).
//
//   warp 0     TMA: Q tile once, then K_j / V_j blocks of 128 keys into a 2- or 3-deep ring
//   warp 1     TMEM allocator + MMA issuer: S_j = Q K_j^T into one of two TMEM S buffers
//              (issued one block ahead), then O_j = P_j V_j into one of two TMEM O buffers
//   warps 2-5  softmax, one query row per thread: scale, causal mask on the diagonal block,
//              running max / sum, P_j = exp2(...) written as bf16 into shared memory in the
//              swizzled K-major layout of the P V operand; folds O_{j-1} into a register
//              accumulator with the rescale of its block (deferred one step so the MMA runs
//              while the exponentials are computed); finally divides by the row sum.
// V is consumed in its natural [key][d] layout as an MN-major B operand.
#pragma once
#include "tc_common.cuh"

namespace dreamer {
namespace tc {

// K-major SW128 descriptor (tile rows of 128 bytes)
__device__ __forceinline__ uint64_t desc_k128(uint32_t addr) { return smem_desc(addr, 128); }
// MN-major SW128 descriptor: 64-element MN chunks `lbo` bytes apart, 8-row K groups 1024 apart
__device__ __forceinline__ uint64_t desc_mn128(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= 2ull << 61;
  return d;
}
// M = 128, N = n, A K-major, B MN-major (bit 16), bf16 -> f32
__host__ __device__ constexpr uint32_t idesc_bf16_m128_bmn(int n) {
  return idesc_bf16_m128(n) | (1u << 16);
}

struct SaArgs {
  int S, H, h, n_qt;      // tokens per sequence, heads, hidden, query tiles per sequence
  int n_items;            // batch * H * n_qt
  bf16 *out;              // attn [T][2h], SA part at columns head*d
  long ldo;
  float scale_log2;       // log2(e) / sqrt(d)
  int *err;
};

template <int D>
struct SaCfg {
  static constexpr int STAGES = D == 64 ? 3 : 2;
  static constexpr int CH = D / 64;                 // 64-column chunks of a head
  static constexpr int TILE = 128 * 128;            // bytes of one [128 x 64] bf16 chunk
  static constexpr int Q_BYTES = CH * TILE;
  static constexpr int KV_BYTES = 2 * CH * TILE;    // K and V of one block
  static constexpr int P_BYTES = 2 * TILE;          // [128 x 128] bf16 in two key chunks
  static constexpr int SMEM = Q_BYTES + STAGES * KV_BYTES + P_BYTES + 1024 + 256;
  static_assert(SMEM <= 227 * 1024, "smem");
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    tc_sa_kernel(const __grid_constant__ CUtensorMap tm, SaArgs a) {
  using C = SaCfg<D>;
  constexpr int ST = C::STAGES, CH = C::CH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sKV = sQ + C::Q_BYTES;
  uint8_t *sP = sKV + ST * C::KV_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sP + C::P_BYTES);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1, *kv_empty = kv_full + ST;
  uint64_t *s_full = kv_empty + ST, *s_free = s_full + 2;
  uint64_t *pv_done = s_free + 2, *o_free = pv_done + 2, *p_full = o_free + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(p_full + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // heaviest tiles first: item -> (query tile from the last, sequence*head)
  const int item = blockIdx.x;
  const int bh = item % (a.n_items / a.n_qt);
  const int qt = a.n_qt - 1 - item / (a.n_items / a.n_qt);
  const int b = bh / a.H, head = bh % a.H;
  const int nb = qt + 1;  // key blocks 0..qt
  const int row0 = b * a.S;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < ST; s++) {
      mbar_init(smem_u32(&kv_full[s]), 1);
      mbar_init(smem_u32(&kv_empty[s]), 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 128);
      mbar_init(smem_u32(&pv_done[i]), 1);
      mbar_init(smem_u32(&o_free[i]), 128);
    }
    mbar_init(smem_u32(p_full), 128);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tm);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S buffers at 0 and 128, O buffers at 256 and 256 + D
  const uint32_t tS = tmem, tO = tmem + 256;

  if (warp == 0) {
    if (lane == 0) {
      const int cq = head * D, ck = a.h + head * D, cv = 2 * a.h + head * D;
      mbar_expect_tx(smem_u32(q_full), C::Q_BYTES);
      for (int c = 0; c < CH; c++)
        tma_load_2d(smem_u32(sQ + c * C::TILE), &tm, smem_u32(q_full), cq + 64 * c,
                    row0 + qt * 128);
      int s = 0;
      uint32_t ph = 0;
      int issued_ph[ST];
      for (int i = 0; i < ST; i++) issued_ph[i] = -1;
      bool ok = true;
      for (int j = 0; j < nb; j++) {
        if (!mbar_wait(smem_u32(&kv_empty[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
        const uint32_t fb = smem_u32(&kv_full[s]);
        uint8_t *kv = sKV + s * C::KV_BYTES;
        mbar_expect_tx(fb, C::KV_BYTES);
        for (int c = 0; c < CH; c++) {
          tma_load_2d(smem_u32(kv + c * C::TILE), &tm, fb, ck + 64 * c, row0 + j * 128);
          tma_load_2d(smem_u32(kv + (CH + c) * C::TILE), &tm, fb, cv + 64 * c, row0 + j * 128);
        }
        issued_ph[s] = (int)ph;
        if (++s == ST) { s = 0; ph ^= 1; }
      }
      // every copy issued lands before the CTA can exit (the Q wait also covers an abort)
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(smem_u32(q_full), 0) && globaltimer() - t0 < WAIT_LIMIT_NS) {
      }
      if (!ok)
        for (int i = 0; i < ST; i++)
          if (issued_ph[i] >= 0) {
            const uint64_t t1 = globaltimer();
            while (!mbar_try_wait(smem_u32(&kv_full[i]), (uint32_t)issued_ph[i]) &&
                   globaltimer() - t1 < WAIT_LIMIT_NS) {
            }
          }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16_m128(128);
      constexpr uint32_t ID_PV = idesc_bf16_m128_bmn(D);
      bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, a.err);
      const uint32_t q0 = smem_u32(sQ), p0 = smem_u32(sP);
      // S_j = Q K_j^T into S buffer j & 1
      auto issue_s = [&](int j) -> bool {
        const int s = j % ST;
        const uint32_t ph = (j / ST) & 1;
        if (!mbar_wait(smem_u32(&kv_full[s]), ph, abort_flag, a.err)) return false;
        if (!mbar_wait(smem_u32(&s_free[j & 1]), ((j >> 1) & 1) ^ 1, abort_flag, a.err)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sKV + s * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < D / 16; k++) {
          const uint32_t off = (k >> 2) * C::TILE + (k & 3) * 32;
          mma_bf16(tS + (j & 1) * 128, desc_k128(q0 + off), desc_k128(k0 + off), ID_S, k != 0);
        }
        mma_commit(smem_u32(&s_full[j & 1]));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; j < nb && ok; j++) {
        if (j + 1 < nb && !issue_s(j + 1)) { ok = false; break; }
        // O_j = P_j V_j into O buffer j & 1
        if (!mbar_wait(smem_u32(p_full), j & 1, abort_flag, a.err)) { ok = false; break; }
        if (!mbar_wait(smem_u32(&o_free[j & 1]), ((j >> 1) & 1) ^ 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const int s = j % ST;
        const uint32_t v0 = smem_u32(sKV + s * C::KV_BYTES + CH * C::TILE);
#pragma unroll
        for (int k = 0; k < 8; k++) {  // 128 keys, 16 per instruction
          const uint32_t poff = (k >> 2) * C::TILE + (k & 3) * 32;
          mma_bf16(tO + (j & 1) * D, desc_k128(p0 + poff), desc_mn128(v0 + k * 2048, C::TILE),
                   ID_PV, k != 0);
        }
        mma_commit(smem_u32(&pv_done[j & 1]));
        mma_commit(smem_u32(&kv_empty[s]));
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int q = warp & 3;
    const int row = q * 32 + lane;                 // query row inside the tile
    const int qi = qt * 128 + row;                 // query position in the sequence
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    float o[D];
#pragma unroll
    for (int i = 0; i < D; i++) o[i] = 0.f;
    float m = -INFINITY, l = 0.f, alpha_prev = 1.f;
    bool ok = true;
    uint8_t *prow0 = sP + row * 128;
    for (int j = 0; j < nb; j++) {
      if (!mbar_wait(smem_u32(&s_full[j & 1]), (j >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sbuf = tS + (j & 1) * 128 + lane_off;
      const bool diag = (j == qt);
      // pass 1: row max of the scaled, masked scores
      float mx = m;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        float sv[32];
        tmem_ld32(sbuf + c, sv);
#pragma unroll
        for (int i = 0; i < 32; i++) {
          const bool masked = diag && (j * 128 + c + i) > qi;
          if (!masked) mx = fmaxf(mx, sv[i] * a.scale_log2);
        }
      }
      const float alpha = exp2f(m - mx);  // 0 on the first block (m = -inf)
      // fold O_{j-1} (kept at the max of block j-1) before P_j overwrites P_{j-1}
      if (j > 0) {
        if (!mbar_wait(smem_u32(&pv_done[(j - 1) & 1]), ((j - 1) >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          float ov[32];
          tmem_ld32(tO + ((j - 1) & 1) * D + c + lane_off, ov);
#pragma unroll
          for (int i = 0; i < 32; i++) o[c + i] = o[c + i] * alpha_prev + ov[i];
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&o_free[(j - 1) & 1]));
      }
      // pass 2: P_j = exp2(s - max) as bf16 into the K-major SW128 operand (key chunk kc at
      // kc * TILE, 16-byte unit u of the row at ((u ^ (row & 7)) << 4))
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 32) {
        float sv[32];
        tmem_ld32(sbuf + c, sv);
#pragma unroll
        for (int i = 0; i < 32; i++) {
          const bool masked = diag && (j * 128 + c + i) > qi;
          const float p = masked ? 0.f : exp2f(sv[i] * a.scale_log2 - mx);
          sv[i] = p;
          rs += p;
        }
        const int kc = c >> 6;
#pragma unroll
        for (int uu = 0; uu < 4; uu++) {
          const int u = ((c & 63) >> 3) + uu;
          uint4 pk;
          __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&pk);
#pragma unroll
          for (int t = 0; t < 4; t++) p2[t] = __floats2bfloat162_rn(sv[uu * 8 + 2 * t], sv[uu * 8 + 2 * t + 1]);
          *reinterpret_cast<uint4 *>(prow0 + kc * C::TILE + ((u ^ (row & 7)) << 4)) = pk;
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[j & 1]));
      l = l * alpha + rs;
      m = mx;
      alpha_prev = alpha;
      fence_proxy_async();
      mbar_arrive(smem_u32(p_full));
    }
    if (ok && mbar_wait(smem_u32(&pv_done[(nb - 1) & 1]), ((nb - 1) >> 1) & 1, abort_flag, a.err)) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        tmem_ld32(tO + ((nb - 1) & 1) * D + c + lane_off, ov);
#pragma unroll
        for (int i = 0; i < 32; i++) o[c + i] = o[c + i] * alpha_prev + ov[i];
      }
      const float inv = 1.0f / l;
      bf16 *dst = a.out + (long)(row0 + qi) * a.ldo + head * D;
#pragma unroll
      for (int c = 0; c < D; c += 8) {
        float t8[8];
#pragma unroll
        for (int i = 0; i < 8; i++) t8[i] = o[c + i] * inv;
        store8(dst + c, t8);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace dreamer

static int tc_attn_init(dreamer_handle *h) { return 0; }

static bool make_tmap(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows,
                      uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows);

static bool tc_sa_ok(dreamer_handle *h) {
  const dreamer_config &c = h->cfg;
  return c.seq % 128 == 0 && (c.head_dim == 64 || c.head_dim == 128) && c.hidden % 64 == 0;
}

// SA of every (sequence, head, query tile): q/k/v from qkv_sa [T][3h], output into the SA
// half of attn [T][2h].
static bool tc_sa(dreamer_handle *h, cudaStream_t s) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int hd = c.hidden, d = c.head_dim;
  const long T = (long)c.batch * c.seq;
  CUtensorMap tm;
  if (!make_tmap(&tm, h->qkv_sa, 3 * hd, T, 3 * hd * 2, 64, 128)) return false;
  tc::SaArgs a{};
  a.S = c.seq; a.H = c.n_heads; a.h = hd; a.n_qt = c.seq / 128;
  a.n_items = c.batch * c.n_heads * a.n_qt;
  a.out = (bf16 *)h->attn; a.ldo = 2 * hd;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  a.err = h->err;
  if (d == 64) {
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(tc::tc_sa_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SaCfg<64>::SMEM);
      set = true;
    }
    tc::tc_sa_kernel<64><<<a.n_items, 192, tc::SaCfg<64>::SMEM, s>>>(tm, a);
  } else {
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(tc::tc_sa_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SaCfg<128>::SMEM);
      set = true;
    }
    tc::tc_sa_kernel<128><<<a.n_items, 192, tc::SaCfg<128>::SMEM, s>>>(tm, a);
  }
  return true;
}
