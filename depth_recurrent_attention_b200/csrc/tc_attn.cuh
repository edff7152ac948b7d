// Causal sequence attention for prefill on tcgen05 (flash-style).  Sequence attention over
// tokens (papernotes "Overall framework": SA keeps the causal interaction across time steps;
// reading R4: scale 1/sqrt(d), key j <= query i).
//
// One CTA = one (sequence, head) and two adjacent 128-query tiles A = 2p, B = 2p + 1 that
// share every K/V block (heaviest pairs first):
//   warp 0      TMA: both Q tiles once, then K_j into a KST-deep ring
//   warp 2      TMA: V_j into a VST-deep ring
//   warp 1      TMEM allocator + MMA issuer: S_t(0) = Q_t K_0^T for both tiles; then per
//               block j and tile t, O_t += P_t(j) V_j with P read from TMEM, and S_t(j+1)
//               into the same TMEM columns (issued after the P.V, so it runs after it);
//               tile B's MMAs keep the tensor core busy while tile A's softmax runs and the
//               other way round
//   warps 3-10  softmax, one query row per thread: tile A on warps 4, 5, 6, 3 and tile B on
//               warps 8, 9, 10, 7 (a warp reads the TMEM lanes of its warp index mod 4), 11
//               warps in all so that a thread may hold a row of 128 scores in registers:
//               the row's 128 scores come out of TMEM in one batch of loads, then the row
//               max, P = exp2(s - m_ref) summed and written as bf16 pairs over the first 64
//               columns of the tile's S (every exponential on MUFU).  O lives in TMEM and is
//               only rescaled when the running max grows by more than 2^8 (P stays <= 256),
//               so most blocks need no O traffic at all; the last step divides O by the sum.
// TMEM: S_A columns 0..127, S_B 128..255, O_A 256.., O_B 256 + D.. (512 allocated).
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

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]),
      "f"(v[15]), "f"(v[16]), "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]),
      "f"(v[22]), "f"(v[23]), "f"(v[24]), "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]),
      "f"(v[29]), "f"(v[30]), "f"(v[31])
      : "memory");
}

// 32 lanes x 32 columns of 32-bit words into TMEM; the wait is a separate tmem_st_wait()
__device__ __forceinline__ void tmem_st32_nowait(uint32_t taddr, const uint32_t *v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T: A (M = 128 rows on the 128 lanes, K packed two bf16 a
// 32-bit column, the lower K in the low half) read from tensor memory, one thread issues.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

struct SaArgs {
  int S, H, h, n_qt;      // tokens per sequence, heads, hidden, query tiles per sequence
  int n_pairs;            // query-tile pairs per sequence
  int bh;                 // batch * H
  bf16 *out;              // attn [T][2h], SA part at columns head*d
  long ldo;
  float scale_log2;       // log2(e) / sqrt(d)
  int *err;
  const int *out_rows;    // output row of token t (grouped projections), or null: t
};

template <int D>
struct SaCfg {
  static constexpr int CH = D / 64;                 // 64-column chunks of a head
  static constexpr int TILE = 128 * 128;            // bytes of one [128 x 64] bf16 chunk
  static constexpr int KST = D == 64 ? 4 : 2;       // K ring depth
  static constexpr int VST = D == 64 ? 4 : 2;       // V ring depth
  static constexpr int Q_BYTES = 2 * CH * TILE;     // both query tiles
  static constexpr int KV_BYTES = CH * TILE;        // one K (or V) block
  static constexpr int SMEM = Q_BYTES + (KST + VST) * KV_BYTES + 1024 + 256;
  static_assert(SMEM <= 227 * 1024, "smem");
};

template <int D>
__global__ void __launch_bounds__(352, 1)
    tc_sa_kernel(const __grid_constant__ CUtensorMap tm, SaArgs a) {
  using C = SaCfg<D>;
  constexpr int CH = C::CH, KST = C::KST, VST = C::VST;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem;
  uint8_t *sK = sQ + C::Q_BYTES;
  uint8_t *sV = sK + KST * C::KV_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sV + VST * C::KV_BYTES);
  uint64_t *q_full = bars;
  uint64_t *k_full = q_full + 1, *k_empty = k_full + KST;
  uint64_t *v_full = k_empty + KST, *v_empty = v_full + VST;
  uint64_t *s_full = v_empty + VST, *p_full = s_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(p_full + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x;
  const int bh = item % a.bh;
  const int pair = a.n_pairs - 1 - item / a.bh;     // heaviest pairs first
  const int b = bh / a.H, head = bh % a.H;
  const int qtA = 2 * pair, qtB = 2 * pair + 1;
  const bool hasB = qtB < a.n_qt;
  const int nbA = qtA + 1, nbB = hasB ? qtB + 1 : 0;
  const int nb = hasB ? nbB : nbA;
  const int row0 = b * a.S;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(q_full), 1);
    for (int s = 0; s < KST; s++) {
      mbar_init(smem_u32(&k_full[s]), 1);
      mbar_init(smem_u32(&k_empty[s]), 1);
    }
    for (int s = 0; s < VST; s++) {
      mbar_init(smem_u32(&v_full[s]), 1);
      mbar_init(smem_u32(&v_empty[s]), 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&p_full[i]), 128);
    }
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
  pdl_wait();     // inputs of the previous kernel are visible from here on
  pdl_trigger();  // after the TMEM allocation (see pdl_trigger)
  // TMEM columns: S_A 0..127, S_B 128..255, O_A 256.., O_B 256 + D..
  const uint32_t tS = tmem, tO = tmem + 256;

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------- producers (warp 0: Q, K; warp 2: V)
    if (lane == 0) {
      const bool isK = warp == 0;
      const int colb = isK ? (a.h + head * D) : (2 * a.h + head * D);
      if (isK) {
        mbar_expect_tx(smem_u32(q_full), (hasB ? 2 : 1) * CH * C::TILE);
        for (int t = 0; t < (hasB ? 2 : 1); t++)
          for (int c = 0; c < CH; c++)
            tma_load_2d(smem_u32(sQ + (t * CH + c) * C::TILE), &tm, smem_u32(q_full),
                        head * D + 64 * c, row0 + (t == 0 ? qtA : qtB) * 128);
      }
      const int NS = isK ? KST : VST;
      uint64_t *fullb = isK ? k_full : v_full, *emptyb = isK ? k_empty : v_empty;
      uint8_t *ring = isK ? sK : sV;
      int issued_ph[4] = {-1, -1, -1, -1};
      bool ok = true;
      for (int j = 0; j < nb; j++) {
        const int s = j % NS;
        const uint32_t ph = (j / NS) & 1;
        if (!mbar_wait(smem_u32(&emptyb[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
        mbar_expect_tx(smem_u32(&fullb[s]), C::KV_BYTES);
        for (int c = 0; c < CH; c++)
          tma_load_2d(smem_u32(ring + s * C::KV_BYTES + c * C::TILE), &tm, smem_u32(&fullb[s]),
                      colb + 64 * c, row0 + j * 128);
        issued_ph[s] = (int)ph;
      }
      // every copy issued lands before the CTA can exit
      const uint64_t t0 = globaltimer();
      if (isK)
        while (!mbar_try_wait(smem_u32(q_full), 0) && globaltimer() - t0 < WAIT_LIMIT_NS) {
        }
      if (!ok)
        for (int i = 0; i < NS; i++)
          if (issued_ph[i] >= 0) {
            const uint64_t t1 = globaltimer();
            while (!mbar_try_wait(smem_u32(&fullb[i]), (uint32_t)issued_ph[i]) &&
                   globaltimer() - t1 < WAIT_LIMIT_NS) {
            }
          }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer
    // Per tile t the order is S_t(0), then for each block j: P_t(j) V_j (P read from the S_t
    // columns in TMEM), S_t(j+1) into the same columns (issued after, so it runs after the
    // P.V has read them), one commit to s_full[t]: the softmax sees S_t(j+1) and, with it, O_t
    // holding every block up to j.  Tile B's work fills the tensor core while tile A's
    // softmax runs, and the other way round.
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16_m128(128);
      constexpr uint32_t ID_PV = idesc_bf16_m128_bmn(D);
      bool ok = mbar_wait(smem_u32(q_full), 0, abort_flag, a.err);
      const uint32_t q0 = smem_u32(sQ);
      auto issue_s = [&](int t, uint32_t k0) {
        const uint32_t qt0 = q0 + t * CH * C::TILE;
#pragma unroll
        for (int k = 0; k < D / 16; k++) {
          const uint32_t off = (k >> 2) * C::TILE + (k & 3) * 32;
          mma_bf16(tS + t * 128, desc_k128(qt0 + off), desc_k128(k0 + off), ID_S, k != 0);
        }
      };
      if (ok && mbar_wait(smem_u32(&k_full[0]), 0, abort_flag, a.err)) {
        tc_fence_after();
        const uint32_t k0 = smem_u32(sK);
        issue_s(0, k0);
        mma_commit(smem_u32(&s_full[0]));
        if (nbB > 0) {
          issue_s(1, k0);
          mma_commit(smem_u32(&s_full[1]));
        }
        mma_commit(smem_u32(&k_empty[0]));
      } else {
        ok = false;
      }
      for (int j = 0; j < nb && ok; j++) {
        const int vs = j % VST;
        if (!mbar_wait(smem_u32(&v_full[vs]), (j / VST) & 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + vs * C::KV_BYTES);
        const bool next = j + 1 < nb;
        const int ks = (j + 1) % KST;
        uint32_t k1 = 0;
        if (next) {
          if (!mbar_wait(smem_u32(&k_full[ks]), ((j + 1) / KST) & 1, abort_flag, a.err)) break;
          tc_fence_after();
          k1 = smem_u32(sK + ks * C::KV_BYTES);
        }
        for (int t = 0; t < 2; t++) {
          const int nbt = t == 0 ? nbA : nbB;
          if (j >= nbt) continue;
          if (!mbar_wait(smem_u32(&p_full[t]), j & 1, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 8; k++)  // 128 keys, 16 per instruction (8 TMEM columns of P)
            mma_bf16_ts(tO + t * D, tS + t * 128 + k * 8, desc_mn128(v0 + k * 2048, C::TILE), ID_PV,
                        (j | k) != 0);
          if (j + 1 < nbt) issue_s(t, k1);
          mma_commit(smem_u32(&s_full[t]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&v_empty[vs]));
        if (next) mma_commit(smem_u32(&k_empty[ks]));
      }
    }
  } else if (warp >= 3) {
    // ------------------------------------------------- softmax (tile A: warps 3-6, B: 7-10)
    const int t = warp < 7 ? 0 : 1;
    const int nbt = t == 0 ? nbA : nbB;
    const int qt = t == 0 ? qtA : qtB;
    if (nbt > 0) {
      const int q = warp & 3;
      const int row = q * 32 + lane;
      const int qi = qt * 128 + row;               // query position in the sequence
      const uint32_t lane_off = (uint32_t)(q * 32) << 16;
      const uint32_t sbuf = tS + t * 128 + lane_off;
      const uint32_t obuf = tO + t * D + lane_off;
      float m_ref = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nbt; j++) {
        if (!mbar_wait(smem_u32(&s_full[t]), j & 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const bool diag = (j == qt);
        const int lim = qi - j * 128;  // diagonal block: last visible key of the row
        // the row's 128 scores into registers with four loads in flight
        float sv[128];
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld32_async(sbuf + c, sv + c);
        tmem_ld_wait();
#pragma unroll
        for (int c = 0; c < 128; c += 32) tmem_ld_fence(sv + c);
        // the diagonal block: keys past the row's own position get -inf (weight 0 below)
        if (diag) {
#pragma unroll
          for (int i = 0; i < 128; i++)
            if (i > lim) sv[i] = -INFINITY;
        }
        // row max of the raw scores (the scale is positive: applied to the max), three a step
        // on four independent chains
        float mc[4] = {sv[0], sv[1], sv[2], sv[3]};
#pragma unroll
        for (int i = 4; i < 124; i += 8)
#pragma unroll
          for (int k = 0; k < 4; k++) mc[k] = max3f(mc[k], sv[i + 2 * k], sv[i + 2 * k + 1]);
        mc[0] = max3f(mc[0], sv[124], sv[125]);
        mc[1] = max3f(mc[1], sv[126], sv[127]);
        const float mraw = max3f(mc[0], mc[1], fmaxf(mc[2], mc[3]));
        const float mx = mraw * a.scale_log2;
        // lazy rescale: move the reference max only when the row max grows by more than 8
        float m_new = m_ref, alpha = 1.f;
        if (j == 0) {
          m_new = mx;
        } else if (mx > m_ref + 8.f) {
          m_new = mx;
          alpha = ex2(m_ref - mx);
        }
        // P = 2^(s * scale - m) as bf16 pairs (the lower key in the low half) into the first
        // 64 columns of this tile's S in TMEM, where the P.V MMA reads it, and summed.  Scale,
        // offset and sum on packed fp32 pairs (masked keys: 2^-inf = 0 exactly).
        const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), nm2 = f2_pack(-m_new, -m_new);
        uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};  // four independent sums of pairs
#pragma unroll
        for (int hh = 0; hh < 2; hh++) {
          uint32_t w[32];
#pragma unroll
          for (int e = 0; e < 32; e++) {
            const int i = hh * 64 + 2 * e;
            const float2 x = f2_unpack(f2_fma(f2_pack(sv[i], sv[i + 1]), sc2, nm2));
            const float p0 = ex2(x.x), p1 = ex2(x.y);
            rs2[e & 3] = f2_add(rs2[e & 3], f2_pack(p0, p1));
            w[e] = bf2_pack_rn(p0, p1);
          }
          tmem_st32_nowait(sbuf + hh * 32, w);
        }
        const float2 rsf = f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])));
        const float rs = rsf.x + rsf.y;
        // O rescaled before P_t(j) V accumulates into it (s_full of block j also means that
        // P_t(j-1) V has completed; P_t(j) V is issued after p_full below)
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            float ov[32];
            tmem_ld32(obuf + c, ov);
#pragma unroll
            for (int i = 0; i < 32; i++) ov[i] *= alpha;
            tmem_st32(obuf + c, ov);
          }
        }
        l = l * alpha + rs;
        m_ref = m_new;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(smem_u32(&p_full[t]));
      }
      // the commit after the last P.V: O_t is final
      if (ok && mbar_wait(smem_u32(&s_full[t]), nbt & 1, abort_flag, a.err)) {
        tc_fence_after();
        const float inv = 1.0f / l;
        const long orow = a.out_rows ? a.out_rows[row0 + qi] : row0 + qi;
        bf16 *dst = a.out + orow * a.ldo + head * D;
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          float ov[32];
          tmem_ld32(obuf + c, ov);
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            float t8[8];
#pragma unroll
            for (int e = 0; e < 8; e++) t8[e] = ov[i + e] * inv;
            store8(dst + c + i, t8);
          }
        }
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

// SA of every (sequence, head, pair of query tiles): q/k/v from qkv_sa [T][3h], output into
// the SA half of attn [T][2h].
static bool tc_sa(dreamer_handle *h, cudaStream_t s, const int *out_rows) {
  using namespace dreamer;
  const dreamer_config &c = h->cfg;
  const int hd = c.hidden, d = c.head_dim;
  const long T = (long)c.batch * c.seq;
  CUtensorMap tm;
  if (!make_tmap(&tm, h->qkv_sa, 3 * hd, T, 3 * hd * 2, 64, 128)) return false;
  tc::SaArgs a{};
  a.S = c.seq; a.H = c.n_heads; a.h = hd; a.n_qt = c.seq / 128;
  a.n_pairs = (a.n_qt + 1) / 2;
  a.bh = c.batch * c.n_heads;
  a.out = (bf16 *)h->attn; a.ldo = 2 * hd;
  a.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  a.err = h->err;
  a.out_rows = out_rows;
  const int grid = a.bh * a.n_pairs;
  ++g_launches_tc;
  if (d == 64) {
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(tc::tc_sa_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SaCfg<64>::SMEM);
      set = true;
    }
    launch_k(h, tc::tc_sa_kernel<64>, dim3(grid), dim3(352), tc::SaCfg<64>::SMEM, s, tm, a);
  } else {
    static bool set = false;
    if (!set) {
      cudaFuncSetAttribute(tc::tc_sa_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SaCfg<128>::SMEM);
      set = true;
    }
    launch_k(h, tc::tc_sa_kernel<128>, dim3(grid), dim3(352), tc::SaCfg<128>::SMEM, s, tm, a);
  }
  return true;
}
