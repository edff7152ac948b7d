// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05), bf16 in, fp32
// accumulated in TMEM:  C[r][n] = sum_k A[row(r)][k] * B_g[n][k]  for the sorted rows r of
// group g, B_g = rows g*b_group_rows + b_row0 .. of B (K contiguous).
//
// Roles (one CTA per SM, tiles of 128 x BN, K-blocks of BK):
//   warp 0      TMA producer: B tile (and A tile unless rows are gathered) per stage
//   warp 1      TMEM allocator + single-thread MMA issuer (tcgen05.mma, commit to barriers)
//   warps 2-5   epilogue: tcgen05.ld of the 128 x BN accumulator, row r per thread, then the
//               caller's epilogue functor on column segments of SEG values (EW = 8: warps
//               2-9, two per TMEM lane quarter, splitting the segments or column passes)
//   next GATHER (gathered rows only: 2 or 4 warps) A producers: 16-byte cp.async of the
//               rows into the 128B-swizzled layout TMA would have written (with four epilogue
//               warps and two gather warps the block stays at 8 warps, so the epilogue may use
//               up to 255 registers a thread)
// Two TMEM accumulators (2 x BN columns) let the epilogue of tile i overlap the MMAs of
// tile i+1.  Every wait is bounded (tc::mbar_wait); on expiry the CTA winds down and the
// device error flag is set.
#pragma once
#include <type_traits>

#include "tc_common.cuh"

namespace dreamer {
namespace tc {

struct TcGemmArgs {
  int N, K, G, M;
  const int *goffs;   // [G+1] sorted-row offsets or null (single group of M rows)
  const int *tiles;   // [G+1] cumulative 128-row tiles per group or null
  const int *arow;    // gathered source row of sorted row r (A row = arow[r] / arow_div)
  int arow_div;
  const bf16 *A;      // gather source [*][lda]
  long lda;
  int b_group_rows, b_row0;
  int *err;
  int skip_loads;     // test-hook build only: the TMA producer issues no loads (0 otherwise)
  const int2 *ttab;   // [tiles] (group, first row | rows << 24) of each 128-row tile, or null
  int mswz;           // row tiles a raster block: the N tiles of mswz row tiles run together
};

// per-row epilogue state: Epi::State for row-pass epilogues, nothing otherwise
struct NoEpiState {};
template <class Epi, bool ROWPASS> struct EpiState { using type = NoEpiState; };
template <class Epi> struct EpiState<Epi, true> { using type = typename Epi::State; };

// group and rows of a tile from its table entry
__device__ __forceinline__ bool tc_tile_unpack(int2 e, int &g, int &m0, int &m1) {
  g = e.x;
  m0 = e.y & 0xffffff;
  m1 = m0 + ((unsigned)e.y >> 24);
  return m0 < m1;
}
__device__ __forceinline__ bool tc_tile_rows(const TcGemmArgs &a, int mt, int &g, int &m0,
                                             int &m1) {
  if (a.goffs && a.ttab) return tc_tile_unpack(a.ttab[mt], g, m0, m1);
  if (!a.goffs) {
    g = 0;
    m0 = mt * 128;
    m1 = min(m0 + 128, a.M);
    return m0 < m1;
  }
  int lo = 0, hi = a.G - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (a.tiles[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  g = lo;
  m0 = a.goffs[g] + (mt - a.tiles[g]) * 128;
  m1 = min(m0 + 128, a.goffs[g + 1]);
  return m0 < m1;
}

// Epilogues that declare STAGED = true get the coalesced store path: each epilogue warp
// passes its 32 rows x up to 64 columns through shared memory so that a row's columns are
// spread over 8 lanes (transform<SEG> runs first in the row-per-thread layout, then
// store_rows<NIT, NV> in the coalesced one, with Epi::Aux values from row_aux(r, token)
// looked up once per tile for each of the lane's rows).
template <class E, class = void> struct EpiStaged { static constexpr bool value = false; };
template <class E> struct EpiStaged<E, std::void_t<decltype(E::STAGED)>> {
  static constexpr bool value = E::STAGED;
};
// Epilogues that declare TMA_STORE = true store plain bf16 rows [r][n] through a TMA tensor
// map (tmC, box 64 columns x 32 rows, 128-byte swizzle): each epilogue warp whose 32 rows are
// all valid writes its 32 x 64 block into a double-buffered shared-memory box and one lane
// issues the tile store; the warp that holds a group's last rows stores them one by one with
// the functor (rows past the group belong to the next group's tile).
template <class E, class = void> struct EpiTma { static constexpr bool value = false; };
template <class E> struct EpiTma<E, std::void_t<decltype(E::TMA_STORE)>> {
  static constexpr bool value = E::TMA_STORE;
};

template <int BN, int BK, int STAGES, int GATHER, bool STAGED = false, int EW_ = 4,
          bool ROWPASS = false, bool TMAST = false>
struct TcGemmCfg {
  static constexpr int A_BYTES = 128 * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int EW = EW_;  // epilogue warps: 4, or 8 (two per TMEM lane quarter)
  static_assert(EW == 4 || EW == 8, "epilogue warps");
  static_assert(GATHER == 0 || GATHER == 2 || GATHER == 4, "gather warps");
  static constexpr int THREADS = 64 + 32 * EW + 32 * GATHER;
  // staged epilogues: EW warps x 32 rows x 64 fp32; row-pass epilogues with two warps a lane
  // quarter: one exchange list of up to 16 (value, raw score, index) a row
  // TMA-store epilogues: two 4 KB boxes a warp, 1024-byte aligned after the barrier block
  static constexpr int STG_BYTES =
      STAGED ? EW * 32 * 64 * 4
             : ((ROWPASS && EW == 8) ? 128 * 16 * 12 : (TMAST ? 768 + EW * 2 * 4096 : 0));
  // at least 120 KB so that a second CTA never shares the SM (and its 512 TMEM columns)
  static constexpr int SMEM_USED =
      STAGES * (A_BYTES + B_BYTES) + 1024 /*align*/ + 256 /*bars*/ + STG_BYTES;
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static_assert(SMEM_USED <= 227 * 1024, "shared memory");
  static constexpr uint32_t IDESC = idesc_bf16_m128(BN);
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "N tile");
  static_assert(BK == 16 || BK == 32 || BK == 64, "K block");
  static_assert(!GATHER || BK == 64, "gathered rows use 128-byte K blocks");
};

// ROWPASS: a CTA takes row tiles mt = blockIdx.x, blockIdx.x + gridDim.x, ... and runs all
// N tiles of each in order, so the epilogue can carry per-row state across the N tiles
// (Epi::State with row_begin / row_apply / row_end); otherwise tiles are strided over CTAs.
template <int BN, int BK, int STAGES, int GATHER, int SEG, class Epi, bool ROWPASS = false,
          int EW = 4>
__global__ void __launch_bounds__(
    TcGemmCfg<BN, BK, STAGES, GATHER, EpiStaged<Epi>::value && !ROWPASS, EW, ROWPASS,
              EpiTma<Epi>::value>::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, TcGemmArgs a, Epi epi) {
  constexpr bool STAGED = EpiStaged<Epi>::value && !ROWPASS;
  constexpr bool TMAST = EpiTma<Epi>::value && !STAGED && !ROWPASS;
  static_assert(!TMAST || SEG == 64, "TMA-store epilogue: 64-column segments");
  using C = TcGemmCfg<BN, BK, STAGES, GATHER, STAGED, EW, ROWPASS, TMAST>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * C::A_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + STAGES * C::B_BYTES);
  uint64_t *full = bars, *empty = bars + STAGES, *tfull = bars + 2 * STAGES, *tempty = tfull + 2;
  uint64_t *xfull = tempty + 2, *xempty = xfull + 4;  // row-pass list exchange, per lane quarter
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(xempty + 4);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  float *stage_buf = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(bars) + 256);
  uint8_t *tma_box = reinterpret_cast<uint8_t *>(bars) + 1024;  // TMAST: 1024-byte aligned

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NT = a.N / BN;
  int mtiles = 0, total = 0;  // read after pdl_wait: the tile table may come from the last kernel
  const int KB = a.K / BK;
  // the i-th tile of this CTA (identical sequence in every role); false past the last one
  auto tile_at = [&](int i, int &mt, int &nt) -> bool {
    if (ROWPASS) {
      mt = blockIdx.x + (i / NT) * gridDim.x;
      nt = i % NT;
      return mt < mtiles;
    }
    // blocks of mswz row tiles; inside a block the row tile changes fastest, so the CTAs
    // working at one time share each B tile (and the block's A tiles stay in L2)
    const int t = blockIdx.x + i * gridDim.x;
    if (a.mswz <= 1) {
      mt = t / NT;
      nt = t % NT;
      return t < total;
    }
    if (t >= total) {
      mt = nt = 0;
      return false;
    }
    const int sw = a.mswz;
    const int per = sw * NT, blk = t / per, u = t - blk * per;
    const int rows = min(sw, mtiles - blk * sw);  // >= 1 since t < mtiles * NT
    nt = u / rows;
    mt = blk * sw + u % rows;
    return true;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(smem_u32(&full[s]), 1 + 32 * GATHER);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(smem_u32(&tfull[i]), 1);
      mbar_init(smem_u32(&tempty[i]), 32 * C::EW);
    }
    for (int i = 0; i < 4; i++) {
      mbar_init(smem_u32(&xfull[i]), 32);
      mbar_init(smem_u32(&xempty[i]), 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmB);
    if (!GATHER) prefetch_tmap(&tmA);
    if (TMAST) prefetch_tmap(&tmC);
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
  mtiles = a.goffs ? a.tiles[a.G] : (a.M + 127) / 128;
  total = mtiles * NT;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      int issued_ph[STAGES];
      for (int i = 0; i < STAGES; i++) issued_ph[i] = -1;
      bool ok = true;
      int mt, nt;
#ifdef DREAMER_TEST_HOOKS
      // the timeout test: no operand ever arrives, so the MMA issuer's bounded wait expires
      if (a.skip_loads) ok = false;
#endif
      // grouped rows: each tile's table entry requested two tiles ahead, so a tile of a single
      // K block does not wait a memory round trip before its loads are issued
      const bool tab = a.goffs && a.ttab;
      auto entry = [&](int i) -> int2 {
        int m_, n_;
        return (tab && tile_at(i, m_, n_)) ? a.ttab[m_] : make_int2(0, 0);
      };
      int2 e1 = entry(0), e2 = entry(1);
      for (int i = 0; ok && tile_at(i, mt, nt); i++) {
        int g, m0, m1;
        const int n0 = nt * BN;
        const int2 e0 = e1;
        e1 = e2;
        e2 = entry(i + 2);
        if (tab) tc_tile_unpack(e0, g, m0, m1);
        else tc_tile_rows(a, mt, g, m0, m1);
        const int brow = g * a.b_group_rows + a.b_row0 + n0;
        for (int kb = 0; kb < KB; kb++) {
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_expect_tx(fb, GATHER ? C::B_BYTES : C::A_BYTES + C::B_BYTES);
          if (!GATHER) tma_load_2d(smem_u32(sA + s * C::A_BYTES), &tmA, fb, kb * BK, m0);
          tma_load_2d(smem_u32(sB + s * C::B_BYTES), &tmB, fb, kb * BK, brow);
          issued_ph[s] = (int)ph;
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        for (int i = 0; i < STAGES; i++)
          if (issued_ph[i] >= 0) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(smem_u32(&full[i]), (uint32_t)issued_ph[i]) &&
                   globaltimer() - t0 < WAIT_LIMIT_NS) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int mt, nt;
      for (int it = 0; ok && tile_at(it, mt, nt); it++) {
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(smem_u32(&tempty[acc]), aph ^ 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * BN;
        for (int kb = 0; kb < KB; kb++) {
          if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, a.err)) { ok = false; break; }
          tc_fence_after();
          if (GATHER) fence_proxy_async();
          const uint32_t a0 = smem_u32(sA + s * C::A_BYTES), b0 = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 16; k++)
            mma_bf16(d, smem_desc(a0 + k * 32, BK * 2), smem_desc(b0 + k * 32, BK * 2), C::IDESC,
                     (kb | k) != 0);
          mma_commit(smem_u32(&empty[s]));
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (ok) mma_commit(smem_u32(&tfull[acc]));
      }
    }
  } else if (warp < 2 + C::EW) {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int half = (warp - 2) >> 2;       // which of the quarter's warps (0, or 1 with 8)
    const int row = q * 32 + lane;
    int mt, nt;
    typename EpiState<Epi, ROWPASS>::type st;
    int rb = 0;  // row blocks finished (row-pass exchange phase)
    int nbox = 0;  // TMAST: tile stores issued by this warp (alternating shared-memory boxes)
    for (int it = 0; tile_at(it, mt, nt); it++) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      int g, m0, m1;
      const int n0 = nt * BN;
      tc_tile_rows(a, mt, g, m0, m1);
      const int r = m0 + row;
      const bool valid = r < m1;
      const int token = valid ? (a.arow ? a.arow[r] / a.arow_div : r) : 0;
      const uint32_t base = tmem + acc * BN + ((uint32_t)(q * 32) << 16);
      if constexpr (STAGED) {
        // Passes of PW = min(SEG, 64) columns.  With PW = 64 lane j of a row holds columns
        // 4j..4j+3 and 32+4j..32+4j+3 (NV = 8), so rotate-half partners 32 apart meet in
        // one lane; 8 lanes cover a row, 4 rows a step.  PW = 32: 4 columns a lane (NV = 4).
        // PW = 16: 4 lanes a row, 8 rows a step.
        constexpr int PW = SEG < 64 ? SEG : 64;
        constexpr int CPR = PW / 4;                 // 16-byte chunks per staged row
        constexpr int LPR = PW == 16 ? 4 : 8;       // lanes per row in the coalesced phase
        constexpr int NV = PW == 64 ? 8 : 4;        // values per lane and row
        constexpr int RPI = 32 / LPR;               // rows per step
        constexpr int NIT = 32 / RPI;               // steps per pass
        constexpr int SW = CPR >= 8 ? 7 : CPR - 1;  // chunk swizzle mask
        float *stg = stage_buf + (warp - 2) * 32 * 64;
        const int cj = lane % LPR;
        // the lane's rows, their per-row values and an L2 prefetch of the tile's inputs, all
        // while the MMAs of this tile are still running
        int crow[NIT], ctok[NIT];
        typename Epi::Aux caux[NIT];
#pragma unroll
        for (int i = 0; i < NIT; i++) {
          const int rr = m0 + q * 32 + i * RPI + lane / LPR;
          crow[i] = rr < m1 ? rr : -1;
          ctok[i] = rr < m1 ? (a.arow ? a.arow[rr] / a.arow_div : rr) : 0;
          caux[i] = epi.row_aux(crow[i], ctok[i]);
        }
        constexpr int NPW = C::EW / 4;  // warps sharing a lane quarter; they split the passes
        epi.template prefetch<NIT>(crow, ctok, caux, n0, BN, cj + half * LPR, LPR * NPW);
        if (!mbar_wait(smem_u32(&tfull[acc]), aph, abort_flag, a.err)) break;
        tc_fence_after();
        // passes of PW columns; pass p of the tile belongs to warp half p % NPW
#pragma unroll 1
        for (int p = half; p < BN / PW && m0 + q * 32 < m1; p += NPW) {
          const int c0 = p * PW;
          __syncwarp();
#pragma unroll
          for (int c = 0; c < PW; c += 32) {  // TMEM -> row-layout transform -> shared memory
            constexpr int W = PW < 32 ? PW : 32;
            float v[W];
            if (W == 32) tmem_ld32(base + c0 + c, v);
            else tmem_ld16(base + c0 + c, v);
            if (valid) epi.template transform<W>(r, token, g, n0 + c0 + c, v);
#pragma unroll
            for (int j = 0; j < W / 4; j++)
              *reinterpret_cast<float4 *>(stg + lane * PW + (((c / 4 + j) ^ (lane & SW)) << 2)) =
                  make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          __syncwarp();
          float cv[NIT][NV];
#pragma unroll
          for (int i = 0; i < NIT; i++) {
            const int rl = i * RPI + lane / LPR;
#pragma unroll
            for (int hh = 0; hh < NV / 4; hh++) {
              const int ch = cj + hh * 8;
              const float4 t4 = *reinterpret_cast<const float4 *>(stg + rl * PW + ((ch ^ (rl & SW)) << 2));
              cv[i][4 * hh] = t4.x; cv[i][4 * hh + 1] = t4.y;
              cv[i][4 * hh + 2] = t4.z; cv[i][4 * hh + 3] = t4.w;
            }
          }
          epi.template store_rows<NIT, NV>(crow, ctok, caux, g, n0 + c0 + cj * 4, cv);
        }
      } else if constexpr (TMAST) {
        if (!mbar_wait(smem_u32(&tfull[acc]), aph, abort_flag, a.err)) break;
        tc_fence_after();
        const bool full_warp = m0 + q * 32 + 31 < m1;
#pragma unroll 1
        for (int sg = half; sg < BN / 64 && m0 + q * 32 < m1; sg += C::EW / 4) {
          float v[64];
          tmem_ld32(base + sg * 64, v);
          tmem_ld32(base + sg * 64 + 32, v + 32);
          if (full_warp) {
            uint8_t *box = tma_box + ((warp - 2) * 2 + (nbox & 1)) * 4096;
            if (lane == 0) bulk_wait_read<1>();  // this box's store of two passes ago has read it
            __syncwarp();
            // row `lane` of the box: 16-byte chunk c at (c ^ (lane & 7)), the 128-byte swizzle
#pragma unroll
            for (int c = 0; c < 8; c++) {
              uint4 pk;
              __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&pk);
#pragma unroll
              for (int j = 0; j < 4; j++) p2[j] = __floats2bfloat162_rn(v[8 * c + 2 * j], v[8 * c + 2 * j + 1]);
              *reinterpret_cast<uint4 *>(box + lane * 128 + ((c ^ (lane & 7)) << 4)) = pk;
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmC, smem_u32(box), n0 + sg * 64, m0 + q * 32);
              bulk_commit();
            }
            nbox++;
          } else if (valid) {
            epi.template operator()<64>(r, token, g, n0 + sg * 64, v);
          }
        }
      } else {
        if (!mbar_wait(smem_u32(&tfull[acc]), aph, abort_flag, a.err)) break;
        tc_fence_after();
        if constexpr (ROWPASS) {
          if (nt == 0) epi.row_begin(st);
        }
        // segments of SEG columns; with eight epilogue warps segment sg belongs to half sg % 2
#pragma unroll 1
        for (int sg = half; sg < BN / SEG && m0 + q * 32 < m1; sg += C::EW / 4) {  // skip warps with no rows
          float v[SEG];
          if (SEG >= 32) {
#pragma unroll
            for (int c = 0; c < SEG; c += 32) tmem_ld32(base + sg * SEG + c, v + c);
          } else {
            tmem_ld16(base + sg * SEG, v);
          }
          if (valid) {
            if constexpr (ROWPASS) epi.template row_apply<SEG>(st, r, token, g, n0 + sg * SEG, v);
            else epi.template operator()<SEG>(r, token, g, n0 + sg * SEG, v);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&tempty[acc]));
      if constexpr (ROWPASS) {
        if (nt == NT - 1) {
          if constexpr (C::EW == 8) {
            // the quarter's two warps hold lists over alternate segments: half 1 hands its
            // list over, half 0 merges and finishes the row
            epi.row_end_pair(st, r, token, valid, half, q * 32 + lane,
                             reinterpret_cast<uint8_t *>(stage_buf), xfull + q, xempty + q, rb,
                             abort_flag, a.err);
            rb++;
          } else if (valid) {
            epi.row_end(st, r, token);
          }
        }
      }
    }
    if constexpr (TMAST) {
      if (lane == 0) bulk_wait_all();  // every tile store of this warp has landed
    }
  } else if (GATHER) {
    // ------------------------------------------------------------- gathered A producers
    constexpr int GT = 32 * (GATHER > 0 ? GATHER : 2), RSUB = GT / 8, NP = 128 / RSUB;
    const int tid = threadIdx.x - (64 + 32 * C::EW);  // 0..GT-1
    const int c = tid & 7;              // 16-byte chunk of the 128-byte row slice
    const int rsub = tid >> 3;          // 0..RSUB-1
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      int g, m0, m1;
      const int mt = t / NT;
      tc_tile_rows(a, mt, g, m0, m1);
      const bf16 *src[NP];
      uint32_t bytes[NP];
#pragma unroll
      for (int p = 0; p < NP; p++) {
        const int rr = p * RSUB + rsub, r = m0 + rr;
        const bool v = r < m1;
        src[p] = a.A + (v ? (long)(a.arow[r] / a.arow_div) * a.lda : 0) + c * 8;
        bytes[p] = v ? 16u : 0u;
      }
      for (int kb = 0; kb < KB; kb++) {
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
        const uint32_t dst0 = smem_u32(sA + s * C::A_BYTES);
#pragma unroll
        for (int p = 0; p < NP; p++) {
          const int rr = p * RSUB + rsub;
          cp_async16(dst0 + rr * 128 + ((c ^ (rr & 7)) << 4), src[p] + kb * 64, bytes[p]);
        }
        cp_async_arrive(smem_u32(&full[s]));
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
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
