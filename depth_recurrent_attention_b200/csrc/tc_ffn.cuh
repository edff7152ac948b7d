// Fused expert FFN on the tensor cores (papernotes "Key design 2": each expert is a small SiLU
// FFN that acts as the value transform of expert attention).  One tile = up to 128 routed rows
// of one expert e, in expert-sorted order:
//   phase 1   H = SiLU(X_rows W1_e)           [128 x m], K = h, fp32 in TMEM
//             -> rounded to bf16 into shared memory, in the K-major swizzled layout that
//                tcgen05.mma reads (the layout TMA writes for a box m elements wide)
//   phase 2   Y_rows = H W2_e in chunks of 256 output columns, K = m, each chunk stored in
//             dtype to Y[sorted row]: an epilogue warp whose 32 rows all belong to the tile
//             writes its 32 x 64 blocks into shared-memory boxes and stores them with TMA
//             (tensor map tmY); the warp holding the expert's last rows stores row by row
// H never leaves the SM.  Rounding points are those of the two-GEMM form (H in bf16, Y in
// bf16), so the result is the same.
//
// Roles (one CTA per SM, tiles strided over CTAs):
//   warp 0      TMA producer: W1_e blocks [m x 64] per stage, W2_e chunks [256 x m]
//   warp 1      TMEM allocator (512 columns) + single-thread MMA issuer
//   warps 2-5   epilogue (TMEM lane quarter warp % 4): SiLU -> H, then the Y chunks
//   warps 6-7   gathered X rows (16-byte cp.async into the 128-byte swizzled layout)
// TMEM is used as two regions of 256 columns; accumulation jobs (a tile's phase 1, then its
// chunks) take regions in turn, so a chunk's epilogue overlaps the next job's MMAs.  Every
// wait is bounded (tc::mbar_wait); on expiry the CTA winds down and the device error flag
// is set.
#pragma once
#include "tc_common.cuh"

namespace dreamer {
namespace tc {

struct TcFfnArgs {
  int H, G, M;         // hidden size (a multiple of 256), experts, routed rows
  const int *goffs;    // [G+1] sorted-row offsets
  const int *tiles;    // [G+1] cumulative 128-row tiles
  const int *arow;     // X row of sorted row r = arow[r] / arow_div
  int arow_div;
  const bf16 *X;
  long ldx;
  bf16 *Y;             // [rows][H], expert-sorted order
  int *err;
  const int2 *ttab;    // [tiles] (expert, first row | rows << 24) of each tile, or null
};

template <int M, int STAGES>
struct TcFfnCfg {
  static_assert(M == 16 || M == 32 || M == 64, "expert hidden size");
  static constexpr int A_BYTES = 128 * 64 * 2;   // 128 gathered rows x one 64-element K block
  static constexpr int B1_BYTES = M * 64 * 2;    // W1_e^T: M rows x 64 K
  static constexpr int B2_BYTES = 256 * M * 2;   // W2_e^T chunk: 256 rows x M K
  static constexpr int H_BYTES = 128 * M * 2;
  static constexpr int THREADS = 256;
  static constexpr int BOX_BYTES = 4 * 2 * 4096;  // two 32 x 64 bf16 boxes per epilogue warp
  static constexpr int SMEM_USED = STAGES * (A_BYTES + B1_BYTES) + 2 * B2_BYTES + H_BYTES +
                                   1024 /*align*/ + 1024 /*bars*/ + BOX_BYTES;
  // at least 120 KB so that a second CTA never shares the SM (and its 512 TMEM columns)
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static_assert(SMEM_USED <= 227 * 1024, "shared memory");
  static constexpr uint32_t IDESC1 = idesc_bf16_m128(M);
  static constexpr uint32_t IDESC2 = idesc_bf16_m128(256);
};

__device__ __forceinline__ void ffn_tile_rows(const TcFfnArgs &a, int mt, int &g, int &m0,
                                              int &m1) {
  if (a.ttab) {
    const int2 e = a.ttab[mt];
    g = e.x;
    m0 = e.y & 0xffffff;
    m1 = m0 + ((unsigned)e.y >> 24);
    return;
  }
  int lo = 0, hi = a.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.tiles[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  g = lo;
  m0 = a.goffs[g] + (mt - a.tiles[g]) * 128;
  m1 = min(m0 + 128, a.goffs[g + 1]);
}

// 16-byte chunk c of row r of a K-major tile whose rows are 2M bytes wide, placed as the
// matching TMA swizzle mode does it (128-, 64- or 32-byte pattern: address bits 4.. XOR
// address bits 7..)
template <int M>
__device__ __forceinline__ int ffn_swz(int r, int c) {
  if (M == 64) return c ^ (r & 7);
  if (M == 32) return c ^ ((r >> 1) & 3);
  return c ^ ((r >> 2) & 1);
}

template <int M, int STAGES>
__global__ void __launch_bounds__(256, 1)
    tc_ffn_kernel(const __grid_constant__ CUtensorMap tmW1, const __grid_constant__ CUtensorMap tmW2,
                  const __grid_constant__ CUtensorMap tmY, TcFfnArgs a) {
  using C = TcFfnCfg<M, STAGES>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem;
  uint8_t *sB1 = sA + STAGES * C::A_BYTES;
  uint8_t *sB2 = sB1 + STAGES * C::B1_BYTES;
  uint8_t *sH = sB2 + 2 * C::B2_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sH + C::H_BYTES);
  uint64_t *full = bars, *empty = full + STAGES;      // phase-1 operand ring
  uint64_t *b2full = empty + STAGES, *b2empty = b2full + 2;  // W2 chunk double buffer
  uint64_t *rfull = b2empty + 2, *rempty = rfull + 2;        // TMEM regions
  uint64_t *hready = rempty + 2, *hfree = hready + 1;        // H in shared memory
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(hfree + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  uint8_t *sbox = reinterpret_cast<uint8_t *>(bars) + 1024;  // 1024-byte aligned store boxes

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = a.H / 64, NC = a.H / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; s++) {
      mbar_init(smem_u32(&full[s]), 1 + 64);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int i = 0; i < 2; i++) {
      mbar_init(smem_u32(&b2full[i]), 1);
      mbar_init(smem_u32(&b2empty[i]), 1);
      mbar_init(smem_u32(&rfull[i]), 1);
      mbar_init(smem_u32(&rempty[i]), 128);
    }
    mbar_init(smem_u32(hready), 128);
    mbar_init(smem_u32(hfree), 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmW1);
    prefetch_tmap(&tmW2);
    prefetch_tmap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();     // the routing tables of the previous kernels are visible from here on
  pdl_trigger();  // after the TMEM allocation (see pdl_trigger)
  const int total = a.tiles[a.G];

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0, q = 0;
      uint32_t ph = 0;
      int issued_ph[STAGES], b2_ph[2] = {-1, -1};
      for (int i = 0; i < STAGES; i++) issued_ph[i] = -1;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
        int g, m0, m1;
        ffn_tile_rows(a, t, g, m0, m1);
        for (int kb = 0; kb < KB; kb++) {
          if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_expect_tx(fb, C::B1_BYTES);
          tma_load_2d(smem_u32(sB1 + s * C::B1_BYTES), &tmW1, fb, kb * 64, g * M);
          issued_ph[s] = (int)ph;
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        for (int c = 0; ok && c < NC; c++, q++) {
          const int slot = q & 1;
          const uint32_t qph = (q >> 1) & 1;
          if (!mbar_wait(smem_u32(&b2empty[slot]), qph ^ 1, abort_flag, a.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&b2full[slot]);
          mbar_expect_tx(fb, C::B2_BYTES);
          tma_load_2d(smem_u32(sB2 + slot * C::B2_BYTES), &tmW2, fb, 0, g * a.H + c * 256);
          b2_ph[slot] = (int)qph;
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
        for (int i = 0; i < 2; i++)
          if (b2_ph[i] >= 0) {
            const uint64_t t0 = globaltimer();
            while (!mbar_try_wait(smem_u32(&b2full[i]), (uint32_t)b2_ph[i]) &&
                   globaltimer() - t0 < WAIT_LIMIT_NS) {
            }
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, q = 0, j = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < total; t += gridDim.x, it++) {
        // phase 1: H accumulator of the tile in region j % 2
        {
          const int rg = j & 1;
          if (!mbar_wait(smem_u32(&rempty[rg]), ((j >> 1) & 1) ^ 1, abort_flag, a.err)) break;
          tc_fence_after();
          const uint32_t d = tmem + rg * 256;
          for (int kb = 0; kb < KB; kb++) {
            if (!mbar_wait(smem_u32(&full[s]), ph, abort_flag, a.err)) { ok = false; break; }
            tc_fence_after();
            fence_proxy_async();  // the gathered rows were written by cp.async
            const uint32_t a0 = smem_u32(sA + s * C::A_BYTES), b0 = smem_u32(sB1 + s * C::B1_BYTES);
#pragma unroll
            for (int k = 0; k < 4; k++)
              mma_bf16(d, smem_desc(a0 + k * 32, 128), smem_desc(b0 + k * 32, 128), C::IDESC1,
                       (kb | k) != 0);
            mma_commit(smem_u32(&empty[s]));
            if (++s == STAGES) { s = 0; ph ^= 1; }
          }
          if (!ok) break;
          mma_commit(smem_u32(&rfull[rg]));
          j++;
        }
        // phase 2: the epilogue has written H of this tile
        if (!mbar_wait(smem_u32(hready), it & 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t h0 = smem_u32(sH);
        for (int c = 0; c < NC; c++, q++, j++) {
          const int rg = j & 1, slot = q & 1;
          if (!mbar_wait(smem_u32(&rempty[rg]), ((j >> 1) & 1) ^ 1, abort_flag, a.err) ||
              !mbar_wait(smem_u32(&b2full[slot]), (q >> 1) & 1, abort_flag, a.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + rg * 256, b0 = smem_u32(sB2 + slot * C::B2_BYTES);
#pragma unroll
          for (int k = 0; k < M / 16; k++)
            mma_bf16(d, smem_desc(h0 + k * 32, 2 * M), smem_desc(b0 + k * 32, 2 * M), C::IDESC2,
                     k != 0);
          mma_commit(smem_u32(&b2empty[slot]));
          mma_commit(smem_u32(&rfull[rg]));
        }
        if (!ok) break;
        mma_commit(smem_u32(hfree));  // H may be overwritten once these MMAs have read it
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------- epilogue
    const int qq = warp & 3;  // TMEM lane quarter
    const int row = qq * 32 + lane;
    int j = 0, it = 0, nbox = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x, it++) {
      int g, m0, m1;
      ffn_tile_rows(a, t, g, m0, m1);
      const int r = m0 + row;
      const bool valid = r < m1;
      {
        const int rg = j & 1;
        if (!mbar_wait(smem_u32(&rfull[rg]), (j >> 1) & 1, abort_flag, a.err)) break;
        if (it > 0 && !mbar_wait(smem_u32(hfree), (it - 1) & 1, abort_flag, a.err)) break;
        tc_fence_after();
        const uint32_t base = tmem + rg * 256 + ((uint32_t)(qq * 32) << 16);
        float v[M];
        if (M == 16) {
          tmem_ld16(base, v);
        } else {
#pragma unroll
          for (int c = 0; c < M; c += 32) tmem_ld32(base + c, v + c);
        }
        // SiLU in fp32, rounded to bf16 (rows past the tile's end hold SiLU(0) = 0)
        uint8_t *hrow = sH + row * (2 * M);
#pragma unroll
        for (int c = 0; c < M / 8; c++) {
          float u[8];
#pragma unroll
          for (int i = 0; i < 8; i++) u[i] = v[8 * c + i] / (1.0f + __expf(-v[8 * c + i]));
          store8(reinterpret_cast<bf16 *>(hrow + (ffn_swz<M>(row, c) << 4)), u);
        }
        fence_proxy_async();  // make the H rows visible to the tensor cores
        tc_fence_before();
        mbar_arrive(smem_u32(&rempty[rg]));
        mbar_arrive(smem_u32(hready));
        j++;
      }
      for (int c = 0; c < NC; c++, j++) {
        const int rg = j & 1;
        if (!mbar_wait(smem_u32(&rfull[rg]), (j >> 1) & 1, abort_flag, a.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = tmem + rg * 256 + ((uint32_t)(qq * 32) << 16);
        bf16 *yr = a.Y + (long)r * a.H + c * 256;
        const bool full_warp = m0 + qq * 32 + 31 < m1;
#pragma unroll 1
        for (int sg = 0; sg < 256; sg += 64) {
          float v[64];
          tmem_ld32(base + sg, v);
          tmem_ld32(base + sg + 32, v + 32);
          if (full_warp) {
            uint8_t *box = sbox + ((warp - 2) * 2 + (nbox & 1)) * 4096;
            if (lane == 0) bulk_wait_read<1>();  // this box's store of two passes ago has read it
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 8; q++) {  // 16-byte chunk q of the row at (q ^ (lane & 7))
              uint4 pk;
              __nv_bfloat162 *p2 = reinterpret_cast<__nv_bfloat162 *>(&pk);
#pragma unroll
              for (int e = 0; e < 4; e++) p2[e] = __floats2bfloat162_rn(v[8 * q + 2 * e], v[8 * q + 2 * e + 1]);
              *reinterpret_cast<uint4 *>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) = pk;
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tmY, smem_u32(box), c * 256 + sg, m0 + qq * 32);
              bulk_commit();
            }
            nbox++;
          } else if (valid) {
#pragma unroll
            for (int i = 0; i < 64; i += 8) store8(yr + sg + i, v + i);
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&rempty[rg]));
      }
    }
    if (lane == 0) bulk_wait_all();  // every tile store of this warp has landed
  } else {
    // ------------------------------------------------------------- gathered X rows
    const int tid = threadIdx.x - 192;  // 0..63
    const int c = tid & 7;              // 16-byte chunk of the 128-byte row slice
    const int rsub = tid >> 3;          // 0..7
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total; t += gridDim.x) {
      int g, m0, m1;
      ffn_tile_rows(a, t, g, m0, m1);
      const bf16 *src[16];
      uint32_t bytes[16];
#pragma unroll
      for (int p = 0; p < 16; p++) {
        const int rr = p * 8 + rsub, r = m0 + rr;
        const bool v = r < m1;
        src[p] = a.X + (v ? (long)(a.arow[r] / a.arow_div) * a.ldx : 0) + c * 8;
        bytes[p] = v ? 16u : 0u;
      }
      for (int kb = 0; kb < KB; kb++) {
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1, abort_flag, a.err)) { ok = false; break; }
        const uint32_t dst0 = smem_u32(sA + s * C::A_BYTES);
#pragma unroll
        for (int p = 0; p < 16; p++) {
          const int rr = p * 8 + rsub;
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
