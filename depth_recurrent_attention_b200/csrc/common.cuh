// Shared device helpers for libdreamer (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dreamer {

typedef __nv_bfloat16 bf16;

// ---- element conversion ---------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// 8 consecutive elements <-> float[8]
__device__ __forceinline__ void load8(const float *p, float *o) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  float4 b = *reinterpret_cast<const float4 *>(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const bf16 *p, float *o) {
  uint4 u = *reinterpret_cast<const uint4 *>(p);
  const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; i++) {
    float2 f = __bfloat1622float2(h2[i]);
    o[2 * i] = f.x;
    o[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(float *p, const float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(bf16 *p, const float *v) {
  uint4 u;
  __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; i++) h2[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}

// 4 consecutive elements <-> float[4]
__device__ __forceinline__ void load4(const float *p, float *o) {
  float4 a = *reinterpret_cast<const float4 *>(p);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
}
__device__ __forceinline__ void load4(const bf16 *p, float *o) {
  uint2 u = *reinterpret_cast<const uint2 *>(p);
  const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
  float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
  o[0] = f0.x; o[1] = f0.y; o[2] = f1.x; o[3] = f1.y;
}
__device__ __forceinline__ void store4(float *p, const float *v) {
  *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16 *p, const float *v) {
  uint2 u;
  __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&u);
  h2[0] = __floats2bfloat162_rn(v[0], v[1]);
  h2[1] = __floats2bfloat162_rn(v[2], v[3]);
  *reinterpret_cast<uint2 *>(p) = u;
}

// L2 prefetch of the 128-byte line holding p
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + __expf(-x)); }

// Routing weights w_s = sigmoid(z_s) / sum_j sigmoid(z_j) over a token's picks, formed as
// exp(ls_s - m) / sum_j exp(ls_j - m) from ls = log sigmoid(z) = min(z, 0) - log(1 + e^-|z|)
// and m = max_j ls_j: the same ratio, finite for every finite z (sigmoids that underflow to
// 0 would give 0/0).
__device__ __forceinline__ float log_sigmoidf_(float z) {
  return fminf(z, 0.f) - log1pf(expf(-fabsf(z)));
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic): {lo, hi} in one 64-bit register ---------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// max of three floats in one instruction
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// two floats rounded to bf16 in one 32-bit word (lo in the low half)
__device__ __forceinline__ uint32_t bf2_pack_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Programmatic dependent launch.  Every kernel of the library calls pdl_wait() before its
// first global memory access (and before any early return), so it may be launched while the
// previous kernel on its stream is still draining; pdl_trigger() lets the next kernel's blocks
// be scheduled.  Kernels that allocate TMEM trigger only after their allocation, so a
// dependent block can never take the columns a running block still needs.  Both are no-ops
// for a kernel launched without the programmatic-serialization attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Device-side error codes written into the handle's flag word (first writer wins).
enum DevErr : int { DEV_OK = 0, DEV_TIMEOUT = 1, DEV_BAD_INDEX = 2 };

// Limit of every bounded device wait (an mbarrier phase, copies in flight), in nanoseconds of
// %globaltimer; on expiry a kernel sets DEV_TIMEOUT and winds down.  The test-hook build
// shortens it so that its timeout test ends quickly.
#ifndef DREAMER_WAIT_LIMIT_NS
#define DREAMER_WAIT_LIMIT_NS 2000000000ull
#endif
__device__ __forceinline__ void raise_dev_error(int *flag, int code) {
  if (flag) atomicCAS(flag, 0, code);
}

}  // namespace dreamer
