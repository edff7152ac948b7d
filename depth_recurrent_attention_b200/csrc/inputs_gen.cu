// Device-side copy of the seeded input generator (see depth_recurrent_attention_b200/
// inputs.py for the definition): splitmix64 outputs mix(key + (i + 1) * golden gamma),
// Box-Muller normals in float64, rounding float64 -> float32 -> bf16 (nearest even).
// This library draws inputs only; it holds none of the Dreamer method.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <cmath>

namespace {
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t raw(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * 0x9E3779B97F4A7C15ull);
}
__host__ __device__ __forceinline__ double u_open0(uint64_t r) {
  return (double)((r >> 11) + 1) * 0x1.0p-53;
}
// element i of the stream as float64
__host__ __device__ __forceinline__ double element(uint64_t key, uint64_t i, int kind, double p) {
  if (kind == 0) {
    uint64_t j = i >> 1;
    double u1 = u_open0(raw(key, 2 * j)), u2 = u_open0(raw(key, 2 * j + 1));
    double rad = sqrt(-2.0 * log(u1));
    double ang = 2.0 * 3.141592653589793 * u2;
    return ((i & 1) ? rad * sin(ang) : rad * cos(ang)) * p;
  }
  if (kind == 1) {
    double u = (double)(raw(key, i) >> 11) * 0x1.0p-53;
    return p * (2.0 * u - 1.0);
  }
  return 1.0;
}
// float32 bits -> bf16 bits, round to nearest even
__host__ __device__ __forceinline__ uint16_t bf16_bits(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  return (uint16_t)((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

__global__ void fill_kernel(void *out, uint64_t key, uint64_t start, uint64_t n, int kind,
                            double p, int dtype) {
  uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (; t < n; t += stride) {
    float f = (float)element(key, start + t, kind, p);
    if (dtype == 0) ((float *)out)[t] = f;
    else ((uint16_t *)out)[t] = bf16_bits(f);
  }
}
}  // namespace

// Host copy: float32 values of the dtype (bf16 values widened back to float32).
extern "C" int dri_fill_host(float *out, uint64_t key, uint64_t start, uint64_t n, int kind,
                             double p, int dtype) {
#pragma omp parallel for schedule(static)
  for (long long t = 0; t < (long long)n; t++) {
    float f = (float)element(key, start + (uint64_t)t, kind, p);
    if (dtype == 1) {
      uint32_t b = (uint32_t)bf16_bits(f) << 16;
      memcpy(&f, &b, 4);
    }
    out[t] = f;
  }
  return 0;
}

extern "C" int dri_fill(void *out, uint64_t key, uint64_t start, uint64_t n, int kind,
                        double p, int dtype, void *stream) {
  if (n == 0) return 0;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 32) blocks = 148 * 32;
  fill_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(out, key, start, n, kind, p, dtype);
  return (int)cudaGetLastError();
}
