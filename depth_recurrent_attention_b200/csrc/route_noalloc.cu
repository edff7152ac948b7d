// Expert routing that allocates no device memory.
//
// Some callers cannot call cudaMalloc on the path where they route: a host application that
// hands the whole device memory to its own pool at start-up and forbids outside allocations,
// a real-time loop where an allocation (which may synchronise the device) is not acceptable,
// or a plugin that only ever receives buffers from its host.  dreamer_route_experts_noalloc
// serves them: it needs no handle, the caller passes inputs, weights and outputs, and the one
// piece of scratch it uses (the expert keys turned by the depth RoPE of the requested depth)
// lives in a fixed array inside this library.
//
// The array is a file-scope __device__ variable of ROUTE_NOALLOC_SCRATCH_FLOATS floats (4 MiB).
// Every GPU that loads the library holds it until the process exits.  All calls share it and
// it keeps the previous call's contents, so calls that overlap on the GPU (two streams, or two
// host threads) race on it: serialise them.  The first call on a device looks up the array's
// device address (cudaGetSymbolAddress) and caches it; make that first call before any stream
// capture on that device.  The cached address belongs to the CUDA context current at that
// first call: it is keyed by device and context, so a new context on the device (after
// cudaDeviceReset, or another context made current) looks the address up again.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "../../include/dreamer.h"
#include "common.cuh"

namespace {

constexpr size_t ROUTE_NOALLOC_SCRATCH_FLOATS = size_t(1) << 20;  // E * d_r <= 1,048,576
static __device__ __align__(256) float g_route_scratch[ROUTE_NOALLOC_SCRATCH_FLOATS];

constexpr int MAX_DEVICES = 64;
static float *g_scratch_addr[MAX_DEVICES] = {nullptr};
static void *g_scratch_ctx[MAX_DEVICES] = {nullptr};  // context the cached address belongs to
static std::mutex g_scratch_mu;

// The CUDA context current on this thread (driver entry point through the runtime, so the
// library needs no link against the driver library); NULL if it cannot be read.
static void *current_context() {
  typedef CUresult (*PFN_ctx_t)(CUcontext *);
  static PFN_ctx_t fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_ctx_t)f;
    looked = true;
  }
  CUcontext c = nullptr;
  if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
  return (void *)c;
}

// Device address of the scratch array on the current device and context (looked up once per
// device and context; in host code the symbol name is only a host-side stand-in and must never
// reach a kernel).
static int scratch_on_current_device(float **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DREAMER_ERR_CUDA;
  if (dev < 0 || dev >= MAX_DEVICES) return DREAMER_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev] || current_context() != g_scratch_ctx[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || !p) return DREAMER_ERR_CUDA;
    g_scratch_addr[dev] = static_cast<float *>(p);
    g_scratch_ctx[dev] = current_context();  // current now: the lookup initialised it
  }
  *out = g_scratch_addr[dev];
  return DREAMER_OK;
}

// Keys of depth l: each key split into halves of d_r/2, each half turned by rotate-half RoPE
// over d_r/2 dims, the first at position l, the second at L-1-l (the depth RoPE of the
// expert keys).  One thread per (expert, pair); angles in double.
template <typename T>
__global__ void rotate_keys_kernel(const T *kE, int E, int dr, int l, int L, double base,
                                   float *out) {
  const int q = dr / 4;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long)E * 2 * q) return;
  const int e = (int)(i / (2 * q)), r = (int)(i % (2 * q));
  const int half = r / q, p = r % q;
  const double pos = half == 0 ? (double)l : (double)(L - 1 - l);
  double sn, cs;
  sincos(pos * pow(base, -2.0 * p / (double)(dr / 2)), &sn, &cs);
  const T *src = kE + (long)e * dr + half * (dr / 2);
  float *dst = out + (long)e * dr + half * (dr / 2);
  const double a = dreamer::to_f(src[p]), b = dreamer::to_f(src[p + q]);
  dst[p] = (float)(a * cs - b * sn);
  dst[p + q] = (float)(b * cs + a * sn);
}

__global__ void zero_kernel(int *p, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = 0;
}

__device__ __forceinline__ bool better(float v1, int e1, float v2, int e2) {
  return v1 > v2 || (v1 == v2 && e1 < e2);
}

// One warp per token: q = y W_qE in fp32 (lanes over the d_r outputs), scores against the
// rotated keys in scratch, each lane keeping its best k of the experts e = lane (mod 32),
// then k warp-wide pops with the lower index winning ties; w = sigmoid(z)/sum over picks.
template <typename T, int DR>
__global__ void __launch_bounds__(256) route_noalloc_kernel(const T *y, int n, int h,
                                                            const T *wq, const float *keys,
                                                            const float *bias, int E, int k,
                                                            int *idx, float *w, int *counts) {
  constexpr int KMAX = 16;
  constexpr int PER = DR / 32;
  __shared__ float qs[8][DR];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + wid;
  if (t >= n) return;
  float acc[PER];
#pragma unroll
  for (int j = 0; j < PER; j++) acc[j] = 0.f;
  const T *yr = y + (long)t * h;
  for (int i = 0; i < h; i++) {
    const float yi = dreamer::to_f(yr[i]);
#pragma unroll
    for (int j = 0; j < PER; j++) acc[j] = fmaf(yi, dreamer::to_f(wq[(long)i * DR + lane + 32 * j]), acc[j]);
  }
#pragma unroll
  for (int j = 0; j < PER; j++) qs[wid][lane + 32 * j] = acc[j];
  __syncwarp();
  const float scale = rsqrtf((float)DR);
  float lv[KMAX];
  int le[KMAX];
#pragma unroll
  for (int i = 0; i < KMAX; i++) {
    lv[i] = -INFINITY;
    le[i] = 0x7fffffff;
  }
  for (int e = lane; e < E; e += 32) {
    const float *kr = keys + (long)e * DR;
    float z = 0.f;
#pragma unroll 8
    for (int i = 0; i < DR; i++) z = fmaf(qs[wid][i], kr[i], z);
    float v = z * scale + bias[e];
    if (v != v) v = -INFINITY;
    if (!better(v, e, lv[k - 1], le[k - 1])) continue;
    int p = k - 1;
    while (p > 0 && better(v, e, lv[p - 1], le[p - 1])) {
      lv[p] = lv[p - 1];
      le[p] = le[p - 1];
      p--;
    }
    lv[p] = v;
    le[p] = e;
  }
  int head = 0, my_e = 0;
  float my_z = 0.f;
  for (int s = 0; s < k; s++) {
    float bv = head < k ? lv[head] : -INFINITY;
    int be = head < k ? le[head] : 0x7fffffff;
    const int mine = be;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (better(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be == mine && head < k) head++;
    // the unbiased score of the pick; lane s keeps pick s
    const float *kr = keys + (long)be * DR;
    float z = 0.f;
    for (int i = 0; i < DR; i++) z = fmaf(qs[wid][i], kr[i], z);
    if (lane == s) {
      my_e = be;
      my_z = z * scale;
    }
  }
  // w = sigmoid(z) / sum over the picks, in the stable form exp(ls - max ls) / sum exp(...)
  // with ls = log sigmoid(z): no 0/0 when every pick's sigmoid underflows
  const float ls = lane < k ? dreamer::log_sigmoidf_(my_z) : -INFINITY;
  const float m = dreamer::warp_max(ls);
  const float ex = lane < k ? expf(ls - m) : 0.f;
  const float ssum = dreamer::warp_sum(ex);
  if (lane < k) {
    idx[(long)t * k + lane] = my_e;
    w[(long)t * k + lane] = ex / ssum;
    if (counts) atomicAdd(counts + my_e, 1);
  }
}

}  // namespace

extern "C" int dreamer_route_experts_noalloc(const dreamer_config *cfg, int depth,
                                             const void *y, int n_tokens, const void *w_qE,
                                             const void *k_E, const float *bias_E,
                                             int32_t *idx, float *w, int32_t *counts,
                                             dreamer_stream stream) {
  if (!cfg || !y || !w_qE || !k_E || !bias_E || !idx || !w) return DREAMER_ERR_ARG;
  const int E = cfg->n_experts, k = cfg->top_k, dr = cfg->router_dim, h = cfg->hidden;
  const int L = cfg->depth;
  if (depth < 0 || depth >= L || n_tokens < 0 || h < 1 || E < 1 || k < 1 || k > E)
    return DREAMER_ERR_ARG;
  if (cfg->dtype != 0 && cfg->dtype != 1) return DREAMER_ERR_ARG;
  if (k > 16 || (dr != 32 && dr != 64 && dr != 128)) return DREAMER_ERR_UNSUPPORTED;
  if ((size_t)E * dr > ROUTE_NOALLOC_SCRATCH_FLOATS) return DREAMER_ERR_UNSUPPORTED;
  float *keys = nullptr;
  int rc = scratch_on_current_device(&keys);
  if (rc != DREAMER_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  if (counts) zero_kernel<<<(E + 255) / 256, 256, 0, s>>>(counts, E);
  if (n_tokens == 0) return cudaGetLastError() == cudaSuccess ? DREAMER_OK : DREAMER_ERR_CUDA;
  const long pairs = (long)E * (dr / 2);
  const int rb = (int)((pairs + 255) / 256);
  const int tb = (n_tokens + 7) / 8;
  if (cfg->dtype == 0) {
    rotate_keys_kernel<float><<<rb, 256, 0, s>>>((const float *)k_E, E, dr, depth, L, cfg->rope_base, keys);
    const float *yy = (const float *)y, *wq = (const float *)w_qE;
    if (dr == 32) route_noalloc_kernel<float, 32><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
    else if (dr == 64) route_noalloc_kernel<float, 64><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
    else route_noalloc_kernel<float, 128><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
  } else {
    using dreamer::bf16;
    rotate_keys_kernel<bf16><<<rb, 256, 0, s>>>((const bf16 *)k_E, E, dr, depth, L, cfg->rope_base, keys);
    const bf16 *yy = (const bf16 *)y, *wq = (const bf16 *)w_qE;
    if (dr == 32) route_noalloc_kernel<bf16, 32><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
    else if (dr == 64) route_noalloc_kernel<bf16, 64><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
    else route_noalloc_kernel<bf16, 128><<<tb, 256, 0, s>>>(yy, n_tokens, h, wq, keys, bias_E, E, k, idx, w, counts);
  }
  return cudaGetLastError() == cudaSuccess ? DREAMER_OK : DREAMER_ERR_CUDA;
}
