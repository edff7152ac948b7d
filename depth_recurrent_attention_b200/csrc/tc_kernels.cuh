// tcgen05 / TMA kernels (bf16 contractions).  Included after the handle definition.
#pragma once

static int tc_init(dreamer_handle *h) { return 0; }
static void tc_destroy(dreamer_handle *h) {}
static bool tc_route_ok(dreamer_handle *h) { return false; }
static void tc_route(dreamer_handle *h, int l, const void *X, int n, int *idx, float *w,
                     int *counts_a, int *counts_b, cudaStream_t s) {}
static bool tc_gemm_ok(dreamer_handle *h, const dreamer::GemmArgs &a) { return false; }
template <typename T>
static void tc_gemm_qkv(dreamer_handle *h, const dreamer::GemmArgs &a,
                        const dreamer::EpiQKV<T> &e, cudaStream_t s) {}
template <typename T>
static void tc_gemm_o(dreamer_handle *h, const dreamer::GemmArgs &a, const dreamer::EpiO<T> &e,
                      cudaStream_t s) {}
static bool tc_sa_ok(dreamer_handle *h) { return false; }
static void tc_sa(dreamer_handle *h, cudaStream_t s) {}
static bool tc_expert_ok(dreamer_handle *h) { return false; }
static void tc_expert(dreamer_handle *h, const void *X, int n, cudaStream_t s) {}
