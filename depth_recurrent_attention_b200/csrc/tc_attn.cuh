// Causal sequence attention (prefill) on tcgen05: placeholder until the flash kernel lands.
#pragma once
static int tc_attn_init(dreamer_handle *h) { return 0; }
static bool tc_sa_ok(dreamer_handle *h) { return false; }
static void tc_sa(dreamer_handle *h, cudaStream_t s) {}
