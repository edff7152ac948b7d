"""The allocation-free expert routing entry point against the handle-based one.

dreamer_route_experts_noalloc exists for callers that cannot allocate device memory where
they route (their host owns all device memory, or allocating is not allowed on their hot
path).  It keeps its scratch in a fixed array inside the library.  This test calls it through
the C ABI twice in a row (the second call finds the first call's scratch contents) and checks
each result against dreamer_route_experts on the same inputs: expert indices equal except at
near ties (k-th and (k+1)-th biased scores within 1e-5 in the float64 oracle), routing
weights within 1e-5, counts equal to the histogram of the returned indices.  This file sorts
last so that a run stopping at the first failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import oracle as O
import parity as PY
from depth_recurrent_attention_b200 import configs, inputs

pytestmark = pytest.mark.gpu


def test_route_noalloc_matches_route_experts(cuda):
    import torch
    from depth_recurrent_attention_b200.dreamer import Dreamer, config_c, lib

    cfg = configs.SMALL
    W = inputs.host_weights(cfg)
    Wd = {k: inputs.to_device(v, "fp32" if k == "bias" else cfg.dtype) for k, v in W.items()}
    dev = Dreamer(cfg, Wd)
    L = lib()
    fn = L.dreamer_route_experts_noalloc
    fn.restype = C.c_int
    fn.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    cc = config_c(cfg)
    n, k, E = cfg.tokens, cfg.top_k, cfg.n_experts
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, l in enumerate((5, 2)):
        y_host = inputs.extra_normal(cfg, 3000 + l, (n, cfg.hidden), 1.0)
        y = inputs.to_device(y_host, cfg.dtype)
        idx_ref, w_ref, cnt_ref = dev.route_experts(l, y)
        idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
        w = torch.empty((n, k), dtype=torch.float32, device="cuda")
        cnt = torch.full((E,), 7, dtype=torch.int32, device="cuda")   # must be cleared
        rc = fn(C.byref(cc), l, C.c_void_p(y.data_ptr()), n, C.c_void_p(Wd["w_qE"].data_ptr()),
                C.c_void_p(Wd["k_E"].data_ptr()), C.c_void_p(Wd["bias"].data_ptr()),
                C.c_void_p(idx.data_ptr()), C.c_void_p(w.data_ptr()), C.c_void_p(cnt.data_ptr()),
                stream)
        assert rc == 0, f"call {call}: {L.dreamer_strerror(rc)}"
        torch.cuda.synchronize()
        a, b = idx.cpu().numpy(), idx_ref.cpu().numpy()
        margin = O.Oracle(cfg, W).route(l, y_host)["margin"]
        same = PY.same_sets(a, b)
        assert np.all(same | (margin <= PY.NEAR_TIE)), f"call {call}: index mismatch"
        assert np.allclose(PY.weights_by_expert(a, w.cpu().numpy())[same],
                           PY.weights_by_expert(b, w_ref.cpu().numpy())[same], atol=1e-5)
        c = cnt.cpu().numpy()
        assert np.array_equal(c, np.bincount(a.ravel(), minlength=E))
        if same.all():
            assert np.array_equal(c, cnt_ref.cpu().numpy())
    # a size beyond the scratch array is refused, nothing is launched
    big = configs.SMALL.with_(n_experts=65536, router_dim=64)
    rc = fn(C.byref(config_c(big)), 0, C.c_void_p(y.data_ptr()), n, C.c_void_p(Wd["w_qE"].data_ptr()),
            C.c_void_p(Wd["k_E"].data_ptr()), C.c_void_p(Wd["bias"].data_ptr()),
            C.c_void_p(idx.data_ptr()), C.c_void_p(w.data_ptr()), None, stream)
    assert rc == -2
    dev.close()
