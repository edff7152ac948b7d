"""The allocation-free expert routing entry point, through the C ABI.

dreamer_route_experts_noalloc exists for callers that cannot allocate device memory where
they route (their host owns all device memory, or allocating is not allowed on their hot
path).  It keeps its scratch in a fixed array inside the library.  Each case calls it twice in
a row (the second call finds the first call's scratch contents) and checks every result
against the float64 oracle's routing of the same inputs (indices equal except at near ties of
the k-th and (k+1)-th biased scores within 1e-5, routing weights within 1e-5, counts the
histogram of the returned indices and the oracle's when nothing flipped) and, where the
handle-based path takes the shape, against dreamer_route_experts.  This file sorts last so
that a run stopping at the first failure has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import oracle as O
import parity as PY
from depth_recurrent_attention_b200 import configs, inputs

pytestmark = pytest.mark.gpu


def _fn():
    from depth_recurrent_attention_b200.dreamer import lib
    fn = lib().dreamer_route_experts_noalloc
    fn.restype = C.c_int
    fn.argtypes = [C.c_void_p, C.c_int, C.c_void_p, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p,
                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]
    return fn


def _call(cfg, l, y, Wd, idx, w, cnt):
    import torch
    from depth_recurrent_attention_b200.dreamer import config_c
    p = lambda t: C.c_void_p(t.data_ptr()) if t is not None else None
    return _fn()(C.byref(config_c(cfg)), l, p(y), y.shape[0], p(Wd["w_qE"]), p(Wd["k_E"]),
                 p(Wd["bias"]), p(idx), p(w), p(cnt),
                 C.c_void_p(torch.cuda.current_stream().cuda_stream))


CASES = {
    "small-bf16-dr64": configs.SMALL,
    "small-bf16-dr128": configs.SMALL.with_(router_dim=128),
    "small-bf16-dr32": configs.SMALL.with_(router_dim=32),          # no handle path in bf16
    "fp32-dr32": configs.TINY.with_(router_dim=32, n_experts=64, top_k=4, batch=8, seq=64),
    "bf16-E24-k16": configs.SMALL.with_(n_experts=24, top_k=16),    # lanes without experts
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_route_noalloc_matches_the_oracle_and_the_handle_path(cuda, name):
    import torch
    from depth_recurrent_attention_b200.dreamer import Dreamer, DreamerError, lib

    cfg = CASES[name]
    W = inputs.host_weights(cfg)
    Wd = {k: inputs.to_device(v, "fp32" if k == "bias" else cfg.dtype) for k, v in W.items()}
    try:
        dev = Dreamer(cfg, Wd)
    except DreamerError:
        dev = None                                  # a shape the handle path does not take
    orc = O.Oracle(cfg, W)
    n, k, E = cfg.tokens, cfg.top_k, cfg.n_experts
    for call, l in enumerate((cfg.depth - 1, 1 % cfg.depth)):
        y_host = inputs.extra_normal(cfg, 3000 + l, (n, cfg.hidden), 1.0)
        y = inputs.to_device(y_host, cfg.dtype)
        idx = torch.empty((n, k), dtype=torch.int32, device="cuda")
        w = torch.empty((n, k), dtype=torch.float32, device="cuda")
        cnt = torch.full((E,), 7, dtype=torch.int32, device="cuda")   # must be cleared
        rc = _call(cfg, l, y, Wd, idx, w, cnt)
        assert rc == 0, f"call {call}: {lib().dreamer_strerror(rc)}"
        torch.cuda.synchronize()
        a, wa, c = idx.cpu().numpy(), w.cpu().numpy(), cnt.cpu().numpy()
        ref = orc.route(l, y_host)
        same, flips = PY.check_routing(cfg, W, l, a, ref["idx"], ref["margin"], strict=True)
        assert np.allclose(PY.weights_by_expert(a, wa)[same],
                           PY.weights_by_expert(ref["idx"], ref["w"])[same], atol=1e-5)
        assert np.array_equal(c, np.bincount(a.ravel(), minlength=E))
        if flips == 0:
            assert np.array_equal(c, ref["counts"])
        print(f"{name} call {call} depth {l}: {flips} near-tie flips against the oracle")
        if dev is not None:
            idx_ref, w_ref, cnt_ref = dev.route_experts(l, y)
            b = idx_ref.cpu().numpy()
            sm = PY.same_sets(a, b)
            assert np.all(sm | (ref["margin"] <= PY.NEAR_TIE)), f"call {call}: index mismatch"
            assert np.allclose(PY.weights_by_expert(a, wa)[sm],
                               PY.weights_by_expert(b, w_ref.cpu().numpy())[sm], atol=1e-5)
            if sm.all():
                assert np.array_equal(c, cnt_ref.cpu().numpy())
    if dev is not None:
        dev.close()


def test_route_noalloc_weights_when_every_sigmoid_underflows(cuda):
    """Every expert picked (E = k) with scores near -100, where each sigmoid underflows to 0
    in float32: the weights must still be the normalised sigmoids (the oracle's, in float64),
    not 0/0."""
    import torch
    cfg = configs.TINY.with_(router_dim=32, n_experts=4, top_k=4, depth=1, batch=1, seq=8)
    W = dict(inputs.host_weights(cfg))
    f = lambda a: np.asarray(a, np.float64)
    row = inputs.extra_normal(cfg, 3000, (1, cfg.hidden), 1.0)
    y_host = np.repeat(row, cfg.tokens, axis=0)                   # every token the same
    q = (f(row) @ f(W["w_qE"]))[0]                                # [d_r]
    # at L = 1 the depth RoPE of depth 0 is the identity, so z_e = q . k_e / sqrt(d_r); keys
    # along -q give z_e = -(100 + 0.3 e)
    W["k_E"] = np.stack([-(100.0 + 0.3 * e) * np.sqrt(cfg.router_dim) * q / (q @ q)
                         for e in range(4)]).astype(np.float32)
    ref = O.Oracle(cfg, W).route(0, y_host)
    zs = (q @ f(W["k_E"]).T) / np.sqrt(cfg.router_dim)
    assert zs.max() < -99, zs.max()                                # sigmoids underflow in fp32
    Wd = {k: inputs.to_device(v, "fp32") for k, v in W.items()}
    y = inputs.to_device(y_host, "fp32")
    idx = torch.empty((cfg.tokens, 4), dtype=torch.int32, device="cuda")
    w = torch.empty((cfg.tokens, 4), dtype=torch.float32, device="cuda")
    assert _call(cfg, 0, y, Wd, idx, w, None) == 0
    torch.cuda.synchronize()
    wa = w.cpu().numpy()
    assert np.isfinite(wa).all()
    # float32 scores of magnitude ~100 carry ~1e-5 relative rounding into exp(z - z_max)
    assert np.allclose(PY.weights_by_expert(idx.cpu().numpy(), wa),
                       PY.weights_by_expert(ref["idx"], ref["w"]), atol=2e-4)


def test_route_noalloc_refuses_sizes_beyond_its_scratch(cuda):
    import torch
    cfg = configs.SMALL
    big = cfg.with_(n_experts=65536, router_dim=64)               # 4 Mi floats > the array
    y = torch.zeros((8, cfg.hidden), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(16, dtype=torch.int32, device="cuda")
    Wd = dict(w_qE=y, k_E=y, bias=t)
    idx = torch.empty((8, cfg.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((8, cfg.top_k), dtype=torch.float32, device="cuda")
    assert _call(big, 0, y, Wd, idx, w, None) == -2               # before anything is launched
