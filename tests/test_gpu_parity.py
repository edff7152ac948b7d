"""GPU parity of libdreamer (through the C ABI) against the CPU oracle on seeded inputs.

Tolerances are the contract's (see tests/parity.py).  Inputs for the oracle and for the GPU
come from the same seeded generator; nothing the GPU computes is fed to the oracle.
"""
import numpy as np
import pytest

import oracle as O
import parity as PY
from depth_recurrent_attention_b200 import configs, inputs

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


def upload(cfg, arrays: dict):
    return {k: inputs.to_device(v, "fp32" if k == "bias" else cfg.dtype) for k, v in arrays.items()}


def make_handle(cfg, W_host, **kw):
    from depth_recurrent_attention_b200.dreamer import Dreamer
    return Dreamer(cfg, upload(cfg, W_host), **kw)


def trace_buffers(cfg, n_tok, with_sa=False):
    torch = _torch()
    L, h, k = cfg.depth, cfg.hidden, cfg.top_k
    dt = torch.float32 if cfg.dtype == "fp32" else torch.bfloat16
    tr = dict(y=torch.zeros((L, n_tok, h), dtype=dt, device="cuda"),
              xhat=torch.zeros((L, n_tok, h), dtype=dt, device="cuda"),
              idx=torch.zeros((L, n_tok, k), dtype=torch.int32, device="cuda"),
              w=torch.zeros((L, n_tok, k), dtype=torch.float32, device="cuda"),
              y_f32=torch.zeros((L, n_tok, h), dtype=torch.float32, device="cuda"),
              x_f32=torch.zeros((L, n_tok, h), dtype=torch.float32, device="cuda"))
    if cfg.n_proj_experts > 0:
        tr["pidx"] = torch.zeros((L, n_tok), dtype=torch.int32, device="cuda")
        tr["psig"] = torch.zeros((L, n_tok), dtype=torch.float32, device="cuda")
    if with_sa:
        tr["sa_k"] = torch.zeros((L, n_tok, h), dtype=dt, device="cuda")
        tr["sa_v"] = torch.zeros((L, n_tok, h), dtype=dt, device="cuda")
    return tr


# ---------------------------------------------------------------------------------------
# tiny, float32, free-running end to end

@pytest.mark.parametrize("kw", [dict(variant=0), dict(variant=1), dict(variant=2),
                                # without depth attention; sliding-window depth attention
                                dict(variant=3), dict(da_window=2), dict(variant=1, da_window=1)])
def test_tiny_forward_fp32(cuda, kw):
    torch = _torch()
    cfg = configs.TINY.with_(**kw)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    ref = O.Oracle(cfg, W).forward(x0)
    dev = make_handle(cfg, W)
    tr = trace_buffers(cfg, cfg.tokens)
    out = dev.forward(inputs.to_device(x0, "fp32"), trace=tr)
    torch.cuda.synchronize()
    for l in range(cfg.depth):
        same, flips = PY.check_routing(cfg, W, l, tr["idx"][l].cpu().numpy(), ref["idx"][l],
                                       ref["margin"][l], strict=True)
        assert flips == 0, "a near tie flipped; later depths are not comparable"
        assert np.allclose(PY.weights_by_expert(tr["idx"][l].cpu().numpy(), PY.to_np(tr["w"][l])),
                           PY.weights_by_expert(ref["idx"][l], ref["w"][l]), atol=1e-5)
        PY.check_hidden(PY.to_np(tr["y"][l]), ref["y"][l], False, f"y depth {l}")
    PY.check_hidden(PY.to_np(out), ref["x_out"], False, "x_L")
    counts = dev.route_counts(on_host=True).numpy()
    assert np.array_equal(counts, ref["counts"])


def test_tiny_depth_ranges_compose(cuda):
    torch = _torch()
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    x0 = inputs.to_device(inputs.host_inputs(cfg)["x0"], "fp32")
    dev = make_handle(cfg, W)
    full = dev.forward(x0).clone()
    da = torch.zeros((cfg.tokens, cfg.depth, 2, cfg.hidden), device="cuda")
    mid = dev.forward(x0, depth_begin=0, depth_end=2, da_kv=da)
    out = dev.forward(mid, depth_begin=2, depth_end=cfg.depth, da_kv=da)
    assert torch.allclose(out, full, atol=1e-5, rtol=0)


# ---------------------------------------------------------------------------------------
# router on identical inputs: strict index parity

@pytest.mark.parametrize("name,l", [("tiny", 1), ("small", 0), ("small", 5)])
def test_router_strict(cuda, name, l):
    cfg = configs.CONFIGS[name]
    W = inputs.host_weights(cfg)
    y = inputs.extra_normal(cfg, 3000 + l, (cfg.tokens, cfg.hidden), 1.0)
    ref = O.Oracle(cfg, W).route(l, y)
    dev = make_handle(cfg, W)
    idx, w, counts = dev.route_experts(l, inputs.to_device(y, cfg.dtype))
    idx = idx.cpu().numpy()
    same, flips = PY.check_routing(cfg, W, l, idx, ref["idx"], ref["margin"], strict=True)
    near = int((ref["margin"] <= PY.NEAR_TIE).sum())
    print(f"router {name} depth {l}: {flips} flips at {near} near ties")
    assert np.allclose(PY.weights_by_expert(idx, PY.to_np(w))[same],
                       PY.weights_by_expert(ref["idx"], ref["w"])[same], atol=1e-5)
    c = counts.cpu().numpy()
    assert np.array_equal(c, np.bincount(idx.ravel(), minlength=cfg.n_experts))
    if flips == 0:
        assert np.array_equal(c, ref["counts"])


@pytest.mark.parametrize("pattern", ["all-equal", "every-third"])
def test_router_exact_ties_on_the_tensor_core_path(cuda, pattern):
    """Scores tied exactly at the selection bound, on the path that stores the scores and picks
    a token's top k from them (9728 tokens: enough 128-row tiles for the tensor-core scores;
    E = 256, k = 4).  Zero router keys make every raw score 0, so the biased score is the bias:
    all equal (every lane's maximum ties, so the candidates exceed a warp and the k rounds of a
    warp-wide best run) or 1 on every third expert and 0 elsewhere.  The picks must be the k
    lowest-index experts among the best, each weighted 1/k."""
    cfg = configs.SMALL.with_(batch=19)
    assert cfg.tokens // 128 >= 74
    W = dict(inputs.host_weights(cfg))
    E, k = cfg.n_experts, cfg.top_k
    W["k_E"] = np.zeros_like(W["k_E"])
    if pattern == "all-equal":
        W["bias"] = np.zeros(E, np.float32)
        want = np.arange(k)
    else:
        W["bias"] = (np.arange(E) % 3 == 0).astype(np.float32)
        want = np.arange(0, 3 * k, 3)
    dev = make_handle(cfg, W)
    y = inputs.extra_normal(cfg, 3000, (cfg.tokens, cfg.hidden), 1.0)
    idx, w, counts = dev.route_experts(0, inputs.to_device(y, cfg.dtype))
    idx, w, counts = idx.cpu().numpy(), PY.to_np(w), counts.cpu().numpy()
    assert np.array_equal(np.sort(idx, axis=-1), np.broadcast_to(want, idx.shape))
    assert np.allclose(w, 1.0 / k, atol=1e-6)
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))


# ---------------------------------------------------------------------------------------
# small, bf16: one depth at a time from seeded states (every depth)

def step_inputs(cfg, l):
    T, L, h = cfg.tokens, cfg.depth, cfg.hidden
    x = inputs.extra_normal(cfg, 1000 + l, (T, h), 1.0)
    hist = np.zeros((T, L, 2, h), np.float32)
    if l > 0:
        hist[:, :l] = inputs.extra_normal(cfg, 2000 + l, (T, l, 2, h), 1.0)
    return x, hist


def router_input(cfg, tr, l):
    return PY.to_np(tr["xhat"][l] if cfg.variant == 2 else tr["y"][l])


def run_step_and_compare(cfg, W, dev, l, orc=None):
    """One depth on seeded x_l and DA history, every token: routing gated on the device's own
    router inputs (strict 1e-5 rule, exact counts), the float32 states against the oracle's
    forward, the stored bf16 values as their exact rounding.  Returns (EA selections that
    differ from the oracle forward's, tokens)."""
    torch = _torch()
    x, hist = step_inputs(cfg, l)
    tr = trace_buffers(cfg, cfg.tokens)
    xd = inputs.to_device(x, cfg.dtype)
    hd = inputs.to_device(hist, cfg.dtype)
    out = dev.forward(xd, depth_begin=l, depth_end=l + 1, da_kv=hd, trace=tr)
    torch.cuda.synchronize()
    bf = cfg.dtype == "bf16"
    g_x, g_y = PY.to_np(out), PY.to_np(tr["y"][l])
    g_y32, g_x32 = PY.to_np(tr["y_f32"][l]), PY.to_np(tr["x_f32"][l])
    g_xh = PY.to_np(tr["xhat"][l])
    g_ein = router_input(cfg, tr, l)
    g_idx = tr["idx"][l].cpu().numpy()
    o = orc or O.Oracle(cfg, W)
    counts = dev.route_counts(on_host=True).numpy()[l]
    PY.gate_router_on_device_input(cfg, W, o, l, g_ein, g_idx, PY.to_np(tr["w"][l]), counts,
                                   what=cfg.name)
    r = o.forward(x, l, l + 1, da_kv=hist.astype(np.float64))
    rx, ry, ridx, rmg = r["x_out"], r["y"][l], r["idx"][l], r["margin"][l]
    rein = r["xhat"][l] if cfg.variant == 2 else ry
    keep = np.ones(cfg.tokens, bool)
    if cfg.n_proj_experts > 0:
        gp = tr["pidx"][l].cpu().numpy()
        PY.gate_proj_router_on_device_input(cfg, o, l, g_xh, gp, PY.to_np(tr["psig"][l]),
                                            what=cfg.name)
        keep = PY.proj_same_as_forward(cfg, W, l, gp, r["pidx"][l], r["pmargin"][l], g_xh,
                                       r["xhat"][l])
        print(f"  {int((~keep).sum())} tokens with another projection expert than the forward's")
    PY.check_hidden(PY.to_np(hd[:, l]), r["da_kv"][:, l], bf, f"DA kv depth {l}")
    PY.check_hidden(g_y[keep], ry[keep], bf, f"y depth {l}", f32=g_y32[keep] if bf else None)
    same, flips = PY.check_routing(cfg, W, l, g_idx[keep], ridx[keep], rmg[keep], g_ein[keep],
                                   rein[keep])
    PY.check_hidden(g_x[keep][same], rx[keep][same], bf, f"x depth {l}",
                    f32=g_x32[keep][same] if bf else None)
    return flips, int(keep.sum())


def test_small_every_depth_bf16(cuda):
    cfg = configs.SMALL
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    orc = O.Oracle(cfg, W)
    for l in range(cfg.depth):
        flips, n = run_step_and_compare(cfg, W, dev, l, orc=orc)
        print(f"small depth {l}: {flips}/{n} selections differ from the oracle forward's, "
              f"each explained by the bf16 rounding of y")


def test_small_linear_moe_step_bf16(cuda):
    """Top-1 linear-MoE QKV/O with 8 projection experts (grouped GEMMs over p*); the oracle
    runs the deployed (absorbed, bf16-stored) weights."""
    cfg = configs.SMALL.with_(n_proj_experts=8, depth=4)
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    orc = O.Oracle(cfg, PY.deployed_weights(cfg, W))
    for l in (0, 3):
        run_step_and_compare(cfg, W, dev, l, orc=orc)


@pytest.mark.parametrize("m", [16, 32])
def test_small_expert_sizes_bf16(cuda, m):
    """Expert hidden sizes 16 and 32 (the fused expert FFN with 32- and 64-byte H rows), about
    32 routed rows per expert, so most tiles are partial."""
    cfg = configs.SMALL.with_(expert_hidden=m, depth=2)
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    orc = O.Oracle(cfg, W)
    for l in (0, 1):
        run_step_and_compare(cfg, W, dev, l, orc=orc)


def test_small_random_norm_gain_bf16(cuda):
    """A random RMSNorm gain (the configurations use g = 1): the first depth's norm, the
    residual rebuilt in the O epilogue and the combine's norm for the next depth all apply it."""
    cfg = configs.SMALL.with_(depth=2)
    W = dict(inputs.host_weights(cfg))
    g = np.random.default_rng(16).uniform(0.5, 1.5, cfg.hidden).astype(np.float32)
    W["g"] = inputs.round_to(g, "bf16").astype(np.float32)
    dev = make_handle(cfg, W)
    orc = O.Oracle(cfg, W)
    for l in (0, 1):
        run_step_and_compare(cfg, W, dev, l, orc=orc)


def test_short_batch_wide_hidden_bf16(cuda):
    """256 tokens at h = 2048 (16 heads of 128): the O projection takes 32-column tiles (two
    row tiles × 64 N tiles), the router its cluster form and the experts their per-row
    form (about 4 routed rows per expert), all in a prefill step."""
    cfg = configs.SMALL.with_(batch=2, seq=128, hidden=2048, n_heads=16, head_dim=128, depth=2)
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    orc = O.Oracle(cfg, W)
    for l in (0, 1):
        run_step_and_compare(cfg, W, dev, l, orc=orc)


@pytest.mark.parametrize("variant", [1, 2])
def test_small_layout_variants_bf16(cuda, variant):
    cfg = configs.SMALL.with_(variant=variant, depth=3)
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    if variant == 1:
        # the serial layout needs every token's DA; run the whole (short) forward
        torch = _torch()
        x0 = inputs.host_inputs(cfg)["x0"]
        orc = O.Oracle(cfg, W)
        ref = orc.forward(x0, 0, 1)
        tr = trace_buffers(cfg, cfg.tokens)
        out = dev.forward(inputs.to_device(x0, "bf16"), depth_end=1, trace=tr)
        torch.cuda.synchronize()
        gy = PY.to_np(tr["y"][0])
        PY.gate_router_on_device_input(cfg, W, orc, 0, gy, tr["idx"][0].cpu().numpy(),
                                       PY.to_np(tr["w"][0]),
                                       dev.route_counts(on_host=True).numpy()[0], what="serial")
        PY.check_hidden(gy, ref["y"][0], True, "y serial", f32=PY.to_np(tr["y_f32"][0]))
        same, flips = PY.check_routing(cfg, W, 0, tr["idx"][0].cpu().numpy(), ref["idx"][0],
                                       ref["margin"][0], gy, ref["y"][0])
        PY.check_hidden(PY.to_np(out)[same], ref["x_out"][same], True, "x serial",
                        f32=PY.to_np(tr["x_f32"][0])[same])
    else:
        for l in (0, 2):
            run_step_and_compare(cfg, W, dev, l)


def test_small_free_running_drift_reported(cuda):
    """Free-running bf16 through all 8 depths: routing flips compound, so the drift is
    reported, not gated; only a gross failure (rel-L2 > 0.5) fails."""
    cfg = configs.SMALL
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    ref = O.Oracle(cfg, W).forward(x0, trace=False)
    dev = make_handle(cfg, W)
    out = PY.to_np(dev.forward(inputs.to_device(x0, "bf16")))
    rl = PY.rel_l2(out, ref["x_out"])
    print(f"small free-running bf16 drift: rel-L2 {rl:.3e}, max-abs "
          f"{np.max(np.abs(out - ref['x_out'])):.3e}")
    assert rl < 0.5


# ---------------------------------------------------------------------------------------
# bf16 through every depth, free-running, where no routing decision can flip

@pytest.mark.parametrize("kw", [dict(n_experts=4, top_k=4, depth=4),
                                dict(n_experts=8, top_k=8, depth=3, n_proj_experts=1),
                                dict(n_experts=4, top_k=4, depth=3, variant=1),
                                dict(n_experts=4, top_k=4, depth=3, variant=2),
                                # head dim 128: q/k columns in the permuted GEMM order
                                dict(n_experts=4, top_k=4, depth=3, n_heads=4, head_dim=128),
                                dict(n_experts=8, top_k=8, depth=2, n_heads=4, head_dim=128,
                                     n_proj_experts=1),
                                dict(n_experts=4, top_k=4, depth=4, da_window=2),
                                dict(n_experts=4, top_k=4, depth=3, variant=3),
                                # expert FFN with 32- and 64-byte H rows, full tiles
                                dict(n_experts=4, top_k=4, depth=2, expert_hidden=16),
                                dict(n_experts=4, top_k=4, depth=2, expert_hidden=32)])
def test_small_flip_free_all_depths_bf16(cuda, kw):
    torch = _torch()
    cfg = configs.SMALL.with_(**kw)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    ref = O.Oracle(cfg, PY.deployed_weights(cfg, W)).forward(x0)
    dev = make_handle(cfg, W)
    tr = trace_buffers(cfg, cfg.tokens)
    out = dev.forward(inputs.to_device(x0, "bf16"), trace=tr)
    torch.cuda.synchronize()
    for l in range(cfg.depth):
        e, rl = PY.check_drift(PY.to_np(tr["y"][l]), ref["y"][l], f"y depth {l}", gate_abs=(l == 0),
                               f32=PY.to_np(tr["y_f32"][l]))
        print(f"  y depth {l}: max-abs {e:.3g} rel-L2 {rl:.3g}")
        if l == 0:  # later depths of a free-running run: weights follow the drift of y
            assert np.allclose(PY.weights_by_expert(tr["idx"][l].cpu().numpy(), PY.to_np(tr["w"][l])),
                               PY.weights_by_expert(ref["idx"][l], ref["w"][l]), atol=5e-3)
    e, rl = PY.check_drift(PY.to_np(out), ref["x_out"], "x_L", gate_abs=False,
                           f32=PY.to_np(tr["x_f32"][cfg.depth - 1]))
    assert np.array_equal(PY.rn_bf16(PY.to_np(tr["x_f32"][cfg.depth - 1])), PY.to_np(out))
    print(f"flip-free {kw}: x_L max-abs {e:.3g} rel-L2 {rl:.3g}")
    assert np.array_equal(dev.route_counts().numpy(), ref["counts"])


# ---------------------------------------------------------------------------------------
# decode

def decode_case(cfg, lens):
    B, L, H, d = cfg.batch, cfg.depth, cfg.n_heads, cfg.head_dim
    cap = cfg.cache_len + 1
    kc = inputs.extra_normal(cfg, 4001, (L, B, H, cap, d), 1.0)
    vc = inputs.extra_normal(cfg, 4002, (L, B, H, cap, d), 1.0)
    x = inputs.extra_normal(cfg, 4003, (B, cfg.hidden), 1.0)
    return x, kc, vc, np.asarray(lens, np.int32)


def flip_free(cfg):
    """E = k and P <= 1: no routing decision can flip, so bf16 runs stay comparable with the
    oracle through every depth."""
    return cfg.n_experts == cfg.top_k and cfg.n_proj_experts <= 1


@pytest.mark.parametrize("base,lens,kw", [
    ("tiny", [12, 5, 0], {}),
    ("small", [300, 1, 77, 299], {}),
    ("small", [300, 1, 77, 299], dict(n_experts=4, top_k=4, depth=4)),
    ("small", [40, 0, 17], dict(n_experts=4, top_k=4, depth=3, n_proj_experts=1)),
    ("small", [300, 1, 77, 299], dict(n_experts=4, top_k=4, depth=3, n_heads=4, head_dim=128)),
    ("small", [300, 1, 77, 299], dict(n_experts=4, top_k=4, depth=4, da_window=2)),
    ("tiny", [12, 5, 0], dict(variant=3)),
    # one sequence with an empty cache; 130 sequences (two row tiles in the projections)
    ("small", [0], {}),
    ("small", [(7 * i) % 61 for i in range(130)], dict(depth=3)),
])
def test_decode_step(cuda, base, lens, kw):
    torch = _torch()
    cfg = configs.CONFIGS[base].with_(batch=len(lens), seq=1, cache_len=max(lens) + 1, **kw)
    W = inputs.host_weights(cfg)
    x, kc, vc, ln = decode_case(cfg, lens)
    dev = make_handle(cfg, W)
    kd, vd = inputs.to_device(kc, cfg.dtype), inputs.to_device(vc, cfg.dtype)
    tr = trace_buffers(cfg, cfg.batch)
    out = dev.decode_step(inputs.to_device(x, cfg.dtype), kd, vd,
                          torch.from_numpy(ln).cuda(), trace=tr)
    torch.cuda.synchronize()
    o = O.Oracle(cfg, PY.deployed_weights(cfg, W))
    bf = cfg.dtype == "bf16"
    g = PY.to_np(out)
    kd_np, vd_np = PY.to_np(kd), PY.to_np(vd)
    for b in range(cfg.batch):
        kcb = kc[:, b].astype(np.float64).copy()
        vcb = vc[:, b].astype(np.float64).copy()
        r = o.decode_seq(x[b], kcb, vcb, int(ln[b]))
        # the new token's key/value went to slot cache_len of every depth (bf16 with real
        # routing: depth 0 only, later depths drift through routing flips)
        PY.check_hidden(kd_np[0:1, b, :, ln[b]], kcb[0:1, :, ln[b]], bf, f"k slot seq {b}")
        PY.check_hidden(vd_np[0:1, b, :, ln[b]], vcb[0:1, :, ln[b]], bf, f"v slot seq {b}")
        if not bf or flip_free(cfg):
            chk = PY.check_hidden if not bf else (lambda a, r_, bf_, w: PY.check_drift(a, r_, w, False))
            chk(kd_np[:, b, :, ln[b]], kcb[:, :, ln[b]], bf, f"k slots seq {b}")
            chk(vd_np[:, b, :, ln[b]], vcb[:, :, ln[b]], bf, f"v slots seq {b}")
        if not bf or flip_free(cfg):
            for l in range(cfg.depth):
                same, flips = PY.check_routing(cfg, W, l, tr["idx"][l, b:b + 1].cpu().numpy(),
                                               r["idx"][l:l + 1], r["margin"][l:l + 1],
                                               strict=True)
                assert flips == 0
                if bf:
                    PY.check_drift(PY.to_np(tr["y"][l, b]), r["y"][l], f"y depth {l} seq {b}",
                                   gate_abs=(l == 0), f32=PY.to_np(tr["y_f32"][l, b]))
                else:
                    PY.check_hidden(PY.to_np(tr["y"][l, b]), r["y"][l], bf, f"y depth {l} seq {b}")
            if bf:
                PY.check_drift(g[b], r["x_out"], f"x_out seq {b}", gate_abs=False,
                               f32=PY.to_np(tr["x_f32"][cfg.depth - 1, b]))
            else:
                PY.check_hidden(g[b], r["x_out"], bf, f"x_out seq {b}")
        else:
            # first depth is comparable token by token; later depths drift by routing flips
            gy = PY.to_np(tr["y"][0, b])
            PY.check_hidden(gy, r["y"][0], True, f"y depth 0 seq {b}",
                            f32=PY.to_np(tr["y_f32"][0, b]))
    # every depth's routing, on the states the device routed (all sequences at once)
    idx_all, w_all = tr["idx"].cpu().numpy(), PY.to_np(tr["w"])
    counts = dev.route_counts(on_host=True).numpy()
    for l in range(cfg.depth):
        PY.gate_router_on_device_input(cfg, W, o, l, PY.to_np(tr["y"][l]), idx_all[l], w_all[l],
                                       counts[l], what="decode")


# ---------------------------------------------------------------------------------------
# bias balance update, error handling, generator

def test_bias_update_matches_oracle(cuda):
    torch = _torch()
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    dev.forward(inputs.to_device(inputs.host_inputs(cfg)["x0"], "fp32"))
    counts = dev.route_counts(on_host=True).numpy()
    new_b = dev.bias_update(0.01).cpu().numpy()
    ref = O.bias_update(counts, 0.01, W["bias"].astype(np.float64))
    assert np.allclose(new_b, ref, atol=1e-7)


def test_bias_update_from_replica_counts(cuda):
    """The update from given counts (this handle's route counts plus another replica's,
    summed as the all-reduce would) matches the oracle's update from the same counts."""
    torch = _torch()
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    dev.forward(inputs.to_device(inputs.host_inputs(cfg)["x0"], "fp32"))
    counts = dev.route_counts(on_host=False)
    rng = np.random.default_rng(7)
    other = rng.integers(0, 9, size=tuple(counts.shape)).astype(np.int32)
    total = counts + torch.from_numpy(other).to(counts.device)
    new_b = dev.bias_update(0.01, counts=total).cpu().numpy()
    ref = O.bias_update(np.ascontiguousarray(total.cpu().numpy()), 0.01,
                        W["bias"].astype(np.float64))
    assert np.allclose(new_b, ref, atol=1e-7)


def test_errors_are_returned_not_faulted(cuda):
    torch = _torch()
    from depth_recurrent_attention_b200.dreamer import Dreamer, DreamerError, ERR_ARG, \
        ERR_UNSUPPORTED, ERR_STATE
    cfg = configs.TINY
    W = upload(cfg, inputs.host_weights(cfg))
    with pytest.raises(DreamerError) as e:
        Dreamer(cfg.with_(hidden=65), W)
    assert e.value.code == ERR_ARG
    with pytest.raises(DreamerError) as e:
        Dreamer(cfg.with_(top_k=17, n_experts=32), W)
    assert e.value.code == ERR_UNSUPPORTED
    with pytest.raises(DreamerError) as e:
        Dreamer(cfg.with_(head_dim=8, n_heads=8), W)
    assert e.value.code == ERR_UNSUPPORTED
    dev = Dreamer(cfg, W)
    x = torch.zeros((cfg.tokens, cfg.hidden), device="cuda")
    with pytest.raises(DreamerError) as e:          # no DA buffer for a later start depth
        dev.forward(x, depth_begin=1)
    assert e.value.code == ERR_ARG
    with pytest.raises(DreamerError) as e:          # misaligned pointer
        xm = x.view(-1)[1:1 + (cfg.tokens - 1) * cfg.hidden].view(cfg.tokens - 1, cfg.hidden)
        dev.forward(xm)
    assert e.value.code == ERR_ARG
    with pytest.raises(DreamerError) as e:          # decode on a handle without a cache
        dev.decode_step(x[:1], x, x, torch.zeros(1, dtype=torch.int32, device="cuda"))
    assert e.value.code == ERR_STATE
    # the context is still usable
    dev.forward(x)
    torch.cuda.synchronize()


def test_device_generator_matches_host(cuda):
    torch = _torch()
    cfg = configs.SMALL
    for spec in inputs.weight_specs(cfg):
        t = inputs.device_tensor(spec, cfg.seed)
        n = min(spec.numel, 1 << 20)
        host = inputs.draw(spec, cfg.seed, 0, n)
        dev = t.float().view(-1)[:n].cpu().numpy()
        mism = int((host != dev).sum())
        assert mism <= max(1, n // 1_000_000), (spec.name, mism)


# ---------------------------------------------------------------------------------------
# the layered comparison arm: L distinct layers without depth attention

@pytest.mark.parametrize("base,kw", [("tiny", {}), ("small", dict(n_experts=4, top_k=4, depth=3))])
def test_layered_stack(cuda, base, kw):
    torch = _torch()
    from depth_recurrent_attention_b200.dreamer import LayeredStack
    cfg = configs.CONFIGS[base].with_(variant=3, **kw)
    Ws = [inputs.host_weights(cfg.with_(seed=cfg.seed + 100 * l)) for l in range(cfg.depth)]
    x0 = inputs.host_inputs(cfg)["x0"]
    stack = LayeredStack(cfg, [upload(cfg, W) for W in Ws])
    out = stack.forward(inputs.to_device(x0, cfg.dtype))
    torch.cuda.synchronize()
    # the oracle layer by layer; the residual leaves each call rounded to dtype (R15)
    x = x0
    for l in range(cfg.depth):
        r = O.Oracle(cfg, PY.deployed_weights(cfg, Ws[l])).forward(x, l, l + 1)
        x = inputs.round_to(r["x_out"], cfg.dtype)
        got = stack.layers[l].route_counts(on_host=True).numpy()[l]
        assert np.array_equal(got, r["counts"][l])
    bf = cfg.dtype == "bf16"
    if bf:
        PY.check_drift(PY.to_np(out), x, "layered x_L", gate_abs=False)
    else:
        PY.check_hidden(PY.to_np(out), x, False, "layered x_L")
    stack.close()


# ---------------------------------------------------------------------------------------
# balance summary of the route counts (Gini, Lorenz) against the oracle's definition

def test_route_balance(cuda):
    torch = _torch()
    cfg = configs.SMALL.with_(depth=2)
    W = inputs.host_weights(cfg)
    dev = make_handle(cfg, W)
    g0, lor0 = dev.route_balance(-1)                  # no call yet: all-zero counts
    torch.cuda.synchronize()
    assert g0.item() == 0.0
    assert np.allclose(lor0.cpu().numpy(), np.arange(cfg.n_experts + 1) / cfg.n_experts)
    dev.forward(inputs.to_device(inputs.host_inputs(cfg)["x0"], cfg.dtype))
    counts = dev.route_counts(on_host=True).numpy()
    for depth in (-1, 0, 1):
        g, lor = dev.route_balance(depth)
        torch.cuda.synchronize()
        n = counts.sum(0) if depth < 0 else counts[depth]
        gr, lr = O.gini_lorenz(n)
        assert abs(g.item() - gr) < 1e-5, (depth, g.item(), gr)
        assert np.allclose(lor.cpu().numpy(), lr, atol=1e-6)
    dev.close()


# ---------------------------------------------------------------------------------------
# which kernels run: bf16 forwards launch no CUDA-core GEMM / attention / top-k kernel

@pytest.mark.parametrize("name", ["small", "medium", "decode"])
def test_bf16_calls_launch_only_tensor_core_and_streaming_kernels(cuda, name):
    torch = _torch()
    from depth_recurrent_attention_b200.dreamer import Dreamer
    cfg = configs.CONFIGS[name]
    dev = Dreamer(cfg, inputs.device_weights(cfg))
    X = inputs.device_inputs(cfg)
    lens = torch.full((cfg.batch,), cfg.cache_len, dtype=torch.int32, device="cuda")
    dev.stats(reset=True)
    for _ in range(3):  # direct, then captured into a graph, then replayed
        if cfg.is_decode:
            dev.decode_step(X["x0"], X["k_cache"], X["v_cache"], lens)
        else:
            dev.forward(X["x0"])
    torch.cuda.synchronize()
    st = dev.stats(reset=True)
    print(f"{name}: {st['launches']} launches, {st['launches_tc']} tcgen05, "
          f"{st['launches_simt']} CUDA-core GEMM/attention/top-k")
    assert st["launches_simt"] == 0
    assert st["launches_tc"] > 0 and st["launches"] >= st["launches_tc"]
    dev.close()


def test_fp32_calls_count_their_cuda_core_kernels(cuda):
    torch = _torch()
    cfg = configs.TINY
    dev = make_handle(cfg, inputs.host_weights(cfg))
    dev.stats(reset=True)
    dev.forward(inputs.to_device(inputs.host_inputs(cfg)["x0"], "fp32"))
    torch.cuda.synchronize()
    st = dev.stats(reset=True)
    assert st["launches_simt"] > 0 and st["launches_tc"] == 0
    dev.close()
