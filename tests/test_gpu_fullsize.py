"""Parity at the full workload sizes, in the launch configuration bench.py times.

The GPU runs every token; the oracle recomputes sampled outputs one by one (a depth step
for selected tokens of one sequence, with that sequence's whole context), the router on all
tokens, and whole decode steps for selected sequences.  GPU inputs are drawn on the device
and the oracle's on the host, from the same counter-based streams (any slice can be drawn on
its own), so no value the GPU computes is fed to the oracle.
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


def handle(cfg):
    from depth_recurrent_attention_b200.dreamer import Dreamer
    return Dreamer(cfg, inputs.device_weights(cfg))


def spec(name, shape, tid, dtype="bf16"):
    return inputs.TensorSpec(name, tuple(shape), "normal", 1.0, dtype, tid)


def host_rows(sp, seed, row0, nrows):
    """Rows [row0, row0 + nrows) of a 2-D view [shape[0]][prod(rest)] of a seeded tensor."""
    per = sp.numel // sp.shape[0]
    return inputs.draw(sp, seed, row0 * per, nrows * per).reshape((nrows,) + sp.shape[1:])


def step_check(cfg, dev, W, l, seq, pos, orc):
    """One depth over every token on seeded inputs; the routing of every token gated on the
    device's own router inputs (strict 1e-5 rule, exact counts), the float32 states of the
    sampled tokens against the oracle's step, the stored bf16 values as their exact rounding."""
    torch = _torch()
    T, L, h = cfg.tokens, cfg.depth, cfg.hidden
    xs = spec("x_l", (T, h), 1000 + l)
    hs = spec("da_hist", (T, L, 2, h), 2000 + l)
    x = inputs.device_tensor(xs, cfg.seed)
    hist = inputs.device_tensor(hs, cfg.seed)
    tr = dict(y=torch.empty((L, T, h), dtype=torch.bfloat16, device="cuda"),
              y_f32=torch.empty((L, T, h), dtype=torch.float32, device="cuda"),
              x_f32=torch.empty((L, T, h), dtype=torch.float32, device="cuda"),
              idx=torch.empty((L, T, cfg.top_k), dtype=torch.int32, device="cuda"),
              w=torch.empty((L, T, cfg.top_k), dtype=torch.float32, device="cuda"))
    if cfg.n_proj_experts:
        tr["xhat"] = torch.empty((L, T, h), dtype=torch.bfloat16, device="cuda")
        tr["pidx"] = torch.empty((L, T), dtype=torch.int32, device="cuda")
        tr["psig"] = torch.empty((L, T), dtype=torch.float32, device="cuda")
    out = dev.forward(x, depth_begin=l, depth_end=l + 1, da_kv=hist, trace=tr)
    torch.cuda.synchronize()
    # routing of every token, on the device's own y (and x^ for the projection router)
    y_all = PY.to_np(tr["y"][l])
    counts = dev.route_counts(on_host=True).numpy()[l]
    PY.gate_router_on_device_input(cfg, W, orc, l, y_all, tr["idx"][l].cpu().numpy(),
                                   PY.to_np(tr["w"][l]), counts, what=cfg.name)
    if cfg.n_proj_experts:
        gp_all = tr["pidx"][l].cpu().numpy()
        PY.gate_proj_router_on_device_input(cfg, orc, l, PY.to_np(tr["xhat"][l]), gp_all,
                                            PY.to_np(tr["psig"][l]), what=cfg.name)
    # the stored bf16 states are the exact rounding of the float32 ones (all tokens)
    assert np.array_equal(PY.rn_bf16(PY.to_np(tr["y_f32"][l])), y_all)
    assert np.array_equal(PY.rn_bf16(PY.to_np(tr["x_f32"][l])), PY.to_np(out))
    del y_all
    # the sampled tokens against the oracle's step with the sequence's whole context
    S = cfg.seq
    tk = seq * S + np.asarray(pos)
    x_seq = host_rows(xs, cfg.seed, seq * S, int(max(pos)) + 1)
    hist_h = np.stack([host_rows(hs, cfg.seed, int(t), 1)[0] for t in tk]).astype(np.float64)
    for j in range(l, L):
        hist_h[:, j] = 0.0
    r = orc.step_tokens(l, x_seq, hist_h, np.asarray(pos, np.int32))
    if cfg.n_proj_experts:
        keep = PY.proj_same_as_forward(cfg, W, l, gp_all[tk], r["pidx"], r["pmargin"],
                                       PY.to_np(tr["xhat"][l, tk]), r["xhat"])
    else:
        keep = np.ones(len(tk), bool)
    gy = PY.to_np(tr["y"][l, tk])
    PY.check_hidden(gy[keep], r["y"][keep], True, f"y depth {l}",
                    f32=PY.to_np(tr["y_f32"][l, tk])[keep])
    same, flips = PY.check_routing(cfg, W, l, tr["idx"][l, tk].cpu().numpy()[keep],
                                   r["idx"][keep], r["margin"][keep], gy[keep], r["y"][keep])
    gx = PY.to_np(out[tk])
    PY.check_hidden(gx[keep][same], r["x_out"][keep][same], True, f"x depth {l}",
                    f32=PY.to_np(tr["x_f32"][l, tk])[keep][same])
    return flips


@pytest.mark.parametrize("name,depths,seq,pos", [
    ("medium", (0, 1, 7, 15), 3, [0, 1, 127, 128, 1000, 2047]),
    ("large", (0, 63), 1, [0, 129, 4095, 8191]),
])
def test_fullsize_step_sampled(cuda, name, depths, seq, pos):
    cfg = configs.CONFIGS[name]
    W = inputs.host_weights(cfg)
    dev = handle(cfg)
    orc = O.Oracle(cfg, PY.deployed_weights(cfg, W))
    for l in depths:
        flips = step_check(cfg, dev, W, l, seq, pos, orc)
        print(f"{name} depth {l}: {flips}/{len(pos)} sampled tokens flipped at near ties")
    dev.close()


@pytest.mark.parametrize("name,l", [("medium", 7), ("large", 40), ("decode", 31)])
def test_fullsize_router_strict(cuda, name, l):
    cfg = configs.CONFIGS[name]
    W = inputs.host_weights(cfg)
    ys = spec("y", (cfg.tokens, cfg.hidden), 3000 + l)
    y_dev = inputs.device_tensor(ys, cfg.seed)
    y_host = inputs.draw_tensor(ys, cfg.seed)
    dev = handle(cfg)
    idx, w, counts = dev.route_experts(l, y_dev)
    ref = O.Oracle(cfg, W).route(l, y_host)
    idx = idx.cpu().numpy()
    same, flips = PY.check_routing(cfg, W, l, idx, ref["idx"], ref["margin"], strict=True)
    print(f"router {name} depth {l}: {flips} flips at "
          f"{int((ref['margin'] <= PY.NEAR_TIE).sum())} near ties over {cfg.tokens} tokens")
    assert np.allclose(PY.weights_by_expert(idx, PY.to_np(w))[same],
                       PY.weights_by_expert(ref["idx"], ref["w"])[same], atol=1e-5)
    c = counts.cpu().numpy()
    assert np.array_equal(c, np.bincount(idx.ravel(), minlength=cfg.n_experts))
    if flips == 0:
        assert np.array_equal(c, ref["counts"])
    dev.close()


def decode_run(cfg, seqs):
    torch = _torch()
    dev = handle(cfg)
    X = inputs.device_inputs(cfg)
    lens = torch.full((cfg.batch,), cfg.cache_len, dtype=torch.int32, device="cuda")
    L, k = cfg.depth, cfg.top_k
    tr = dict(y=torch.empty((L, cfg.batch, cfg.hidden), dtype=torch.bfloat16, device="cuda"),
              y_f32=torch.empty((L, cfg.batch, cfg.hidden), dtype=torch.float32, device="cuda"),
              x_f32=torch.empty((L, cfg.batch, cfg.hidden), dtype=torch.float32, device="cuda"),
              idx=torch.empty((L, cfg.batch, k), dtype=torch.int32, device="cuda"),
              w=torch.empty((L, cfg.batch, k), dtype=torch.float32, device="cuda"))
    out = dev.decode_step(X["x0"], X["k_cache"], X["v_cache"], lens, trace=tr)
    torch.cuda.synchronize()
    kslot = PY.to_np(X["k_cache"][:, :, :, cfg.cache_len])   # [L][B][H][d]
    res = dict(out=PY.to_np(out), y=PY.to_np(tr["y"]), idx=tr["idx"].cpu().numpy(), kslot=kslot,
               y_f32=PY.to_np(tr["y_f32"]), x_f32=PY.to_np(tr["x_f32"]), w=PY.to_np(tr["w"]),
               counts=dev.route_counts(on_host=True).numpy())
    del X
    dev.close()
    W = inputs.host_weights(cfg)
    # every depth's routing of all sequences, on the states the device routed
    orc_all = O.Oracle(cfg, PY.deployed_weights(cfg, W))
    for l in range(L):
        PY.gate_router_on_device_input(cfg, W, orc_all, l, res["y"][l], res["idx"][l],
                                       res["w"][l], res["counts"][l], what=cfg.name)
    assert np.array_equal(PY.rn_bf16(res["y_f32"]), res["y"])
    assert np.array_equal(PY.rn_bf16(res["x_f32"][L - 1]), res["out"])
    o = O.Oracle(cfg.with_(batch=1), PY.deployed_weights(cfg, W))
    sp = {s.name: s for s in inputs.input_specs(cfg)}
    H, d, cap = cfg.n_heads, cfg.head_dim, cfg.cache_len + 1
    refs = {}
    for b in seqs:
        kc = np.empty((L, H, cap, d))
        vc = np.empty((L, H, cap, d))
        per = H * cap * d
        for l in range(L):
            off = (l * cfg.batch + b) * per
            kc[l] = inputs.draw(sp["k_cache"], cfg.seed, off, per).reshape(H, cap, d)
            vc[l] = inputs.draw(sp["v_cache"], cfg.seed, off, per).reshape(H, cap, d)
        x = inputs.draw(sp["x0"], cfg.seed, b * cfg.hidden, cfg.hidden)
        refs[b] = (o.decode_seq(x, kc, vc, cfg.cache_len), kc[:, :, cfg.cache_len].copy())
    return res, refs, W


def test_fullsize_decode_first_depth(cuda):
    """Real routing: the routing of every depth is gated on the states the device routed;
    depth 0's states are compared token by token with the oracle's decode (later depths of a
    free-running bf16 decode follow routing flips at near ties)."""
    cfg = configs.DECODE
    res, refs, W = decode_run(cfg, (0, 37))
    for b, (r, kslot) in refs.items():
        PY.check_hidden(res["y"][0, b], r["y"][0], True, f"y depth 0 seq {b}",
                        f32=res["y_f32"][0, b])
        PY.check_hidden(res["kslot"][0, b], kslot[0], True, f"k slot depth 0 seq {b}")
        PY.check_routing(cfg, W, 0, res["idx"][0, b:b + 1], r["idx"][0:1], r["margin"][0:1],
                         res["y"][0, b:b + 1], r["y"][0:1])


def test_fullsize_decode_flip_free_all_depths(cuda):
    """Decode shapes (64 sequences, 4096 cached tokens, 32 depths, h 1024) with E = k = 16,
    so no routing decision can flip and all 32 depths stay comparable."""
    cfg = configs.DECODE.with_(n_experts=16, top_k=16)
    res, refs, W = decode_run(cfg, (0, 63))
    for b, (r, kslot) in refs.items():
        for l in range(cfg.depth):
            PY.check_drift(res["y"][l, b], r["y"][l], f"y depth {l} seq {b}", gate_abs=(l == 0),
                           f32=res["y_f32"][l, b])
        PY.check_drift(res["kslot"][:, b], kslot, f"k slots seq {b}", gate_abs=False)
        e, rl = PY.check_drift(res["out"][b], r["x_out"], f"x_out seq {b}", gate_abs=False,
                               f32=res["x_f32"][cfg.depth - 1, b])
        print(f"decode flip-free seq {b}: x_out max-abs {e:.3g} rel-L2 {rl:.3g}")
