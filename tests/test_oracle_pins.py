"""Pins of the CPU oracle to what the pages and the mathematics fix (no GPU).

Each test states the fact it checks and where that fact comes from.  None of them re-types
the oracle's own code: they use closed forms, invariants, special cases that reduce to a
textbook result, and brute force with library routines on tiny inputs.
"""
import numpy as np
import pytest

import oracle as O
from depth_recurrent_attention_b200 import configs, inputs

RNG = np.random.default_rng(1234)


def tiny_cfg(**kw):
    return configs.TINY.with_(**kw)


def rand_weights(cfg, seed=0, scale_o=1.0):
    """Seeded fp32 weights for a small hand-made configuration."""
    W = inputs.host_weights(cfg.with_(seed=seed))
    if scale_o != 1.0:
        W["w_o"] = (W["w_o"] * scale_o).astype(np.float32)
    return W


# ---------------------------------------------------------------------------------------
# RMSNorm (papernotes "Overall framework": RMSNorm on the residual stream)

def test_rmsnorm_worked_example():
    # x = (3, 4): mean square 12.5, so x^ = (3, 4) / sqrt(12.5)
    out = O.rmsnorm([3.0, 4.0], np.ones(2, np.float32), 0.0)
    assert np.allclose(out, [3 / np.sqrt(12.5), 4 / np.sqrt(12.5)], rtol=0, atol=1e-15)


def test_rmsnorm_unit_mean_square_and_scale_invariance():
    x = RNG.normal(size=257) * 7.3
    g = np.ones(257, np.float32)
    eps = 1e-6
    out = O.rmsnorm(x, g, eps)
    ms = np.mean(x ** 2)
    assert abs(np.mean(out ** 2) - ms / (ms + eps)) < 1e-12
    out2 = O.rmsnorm(x * 1e3, g, 0.0)
    assert np.allclose(out2, O.rmsnorm(x, g, 0.0), rtol=1e-13, atol=1e-13)
    gg = RNG.normal(size=257).astype(np.float32)
    assert np.allclose(O.rmsnorm(x, gg, eps), gg * out, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------------------
# RoPE (rotate-half convention, Su et al. RoFormer) and depth RoPE with a reversed half
# (papernotes "Key design 1"; gist.science "Methodology")

def test_rope_two_dims_is_plain_rotation():
    # n = 2: the single pair turns by pos * base^0 = pos radians
    for pos in (0.0, 1.0, 2.5, 17.0):
        v = O.rope([1.0, 0.0], pos)
        assert np.allclose(v, [np.cos(pos), np.sin(pos)], atol=1e-15)
        v = O.rope([0.0, 1.0], pos)
        assert np.allclose(v, [-np.sin(pos), np.cos(pos)], atol=1e-15)


def test_rope_pairing_and_ladder_special_values():
    n = 16
    for i in range(n // 2):
        e = np.zeros(n)
        e[i] = 1.0
        v = O.rope(e, 3.0)
        support = set(np.nonzero(np.abs(v) > 1e-15)[0].tolist())
        assert support <= {i, i + n // 2}            # rotate-half pairs (i, i + n/2)
    # n = 4, base 10^4: second pair turns 10^4^(-1/2) = 0.01 rad per position
    e = np.array([0.0, 1.0, 0.0, 0.0])
    v = O.rope(e, 1.0)
    assert np.isclose(np.arctan2(v[3], v[1]), 0.01, atol=1e-15)


def test_rope_norm_identity_and_relative_position():
    d = 64
    q, k = RNG.normal(size=d), RNG.normal(size=d)
    assert np.allclose(O.rope(q, 0.0), q, atol=0)
    assert np.isclose(np.linalg.norm(O.rope(q, 123.0)), np.linalg.norm(q), rtol=1e-14)
    s1 = O.rope(q, 10.0) @ O.rope(k, 3.0)
    s2 = O.rope(q, 57.0) @ O.rope(k, 50.0)
    assert abs(s1 - s2) < 1e-11
    # group property R_a R_b = R_{a+b}
    assert np.allclose(O.rope(O.rope(q, 5.0), 9.0), O.rope(q, 14.0), atol=1e-12)


def test_depth_rope_forward_half_depends_on_depth_difference_only():
    d, L = 64, 16
    q, k = RNG.normal(size=d), RNG.normal(size=d)
    h2 = d // 2
    for (l, j, c) in [(5, 2, 3), (7, 0, 6), (4, 4, 9)]:
        a = O.depth_rope(q, l, L)[:h2] @ O.depth_rope(k, j, L)[:h2]
        b = O.depth_rope(q, l + c, L)[:h2] @ O.depth_rope(k, j + c, L)[:h2]
        assert abs(a - b) < 1e-11


def test_depth_rope_reversed_half():
    d, L = 64, 16
    q, k = RNG.normal(size=d), RNG.normal(size=d)
    h2 = d // 2
    # second half sits at L-1-l: its score depends on j - l, i.e. the same shift reversed
    a = O.depth_rope(q, 5, L)[h2:] @ O.depth_rope(k, 2, L)[h2:]
    b = O.depth_rope(q, 8, L)[h2:] @ O.depth_rope(k, 5, L)[h2:]
    assert abs(a - b) < 1e-11
    # at depth 0 the first half is untouched and the second half turns to position L-1
    v0 = O.depth_rope(q, 0, L)
    assert np.array_equal(v0[:h2], q[:h2])
    assert np.allclose(v0[h2:], O.rope(q[h2:], L - 1), atol=1e-15)
    # at the last depth the roles swap
    vL = O.depth_rope(q, L - 1, L)
    assert np.allclose(vL[:h2], O.rope(q[:h2], L - 1), atol=1e-15)
    assert np.array_equal(vL[h2:], q[h2:])
    # and the two halves are not rotated alike at depths other than the middle one
    assert not np.allclose(O.depth_rope(q, 2, L)[:h2] @ q[:h2],
                           O.depth_rope(q, 2, L)[h2:] @ q[h2:])
    assert np.isclose(np.linalg.norm(O.depth_rope(q, 3, L)), np.linalg.norm(q), rtol=1e-14)


# ---------------------------------------------------------------------------------------
# scaled dot-product attention / softmax

def test_softmax_rows_sum_to_one_and_closed_forms():
    d = 16
    q = RNG.normal(size=d)
    K = RNG.normal(size=(37, d))
    V = RNG.normal(size=(37, d))
    out, p = O.attend(q, K, V)
    assert abs(p.sum() - 1.0) < 1e-12 * 37
    # one key: the output is that key's value exactly (DA at depth 0 equals its V)
    out1, p1 = O.attend(q, K[:1], V[:1])
    assert np.array_equal(out1, V[0]) and p1[0] == 1.0
    # identical keys: uniform weights, output is the mean of the values
    Ke = np.repeat(K[:1], 5, axis=0)
    oute, pe = O.attend(q, Ke, V[:5])
    assert np.allclose(pe, 0.2, atol=1e-15) and np.allclose(oute, V[:5].mean(0), atol=1e-14)
    # two keys: weight of key 1 is sigmoid(s1 - s0), scores scaled by 1/sqrt(d)
    s = K[:2] @ q / np.sqrt(d)
    _, p2 = O.attend(q, K[:2], V[:2])
    assert np.isclose(p2[1], 1 / (1 + np.exp(-(s[1] - s[0]))), rtol=1e-13)


# ---------------------------------------------------------------------------------------
# routing sigma(x) = norm(TopK(sigmoid(x), x + b, k))   (papernotes "Key design 2")

def test_topk_matches_sort_with_index_tiebreak():
    for E, k in [(16, 2), (256, 4), (1024, 8), (33, 33)]:
        z = RNG.normal(size=E)
        b = RNG.uniform(-0.1, 0.1, size=E).astype(np.float32)
        idx, w, margin = O.topk(z, b, k)
        key = z + b.astype(np.float64)
        order = sorted(range(E), key=lambda e: (-key[e], e))
        assert list(idx) == order[:k]
        assert abs(w.sum() - 1.0) < 1e-12
        sg = 1 / (1 + np.exp(-z[idx]))
        assert np.allclose(w, sg / sg.sum(), rtol=1e-13)
        if k < E:
            assert np.isclose(margin, key[order[k - 1]] - key[order[k]], atol=1e-15)
        else:
            assert margin == np.inf


def test_topk_zero_bias_equals_topk_of_sigmoid():
    z = RNG.normal(size=300) * 3
    idx, _, _ = O.topk(z, np.zeros(300, np.float32), 7)
    s = 1 / (1 + np.exp(-z))
    assert set(idx.tolist()) == set(np.argsort(-s, kind="stable")[:7].tolist())


def test_topk_bias_chooses_but_does_not_weight():
    z = np.array([0.0, 0.1, 0.2, 0.3])
    b = np.array([5.0, 0.0, 0.0, 0.0], np.float32)
    idx, w, _ = O.topk(z, b, 2)
    assert list(idx) == [0, 3]                       # bias lifts expert 0 into the picks
    s = 1 / (1 + np.exp(-np.array([0.0, 0.3])))
    assert np.allclose(w, s / s.sum())               # weights come from sigmoid(z), not z+b


def test_topk_ties_go_to_lower_index():
    idx, w, margin = O.topk(np.zeros(10), np.zeros(10, np.float32), 3)
    assert list(idx) == [0, 1, 2] and margin == 0.0 and np.allclose(w, 1 / 3)


def test_bias_update_closed_form():
    # N = (1, 5, 3, 3) summed over depths -> sorted (1, 3, 3, 5), lower median 3
    counts = np.array([[1, 2, 1, 2], [0, 3, 2, 1]], np.int32)
    b = O.bias_update(counts, 0.01, np.zeros(4))
    assert np.allclose(b, [0.01, -0.01, 0.0, 0.0])


# ---------------------------------------------------------------------------------------
# linear-MoE projection with the absorbed shared expert (papernotes "Key design 3")

def test_absorbed_shared_expert_identity():
    Wp = RNG.normal(size=(48, 80)).astype(np.float32)
    Ws = RNG.normal(size=(48, 80)).astype(np.float32)
    x = RNG.normal(size=48)
    for sigma in (0.51, 0.93):
        a = O.linear_moe(x, Wp, Ws, sigma)
        b = O.linear_moe(x, Wp, Ws, sigma, absorbed=True)
        assert np.allclose(a, b, rtol=1e-12, atol=1e-12)
        assert np.allclose(a, sigma * (x @ Wp.astype(np.float64)) + sigma * (x @ Ws.astype(np.float64)),
                           rtol=1e-12, atol=1e-12)


def test_expert_ffn_scalar_case():
    # h = 1, m = 1: SiLU(y w1) w2
    y, w1, w2 = 0.7, 1.3, -2.1
    u = y * w1
    out = O.expert(np.array([y]), np.array([[w1]], np.float32), np.array([[w2]], np.float32))
    w1f, w2f = np.float32(w1), np.float32(w2)
    u = y * float(w1f)
    assert np.isclose(out[0], u / (1 + np.exp(-u)) * float(w2f), rtol=1e-14)


# ---------------------------------------------------------------------------------------
# whole block

def _closed_form_single_token(cfg, W, x0):
    """L = 1, s = 1, E = k: SA over one key returns v_SA, DA at depth 0 returns v_DA,
    all experts are picked.  Everything reduces to plain matrix products.  With P projection
    experts each token takes p* = argmax_p z_P (numpy's argmax: the first of equal maxima)
    and runs sigma (W_p* + W_shared) with sigma = sigmoid(z_P[p*]) (papernotes "Key design
    3": sigma x W + max(sigma^) x W_shared, the router shared by QKV and O).  Returns
    (x_out, p*, sigma)."""
    h, dr = cfg.hidden, cfg.router_dim
    f = lambda a: np.asarray(a, np.float64)
    x = f(x0)
    T = x.shape[0]
    xh = x / np.sqrt(np.mean(x ** 2, axis=-1, keepdims=True) + cfg.rms_eps) * f(W["g"])
    P = cfg.n_proj_experts
    if P > 0:
        # at L = 1 the depth RoPE of depth 0 rotates both halves by position 0: the identity
        kP = np.stack([O.depth_rope(f(k), 0, 1) for k in W["k_P"]])       # [P][d_r]
        zP = (xh @ f(W["w_qP"])) @ kP.T / np.sqrt(dr)                     # [T][P]
        pstar = np.argmax(zP, axis=1)
        sig = 1 / (1 + np.exp(-zP[np.arange(T), pstar]))
        Wqkv = sig[:, None, None] * (f(W["w_qkv"])[pstar] + f(W["w_qkv_shared"])[None])
        Wo = sig[:, None, None] * (f(W["w_o"])[pstar] + f(W["w_o_shared"])[None])
        qkv = np.einsum("ti,tij->tj", xh, Wqkv)
    else:
        qkv = xh @ f(W["w_qkv"][0])
        Wo, pstar, sig = None, np.zeros(T, int), np.ones(T)
    v_sa, v_da = qkv[:, 2 * h:3 * h], qkv[:, 5 * h:6 * h]
    cat = np.concatenate([v_sa, v_da], axis=1)
    o = np.einsum("ti,tij->tj", cat, Wo) if Wo is not None else cat @ f(W["w_o"][0])
    y = xh + o
    kE = np.stack([O.depth_rope(f(k), 0, 1) for k in W["k_E"]])
    z = (y @ f(W["w_qE"])) @ kE.T / np.sqrt(dr)
    s = 1 / (1 + np.exp(-z))
    w = s / s.sum(1, keepdims=True)
    out = y.copy()
    for e in range(cfg.n_experts):
        u = y @ f(W["w1"][e])
        out += w[:, e:e + 1] * ((u / (1 + np.exp(-u))) @ f(W["w2"][e]))
    return out, pstar, sig


@pytest.mark.parametrize("P", [0, 1])
def test_block_reduces_to_closed_form(P):
    cfg = tiny_cfg(batch=3, seq=1, depth=1, n_experts=3, top_k=3, n_proj_experts=P)
    W = rand_weights(cfg, seed=11)
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    ref, _, _ = _closed_form_single_token(cfg, W, x0)
    assert np.allclose(r["x_out"], ref, rtol=1e-11, atol=1e-11)


def test_block_closed_form_with_a_non_unit_norm_gain():
    """The same single-token closed form with a random RMSNorm gain g (the configurations all
    use g = 1): the block's normalised state is g * x / rms(x) wherever it is used (QKV input,
    residual, projection router)."""
    cfg = tiny_cfg(batch=3, seq=1, depth=1, n_experts=3, top_k=3, n_proj_experts=1)
    W = dict(rand_weights(cfg, seed=15))
    W["g"] = (0.5 + np.random.default_rng(15).random(cfg.hidden)).astype(np.float32)
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    ref, _, _ = _closed_form_single_token(cfg, W, x0)
    assert np.allclose(r["x_out"], ref, rtol=1e-11, atol=1e-11)


def test_block_with_three_projection_experts_closed_form():
    """P = 3 projection experts with distinct QKV/O matrices; the keys are built so that the
    six tokens pick all three experts (token t aligns with expert t mod 3) and the argmin
    differs from the argmax for every token.  The oracle's p*, sigma, margin and output
    must equal the numpy chain; so an argmin for the argmax, a wrong expert offset into the
    stacked matrices, or a sigma from another expert's score fails here."""
    P = 3
    cfg = tiny_cfg(batch=6, seq=1, depth=1, n_experts=3, top_k=3, n_proj_experts=P)
    W = dict(rand_weights(cfg, seed=12))
    x0 = inputs.host_inputs(cfg)["x0"]
    f = lambda a: np.asarray(a, np.float64)
    x = f(x0)
    xh = x / np.sqrt(np.mean(x ** 2, axis=-1, keepdims=True) + cfg.rms_eps)
    q = xh @ f(W["w_qP"])
    W["k_P"] = np.stack([3.0 * q[p] / np.linalg.norm(q[p]) for p in range(P)]).astype(np.float32)
    # the stacked expert matrices differ from one another
    for name in ("w_qkv", "w_o"):
        for a in range(P):
            for b in range(a + 1, P):
                assert np.abs(W[name][a] - W[name][b]).max() > 0.1
    ref, pstar, sig = _closed_form_single_token(cfg, W, x0)
    kP = f(W["k_P"])
    zP = q @ kP.T / np.sqrt(cfg.router_dim)
    assert sorted(set(pstar.tolist())) == [0, 1, 2], pstar
    assert np.all(np.argmin(zP, axis=1) != pstar)
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    assert np.array_equal(r["pidx"][0], pstar)
    assert np.allclose(r["psig"][0], sig, rtol=1e-12, atol=0)
    second = np.sort(zP, axis=1)[:, -2]
    assert np.allclose(r["pmargin"][0], zP.max(1) - second, rtol=1e-10, atol=1e-12)
    assert np.allclose(r["x_out"], ref, rtol=1e-11, atol=1e-11)
    # the router alone (the entry the GPU parity tests route the device's x^ with)
    pr = O.Oracle(cfg, W, threads=1).proj_route(0, xh.astype(np.float32))
    xh32 = f(xh.astype(np.float32))
    z32 = (xh32 @ f(W["w_qP"])) @ kP.T / np.sqrt(cfg.router_dim)
    assert np.array_equal(pr["pidx"], np.argmax(z32, axis=1))
    assert np.allclose(pr["psig"], 1 / (1 + np.exp(-z32.max(1))), rtol=1e-12, atol=0)


def test_projection_router_rotates_keys_by_the_depth():
    """At depth l of L the projection keys carry the depth RoPE of l (reading R12, the same
    form as expert attention): the router alone equals argmax over (x^ W_qP) . R_l k_p."""
    cfg = tiny_cfg(batch=4, seq=2, depth=3, n_proj_experts=5)
    W = rand_weights(cfg, seed=13)
    xh = RNG.normal(size=(cfg.tokens, cfg.hidden)).astype(np.float32)
    f = lambda a: np.asarray(a, np.float64)
    q = f(xh) @ f(W["w_qP"])
    for l in range(cfg.depth):
        kP = np.stack([O.depth_rope(f(k), l, cfg.depth) for k in W["k_P"]])
        z = q @ kP.T / np.sqrt(cfg.router_dim)
        r = O.Oracle(cfg, W, threads=1).proj_route(l, xh)
        assert np.array_equal(r["pidx"], np.argmax(z, axis=1))
        assert np.allclose(r["psig"], 1 / (1 + np.exp(-z.max(1))), rtol=1e-12, atol=0)
        assert np.allclose(r["pmargin"], z.max(1) - np.sort(z, axis=1)[:, -2], rtol=1e-9, atol=1e-12)


def test_da_reshape_equals_explicit_loops():
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=2)
    a = o.forward(x0)
    b = o.forward(x0, da_loops=True)
    assert np.allclose(a["x_out"], b["x_out"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(a["idx"], b["idx"])


def test_da_at_depth_zero_returns_its_value():
    # SA rows of W_O zero, DA rows identity, experts off: x_1 = x^ + v_DA(x^)
    cfg = tiny_cfg(depth=1, n_experts=2, top_k=1)
    W = rand_weights(cfg, seed=3)
    h = cfg.hidden
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, h:, :] = np.eye(h, dtype=np.float32)
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    x = x0.astype(np.float64)
    xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
    v_da = xh @ W["w_qkv"][0][:, 5 * h:6 * h].astype(np.float64)
    assert np.allclose(r["x_out"], xh + v_da, rtol=1e-12, atol=1e-12)


def test_sa_causality_and_single_token():
    cfg = tiny_cfg(batch=2, seq=8, depth=2)
    W = rand_weights(cfg, seed=5)
    x0 = inputs.host_inputs(cfg)["x0"].copy()
    o = O.Oracle(cfg, W, threads=1)
    a = o.forward(x0)["x_out"]
    x1 = x0.copy()
    x1[5] += 1.0                        # token 5 of sequence 0
    b = o.forward(x1)["x_out"]
    assert np.array_equal(a[:5], b[:5])          # earlier tokens bit-identical
    assert not np.allclose(a[5:8], b[5:8])
    assert np.array_equal(a[8:], b[8:])          # other sequence untouched


def test_sa_with_zero_keys_is_the_causal_running_mean_of_values():
    """Sequence attention with every key zero: all scores are 0, so the causal softmax gives
    each of the keys 0..t the weight 1/(t+1) and position t returns the running mean of v over
    its own sequence (papernotes "Overall framework": causal attention over time steps;
    reading R4).  A dropped mask would average over the whole sequence, a wrong limit or a
    missing normaliser would change the count.  L = 1, the DA rows of W_O and the experts'
    W2 zero, the SA rows of W_O the identity: x_1 = x^ + running_mean(x^ W_v)."""
    cfg = tiny_cfg(batch=2, seq=8, depth=1, n_experts=2, top_k=1)
    W = rand_weights(cfg, seed=11)
    h, s = cfg.hidden, cfg.seq
    W["w_qkv"] = W["w_qkv"].copy()
    W["w_qkv"][0][:, h:2 * h] = 0.0                   # k_SA = 0
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, :h, :] = np.eye(h, dtype=np.float32)   # SA rows: identity; DA rows: 0
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    x = x0.astype(np.float64)
    xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
    v = (xh @ W["w_qkv"][0][:, 2 * h:3 * h].astype(np.float64)).reshape(cfg.batch, s, h)
    run_mean = np.cumsum(v, axis=1) / np.arange(1, s + 1)[None, :, None]
    assert np.allclose(r["x_out"], xh + run_mean.reshape(-1, h), rtol=1e-12, atol=1e-12)


def test_sa_rotates_queries_and_keys_by_their_positions_in_the_sequence():
    """Sequence attention over two tokens with one head of 4 dims, worked by hand: queries and
    keys turn by their position inside the sequence (rotate-half pairs (0, 2) and (1, 3) at
    angles p and p / 100, i.e. base 10000 over d = 4: reading R5), so the second token scores
    the first by (R_1 q_1) . k_0 and itself by q_1 . k_1 (a rotation keeps the dot product);
    values are not rotated.  SA rows of W_O the identity, DA rows and experts off, L = 1."""
    cfg = tiny_cfg(batch=1, seq=2, hidden=4, n_heads=1, head_dim=4, depth=1, n_experts=2,
                   top_k=1, router_dim=4)
    W = rand_weights(cfg, seed=13)
    h = cfg.hidden
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, :h, :] = np.eye(h, dtype=np.float32)
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    x = x0.astype(np.float64)
    xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
    Wf = W["w_qkv"][0].astype(np.float64)
    q, k, v = xh @ Wf[:, 0:4], xh @ Wf[:, 4:8], xh @ Wf[:, 8:12]

    def turn(u, p):   # angles p * 1 and p * 0.01 on the pairs (0, 2) and (1, 3)
        a0, a1 = p * 1.0, p * 0.01
        return np.array([u[0] * np.cos(a0) - u[2] * np.sin(a0),
                         u[1] * np.cos(a1) - u[3] * np.sin(a1),
                         u[0] * np.sin(a0) + u[2] * np.cos(a0),
                         u[1] * np.sin(a1) + u[3] * np.cos(a1)])
    s10 = turn(q[1], 1) @ k[0] / 2.0          # k_0 at position 0 is not turned
    s11 = q[1] @ k[1] / 2.0
    p0 = 1.0 / (1.0 + np.exp(s11 - s10))
    a = np.stack([v[0], p0 * v[0] + (1 - p0) * v[1]])
    assert abs(s10 - q[1] @ k[0] / 2.0) > 1e-3           # the rotation matters here
    assert np.allclose(r["x_out"], xh + a, rtol=1e-12, atol=1e-12)


def test_da_rotates_by_depth_with_the_second_half_reversed_worked_by_hand():
    """Depth attention of one token over depths 0 and 1 (L = 2) with one head of 4 dims,
    worked by hand: each half of the head (2 dims, one rotate-half pair at base^0 = 1 rad a
    step) turns by the depth for the first half and by L - 1 - depth for the second (reading
    R6, the pages' half-reversed depth RoPE), queries and keys alike; values are not turned.
    SA rows of W_O and the experts off, DA rows of W_O the identity."""
    cfg = tiny_cfg(batch=1, seq=1, hidden=4, n_heads=1, head_dim=4, depth=2, n_experts=2,
                   top_k=1, router_dim=4)
    W = rand_weights(cfg, seed=14)
    h = cfg.hidden
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, h:, :] = np.eye(h, dtype=np.float32)
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    Wf = W["w_qkv"][0].astype(np.float64)
    norm = lambda x: x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)

    def turn(u, l):   # first half by l, second half by L - 1 - l (1 rad a step)
        a, b = float(l), float(cfg.depth - 1 - l)
        return np.array([u[0] * np.cos(a) - u[1] * np.sin(a), u[0] * np.sin(a) + u[1] * np.cos(a),
                         u[2] * np.cos(b) - u[3] * np.sin(b), u[2] * np.sin(b) + u[3] * np.cos(b)])
    xh0 = norm(x0.astype(np.float64))
    k0, v0 = turn((xh0 @ Wf[:, 16:20])[0], 0), (xh0 @ Wf[:, 20:24])[0]
    xh1 = norm(xh0 + v0)                      # depth 0 attends to itself only: a_0 = v_0
    q1, k1, v1 = (xh1 @ Wf[:, 12:16])[0], (xh1 @ Wf[:, 16:20])[0], (xh1 @ Wf[:, 20:24])[0]
    q1, k1 = turn(q1, 1), turn(k1, 1)
    s0, s1 = q1 @ k0 / 2.0, q1 @ k1 / 2.0
    p0 = 1.0 / (1.0 + np.exp(s1 - s0))
    want = xh1 + p0 * v0 + (1 - p0) * v1
    assert np.allclose(r["x_out"][0], want[0], rtol=1e-12, atol=1e-12)


def test_expert_attention_scores_depth_rotated_keys_worked_by_hand():
    """Expert attention of one token over two depths (L = 2), two experts, top-1, worked by
    hand: the unrotated query q = y W_qE against each expert key turned by the half-reversed
    depth rotation of the depth (reading R8: "depth-RoPE'd expert keys"), the pick by z + b
    (R9), weight 1 (R10), x_{l+1} = y + SiLU(y W1_e) W2_e (R11).  W_O zero, so y_l = x^_l.
    The seed is one where unrotated keys would pick another expert at both depths."""
    cfg = tiny_cfg(batch=1, seq=1, hidden=4, n_heads=1, head_dim=4, depth=2, n_experts=2,
                   top_k=1, router_dim=4, seed=21)
    W = dict(inputs.host_weights(cfg))
    W["w_o"] = np.zeros_like(W["w_o"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    f = lambda a: np.asarray(a, np.float64)
    norm = lambda x: x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)

    def turn(u, l):   # first half by l, second half by L - 1 - l (1 rad a step)
        a, b = float(l), float(cfg.depth - 1 - l)
        return np.array([u[0] * np.cos(a) - u[1] * np.sin(a), u[0] * np.sin(a) + u[1] * np.cos(a),
                         u[2] * np.cos(b) - u[3] * np.sin(b), u[2] * np.sin(b) + u[3] * np.cos(b)])
    x, picks, unrotated = f(x0), [], []
    for l in range(cfg.depth):
        y = norm(x)
        q = (y @ f(W["w_qE"]))[0]
        z = np.array([q @ turn(f(W["k_E"][e]), l) / 2.0 for e in range(2)])
        z_plain = np.array([q @ f(W["k_E"][e]) / 2.0 for e in range(2)])
        e = int(np.argmax(z + f(W["bias"])))
        picks.append(e)
        unrotated.append(int(np.argmax(z_plain + f(W["bias"]))))
        u = y @ f(W["w1"][e])
        x = y + (u / (1.0 + np.exp(-u))) @ f(W["w2"][e])
    assert picks != unrotated                              # the rotation decides here
    assert [int(r["idx"][l][0][0]) for l in range(cfg.depth)] == picks
    assert np.allclose(r["x_out"], x, rtol=1e-12, atol=1e-12)


def test_da_with_zero_keys_is_the_running_mean_over_depths():
    """Depth attention with every key zero: the token's scores over depths 0..l are all 0, so
    depth l returns the mean of v_DA over depths 0..l, the current one included (papernotes
    "Key design 1": attention over the token's own earlier depth states; reading R2).  SA rows
    of W_O and the experts' W2 zero, the DA rows of W_O the identity, L = 4: the recurrence
    x^_l = RMSNorm(x_l), v_l = x^_l W_v, x_{l+1} = x^_l + mean(v_0..v_l) in closed form.  An
    exclusive slice, a missing normaliser or a depth read from the wrong slot all fail."""
    cfg = tiny_cfg(batch=1, seq=4, depth=4, n_experts=2, top_k=1)
    W = rand_weights(cfg, seed=12)
    h = cfg.hidden
    W["w_qkv"] = W["w_qkv"].copy()
    W["w_qkv"][0][:, 4 * h:5 * h] = 0.0                # k_DA = 0
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, h:, :] = np.eye(h, dtype=np.float32)   # DA rows: identity; SA rows: 0
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    Wv = W["w_qkv"][0][:, 5 * h:6 * h].astype(np.float64)
    x = x0.astype(np.float64)
    vs = []
    for _ in range(cfg.depth):
        xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
        vs.append(xh @ Wv)
        x = xh + np.mean(vs, axis=0)
    assert np.allclose(r["x_out"], x, rtol=1e-12, atol=1e-12)


def test_batch_permutation_equivariance():
    cfg = tiny_cfg(batch=3, seq=4, depth=2)
    W = rand_weights(cfg, seed=6)
    x0 = inputs.host_inputs(cfg)["x0"].reshape(3, 4, -1)
    o = O.Oracle(cfg, W, threads=1)
    a = o.forward(x0.reshape(12, -1))["x_out"].reshape(3, 4, -1)
    b = o.forward(x0[[2, 0, 1]].reshape(12, -1))["x_out"].reshape(3, 4, -1)
    assert np.array_equal(a[[2, 0, 1]], b)


def test_counts_are_histogram_of_indices():
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    r = O.Oracle(cfg, W, threads=1).forward(inputs.host_inputs(cfg)["x0"])
    T, k, L, E = cfg.tokens, cfg.top_k, cfg.depth, cfg.n_experts
    assert np.all(r["counts"].sum(1) == T * k)
    for l in range(L):
        assert np.array_equal(r["counts"][l], np.bincount(r["idx"][l].ravel(), minlength=E))
        for t in range(T):
            assert len(set(r["idx"][l, t].tolist())) == k
    assert np.allclose(r["w"].sum(-1), 1.0, atol=1e-12)


def test_depth_range_composes():
    """Running depths [0, 2) then [2, L) through the DA buffer equals [0, L)."""
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=1)
    full = o.forward(x0)
    a = o.forward(x0, 0, 2)
    b = o.forward(a["x_out"].astype(np.float32), 2, cfg.depth, da_kv=a["da_kv"])
    # the middle state passes through float32, so compare loosely
    assert np.allclose(b["x_out"], full["x_out"], rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("variant", [0, 2])
def test_step_tokens_equals_forward_rows(variant):
    cfg = tiny_cfg(batch=2, seq=8, depth=3, variant=variant)
    W = rand_weights(cfg, seed=8)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=1)
    full = o.forward(x0, 0, 2)
    x2 = full["x_out"].astype(np.float32)
    ref = o.forward(x2, 2, 3, da_kv=full["da_kv"])
    seq = 1
    pos = np.array([0, 3, 7], np.int32)
    toks = seq * cfg.seq + pos
    st = o.step_tokens(2, x2[seq * cfg.seq:(seq + 1) * cfg.seq], full["da_kv"][toks], pos)
    assert np.allclose(st["x_out"], ref["x_out"][toks], rtol=1e-12, atol=1e-12)
    assert np.array_equal(st["idx"], ref["idx"][2][toks])


@pytest.mark.parametrize("P,variant", [(0, 0), (2, 0), (0, 1), (0, 2)])
def test_decode_equals_last_row_of_longer_prefill(P, variant):
    cfg = tiny_cfg(batch=1, seq=6, depth=3, n_proj_experts=P, variant=variant)
    W = rand_weights(cfg, seed=9)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=1)
    full = o.forward(x0)                       # prefill of s + 1 = 6 tokens
    L, H, d, h = cfg.depth, cfg.n_heads, cfg.head_dim, cfg.hidden
    s = 5
    cap = 8
    kc = np.zeros((L, H, cap, d))
    vc = np.zeros((L, H, cap, d))
    for l in range(L):
        kc[l, :, :s] = full["sa_k"][l, :s].reshape(s, H, d).transpose(1, 0, 2)
        vc[l, :, :s] = full["sa_v"][l, :s].reshape(s, H, d).transpose(1, 0, 2)
    dec = o.decode_seq(x0[s], kc, vc, s)
    assert np.allclose(dec["x_out"], full["x_out"][s], rtol=1e-12, atol=1e-12)
    assert np.array_equal(dec["idx"].reshape(L, -1), full["idx"][:, s])
    # the decode step wrote the new token's keys at slot s
    for l in range(L):
        assert np.allclose(kc[l, :, s], full["sa_k"][l, s].reshape(H, d), atol=1e-12)


def test_decode_empty_cache_single_depth_is_one_token_block():
    cfg = tiny_cfg(batch=1, seq=1, depth=1)
    W = rand_weights(cfg, seed=10)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=1)
    ref = o.forward(x0)["x_out"][0]
    kc = np.zeros((1, cfg.n_heads, 4, cfg.head_dim))
    vc = np.zeros_like(kc)
    dec = o.decode_seq(x0[0], kc, vc, 0)
    assert np.allclose(dec["x_out"], ref, rtol=1e-13, atol=1e-13)


def test_serial_layout_closed_form():
    """Serial DA -> SA -> EA at L = 1, s = 1, E = k: u = x^ + v_DA W_O^DA;
    v = u + v_SA(u) W_O^SA; x_1 = v + mixture(v)."""
    cfg = tiny_cfg(batch=2, seq=1, depth=1, n_experts=2, top_k=2, variant=1)
    W = rand_weights(cfg, seed=12)
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    h, dr = cfg.hidden, cfg.router_dim
    f = lambda a: np.asarray(a, np.float64)
    x = f(x0)
    xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
    Wq, Wo = f(W["w_qkv"][0]), f(W["w_o"][0])
    u = xh + (xh @ Wq[:, 5 * h:]) @ Wo[h:]
    v = u + (u @ Wq[:, 2 * h:3 * h]) @ Wo[:h]
    kE = np.stack([O.depth_rope(f(k), 0, 1) for k in W["k_E"]])
    z = (v @ f(W["w_qE"])) @ kE.T / np.sqrt(dr)
    s = 1 / (1 + np.exp(-z))
    w = s / s.sum(1, keepdims=True)
    out = v.copy()
    for e in range(2):
        a = v @ f(W["w1"][e])
        out += w[:, e:e + 1] * ((a / (1 + np.exp(-a))) @ f(W["w2"][e]))
    assert np.allclose(r["x_out"], out, rtol=1e-11, atol=1e-11)


def test_fully_parallel_layout_routes_normed_state():
    """Fully parallel DA + SA + EA: with W_O = 0 the output is x^ + mixture(x^)."""
    cfg = tiny_cfg(batch=1, seq=3, depth=1, n_experts=4, top_k=4, variant=2)
    W = rand_weights(cfg, seed=13)
    W["w_o"] = np.zeros_like(W["w_o"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    f = lambda a: np.asarray(a, np.float64)
    x = f(x0)
    xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
    kE = np.stack([O.depth_rope(f(k), 0, 1) for k in W["k_E"]])
    z = (xh @ f(W["w_qE"])) @ kE.T / np.sqrt(cfg.router_dim)
    s = 1 / (1 + np.exp(-z))
    w = s / s.sum(1, keepdims=True)
    out = xh.copy()
    for e in range(4):
        a = xh @ f(W["w1"][e])
        out += w[:, e:e + 1] * ((a / (1 + np.exp(-a))) @ f(W["w2"][e]))
    assert np.allclose(r["x_out"], out, rtol=1e-11, atol=1e-11)


def test_route_entry_matches_forward_trace():
    cfg = configs.TINY
    W = inputs.host_weights(cfg)
    o = O.Oracle(cfg, W, threads=1)
    full = o.forward(inputs.host_inputs(cfg)["x0"])
    y1 = full["y"][1].astype(np.float32)
    r = o.route(1, y1)
    # routing from the float32-rounded y picks the same experts except at near ties
    same = np.all(np.sort(r["idx"], 1) == np.sort(full["idx"][1], 1), axis=1)
    assert np.all(same | (full["margin"][1] < 1e-5))


def test_route_on_bf16_input_changes_only_near_ties():
    """Taking the routing decision on the bf16-rounded state moves a selection only where
    the float64 margin is below the effect of that rounding."""
    cfg = configs.SMALL.with_(batch=1, seq=64, depth=2)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    a = O.Oracle(cfg, W, threads=2, route_bf16=False).forward(x0, 0, 1)
    b = O.Oracle(cfg, W, threads=2, route_bf16=True).forward(x0, 0, 1)
    assert np.array_equal(a["y"], b["y"])                      # states are untouched
    same = np.all(np.sort(a["idx"][0], 1) == np.sort(b["idx"][0], 1), axis=1)
    assert np.all(same | (a["margin"][0] < 0.05))


# ---------------------------------------------------------------------------------------
# Sliding-window depth attention and the layout without DA (the pages' comparison arms and
# sparse-DA outlook): window W reads depths max(0, l-W+1)..l; variant 3 has no DA at all.

def test_window_covering_all_depths_is_full_da():
    cfg = tiny_cfg(depth=4)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    full = O.Oracle(cfg, W, threads=2).forward(x0)
    for win in (4, 9):
        r = O.Oracle(cfg.with_(da_window=win), W, threads=2).forward(x0)
        assert np.array_equal(r["x_out"], full["x_out"])
    short = O.Oracle(cfg.with_(da_window=2), W, threads=2).forward(x0)
    assert not np.allclose(short["x_out"], full["x_out"])  # depths 2, 3 lose history


def test_window_one_returns_the_depths_own_value_closed_form():
    # W = 1: softmax over one depth is 1, so DA = v_DA(x^_l) at every depth.  SA rows of
    # W_O zero, DA rows identity, experts off: x_{l+1} = x^_l + x^_l W_v, iterated.
    cfg = tiny_cfg(depth=3, n_experts=2, top_k=1, da_window=1)
    W = rand_weights(cfg, seed=5)
    h = cfg.hidden
    W["w_o"] = np.zeros_like(W["w_o"])
    W["w_o"][0, h:, :] = np.eye(h, dtype=np.float32)
    W["w2"] = np.zeros_like(W["w2"])
    x0 = inputs.host_inputs(cfg)["x0"]
    r = O.Oracle(cfg, W, threads=1).forward(x0)
    x = x0.astype(np.float64)
    wv = W["w_qkv"][0][:, 5 * h:6 * h].astype(np.float64)
    for _ in range(cfg.depth):
        xh = x / np.sqrt(np.mean(x ** 2, 1, keepdims=True) + cfg.rms_eps)
        x = xh + xh @ wv
    assert np.allclose(r["x_out"], x, rtol=1e-12, atol=1e-12)


def test_window_ignores_depths_before_it():
    # one step at depth 3 with W = 2 reads the history rows of depths 2 (and its own 3)
    cfg = tiny_cfg(batch=1, seq=6, depth=5, da_window=2)
    W = rand_weights(cfg, seed=9)
    x = inputs.extra_normal(cfg, 1101, (cfg.seq, cfg.hidden), 1.0, dtype="fp32")
    hist = inputs.extra_normal(cfg, 1102, (2, cfg.depth, 2, cfg.hidden), 1.0, dtype="fp32")
    hist = hist.astype(np.float64)
    pos = np.array([1, 5], np.int32)
    o = O.Oracle(cfg, W, threads=1)
    base = o.step_tokens(3, x, hist, pos)["x_out"]
    h2 = hist.copy()
    h2[:, 0:2] += 3.0                                   # depths 0, 1: outside the window
    assert np.array_equal(o.step_tokens(3, x, h2, pos)["x_out"], base)
    h3 = hist.copy()
    h3[:, 2] += 3.0                                     # depth 2: inside
    assert not np.allclose(o.step_tokens(3, x, h3, pos)["x_out"], base)
    full = O.Oracle(cfg.with_(da_window=0), W, threads=1)
    assert not np.allclose(full.step_tokens(3, x, h2, pos)["x_out"],
                           full.step_tokens(3, x, hist, pos)["x_out"])


def test_window_reshape_equals_explicit_loops():
    cfg = tiny_cfg(depth=4, da_window=2)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    o = O.Oracle(cfg, W, threads=2)
    a, b = o.forward(x0), o.forward(x0, da_loops=True)
    assert np.allclose(a["x_out"], b["x_out"], rtol=1e-12, atol=1e-12)


def _zero_da_rows(cfg, W):
    W2 = dict(W)
    W2["w_o"] = W["w_o"].copy()
    W2["w_o"][:, cfg.hidden:, :] = 0.0
    return W2


def test_no_da_layout_equals_zeroed_da_rows():
    # without DA, y = x^ + SA W_O[SA rows]: the same as the default layout whose W_O rows
    # for a_DA are zero (adding exact zeros), in forward, one-step and decode form
    cfg = tiny_cfg(depth=3)
    W = inputs.host_weights(cfg)
    x0 = inputs.host_inputs(cfg)["x0"]
    nda = O.Oracle(cfg.with_(variant=3), W, threads=2)
    ref = O.Oracle(cfg, _zero_da_rows(cfg, W), threads=2)
    a, b = nda.forward(x0), ref.forward(x0)
    assert np.array_equal(a["x_out"], b["x_out"]) and np.array_equal(a["idx"], b["idx"])
    full = O.Oracle(cfg, W, threads=2).forward(x0)
    assert not np.allclose(a["x_out"], full["x_out"])
    dc = configs.TINY.with_(batch=1, seq=1, cache_len=8, depth=3)
    Wd = inputs.host_weights(dc)
    H, d = dc.n_heads, dc.head_dim
    kc = RNG.standard_normal((dc.depth, H, 9, d))
    vc = RNG.standard_normal((dc.depth, H, 9, d))
    xn = inputs.host_inputs(dc)["x0"][0]
    r1 = O.Oracle(dc.with_(variant=3), Wd, threads=1).decode_seq(xn, kc.copy(), vc.copy(), 5)
    r2 = O.Oracle(dc, _zero_da_rows(dc, Wd), threads=1).decode_seq(xn, kc.copy(), vc.copy(), 5)
    assert np.array_equal(r1["x_out"], r2["x_out"])


# ---------------------------------------------------------------------------------------
# Balance summary of the route counts (f2): Gini and Lorenz

def test_gini_lorenz_closed_forms():
    g, lor = O.gini_lorenz(np.full(16, 7))
    assert g == 0.0 and np.allclose(lor, np.arange(17) / 16)        # perfect equality
    one = np.zeros(16)
    one[5] = 40
    g, lor = O.gini_lorenz(one)
    assert g == pytest.approx(1 - 1 / 16) and lor[15] == 0 and lor[16] == 1   # one expert
    g, lor = O.gini_lorenz([1, 3])                                   # |1-3|*2 / (2*4*2)
    assert g == pytest.approx(0.25) and np.allclose(lor, [0, 0.25, 1])
    g, _ = O.gini_lorenz(np.zeros(8))
    assert g == 0.0


def test_gini_equals_one_minus_twice_lorenz_area():
    # the pairwise definition and the area under the Lorenz curve agree (trapezoid rule on
    # the piecewise-linear curve is exact)
    for n in (5, 64, 300):
        x = RNG.integers(0, 50, n)
        g, lor = O.gini_lorenz(x)
        area = np.sum((lor[1:] + lor[:-1]) / 2) / n
        assert g == pytest.approx(1 - 2 * area, abs=1e-12)
        assert np.all(np.diff(lor) >= 0) and np.all(np.diff(lor, 2) >= -1e-15)  # convex
