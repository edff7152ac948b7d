"""Helpers of the GPU-vs-oracle parity tests.

Tolerances (the stated bounds of the Dreamer core-forward contract):
  * float32 mode: hidden states max-abs <= 1e-4; expert indices bit-exact except where the
    oracle's k-th and (k+1)-th biased scores lie within 1e-5 (counted, reported).
  * bfloat16 mode: hidden states max-abs <= 3e-2 and relative L2 <= 1e-2.
  * route counts exact.

How the bf16 bounds are applied.  The residual stream is carried in float32 inside a call;
the states y_l and x_{l+1} leave it rounded to bf16.  The library dumps both forms (trace
fields y_f32 / x_f32 next to y and the call's output), so:
  * the float32 dump is held to max-abs 3e-2 and rel-L2 1e-2 against the oracle as it is,
    with no allowance for rounding;
  * the bf16 value must equal the float32 dump rounded to nearest even, bit for bit.
Values that exist only in bf16 (the DA key/value slots, SA cache slots) must be the bf16
rounding of some real within 3e-2 of the oracle: RN(ref - 3e-2) <= got <= RN(ref + 3e-2)
(RN is monotone, so this says the exact value before the store was within the bound).
Every check reports how many elements the final rounding alone puts beyond 3e-2.

Routing is gated on the device's own router inputs: the oracle routes the bf16 y (or x^)
the device dumped, and the device's picks must equal the oracle's except where the oracle's
k-th and (k+1)-th biased scores lie within 1e-5; counts exact.  The projection router (P > 0)
likewise on the device's x^.  Comparing x_{l+1} with the oracle's own forward, a token whose
selection differs from the forward's is excluded only where the forward's margin is below
what the difference between the two y's can move a score (Cauchy-Schwarz:
|dz_e| <= ||y_gpu - y_orc||_2 * ||W_qE k~_e||_2 / sqrt(d_r)).
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


def rn_bf16(x) -> np.ndarray:
    """float64 -> nearest bfloat16 value (ties to even), as float64; normal range only."""
    x = np.asarray(x, np.float64)
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    ulp = 2.0 ** (e - 7)
    return np.where(ax > 0, np.round(x / ulp) * ulp, 0.0)


def router_lipschitz(cfg, W, l, proj=False) -> float:
    """max_e ||W_q k~_e||_2 / sqrt(d_r) at depth l (expert router, or the projection router)."""
    wq = np.asarray(W["w_qP" if proj else "w_qE"], np.float64)
    keys = W["k_P" if proj else "k_E"]
    kr = np.stack([O.depth_rope(np.asarray(k, np.float64), l, cfg.depth, cfg.rope_base)
                   for k in keys])
    cols = wq @ kr.T                      # [h][E]
    return float(np.max(np.linalg.norm(cols, axis=0)) / np.sqrt(cfg.router_dim))


def same_sets(a, b) -> np.ndarray:
    return np.all(np.sort(a, axis=-1) == np.sort(b, axis=-1), axis=-1)


def check_routing(cfg, W, l, gpu_idx, orc_idx, orc_margin, gpu_y=None, orc_y=None,
                  strict=False):
    """Returns (same mask, n_flips).  strict (or no y given): mismatches only at near ties of
    1e-5; otherwise also where the y difference can move the scores across the margin
    (Cauchy-Schwarz).  Raises AssertionError on an unexplained mismatch."""
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


def gate_router_on_device_input(cfg, W, orc, l, gpu_ein, gpu_idx, gpu_w, gpu_counts=None,
                                what=""):
    """The oracle routes the device's own router input (bf16 y, or x^ in the fully parallel
    layout): picks equal except at near ties of 1e-5, weights (by expert) within 1e-5 where
    the sets agree, counts exact (the histogram of the device's picks, equal to the oracle's
    when nothing flipped).  Returns the number of near-tie flips."""
    ref = orc.route(l, gpu_ein)
    same, flips = check_routing(cfg, W, l, gpu_idx, ref["idx"], ref["margin"], strict=True)
    assert np.allclose(weights_by_expert(gpu_idx, gpu_w)[same],
                       weights_by_expert(ref["idx"], ref["w"])[same], atol=1e-5), what
    if gpu_counts is not None:
        hist = np.bincount(np.asarray(gpu_idx).ravel(), minlength=cfg.n_experts)
        assert np.array_equal(gpu_counts, hist), f"{what}: counts are not the picks' histogram"
        if flips == 0:
            assert np.array_equal(gpu_counts, ref["counts"]), f"{what}: counts differ"
    near = int((ref["margin"] <= NEAR_TIE).sum())
    print(f"  router {what} depth {l}: {flips} flips at {near} near ties (device input)")
    return flips


def gate_proj_router_on_device_input(cfg, orc, l, gpu_xhat, gpu_pidx, gpu_psig=None, what=""):
    """The projection router (P > 0) on the device's own x^: p* equal except at near ties of
    1e-5; sigma within 1e-5 where p* agrees."""
    ref = orc.proj_route(l, gpu_xhat)
    diff = gpu_pidx != ref["pidx"]
    bad = diff & (ref["pmargin"] > NEAR_TIE)
    assert not bad.any(), f"{what} depth {l}: {int(bad.sum())} projection routing mismatches"
    if gpu_psig is not None:
        assert np.allclose(gpu_psig[~diff], ref["psig"][~diff], atol=1e-5), what
    print(f"  projection router {what} depth {l}: {int(diff.sum())} near-tie flips")
    return ~diff


def proj_same_as_forward(cfg, W, l, gpu_pidx, orc_pidx, orc_pmargin, gpu_xhat, orc_xhat):
    """Tokens whose p* equals the oracle forward's; a difference must be explained by the x^
    difference (Cauchy-Schwarz, as for expert routing)."""
    same = gpu_pidx == orc_pidx
    dx = np.linalg.norm(gpu_xhat - orc_xhat, axis=-1)
    delta = 2.0 * dx * router_lipschitz(cfg, W, l, proj=True) + NEAR_TIE
    bad = (~same) & (orc_pmargin > delta)
    assert not bad.any(), f"depth {l}: {int(bad.sum())} projection flips not explained"
    return same


def check_hidden(got, ref, bf16: bool, what: str, f32=None):
    """Hidden states against the oracle.  float32 mode: max-abs 1e-4.  bf16 mode with the
    float32 dump `f32`: that dump within 3e-2 / rel-L2 1e-2 and `got` its exact rounding;
    without one: the interval rule for a value stored once in bf16 (module docstring)."""
    if got.size == 0:
        return 0.0, 0.0
    err = float(np.max(np.abs(got - ref)))
    if not bf16:
        assert err <= TOL_F32_ABS, f"{what}: max-abs {err:.3g} (<= {TOL_F32_ABS})"
        return err, 0.0
    n_round = int((np.abs(got - ref) > TOL_BF16_ABS).sum())
    if f32 is not None:
        e32 = float(np.max(np.abs(f32 - ref)))
        rl = rel_l2(f32, ref)
        assert e32 <= TOL_BF16_ABS and rl <= TOL_BF16_REL, \
            f"{what}: float32 state max-abs {e32:.3g} (<= {TOL_BF16_ABS}), rel-L2 {rl:.3g}"
        mism = int((rn_bf16(f32) != got).sum())
        assert mism == 0, f"{what}: {mism} stored bf16 values are not the rounding of the state"
        print(f"  {what}: max-abs {e32:.3g} rel-L2 {rl:.3g} (float32 state); "
              f"{n_round} stored elements beyond {TOL_BF16_ABS} by their rounding")
        return e32, rl
    rl = rel_l2(got, ref)
    lo, hi = rn_bf16(ref - TOL_BF16_ABS), rn_bf16(ref + TOL_BF16_ABS)
    out = (got < lo) | (got > hi)
    assert not out.any() and rl <= TOL_BF16_REL, \
        f"{what}: {int(out.sum())} stored values not the rounding of a value within " \
        f"{TOL_BF16_ABS} (max-abs {err:.3g}), rel-L2 {rl:.3g} (<= {TOL_BF16_REL})"
    if n_round:
        print(f"  {what}: {n_round} stored elements beyond {TOL_BF16_ABS} by their rounding")
    return err, rl


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


def check_drift(got, ref, what: str, gate_abs: bool, f32=None):
    """Free-running comparison: relative L2 gated; max-abs gated only where asked (the first
    depth, through check_hidden), otherwise reported."""
    if gate_abs:
        return check_hidden(got, ref, True, what, f32=f32)
    src = f32 if f32 is not None else got
    err = float(np.max(np.abs(src - ref))) if src.size else 0.0
    rl = rel_l2(src, ref) if src.size else 0.0
    assert rl <= TOL_BF16_REL, f"{what}: rel-L2 {rl:.3g} (<= {TOL_BF16_REL}); max-abs {err:.3g}"
    return err, rl


def weights_by_expert(idx, w) -> np.ndarray:
    """Routing weights reordered by expert index (the pick order of two nearly equal
    scores may differ between the two sides; the (expert, weight) pairs may not)."""
    o = np.argsort(idx, axis=-1)
    return np.take_along_axis(np.asarray(w, np.float64), o, axis=-1)
