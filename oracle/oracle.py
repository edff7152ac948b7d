"""ctypes binding of the CPU oracle (oracle/dreamer_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
CPU-baseline / reference leg.  The product library never imports this module.
"""
from __future__ import annotations

import ctypes as C
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)
import build as _build  # noqa: E402

_lib = None

f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")


class OrcCfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("B", "S", "h", "H", "d", "L", "E", "k", "m", "dr", "P")] + \
               [("rope_base", C.c_double), ("eps", C.c_double), ("variant", C.c_int),
                ("route_bf16", C.c_int), ("da_window", C.c_int)]


_WNAMES = ("g", "w_qkv", "w_qkv_sh", "w_o", "w_o_sh", "w_qP", "k_P", "w_qE", "k_E", "bias",
           "w1", "w2")


class OrcWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _WNAMES]


_TNAMES = ("xhat", "y", "idx", "w", "margin", "zsel", "counts", "sa_k", "sa_v", "pidx",
           "psig", "pmargin")


class OrcTrace(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in _TNAMES]


def lib():
    global _lib
    if _lib is None:
        L = C.CDLL(_build.build())
        L.orc_set_threads.argtypes = [C.c_int]
        vp = C.c_void_p
        L.orc_forward.argtypes = [vp, vp, f32p, C.c_int, C.c_int, f64p, f64p, vp]
        L.orc_forward_da_loops.argtypes = L.orc_forward.argtypes
        L.orc_step_tokens.argtypes = [vp, vp, C.c_int, f32p, C.c_int, f64p, i32p, C.c_int,
                                      f64p, vp]
        L.orc_decode_seq.argtypes = [vp, vp, f32p, f64p, f64p, C.c_int, C.c_int, f64p, vp]
        L.orc_route.argtypes = [vp, vp, C.c_int, f32p, C.c_int, i32p, f64p, vp, vp, vp]
        L.orc_proj_route.argtypes = [vp, vp, C.c_int, f32p, C.c_int, i32p, f64p, vp]
        L.orc_rmsnorm.argtypes = [C.c_int, f64p, f32p, C.c_double, f64p]
        L.orc_rope.argtypes = [f64p, C.c_int, C.c_double, C.c_double]
        L.orc_depth_rope.argtypes = [f64p, C.c_int, C.c_int, C.c_int, C.c_double]
        L.orc_attend.argtypes = [f64p, f64p, f64p, C.c_int, C.c_int, C.c_long, f64p, f64p]
        L.orc_topk.argtypes = [f64p, f32p, C.c_int, C.c_int, i32p, f64p, vp]
        L.orc_linear_moe.argtypes = [C.c_int, C.c_int, f64p, f32p, f32p, C.c_double, f64p]
        L.orc_linear_moe_absorbed.argtypes = L.orc_linear_moe.argtypes
        L.orc_expert.argtypes = [C.c_int, C.c_int, f64p, f32p, f32p, f64p]
        L.orc_bias_update.argtypes = [C.c_int, C.c_int, i32p, C.c_double, f64p]
        for f in ("orc_forward", "orc_forward_da_loops", "orc_step_tokens", "orc_decode_seq",
                  "orc_route", "orc_proj_route"):
            getattr(L, f).restype = C.c_int
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32)


class Oracle:
    """The oracle bound to one configuration and one weight set (float32 arrays holding
    exact bf16/fp32 values)."""

    def __init__(self, cfg, weights: dict, threads: int | None = None,
                 route_bf16: bool | None = None):
        """route_bf16 (default: the config is bf16) makes routing decisions read their input
        rounded to bf16, as the bf16 kernels store it."""
        self.cfg = cfg
        rb = (cfg.dtype == "bf16") if route_bf16 is None else route_bf16
        self.c = OrcCfg(cfg.batch, cfg.seq, cfg.hidden, cfg.n_heads, cfg.head_dim, cfg.depth,
                        cfg.n_experts, cfg.top_k, cfg.expert_hidden, cfg.router_dim,
                        cfg.n_proj_experts, float(cfg.rope_base), float(cfg.rms_eps),
                        int(cfg.variant), int(rb), int(getattr(cfg, "da_window", 0)))
        self._keep = {}
        ptrs = {}
        alias = {"w_qkv_sh": "w_qkv_shared", "w_o_sh": "w_o_shared"}
        for n in _WNAMES:
            src = weights.get(alias.get(n, n))
            if src is None:
                ptrs[n] = None
                continue
            a = _f32(src)
            self._keep[n] = a
            ptrs[n] = a.ctypes.data
        self.W = OrcWeights(**ptrs)
        set_threads(threads if threads is not None else (os.cpu_count() or 1))

    # -- trace helpers -------------------------------------------------------------------
    def _trace(self, rows: int, want: bool):
        if not want:
            return None, {}
        cfg = self.cfg
        h, k, E = cfg.hidden, cfg.top_k, cfg.n_experts
        bufs = dict(
            xhat=np.zeros((rows, h)), y=np.zeros((rows, h)),
            idx=np.zeros((rows, k), np.int32), w=np.zeros((rows, k)),
            margin=np.zeros(rows), zsel=np.zeros((rows, k + 1)),
            pidx=np.zeros(rows, np.int32), psig=np.zeros(rows), pmargin=np.zeros(rows),
            sa_k=np.zeros((rows, h)), sa_v=np.zeros((rows, h)))
        return bufs, E

    @staticmethod
    def _trace_struct(bufs, counts):
        ptr = {n: (bufs[n].ctypes.data if n in bufs else None) for n in _TNAMES if n != "counts"}
        ptr["counts"] = counts.ctypes.data if counts is not None else None
        return OrcTrace(**ptr)

    # -- entry points --------------------------------------------------------------------
    def forward(self, x_in, l0: int = 0, l1: int | None = None, da_kv=None,
                trace: bool = True, da_loops: bool = False) -> dict:
        cfg = self.cfg
        T, h, L, k = cfg.tokens, cfg.hidden, cfg.depth, cfg.top_k
        l1 = L if l1 is None else l1
        da = np.zeros((T, L, 2, h)) if da_kv is None else np.ascontiguousarray(da_kv, np.float64)
        x_out = np.zeros((T, h))
        bufs, E = self._trace(L * T, trace)
        counts = np.zeros((L, cfg.n_experts), np.int32)
        tr = self._trace_struct(bufs, counts) if trace else None
        fn = lib().orc_forward_da_loops if da_loops else lib().orc_forward
        rc = fn(C.byref(self.c), C.byref(self.W), _f32(x_in).reshape(T, h), l0, l1, da, x_out,
                C.byref(tr) if tr is not None else None)
        if rc != 0:
            raise RuntimeError(f"orc_forward failed: {rc}")
        out = dict(x_out=x_out, da_kv=da, counts=counts)
        if trace:
            for n, b in bufs.items():
                out[n] = b.reshape((L, T) + b.shape[1:])
        return out

    def step_tokens(self, l: int, x_seq, da_hist, pos) -> dict:
        cfg = self.cfg
        h, L, k = cfg.hidden, cfg.depth, cfg.top_k
        x_seq = _f32(x_seq)
        n_ctx = x_seq.shape[0]
        pos = np.ascontiguousarray(pos, np.int32)
        n_s = len(pos)
        da_hist = np.ascontiguousarray(da_hist, np.float64).reshape(n_s, L, 2, h)
        x_out = np.zeros((n_s, h))
        bufs, _ = self._trace(n_s, True)
        counts = np.zeros(cfg.n_experts, np.int32)
        tr = self._trace_struct(bufs, counts)
        rc = lib().orc_step_tokens(C.byref(self.c), C.byref(self.W), l, x_seq, n_ctx, da_hist,
                                   pos, n_s, x_out, C.byref(tr))
        if rc != 0:
            raise RuntimeError(f"orc_step_tokens failed: {rc}")
        return dict(x_out=x_out, counts=counts, **bufs)

    def decode_seq(self, x_new, kc, vc, length: int) -> dict:
        """kc, vc: [L][H][cap][d] (float64, updated in place)."""
        cfg = self.cfg
        h, L = cfg.hidden, cfg.depth
        cap = kc.shape[2]
        x_out = np.zeros(h)
        bufs, _ = self._trace(L, True)
        counts = np.zeros((L, cfg.n_experts), np.int32)
        tr = self._trace_struct(bufs, counts)
        rc = lib().orc_decode_seq(C.byref(self.c), C.byref(self.W), _f32(x_new).reshape(h), kc,
                                  vc, cap, int(length), x_out, C.byref(tr))
        if rc != 0:
            raise RuntimeError(f"orc_decode_seq failed: {rc}")
        return dict(x_out=x_out, counts=counts, **bufs)

    def route(self, l: int, y, want_zsel: bool = True) -> dict:
        cfg = self.cfg
        y = _f32(y)
        T = y.shape[0]
        k = cfg.top_k
        idx = np.zeros((T, k), np.int32)
        w = np.zeros((T, k))
        margin = np.zeros(T)
        zsel = np.zeros((T, k + 1))
        counts = np.zeros(cfg.n_experts, np.int32)
        rc = lib().orc_route(C.byref(self.c), C.byref(self.W), l, y, T, idx, w,
                             margin.ctypes.data, zsel.ctypes.data if want_zsel else None,
                             counts.ctypes.data)
        if rc != 0:
            raise RuntimeError(f"orc_route failed: {rc}")
        return dict(idx=idx, w=w, margin=margin, zsel=zsel, counts=counts)

    def proj_route(self, l: int, xh) -> dict:
        """Projection router alone on normalised states x^ [T][h] at depth l (P > 0)."""
        xh = _f32(xh)
        T = xh.shape[0]
        pidx = np.zeros(T, np.int32)
        psig = np.zeros(T)
        pmargin = np.zeros(T)
        rc = lib().orc_proj_route(C.byref(self.c), C.byref(self.W), l, xh, T, pidx, psig,
                                  pmargin.ctypes.data)
        if rc != 0:
            raise RuntimeError(f"orc_proj_route failed: {rc}")
        return dict(pidx=pidx, psig=psig, pmargin=pmargin)


# -- building blocks (for the pins) ------------------------------------------------------
def rmsnorm(x, g, eps):
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros_like(x)
    lib().orc_rmsnorm(x.size, x, _f32(g), float(eps), out)
    return out


def rope(v, pos, base=10000.0):
    v = np.array(v, np.float64)
    lib().orc_rope(v, v.size, float(pos), float(base))
    return v


def depth_rope(v, l, L, base=10000.0):
    v = np.array(v, np.float64)
    lib().orc_depth_rope(v, v.size, int(l), int(L), float(base))
    return v


def attend(q, K, V):
    q = np.ascontiguousarray(q, np.float64)
    K = np.ascontiguousarray(K, np.float64)
    V = np.ascontiguousarray(V, np.float64)
    nk, d = K.shape
    out = np.zeros(d)
    probs = np.zeros(max(nk, 1))
    lib().orc_attend(q, K, V, nk, d, d, out, probs)
    return out, probs[:nk]


def topk(z, bias, k):
    z = np.ascontiguousarray(z, np.float64)
    E = z.size
    idx = np.zeros(k, np.int32)
    w = np.zeros(k)
    margin = np.zeros(1)
    lib().orc_topk(z, _f32(bias), E, k, idx, w, margin.ctypes.data)
    return idx, w, float(margin[0])


def linear_moe(x, Wp, Wsh, sigma, absorbed=False):
    x = np.ascontiguousarray(x, np.float64)
    Wp = _f32(Wp)
    n_in, n_out = Wp.shape
    y = np.zeros(n_out)
    fn = lib().orc_linear_moe_absorbed if absorbed else lib().orc_linear_moe
    fn(n_in, n_out, x, Wp, _f32(Wsh), float(sigma), y)
    return y


def expert(y, w1e, w2e):
    y = np.ascontiguousarray(y, np.float64)
    w1e = _f32(w1e)
    h, m = w1e.shape
    out = np.zeros(h)
    lib().orc_expert(h, m, y, w1e, _f32(w2e), out)
    return out


def bias_update(counts, lam, bias):
    counts = np.ascontiguousarray(counts, np.int32)
    L, E = counts.shape
    b = np.array(bias, np.float64)
    lib().orc_bias_update(L, E, counts, float(lam), b)
    return b


def gini_lorenz(counts):
    """Balance of expert use (papernotes "Key design 2": the bias keeps experts balanced):
    Lorenz curve of the per-expert counts (sorted ascending, cumulative share at e/E for
    e = 0..E) and the Gini coefficient by its definition, the mean absolute difference over
    all pairs divided by twice the mean.  All-zero counts: the diagonal and 0."""
    x = np.sort(np.asarray(counts, np.float64).ravel())
    E = x.size
    tot = x.sum()
    if tot <= 0:
        return 0.0, np.arange(E + 1) / E
    lorenz = np.concatenate([[0.0], np.cumsum(x) / tot])
    g = np.abs(x[:, None] - x[None, :]).sum() / (2.0 * E * E * (tot / E))
    return float(g), lorenz
