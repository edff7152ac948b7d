"""Python binding of libdreamer (include/dreamer.h): argument marshalling only.

Every step of the depth-recurrent forward runs in the library's CUDA kernels; PyTorch only
supplies device memory and streams.  If libdreamer.so is missing this module raises: there is
no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

from .configs import DreamerConfig

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdreamer.so")
# test infrastructure only: the same sources with the timeout-test hook (dreamer_test_inject)
# and a 20 ms device wait limit
TESTHOOKS_PATH = os.path.join(_HERE, "libdreamer_testhooks.so")
_libs = {}

OK = 0
ERR_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_OOM, ERR_TIMEOUT, ERR_STATE = -1, -2, -3, -4, -5, -6


class DreamerError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {lib().dreamer_strerror(code).decode()} ({code})")
        self.code = code


class ConfigC(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "batch", "seq", "hidden", "n_heads", "head_dim", "depth", "n_experts", "top_k",
        "expert_hidden", "router_dim", "n_proj_experts", "dtype")] + \
        [("rope_base", C.c_float), ("rms_eps", C.c_float), ("max_cache_len", C.c_int),
         ("variant", C.c_int), ("da_window", C.c_int)]


WEIGHT_FIELDS = ("rms_gain", "w_qkv", "w_qkv_shared", "w_o", "w_o_shared", "w_qP", "k_P",
                 "w_qE", "k_E", "bias_E", "w1", "w2")
# names used by inputs.weight_specs for the same tensors
WEIGHT_SOURCE = dict(rms_gain="g", bias_E="bias")


class WeightsC(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in WEIGHT_FIELDS]


STAGES = ("norm", "proj_route", "qkv", "da", "sa", "o_proj", "ea_route", "permute",
          "experts", "finish")


class StatsC(C.Structure):
    _fields_ = [("launches", C.c_uint64), ("ms", C.c_double * len(STAGES)),
                ("count", C.c_uint64 * len(STAGES)), ("launches_tc", C.c_uint64),
                ("launches_simt", C.c_uint64)]


TRACE_FIELDS = ("xhat", "y", "idx", "w", "sa_k", "sa_v", "pidx", "psig", "y_f32", "x_f32")


class TraceC(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in TRACE_FIELDS]


def lib(path: str = LIB_PATH):
    if path not in _libs:
        if not os.path.exists(path):
            raise RuntimeError(f"{path} not built: run __graft_entry__.build()")
        L = C.CDLL(path)
        vp, i = C.c_void_p, C.c_int
        L.dreamer_init.argtypes = [C.POINTER(ConfigC), C.POINTER(WeightsC), vp, C.POINTER(vp)]
        L.dreamer_core_forward.argtypes = [vp, vp, vp, i, i, vp, vp, vp]
        L.dreamer_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
        L.dreamer_route_counts.argtypes = [vp, vp, i, vp]
        L.dreamer_route_experts.argtypes = [vp, i, vp, i, vp, vp, vp, vp]
        L.dreamer_bias_update.argtypes = [vp, C.c_float, vp, vp]
        L.dreamer_bias_update_counts.argtypes = [vp, C.c_float, vp, i, vp, vp]
        L.dreamer_route_balance.argtypes = [vp, i, vp, vp, vp]
        L.dreamer_set_profiling.argtypes = [vp, i]
        L.dreamer_get_stats.argtypes = [vp, C.POINTER(StatsC), i]
        L.dreamer_destroy.argtypes = [vp]
        L.dreamer_destroy.restype = None
        L.dreamer_strerror.argtypes = [i]
        L.dreamer_strerror.restype = C.c_char_p
        for f in ("dreamer_init", "dreamer_core_forward", "dreamer_decode_step",
                  "dreamer_route_counts", "dreamer_route_experts", "dreamer_bias_update",
                  "dreamer_bias_update_counts", "dreamer_route_balance",
                  "dreamer_set_profiling", "dreamer_get_stats"):
            getattr(L, f).restype = i
        if hasattr(L, "dreamer_test_inject"):
            L.dreamer_test_inject.argtypes = [vp, i]
            L.dreamer_test_inject.restype = i
        _libs[path] = L
    return _libs[path]


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _check(rc, what):
    if rc != OK:
        raise DreamerError(rc, what)


def torch_dtype(cfg: DreamerConfig):
    return torch.float32 if cfg.dtype == "fp32" else torch.bfloat16


def config_c(cfg: DreamerConfig) -> ConfigC:
    return ConfigC(cfg.batch, cfg.seq, cfg.hidden, cfg.n_heads, cfg.head_dim, cfg.depth,
                   cfg.n_experts, cfg.top_k, cfg.expert_hidden, cfg.router_dim,
                   cfg.n_proj_experts, 0 if cfg.dtype == "fp32" else 1, cfg.rope_base,
                   cfg.rms_eps, (cfg.cache_len + 1) if cfg.is_decode else 0, cfg.variant,
                   cfg.da_window)


class Dreamer:
    """A libdreamer handle for one configuration and weight set.

    weights: dict of device tensors named as in inputs.weight_specs (g, w_qkv, w_o, w_qE,
    k_E, bias, w1, w2 and, with projection experts, w_qkv_shared, w_o_shared, w_qP, k_P).
    """

    def __init__(self, cfg: DreamerConfig, weights: dict, stream=None, max_cache_len=None,
                 lib_path: str = LIB_PATH):
        self.cfg = cfg
        self.L = lib(lib_path)
        self.cc = config_c(cfg)
        if max_cache_len is not None:
            self.cc.max_cache_len = int(max_cache_len)
        ptrs = {}
        for f in WEIGHT_FIELDS:
            src = WEIGHT_SOURCE.get(f, f)
            t = weights.get(src)
            ptrs[f] = _ptr(t) if t is not None else None
        self.wc = WeightsC(**ptrs)
        self.h = C.c_void_p()
        _check(self.L.dreamer_init(C.byref(self.cc), C.byref(self.wc), _stream(stream),
                                  C.byref(self.h)), "dreamer_init")

    def close(self):
        if self.h:
            self.L.dreamer_destroy(self.h)
            self.h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @staticmethod
    def _trace(trace: dict | None):
        if not trace:
            return None
        return TraceC(**{f: _ptr(trace.get(f)) for f in TRACE_FIELDS})

    def forward(self, x_in, x_out=None, depth_begin=0, depth_end=None, da_kv=None,
                trace: dict | None = None, stream=None):
        cfg = self.cfg
        depth_end = cfg.depth if depth_end is None else depth_end
        if x_out is None:
            x_out = torch.empty_like(x_in)
        tr = self._trace(trace)
        _check(self.L.dreamer_core_forward(self.h, _ptr(x_in), _ptr(x_out), int(depth_begin),
                                          int(depth_end), _ptr(da_kv),
                                          C.byref(tr) if tr is not None else None,
                                          _stream(stream)), "dreamer_core_forward")
        return x_out

    def decode_step(self, x_new, k_cache, v_cache, cache_len, x_out=None,
                    trace: dict | None = None, stream=None):
        if x_out is None:
            x_out = torch.empty_like(x_new)
        tr = self._trace(trace)
        _check(self.L.dreamer_decode_step(self.h, _ptr(x_new), _ptr(k_cache), _ptr(v_cache),
                                         _ptr(cache_len), _ptr(x_out),
                                         C.byref(tr) if tr is not None else None,
                                         _stream(stream)), "dreamer_decode_step")
        return x_out

    def route_balance(self, depth: int = -1, stream=None):
        """(Gini coefficient, Lorenz curve [E+1]) of the last call's route counts (depth < 0:
        summed over depths), as device tensors."""
        lor = torch.empty(self.cfg.n_experts + 1, dtype=torch.float32, device="cuda")
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        _check(self.L.dreamer_route_balance(self.h, int(depth), _ptr(lor), _ptr(g),
                                           _stream(stream)), "dreamer_route_balance")
        return g, lor

    def route_counts(self, on_host: bool = True, stream=None):
        cfg = self.cfg
        if on_host:
            out = torch.zeros((cfg.depth, cfg.n_experts), dtype=torch.int32)
            _check(self.L.dreamer_route_counts(self.h, C.c_void_p(out.data_ptr()), 1,
                                              _stream(stream)), "dreamer_route_counts")
            return out
        out = torch.zeros((cfg.depth, cfg.n_experts), dtype=torch.int32, device="cuda")
        _check(self.L.dreamer_route_counts(self.h, _ptr(out), 0, _stream(stream)),
               "dreamer_route_counts")
        return out

    def route_experts(self, depth: int, y, stream=None):
        cfg = self.cfg
        n = y.shape[0]
        idx = torch.empty((n, cfg.top_k), dtype=torch.int32, device=y.device)
        w = torch.empty((n, cfg.top_k), dtype=torch.float32, device=y.device)
        counts = torch.empty(cfg.n_experts, dtype=torch.int32, device=y.device)
        _check(self.L.dreamer_route_experts(self.h, int(depth), _ptr(y), int(n), _ptr(idx),
                                           _ptr(w), _ptr(counts), _stream(stream)),
               "dreamer_route_experts")
        return idx, w, counts

    def bias_update(self, lam: float, counts=None, stream=None):
        """b_e += lam * sign(median(N) - N_e) on the handle's bias; returns the new bias.
        N = the last call's route counts summed over depths, or, when `counts` is given (a
        CUDA int32 tensor [R][E] or [E], e.g. the counts of all replicas from
        allreduce_route_counts), those summed over their rows."""
        out = torch.empty(self.cfg.n_experts, dtype=torch.float32, device="cuda")
        if counts is None:
            _check(self.L.dreamer_bias_update(self.h, float(lam), _ptr(out), _stream(stream)),
                   "dreamer_bias_update")
            return out
        c = counts.reshape(-1, self.cfg.n_experts)
        if c.dtype != torch.int32 or not c.is_cuda or not c.is_contiguous():
            raise ValueError("counts: a contiguous CUDA int32 tensor [R][E] or [E]")
        _check(self.L.dreamer_bias_update_counts(self.h, float(lam), _ptr(c), int(c.shape[0]),
                                                _ptr(out), _stream(stream)),
               "dreamer_bias_update_counts")
        return out

    def set_profiling(self, enable: bool):
        _check(self.L.dreamer_set_profiling(self.h, int(bool(enable))), "dreamer_set_profiling")

    def test_inject(self, what: int):
        """Test-hook library only: what = 1 makes the next call's first QKV GEMM load no
        operands, so that its bounded wait expires (DREAMER_ERR_TIMEOUT)."""
        _check(self.L.dreamer_test_inject(self.h, int(what)), "dreamer_test_inject")

    def stats(self, reset: bool = True) -> dict:
        st = StatsC()
        _check(self.L.dreamer_get_stats(self.h, C.byref(st), int(bool(reset))), "dreamer_get_stats")
        return dict(launches=int(st.launches), launches_tc=int(st.launches_tc),
                    launches_simt=int(st.launches_simt),
                    ms={n: float(st.ms[i]) for i, n in enumerate(STAGES)},
                    count={n: int(st.count[i]) for i, n in enumerate(STAGES)})


def allreduce_route_counts(counts, group=None):
    """Sum route counts ([L][E] int32, from Dreamer.route_counts) over the ranks of `group` in
    place and return them: the one exchange of data-parallel replicas, after which every
    replica's bias update (Dreamer.bias_update(lam, counts=...)) sees the global expert use.
    NCCL for CUDA tensors (NVLink), gloo for CPU ones; a no-op without a process group of
    more than one rank."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    return counts


class LayeredStack:
    """The layered (LA) comparison arm: L distinct layers, each the Dreamer block without depth
    attention (SA, then expert attention), layer l with its own weights.  Built from one
    handle per layer (configuration `variant` 3); layer l runs depth l of its handle, so the
    expert keys take the depth-RoPE of their layer index and each handle counts its own row
    of the route histogram.  weights: a list of L device weight dicts."""

    def __init__(self, cfg: DreamerConfig, weights: list, stream=None):
        if cfg.variant != 3:
            raise ValueError("the layered arm has no depth attention: use variant 3")
        if len(weights) != cfg.depth:
            raise ValueError("one weight set per layer")
        self.cfg = cfg
        self.layers = [Dreamer(cfg, w, stream=stream) for w in weights]
        self._tmp = None

    def forward(self, x_in, x_out=None, stream=None):
        x = x_in
        if self._tmp is None or self._tmp[0].shape != x_in.shape or self._tmp[0].dtype != x_in.dtype:
            self._tmp = (torch.empty_like(x_in), torch.empty_like(x_in))
        if x_out is None:
            x_out = torch.empty_like(x_in)
        L = self.cfg.depth
        for l, layer in enumerate(self.layers):
            dst = x_out if l == L - 1 else self._tmp[l % 2]
            layer.forward(x, x_out=dst, depth_begin=l, depth_end=l + 1, stream=stream)
            x = dst
        return x_out

    def close(self):
        for layer in self.layers:
            layer.close()
        self.layers = []
