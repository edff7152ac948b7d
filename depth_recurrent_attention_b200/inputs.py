"""Seeded synthetic inputs shared by the CUDA path's tests/bench and by the oracle.

This module holds no arithmetic of the Dreamer method.  It only draws numbers.

Generator (counter-based, so any slice of any tensor can be drawn on its own):
  * splitmix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014): output i of the stream keyed by K is mix(K + (i + 1) * 0x9E3779B97F4A7C15)
    with mix(z) = z ^= z >> 30, z *= 0xBF58476D1CE4E5B9, z ^= z >> 27,
    z *= 0x94D049BB133111EB, z ^= z >> 31 (all mod 2^64).
  * stream key of (seed, tensor_id): mix((seed << 32) ^ tensor_id ^ 0x243F6A8885A308D3).
  * uniform in (0, 1]: ((r >> 11) + 1) * 2^-53.
  * normal: Box-Muller (Box and Muller, 1958) on the pair (u1, u2) = (U(2j), U(2j + 1)):
    element 2j = sqrt(-2 ln u1) cos(2 pi u2), element 2j + 1 = sqrt(-2 ln u1) sin(2 pi u2),
    evaluated in float64, then scaled by std.
  * uniform(-a, a): a * (2 * ((r >> 11) * 2^-53) - 1).
  * rounding: float64 -> float32 (round to nearest even); bf16 = float32 rounded to nearest
    even at bit 16.

The same generator exists as a CUDA fill kernel (csrc/inputs_gen.cu, library
libdreamer_inputs.so) so that multi-GB tensors (the decode KV cache, large-config weights) can
be drawn directly in device memory.  Both follow the definitions above.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np

from .configs import DreamerConfig

GAMMA = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
MASK = (1 << 64) - 1

# tensor ids (one independent stream per tensor)
TID = dict(x0=1, g=2, w_qkv=3, w_qkv_shared=4, w_o=5, w_o_shared=6, w_qP=7, k_P=8, w_qE=9,
           k_E=10, bias=11, w1=12, w2=13, k_cache=14, v_cache=15, cache_len=16)
# ids >= 1000 are free for tests (step inputs, histories, perturbations)


def _mix_int(z: int) -> int:
    z &= MASK
    z = ((z ^ (z >> 30)) * M1) & MASK
    z = ((z ^ (z >> 27)) * M2) & MASK
    return z ^ (z >> 31)


def stream_key(seed: int, tensor_id: int) -> int:
    return _mix_int((seed << 32) ^ tensor_id ^ 0x243F6A8885A308D3)


def _raw(key: int, start: int, n: int) -> np.ndarray:
    """splitmix64 outputs start .. start+n-1 of stream `key` (uint64)."""
    with np.errstate(over="ignore"):
        i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        z = np.uint64(key) + i * np.uint64(GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(M2)
        return z ^ (z >> np.uint64(31))


def _u01_open0(r: np.ndarray) -> np.ndarray:
    return ((r >> np.uint64(11)) + np.uint64(1)).astype(np.float64) * (2.0 ** -53)


def normal(key: int, start: int, n: int, std: float = 1.0) -> np.ndarray:
    """float64 N(0, std^2) elements start .. start+n-1 of the stream."""
    if n <= 0:
        return np.zeros(0, np.float64)
    j0 = start // 2
    j1 = (start + n - 1) // 2 + 1
    r = _raw(key, 2 * j0, 2 * (j1 - j0))
    u1 = _u01_open0(r[0::2])
    u2 = _u01_open0(r[1::2])
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = 2.0 * np.pi * u2
    out = np.empty(2 * (j1 - j0), np.float64)
    out[0::2] = rad * np.cos(ang)
    out[1::2] = rad * np.sin(ang)
    off = start - 2 * j0
    return out[off:off + n] * std


def uniform(key: int, start: int, n: int, a: float) -> np.ndarray:
    r = _raw(key, start, n)
    u = (r >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
    return a * (2.0 * u - 1.0)


def to_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, np.float64).astype(np.float32)


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(x32, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """float64 -> values of `dtype` ("fp32" or "bf16"), returned as float32."""
    x32 = to_f32(x)
    if dtype == "fp32":
        return x32
    return bf16_bits_to_f32(f32_to_bf16_bits(x32))


@dataclass
class TensorSpec:
    name: str
    shape: tuple
    kind: str        # "normal", "uniform", "ones"
    param: float     # std or half-range
    dtype: str       # "fp32" or "bf16"
    tid: int

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= s
        return n


def weight_specs(cfg: DreamerConfig) -> list[TensorSpec]:
    """Shapes and distributions of every weight: W ~ N(0, 1/fan_in), keys ~ N(0, 1),
    gain 1, bias ~ U(-a, a) (fp32)."""
    h, dr, E, m, P = cfg.hidden, cfg.router_dim, cfg.n_experts, cfg.expert_hidden, cfg.n_proj_experts
    dt = cfg.dtype
    sh = 1.0 / np.sqrt(h)
    specs = [
        TensorSpec("g", (h,), "ones", 1.0, dt, TID["g"]),
        TensorSpec("w_qkv", (max(P, 1), h, 6 * h), "normal", sh, dt, TID["w_qkv"]),
        TensorSpec("w_o", (max(P, 1), 2 * h, h), "normal", sh, dt, TID["w_o"]),
        TensorSpec("w_qE", (h, dr), "normal", sh, dt, TID["w_qE"]),
        TensorSpec("k_E", (E, dr), "normal", 1.0, dt, TID["k_E"]),
        TensorSpec("bias", (E,), "uniform", cfg.bias_range, "fp32", TID["bias"]),
        TensorSpec("w1", (E, h, m), "normal", sh, dt, TID["w1"]),
        TensorSpec("w2", (E, m, h), "normal", 1.0 / np.sqrt(m), dt, TID["w2"]),
    ]
    if P > 0:
        specs += [
            TensorSpec("w_qkv_shared", (h, 6 * h), "normal", sh, dt, TID["w_qkv_shared"]),
            TensorSpec("w_o_shared", (2 * h, h), "normal", sh, dt, TID["w_o_shared"]),
            TensorSpec("w_qP", (h, dr), "normal", sh, dt, TID["w_qP"]),
            TensorSpec("k_P", (P, dr), "normal", 1.0, dt, TID["k_P"]),
        ]
    return specs


def input_specs(cfg: DreamerConfig) -> list[TensorSpec]:
    T, h = cfg.tokens, cfg.hidden
    specs = [TensorSpec("x0", (T, h), "normal", 1.0, cfg.dtype, TID["x0"])]
    if cfg.is_decode:
        cap = cfg.cache_len + 1
        shp = (cfg.depth, cfg.batch, cfg.n_heads, cap, cfg.head_dim)
        specs += [TensorSpec("k_cache", shp, "normal", 1.0, cfg.dtype, TID["k_cache"]),
                  TensorSpec("v_cache", shp, "normal", 1.0, cfg.dtype, TID["v_cache"])]
    return specs


def draw(spec: TensorSpec, seed: int, start: int = 0, n: int | None = None,
         use_c: bool = True) -> np.ndarray:
    """Flat elements [start, start+n) of a tensor, as float32 values of spec.dtype.

    Uses the C copy of the generator (libdreamer_inputs.so, OpenMP) when it is built, else
    the numpy definition below."""
    n = spec.numel - start if n is None else n
    if use_c and _lib_available():
        out = np.empty(n, np.float32)
        _lib().dri_fill_host(out.ctypes.data_as(ctypes.c_void_p),
                             ctypes.c_uint64(stream_key(seed, spec.tid)), ctypes.c_uint64(start),
                             ctypes.c_uint64(n), KIND_CODE[spec.kind], float(spec.param),
                             DTYPE_CODE[spec.dtype])
        return out
    if spec.kind == "ones":
        v = np.ones(n, np.float64)
    elif spec.kind == "normal":
        v = normal(stream_key(seed, spec.tid), start, n, spec.param)
    elif spec.kind == "uniform":
        v = uniform(stream_key(seed, spec.tid), start, n, spec.param)
    else:
        raise ValueError(spec.kind)
    return round_to(v, spec.dtype)


def draw_tensor(spec: TensorSpec, seed: int, chunk: int = 1 << 24) -> np.ndarray:
    out = np.empty(spec.numel, np.float32)
    for s in range(0, spec.numel, chunk):
        e = min(spec.numel, s + chunk)
        out[s:e] = draw(spec, seed, s, e - s)
    return out.reshape(spec.shape)


def host_weights(cfg: DreamerConfig) -> dict[str, np.ndarray]:
    return {s.name: draw_tensor(s, cfg.seed) for s in weight_specs(cfg)}


def host_inputs(cfg: DreamerConfig) -> dict[str, np.ndarray]:
    return {s.name: draw_tensor(s, cfg.seed) for s in input_specs(cfg)}


def extra_normal(cfg: DreamerConfig, tid: int, shape, std: float = 1.0,
                 dtype: str | None = None) -> np.ndarray:
    """A further seeded tensor (tests' step inputs, DA histories); tid >= 1000."""
    spec = TensorSpec("extra", tuple(shape), "normal", std, dtype or cfg.dtype, tid)
    return draw_tensor(spec, cfg.seed)


# ----------------------------------------------------------------------------------------
# device-side fill (same generator, CUDA kernel in libdreamer_inputs.so)
# ----------------------------------------------------------------------------------------
_LIB = None
_HERE = os.path.dirname(os.path.abspath(__file__))


def _lib_available() -> bool:
    return os.path.exists(os.path.join(_HERE, "libdreamer_inputs.so"))


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "libdreamer_inputs.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build() first")
        lib = ctypes.CDLL(path)
        lib.dri_fill.restype = ctypes.c_int
        lib.dri_fill.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                 ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
                                 ctypes.c_int, ctypes.c_void_p]
        lib.dri_fill_host.restype = ctypes.c_int
        lib.dri_fill_host.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_uint64,
                                      ctypes.c_uint64, ctypes.c_int, ctypes.c_double,
                                      ctypes.c_int]
        _LIB = lib
    return _LIB


KIND_CODE = {"normal": 0, "uniform": 1, "ones": 2}
DTYPE_CODE = {"fp32": 0, "bf16": 1}


def fill_device(ptr: int, spec: TensorSpec, seed: int, stream: int = 0,
                start: int = 0, n: int | None = None) -> None:
    """Draw elements [start, start+n) of `spec` straight into device memory at ptr."""
    n = spec.numel - start if n is None else n
    rc = _lib().dri_fill(ctypes.c_void_p(ptr), ctypes.c_uint64(stream_key(seed, spec.tid)),
                         ctypes.c_uint64(start), ctypes.c_uint64(n), KIND_CODE[spec.kind],
                         float(spec.param), DTYPE_CODE[spec.dtype], ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"dri_fill failed with CUDA error {rc}")


def device_tensor(spec: TensorSpec, seed: int, stream=None):
    """A torch CUDA tensor drawn in place by the device copy of the generator."""
    import torch
    dt = torch.float32 if spec.dtype == "fp32" else torch.bfloat16
    t = torch.empty(spec.shape, dtype=dt, device="cuda")
    s = stream if stream is not None else torch.cuda.current_stream()
    fill_device(t.data_ptr(), spec, seed, stream=s.cuda_stream)
    return t


def device_weights(cfg: DreamerConfig) -> dict:
    return {s.name: device_tensor(s, cfg.seed) for s in weight_specs(cfg)}


def device_inputs(cfg: DreamerConfig) -> dict:
    return {s.name: device_tensor(s, cfg.seed) for s in input_specs(cfg)}


def to_device(arr: np.ndarray, dtype: str):
    """Upload float32 host values (exact in dtype) as a CUDA tensor of dtype."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr, np.float32))
    return t.to("cuda").to(torch.float32 if dtype == "fp32" else torch.bfloat16)
